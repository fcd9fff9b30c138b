// Chunked prefill of the gated delta rule on the sm_100a tensor cores
// (tcgen05 MMA from shared-memory operands into TMEM accumulators), for bf16
// inputs with d_k = d_v = 128.
//
// The recurrence ("Qwen3.8-Flash-Next: architecture, efficiency and technical
// lineage", section 03 "Gated DeltaNet", update equations) is regrouped per
// chunk of C = 64 tokens.  With the entering state S (d_k x d_v),
// G_t = sum_{s<=t} log alpha_s, gamma_t = exp(G_t), K^, Q^ the L2-normalised
// keys/queries (rows t):
//
//   A   = strict_lower(diag(beta) (exp(G_t - G_i)) o K^ K^T)
//   T   = (I + A)^{-1}                                  (fp32, CUDA cores)
//   W   = T diag(beta gamma) K^        U = T diag(beta) V
//   Delta = U - W S                                     (values written)
//   Y   = diag(gamma) Q^ S + (lower(exp(G_t - G_i)) o Q^ K^T) Delta
//   S  <- gamma_C S + (diag(exp(G_C - G)) K^)^T Delta
//
// Every product is computed transposed so that the 128 TMEM lanes index d_v
// (or d_k) and all MMAs are M = 128:
//   MMA0  [K; Q] K^T   raw bf16 inputs, exact products; the L2-norm factors
//                      are applied afterwards in fp32
//   MMAW  W^T  = K^T (T diag(beta gamma))^T      (128 x 64)
//   MMAU  U^T  = V^T (T diag(beta))^T            (128 x 64)
//   MMA1  D^T  = U^T - S^T W^T                   (128 x 64, A negated)
//   MMA2  Y^T  = S^T (diag(gamma) Q^)^T          (128 x 64)
//   MMA3  S^T += D^T diag(exp(G_C - G)) K^       (128 x 128)
//   MMA4  Y^T += D^T P^T                         (128 x 64)
//
// Precision.  The state S^T stays in TMEM in fp32 for the whole sequence.
// MMA0 multiplies the raw bf16 q, k (exact, so q.k for near-orthogonal pairs
// keeps its sign and size).  Every other MMA takes fp16 operands (11-bit
// significand, 8x finer than bf16), with exact power-of-two scaling to stay
// inside fp16 range: per chunk, an exponent e is chosen from the block maxima
// of |V| and |S| and every value-like quantity (V, S, Delta, Y) enters the
// tensor core multiplied by 2^-e; T enters as T 2^-f, f chosen from max |T|.
// The fp32 TMEM state carries its own exponent; the scales are undone in the
// fp32 epilogue and in the final state.
//
// One CTA (8 warps) per (sequence, value head).  Warps 0-3 and 4-7 reach the
// same TMEM lanes (lane quarter = warp % 4) and split the columns.  Thread 0
// issues the MMAs; completion is tracked with one mbarrier whose waits are
// bounded: a wait that runs out flags the device error word and the CTA
// stops (after a second bounded wait for its own MMAs) without faulting.
#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_sm100.cuh"

// Section timing hook for tuning builds; compiles to nothing by default.
#ifndef GDN_TRACE_POINT
#define GDN_TRACE_POINT(i)
#endif

namespace gdn {
namespace {

using namespace sm100;

constexpr int kC = 64;    // chunk length
constexpr int kD = 128;   // head dim (d_k = d_v)
constexpr int kNT = 256;  // threads per CTA

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // [K; Q] raw bf16 128 x 128, 2 panels x 16 KB
constexpr uint32_t OFF_KH = 32768;      // K^ fp16          64 x 128, 2 panels x 8 KB
constexpr uint32_t OFF_QG = 49152;      // gamma Q^ fp16    64 x 128
constexpr uint32_t OFF_KT = 65536;      // dec K^ fp16      64 x 128
constexpr uint32_t OFF_VT = 81920;      // V 2^-e fp16      64 x 128
constexpr uint32_t OFF_TB = 98304;      // T b 2^-f fp16    64 x 64
constexpr uint32_t OFF_TBG = 106496;    // T b g 2^-f fp16  64 x 64
constexpr uint32_t OFF_P = 114688;      // P fp16           64 x 64
constexpr uint32_t OFF_WT = 122880;     // W^T fp16        128 x 64
constexpr uint32_t OFF_S0T = 139264;    // S^T 2^-e fp16   128 x 128, 2 panels x 16 KB
constexpr uint32_t OFF_DT = 172032;     // Delta^T fp16    128 x 64
// A and T (fp32 64 x 64 each) live in the [K; Q] region, which is dead once
// MMA0 has completed and is rewritten only after T has been consumed.
constexpr uint32_t OFF_A = OFF_KQ;
constexpr uint32_t OFF_T = OFF_KQ + 16384;
constexpr int kLZ = 52;
constexpr uint32_t OFF_Z = 188416;                   // Z fp32 [16][52]
constexpr uint32_t OFF_GATE = OFF_Z + 16 * kLZ * 4;  // G, beta, gamma, dec, rk, rq: 6 x 64
constexpr uint32_t OFF_RED = OFF_GATE + 6 * 64 * 4;  // red[4][64], rr[64], max[16]
constexpr uint32_t OFF_BAR = OFF_RED + 5 * 64 * 4 + 64;
constexpr uint32_t kSmemBytes = OFF_BAR + 64 + 1024;  // + alignment slack

// TMEM columns (fp32, 128 lanes)
constexpr uint32_t TM_S = 0, TM_KQ = 128, TM_W = 192, TM_D = 256, TM_Y = 320;
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kWaitLimit = 1u << 24;

constexpr uint32_t ID_BF_KK = idesc_f16(128, 64, false, false, false, false);  // MMA0
constexpr uint32_t ID_KK = idesc_f16(128, 64, false, false, false, true);
constexpr uint32_t ID_MK = idesc_f16(128, 64, true, false, false, true);
constexpr uint32_t ID_KM_NEG = idesc_f16(128, 64, false, true, true, true);
constexpr uint32_t ID_KM128 = idesc_f16(128, 128, false, true, false, true);

// fp32 64 x 64 scratch with an XOR swizzle on float4 groups (no padding)
__device__ __forceinline__ int fidx(int r, int c) { return r * 64 + (c ^ ((r & 7) << 2)); }

__device__ __forceinline__ void rs_stage(float* v, int H, int lane) {
  const bool up = (lane & H) != 0;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    if (k < H) {
      const float send = up ? v[k] : v[k + H];
      const float keep = up ? v[k + H] : v[k];
      v[k] = keep + __shfl_xor_sync(0xffffffffu, send, H);
    }
  }
}

// Block-wide max of non-negative values (every thread gets the result).
__device__ __forceinline__ float block_max(float x, float* sMax, int warp, int lane) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  if (lane == 0) sMax[warp] = x;
  __syncthreads();
  float m = sMax[0];
#pragma unroll
  for (int w = 1; w < kNT / 32; ++w) m = fmaxf(m, sMax[w]);
  __syncthreads();  // sMax reusable afterwards
  return m;
}

// Exponent e with x * 2^-e <= 2^target (x >= 0); 0 for x == 0 or non-finite.
__device__ __forceinline__ int scale_exp(float x, int target) {
  if (!(x > 0.f) || !(x < 3.0e38f)) return 0;
  int ex;
  frexpf(x, &ex);  // x = m 2^ex, m in [0.5, 1)
  return ex - target;
}

__device__ __forceinline__ void st_chunk_f16(uint32_t addr, const float* v, float s) {
  st_shared_v4(addr, pack_f16(v[0] * s, v[1] * s), pack_f16(v[2] * s, v[3] * s),
               pack_f16(v[4] * s, v[5] * s), pack_f16(v[6] * s, v[7] * s));
}

__global__ void __launch_bounds__(kNT, 1) gdn_prefill_tc_kernel(const PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* gb = smem_raw + (sb - raw);
  float* sA = reinterpret_cast<float*>(gb + OFF_A);
  float* sT = reinterpret_cast<float*>(gb + OFF_T);
  float* sZ = reinterpret_cast<float*>(gb + OFF_Z);
  float* sG = reinterpret_cast<float*>(gb + OFF_GATE);
  float* sBeta = sG + 64;
  float* sGam = sG + 128;
  float* sDec = sG + 192;
  float* sRk = sG + 256;
  float* sRq = sG + 320;
  float* sRed = reinterpret_cast<float*>(gb + OFF_RED);  // [4][64]
  float* sRr = sRed + 256;                                // [64]
  float* sMax = sRed + 320;                               // [16]
  uint64_t* bar = reinterpret_cast<uint64_t*>(gb + OFF_BAR);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(gb + OFF_BAR + 8);

  const int seq = blockIdx.x / a.H_v;
  const int h = blockIdx.x % a.H_v;
  const int hq = h / (a.H_v / a.H_qk);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = tid & 127;   // TMEM lane of this thread
  const int half = tid >> 7;   // which half of the columns
  int64_t t_begin, t_end;
  if (!seq_bounds(a.cu_seqlens, seq, a.total_T, &t_begin, &t_end, a.err)) return;

  const __nv_bfloat16* Qg = static_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* Kg = static_cast<const __nv_bfloat16*>(a.k);
  const __nv_bfloat16* Vg = static_cast<const __nv_bfloat16*>(a.v);
  const __nv_bfloat16* Gg = static_cast<const __nv_bfloat16*>(a.g);
  __nv_bfloat16* Yg = static_cast<__nv_bfloat16*>(a.y);
  const size_t st_off = ((size_t)seq * a.H_v + h) * (size_t)(kD * kD);

  if (warp == 0) tmem_alloc(tslot, kTmemCols);
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tbase = *tslot;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t tS = tbase + lane_off + TM_S, tKQ = tbase + lane_off + TM_KQ;
  const uint32_t tW = tbase + lane_off + TM_W, tD = tbase + lane_off + TM_D;
  const uint32_t tY = tbase + lane_off + TM_Y;

  // initial state -> TMEM S^T (lane j = column j of S, columns d), exponent 0
  {
    float v[32];
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) {
      const int d0 = half * 64 + cb * 32;
#pragma unroll
      for (int x = 0; x < 32; ++x)
        v[x] = a.initial_state ? __ldg(a.initial_state + st_off + (size_t)(d0 + x) * kD + row)
                               : 0.f;
      tmem_st32(tS + d0, v);
    }
    tmem_wait_st();
  }
  int s_exp = 0;  // S_true = S_tmem * 2^s_exp

  uint32_t phase = 0;
  bool ok = true;
  const bool has_g = Gg != nullptr;
  float wj = 0.f;
  if (has_g && a.norm_w) wj = __ldg(a.norm_w + row);

  for (int64_t c0 = t_begin; c0 < t_end; c0 += kC) {
    const int n = (t_end - c0) < kC ? (int)(t_end - c0) : kC;

    GDN_TRACE_POINT(0);
    // ---- gates: cumsum of log alpha, beta, gamma, exp(G_C - G) --------------
    if (warp == 0) {
      float carry = 0.f;
      float Gv[2], bv[2];
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        const int t = hb * 32 + lane;
        float x = t < n ? __ldg(a.log_alpha + (size_t)(c0 + t) * a.H_v + h) : 0.f;
        bv[hb] = t < n ? __ldg(a.beta + (size_t)(c0 + t) * a.H_v + h) : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float u = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += u;
        }
        Gv[hb] = x + carry;
        carry += __shfl_sync(0xffffffffu, x, 31);
      }
      const float GC = carry;
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        const int t = hb * 32 + lane;
        sG[t] = Gv[hb];
        sBeta[t] = bv[hb];
        sGam[t] = expf(Gv[hb]);
        sDec[t] = expf(GC - Gv[hb]);
      }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    GDN_TRACE_POINT(1);
    // ---- q, k rows -> operand tiles; v rows kept in registers -----------------
    // warp w owns rows 8w .. 8w+7; lane l owns columns 4l .. 4l+3
    float4 vv[8];
    float vmax = 0.f;
#pragma unroll
    for (int rp = 0; rp < 2; ++rp) {
      uint2 kr[4], qr[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = warp * 8 + rp * 4 + u;
        if (r < n) {
          const size_t qo = ((size_t)(c0 + r) * a.H_qk + hq) * kD + 4 * lane;
          kr[u] = __ldg(reinterpret_cast<const uint2*>(Kg + qo));
          qr[u] = __ldg(reinterpret_cast<const uint2*>(Qg + qo));
          vv[rp * 4 + u] =
              Elem<__nv_bfloat16>::load4(Vg + ((size_t)(c0 + r) * a.H_v + h) * kD + 4 * lane);
        } else {
          kr[u] = qr[u] = make_uint2(0u, 0u);
          vv[rp * 4 + u] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = warp * 8 + rp * 4 + u;
        const float2 k01 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&kr[u].x));
        const float2 k23 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&kr[u].y));
        const float2 q01 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&qr[u].x));
        const float2 q23 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&qr[u].y));
        float nk = k01.x * k01.x + k01.y * k01.y + k23.x * k23.x + k23.y * k23.y;
        float nq = q01.x * q01.x + q01.y * q01.y + q23.x * q23.x + q23.y * q23.y;
        nk = warp_sum(nk);
        nq = warp_sum(nq);
        const float rk = (a.l2norm && r < n) ? rsqrtf(nk + a.eps_l2) : 1.f;
        const float rq = (a.l2norm && r < n) ? rsqrtf(nq + a.eps_l2) : 1.f;
        if (lane == 0) {
          sRk[r] = rk;
          sRq[r] = rq;
        }
        const int col = 4 * lane;
        // raw bf16 rows for the exact q.k / k.k products
        st_shared_v2(sb + OFF_KQ + sw128_off(r, col, 128), kr[u].x, kr[u].y);
        st_shared_v2(sb + OFF_KQ + sw128_off(64 + r, col, 128), qr[u].x, qr[u].y);
        const float gq = sGam[r] * rq, dk = sDec[r] * rk;
        st_shared_v2(sb + OFF_KH + sw128_off(r, col, 64), pack_f16(rk * k01.x, rk * k01.y),
                     pack_f16(rk * k23.x, rk * k23.y));
        st_shared_v2(sb + OFF_QG + sw128_off(r, col, 64), pack_f16(gq * q01.x, gq * q01.y),
                     pack_f16(gq * q23.x, gq * q23.y));
        st_shared_v2(sb + OFF_KT + sw128_off(r, col, 64), pack_f16(dk * k01.x, dk * k01.y),
                     pack_f16(dk * k23.x, dk * k23.y));
        const float4 x = vv[rp * 4 + u];
        vmax = fmaxf(vmax, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
      }
    }

    GDN_TRACE_POINT(2);
    // ---- S^T from TMEM, block maxima, chunk exponent e ---------------------------
    float sv[64];
    tmem_ld32(tS + half * 64, sv);
    tmem_ld32(tS + half * 64 + 32, sv + 32);
    tmem_wait_ld();
    float smax = 0.f;
#pragma unroll
    for (int x = 0; x < 64; ++x) smax = fmaxf(smax, fabsf(sv[x]));
    const float mV = block_max(vmax, sMax, warp, lane);
    const float mS = ldexpf(block_max(smax, sMax, warp, lane), s_exp);
    // |Delta| <= |v| + |S| ||k^||_1 <= max|V| + 12 max|S|; keep that <= 2^12
    const int e = scale_exp(mV + 12.f * mS, 12);
    {
      const float sv_scale = ldexpf(1.f, -e);
      // V rows 2^-e -> fp16 tile (rows i, columns j)
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int r = warp * 8 + u;
        const float4 x = vv[u];
        st_shared_v2(sb + OFF_VT + sw128_off(r, 4 * lane, 64), pack_f16(x.x * sv_scale, x.y * sv_scale),
                     pack_f16(x.z * sv_scale, x.w * sv_scale));
      }
      // S^T 2^-e -> fp16 tile; fp32 state rescaled by gamma_C and to exponent e
      const float to_e = ldexpf(1.f, s_exp - e);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        st_chunk_f16(sb + OFF_S0T + sw128_chunk(row, half * 8 + q, 128), sv + 8 * q, to_e);
      const float upd = sGam[63] * to_e;
#pragma unroll
      for (int x = 0; x < 64; ++x) sv[x] *= upd;
      tmem_st32(tS + half * 64, sv);
      tmem_st32(tS + half * 64 + 32, sv + 32);
      tmem_wait_st();
      s_exp = e;
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();

    GDN_TRACE_POINT(3);
    // ---- MMA0: [K;Q] K^T (bf16, exact);  MMA2: S^T (gamma Q^)^T (fp16) -----------
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t d = sdesc(sb + OFF_KQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
        mma_f16(tbase + TM_KQ, d, d, ID_BF_KK, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t da = sdesc(sb + OFF_S0T + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
        const uint64_t db = sdesc(sb + OFF_QG + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
        mma_f16(tbase + TM_Y, da, db, ID_KK, kk > 0);
      }
      mma_commit(bar);
    }
    ok = mbar_wait(bar, phase, kWaitLimit);
    phase ^= 1;
    if (!__syncthreads_and(ok)) { ok = false; break; }
    fence_after_sync();

    GDN_TRACE_POINT(4);
    // ---- A (fp32) and P (fp16) from the raw products (warps 0-3) --------------
    if (tid < 128) {
      const int t = tid & 63;
      float v[64];
      tmem_ld32(tKQ, v);
      tmem_ld32(tKQ + 32, v + 32);
      tmem_wait_ld();
      const float Gt = sG[t];
      if (tid < 64) {
        const float bt = sBeta[t] * sRk[t];
#pragma unroll
        for (int i = 0; i < 64; i += 4) {
          float4 o;
          o.x = (i + 0 < t) ? bt * sRk[i + 0] * expf(Gt - sG[i + 0]) * v[i + 0] : 0.f;
          o.y = (i + 1 < t) ? bt * sRk[i + 1] * expf(Gt - sG[i + 1]) * v[i + 1] : 0.f;
          o.z = (i + 2 < t) ? bt * sRk[i + 2] * expf(Gt - sG[i + 2]) * v[i + 2] : 0.f;
          o.w = (i + 3 < t) ? bt * sRk[i + 3] * expf(Gt - sG[i + 3]) * v[i + 3] : 0.f;
          *reinterpret_cast<float4*>(sA + fidx(t, i)) = o;
        }
      } else {
        const float qt = sRq[t];
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          uint32_t pk[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i0 = 8 * c8 + 2 * u, i1 = i0 + 1;
            const float p0 = (i0 <= t) ? qt * sRk[i0] * expf(Gt - sG[i0]) * v[i0] : 0.f;
            const float p1 = (i1 <= t) ? qt * sRk[i1] * expf(Gt - sG[i1]) * v[i1] : 0.f;
            pk[u] = pack_f16(p0, p1);
          }
          st_shared_v4(sb + OFF_P + sw128_chunk(t, c8, 64), pk[0], pk[1], pk[2], pk[3]);
        }
      }
    }
    fence_before_sync();
    __syncthreads();

    GDN_TRACE_POINT(5);
    // ---- T = (I + A)^{-1}: 16 x 16 diagonal blocks by substitution -------------
    if (tid < 64) {
      const int b = tid >> 4, c = tid & 15;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float s = (r == c) ? 1.f : 0.f;
#pragma unroll
        for (int m = 0; m < r; ++m) s -= sA[fidx(16 * b + r, 16 * b + m)] * x[m];
        x[r] = s;
      }
#pragma unroll
      for (int r = 0; r < 16; ++r) sT[fidx(16 * b + r, 16 * b + c)] = x[r];
    }
    __syncthreads();
    // off-diagonal blocks: T_rc = -T_rr sum_{m=c}^{r-1} A_rm T_mc, block row by row
#pragma unroll 1
    for (int rb = 1; rb < 4; ++rb) {
      const int ncols = 16 * rb, total = 16 * ncols;
      for (int e2 = tid; e2 < total; e2 += kNT) {
        const int p = e2 / ncols, q = e2 % ncols;
        float s = 0.f;
        for (int m = 16 * (q >> 4); m < 16 * rb; ++m) s += sA[fidx(16 * rb + p, m)] * sT[fidx(m, q)];
        sZ[p * kLZ + q] = s;
      }
      __syncthreads();
      for (int e2 = tid; e2 < total; e2 += kNT) {
        const int p = e2 / ncols, q = e2 % ncols;
        float s = 0.f;
        for (int u = 0; u <= p; ++u) s += sT[fidx(16 * rb + p, 16 * rb + u)] * sZ[u * kLZ + q];
        sT[fidx(16 * rb + p, q)] = -s;
      }
      __syncthreads();
    }

    GDN_TRACE_POINT(6);
    // ---- scale exponent of T; T diag(b) 2^-f, T diag(b g) 2^-f -> fp16 ---------
    float tmax = 0.f;
    if (tid < 128) {
      const int t = tid & 63;
      for (int i = (tid >> 6) * 32; i < (tid >> 6) * 32 + 32; ++i)
        if (i <= t) tmax = fmaxf(tmax, fabsf(sT[fidx(t, i)]));
    }
    const int f = max(0, scale_exp(block_max(tmax, sMax, warp, lane), 8));
    if (tid < 128) {
      const int t = tid & 63;
      const bool withg = tid >= 64;
      const float sf = ldexpf(1.f, -f);
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        uint32_t pk[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i0 = 8 * c8 + 2 * u, i1 = i0 + 1;
          float x0 = (i0 <= t) ? sT[fidx(t, i0)] * sBeta[i0] * sf : 0.f;
          float x1 = (i1 <= t) ? sT[fidx(t, i1)] * sBeta[i1] * sf : 0.f;
          if (withg) {
            x0 *= sGam[i0];
            x1 *= sGam[i1];
          }
          pk[u] = pack_f16(x0, x1);
        }
        st_shared_v4(sb + (withg ? OFF_TBG : OFF_TB) + sw128_chunk(t, c8, 64), pk[0], pk[1],
                     pk[2], pk[3]);
      }
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();

    GDN_TRACE_POINT(7);
    // ---- MMAW: W^T = K^T (T diag(b g))^T;  MMAU: U^T = V^T (T diag(b))^T -------
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t da = sdesc(sb + OFF_KH + kk * 2048, 8192, 1024);
        const uint64_t db = sdesc(sb + OFF_TBG + kk * 32, 16, 1024);
        mma_f16(tbase + TM_W, da, db, ID_MK, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t da = sdesc(sb + OFF_VT + kk * 2048, 8192, 1024);
        const uint64_t db = sdesc(sb + OFF_TB + kk * 32, 16, 1024);
        mma_f16(tbase + TM_D, da, db, ID_MK, kk > 0);
      }
      mma_commit(bar);
    }
    ok = mbar_wait(bar, phase, kWaitLimit);
    phase ^= 1;
    if (!__syncthreads_and(ok)) { ok = false; break; }
    fence_after_sync();

    GDN_TRACE_POINT(8);
    // ---- W^T 2^-f (fp32) -> fp16 tile, rows d, columns t ------------------------
    {
      float v[32];
      tmem_ld32(tW + half * 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 4; ++q)
        st_chunk_f16(sb + OFF_WT + sw128_chunk(row, half * 4 + q, 128), v + 8 * q, 1.f);
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();

    GDN_TRACE_POINT(9);
    // ---- MMA1: Delta^T 2^-(e+f) = U^T - S^T W^T ---------------------------------------
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t da = sdesc(sb + OFF_S0T + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
        const uint64_t db = sdesc(sb + OFF_WT + kk * 2048, 16384, 1024);
        mma_f16(tbase + TM_D, da, db, ID_KM_NEG, 1);
      }
      mma_commit(bar);
    }
    ok = mbar_wait(bar, phase, kWaitLimit);
    phase ^= 1;
    if (!__syncthreads_and(ok)) { ok = false; break; }
    fence_after_sync();

    GDN_TRACE_POINT(10);
    // ---- Delta^T 2^-e -> fp16 tile, rows j, columns i -------------------------------
    {
      float v[32];
      tmem_ld32(tD + half * 32, v);
      tmem_wait_ld();
      const float sf = ldexpf(1.f, f);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        st_chunk_f16(sb + OFF_DT + sw128_chunk(row, half * 4 + q, 128), v + 8 * q, sf);
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();

    GDN_TRACE_POINT(11);
    // ---- MMA3: S^T += Delta^T (dec K^);  MMA4: Y^T += Delta^T P^T ---------------------
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t da = sdesc(sb + OFF_DT + kk * 32, 16, 1024);
        const uint64_t db = sdesc(sb + OFF_KT + kk * 2048, 8192, 1024);
        mma_f16(tbase + TM_S, da, db, ID_KM128, 1);
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t da = sdesc(sb + OFF_DT + kk * 32, 16, 1024);
        const uint64_t db = sdesc(sb + OFF_P + kk * 32, 16, 1024);
        mma_f16(tbase + TM_Y, da, db, ID_KK, 1);
      }
      mma_commit(bar);
    }
    ok = mbar_wait(bar, phase, kWaitLimit);
    phase ^= 1;
    if (!__syncthreads_and(ok)) { ok = false; break; }
    fence_after_sync();

    GDN_TRACE_POINT(12);
    // ---- epilogue: Y^T 2^-e -> y (optional RMSNorm x sigmoid(g)) ----------------------
    {
      float v[32];
      tmem_ld32(tY + half * 32, v);
      tmem_wait_ld();
      const float ys = ldexpf(a.scale, e);
#pragma unroll
      for (int x = 0; x < 32; ++x) v[x] *= ys;
      if (has_g) {
        float s2[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) s2[x] = v[x] * v[x];
        rs_stage(s2, 16, lane);
        rs_stage(s2, 8, lane);
        rs_stage(s2, 4, lane);
        rs_stage(s2, 2, lane);
        rs_stage(s2, 1, lane);
        sRed[(warp & 3) * 64 + half * 32 + lane] = s2[0];
        __syncthreads();
        if (tid < 64)
          sRr[tid] = rsqrtf((sRed[tid] + sRed[64 + tid] + sRed[128 + tid] + sRed[192 + tid]) /
                                (float)kD + a.eps_norm);
        __syncthreads();
      }
#pragma unroll 4
      for (int x = 0; x < 32; ++x) {
        const int t = half * 32 + x;
        if (t < n) {
          const size_t yo = ((size_t)(c0 + t) * a.H_v + h) * kD + row;
          float o = v[x];
          if (has_g) {
            const float gg = __bfloat162float(Gg[yo]);
            o = o * sRr[t] * (1.f + wj) / (1.f + __expf(-gg));
          }
          Yg[yo] = __float2bfloat16_rn(o);
        }
      }
    }
    fence_before_sync();
    __syncthreads();
    GDN_TRACE_POINT(13);
  }

  if (ok) {
    // final state from TMEM, undoing the state exponent
    if (a.final_state) {
      const float sc = ldexpf(1.f, s_exp);
      float v[32];
#pragma unroll 1
      for (int cb = 0; cb < 2; ++cb) {
        const int d0 = half * 64 + cb * 32;
        tmem_ld32(tS + d0, v);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x)
          a.final_state[st_off + (size_t)(d0 + x) * kD + row] = v[x] * sc;
      }
    }
  } else {
    if (tid == 0) atomicOr(a.err, kErrTimeout);
    // give in-flight MMAs a second bounded chance to drain before TMEM is freed
    mbar_wait(bar, phase ^ 1, kWaitLimit);
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tbase, kTmemCols);
}

}  // namespace

bool prefill_tc_supports(const PrefillArgs& a) {
  return a.dtype == GDN_BF16 && a.d_k == kD && a.d_v == kD;
}

gdn_status launch_prefill_tc(const PrefillArgs& a, cudaStream_t stream) {
  if (!prefill_tc_supports(a)) return GDN_ERR_UNSUPPORTED;
  // the shared-memory opt-in is per device; set it once for each
  static bool attr_set[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    if (cudaFuncSetAttribute(gdn_prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes) != cudaSuccess)
      return GDN_ERR_CUDA;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const unsigned grid = (unsigned)a.n_seq * (unsigned)a.H_v;
  gdn_prefill_tc_kernel<<<grid, kNT, kSmemBytes, stream>>>(a);
  return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn
