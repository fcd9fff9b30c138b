// Chunked prefill of the gated delta rule on the sm_100a tensor cores
// (tcgen05 MMA from shared-memory and TMEM operands into TMEM accumulators), for bf16
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
// (or d_k) and the state-side MMAs are M = 128:
//   MMA0  [K; Q] K^T     raw bf16 inputs, exact products; the L2-norm factors
//                        are applied afterwards in fp32
//   MMAW  W = (T diag(beta gamma)) K^        (M = 64 tokens x N = 128), stored
//                        negated and K-major beside gamma Q^
//   MMA1  [Delta^T | Y^T] = S^T [-W; gamma Q^]^T   (one N = 128 product)
//   MMAU  Delta^T += V^T (T diag(beta))^T  (= U^T)
//   MMA3  S^T += Delta^T diag(exp(G_C - G)) K^     (128 x 128)
//   MMA4  Y^T += Delta^T P^T
// The fp16 copies of S^T and Delta^T that MMA1 / MMA3 / MMA4 read are written
// straight into TMEM (tcgen05.st) and used as TMEM A operands.
//
// Precision.  The state S^T stays in TMEM in fp32 for the whole sequence.
// MMA0 multiplies the raw bf16 q, k (exact, so q.k for near-orthogonal pairs
// keeps its sign and size).  Every other MMA takes fp16 operands (11-bit
// significand, 8x finer than bf16), with exact power-of-two scaling to stay
// inside fp16 range: per chunk, an exponent e is chosen from the block maxima
// of |V| and |S| and every value-like quantity (V, S, Delta, Y) enters the
// tensor core multiplied by 2^-e; T enters as T 2^-f, f chosen from max |T|,
// and T diag(beta gamma) as an fp16 hi + lo pair (W is a cancellation when
// keys repeat).  The fp32 TMEM state carries its own exponent; the scales are
// undone in the fp32 epilogue and in the final state.
//
// Layouts: one CTA (8 warps) per (sequence, value head) for large batches
// (gdn_prefill_tc_kernel); for small batches without a workspace a chain CTA
// plus preparation CTAs per item in a cluster (gdn_prefill_tc_pair_kernel,
// below; with a workspace the scan layout of gdn_prefill_scan.cu runs
// instead).  Warps 0-3 and 4-7 reach
// the same TMEM lanes (lane quarter = warp % 4) and split the columns.  One
// thread issues the MMAs; completion is tracked with mbarriers whose waits are
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

// shared memory map of the one-CTA kernel (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // [K; Q] raw bf16 128 x 128 (cp.async target), 2 x 16 KB
constexpr uint32_t OFF_KH = 32768;      // K^ fp16          64 x 128, 2 panels x 8 KB
constexpr uint32_t OFF_KT = 49152;      // dec K^ fp16      64 x 128
constexpr uint32_t OFF_VT = 65536;      // V: raw bf16 (cp.async), then V 2^-e fp16 in place
constexpr uint32_t OFF_TB = 81920;      // T b 2^-f fp16    64 x 64
constexpr uint32_t OFF_TBG = 90112;     // T b g 2^-f fp16  64 x 64 (rounded part)
constexpr uint32_t OFF_P = 98304;       // P fp16           64 x 64
constexpr uint32_t OFF_WQ = 106496;     // [-W; gamma Q^] fp16 128 x 128 K-major, 2 panels x 16 KB
constexpr uint32_t OFF_A = 139264;      // A fp32 64 x 64
constexpr uint32_t OFF_T = 155648;      // T fp32 64 x 64
constexpr uint32_t OFF_TBG_LO = OFF_A;  // rounding remainder of T diag(b g), after A is dead
constexpr uint32_t OFF_STG = 172032;    // output staging [64][128] 16-bit
constexpr uint32_t OFF_GS = 188416;     // g (-> gate factors in place), 2 buffers x [64][128]
constexpr uint32_t OFF_Z = 221184;      // Z fp32 [1024]
constexpr uint32_t OFF_GATEBUF = 225280;  // [2 buffers][log alpha, beta][64] fp32
constexpr uint32_t OFF_GATE = 226304;   // G2, beta, gamma, dec, rk, rq: 6 x 64 fp32
constexpr uint32_t OFF_RED = 227840;    // red[4][64], rr[64], max[16]
constexpr uint32_t OFF_BAR = 229248;
constexpr uint32_t kSmemBytes = OFF_BAR + 64 + 1024;  // + alignment slack

// TMEM columns (fp32, 128 lanes): S^T, [K;Q]K^T (then W, M = 64 x N = 128),
// Delta^T | Y^T (adjacent: one N = 128 product writes both), and the fp16
// MMA A operands S^T 2^-e and Delta^T 2^-e
constexpr uint32_t TM_S = 0, TM_KQ = 128, TM_W = 128, TM_D = 256, TM_Y = 320, TM_SA = 384,
                   TM_DA = 448;
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kWaitLimit = 1u << 24;
constexpr float kLog2e = 1.4426950408889634f;

constexpr uint32_t ID_BF_KK = idesc_f16(128, 64, false, false, false, false);  // MMA0
constexpr uint32_t ID_KK = idesc_f16(128, 64, false, false, false, true);
constexpr uint32_t ID_MK = idesc_f16(128, 64, true, false, false, true);
constexpr uint32_t ID_KM128 = idesc_f16(128, 128, false, true, false, true);
constexpr uint32_t ID_KK128 = idesc_f16(128, 128, false, false, false, true);
constexpr uint32_t ID_W64 = idesc_f16(64, 128, false, true, false, true);

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

// Block-wide maxima of two non-negative values with one exchange (sMax
// holds 2 x 8 floats).
__device__ __forceinline__ float2 block_max2(float x, float y, float* sMax, int warp, int lane) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    y = fmaxf(y, __shfl_xor_sync(0xffffffffu, y, o));
  }
  if (lane == 0) {
    sMax[warp] = x;
    sMax[8 + warp] = y;
  }
  __syncthreads();
  float mx = sMax[0], my = sMax[8];
#pragma unroll
  for (int w = 1; w < kNT / 32; ++w) {
    mx = fmaxf(mx, sMax[w]);
    my = fmaxf(my, sMax[8 + w]);
  }
  __syncthreads();  // sMax reusable afterwards
  return make_float2(mx, my);
}

// Exponent e with x * 2^-e <= 2^target (x >= 0); 0 for x == 0 or non-finite.
__device__ __forceinline__ int scale_exp(float x, int target) {
  if (!(x > 0.f) || !(x < 3.0e38f)) return 0;
  int ex;
  frexpf(x, &ex);  // x = m 2^ex, m in [0.5, 1)
  return ex - target;
}

// fp16 pair split into a rounded part and the rounding remainder:
// hi + lo carries the fp32 value to ~2^-22 relative.
__device__ __forceinline__ void split_pack_f16(float x0, float x1, uint32_t* hi, uint32_t* lo) {
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 hf = __half22float2(h);
  *hi = *reinterpret_cast<const uint32_t*>(&h);
  *lo = pack_f16(x0 - hf.x, x1 - hf.y);
}

__device__ __forceinline__ void st_chunk_f16(uint32_t addr, const float* v, float s) {
  st_shared_v4(addr, pack_f16(v[0] * s, v[1] * s), pack_f16(v[2] * s, v[3] * s),
               pack_f16(v[4] * s, v[5] * s), pack_f16(v[6] * s, v[7] * s));
}

__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__device__ __forceinline__ void unpack_bf16x8(const uint4 u, float* f) {
  float2 p;
  p = bf2_to_f2(u.x); f[0] = p.x; f[1] = p.y;
  p = bf2_to_f2(u.y); f[2] = p.x; f[3] = p.y;
  p = bf2_to_f2(u.z); f[4] = p.x; f[5] = p.y;
  p = bf2_to_f2(u.w); f[6] = p.x; f[7] = p.y;
}

__device__ __forceinline__ float2 h2_to_f2(uint32_t w) {
  __half2 h;
  memcpy(&h, &w, 4);
  return __half22float2(h);
}

__device__ __forceinline__ void unpack_f16x8(const uint4 u, float* f) {
  float2 p;
  p = h2_to_f2(u.x); f[0] = p.x; f[1] = p.y;
  p = h2_to_f2(u.y); f[2] = p.x; f[3] = p.y;
  p = h2_to_f2(u.z); f[4] = p.x; f[5] = p.y;
  p = h2_to_f2(u.w); f[6] = p.x; f[7] = p.y;
}


// One recursive-doubling level of the unit-lower-triangular inverse: for
// every pair of BS x BS diagonal blocks [[T1, 0], [A21, T2]] of I + A, writes
// the off-diagonal block X = -T2 (A21 T1) of the inverse.  All 256 threads;
// each computes an R x 2 (BS >= 16) or 1 x 1 (BS = 8) block of outputs with
// the sums over m unrolled in steps of 4 (float4 rows of A / T, float2
// columns of T / Z).  T's strictly upper entries must be zero.
template <int BS>
__device__ __forceinline__ void tinv_level(const float* sA, float* sT, float* sZ, int tid) {
  constexpr int NP = 64 / (2 * BS);                  // pairs
  constexpr int EPT = NP * BS * BS / kNT;            // outputs per thread
  constexpr int RC = EPT >= 2 ? 2 : 1;               // columns per thread
  constexpr int RR = EPT / RC;                       // rows per thread
  constexpr int CB = BS / RC;                        // column blocks per row
  constexpr int TPP = (BS / RR) * CB;                // threads per pair
  const int p = tid / TPP, q = tid % TPP;
  const int r0 = (q / CB) * RR, c0 = (q % CB) * RC;
  const int top = 2 * BS * p, bot = top + BS;
  float acc[RR][RC];
  // Z = A21 T1
#pragma unroll
  for (int i = 0; i < RR; ++i)
#pragma unroll
    for (int j = 0; j < RC; ++j) acc[i][j] = 0.f;
#pragma unroll
  for (int m = 0; m < BS; m += 4) {
    float4 ar[RR];
#pragma unroll
    for (int i = 0; i < RR; ++i) ar[i] = *reinterpret_cast<const float4*>(sA + fidx(bot + r0 + i, top + m));
#pragma unroll
    for (int mm = 0; mm < 4; ++mm) {
      float tc[RC];
      if (RC == 2) {
        const float2 t2 = *reinterpret_cast<const float2*>(sT + fidx(top + m + mm, top + c0));
        tc[0] = t2.x;
        tc[RC - 1] = t2.y;
      } else {
        tc[0] = sT[fidx(top + m + mm, top + c0)];
      }
#pragma unroll
      for (int i = 0; i < RR; ++i) {
        const float av = mm == 0 ? ar[i].x : mm == 1 ? ar[i].y : mm == 2 ? ar[i].z : ar[i].w;
#pragma unroll
        for (int j = 0; j < RC; ++j) acc[i][j] += av * tc[j];
      }
    }
  }
#pragma unroll
  for (int i = 0; i < RR; ++i)
#pragma unroll
    for (int j = 0; j < RC; ++j) sZ[p * BS * BS + (r0 + i) * BS + c0 + j] = acc[i][j];
  __syncthreads();
  // X = -T2 Z
#pragma unroll
  for (int i = 0; i < RR; ++i)
#pragma unroll
    for (int j = 0; j < RC; ++j) acc[i][j] = 0.f;
#pragma unroll
  for (int m = 0; m < BS; m += 4) {
    float4 tr[RR];
#pragma unroll
    for (int i = 0; i < RR; ++i) tr[i] = *reinterpret_cast<const float4*>(sT + fidx(bot + r0 + i, bot + m));
#pragma unroll
    for (int mm = 0; mm < 4; ++mm) {
      float zc[RC];
      if (RC == 2) {
        const float2 z2 = *reinterpret_cast<const float2*>(sZ + p * BS * BS + (m + mm) * BS + c0);
        zc[0] = z2.x;
        zc[RC - 1] = z2.y;
      } else {
        zc[0] = sZ[p * BS * BS + (m + mm) * BS + c0];
      }
#pragma unroll
      for (int i = 0; i < RR; ++i) {
        const float tv = mm == 0 ? tr[i].x : mm == 1 ? tr[i].y : mm == 2 ? tr[i].z : tr[i].w;
#pragma unroll
        for (int j = 0; j < RC; ++j) acc[i][j] -= tv * zc[j];
      }
    }
  }
#pragma unroll
  for (int i = 0; i < RR; ++i) {
    if (RC == 2) {
      *reinterpret_cast<float2*>(sT + fidx(bot + r0 + i, top + c0)) = make_float2(acc[i][0], acc[i][RC - 1]);
    } else {
      sT[fidx(bot + r0 + i, top + c0)] = acc[i][0];
    }
  }
  __syncthreads();
}


// A (fp32, strictly lower) and P (fp16 tile, lower incl. diagonal) for one
// row t of the chunk from 32 raw products v of this thread's TMEM lane:
//   A_ti = beta_t rk_t rk_i 2^(G2_t - G2_i) (k.k)_ti      (i < t)
//   P_ti = rq_t rk_i 2^(G2_t - G2_i) (q.k)_ti             (i <= t)
// columns i0 .. i0+31.  Blocks of columns entirely above the diagonal are
// skipped (whole warps skip them together, rows are warp-contiguous).
__device__ __forceinline__ void chunk_ap(const float* v, int t, int i0, bool is_a,
                                         const float* sG2, const float* sBeta, const float* sRk,
                                         const float* sRq, float* sA, uint32_t p_tile) {
  const float Gt = sG2[t];
  if (is_a) {
    const float bt = sBeta[t] * sRk[t];
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i0 + i < t) {
        const float4 g4 = *reinterpret_cast<const float4*>(sG2 + i0 + i);
        const float4 k4 = *reinterpret_cast<const float4*>(sRk + i0 + i);
        o.x = bt * k4.x * ex2_approx(Gt - g4.x) * v[i + 0];
        o.y = (i0 + i + 1 < t) ? bt * k4.y * ex2_approx(Gt - g4.y) * v[i + 1] : 0.f;
        o.z = (i0 + i + 2 < t) ? bt * k4.z * ex2_approx(Gt - g4.z) * v[i + 2] : 0.f;
        o.w = (i0 + i + 3 < t) ? bt * k4.w * ex2_approx(Gt - g4.w) * v[i + 3] : 0.f;
      }
      *reinterpret_cast<float4*>(sA + fidx(t, i0 + i)) = o;
    }
  } else {
    const float qt = sRq[t];
#pragma unroll
    for (int c8 = 0; c8 < 4; ++c8) {
      uint32_t pk[4] = {0u, 0u, 0u, 0u};
      if (i0 + 8 * c8 <= t) {
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {
          const int ib = i0 + 8 * c8 + 4 * hq;
          const float4 g4 = *reinterpret_cast<const float4*>(sG2 + ib);
          const float4 k4 = *reinterpret_cast<const float4*>(sRk + ib);
          const float* vv = v + 8 * c8 + 4 * hq;
          const float p0 = (ib + 0 <= t) ? qt * k4.x * ex2_approx(Gt - g4.x) * vv[0] : 0.f;
          const float p1 = (ib + 1 <= t) ? qt * k4.y * ex2_approx(Gt - g4.y) * vv[1] : 0.f;
          const float p2 = (ib + 2 <= t) ? qt * k4.z * ex2_approx(Gt - g4.z) * vv[2] : 0.f;
          const float p3 = (ib + 3 <= t) ? qt * k4.w * ex2_approx(Gt - g4.w) * vv[3] : 0.f;
          pk[2 * hq] = pack_f16(p0, p1);
          pk[2 * hq + 1] = pack_f16(p2, p3);
        }
      }
      st_shared_v4(p_tile + sw128_chunk(t, i0 / 8 + c8, 64), pk[0], pk[1], pk[2], pk[3]);
    }
  }
}

struct ChunkLoader {
  const __nv_bfloat16 *Qg, *Kg, *Vg, *Gg;
  const float *la, *beta;
  int H_qk, H_v, h, hq, tid;
  uint32_t sb;
  uint32_t off_kq = OFF_KQ, off_vt = OFF_VT, off_gs = OFF_GS, off_gate = OFF_GATEBUF;
  // raw q, k rows of the chunk into the [K; Q] tile (rows >= nn zero filled)
  __device__ void qk(int64_t c0, int nn) const {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int idx = tid + kNT * k;  // 2048 16-byte pieces
      const int which = idx >> 10, rr = (idx >> 4) & 63, ch = idx & 15;
      const bool ok = rr < nn;
      const __nv_bfloat16* base = which ? Qg : Kg;
      const __nv_bfloat16* src =
          base + (ok ? ((size_t)(c0 + rr) * H_qk + hq) * kD + ch * 8 : 0);
      cp_async16(sb + off_kq + sw128_chunk(which * 64 + rr, ch, 128), src, ok);
    }
  }
  __device__ void v(int64_t c0, int nn) const {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int idx = tid + kNT * k;  // 1024 pieces
      const int rr = idx >> 4, ch = idx & 15;
      const bool ok = rr < nn;
      const __nv_bfloat16* src = Vg + (ok ? ((size_t)(c0 + rr) * H_v + h) * kD + ch * 8 : 0);
      cp_async16(sb + off_vt + sw128_chunk(rr, ch, 64), src, ok);
    }
  }
  __device__ void g(int64_t c0, int nn, int buf) const {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int idx = tid + kNT * k;
      const int rr = idx >> 4, ch = idx & 15;
      const bool ok = rr < nn;
      const __nv_bfloat16* src = Gg + (ok ? ((size_t)(c0 + rr) * H_v + h) * kD + ch * 8 : 0);
      cp_async16(sb + off_gs + buf * 16384 + rr * 256 + ch * 16, src, ok);
    }
  }
  __device__ void gates(int64_t c0, int nn, int buf) const {
    if (tid < 128) {
      const int which = tid >> 6, t = tid & 63;
      const bool ok = t < nn;
      const float* src = (which ? beta : la) + (ok ? (size_t)(c0 + t) * H_v + h : 0);
      cp_async4(sb + off_gate + (buf * 2 + which) * 256 + t * 4, src, ok);
    }
  }
};

__global__ void __launch_bounds__(kNT, 1) gdn_prefill_tc_kernel(const PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* gb = smem_raw + (sb - raw);
  float* sA = reinterpret_cast<float*>(gb + OFF_A);
  float* sT = reinterpret_cast<float*>(gb + OFF_T);
  float* sZ = reinterpret_cast<float*>(gb + OFF_Z);
  const float* sGateBuf = reinterpret_cast<const float*>(gb + OFF_GATEBUF);
  float* sG2 = reinterpret_cast<float*>(gb + OFF_GATE);
  float* sBeta = sG2 + 64;
  float* sGam = sG2 + 128;
  float* sDec = sG2 + 192;
  float* sRk = sG2 + 256;
  float* sRq = sG2 + 320;
  float* sRed = reinterpret_cast<float*>(gb + OFF_RED);  // [4][64]
  float* sRr = sRed + 256;                                // [64]
  float* sMax = sRed + 320;                               // [16]
  uint64_t* bar = reinterpret_cast<uint64_t*>(gb + OFF_BAR);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(gb + OFF_BAR + 8);

  // (sequence, value head) item: sequences longest first when the order is
  // given, so that the long ones do not start in the last wave
  const int seq = a.seq_order ? a.seq_order[blockIdx.x / a.H_v] : (int)(blockIdx.x / a.H_v);
  const int h = blockIdx.x % a.H_v;
  const int hq = h / (a.H_v / a.H_qk);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = tid & 127;   // TMEM lane of this thread
  const int half = tid >> 7;   // which half of the columns
  int64_t t_begin, t_end;
  if (!seq_bounds(a.cu_seqlens, seq, a.total_T, &t_begin, &t_end, a.err)) return;

  const __nv_bfloat16* Gg = static_cast<const __nv_bfloat16*>(a.g);
  __nv_bfloat16* Yg = static_cast<__nv_bfloat16*>(a.y);
  const size_t st_off = ((size_t)seq * a.H_v + h) * (size_t)(kD * kD);
  ChunkLoader ld;
  ld.Qg = static_cast<const __nv_bfloat16*>(a.q);
  ld.Kg = static_cast<const __nv_bfloat16*>(a.k);
  ld.Vg = static_cast<const __nv_bfloat16*>(a.v);
  ld.Gg = Gg;
  ld.la = a.log_alpha;
  ld.beta = a.beta;
  ld.H_qk = a.H_qk;
  ld.H_v = a.H_v;
  ld.h = h;
  ld.hq = hq;
  ld.tid = tid;
  ld.sb = sb;
  const bool has_g = Gg != nullptr;

  // first chunk's inputs in flight while TMEM and the state are set up
  if (t_begin < t_end) {
    const int n0 = (t_end - t_begin) < kC ? (int)(t_end - t_begin) : kC;
    ld.qk(t_begin, n0);
    ld.v(t_begin, n0);
    if (has_g) ld.g(t_begin, n0, 0);
    ld.gates(t_begin, n0, 0);
    cp_async_commit();
  }

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
  const uint32_t tSA = tbase + lane_off + TM_SA, tDA = tbase + lane_off + TM_DA;

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

  // 1 + w for the 8 output columns this thread gates and stores (the same
  // in every chunk: piece index p has column block p % 16 = tid % 16)
  float wv[8];
#pragma unroll
  for (int j2 = 0; j2 < 8; ++j2)
    wv[j2] = 1.f + ((has_g && a.norm_w) ? __ldg(a.norm_w + (tid & 15) * 8 + j2) : 0.f);

  uint32_t phase = 0;
  bool ok = true;

  int ci = 0;
  for (int64_t c0 = t_begin; c0 < t_end; c0 += kC, ++ci) {
    const int n = (t_end - c0) < kC ? (int)(t_end - c0) : kC;
    const bool has_next = c0 + kC < t_end;
    const int nn = has_next ? ((t_end - c0 - kC) < kC ? (int)(t_end - c0 - kC) : kC) : 0;
    const int buf = ci & 1;
    const uint32_t gsb = sb + OFF_GS + buf * 16384;  // this chunk's g -> gate factors

    cp_async_wait_all();
    fence_proxy_async();  // the raw [K; Q] tile is read by MMA0 below
    __syncthreads();
    GDN_TRACE_POINT(0);

    // ---- MMA0: [K;Q] K^T on the raw bf16 inputs (exact), while the gates,
    // norms and conversions run --------------------------------------------------
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t d = sdesc(sb + OFF_KQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
        mma_f16(tbase + TM_KQ, d, d, ID_BF_KK, kk > 0);
      }
      mma_commit(bar);
    }

    // ---- gates: cumsum of log alpha (log2 units), beta, gamma, exp(G_C - G) ----
    if (warp == 1) {
      const float* gl = sGateBuf + buf * 128;
      float carry = 0.f;
      float Gv[2], bv[2];
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        const int t = hb * 32 + lane;
        float x = gl[t] * kLog2e;
        bv[hb] = gl[64 + t];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float u = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += u;
        }
        Gv[hb] = x + carry;
        carry += __shfl_sync(0xffffffffu, x, 31);
      }
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        const int t = hb * 32 + lane;
        sG2[t] = Gv[hb];
        sBeta[t] = bv[hb];
        sGam[t] = ex2_approx(Gv[hb]);
        sDec[t] = ex2_approx(carry - Gv[hb]);
      }
    }
    // next chunk's gates and g go into the other buffers now
    if (has_next) {
      if (has_g) ld.g(c0 + kC, nn, buf ^ 1);
      ld.gates(c0 + kC, nn, buf ^ 1);
    }
    cp_async_commit();
    __syncthreads();
    GDN_TRACE_POINT(1);

    // ---- L2 norms; K^, dec K^ and gamma Q^ (rows 64-127 of [-W; gamma Q^]) -----
    // warp w owns rows 8w .. 8w+7; 4 lanes per row, 32 columns (4 chunks) each
    {
      const int r = warp * 8 + (lane >> 2);
      const int qc = (lane & 3) * 4;  // first 16-byte chunk of this lane
      float kf[32], qf[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        unpack_bf16x8(ld_shared_v4(sb + OFF_KQ + sw128_chunk(r, qc + c, 128)), kf + 8 * c);
        unpack_bf16x8(ld_shared_v4(sb + OFF_KQ + sw128_chunk(64 + r, qc + c, 128)), qf + 8 * c);
      }
      float nk = 0.f, nq = 0.f;
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        nk += kf[x] * kf[x];
        nq += qf[x] * qf[x];
      }
      nk = group_sum<4>(nk);
      nq = group_sum<4>(nq);
      const float rk = (a.l2norm && r < n) ? rsqrtf(nk + a.eps_l2) : 1.f;
      const float rq = (a.l2norm && r < n) ? rsqrtf(nq + a.eps_l2) : 1.f;
      if ((lane & 3) == 0) {
        sRk[r] = rk;
        sRq[r] = rq;
      }
      const float gq = sGam[r] * rq, dk = sDec[r] * rk;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        st_chunk_f16(sb + OFF_KH + sw128_chunk(r, qc + c, 64), kf + 8 * c, rk);
        st_chunk_f16(sb + OFF_WQ + sw128_chunk(64 + r, qc + c, 128), qf + 8 * c, gq);
        st_chunk_f16(sb + OFF_KT + sw128_chunk(r, qc + c, 64), kf + 8 * c, dk);
      }
    }

    // ---- block maxima of |V| and |S|, chunk exponent e ---------------------------
    float vf[32];
    float vmax = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int idx = tid + kNT * k;
      unpack_bf16x8(ld_shared_v4(sb + OFF_VT + sw128_chunk(idx >> 4, idx & 15, 64)), vf + 8 * k);
    }
#pragma unroll
    for (int x = 0; x < 32; ++x) vmax = fmaxf(vmax, fabsf(vf[x]));
    float sv[64];
    tmem_ld32(tS + half * 64, sv);
    tmem_ld32(tS + half * 64 + 32, sv + 32);
    tmem_wait_ld();
    float smax = 0.f;
#pragma unroll
    for (int x = 0; x < 64; ++x) smax = fmaxf(smax, fabsf(sv[x]));
    const float2 mx = block_max2(vmax, smax, sMax, warp, lane);
    const float mV = mx.x;
    const float mS = ldexpf(mx.y, s_exp);
    // |Delta| <= |v| + |S| ||k^||_1 <= max|V| + 12 max|S|; keep that <= 2^12
    const int e = scale_exp(mV + 12.f * mS, 12);
    {
      const float sv_scale = ldexpf(1.f, -e);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int idx = tid + kNT * k;
        st_chunk_f16(sb + OFF_VT + sw128_chunk(idx >> 4, idx & 15, 64), vf + 8 * k, sv_scale);
      }
      const float to_e = ldexpf(1.f, s_exp - e);
      {
        // S^T 2^-e as the fp16 A operand, in TMEM (d_k pairs per column)
        uint32_t pk[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) pk[x] = pack_f16(sv[2 * x] * to_e, sv[2 * x + 1] * to_e);
        tmem_st32(tSA + half * 32, reinterpret_cast<const float*>(pk));
      }
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
    ok = mbar_wait(bar, phase, kWaitLimit);  // MMA0
    phase ^= 1;
    if (!__syncthreads_and(ok)) { ok = false; break; }
    fence_after_sync();
    // the raw [K; Q] tile is free (MMA0 done, norms read it): next chunk's q, k
    if (has_next) ld.qk(c0 + kC, nn);
    cp_async_commit();
    GDN_TRACE_POINT(2);

    // ---- A (fp32) and P (fp16) from the raw products: all 256 threads -----------
    {
      float v[32];
      tmem_ld32(tKQ + half * 32, v);
      tmem_wait_ld();
      chunk_ap(v, row & 63, half * 32, row < 64, sG2, sBeta, sRk, sRq, sA, sb + OFF_P);
    }
    // T starts from zero (its strictly upper blocks are never computed)
#pragma unroll
    for (int k = 0; k < 4; ++k) reinterpret_cast<float4*>(sT)[tid + kNT * k] = make_float4(0.f, 0.f, 0.f, 0.f);
    fence_before_sync();
    __syncthreads();
    GDN_TRACE_POINT(3);

    // ---- T = (I + A)^{-1} by recursive doubling ---------------------------------
    // 8 x 8 diagonal blocks by substitution, then for block sizes b = 8, 16, 32:
    //   [[T1, 0], [A21, T2]] -> off-diagonal block X = -T2 (A21 T1)
    if (tid < 64) {
      const int b = tid >> 3, c = tid & 7;
      float ab[8][8];
#pragma unroll
      for (int r = 1; r < 8; ++r) {
        const float4 lo = *reinterpret_cast<const float4*>(sA + fidx(8 * b + r, 8 * b));
        const float4 hi = *reinterpret_cast<const float4*>(sA + fidx(8 * b + r, 8 * b + 4));
        ab[r][0] = lo.x; ab[r][1] = lo.y; ab[r][2] = lo.z; ab[r][3] = lo.w;
        ab[r][4] = hi.x; ab[r][5] = hi.y; ab[r][6] = hi.z; ab[r][7] = hi.w;
      }
      float x[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        float s = (r == c) ? 1.f : 0.f;
#pragma unroll
        for (int m = 0; m < r; ++m) s -= ab[r][m] * x[m];
        x[r] = s;
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) sT[fidx(8 * b + r, 8 * b + c)] = x[r];
    }
    __syncthreads();
    tinv_level<8>(sA, sT, sZ, tid);
    tinv_level<16>(sA, sT, sZ, tid);
    tinv_level<32>(sA, sT, sZ, tid);
    GDN_TRACE_POINT(4);

    // ---- scale exponent of T; T diag(b) 2^-f, T diag(b g) 2^-f -> fp16 ---------
    {
      const int t = row & 63;
      const bool withg = row >= 64;
      float tv[32];
      float tmax = 0.f;
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        const float4 x = *reinterpret_cast<const float4*>(sT + fidx(t, half * 32 + i));
        tv[i] = x.x; tv[i + 1] = x.y; tv[i + 2] = x.z; tv[i + 3] = x.w;
        tmax = fmaxf(tmax, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
      }
      const int f = max(0, scale_exp(block_max(tmax, sMax, warp, lane), 8));
      const float sf = ldexpf(1.f, -f);
      // T diag(b g) feeds W, a cancellation when keys repeat: it goes in as
      // fp16 hi + lo (the lo tile reuses the dead A scratch)
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        uint32_t pk[4], pl[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int ia = half * 32 + 8 * c8 + 2 * u;
          float x0 = tv[8 * c8 + 2 * u] * sBeta[ia] * sf;
          float x1 = tv[8 * c8 + 2 * u + 1] * sBeta[ia + 1] * sf;
          if (withg) {
            x0 *= sGam[ia];
            x1 *= sGam[ia + 1];
          }
          split_pack_f16(x0, x1, &pk[u], &pl[u]);
        }
        const uint32_t off = sw128_chunk(t, half * 4 + c8, 64);
        st_shared_v4(sb + (withg ? OFF_TBG : OFF_TB) + off, pk[0], pk[1], pk[2], pk[3]);
        if (withg) st_shared_v4(sb + OFF_TBG_LO + off, pl[0], pl[1], pl[2], pl[3]);
      }
      if (tid == 0) sMax[8] = (float)f;
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    const int f = (int)sMax[8];
    GDN_TRACE_POINT(5);

    // ---- W = (T diag(b g)) K^ (M = 64 tokens, N = 128; hi + lo parts), into
    // TMEM columns TM_W .. +127 ([K; Q] K^T is consumed) ---------------------------
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t da = sdesc(sb + OFF_TBG + kk * 32, 16, 1024);
        const uint64_t db = sdesc(sb + OFF_KH + kk * 2048, 8192, 1024);
        mma_f16(tbase + TM_W, da, db, ID_W64, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t da = sdesc(sb + OFF_TBG_LO + kk * 32, 16, 1024);
        const uint64_t db = sdesc(sb + OFF_KH + kk * 2048, 8192, 1024);
        mma_f16(tbase + TM_W, da, db, ID_W64, 1);
      }
      mma_commit(bar);
    }
    if (has_g && tid >= 32) {
      // meanwhile, warps 1-7: this chunk's gate factors (1 + w) sigmoid(g),
      // in place as fp16 (g landed before the loop-top barrier).  Piece
      // p = tid - 32 + 224 k has column block p % 16 = tid % 16.
#pragma unroll 1
      for (int pc = tid - 32; pc < 1024; pc += 224) {
        const uint32_t addr = gsb + (pc >> 4) * 256 + (pc & 15) * 16;
        float gf[8];
        unpack_bf16x8(ld_shared_v4(addr), gf);
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          o[q] = pack_f16(__fdividef(wv[2 * q], 1.f + __expf(-gf[2 * q])),
                          __fdividef(wv[2 * q + 1], 1.f + __expf(-gf[2 * q + 1])));
        st_shared_v4(addr, o[0], o[1], o[2], o[3]);
      }
    }
    ok = mbar_wait(bar, phase, kWaitLimit);
    phase ^= 1;
    if (!__syncthreads_and(ok)) { ok = false; break; }
    fence_after_sync();
    GDN_TRACE_POINT(6);

    // ---- -W -> rows 0-63 of [-W; gamma Q^] (M = 64 accumulator: row t sits in
    // TMEM lane (t % 16) + 32 (t / 16); warps w and w + 4 take the d_k halves) ---
    {
      float v[64];
      tmem_ld32(tW + half * 64, v);
      tmem_ld32(tW + half * 64 + 32, v + 32);
      tmem_wait_ld();
      if (lane < 16) {
        const int t = 16 * (warp & 3) + lane;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          st_chunk_f16(sb + OFF_WQ + sw128_chunk(t, half * 8 + q, 128), v + 8 * q, -1.f);
      }
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    GDN_TRACE_POINT(7);

    // ---- [Delta^T | Y^T] = S^T [-W; gamma Q^]^T (one N = 128 product per K step),
    // then Delta^T += U^T = V^T (T diag b)^T ---------------------------------------
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t db = sdesc(sb + OFF_WQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
        mma_f16_ta(tbase + TM_D, tbase + TM_SA + kk * 8, db, ID_KK128, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t da = sdesc(sb + OFF_VT + kk * 2048, 8192, 1024);
        const uint64_t db = sdesc(sb + OFF_TB + kk * 32, 16, 1024);
        mma_f16(tbase + TM_D, da, db, ID_MK, 1);
      }
      mma_commit(bar);
    }
    ok = mbar_wait(bar, phase, kWaitLimit);
    phase ^= 1;
    if (!__syncthreads_and(ok)) { ok = false; break; }
    fence_after_sync();
    // the V tile is free: next chunk's v
    if (has_next) ld.v(c0 + kC, nn);
    cp_async_commit();
    GDN_TRACE_POINT(8);

    // ---- Delta^T 2^-e -> fp16 A operand in TMEM (token pairs per column) -------
    {
      float v[32];
      tmem_ld32(tD + half * 32, v);
      tmem_wait_ld();
      const float sf = ldexpf(1.f, f);
      uint32_t pk[16];
#pragma unroll
      for (int x = 0; x < 16; ++x) pk[x] = pack_f16(v[2 * x] * sf, v[2 * x + 1] * sf);
      tmem_st16(tDA + half * 16, pk);
      tmem_wait_st();
    }
    fence_before_sync();
    __syncthreads();
    GDN_TRACE_POINT(9);

    // ---- S^T += Delta^T (dec K^);  Y^T += Delta^T P^T ------------------------------
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t db = sdesc(sb + OFF_KT + kk * 2048, 8192, 1024);
        mma_f16_ta(tbase + TM_S, tbase + TM_DA + kk * 8, db, ID_KM128, 1);
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t db = sdesc(sb + OFF_P + kk * 32, 16, 1024);
        mma_f16_ta(tbase + TM_Y, tbase + TM_DA + kk * 8, db, ID_KK, 1);
      }
      mma_commit(bar);
    }
    ok = mbar_wait(bar, phase, kWaitLimit);
    phase ^= 1;
    if (!__syncthreads_and(ok)) { ok = false; break; }
    fence_after_sync();
    GDN_TRACE_POINT(10);

    // ---- epilogue: y = scale 2^e Y^T; with the gate, out = y rr (1 + w) sigmoid(g)
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
        // y rr (|y rr| <= sqrt(d_v)) as fp16, token-major, into the staging tile
        __half* yst = reinterpret_cast<__half*>(gb + OFF_STG) + half * 32 * kD + row;
        const float4* rr4 = reinterpret_cast<const float4*>(sRr + half * 32);
#pragma unroll
        for (int x4 = 0; x4 < 8; ++x4) {
          const float4 r = rr4[x4];
          yst[(4 * x4 + 0) * kD] = __float2half_rn(v[4 * x4 + 0] * r.x);
          yst[(4 * x4 + 1) * kD] = __float2half_rn(v[4 * x4 + 1] * r.y);
          yst[(4 * x4 + 2) * kD] = __float2half_rn(v[4 * x4 + 2] * r.z);
          yst[(4 * x4 + 3) * kD] = __float2half_rn(v[4 * x4 + 3] * r.w);
        }
        __syncthreads();
        // 8 consecutive outputs of one token per piece, times the gate factors
        const int ch = tid & 15;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int rr = (tid >> 4) + 16 * k;
          if (rr < n) {
            float yf[8], gf[8];
            unpack_f16x8(ld_shared_v4(sb + OFF_STG + rr * 256 + ch * 16), yf);
            unpack_f16x8(ld_shared_v4(gsb + rr * 256 + ch * 16), gf);
            uint32_t o[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
              o[q] = pack_bf16(yf[2 * q] * gf[2 * q], yf[2 * q + 1] * gf[2 * q + 1]);
            *reinterpret_cast<uint4*>(Yg + ((size_t)(c0 + rr) * a.H_v + h) * kD + ch * 8) =
                make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      } else {
        // no gate: y as bf16 through the staging tile, coalesced stores
        __nv_bfloat16* gs = reinterpret_cast<__nv_bfloat16*>(gb + OFF_STG);
#pragma unroll
        for (int x = 0; x < 32; ++x) gs[(half * 32 + x) * kD + row] = __float2bfloat16_rn(v[x]);
        __syncthreads();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int idx = tid + kNT * k;
          const int rr = idx >> 4, ch = idx & 15;
          if (rr < n) {
            const uint4 val = ld_shared_v4(sb + OFF_STG + rr * 256 + ch * 16);
            *reinterpret_cast<uint4*>(Yg + ((size_t)(c0 + rr) * a.H_v + h) * kD + ch * 8) = val;
          }
        }
      }
    }
    fence_before_sync();
    GDN_TRACE_POINT(11);
  }
  cp_async_wait_all();

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

// ============================================================================
// Small-batch layouts: per (sequence, value head) item, a "chain" CTA and
// NPREP "preparation" CTAs.  A preparation CTA does everything that does not
// depend on the state -- L2 norms, [K; Q] K^T, A and P, the triangular
// inverse, T diag(beta), and W (an M = 64 x N = 128 product, stored negated
// and K-major beside gamma Q^) -- and ships the chain's operand tiles per
// chunk: dec K^, [-W; gamma Q^], P and T diag(beta), 64 KB.  The chain CTA
// keeps the state in TMEM, converts S^T and Delta^T to fp16 straight into
// TMEM (MMA A operands), and runs [Delta | Y] = S^T [-W; gamma Q^]^T,
// Delta += U, the state update, Y += Delta P^T and the epilogue.
//
// One 2- or 3-CTA cluster per item; the tiles go over distributed shared
// memory with bulk copies (shared::cta -> shared::cluster, no multicast),
// double-buffered.  "full" barriers in the chain CTA (arrive + expected
// bytes, completed by the copies), "empty" barriers in the preparation CTA
// (arrived by the chain CTA once its MMAs have read a buffer), "staging
// free" barriers in the preparation CTA (arrived once a copy has landed, so
// its source may be overwritten).  Every wait is bounded.  (The workspace
// form of these roles, without a cluster, is the scan layout in
// gdn_prefill_scan.cu.)
// ============================================================================

// chain CTA (rank 0) shared memory
// shipped tiles: dec K^ [t][d_k]; [-W; gamma Q^] [128][d_k] (K-major, rows 0-63
// -W, rows 64-127 gamma Q^: one N = 128 MMA gives [Delta^T | Y^T]); P; T diag(b)
constexpr uint32_t SH_KT = 0, SH_WQ = 16384, SH_P = 49152, SH_TB = 57344;
constexpr uint32_t kShipBytes = 65536;
constexpr uint32_t C_SHIP = 0;            // 2 ship buffers; then V raw -> fp16, the output
                                          // staging tile and g: see the kernel
constexpr uint32_t C_SCAL = 229376;       // shipped scalars [2][4]
constexpr uint32_t C_RED = 229632;        // red[4][64], rr[64], max[16]
constexpr uint32_t C_BAR = 231040;        // full[2], mma, tmem slot
// prep CTA (rank 1) shared memory
constexpr uint32_t P_KQ = 0;              // raw [K; Q] bf16
constexpr uint32_t P_KH = 32768;          // K^ fp16
constexpr uint32_t P_TBG = 49152;         // T diag(b g) 2^-f fp16
constexpr uint32_t P_A = 57344;           // A fp32
constexpr uint32_t P_T = 73728;           // T fp32
constexpr uint32_t P_TBG_LO = P_A;        // remainder of T diag(b g), after A is dead
constexpr uint32_t P_STG = 90112;         // ship staging, 2 x 64 KB
constexpr uint32_t P_Z = 221184;          // Z fp32 [1024]
constexpr uint32_t P_GATEBUF = 225280;    // [2][la, beta][64]
constexpr uint32_t P_GATE = 226304;       // G2, beta, gamma, dec, rk, rq
constexpr uint32_t P_SCAL = 227840;       // scalar staging [2][4]
constexpr uint32_t P_MAX = 227872;        // block-max scratch [16]
constexpr uint32_t P_BAR = 227936;        // empty[2], mma, tmem slot, staging free[2]
constexpr uint32_t kPairSmemBytes = 231072 + 1024;  // the chain CTA's map is the larger

template <int NPREP>
__global__ void __launch_bounds__(kNT, 1) gdn_prefill_tc_pair_kernel(const PrefillArgs a) {
  // chain CTA map: 2 ship buffers (64 KB of tiles each), V, the output
  // staging tile, and 2 buffers for g (converted in place to the gate
  // factors); then C_SCAL / C_RED / C_BAR at fixed offsets.
  // TMEM (512 columns): S^T fp32 0-127, [Delta^T | Y^T] 128-255, and the fp16
  // MMA A operands S^T 2^-e (256-319) and Delta^T 2^-e (320-351).
  constexpr uint32_t kShipStride = kShipBytes;
  constexpr uint32_t X_VT = C_SHIP + 2 * kShipStride;
  constexpr uint32_t X_DT = X_VT + 16384;  // output staging (16 KB)
  constexpr uint32_t X_GS = X_DT + 16384;
  static_assert(X_GS + 2 * 16384 <= C_SCAL, "chain shared-memory map overlaps");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* gb = smem_raw + (sb - raw);
  const uint32_t rank = cluster_ctarank();
  const int item = blockIdx.x / (1 + NPREP);
  const int seq = item / a.H_v;
  const int h = item % a.H_v;
  const int hq = h / (a.H_v / a.H_qk);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = tid & 127;
  const int half = tid >> 7;
  int64_t t_begin, t_end;
  // both CTAs see the same bounds, so both leave before touching the other
  if (!seq_bounds(a.cu_seqlens, seq, a.total_T, &t_begin, &t_end, rank == 0 ? a.err : nullptr))
    return;
  const bool has_g = a.g != nullptr;
  ChunkLoader ld;
  ld.Qg = static_cast<const __nv_bfloat16*>(a.q);
  ld.Kg = static_cast<const __nv_bfloat16*>(a.k);
  ld.Vg = static_cast<const __nv_bfloat16*>(a.v);
  ld.Gg = static_cast<const __nv_bfloat16*>(a.g);
  ld.la = a.log_alpha;
  ld.beta = a.beta;
  ld.H_qk = a.H_qk;
  ld.H_v = a.H_v;
  ld.h = h;
  ld.hq = hq;
  ld.tid = tid;
  ld.sb = sb;
  ld.off_kq = P_KQ;
  ld.off_vt = X_VT;
  ld.off_gs = X_GS;
  ld.off_gate = P_GATEBUF;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  uint32_t phase = 0;
  bool ok = true;

  if (rank == 0) {
    // =========================== chain CTA ===========================
    uint64_t* full = reinterpret_cast<uint64_t*>(gb + C_BAR);
    uint64_t* mbar = reinterpret_cast<uint64_t*>(gb + C_BAR + 16);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(gb + C_BAR + 24);
    float* sRed = reinterpret_cast<float*>(gb + C_RED);
    float* sRr = sRed + 256;
    float* sMax = sRed + 320;
    const float* sScal = reinterpret_cast<const float*>(gb + C_SCAL);
    __nv_bfloat16* Yg = static_cast<__nv_bfloat16*>(a.y);
    const size_t st_off = ((size_t)seq * a.H_v + h) * (size_t)(kD * kD);
    // Copies: V_c+1 is issued after chunk c's first MMA batch, g_c+1 (into
    // buffer (c+1) & 1) at the top of chunk c; the loop top waits for all.
    if (t_begin < t_end) {
      const int n0 = (t_end - t_begin) < kC ? (int)(t_end - t_begin) : kC;
      ld.v(t_begin, n0);
      if (has_g) ld.g(t_begin, n0, 0);
    }
    cp_async_commit();
    if (warp == 0) tmem_alloc(tslot, 512);
    if (tid == 0) {
      mbar_init(&full[0], 1);
      mbar_init(&full[1], 1);
      mbar_init(mbar, 1);
      fence_mbar_init();
    }
    fence_before_sync();
    __syncthreads();
    cluster_sync();
    fence_after_sync();
    const uint32_t tbase = *tslot;
    const uint32_t tS = tbase + lane_off;
    const uint32_t tSA = tbase + lane_off + 256, tDA = tbase + lane_off + 320;
    // TMEM column of [Delta^T | Y^T]
    constexpr uint32_t kDY = 128;
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
    int s_exp = 0;
    // 1 + w for the 8 output columns this thread stores (the same in every
    // chunk: piece index tid + 256 k has column block tid % 16)
    float wv[8];
#pragma unroll
    for (int j2 = 0; j2 < 8; ++j2)
      wv[j2] = 1.f + ((has_g && a.norm_w) ? __ldg(a.norm_w + (tid & 15) * 8 + j2) : 0.f);

    // Epilogue of one chunk in two parts.  (A) Y^T from TMEM, scaled back,
    // with the gate: per-token RMS over d_v and y rr staged as fp16, token-
    // major; without: y staged as bf16.  (B) with the gate: 8 consecutive
    // outputs of one token per piece times the gate factors (gfa), packed to
    // bf16 and stored; without: the staged rows copied out.  Between (A) and
    // (B), and after (B) before the next (A), the caller provides a barrier.
    auto epi_a = [&](uint32_t ty, int ee) {
      float v[32];
      tmem_ld32(ty + half * 32, v);
      tmem_wait_ld();
      const float ys = ldexpf(a.scale, ee);
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
        // y rr (|y rr| <= sqrt(d_v)) as fp16, token-major, into the staging tile
        __half* yst = reinterpret_cast<__half*>(gb + X_DT) + half * 32 * kD + row;
        const float4* rr4 = reinterpret_cast<const float4*>(sRr + half * 32);
#pragma unroll
        for (int x4 = 0; x4 < 8; ++x4) {
          const float4 r = rr4[x4];
          yst[(4 * x4 + 0) * kD] = __float2half_rn(v[4 * x4 + 0] * r.x);
          yst[(4 * x4 + 1) * kD] = __float2half_rn(v[4 * x4 + 1] * r.y);
          yst[(4 * x4 + 2) * kD] = __float2half_rn(v[4 * x4 + 2] * r.z);
          yst[(4 * x4 + 3) * kD] = __float2half_rn(v[4 * x4 + 3] * r.w);
        }
      } else {
        __nv_bfloat16* gs = reinterpret_cast<__nv_bfloat16*>(gb + X_DT);
#pragma unroll
        for (int x = 0; x < 32; ++x) gs[(half * 32 + x) * kD + row] = __float2bfloat16_rn(v[x]);
      }
    };
    auto epi_b = [&](int64_t cc0, int nc, uint32_t gfa) {
      const int ch = tid & 15;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int rr = (tid >> 4) + 16 * k;
        if (rr < nc) {
          uint4 val = ld_shared_v4(sb + X_DT + rr * 256 + ch * 16);
          if (has_g) {
            float yf[8], gf[8];
            unpack_f16x8(val, yf);
            unpack_f16x8(ld_shared_v4(gfa + rr * 256 + ch * 16), gf);
            val = make_uint4(pack_bf16(yf[0] * gf[0], yf[1] * gf[1]),
                             pack_bf16(yf[2] * gf[2], yf[3] * gf[3]),
                             pack_bf16(yf[4] * gf[4], yf[5] * gf[5]),
                             pack_bf16(yf[6] * gf[6], yf[7] * gf[7]));
          }
          *reinterpret_cast<uint4*>(Yg + ((size_t)(cc0 + rr) * a.H_v + h) * kD + ch * 8) = val;
        }
      }
    };
    int ci = 0;
    for (int64_t c0 = t_begin; c0 < t_end; c0 += kC, ++ci) {
      const int n = (t_end - c0) < kC ? (int)(t_end - c0) : kC;
      const bool has_next = c0 + kC < t_end;
      const int nn = has_next ? ((t_end - c0 - kC) < kC ? (int)(t_end - c0 - kC) : kC) : 0;
      const int b = ci & 1;
      const uint32_t ship = sb + C_SHIP + b * kShipStride;
      // this chunk's gate factors, computed here from g in place (buffer b)
      const uint32_t gsb = sb + X_GS + b * 16384;
      cp_async_wait_all();
      // the other g buffer was last read by the previous chunk's epilogue
      if (has_next && has_g) ld.g(c0 + kC, nn, b ^ 1);
      cp_async_commit();
      bool okw = true;
      __syncthreads();
      GDN_TRACE_POINT(0);
      okw = mbar_wait_cluster(&full[b], (ci >> 1) & 1, kWaitLimit);
      if (!__syncthreads_and(okw)) { ok = false; break; }
      // the copy has landed: its source staging buffer may be reused
      if (tid == 0)
        mbar_remote_arrive(
            mapa_shared(sb + P_BAR + 32 + 8 * ((ci / NPREP) & 1), 1 + ci % NPREP));
      GDN_TRACE_POINT(1);
      const float gC = sScal[b * 4 + 0];
      const int f = (int)sScal[b * 4 + 1];

      // V, S maxima -> e; V 2^-e and S^T 2^-e to fp16; state rescaled
      float vf[32];
      float vmax = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int idx = tid + kNT * k;
        unpack_bf16x8(ld_shared_v4(sb + X_VT + sw128_chunk(idx >> 4, idx & 15, 64)), vf + 8 * k);
      }
#pragma unroll
      for (int x = 0; x < 32; ++x) vmax = fmaxf(vmax, fabsf(vf[x]));
      float sv[64];
      tmem_ld32(tS + half * 64, sv);
      tmem_ld32(tS + half * 64 + 32, sv + 32);
      tmem_wait_ld();
      float smax = 0.f;
#pragma unroll
      for (int x = 0; x < 64; ++x) smax = fmaxf(smax, fabsf(sv[x]));
      const float2 mx = block_max2(vmax, smax, sMax, warp, lane);
      const float mV = mx.x;
      const float mS = ldexpf(mx.y, s_exp);
      const int e = scale_exp(mV + 12.f * mS, 12);
      {
        const float sv_scale = ldexpf(1.f, -e);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int idx = tid + kNT * k;
          st_chunk_f16(sb + X_VT + sw128_chunk(idx >> 4, idx & 15, 64), vf + 8 * k, sv_scale);
        }
        const float to_e = ldexpf(1.f, s_exp - e);
        {
          // S^T 2^-e as the fp16 A operand, in TMEM (d_k pairs per column)
          uint32_t pk[32];
#pragma unroll
          for (int x = 0; x < 32; ++x) pk[x] = pack_f16(sv[2 * x] * to_e, sv[2 * x + 1] * to_e);
          tmem_st32(tSA + half * 32, reinterpret_cast<const float*>(pk));
        }
        const float upd = gC * to_e;
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
      GDN_TRACE_POINT(2);

      // [Delta^T | Y^T] = S^T [-W; gamma Q^]^T (one N = 128 product), then
      // Delta^T += U^T = V^T (T diag b)^T
      if (tid == 0) {
        fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t db = sdesc(ship + SH_WQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          mma_f16_ta(tbase + kDY, tbase + 256 + kk * 8, db, ID_KK128, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t da = sdesc(sb + X_VT + kk * 2048, 8192, 1024);
          const uint64_t db = sdesc(ship + SH_TB + kk * 32, 16, 1024);
          mma_f16(tbase + kDY, da, db, ID_MK, 1);
        }
        mma_commit(mbar);
      }
      if (has_g && tid >= 64) {
        // Also while the MMAs run: this chunk's gate factors (1 + w)
        // sigmoid(g), in place as fp16 (g landed before the loop-top
        // barrier).  Warps 2-7 only: warp 0 issues the MMAs, warp 1 fetches.
        // Piece p = tid - 64 + 192 k has column block p % 16 = tid % 16.
#pragma unroll 1
        for (int pc = tid - 64; pc < 1024; pc += 192) {
          const uint32_t addr = gsb + (pc >> 4) * 256 + (pc & 15) * 16;
          float gf[8];
          unpack_bf16x8(ld_shared_v4(addr), gf);
          uint32_t o[4];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            o[q] = pack_f16(__fdividef(wv[2 * q], 1.f + __expf(-gf[2 * q])),
                            __fdividef(wv[2 * q + 1], 1.f + __expf(-gf[2 * q + 1])));
          st_shared_v4(addr, o[0], o[1], o[2], o[3]);
        }
      }
      okw = mbar_wait(mbar, phase, kWaitLimit);
      phase ^= 1;
      if (!__syncthreads_and(okw)) { ok = false; break; }
      fence_after_sync();
      if (has_next) ld.v(c0 + kC, nn);
      cp_async_commit();
      GDN_TRACE_POINT(3);

      // Delta^T 2^-e -> fp16 A operand in TMEM (token pairs per column)
      {
        float v[32];
        tmem_ld32(tbase + lane_off + kDY + half * 32, v);
        tmem_wait_ld();
        const float sf = ldexpf(1.f, f);
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) pk[x] = pack_f16(v[2 * x] * sf, v[2 * x + 1] * sf);
        tmem_st16(tDA + half * 16, pk);
        tmem_wait_st();
      }
      fence_before_sync();
      __syncthreads();
      GDN_TRACE_POINT(4);

      // S^T += Delta^T (dec K^);  Y^T += Delta^T P^T
      if (tid == 0) {
        fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t db = sdesc(ship + SH_KT + kk * 2048, 8192, 1024);
          mma_f16_ta(tbase, tbase + 320 + kk * 8, db, ID_KM128, 1);
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t db = sdesc(ship + SH_P + kk * 32, 16, 1024);
          mma_f16_ta(tbase + kDY + 64, tbase + 320 + kk * 8, db, ID_KK, 1);
        }
        mma_commit(mbar);
      }
      okw = mbar_wait(mbar, phase, kWaitLimit);
      phase ^= 1;
      if (!__syncthreads_and(okw)) { ok = false; break; }
      fence_after_sync();
      // this chunk's shipped tiles are no longer read: hand the buffer back
      if (tid == 0) mbar_remote_arrive(mapa_shared(sb + P_BAR + 8 * b, 1 + ci % NPREP));
      GDN_TRACE_POINT(5);

      // epilogue now (its gate factors were converted in place, buffer b)
      epi_a(tbase + lane_off + kDY + 64, e);
      __syncthreads();
      epi_b(c0, n, gsb);
      __syncthreads();  // staging reads done: g buffer and staging tile reusable
      fence_before_sync();
      GDN_TRACE_POINT(6);
    }
    cp_async_wait_all();
    if (ok) {
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
      mbar_wait(mbar, phase ^ 1, kWaitLimit);
      // a copy into this CTA's buffers that may still be landing
      if (t_begin + (int64_t)(ci + 1) * kC < t_end)
        mbar_wait_cluster(&full[(ci + 1) & 1], ((ci + 1) >> 1) & 1, kWaitLimit >> 6);
    }
    fence_before_sync();
    __syncthreads();
    cluster_sync();
    if (warp == 0) tmem_dealloc(tbase, 512);
  } else {
    // =========================== prep CTA ============================
    uint64_t* empty = reinterpret_cast<uint64_t*>(gb + P_BAR);
    uint64_t* mbar = reinterpret_cast<uint64_t*>(gb + P_BAR + 16);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(gb + P_BAR + 24);
    uint64_t* stg_free = reinterpret_cast<uint64_t*>(gb + P_BAR + 32);
    float* sA = reinterpret_cast<float*>(gb + P_A);
    float* sT = reinterpret_cast<float*>(gb + P_T);
    float* sZ = reinterpret_cast<float*>(gb + P_Z);
    const float* sGateBuf = reinterpret_cast<const float*>(gb + P_GATEBUF);
    float* sG2 = reinterpret_cast<float*>(gb + P_GATE);
    float* sBeta = sG2 + 64;
    float* sGam = sG2 + 128;
    float* sDec = sG2 + 192;
    float* sRk = sG2 + 256;
    float* sRq = sG2 + 320;
    float* sScal = reinterpret_cast<float*>(gb + P_SCAL);
    float* sMax = reinterpret_cast<float*>(gb + P_MAX);
    // prep CTA r handles chunks r-1, r-1+NPREP, ...
    const int first = (int)rank - 1;
    const int64_t c_first = t_begin + (int64_t)kC * first;
    if (c_first < t_end) {
      const int n0 = (t_end - c_first) < kC ? (int)(t_end - c_first) : kC;
      ld.qk(c_first, n0);
      ld.gates(c_first, n0, 0);
      cp_async_commit();
    }
    if (warp == 0) tmem_alloc(tslot, 128);
    if (tid == 0) {
      mbar_init(&empty[0], 1);
      mbar_init(&empty[1], 1);
      mbar_init(mbar, 1);
      mbar_init(&stg_free[0], 1);
      mbar_init(&stg_free[1], 1);
      fence_mbar_init();
    }
    fence_before_sync();
    __syncthreads();
    cluster_sync();
    fence_after_sync();
    const uint32_t tbase = *tslot;
    const uint32_t tKQ = tbase + lane_off, tW = tbase + lane_off;
    const uint32_t full_cl0 = mapa_shared(sb + C_BAR, 0);
    const uint32_t ship_cl0 = mapa_shared(sb + C_SHIP, 0);
    const uint32_t scal_cl0 = mapa_shared(sb + C_SCAL, 0);

    int ci = first, lc = 0;  // chunk index, local count
    for (int64_t c0 = c_first; c0 < t_end; c0 += (int64_t)kC * NPREP, ci += NPREP, ++lc) {
      const int n = (t_end - c0) < kC ? (int)(t_end - c0) : kC;
      const int64_t cnext = c0 + (int64_t)kC * NPREP;
      const bool has_next = cnext < t_end;
      const int nn = has_next ? ((t_end - cnext) < kC ? (int)(t_end - cnext) : kC) : 0;
      const int b = ci & 1;       // buffer in the chain CTA
      const int lb = lc & 1;      // local staging / prefetch buffer
      const uint32_t stg = sb + P_STG + lb * kShipBytes;
      cp_async_wait_all();
      fence_proxy_async();  // the raw [K; Q] tile is read by MMA0 below
      bool okw = true;
      // staging buffer lb was the source of the copy two local chunks ago;
      // the chain CTA reports when that copy has landed
      if (tid == 0 && lc >= 2)
        okw = mbar_wait_cluster(&stg_free[lb], ((lc - 2) >> 1) & 1, kWaitLimit);
      if (!__syncthreads_and(okw)) { ok = false; break; }
      GDN_TRACE_POINT(20);

      // [K; Q] K^T on the raw inputs, overlapped with the gates and norms
      if (tid == 0) {
        fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t d = sdesc(sb + P_KQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          mma_f16(tbase, d, d, ID_BF_KK, kk > 0);
        }
        mma_commit(mbar);
      }

      // gates (warp 1: thread 0 of warp 0 has just issued the MMAs)
      if (warp == 1) {
        const float* gl = sGateBuf + lb * 128;
        float carry = 0.f;
        float Gv[2], bv[2];
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
          const int t = hb * 32 + lane;
          float x = gl[t] * kLog2e;
          bv[hb] = gl[64 + t];
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += u;
          }
          Gv[hb] = x + carry;
          carry += __shfl_sync(0xffffffffu, x, 31);
        }
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
          const int t = hb * 32 + lane;
          sG2[t] = Gv[hb];
          sBeta[t] = bv[hb];
          sGam[t] = ex2_approx(Gv[hb]);
          sDec[t] = ex2_approx(carry - Gv[hb]);
        }
        if (lane == 0) sScal[lb * 4 + 0] = ex2_approx(carry);
      }
      if (has_next) ld.gates(cnext, nn, lb ^ 1);
      cp_async_commit();
      GDN_TRACE_POINT(21);
      __syncthreads();

      // norms -> K^ (local), gamma Q^ and dec K^ (shipped)
      {
        const int r = warp * 8 + (lane >> 2);
        const int qc = (lane & 3) * 4;
        float kf[32], qf[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          unpack_bf16x8(ld_shared_v4(sb + P_KQ + sw128_chunk(r, qc + c, 128)), kf + 8 * c);
          unpack_bf16x8(ld_shared_v4(sb + P_KQ + sw128_chunk(64 + r, qc + c, 128)), qf + 8 * c);
        }
        float nk = 0.f, nq = 0.f;
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          nk += kf[x] * kf[x];
          nq += qf[x] * qf[x];
        }
        nk = group_sum<4>(nk);
        nq = group_sum<4>(nq);
        const float rk = (a.l2norm && r < n) ? rsqrtf(nk + a.eps_l2) : 1.f;
        const float rq = (a.l2norm && r < n) ? rsqrtf(nq + a.eps_l2) : 1.f;
        if ((lane & 3) == 0) {
          sRk[r] = rk;
          sRq[r] = rq;
        }
        const float gq = sGam[r] * rq, dk = sDec[r] * rk;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          st_chunk_f16(sb + P_KH + sw128_chunk(r, qc + c, 64), kf + 8 * c, rk);
          st_chunk_f16(stg + SH_WQ + sw128_chunk(64 + r, qc + c, 128), qf + 8 * c, gq);
          st_chunk_f16(stg + SH_KT + sw128_chunk(r, qc + c, 64), kf + 8 * c, dk);
        }
      }
      fence_proxy_async();
      fence_before_sync();
      okw = mbar_wait(mbar, phase, kWaitLimit);
      phase ^= 1;
      if (!__syncthreads_and(okw)) { ok = false; break; }
      fence_after_sync();
      if (has_next) ld.qk(cnext, nn);
      cp_async_commit();
      GDN_TRACE_POINT(22);

      // A (fp32) and P (fp16, shipped)
      {
        float v[32];
        tmem_ld32(tKQ + half * 32, v);
        tmem_wait_ld();
        chunk_ap(v, row & 63, half * 32, row < 64, sG2, sBeta, sRk, sRq, sA, stg + SH_P);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k)
        reinterpret_cast<float4*>(sT)[tid + kNT * k] = make_float4(0.f, 0.f, 0.f, 0.f);
      fence_before_sync();
      __syncthreads();
      GDN_TRACE_POINT(23);

      // T = (I + A)^{-1}
      if (tid < 64) {
        const int bq = tid >> 3, c = tid & 7;
        float ab[8][8];
#pragma unroll
        for (int r = 1; r < 8; ++r) {
          const float4 lo = *reinterpret_cast<const float4*>(sA + fidx(8 * bq + r, 8 * bq));
          const float4 hi = *reinterpret_cast<const float4*>(sA + fidx(8 * bq + r, 8 * bq + 4));
          ab[r][0] = lo.x; ab[r][1] = lo.y; ab[r][2] = lo.z; ab[r][3] = lo.w;
          ab[r][4] = hi.x; ab[r][5] = hi.y; ab[r][6] = hi.z; ab[r][7] = hi.w;
        }
        float x[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          float s = (r == c) ? 1.f : 0.f;
#pragma unroll
          for (int m = 0; m < r; ++m) s -= ab[r][m] * x[m];
          x[r] = s;
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) sT[fidx(8 * bq + r, 8 * bq + c)] = x[r];
      }
      __syncthreads();
      tinv_level<8>(sA, sT, sZ, tid);
      tinv_level<16>(sA, sT, sZ, tid);
      tinv_level<32>(sA, sT, sZ, tid);
      GDN_TRACE_POINT(24);

      // f; T diag(b) 2^-f (shipped), T diag(b g) 2^-f (local)
      {
        const int t = row & 63;
        const bool withg = row >= 64;
        float tv[32];
        float tmax = 0.f;
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 x = *reinterpret_cast<const float4*>(sT + fidx(t, half * 32 + i));
          tv[i] = x.x; tv[i + 1] = x.y; tv[i + 2] = x.z; tv[i + 3] = x.w;
          tmax = fmaxf(tmax, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
        }
        const int f = max(0, scale_exp(block_max(tmax, sMax, warp, lane), 8));
        const float sf = ldexpf(1.f, -f);
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          uint32_t pk[4], pl[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int ia = half * 32 + 8 * c8 + 2 * u;
            float x0 = tv[8 * c8 + 2 * u] * sBeta[ia] * sf;
            float x1 = tv[8 * c8 + 2 * u + 1] * sBeta[ia + 1] * sf;
            if (withg) {
              x0 *= sGam[ia];
              x1 *= sGam[ia + 1];
            }
            split_pack_f16(x0, x1, &pk[u], &pl[u]);
          }
          const uint32_t off = sw128_chunk(t, half * 4 + c8, 64);
          st_shared_v4((withg ? sb + P_TBG : stg + SH_TB) + off, pk[0], pk[1], pk[2], pk[3]);
          if (withg) st_shared_v4(sb + P_TBG_LO + off, pl[0], pl[1], pl[2], pl[3]);
        }
        if (tid == 0) sScal[lb * 4 + 1] = (float)f;
      }
      fence_proxy_async();
      fence_before_sync();
      __syncthreads();
      GDN_TRACE_POINT(25);

      // W = (T diag(b g)) K^ (M = 64 tokens, N = 128 = d_k; hi + lo parts
      // of T diag(b g)), into TMEM columns 0-127 ([K; Q] K^T is consumed)
      if (tid == 0) {
        fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t da = sdesc(sb + P_TBG + kk * 32, 16, 1024);
          const uint64_t db = sdesc(sb + P_KH + kk * 2048, 8192, 1024);
          mma_f16(tbase, da, db, ID_W64, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t da = sdesc(sb + P_TBG_LO + kk * 32, 16, 1024);
          const uint64_t db = sdesc(sb + P_KH + kk * 2048, 8192, 1024);
          mma_f16(tbase, da, db, ID_W64, 1);
        }
        mma_commit(mbar);
      }
      okw = mbar_wait(mbar, phase, kWaitLimit);
      phase ^= 1;
      if (!__syncthreads_and(okw)) { ok = false; break; }
      fence_after_sync();
      {
        // M = 64 accumulator: row t sits in TMEM lane (t % 16) + 32 (t / 16),
        // i.e. lanes 0-15 of warp quarter t / 16; warps w and w + 4 take the
        // two halves of d_k.  -W goes to rows 0-63 of the merged tile.
        float v[64];
        tmem_ld32(tW + half * 64, v);
        tmem_ld32(tW + half * 64 + 32, v + 32);
        tmem_wait_ld();
        if (lane < 16) {
          const int t = 16 * (warp & 3) + lane;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            st_chunk_f16(stg + SH_WQ + sw128_chunk(t, half * 8 + q, 128), v + 8 * q, -1.f);
        }
      }
      fence_proxy_async();
      fence_before_sync();
      __syncthreads();
      GDN_TRACE_POINT(26);

      // ship this chunk's tiles once the chain CTA has released buffer b
      okw = true;
      if (tid == 0) {
        okw = mbar_wait_cluster(&empty[b], ((ci >> 1) & 1) ^ 1, kWaitLimit);
        if (okw) {
          // the cluster window keeps the peer's layout: offsets carry over
          const uint32_t full_cl = full_cl0 + 8 * b;
          const uint32_t ship_cl = ship_cl0 + b * kShipBytes;
          mbar_remote_arrive_expect_tx(full_cl, kShipBytes + 16);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            bulk_copy_to_peer(ship_cl + 16384 * k, stg + 16384 * k, 16384, full_cl);
          bulk_copy_to_peer(scal_cl0 + 16 * b, sb + P_SCAL + 16 * lb, 16, full_cl);
        }
      }
      if (!__syncthreads_and(okw)) { ok = false; break; }
      GDN_TRACE_POINT(27);
    }
    cp_async_wait_all();
    if (!ok) {
      if (tid == 0) atomicOr(a.err, kErrTimeout);
      mbar_wait(mbar, phase ^ 1, kWaitLimit);
    }
    fence_before_sync();
    __syncthreads();
    cluster_sync();
    if (warp == 0) tmem_dealloc(tbase, 128);
  }
}

// Larger batches (more than kScanMaxItems items, at most kMaxOrderSeqs
// sequences) with a workspace: the one-CTA layout takes the sequences
// longest first.
constexpr int kMaxOrderSeqs = 1024;

// order[r] = the sequence of rank r by decreasing length (ties: lower index
// first); one CTA of kMaxOrderSeqs threads, one sequence each.  cu_seqlens
// is only read: the prefill kernel validates it.
__global__ void __launch_bounds__(kMaxOrderSeqs) order_by_length_kernel(const int32_t* cu,
                                                                        int n_seq,
                                                                        int64_t total_T,
                                                                        int32_t* order) {
  __shared__ int64_t len[kMaxOrderSeqs];
  const int s = threadIdx.x;
  if (s < n_seq) len[s] = cu ? (int64_t)cu[s + 1] - cu[s] : total_T;
  __syncthreads();
  if (s < n_seq) {
    const int64_t ls = len[s];
    int rank = 0;
    for (int j = 0; j < n_seq; ++j) rank += (len[j] > ls || (len[j] == ls && j < s)) ? 1 : 0;
    order[rank] = s;
  }
}

}  // namespace

bool prefill_tc_supports(const PrefillArgs& a) {
  return a.dtype == GDN_BF16 && a.d_k == kD && a.d_v == kD;
}

// Workspace: batches of at most kScanMaxItems items take the scan layout
// (gdn_prefill_scan.cu), whose hand-off ring lives in it (scan_ws_bytes).
// Larger batches of at most kMaxOrderSeqs sequences use the workspace for
// the one-CTA layout's sequence order instead (n_seq int32, longest first).
size_t prefill_tc_workspace_bytes(int32_t n_seq, int32_t H_v, int32_t d_k, int32_t d_v,
                                  gdn_dtype dtype) {
  const long long items = (long long)n_seq * H_v;
  if (dtype != GDN_BF16 || d_k != kD || d_v != kD || items < 1) return 0;
  if (items > kScanMaxItems)
    return n_seq <= kMaxOrderSeqs ? (((size_t)n_seq * sizeof(int32_t) + 255) & ~(size_t)255) : 0;
  return scan_ws_bytes(items);
}

void prefill_tc_workspace_layout(void* ws, int32_t n_seq, int32_t H_v, PrefillArgs* a) {
  const long long items = (long long)n_seq * H_v;
  if (items > kScanMaxItems) {
    a->seq_order = static_cast<int32_t*>(ws);
    return;
  }
  a->ring_flags = static_cast<unsigned long long*>(ws);
  a->ring = static_cast<uint8_t*>(ws) + scan_flag_bytes(items);
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
  static bool pair_attr_set[64][2] = {{false}};
  const long long items = (long long)a.n_seq * a.H_v;
  // Scan layout (needs the workspace): a chain CTA and two preparation CTAs
  // per item in one cooperative launch, when every CTA can be resident.
  auto scan_fits = [&]() -> bool {
    return a.ring != nullptr && a.ring_flags != nullptr && items <= kScanMaxItems &&
           items <= prefill_scan_capacity();
  };
  if (a.tc_variant == 3 || (a.tc_variant == 0 && a.total_T >= kC && scan_fits())) {
    if (!scan_fits()) return GDN_ERR_UNSUPPORTED;
    return launch_prefill_scan(a, stream);
  }
  // While there are too few (sequence, head) items to fill the GPU, give each
  // a cluster: one chain CTA plus one or two preparation CTAs -- but only a
  // cluster size whose clusters all fit on the GPU at once (a second wave
  // would double the time).
  static int max_clusters[64][2] = {{0}};
  auto fits = [&](int np) -> bool {
    if (dev < 0 || dev >= 64) return false;
    if (max_clusters[dev][np - 1] == 0) {
      const void* fn = np == 2 ? (const void*)gdn_prefill_tc_pair_kernel<2>
                               : (const void*)gdn_prefill_tc_pair_kernel<1>;
      if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kPairSmemBytes) != cudaSuccess)
        return false;
      pair_attr_set[dev][np - 1] = true;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)(1 + np), 1, 1);
      cfg.blockDim = dim3(kNT, 1, 1);
      cfg.dynamicSmemBytes = kPairSmemBytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 1 + np;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int mc = 0;
      if (cudaOccupancyMaxActiveClusters(&mc, fn, &cfg) != cudaSuccess) mc = -1;
      max_clusters[dev][np - 1] = mc;
    }
    return max_clusters[dev][np - 1] >= items;
  };
  int nprep = 0;
  if (a.tc_variant == 1) nprep = fits(2) ? 2 : 1;
  else if (a.tc_variant == 0) nprep = fits(2) ? 2 : (fits(1) ? 1 : 0);
  if (nprep > 0) {
    const void* fn = nprep == 2 ? (const void*)gdn_prefill_tc_pair_kernel<2>
                                : (const void*)gdn_prefill_tc_pair_kernel<1>;
    if (dev < 0 || dev >= 64 || !pair_attr_set[dev][nprep - 1]) {
      if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kPairSmemBytes) != cudaSuccess)
        return GDN_ERR_CUDA;
      if (dev >= 0 && dev < 64) pair_attr_set[dev][nprep - 1] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((1 + nprep) * items), 1, 1);
    cfg.blockDim = dim3(kNT, 1, 1);
    cfg.dynamicSmemBytes = kPairSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1 + nprep;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t err = nprep == 2 ? cudaLaunchKernelEx(&cfg, gdn_prefill_tc_pair_kernel<2>, a)
                                 : cudaLaunchKernelEx(&cfg, gdn_prefill_tc_pair_kernel<1>, a);
    if (err != cudaSuccess) return GDN_ERR_CUDA;
  } else {
    if (a.seq_order != nullptr) {
      order_by_length_kernel<<<1, kMaxOrderSeqs, 0, stream>>>(a.cu_seqlens, a.n_seq, a.total_T,
                                                              a.seq_order);
    }
    gdn_prefill_tc_kernel<<<(unsigned)items, kNT, kSmemBytes, stream>>>(a);
  }
  return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn
