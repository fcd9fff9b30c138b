// Chunked prefill of the gated delta rule on the sm_100a tensor cores, for
// small batches: the "scan" layout.  bf16 inputs, d_k = d_v = 128.
//
// The recurrence ("Qwen3.8-Flash-Next: architecture, efficiency and technical
// lineage", section 03 "Gated DeltaNet", update equations) is regrouped per
// chunk of C = 64 tokens.  With the entering state S (d_k x d_v),
// G_t = sum_{s<=t} log alpha_s, K^, Q^ the L2-normalised keys / queries:
//
//   A     = strict_lower(diag(beta) (exp(G_t - G_i)) o K^ K^T),  T = (I + A)^{-1}
//   W     = T diag(beta gamma) K^            U = T diag(beta) V
//   Delta = U - W S                          (the values the chunk writes)
//   Y     = diag(gamma) Q^ S + P Delta,      P = lower(exp(G_t - G_i)) o Q^ K^T
//   S    <- gamma_C S + (diag(exp(G_C - G)) K^)^T Delta
//
// Only S depends on the previous chunk.  Per (sequence, value head) item the
// work is split accordingly:
//
//   * four preparation sub-pipelines (two CTAs, each with two sub-pipelines
//     of four compute warps and one control thread) take the chunks in turn
//     (chunk c goes to sub-pipeline c % 4) and do everything that does not
//     need S: q, k, v arrive by TMA (3-D tiles, 128-byte swizzle, straight
//     into the MMA operand layout); [K; Q] K^T on the raw bf16 inputs (exact
//     products, norms applied in fp32); A and P; T by recursive doubling
//     (fp32); W and U^T as bf16 MMAs on the raw k and v tiles with T diag(.)
//     split into bf16 hi + lo parts (about 16 significant bits).  fp16 -W,
//     dec K^, gamma Q^, U^T 2^-e_u and P (72 KB) are staged in shared memory
//     in the slot's layout and bulk-copied into a slot of a per-item ring in
//     the workspace (L2); the control thread then publishes the slot with a
//     release flag;
//   * one chain CTA keeps S in the registers of its eight compute warps
//     (fp32, 64 values per thread) and writes fp16 S^T 2^-e and Delta^T 2^-e
//     into tensor memory as the A operands of the per-chunk products, whose
//     B operands come from the slot in shared memory: [Delta^T | Y^T] =
//     S^T [-W; gamma Q^]^T (Delta^T then gains U^T in fp32), S^T += Delta^T K~
//     (K~ = dec K^) and Y^T += Delta^T P^T.  One thread issues the products,
//     one thread loads the slot (in three parts, each as soon as its buffer
//     is free) and the raw g by TMA, and two epilogue warps apply RMSNorm x
//     (1 + w) sigmoid(g) to chunk c - 1's staged Y while chunk c runs.  The
//     fp16 copies of S and Delta carry a per-chunk power-of-two exponent e
//     from max|V| + 12 max|S| (|Delta| <= |v| + |S| ||k^||_1).
//
// All CTAs (chain + two preparation CTAs per item, 384 threads each) are one
// cooperative launch, so they are co-resident.  Every wait is bounded; a
// wait that runs out sets the device error word and the CTA winds down
// without faulting.
#include <cuda.h>

#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_sm100.cuh"

// Section timing hook for tuning builds (role 0: chain thread 0; role 1:
// preparation thread 0 of sub-pipeline 0); compiles to nothing by default.
#ifndef GDN_SCAN_TRACE
#define GDN_SCAN_TRACE(role, id)
#define GDN_SCAN_TRACE_INIT()
#endif

namespace gdn {
namespace {

using namespace sm100;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kCta = 384;      // threads per CTA (12 warps, both roles)
constexpr int kSubT = 128;     // compute threads of a preparation sub-pipeline (4 warps)
constexpr int kSubs = 2;       // sub-pipelines per preparation CTA
constexpr int kPrepCtas = 2;   // preparation CTAs per item
constexpr int kLanes = kSubs * kPrepCtas;  // sub-pipelines per item: chunk c goes to c % kLanes
constexpr int kRingS = kScanRing;
constexpr int kChainT = 256;   // compute threads of the chain CTA (8 warps)
constexpr int kCtrlWarp = 8;   // the chain CTA's MMA warp
constexpr int kLoadWarp = 11;  // the chain CTA's loader warp (slot and g copies)
constexpr int kEpiWarp = 9;    // first of the chain CTA's two epilogue warps
constexpr int kEpiT = 64;

constexpr uint32_t kWait = 1u << 24;
constexpr uint32_t kDrain = 1u << 16;
constexpr float kLog2e = 1.4426950408889634f;

// ---- a ring slot (global image) ---------------------------------------------------
// The chain CTA bulk-loads the slot (MMA operands, scalars and U^T) into
// shared memory, in three parts.
constexpr uint32_t SL_WQ = 0;       // [-W; gamma Q^] fp16 [128 rows][128 d_k], SW128, 2 panels
                                    //   x 16 KB: rows 0-63 -W (token t), rows 64-127 gamma Q^
constexpr uint32_t SL_K = 32768;    // dec K^ fp16 [64 t][128 d_k], SW128, 2 panels x 8 KB
constexpr uint32_t SL_P = 49152;    // P fp16 [64 t][64 i], SW128, 1 panel
constexpr uint32_t SL_SCAL = 57344; // gamma_C, e_u, max|V|, valid rows (fp32 x 4)
constexpr uint32_t SL_U = 57600;    // U^T 2^-e_u fp16 [128 d_v][64 t], 16-byte chunks of row j
                                    //   at position chunk ^ (j % 8)
constexpr uint32_t kSlotLoadBytes = SL_U + 16384;
static_assert(kScanSlotBytes >= kSlotLoadBytes && kScanSlotBytes % 256 == 0, "slot size");

// ---- chain CTA shared memory ------------------------------------------------------
constexpr uint32_t kSlotStride = 74752;           // a slot copy (chunk c in buffer c % 2)
constexpr uint32_t C_YS = 2 * kSlotStride;        // Y^T 2^-e stages: 2 x fp16 [64 t][128 j],
                                                  //   16-byte chunk c of row t at c ^ (t % 16)
constexpr uint32_t C_GS = C_YS + 32768;           // raw g of the staged chunks (TMA): 2 x
                                                  //   bf16 [64 t][128 j], SW128, 2 panels
constexpr uint32_t C_WN = C_GS + 32768;           // 1 + norm_w [128] fp32
constexpr uint32_t C_MISC = C_WN + 512;           // warp maxima [2][8], stage exponents [2]
constexpr uint32_t C_BAR = C_MISC + 128;           // fullA[2] bar1 bar3 barY[2] ysfull[2]
                                                  //   ysempty[2] sready dready gfull[2]
                                                  //   fullB[2] fullC[2] bar1b[2] ufree[2],
                                                  //   TMEM slot
constexpr uint32_t kChainSmem = C_BAR + 256;

// ---- preparation sub-pipeline shared memory (two per CTA) -------------------------
constexpr uint32_t P_KQ = 0;           // [K; Q] raw bf16 [128][128], SW128, 2 panels x 16 KB
constexpr uint32_t P_V = 32768;        // V raw bf16 [64][128], 2 panels x 8 KB
constexpr uint32_t P_A = 49152;        // A fp32 64 x 64; after the inverse: W splits
constexpr uint32_t P_TWH = P_A;        // T diag(beta gamma rk) hi, bf16 [64][64]
constexpr uint32_t P_TWL = P_A + 8192; //   ... lo
constexpr uint32_t P_T = 65536;        // T fp32 64 x 64
constexpr uint32_t P_TBH = 81920;      // T diag(beta) hi, bf16 [64][64]
constexpr uint32_t P_TBL = 90112;      //   ... lo
constexpr uint32_t P_Z = 98304;        // doubling scratch, fp32 [1024]
constexpr uint32_t P_GB = 102400;      // gate staging [log alpha, beta][64] fp32
constexpr uint32_t P_G = 102912;       // G2, beta, gamma, dec, rk, rq: 6 x 64 fp32
constexpr uint32_t P_MAX = 104448;     // max|V| per warp [4], max|U| per warp [4], gamma_C
constexpr uint32_t P_BAR = 105088;     // tma full, mma0 done, W/U done, slot free, TMEM slot
// Stages of the slot parts (the slot's own layouts), bulk-copied to the ring:
constexpr uint32_t P_SK = P_TBH;       // dec K^ (P2; the splits come later)
constexpr uint32_t P_SQ = P_T;         // gamma Q^ (P2; T is built later)
constexpr uint32_t P_SP = P_KQ + 8192; // P (P3; raw Q rows of panel 0, dead after [K; Q] K^T)
constexpr uint32_t P_SW = P_TBH;       // -W (P6; the W / U products are done)
constexpr uint32_t P_SU = P_A;         // U^T (P6)
constexpr uint32_t kSubStride = 105472;
constexpr uint32_t kPrepSmem = kSubs * kSubStride;

constexpr uint32_t kSmem = (kChainSmem > kPrepSmem ? kChainSmem : kPrepSmem) + 1024;

// instruction descriptors
constexpr uint32_t ID_KQ = idesc_f16(128, 64, false, false, false, false);   // [K;Q] K^T, bf16
constexpr uint32_t ID_W = idesc_f16(64, 128, false, true, false, false);     // W, bf16
constexpr uint32_t ID_U = idesc_f16(128, 64, true, false, false, false);     // U^T, bf16
constexpr uint32_t ID_S = idesc_f16(128, 128, false, true, false, true);     // S^T increment
constexpr uint32_t ID_Y = idesc_f16(128, 64, false, false, false, true);     // Y^T += Delta^T P^T

struct ScanParams {
  PrefillArgs a;
  CUtensorMap tq, tk, tv;  // [total_T, H, 128] bf16, boxes of 64 x 1 x 64
  CUtensorMap tg;          // g, the same shape as v (set when g is given)
  int items;
  int has_tiles;           // total_T > 0 (otherwise the maps are unset and unused)
};

__device__ __forceinline__ int fidx(int r, int c) { return r * 64 + (c ^ ((r & 7) << 2)); }

// Two mbarrier parities packed in one register (bit b: buffer b), so that
// a buffer index known only at run time does not put them in local memory.
__device__ __forceinline__ uint32_t par(uint32_t bits, int b) { return (bits >> b) & 1u; }

__device__ __forceinline__ float a_norm_w_or_zero(const PrefillArgs& a, int j) {
  return (a.g != nullptr && a.norm_w != nullptr) ? a.norm_w[j] : 0.f;
}

__device__ __forceinline__ int scale_exp(float x, int target) {
  if (!(x > 0.f) || !(x < 3.0e38f)) return 0;
  int ex;
  frexpf(x, &ex);
  return ex - target;
}

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack_b2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 h2f(uint32_t w) {
  __half2 h;
  memcpy(&h, &w, 4);
  return __half22float2(h);
}

// bf16 hi + lo parts of a pair: hi = bf16(x), lo = bf16(x - hi)
__device__ __forceinline__ void split_b2(float x0, float x1, uint32_t* hi, uint32_t* lo) {
  const uint32_t h = pack_b2(x0, x1);
  *hi = h;
  *lo = pack_b2(x0 - bf_lo(h), x1 - bf_hi(h));
}

// One recursive-doubling level of the unit-lower-triangular inverse over the
// kSubT threads of a sub-pipeline (barrier `bid`): for every pair of BS x BS
// diagonal blocks [[T1, 0], [A21, T2]] of I + A, X = -T2 (A21 T1).
template <int BS>
__device__ __forceinline__ void tinv_level(const float* sA, float* sT, float* sZ, int tid,
                                           uint32_t bid) {
  constexpr int NP = 64 / (2 * BS);
  constexpr int EPT = NP * BS * BS / kSubT;
  constexpr int RC = EPT >= 2 ? 2 : 1;
  constexpr int RR = EPT / RC;
  constexpr int CB = BS / RC;
  constexpr int TPP = (BS / RR) * CB;
  const int p = tid / TPP, q = tid % TPP;
  const int r0 = (q / CB) * RR, c0 = (q % CB) * RC;
  const int top = 2 * BS * p, bot = top + BS;
  float acc[RR][RC];
#pragma unroll
  for (int i = 0; i < RR; ++i)
#pragma unroll
    for (int j = 0; j < RC; ++j) acc[i][j] = 0.f;
  // Z = A21 T1 (T1 lower triangular: rows m >= c0 only)
#pragma unroll 2
  for (int m = 0; m < BS; m += 4) {
    float4 ar[RR];
#pragma unroll
    for (int i = 0; i < RR; ++i)
      ar[i] = *reinterpret_cast<const float4*>(sA + fidx(bot + r0 + i, top + m));
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
  named_sync(bid, kSubT);
  // X = -T2 Z
#pragma unroll
  for (int i = 0; i < RR; ++i)
#pragma unroll
    for (int j = 0; j < RC; ++j) acc[i][j] = 0.f;
#pragma unroll 2
  for (int m = 0; m < BS; m += 4) {
    float4 tr[RR];
#pragma unroll
    for (int i = 0; i < RR; ++i)
      tr[i] = *reinterpret_cast<const float4*>(sT + fidx(bot + r0 + i, bot + m));
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
      *reinterpret_cast<float2*>(sT + fidx(bot + r0 + i, top + c0)) =
          make_float2(acc[i][0], acc[i][RC - 1]);
    } else {
      sT[fidx(bot + r0 + i, top + c0)] = acc[i][0];
    }
  }
  named_sync(bid, kSubT);
}

// ============================================================================
// Preparation sub-pipeline: chunks lane_id, lane_id + kLanes, ... of one item.
// Four compute warps (threads `st` 0-127, named barrier bA) and one control
// thread that waits for the output slot, issues the TMA loads and the MMAs,
// and publishes the slot; they hand off through mbarriers, all of whose
// waits are bounded.
// ============================================================================
struct PrepBars {
  uint64_t* tma;     // q, k, v tiles landed
  uint64_t* mma0;    // [K; Q] K^T done
  uint64_t* wu;      // W and U^T done
  uint64_t* slot;    // the output slot may be written (arrived by the control thread)
  uint64_t* splits;  // the T diag(.) splits are in shared memory (the compute threads)
  uint64_t* stored;  // the slot is stored (the compute threads)
};

__device__ void prep_compute(const ScanParams& P, uint8_t* gb, uint32_t sb, uint32_t tb,
                             int item, int lane_id, int st, uint32_t bA, const PrepBars& B) {
  const PrefillArgs& a = P.a;
  const int seq = item / a.H_v, h = item % a.H_v;
  const int warp = st >> 5, lane = st & 31;
  int64_t t_begin, t_end;
  if (!seq_bounds(a.cu_seqlens, seq, a.total_T, &t_begin, &t_end, nullptr)) return;
  const int nch = (int)((t_end - t_begin + kC - 1) / kC);

  float* sA = reinterpret_cast<float*>(gb + P_A);
  float* sT = reinterpret_cast<float*>(gb + P_T);
  float* sZ = reinterpret_cast<float*>(gb + P_Z);
  const float* sGB = reinterpret_cast<const float*>(gb + P_GB);
  float* sG2 = reinterpret_cast<float*>(gb + P_G);
  float* sBeta = sG2 + 64;
  float* sGam = sG2 + 128;
  float* sDec = sG2 + 192;
  float* sRk = sG2 + 256;
  float* sRq = sG2 + 320;
  float* sMax = reinterpret_cast<float*>(gb + P_MAX);
  uint8_t* ring = static_cast<uint8_t*>(a.ring) + (size_t)item * kRingS * kScanSlotBytes;
  const bool l2n = a.l2norm != 0;
  const uint32_t lane_off = (uint32_t)(32 * warp) << 16;

  auto load_gates = [&](int c) {
    const int64_t c0 = t_begin + (int64_t)c * kC;
    const int n = (int)(t_end - c0 < kC ? t_end - c0 : kC);
    const int which = st >> 6, t = st & 63;
    const bool ok = t < n;
    const float* src = (which ? a.beta : a.log_alpha) + (ok ? (size_t)(c0 + t) * a.H_v + h : 0);
    cp_async4(sb + P_GB + which * 256 + t * 4, src, ok);
    cp_async_commit();
  };
  if (lane_id < nch) load_gates(lane_id);

  uint32_t ph_tma = 0, ph_mma0 = 0, ph_wu = 0, ph_slot = 0;
  bool ok = true;
  for (int c = lane_id; c < nch; c += kLanes) {
    const int64_t c0 = t_begin + (int64_t)c * kC;
    const int n = (int)(t_end - c0 < kC ? t_end - c0 : kC);
    uint8_t* slot = ring + (size_t)(c % kRingS) * kScanSlotBytes;

    GDN_SCAN_TRACE(1, 18);
    // ---- P1: gates (warp 1): G2 = cumsum(log alpha) log2 e; gamma = 2^G2;
    // dec = 2^(G2_C - G2) ------------------------------------------------------
    cp_async_wait_all();
    named_sync(bA, kSubT);
    if (warp == 1) {
      float carry = 0.f;
      float Gv[2], bv[2];
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        const int t = hb * 32 + lane;
        float x = sGB[t] * kLog2e;
        bv[hb] = sGB[64 + t];
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
      if (lane == 0) sMax[8] = ex2_approx(carry);  // gamma_C
    }
    // the tiles have landed (TMA) and the slot is free (control thread)
    bool okw = mbar_wait(B.tma, ph_tma, kWait);
    ph_tma ^= 1;
    okw = mbar_wait(B.slot, ph_slot, kWait) && okw;
    ph_slot ^= 1;
    if (!named_sync_and(bA, kSubT, okw)) { ok = false; break; }
    if (c + kLanes < nch) load_gates(c + kLanes);
    GDN_SCAN_TRACE(1, 10);

    // ---- P2: norms; dec K^ and gamma Q^ into the slot; max|V| ---------------
    {
      const int r = st;   // row of [K; Q]
      const int t = r & 63;
      const bool is_k = r < 64;
      float ss = 0.f;
#pragma unroll 4
      for (int ch = 0; ch < 16; ++ch) {
        const uint4 u = ld_shared_v4(sb + P_KQ + sw128_chunk(r, ch, 128));
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) ss += bf_lo(w4[e]) * bf_lo(w4[e]) + bf_hi(w4[e]) * bf_hi(w4[e]);
      }
      GDN_SCAN_TRACE(1, 21);
      const bool valid = t < n;
      const float rn = valid ? (l2n ? rsqrtf(ss + a.eps_l2) : 1.f) : 0.f;
      (is_k ? sRk : sRq)[t] = rn;
      const float f = rn * (is_k ? sDec[t] : sGam[t]);
      // dec K^ rows into the K stage, gamma Q^ rows into the Q stage (the
      // slot's layouts; bulk-copied out below)
      const uint32_t stage = sb + (is_k ? P_SK : P_SQ) + t * 128;
      // a panel's loads are all issued before its stores (the shared-memory
      // accesses keep their program order)
#pragma unroll 1
      for (int pn = 0; pn < 2; ++pn) {
        uint4 u[8];
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) u[c8] = ld_shared_v4(sb + P_KQ + sw128_chunk(r, 8 * pn + c8, 128));
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8)
          st_shared_v4(stage + pn * 8192 + ((c8 ^ (t & 7)) << 4),
                       pack_h2(bf_lo(u[c8].x) * f, bf_hi(u[c8].x) * f),
                       pack_h2(bf_lo(u[c8].y) * f, bf_hi(u[c8].y) * f),
                       pack_h2(bf_lo(u[c8].z) * f, bf_hi(u[c8].z) * f),
                       pack_h2(bf_lo(u[c8].w) * f, bf_hi(u[c8].w) * f));
      }
      GDN_SCAN_TRACE(1, 22);
      // max |V| over the valid rows: 8 pieces of 8 per thread
      float vm = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int idx = st + kSubT * k, vr = idx >> 4, vc = idx & 15;
        if (vr < n) {
          const uint4 u = ld_shared_v4(sb + P_V + sw128_chunk(vr, vc, 64));
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) vm = fmaxf(vm, fmaxf(fabsf(bf_lo(w4[e])), fabsf(bf_hi(w4[e]))));
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, o));
      if (lane == 0) sMax[warp] = vm;
    }
    fence_proxy_async();  // the staged rows before the bulk copies
    named_sync(bA, kSubT);
    if (st == 0) {
      fence_proxy_async_global();
      bulk_store_s2g(slot + SL_K, sb + P_SK, 16384);
      bulk_store_s2g(slot + SL_WQ + 8192, sb + P_SQ, 8192);
      bulk_store_s2g(slot + SL_WQ + 16384 + 8192, sb + P_SQ + 8192, 8192);
      bulk_commit();
    }
    GDN_SCAN_TRACE(1, 11);

    // ---- P3: A (fp32, shared) and P (fp16, slot) from the products ----------
    okw = mbar_wait(B.mma0, ph_mma0, kWait);
    ph_mma0 ^= 1;
    fence_after_sync();
    GDN_SCAN_TRACE(1, 31);
    {
      // lanes 0-63: K rows, A_ti = beta_t rk_t rk_i 2^(G2_t - G2_i) (k.k)_ti, i < t;
      // lanes 64-127: Q rows, P_ti = rq_t rk_i 2^(G2_t - G2_i) (q.k)_ti, i <= t
      const int row = 32 * warp + lane;
      const int t = row & 63;
      const bool is_a = row < 64;
      const float Gt = sG2[t];
      const float sc = is_a ? sBeta[t] * sRk[t] : sRq[t];
      const int lim = is_a ? t : t + 1;  // columns i < lim are kept
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {
        const int i0 = 32 * hh;
        float v[32];
        tmem_ld32(tb + lane_off + i0, v);
        // the half's column factors rk_i and G2_i
        float rkv[32], gv[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 r4 = *reinterpret_cast<const float4*>(sRk + i0 + 4 * q);
          const float4 g4 = *reinterpret_cast<const float4*>(sG2 + i0 + 4 * q);
          rkv[4 * q] = r4.x; rkv[4 * q + 1] = r4.y; rkv[4 * q + 2] = r4.z; rkv[4 * q + 3] = r4.w;
          gv[4 * q] = g4.x; gv[4 * q + 1] = g4.y; gv[4 * q + 2] = g4.z; gv[4 * q + 3] = g4.w;
        }
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          // masked entries take 2^-inf = 0 (no branch around the exponential)
          const float d = i0 + x < lim ? Gt - gv[x] : -INFINITY;
          v[x] = sc * rkv[x] * ex2_approx(d) * v[x];
        }
        if (is_a) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(sA + fidx(t, i0 + i)) =
                make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        } else {
          // P row t into its stage (the slot's layout)
          uint8_t* dst = gb + P_SP + t * 128;
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8)
            *reinterpret_cast<uint4*>(dst + (((4 * hh + c8) ^ (t & 7)) << 4)) =
                make_uint4(pack_h2(v[8 * c8], v[8 * c8 + 1]), pack_h2(v[8 * c8 + 2], v[8 * c8 + 3]),
                           pack_h2(v[8 * c8 + 4], v[8 * c8 + 5]),
                           pack_h2(v[8 * c8 + 6], v[8 * c8 + 7]));
        }
      }
    }
    fence_proxy_async();
    fence_before_sync();
    GDN_SCAN_TRACE(1, 32);
    // the K and Q stages are read out before T and the splits reuse them
    if (st == 0) bulk_wait_read_all();
    GDN_SCAN_TRACE(1, 33);
    if (!named_sync_and(bA, kSubT, okw)) { ok = false; break; }
    if (st == 0) {
      bulk_store_s2g(slot + SL_P, sb + P_SP, 8192);
      bulk_commit();
    }
    GDN_SCAN_TRACE(1, 12);

    // ---- P4: T = (I + A)^{-1}: 8 x 8 diagonal blocks by substitution, then
    // doubling 8 -> 16 -> 32 -> 64 -----------------------------------------------
    if (st < 64) {
      const int bq = st >> 3, cc = st & 7;
      float ab[8][8];
#pragma unroll
      for (int r = 1; r < 8; ++r) {
        const float4 lo = *reinterpret_cast<const float4*>(sA + fidx(8 * bq + r, 8 * bq));
        const float4 hi = *reinterpret_cast<const float4*>(sA + fidx(8 * bq + r, 8 * bq + 4));
        ab[r][0] = lo.x; ab[r][1] = lo.y; ab[r][2] = lo.z; ab[r][3] = lo.w;
        ab[r][4] = hi.x; ab[r][5] = hi.y; ab[r][6] = hi.z; ab[r][7] = hi.w;
      }
      float xs[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        float s = (r == cc) ? 1.f : 0.f;
#pragma unroll
        for (int m = 0; m < r; ++m) s -= ab[r][m] * xs[m];
        xs[r] = s;
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) sT[fidx(8 * bq + r, 8 * bq + cc)] = xs[r];
    } else {
      // T above the 8 x 8 block diagonal is zero (the doubling reads it):
      // row r, columns from 8 (r / 8 + 1), 4 at a time
      const int r = st - 64;
      for (int c4 = 8 * ((r >> 3) + 1); c4 < 64; c4 += 4)
        *reinterpret_cast<float4*>(sT + fidx(r, c4)) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    named_sync(bA, kSubT);
    GDN_SCAN_TRACE(1, 23);
    tinv_level<8>(sA, sT, sZ, st, bA);
    GDN_SCAN_TRACE(1, 24);
    tinv_level<16>(sA, sT, sZ, st, bA);
    GDN_SCAN_TRACE(1, 25);
    tinv_level<32>(sA, sT, sZ, st, bA);
    GDN_SCAN_TRACE(1, 13);

    // ---- P5: bf16 hi / lo parts of T diag(beta gamma rk) (W) and T diag(beta)
    // (U^T); the A scratch is dead ---------------------------------------------------
    {
      const int t = st >> 1, q4 = (st & 1) * 32;
#pragma unroll 1
      for (int hp = 0; hp < 4; hp += 2) {
        // T row t and the column factors of blocks hp, hp + 1 (loads first)
        float tv[16], bv[16], gr[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = q4 + 8 * hp + 4 * q;
          const float4 x = *reinterpret_cast<const float4*>(sT + fidx(t, col));
          const float4 bb = *reinterpret_cast<const float4*>(sBeta + col);
          const float4 gg = *reinterpret_cast<const float4*>(sGam + col);
          const float4 rr = *reinterpret_cast<const float4*>(sRk + col);
          tv[4 * q] = x.x; tv[4 * q + 1] = x.y; tv[4 * q + 2] = x.z; tv[4 * q + 3] = x.w;
          bv[4 * q] = bb.x; bv[4 * q + 1] = bb.y; bv[4 * q + 2] = bb.z; bv[4 * q + 3] = bb.w;
          gr[4 * q] = gg.x * rr.x; gr[4 * q + 1] = gg.y * rr.y;
          gr[4 * q + 2] = gg.z * rr.z; gr[4 * q + 3] = gg.w * rr.w;
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t wh[4], wl[4], uh[4], ul[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int x = 8 * hh + 2 * u;
            const float b0 = bv[x] * tv[x], b1 = bv[x + 1] * tv[x + 1];
            split_b2(b0, b1, &uh[u], &ul[u]);
            split_b2(b0 * gr[x], b1 * gr[x + 1], &wh[u], &wl[u]);
          }
          const uint32_t off = sw128_chunk(t, q4 / 8 + hp + hh, 64);
          st_shared_v4(sb + P_TWH + off, wh[0], wh[1], wh[2], wh[3]);
          st_shared_v4(sb + P_TWL + off, wl[0], wl[1], wl[2], wl[3]);
          st_shared_v4(sb + P_TBH + off, uh[0], uh[1], uh[2], uh[3]);
          st_shared_v4(sb + P_TBL + off, ul[0], ul[1], ul[2], ul[3]);
        }
      }
    }
    fence_proxy_async();
    fence_before_sync();
    // the P stage is read out before the control thread loads the next tiles
    // over it (after the W / U products)
    if (st == 0) bulk_wait_read_all();
    mbar_arrive(B.splits);  // the control thread issues W and U^T
    GDN_SCAN_TRACE(1, 14);

    GDN_SCAN_TRACE(1, 15);

    // ---- P6: -W and U^T 2^-e_u into the slot ----------------------------------------
    okw = mbar_wait(B.wu, ph_wu, kWait);
    ph_wu ^= 1;
    fence_after_sync();
    GDN_SCAN_TRACE(1, 16);
    {
      float v[32];
      // W: M = 64 accumulator, row t in lane (t % 16) + 32 (t / 16)
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        tmem_ld32(tb + lane_off + 64 + 32 * q, v);
        tmem_wait_ld();
        if (lane < 16) {
          const int t = 16 * warp + lane;
          const uint32_t dst = sb + P_SW + (q >> 1) * 8192 + t * 128;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const int ch = 4 * (q & 1) + c4;
            st_shared_v4(dst + ((ch ^ (t & 7)) << 4), pack_h2(-v[8 * c4], -v[8 * c4 + 1]),
                         pack_h2(-v[8 * c4 + 2], -v[8 * c4 + 3]),
                         pack_h2(-v[8 * c4 + 4], -v[8 * c4 + 5]),
                         pack_h2(-v[8 * c4 + 6], -v[8 * c4 + 7]));
          }
        }
      }
      GDN_SCAN_TRACE(1, 27);
      // U^T: row j = d_v index (this thread's TMEM lane), 64 token columns
      float u[64];
      tmem_ld32(tb + lane_off + 192, u);
      tmem_ld32(tb + lane_off + 224, u + 32);
      tmem_wait_ld();
      float um = 0.f;
#pragma unroll
      for (int x = 0; x < 64; ++x) um = fmaxf(um, fabsf(u[x]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) um = fmaxf(um, __shfl_xor_sync(0xffffffffu, um, o));
      if (lane == 0) sMax[4 + warp] = um;
      fence_proxy_async();
      fence_before_sync();
      named_sync(bA, kSubT);
      if (st == 0) {
        bulk_store_s2g(slot + SL_WQ, sb + P_SW, 8192);
        bulk_store_s2g(slot + SL_WQ + 16384, sb + P_SW + 8192, 8192);
        bulk_commit();
      }
      const float mu = fmaxf(fmaxf(sMax[4], sMax[5]), fmaxf(sMax[6], sMax[7]));
      const int eu = scale_exp(mu, 14);
      const float su = ldexpf(1.f, -eu);
      const int j = 32 * warp + lane;
      const uint32_t dst = sb + P_SU + j * 128;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch)
        st_shared_v4(dst + ((ch ^ (j & 7)) << 4), pack_h2(u[8 * ch] * su, u[8 * ch + 1] * su),
                     pack_h2(u[8 * ch + 2] * su, u[8 * ch + 3] * su),
                     pack_h2(u[8 * ch + 4] * su, u[8 * ch + 5] * su),
                     pack_h2(u[8 * ch + 6] * su, u[8 * ch + 7] * su));
      fence_proxy_async();
      named_sync(bA, kSubT);
      if (st == 0) {
        const float mv = fmaxf(fmaxf(sMax[0], sMax[1]), fmaxf(sMax[2], sMax[3]));
        *reinterpret_cast<float4*>(slot + SL_SCAL) = make_float4(sMax[8], (float)eu, mv, (float)n);
        bulk_store_s2g(slot + SL_U, sb + P_SU, 16384);
        bulk_commit();
        GDN_SCAN_TRACE(1, 34);
        // every copy of the chunk has landed before the slot is published
        bulk_wait_all();
        GDN_SCAN_TRACE(1, 35);
        fence_proxy_async_global();
      }
    }
    // ---- P7: the slot is stored: the control thread publishes it --------------
    fence_before_sync();
    mbar_arrive(B.stored);
    if (!okw) { ok = false; break; }
    GDN_SCAN_TRACE(1, 17);
  }
  cp_async_wait_all();
  if (st == 0) bulk_wait_all();  // no copy still reads shared memory at exit
  GDN_SCAN_TRACE(1, 19);
  if (!ok && st == 0) atomicOr(a.err, kErrTimeout);
}

// The control thread of a preparation sub-pipeline.
__device__ void prep_control(const ScanParams& P, uint32_t sb, uint32_t tb, int item, int lane_id,
                             const PrepBars& B) {
  const PrefillArgs& a = P.a;
  const int seq = item / a.H_v, h = item % a.H_v, hq = h / (a.H_v / a.H_qk);
  int64_t t_begin, t_end;
  if (!seq_bounds(a.cu_seqlens, seq, a.total_T, &t_begin, &t_end, nullptr)) return;
  const int nch = (int)((t_end - t_begin + kC - 1) / kC);
  unsigned long long* ready = a.ring_flags + (size_t)item * 2 * kRingS;
  unsigned long long* consumed = ready + kRingS;
  // chunk c's q / k / v tiles into L2 ahead of their loads (the loads land
  // only a few thousand cycles before the compute threads need them)
  auto prefetch_tiles = [&](int c) {
    const int z = (int)(t_begin + (int64_t)c * kC);
#pragma unroll 1
    for (int pp = 0; pp < 2; ++pp) {
      tma_prefetch_3d(&P.tk, 64 * pp, hq, z);
      tma_prefetch_3d(&P.tq, 64 * pp, hq, z);
      tma_prefetch_3d(&P.tv, 64 * pp, h, z);
    }
  };
  auto load_tiles = [&](int c) {
    const int z = (int)(t_begin + (int64_t)c * kC);
    mbar_arrive_expect_tx(B.tma, 49152);
#pragma unroll 1
    for (int pp = 0; pp < 2; ++pp) {
      tma_load_3d(sb + P_KQ + pp * 16384, &P.tk, 64 * pp, hq, z, B.tma);
      tma_load_3d(sb + P_KQ + pp * 16384 + 8192, &P.tq, 64 * pp, hq, z, B.tma);
      tma_load_3d(sb + P_V + pp * 8192, &P.tv, 64 * pp, h, z, B.tma);
    }
  };
  uint32_t ph_tma = 0, ph_wu = 0, ph_sp = 0, ph_st = 0;
  bool ok = true;
  // The compute threads may start chunk c once its output slot (which held
  // chunk c - ring: the chain side must be done with it) is free.  The next
  // chunk's slot is handed over before this chunk is published, so that they
  // do not wait for the publication.
  auto open_slot = [&](int c) -> bool {
    if (c >= kRingS &&
        !wait_flag_ge(&consumed[c % kRingS], (unsigned long long)(c - kRingS) + 1, kWait))
      return false;
    mbar_arrive(B.slot);
    return true;
  };
  if (lane_id < nch) {
    load_tiles(lane_id);
    ok = open_slot(lane_id);
  }
  for (int c = lane_id; ok && c < nch; c += kLanes) {
    // [K; Q] K^T once the tiles have landed
    ok = mbar_wait(B.tma, ph_tma, kWait);
    ph_tma ^= 1;
    if (!ok) break;
#pragma unroll 1
    for (int kk = 0; kk < 8; ++kk) {
      const uint64_t d = sdesc(sb + P_KQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
      mma_f16(tb, d, d, ID_KQ, kk > 0);
    }
    mma_commit(B.mma0);
    // the next chunk's tiles into L2 while this one is prepared
    if (c + kLanes < nch) prefetch_tiles(c + kLanes);
    // W = T diag(beta gamma rk) K_raw (M = 64, N = 128) and U^T = V^T (T
    // diag(beta))^T (M = 128, N = 64), hi then lo parts, once the splits are in
    ok = mbar_wait(B.splits, ph_sp, kWait);
    ph_sp ^= 1;
    if (!ok) break;
    fence_after_sync();
#pragma unroll 1
    for (int part = 0; part < 2; ++part) {
      const uint32_t aw = sb + (part ? P_TWL : P_TWH);
      const uint32_t bu = sb + (part ? P_TBL : P_TBH);
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk) {
        mma_f16(tb + 64, sdesc(aw + kk * 32, 16, 1024), sdesc(sb + P_KQ + kk * 2048, 16384, 1024),
                ID_W, part | (kk > 0));
        mma_f16(tb + 192, sdesc(sb + P_V + kk * 2048, 8192, 1024), sdesc(bu + kk * 32, 16, 1024),
                ID_U, part | (kk > 0));
      }
    }
    mma_commit(B.wu);
    // the raw tiles are free once the products are done: the next chunk's
    ok = mbar_wait(B.wu, ph_wu, kWait);
    ph_wu ^= 1;
    if (!ok) break;
    if (c + kLanes < nch) {
      fence_proxy_async();  // the generic reads of the raw tiles precede the TMA writes
      load_tiles(c + kLanes);
      ok = open_slot(c + kLanes);
      if (!ok) break;
    }
    // the compute threads have stored the slot: publish it
    ok = mbar_wait(B.stored, ph_st, kWait);
    ph_st ^= 1;
    if (!ok) break;
    __threadfence();
    st_release_u64(&ready[c % kRingS], (unsigned long long)c + 1);
  }
  if (!ok) atomicOr(a.err, kErrTimeout);
}

// ============================================================================
// Chain CTA.  Compute warps 0-7: thread (warp w, lane l) owns d_v index
// j = 32 (w % 4) + l (its TMEM lane) and the state entries S[i][j],
// i in [64 cg, 64 cg + 64), cg = w / 4, in registers.  MMA warp 8 (lane 0)
// issues the products; loader warp 11 (lane 0) loads the slots and the raw g.
// Epilogue warps 9-10 apply RMSNorm x gate to staged Y rows and store y.
// TMEM columns: S^T 2^-e A operand 0-63 (two fp16 K elements per column),
// Delta^T 2^-e A operand 64-95, S^T increment 128-255, and two
// [Delta^T | Y^T] accumulators 256-383 / 384-511 (chunk c in c & 1).
// Named barriers: 1 compute warps, 4 epilogue warps, 5 teardown; the roles
// hand off through mbarriers, all of whose waits are bounded.
// ============================================================================
struct ChainBars {
  uint64_t* fullA;    // [2] [-W; gamma Q^] of the slot in buffer c % 2 landed
  uint64_t* bar1;     // [Delta^T | Y^T] = S^T [-W; gamma Q^]^T done
  uint64_t* bar3;     // S^T increment done
  uint64_t* barY;     // [2] Y^T of chunk c complete (accumulator c % 2)
  uint64_t* ysfull;   // [2] Y stage written (compute warps)
  uint64_t* ysempty;  // [2] Y stage read (epilogue warps)
  uint64_t* sready;   // S^T operand of the next chunk in TMEM (compute warps)
  uint64_t* dready;   // Delta^T operand in TMEM (compute warps)
  uint64_t* gfull;    // [2] raw g of the chunk in stage c % 2 landed (TMA)
  uint64_t* fullB;    // [2] the scalars and U^T landed
  uint64_t* fullC;    // [2] dec K^ and P landed
  uint64_t* bar1b;    // [2] both S^T [-W; gamma Q^]^T products done ([-W; gamma Q^] free)
  uint64_t* ufree;    // [2] the scalars and U^T read (arrived by the MMA thread after dready)
};

__device__ void chain_compute(const ScanParams& P, uint8_t* gb, uint32_t sb, uint32_t tbase,
                              int item, const ChainBars& B) {
  const PrefillArgs& a = P.a;
  const int seq = item / a.H_v, h = item % a.H_v;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, cg = warp >> 2;
  const int j = 32 * qd + lane;
  const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
  int64_t t_begin, t_end;
  const bool bounds_ok =
      seq_bounds(a.cu_seqlens, seq, a.total_T, &t_begin, &t_end, tid == 0 ? a.err : nullptr);
  const int nch = bounds_ok ? (int)((t_end - t_begin + kC - 1) / kC) : 0;
  float* sMaxw = reinterpret_cast<float*>(gb + C_MISC);
  int* sYExp = reinterpret_cast<int*>(gb + C_MISC + 64);  // exponent of each Y stage
  const size_t st_off = ((size_t)seq * a.H_v + h) * (size_t)(kD * kD);
  const uint32_t tSA = tbase + lane_off + 32 * cg;
  const uint32_t tDA = tbase + lane_off + 64 + 16 * cg;
  const uint32_t tDS = tbase + lane_off + 128 + 64 * cg;
  auto tD1 = [&](int b) -> uint32_t { return tbase + lane_off + 256 + 128 * b; };

  // the initial state (zero without one); plain loads under a branch, so that
  // no load from a null initial state can be speculated
  float S[64];
  if (a.initial_state != nullptr) {
    const float* s0 = a.initial_state + st_off + (size_t)(64 * cg) * kD + j;
#pragma unroll
    for (int x = 0; x < 64; ++x) S[x] = s0[(size_t)x * kD];
  } else {
#pragma unroll
    for (int x = 0; x < 64; ++x) S[x] = 0.f;
  }

  uint32_t ph_full = 0, ph1 = 0, ph3 = 0, phY = 0, phE = 0;  // parity bits per buffer
  bool ok = true;
  int e_cur = 0, e_prev = 0;

  // S^T 2^-e of chunk c into TMEM (slot c landed, e from max|V_c| and
  // max|S|), then "S^T ready".  Returns e, or INT32_MIN when a wait ran out.
  auto state_operand = [&](int c, float smax, bool okin) -> int {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, o));
    // per-warp maxima in the half of the scratch for chunk parity c % 2 (a warp
    // still reading chunk c - 1's maxima is not overwritten)
    float* mx = sMaxw + 8 * (c & 1);
    if (lane == 0) mx[warp] = smax;
    // the slot's scalars (and U^T) have landed
    bool okw = mbar_wait(&B.fullB[c & 1], par(ph_full, c & 1), kWait) && okin;
    ph_full ^= 1u << (c & 1);
    if (!named_sync_and(1, kChainT, okw)) return INT32_MIN;
    float mS = mx[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) mS = fmaxf(mS, mx[w]);
    const float mV = reinterpret_cast<const float*>(gb + (c & 1) * kSlotStride + SL_SCAL)[2];
    const int e = scale_exp(mV + 12.f * mS, 12);
    const float se = ldexpf(1.f, -e);
    uint32_t pk[32];
#pragma unroll
    for (int m2 = 0; m2 < 32; ++m2) pk[m2] = pack_h2(S[2 * m2] * se, S[2 * m2 + 1] * se);
    tmem_st32(tSA, reinterpret_cast<const float*>(pk));
    tmem_wait_st();
    fence_before_sync();
    mbar_arrive(B.sready);
    return e;
  };
  // Y^T 2^-e of chunk pc (exponent pe) from its accumulator into stage pc % 2,
  // token-major
  auto export_y = [&](int pc, int pe) -> bool {
    const int b = pc & 1;
    bool okw = mbar_wait(&B.barY[b], par(phY, b), kWait);
    phY ^= 1u << b;
    if (pc >= 2) {
      okw = mbar_wait(&B.ysempty[b], par(phE, b), kWait) && okw;
      phE ^= 1u << b;
    }
    fence_after_sync();
    float v[32];
    tmem_ld32(tD1(b) + 64 + 32 * cg, v);
    tmem_wait_ld();
    uint8_t* ys = gb + C_YS + b * 16384;
#pragma unroll
    for (int x = 0; x < 32; ++x) {
      const int t = 32 * cg + x;
      *reinterpret_cast<__half*>(ys + t * 256 + ((((j >> 3) ^ (t & 15))) << 4) + (j & 7) * 2) =
          __float2half_rn(v[x]);
    }
    if (tid == 0) sYExp[b] = pe;
    mbar_arrive(&B.ysfull[b]);
    return okw;
  };

  float smax = 0.f, gC = 1.f;
#pragma unroll
  for (int x = 0; x < 64; ++x) smax = fmaxf(smax, fabsf(S[x]));
  bool okw = true;
  // Iteration c: the state operand and Delta of chunk c, the Y stage of chunk
  // c - 1 (while chunk c's state products run), the state update of chunk c;
  // iteration nch only stages the last Y.
  for (int c = 0; c <= nch && nch > 0; ++c) {
    const bool live = c < nch;
    const int b = c & 1;
    if (live) {
      e_cur = state_operand(c, smax, okw);
      if (e_cur == INT32_MIN) { ok = false; break; }
      // slot c's scalars: read before its products complete (buffer b then takes
      // chunk c + 2)
      const float* scal = reinterpret_cast<const float*>(gb + b * kSlotStride + SL_SCAL);
      gC = scal[0];
      const int eu = (int)scal[1];
      GDN_SCAN_TRACE(0, 0);

      // ---- Delta^T 2^-e = acc + U^T 2^(e_u - e) -> fp16 A operand ------------------
      okw = mbar_wait(B.bar1, ph1, kWait);
      ph1 ^= 1;
      fence_after_sync();
      GDN_SCAN_TRACE(0, 2);
      {
        float v[32];
        tmem_ld32(tD1(b) + 32 * cg, v);
        uint4 uq[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          uq[q] = ld_shared_v4(sb + b * kSlotStride + SL_U + j * 128 + (((4 * cg + q) ^ (j & 7)) << 4));
        tmem_wait_ld();
        const float su = ldexpf(1.f, eu - e_cur);
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t uw[4] = {uq[q].x, uq[q].y, uq[q].z, uq[q].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 uf = h2f(uw[e]);
            const int x = 8 * q + 2 * e;
            pk[4 * q + e] = pack_h2(v[x] + uf.x * su, v[x + 1] + uf.y * su);
          }
        }
        tmem_st16(tDA, pk);
        tmem_wait_st();
      }
      fence_before_sync();
      mbar_arrive(B.dready);
      GDN_SCAN_TRACE(0, 3);
    }
    // the previous chunk's Y^T to the stage while the state products run
    if (c > 0) okw = export_y(c - 1, e_prev) && okw;
    GDN_SCAN_TRACE(0, 4);
    if (!live) break;

    // ---- S <- gamma_C S + 2^e increment --------------------------------------------
    okw = mbar_wait(B.bar3, ph3, kWait) && okw;
    ph3 ^= 1;
    fence_after_sync();
    GDN_SCAN_TRACE(0, 5);
    smax = 0.f;
    {
      float v[64];
      tmem_ld32(tDS, v);
      tmem_ld32(tDS + 32, v + 32);
      tmem_wait_ld();
      const float se = ldexpf(1.f, e_cur);
#pragma unroll
      for (int x = 0; x < 64; ++x) {
        S[x] = gC * S[x] + se * v[x];
        smax = fmaxf(smax, fabsf(S[x]));
      }
    }
    GDN_SCAN_TRACE(0, 6);
    e_prev = e_cur;
    GDN_SCAN_TRACE(0, 7);
  }
  ok = ok && okw;
  if (ok && a.final_state && bounds_ok) {
    float* fs = a.final_state + st_off + (size_t)(64 * cg) * kD + j;
#pragma unroll
    for (int x = 0; x < 64; ++x) fs[(size_t)x * kD] = S[x];
  }
  GDN_SCAN_TRACE(0, 8);
  if (!ok) {
    if (tid == 0) atomicOr(a.err, kErrTimeout);
    // products possibly in flight get a short bounded chance to finish
    mbar_wait(B.bar3, ph3, kDrain);
    mbar_wait(&B.barY[0], par(phY, 0), kDrain);
    mbar_wait(&B.barY[1], par(phY, 1), kDrain);
  }
}

// The chain CTA's MMA thread (control warp): per chunk, the products as soon
// as their operands are in tensor memory.
__device__ void chain_mma(const ScanParams& P, uint32_t sb, uint32_t tbase, int item,
                          const ChainBars& B) {
  const PrefillArgs& a = P.a;
  const int seq = item / a.H_v;
  int64_t t_begin, t_end;
  if (!seq_bounds(a.cu_seqlens, seq, a.total_T, &t_begin, &t_end, nullptr)) return;
  const int nch = (int)((t_end - t_begin + kC - 1) / kC);
  unsigned long long* consumed = a.ring_flags + (size_t)item * 2 * kRingS + kRingS;
  uint32_t ph_s = 0, ph_d = 0, phA = 0, phC = 0;  // phA, phC: parity bits per buffer
  bool ok = true;
  for (int c = 0; ok && c < nch; ++c) {
    const int b = c & 1;
    const uint32_t slot = sb + b * kSlotStride;
    // S^T of chunk c is in TMEM (the compute warps saw slot c's scalars land)
    // and [-W; gamma Q^] of chunk c has landed
    ok = mbar_wait(B.sready, ph_s, kWait);
    ph_s ^= 1;
    ok = ok && mbar_wait(&B.fullA[b], par(phA, b), kWait);
    phA ^= 1u << b;
    if (!ok) break;
    fence_after_sync();
    GDN_SCAN_TRACE(2, 50);
    // Delta^T part first (its own commit: the state step waits only for it),
    // then the gamma Q^ part of Y^T
#pragma unroll 1
    for (int kk = 0; kk < 8; ++kk)
      mma_f16_ta(tbase + 256 + 128 * b, tbase + 8 * kk,
                 sdesc(slot + SL_WQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024), ID_Y, kk > 0);
    mma_commit(B.bar1);
#pragma unroll 1
    for (int kk = 0; kk < 8; ++kk)
      mma_f16_ta(tbase + 256 + 128 * b + 64, tbase + 8 * kk,
                 sdesc(slot + SL_WQ + (kk >> 2) * 16384 + 8192 + (kk & 3) * 32, 16, 1024), ID_Y,
                 kk > 0);
    mma_commit(&B.bar1b[b]);  // buffer b's [-W; gamma Q^] may take chunk c + 2's
    GDN_SCAN_TRACE(2, 51);
    ok = mbar_wait(B.dready, ph_d, kWait);  // Delta^T of chunk c is in TMEM
    ph_d ^= 1;
    if (!ok) break;
    // the compute warps have read the scalars and U^T: buffer b may take
    // chunk c + 2's
    mbar_arrive(&B.ufree[b]);
    // dec K^ and P of chunk c have landed
    ok = mbar_wait(&B.fullC[b], par(phC, b), kWait);
    phC ^= 1u << b;
    if (!ok) break;
    fence_after_sync();
    GDN_SCAN_TRACE(2, 52);
#pragma unroll 1
    for (int kk = 0; kk < 4; ++kk)
      mma_f16_ta(tbase + 128, tbase + 64 + 8 * kk, sdesc(slot + SL_K + kk * 2048, 8192, 1024),
                 ID_S, kk > 0);
    mma_commit(B.bar3);
#pragma unroll 1
    for (int kk = 0; kk < 4; ++kk)
      mma_f16_ta(tbase + 256 + 128 * b + 64, tbase + 64 + 8 * kk,
                 sdesc(slot + SL_P + kk * 32, 16, 1024), ID_Y, 1);
    mma_commit(&B.barY[b]);
    // every part of slot c is in shared memory: its global image may be
    // reused (a release store waits for this thread's earlier stores, so it
    // comes after the products are issued)
    st_release_u64(&consumed[c % kRingS], (unsigned long long)c + 1);
    GDN_SCAN_TRACE(2, 53);
  }
  if (!ok) atomicOr(a.err, kErrTimeout);
}

// The chain CTA's loader thread: slot c into buffer c % 2 once it is published
// and chunk c - 2's products are done with that buffer, and chunk c's raw g
// into stage c % 2 once chunk c - 2's epilogue has read it.
__device__ void chain_loader(const ScanParams& P, uint32_t sb, int item, const ChainBars& B) {
  const PrefillArgs& a = P.a;
  const int seq = item / a.H_v, h = item % a.H_v;
  int64_t t_begin, t_end;
  if (!seq_bounds(a.cu_seqlens, seq, a.total_T, &t_begin, &t_end, nullptr)) return;
  const int nch = (int)((t_end - t_begin + kC - 1) / kC);
  const uint8_t* ring =
      static_cast<const uint8_t*>(a.ring) + (size_t)item * kRingS * kScanSlotBytes;
  unsigned long long* ready = a.ring_flags + (size_t)item * 2 * kRingS;
  // parity bits per buffer of the barriers that free each part of it
  uint32_t ph1b = 0, phU = 0, phY = 0, phE = 0;
  // chunks whose copies were issued, per part (for the drain)
  int nA = 0, nB = 0, nC = 0, ngs = 0;
  bool ok = true;
  // Chunk c into buffer c % 2 in three parts, each as soon as chunk c - 2 is
  // done with that part of the buffer: [-W; gamma Q^] after both products
  // that read it, the scalars and U^T after the Delta step, dec K^ and P
  // after the last products of chunk c - 2.
  for (int c = 0; ok && c < nch; ++c) {
    const int b = c & 1;
    const uint8_t* src = ring + (size_t)(c % kRingS) * kScanSlotBytes;
    const uint32_t dst = sb + b * kSlotStride;
    ok = wait_flag_ge(&ready[c % kRingS], (unsigned long long)c + 1, kWait);
    if (!ok) break;
    fence_proxy_async_global();
    if (c >= 2) {
      ok = mbar_wait(&B.bar1b[b], par(ph1b, b), kWait);
      ph1b ^= 1u << b;
      if (!ok) break;
    }
    mbar_arrive_expect_tx(&B.fullA[b], 32768);
    bulk_load_g2s(dst + SL_WQ, src + SL_WQ, 16384, &B.fullA[b]);
    bulk_load_g2s(dst + SL_WQ + 16384, src + SL_WQ + 16384, 16384, &B.fullA[b]);
    nA = c + 1;
    if (c >= 2) {
      ok = mbar_wait(&B.ufree[b], par(phU, b), kWait);
      phU ^= 1u << b;
      if (!ok) break;
    }
    fence_proxy_async();  // the compute warps' reads of the old scalars / U^T precede the copy
    mbar_arrive_expect_tx(&B.fullB[b], (SL_U - SL_SCAL) + 16384);
    bulk_load_g2s(dst + SL_SCAL, src + SL_SCAL, SL_U - SL_SCAL, &B.fullB[b]);
    bulk_load_g2s(dst + SL_U, src + SL_U, 16384, &B.fullB[b]);
    nB = c + 1;
    if (c >= 2) {
      ok = mbar_wait(&B.barY[b], par(phY, b), kWait);
      phY ^= 1u << b;
      if (!ok) break;
    }
    mbar_arrive_expect_tx(&B.fullC[b], SL_SCAL - SL_K);
    bulk_load_g2s(dst + SL_K, src + SL_K, SL_SCAL - SL_K, &B.fullC[b]);
    nC = c + 1;
    if (c >= 2) {
      ok = mbar_wait(&B.ysempty[b], par(phE, b), kWait);
      phE ^= 1u << b;
    }
    if (ok && a.g != nullptr) {
      const int z = (int)(t_begin + (int64_t)c * kC);
      fence_proxy_async();  // the epilogue's reads of the stage precede the TMA writes
      mbar_arrive_expect_tx(&B.gfull[b], 16384);
      tma_load_3d(sb + C_GS + 16384 * b, &P.tg, 0, h, z, &B.gfull[b]);
      tma_load_3d(sb + C_GS + 16384 * b + 8192, &P.tg, 64, h, z, &B.gfull[b]);
      ngs = c + 1;
    } else if (ok) {
      mbar_arrive(&B.gfull[b]);
    }
  }
  if (!ok) {
    atomicOr(a.err, kErrTimeout);
    // copies still landing get a short bounded chance before the CTA may exit:
    // the last chunk issued into each buffer completes that buffer's phase
    // (chunk index / 2) % 2
    for (int c = nA - 2 < 0 ? 0 : nA - 2; c < nA; ++c)
      mbar_wait(&B.fullA[c & 1], (uint32_t)(c >> 1) & 1u, kDrain);
    for (int c = nB - 2 < 0 ? 0 : nB - 2; c < nB; ++c)
      mbar_wait(&B.fullB[c & 1], (uint32_t)(c >> 1) & 1u, kDrain);
    for (int c = nC - 2 < 0 ? 0 : nC - 2; c < nC; ++c)
      mbar_wait(&B.fullC[c & 1], (uint32_t)(c >> 1) & 1u, kDrain);
    for (int c = ngs - 2 < 0 ? 0 : ngs - 2; c < ngs; ++c)
      mbar_wait(&B.gfull[c & 1], (uint32_t)(c >> 1) & 1u, kDrain);
  }
}

// The chain CTA's epilogue warps: token t = thread index; per chunk, the staged
// Y row and the raw g row (TMA), RMSNorm x (1 + w) sigmoid(g), bf16 out.
__device__ void chain_epilogue(const ScanParams& P, uint8_t* gb, int item, const ChainBars& B) {
  const PrefillArgs& a = P.a;
  const int seq = item / a.H_v, h = item % a.H_v;
  const int et = threadIdx.x - 32 * kEpiWarp;
  int64_t t_begin, t_end;
  if (!seq_bounds(a.cu_seqlens, seq, a.total_T, &t_begin, &t_end, nullptr)) return;
  const int nch = (int)((t_end - t_begin + kC - 1) / kC);
  const float* sWn = reinterpret_cast<const float*>(gb + C_WN);
  const int* sExp = reinterpret_cast<const int*>(gb + C_MISC + 64);
  const bool has_g = a.g != nullptr;
  uint32_t phF = 0, phG = 0;  // parity bits per stage
  bool ok = true;
  for (int pc = 0; pc < nch; ++pc) {
    const int b = pc & 1;
    const int64_t c0 = t_begin + (int64_t)pc * kC;
    const int n = (int)(t_end - c0 < kC ? t_end - c0 : kC);
    ok = mbar_wait(&B.ysfull[b], par(phF, b), kWait);
    phF ^= 1u << b;
    ok = mbar_wait(&B.gfull[b], par(phG, b), kWait) && ok;
    phG ^= 1u << b;
    if (!named_sync_and(4, kEpiT, ok)) { ok = false; break; }
    const float ys = ldexpf(a.scale, sExp[b]);
    const uint8_t* yst = gb + C_YS + b * 16384 + et * 256;
    const int t = et;
    if (t < n) {
      uint8_t* dst = reinterpret_cast<uint8_t*>(static_cast<__nv_bfloat16*>(a.y) +
                                                ((size_t)(c0 + t) * a.H_v + h) * kD);
      // RMSNorm x gate when g is given (gate factor (1 + w_j) sigmoid(g_tj)),
      // the plain scaled rows otherwise
      float rr = ys;
      if (has_g) {
        float ss = 0.f;
#pragma unroll 4
        for (int ch = 0; ch < 16; ++ch) {
          const uint4 u = *reinterpret_cast<const uint4*>(yst + ((ch ^ (t & 15)) << 4));
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = h2f(w4[e]);
            ss += f.x * f.x + f.y * f.y;
          }
        }
        rr = ys * rsqrtf(ss * ys * ys / (float)kD + a.eps_norm);
      }
      // raw g row t: 16-byte chunk cc of panel p at cc ^ (t % 8) (TMA, SW128)
      const uint8_t* gsrc = gb + C_GS + b * 16384 + t * 128;
      // two 16-byte chunks at a time, their loads ahead of their stores
#pragma unroll 1
      for (int cb = 0; cb < 16; cb += 2) {
        uint4 u[2], gq[2];
        float4 w[4];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int ch = cb + k;
          u[k] = *reinterpret_cast<const uint4*>(yst + ((ch ^ (t & 15)) << 4));
          gq[k] = *reinterpret_cast<const uint4*>(gsrc + (ch >> 3) * 8192 +
                                                  (((ch & 7) ^ (t & 7)) << 4));
          w[2 * k] = *reinterpret_cast<const float4*>(sWn + 8 * ch);
          w[2 * k + 1] = *reinterpret_cast<const float4*>(sWn + 8 * ch + 4);
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const float wv[8] = {w[2 * k].x,     w[2 * k].y,     w[2 * k].z,     w[2 * k].w,
                               w[2 * k + 1].x, w[2 * k + 1].y, w[2 * k + 1].z, w[2 * k + 1].w};
          const uint32_t w4[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
          const uint32_t g4[4] = {gq[k].x, gq[k].y, gq[k].z, gq[k].w};
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            // (1 + w_j) sigmoid(g_tj) y_tj / rms (w = 0 and no gate without g)
            const float2 f = h2f(w4[e]);
            const float s0 = has_g ? rcp_approx(1.f + ex2_approx(-kLog2e * bf_lo(g4[e]))) : 1.f;
            const float s1 = has_g ? rcp_approx(1.f + ex2_approx(-kLog2e * bf_hi(g4[e]))) : 1.f;
            o[e] = pack_b2(f.x * rr * (wv[2 * e] * s0), f.y * rr * (wv[2 * e + 1] * s1));
          }
          st_global_v4(dst + 16 * (cb + k), o[0], o[1], o[2], o[3]);
        }
      }
    }
    mbar_arrive(&B.ysempty[b]);
  }
  if (!ok && et == 0) atomicOr(a.err, kErrTimeout);
}

__global__ void __launch_bounds__(kCta, 1)
    gdn_prefill_scan_kernel(const __grid_constant__ ScanParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* gb = smem_raw + (sb - raw);
  GDN_SCAN_TRACE_INIT();
  const int bx = (int)blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5;
  if (bx < p.items) {
    // ---- chain CTA ----
    uint64_t* bars = reinterpret_cast<uint64_t*>(gb + C_BAR);
    ChainBars B{bars,      bars + 2,  bars + 3,  bars + 4,  bars + 6,  bars + 8, bars + 10,
                bars + 11, bars + 12, bars + 14, bars + 16, bars + 18, bars + 20};
    if (tid < kD) reinterpret_cast<float*>(gb + C_WN)[tid] = 1.f + a_norm_w_or_zero(p.a, tid);
    if (tid == 32 * kLoadWarp && p.has_tiles && p.a.g != nullptr) prefetch_tmap(&p.tg);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(gb + C_BAR + 176);
    if (warp == 0) tmem_alloc(tslot, 512);
    if (tid == 0) {
      for (int k = 0; k < 22; ++k) {
        // ysfull, sready, dready count the compute threads, ysempty the
        // epilogue threads, the others one arrival (commit, copy, control)
        const uint32_t cnt = (k == 6 || k == 7 || k == 10 || k == 11)
                                 ? kChainT
                                 : ((k == 8 || k == 9) ? kEpiT : 1);
        mbar_init(bars + k, cnt);
      }
      fence_mbar_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tslot;
    if (warp < 8) {
      chain_compute(p, gb, sb, tbase, bx, B);
      // every MMA is complete (the compute warps waited for the last Y^T)
      fence_before_sync();
      named_sync(5, kChainT);
      if (warp == 0) tmem_dealloc(tbase, 512);
    } else if (tid == 32 * kCtrlWarp) {
      chain_mma(p, sb, tbase, bx, B);
    } else if (tid == 32 * kLoadWarp) {
      chain_loader(p, sb, bx, B);
    } else if (warp == kEpiWarp || warp == kEpiWarp + 1) {
      chain_epilogue(p, gb, bx, B);
    }
    return;
  }
  // ---- preparation CTA: two sub-pipelines (compute warps 4 s .. 4 s + 3,
  // control warp 8 + s) ----
  const int pidx = bx - p.items;
  const int item = pidx / kPrepCtas;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(gb + P_BAR + 48);
  if (warp == 0) tmem_alloc(tslot, 512);
  if (tid < 2) {
    uint64_t* bars = reinterpret_cast<uint64_t*>(gb + tid * kSubStride + P_BAR);
    // tma, mma0, wu, slot: one arrival; splits, stored: the compute threads
    for (int k = 0; k < 6; ++k) mbar_init(bars + k, k < 4 ? 1 : kSubT);
    fence_mbar_init();
  }
  if (tid == 0 && p.has_tiles) {
    prefetch_tmap(&p.tq);
    prefetch_tmap(&p.tk);
    prefetch_tmap(&p.tv);
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tbase = *tslot;
  const int sub = warp < 8 ? warp >> 2 : warp - 8;
  if (warp >= 10) return;
  uint64_t* bars = reinterpret_cast<uint64_t*>(gb + sub * kSubStride + P_BAR);
  PrepBars B{bars, bars + 1, bars + 2, bars + 3, bars + 4, bars + 5};
  const int lane_id = (pidx % kPrepCtas) * kSubs + sub;
  const uint32_t bA = 1 + sub;
  if (warp < 8) {
    prep_compute(p, gb + sub * kSubStride, sb + sub * kSubStride, tbase + 256 * sub, item, lane_id,
                 tid & 127, bA, B);
    fence_before_sync();
    named_sync(7, 2 * kSubT);  // both sub-pipelines' MMAs are done
    if (warp == 0) tmem_dealloc(tbase, 512);
  } else if ((tid & 31) == 0) {
    prep_control(p, sb + sub * kSubStride, tbase + 256 * sub, item, lane_id, B);
  }
}

// ---- host: tensor maps ------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [T, H, 128] bf16 with boxes of 64 (feature) x 1 (head) x 64 (token), 128-byte swizzle
bool make_tmap(CUtensorMap* m, const void* base, int64_t T, int H) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr || T < 1) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2};
  const cuuint32_t box[3] = {64, 1, 64};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int prefill_scan_capacity() {
  static int cap[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cap[dev] == 0) {
    int c = -1;
    int coop = 0, sms = 0, per_sm = 0;
    if (cudaFuncSetAttribute(gdn_prefill_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmem) == cudaSuccess &&
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gdn_prefill_scan_kernel, kCta,
                                                      kSmem) == cudaSuccess &&
        coop && encode_fn() != nullptr)
      c = per_sm * sms;
    cap[dev] = c;
  }
  return cap[dev] > 0 ? cap[dev] / (1 + kPrepCtas) : 0;
}

gdn_status launch_prefill_scan(const PrefillArgs& a, cudaStream_t stream) {
  const long long items = (long long)a.n_seq * a.H_v;
  if (a.ring == nullptr || a.ring_flags == nullptr || items < 1 || items > kScanMaxItems ||
      items > prefill_scan_capacity())
    return GDN_ERR_UNSUPPORTED;
  ScanParams p;
  p.a = a;
  p.items = (int)items;
  p.has_tiles = a.total_T > 0;
  // TMA coordinates are 32-bit
  if (a.total_T > 0x7fffff00LL) return GDN_ERR_UNSUPPORTED;
  if (p.has_tiles) {
    // a box spans 64 tokens; rows past total_T (or a shorter tensor) read as zeros
    if (!make_tmap(&p.tq, a.q, a.total_T, a.H_qk) || !make_tmap(&p.tk, a.k, a.total_T, a.H_qk) ||
        !make_tmap(&p.tv, a.v, a.total_T, a.H_v))
      return GDN_ERR_CUDA;
  } else {
    memset(&p.tq, 0, sizeof(p.tq));
    memset(&p.tk, 0, sizeof(p.tk));
    memset(&p.tv, 0, sizeof(p.tv));
  }
  if (p.has_tiles && a.g != nullptr) {
    if (!make_tmap(&p.tg, a.g, a.total_T, a.H_v)) return GDN_ERR_CUDA;
  } else {
    memset(&p.tg, 0, sizeof(p.tg));
  }
  if (cudaMemsetAsync(a.ring_flags, 0, scan_flag_bytes(items), stream) != cudaSuccess)
    return GDN_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((1 + kPrepCtas) * items), 1, 1);
  cfg.blockDim = dim3(kCta, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, gdn_prefill_scan_kernel, p) != cudaSuccess) return GDN_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn
