// Backward of the chunked gated delta rule on CUDA cores, fp32 throughout.
// Tiles move into shared memory with 16-byte asynchronous copies; the two
// chains keep their state slice in registers and run two CTAs per SM.
//
// The forward is the recurrence of "Qwen3.8-Flash-Next: architecture,
// efficiency and technical lineage", section 03 "Gated DeltaNet" (update
// equations), with the optional RMSNorm x sigmoid(g) output epilogue of the
// same section.  Its chunkwise form, per chunk of C = 64 tokens with
// entering state S0, Qs = scale Q^, E_ti = exp(G_t - G_i), gamma = exp(G),
// b = exp(G_C - G):
//
//   A = diag(beta) (K K^T o E)_strict      T = (I + A)^-1
//   W = T diag(beta gamma) K               U = T diag(beta) V
//   Delta = U - W S0                       P = (Qs K^T o E)_lower-incl
//   O  = diag(gamma) Qs S0 + P Delta       S1 = gamma_C S0 + (diag(b) K)^T Delta
//
// is differentiated by hand.  Given dO and dS1 (the gradient of the state
// leaving the chunk):
//
//   chains (the d_v columns of the state are independent):
//     dDelta = P^T dO + diag(b) K dS1
//     dS0    = (diag(gamma) Qs)^T dO + gamma_C dS1 - W^T dDelta
//   per chunk:
//     TdD = T^T dDelta, dV = diag(beta) TdD, R = (I + A) Delta,
//     dT = dDelta R^T, dA = -(T^T dT T^T)_strict, dP = (dO Delta^T)_lower-incl,
//     L1 = dO S0^T, L2 = TdD S0^T, L3 = Delta dS1^T,
//     dQs = diag(gamma) L1 + (dP o E) K,
//     dK  = (dP o E)^T Qs + diag(b) L3 - diag(beta gamma) L2 + (B + B^T) K,
//           B = dA o E o beta_t,
//   and the gate gradients collected per row (dbeta directly, dG then a
//   reverse cumulative sum within the chunk for dlog alpha).
//
// Kernels, in launch order (all per value head h; "chunk" is an entry of a
// device-built table of (sequence, first token, length)):
//   chunk_table  chunk list and each sequence's first chunk
//   normalise    q^, k^ in fp32
//   prep         per chunk: G, T, K K^T o E, P, W (and W^T), U
//   fwd_chain    per (sequence, 32 state columns): S entering each chunk, Delta
//   dout         per chunk: dO (with the epilogue: O recomputed, then dy taken
//                back through the gate and the RMS norm), and the dO-only
//                products X1 = P^T dO, X2 = (diag(gamma) Qs)^T dO
//   bwd_chain    per (sequence, 32 state columns): dS1 of each chunk,
//                dDelta = X1 + diag(b) K dS1
//   chunk_a      per chunk: TdD, dV, R, dT, dA, dP and their row terms
//   chunk_b      per chunk: L1..L3, dq^ and dk^ of this value head, dbeta, dlog alpha
//   qk_final     sum over the value heads of a QK head, then the L2 norm
//   dw_reduce    the norm weight's gradient, summed over chunks
#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_sm100.cuh"

namespace gdn {
namespace {

using sm100::cp_async16;
using sm100::cp_async_commit;
using sm100::cp_async_wait_all;
using sm100::smem_u32;

constexpr int kC = 64;    // chunk length
constexpr int kNT = 256;  // threads per CTA; (ty, tx) = (tid / 16, tid % 16)
constexpr int kLC = kC + 4;  // padded row length of C x C tiles (16-byte rows)

struct ChunkEnt {
  long long t0;  // first token
  int seq;
  int n;         // tokens in this chunk (1..64)
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

int64_t max_chunks_of(int32_t n_seq, int64_t total_T) { return (total_T + kC - 1) / kC + n_seq; }

// ---------------------------------------------------------------------------
// Shared-memory tiles are row-major, rows padded by 4 floats (16-byte rows).

// rows x cols fp32 (cols % 4 == 0) from global rows of stride gstride floats
// (16-byte aligned) into shared memory, asynchronously; rows >= valid are
// zero-filled.  Completes at cp_async_wait_all() + __syncthreads().
__device__ __forceinline__ void cp_tile(float* s, int ld, const float* g, size_t gstride, int rows,
                                        int valid, int cols) {
  const int c4 = cols / 4;
  for (int e = threadIdx.x; e < rows * c4; e += kNT) {
    const int r = e / c4, c = (e % c4) * 4;
    const bool ok = r < valid;
    cp_async16(smem_u32(s + r * ld + c), ok ? g + (size_t)r * gstride + c : g, ok);
  }
}

// The same for input-dtype rows (bf16 or fp32), converted to fp32; synchronous.
template <typename Tin>
__device__ __forceinline__ void ld_rows_in(float* s, int ld, const Tin* g, size_t gstride, int rows,
                                           int valid, int cols) {
  const int c4 = cols / 4;
  for (int e = threadIdx.x; e < rows * c4; e += kNT) {
    const int r = e / c4, c = (e % c4) * 4;
    const float4 x = r < valid ? Elem<Tin>::load4(g + (size_t)r * gstride + c)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<float4*>(s + r * ld + c) = x;
  }
}

__device__ __forceinline__ bool chunk_of(const BwdArgs& a, const ChunkEnt** ent) {
  const int count = a.seq_first[a.n_seq];
  if ((int)blockIdx.x >= count) return false;
  *ent = reinterpret_cast<const ChunkEnt*>(a.chunks) + blockIdx.x;
  return true;
}

// ---------------------------------------------------------------------------
// chunk_table: one CTA.  seq_first[s] = index of sequence s's first chunk,
// seq_first[n_seq] = number of chunks.

__global__ void __launch_bounds__(kNT) bwd_chunk_table_kernel(const BwdArgs a) {
  __shared__ int s_warp[kNT / 32];
  __shared__ int s_carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_carry = 0;
  __syncthreads();
  for (int base = 0; base < a.n_seq; base += kNT) {
    const int s = base + tid;
    int nch = 0;
    if (s < a.n_seq) {
      int64_t t0, t1;
      if (seq_bounds(a.cu_seqlens, s, a.total_T, &t0, &t1, a.err)) nch = (int)((t1 - t0 + kC - 1) / kC);
    }
    int x = nch;  // inclusive scan over the block
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += u;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    int before = s_carry;
    for (int w = 0; w < warp; ++w) before += s_warp[w];
    if (s < a.n_seq) a.seq_first[s] = before + x - nch;
    __syncthreads();
    if (tid == kNT - 1) s_carry = before + x;
    __syncthreads();
  }
  if (tid == 0) a.seq_first[a.n_seq] = s_carry;
  __syncthreads();
  ChunkEnt* ents = reinterpret_cast<ChunkEnt*>(a.chunks);
  for (int s = tid; s < a.n_seq; s += kNT) {
    int64_t t0, t1;
    if (!seq_bounds(a.cu_seqlens, s, a.total_T, &t0, &t1, nullptr)) continue;
    const int first = a.seq_first[s];
    for (int64_t c0 = t0, c = 0; c0 < t1; c0 += kC, ++c) {
      ChunkEnt e;
      e.t0 = c0;
      e.seq = s;
      e.n = (int)((t1 - c0) < kC ? (t1 - c0) : kC);
      ents[first + c] = e;
    }
  }
}

// ---------------------------------------------------------------------------
// normalise: one warp per (token, QK head); q^ and k^ in fp32.

template <int DK, typename Tin>
__global__ void __launch_bounds__(kNT) bwd_normalise_kernel(const BwdArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (kNT / 32) + (threadIdx.x >> 5);
  if (row >= a.total_T * a.H_qk) return;
  const Tin* Q = static_cast<const Tin*>(a.q) + row * DK;
  const Tin* K = static_cast<const Tin*>(a.k) + row * DK;
  float qv[(DK + 31) / 32], kv[(DK + 31) / 32];
  float nq = 0.f, nk = 0.f;
#pragma unroll
  for (int m = 0; m < (DK + 31) / 32; ++m) {
    const int d = lane + 32 * m;
    qv[m] = d < DK ? Elem<Tin>::load(Q + d) : 0.f;
    kv[m] = d < DK ? Elem<Tin>::load(K + d) : 0.f;
    nq += qv[m] * qv[m];
    nk += kv[m] * kv[m];
  }
  nq = warp_sum(nq);
  nk = warp_sum(nk);
  const float rq = a.l2norm ? rsqrtf(nq + a.eps_l2) : 1.f;
  const float rk = a.l2norm ? rsqrtf(nk + a.eps_l2) : 1.f;
#pragma unroll
  for (int m = 0; m < (DK + 31) / 32; ++m) {
    const int d = lane + 32 * m;
    if (d < DK) {
      a.qh[row * DK + d] = qv[m] * rq;
      a.kh[row * DK + d] = kv[m] * rk;
    }
  }
}

// ---------------------------------------------------------------------------
// prep: per (chunk, value head).  Two CTAs per SM.

template <int DK, int DV>
struct PrepSmem {
  static constexpr int LK = DK + 4, LQV = (DK > DV ? DK : DV) + 4;
  static constexpr int oK = 0, oQV = oK + kC * LK, oA = oQV + kC * LQV, oT = oA + kC * kLC,
                       oG = oT + kC * kLC, oB = oG + kC, total = oB + kC;
  static constexpr size_t bytes = sizeof(float) * total;
};

// Inclusive cumsum of log alpha over one chunk into sG, beta into sB (warp 0;
// rows >= n get log alpha = 0, beta = 0).
__device__ __forceinline__ void load_gates(const BwdArgs& a, const ChunkEnt& e, int h, float* sG,
                                           float* sB) {
  const int lane = threadIdx.x & 31;
  if ((threadIdx.x >> 5) != 0) return;
  float carry = 0.f;
  for (int base = 0; base < kC; base += 32) {
    const int r = base + lane;
    float x = r < e.n ? __ldg(a.log_alpha + (size_t)(e.t0 + r) * a.H_v + h) : 0.f;
    const float b = r < e.n ? __ldg(a.beta + (size_t)(e.t0 + r) * a.H_v + h) : 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += u;
    }
    sG[r] = x + carry;
    sB[r] = b;
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
}

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(kNT, 2) bwd_prep_kernel(const BwdArgs a) {
  using L = PrepSmem<DK, DV>;
  constexpr int NK = DK / 16, NV = DV / 16;
  extern __shared__ __align__(16) float smem[];
  const ChunkEnt* e;
  if (!chunk_of(a, &e)) return;
  const int h = blockIdx.y, hq = h / (a.H_v / a.H_qk);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, ty = tid / 16, tx = tid % 16;
  float *sK = smem + L::oK, *sQV = smem + L::oQV, *sA = smem + L::oA, *sT = smem + L::oT,
        *sG = smem + L::oG, *sB = smem + L::oB;
  const size_t ch = (size_t)blockIdx.x * a.H_v + h;
  const int n = e->n;
  const size_t krow = (size_t)a.H_qk * DK;
  cp_tile(sK, L::LK, a.kh + ((size_t)e->t0 * a.H_qk + hq) * DK, krow, kC, n, DK);
  cp_tile(sQV, L::LQV, a.qh + ((size_t)e->t0 * a.H_qk + hq) * DK, krow, kC, n, DK);
  cp_async_commit();
  load_gates(a, *e, h, sG, sB);
  cp_async_wait_all();
  __syncthreads();

  // K K^T o E (strictly lower) -> global and A = beta_t (.) into sA; P -> global
  {
    float kk[4][4], qk[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < 4; ++w) kk[u][w] = qk[u][w] = 0.f;
    for (int d = 0; d < DK; ++d) {
      float kt[4], qt[4], ki[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        kt[u] = sK[(ty + 16 * u) * L::LK + d];
        qt[u] = sQV[(ty + 16 * u) * L::LQV + d];
        ki[u] = sK[(tx + 16 * u) * L::LK + d];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          kk[u][w] += kt[u] * ki[w];
          qk[u][w] += qt[u] * ki[w];
        }
    }
    float* gKKE = a.KKE + ch * kC * kC;
    float* gP = a.P + ch * kC * kC;
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int t = ty + 16 * u, i = tx + 16 * w;
        const float E = i <= t ? expf(sG[t] - sG[i]) : 0.f;
        const float kke = i < t ? kk[u][w] * E : 0.f;
        gKKE[t * kC + i] = kke;
        sA[t * kLC + i] = sB[t] * kke;
        gP[t * kC + i] = i <= t ? a.scale * qk[u][w] * E : 0.f;
      }
  }
  // this thread's share of V, fetched while T is being formed
  float vr[kC * DV / kNT];
  {
    const Tin* V = static_cast<const Tin*>(a.v) + ((size_t)e->t0 * a.H_v + h) * DV;
#pragma unroll
    for (int m = 0; m < kC * DV / (4 * kNT); ++m) {
      const int x = (tid + m * kNT) * 4, r = x / DV, c = x % DV;
      const float4 f = r < n ? Elem<Tin>::load4(V + (size_t)r * a.H_v * DV + c)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
      vr[4 * m] = f.x;
      vr[4 * m + 1] = f.y;
      vr[4 * m + 2] = f.z;
      vr[4 * m + 3] = f.w;
    }
  }
  __syncthreads();  // sA complete; Q^ no longer read

  // T = (I + A)^-1, row by row: T_t = e_t - sum_{i<t} A_ti T_i.  Each warp
  // owns 8 columns, 4 lanes per column split the sum.
  {
    const int j = warp * 8 + lane / 4, p = lane % 4;
    for (int t = 0; t < kC; ++t) {
      float s = 0.f;
      for (int i = j + p; i < t; i += 4) s += sA[t * kLC + i] * sT[i * kLC + j];
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (p == 0) sT[t * kLC + j] = (t == j ? 1.f : 0.f) - (t > j ? s : 0.f);
      __syncwarp();
    }
  }
#pragma unroll
  for (int m = 0; m < kC * DV / (4 * kNT); ++m) {
    const int x = (tid + m * kNT) * 4, r = x / DV, c = x % DV;
    *reinterpret_cast<float4*>(sQV + r * L::LQV + c) =
        make_float4(vr[4 * m], vr[4 * m + 1], vr[4 * m + 2], vr[4 * m + 3]);
  }
  __syncthreads();

  // W = T diag(beta gamma) K, U = T diag(beta) V
  {
    float wacc[4][NK], uacc[4][NV];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
#pragma unroll
      for (int w = 0; w < NK; ++w) wacc[u][w] = 0.f;
#pragma unroll
      for (int w = 0; w < NV; ++w) uacc[u][w] = 0.f;
    }
    for (int i = 0; i < kC; ++i) {
      const float bi = sB[i], bgi = bi * expf(sG[i]);
      float tr[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) tr[u] = sT[(ty + 16 * u) * kLC + i];
#pragma unroll
      for (int w = 0; w < NK; ++w) {
        const float kv = bgi * sK[i * L::LK + tx + 16 * w];
#pragma unroll
        for (int u = 0; u < 4; ++u) wacc[u][w] += tr[u] * kv;
      }
#pragma unroll
      for (int w = 0; w < NV; ++w) {
        const float vv = bi * sQV[i * L::LQV + tx + 16 * w];
#pragma unroll
        for (int u = 0; u < 4; ++u) uacc[u][w] += tr[u] * vv;
      }
    }
    float* gW = a.W + ch * kC * DK;
    float* gWT = a.WT + ch * kC * DK;
    float* gU = a.UT + ch * kC * DV;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = ty + 16 * u;
#pragma unroll
      for (int w = 0; w < NK; ++w) {
        gW[t * DK + tx + 16 * w] = wacc[u][w];
        gWT[(tx + 16 * w) * kC + t] = wacc[u][w];
      }
#pragma unroll
      for (int w = 0; w < NV; ++w) gU[t * DV + tx + 16 * w] = uacc[u][w];
    }
  }
  for (int x = tid; x < kC * kC; x += kNT) a.T[ch * kC * kC + x] = sT[(x / kC) * kLC + x % kC];
  if (tid < kC) a.G[ch * kC + tid] = sG[tid];
}

// ---------------------------------------------------------------------------
// Chains: per (sequence, value head, slice of SW state columns).  The state
// columns evolve independently, so each slice is its own recurrence.  Two
// CTAs per SM: one's loads overlap the other's arithmetic.

template <int DV>
struct Slice {
  static constexpr int SW = DV < 32 ? DV : 32;
  static constexpr int NS = DV / SW;
  static constexpr int NW = SW / 16;  // column blocks per thread
};

template <int DK, int DV>
struct ChainSmem {
  static constexpr int LK = DK + 4, LS = Slice<DV>::SW + 4, LT = kC + 4;
  // fwd_chain: W^T [DK][LT]; bwd_chain: W [C][LK] (the larger of the two)
  static constexpr int WSZ = (DK * LT > kC * LK) ? DK * LT : kC * LK;
  static constexpr int oW = 0, oK = oW + WSZ, oS = oK + kC * LK, oD = oS + DK * LS,
                       oB = oD + kC * LS, oG = oB + kC, total = oG + kC;
  static constexpr size_t bytes = sizeof(float) * total;
};

// N consecutive floats from shared memory (N = 1, 2, 4 or 8; 4N-byte aligned)
template <int N>
__device__ __forceinline__ void lds_row(const float* p, float* x) {
  if constexpr (N == 8) {
    const float4 a = reinterpret_cast<const float4*>(p)[0];
    const float4 b = reinterpret_cast<const float4*>(p)[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  } else if constexpr (N == 4) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  } else if constexpr (N == 2) {
    const float2 a = *reinterpret_cast<const float2*>(p);
    x[0] = a.x; x[1] = a.y;
  } else {
    x[0] = p[0];
  }
}

// L2 prefetch of `rows` rows of `row_floats` floats (a multiple of 32: whole
// 128-byte lines), `stride` floats apart, spread over the CTA's threads.
__device__ __forceinline__ void prefetch_rows(const float* p, int rows, size_t stride,
                                              int row_floats) {
  const int lines = row_floats / 32;
  for (int x = threadIdx.x; x < rows * lines; x += kNT)
    sm100::prefetch_l2(p + (size_t)(x / lines) * stride + (x % lines) * 32);
}

// b_t = exp(G_C - G_t) for the chunk (warp 0), once per chunk
__device__ __forceinline__ void chunk_decay(const float* sG, float* sB) {
  if (threadIdx.x < kC) sB[threadIdx.x] = expf(sG[kC - 1] - sG[threadIdx.x]);
}

// fwd_chain: S entering each chunk -> ws S; Delta = U - W S -> ws D.  The
// state slice lives in registers, thread (ty, tx) holding rows NK ty .. NK ty
// + NK - 1 (consecutive, for vector loads of K^) and columns tx + 16 w.
template <int DK, int DV>
__global__ void __launch_bounds__(kNT, 2) bwd_fwd_chain_kernel(const BwdArgs a) {
  using L = ChainSmem<DK, DV>;
  using SL = Slice<DV>;
  constexpr int SW = SL::SW, NW = SL::NW, NK = DK / 16;
  extern __shared__ __align__(16) float smem[];
  float *sWt = smem + L::oW, *sK = smem + L::oK, *sS = smem + L::oS, *sD = smem + L::oD,
        *sB = smem + L::oB, *sG = smem + L::oG;
  const int seq = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * SW;
  const int hq = h / (a.H_v / a.H_qk);
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const size_t st = ((size_t)seq * a.H_v + h) * DK * DV;
  float sr[NK][NW];
#pragma unroll
  for (int u = 0; u < NK; ++u)
#pragma unroll
    for (int w = 0; w < NW; ++w)
      sr[u][w] = a.initial_state
                     ? __ldg(a.initial_state + st + (size_t)(NK * ty + u) * DV + j0 + tx + 16 * w)
                     : 0.f;
  const int c_begin = a.seq_first[seq], c_end = a.seq_first[seq + 1];
  const ChunkEnt* ents = reinterpret_cast<const ChunkEnt*>(a.chunks);
  for (int c = c_begin; c < c_end; ++c) {
    const ChunkEnt e = ents[c];
    const size_t ch = (size_t)c * a.H_v + h;
    __syncthreads();  // the previous chunk is done with every buffer
    cp_tile(sWt, L::LT, a.WT + ch * DK * kC, kC, DK, DK, kC);
    cp_tile(sK, L::LK, a.kh + ((size_t)e.t0 * a.H_qk + hq) * DK, (size_t)a.H_qk * DK, kC, e.n, DK);
    cp_tile(sG, kC, a.G + ch * kC, kC, 1, 1, kC);
    cp_async_commit();
    float* gS = a.S + ch * DK * DV + j0;
#pragma unroll
    for (int u = 0; u < NK; ++u)
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const int i = NK * ty + u, j = tx + 16 * w;
        sS[i * L::LS + j] = sr[u][w];
        gS[(size_t)i * DV + j] = sr[u][w];
      }
    float acc[4][NW];  // Delta rows 4 ty + u
    const float* gU = a.UT + ch * kC * DV + j0;
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < NW; ++w) acc[u][w] = __ldg(gU + (size_t)(4 * ty + u) * DV + tx + 16 * w);
    cp_async_wait_all();
    __syncthreads();
    chunk_decay(sG, sB);
    if (c + 1 < c_end) {
      // the next chunk's inputs into L2 while this one is computed
      const ChunkEnt e1 = ents[c + 1];
      const size_t ch1 = (size_t)(c + 1) * a.H_v + h;
      prefetch_rows(a.WT + ch1 * DK * kC, 1, 0, DK * kC);
      prefetch_rows(a.kh + ((size_t)e1.t0 * a.H_qk + hq) * DK, e1.n, (size_t)a.H_qk * DK, DK);
      prefetch_rows(a.UT + ch1 * kC * DV + j0, kC, DV, SW);
      if (threadIdx.x == 0) sm100::prefetch_l2(a.G + ch1 * kC);
    }
    // Delta = U - W S   (W^T rows give each thread's 4 rows in one load)
#pragma unroll 8
    for (int i = 0; i < DK; ++i) {
      float sv[NW], wv[4];
#pragma unroll
      for (int w = 0; w < NW; ++w) sv[w] = sS[i * L::LS + tx + 16 * w];
      lds_row<4>(sWt + i * L::LT + 4 * ty, wv);
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < NW; ++w) acc[u][w] -= wv[u] * sv[w];
    }
    float* gD = a.D + ch * kC * DV + j0;
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const int t = 4 * ty + u, j = tx + 16 * w;
        sD[t * L::LS + j] = acc[u][w];
        gD[(size_t)t * DV + j] = acc[u][w];
      }
    __syncthreads();
    // S <- gamma_C S + (diag(b) K)^T Delta
    const float gC = expf(sG[kC - 1]);
#pragma unroll
    for (int u = 0; u < NK; ++u)
#pragma unroll
      for (int w = 0; w < NW; ++w) sr[u][w] *= gC;
#pragma unroll 8
    for (int t = 0; t < kC; ++t) {
      const float bt = sB[t];
      float dv[NW], kv[NK];
#pragma unroll
      for (int w = 0; w < NW; ++w) dv[w] = sD[t * L::LS + tx + 16 * w];
      lds_row<NK>(sK + t * L::LK + NK * ty, kv);
#pragma unroll
      for (int u = 0; u < NK; ++u) {
        const float kb = bt * kv[u];
#pragma unroll
        for (int w = 0; w < NW; ++w) sr[u][w] += kb * dv[w];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// dout: per (chunk, value head).  dO = dy without the epilogue; with it, O is
// recomputed and dy is taken back through sigmoid(g), (1 + w) and the RMS
// norm (also writing dg and this chunk's share of dw).  Then the two
// products the state-gradient chain needs from dO alone:
//   X1 = P^T dO -> ws dD (the chain turns it into dDelta in place)
//   X2 = scale (diag(gamma) Q^)^T dO -> ws dS (read by the chain before it
//        stores dS1 there)

template <int DK, int DV, bool EPI>
struct DoutSmem {
  static constexpr int LK = DK + 4, LV = DV + 4;
  static constexpr int oQ = 0, oP = oQ + kC * LK, oO = oP + kC * kLC, oS = oO + kC * LV,
                       oD = oS + (EPI ? DK * LV : 0), oW = oD + (EPI ? kC * LV : 0),
                       oG = oW + (EPI ? 16 * DV : 0), total = oG + kC;
  static constexpr size_t bytes = sizeof(float) * total;
};

template <int DK, int DV, typename Tin, bool EPI>
__global__ void __launch_bounds__(kNT, EPI ? 1 : 2) bwd_dout_kernel(const BwdArgs a) {
  using L = DoutSmem<DK, DV, EPI>;
  constexpr int NK = DK / 16, NV = DV / 16;
  extern __shared__ __align__(16) float smem[];
  const ChunkEnt* e;
  if (!chunk_of(a, &e)) return;
  const int h = blockIdx.y, hq = h / (a.H_v / a.H_qk);
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const size_t ch = (size_t)blockIdx.x * a.H_v + h;
  const int n = e->n;
  float *sQ = smem + L::oQ, *sP = smem + L::oP, *sO = smem + L::oO, *sS = smem + L::oS,
        *sD = smem + L::oD, *sWr = smem + L::oW, *sG = smem + L::oG;
  cp_tile(sQ, L::LK, a.qh + ((size_t)e->t0 * a.H_qk + hq) * DK, (size_t)a.H_qk * DK, kC, n, DK);
  cp_tile(sP, kLC, a.P + ch * kC * kC, kC, kC, kC, kC);
  cp_tile(sG, kC, a.G + ch * kC, kC, 1, 1, kC);
  if (EPI) {
    cp_tile(sS, L::LV, a.S + ch * DK * DV, DV, DK, DK, DV);
    cp_tile(sD, L::LV, a.D + ch * kC * DV, DV, kC, kC, DV);
  }
  cp_async_commit();
  const Tin* dY = static_cast<const Tin*>(a.dy);
  const size_t row0 = (size_t)e->t0 * a.H_v + h;  // row of token t0, this head
  // this thread's tile of dy: rows ty + 16u, columns tx + 16w
  float dyr[4][NV];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int t = ty + 16 * u;
#pragma unroll
    for (int w = 0; w < NV; ++w)
      dyr[u][w] = t < n ? Elem<Tin>::load(dY + (row0 + (size_t)t * a.H_v) * DV + tx + 16 * w) : 0.f;
  }
  cp_async_wait_all();
  __syncthreads();
  if (EPI) {
    // O = scale diag(gamma) Q^ S0 + P Delta, in registers
    float o[4][NV], pacc[4][NV];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < NV; ++w) o[u][w] = pacc[u][w] = 0.f;
    for (int i = 0; i < DK; ++i) {
      float sv[NV];
#pragma unroll
      for (int w = 0; w < NV; ++w) sv[w] = sS[i * L::LV + tx + 16 * w];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float qv = sQ[(ty + 16 * u) * L::LK + i];
#pragma unroll
        for (int w = 0; w < NV; ++w) o[u][w] += qv * sv[w];
      }
    }
    for (int i = 0; i < kC; ++i) {
      float dv[NV];
#pragma unroll
      for (int w = 0; w < NV; ++w) dv[w] = sD[i * L::LV + tx + 16 * w];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float pv = sP[(ty + 16 * u) * kLC + i];
#pragma unroll
        for (int w = 0; w < NV; ++w) pacc[u][w] += pv * dv[w];
      }
    }
    const Tin* Gg = static_cast<const Tin*>(a.g);
    float wsum[NV];
#pragma unroll
    for (int w = 0; w < NV; ++w) wsum[w] = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = ty + 16 * u;
      const float sg0 = a.scale * expf(sG[t]);
      float ss = 0.f;
#pragma unroll
      for (int w = 0; w < NV; ++w) {
        o[u][w] = sg0 * o[u][w] + pacc[u][w];
        ss += o[u][w] * o[u][w];
      }
      ss = group_sum<16>(ss);
      const float rs = rsqrtf(ss / (float)DV + a.eps_norm);
      float dot = 0.f;
#pragma unroll
      for (int w = 0; w < NV; ++w) {
        const int j = tx + 16 * w;
        const float wj = a.norm_w ? __ldg(a.norm_w + j) : 0.f;
        const float gv = t < n ? Elem<Tin>::load(Gg + (row0 + (size_t)t * a.H_v) * DV + j) : 0.f;
        const float sgm = sigmoidf_(gv);
        const float nv = o[u][w] * rs;
        const float dyj = dyr[u][w];
        if (t < n) a.dg[(row0 + (size_t)t * a.H_v) * DV + j] = dyj * nv * (1.f + wj) * sgm * (1.f - sgm);
        wsum[w] += dyj * nv * sgm;
        const float dn = dyj * (1.f + wj) * sgm;
        pacc[u][w] = nv;   // keep n
        dyr[u][w] = dn;    // dn in place of dy
        dot += dn * nv;
      }
      dot = group_sum<16>(dot) / (float)DV;
#pragma unroll
      for (int w = 0; w < NV; ++w) dyr[u][w] = rs * (dyr[u][w] - pacc[u][w] * dot);
    }
#pragma unroll
    for (int w = 0; w < NV; ++w) sWr[ty * DV + tx + 16 * w] = wsum[w];
  }
  // dO -> ws (valid rows) and shared memory (all rows; padded rows are 0)
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int t = ty + 16 * u;
#pragma unroll
    for (int w = 0; w < NV; ++w) {
      const int j = tx + 16 * w;
      sO[t * L::LV + j] = dyr[u][w];
      if (t < n) a.dO[(row0 + (size_t)t * a.H_v) * DV + j] = dyr[u][w];
    }
  }
  __syncthreads();
  if (EPI) {
    for (int j = tid; j < DV; j += kNT) {
      float s = 0.f;
      for (int r = 0; r < 16; ++r) s += sWr[r * DV + j];
      a.dw[ch * DV + j] = s;
    }
  }
  // X1 = P^T dO: X1_tj = sum_{s >= t} P_st dO_sj
  {
    float acc[4][NV];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < NV; ++w) acc[u][w] = 0.f;
    for (int s = 0; s < kC; ++s) {
      float yv[NV];
#pragma unroll
      for (int w = 0; w < NV; ++w) yv[w] = sO[s * L::LV + tx + 16 * w];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float pv = sP[s * kLC + ty + 16 * u];
#pragma unroll
        for (int w = 0; w < NV; ++w) acc[u][w] += pv * yv[w];
      }
    }
    float* gX1 = a.dD + ch * kC * DV;
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < NV; ++w) gX1[(size_t)(ty + 16 * u) * DV + tx + 16 * w] = acc[u][w];
  }
  // X2 = scale sum_t gamma_t q^_t dO_t^T (d_k x d_v)
  {
    float acc[NK][NV];
#pragma unroll
    for (int u = 0; u < NK; ++u)
#pragma unroll
      for (int w = 0; w < NV; ++w) acc[u][w] = 0.f;
    for (int t = 0; t < kC; ++t) {
      const float sg0 = a.scale * expf(sG[t]);
      float yv[NV];
#pragma unroll
      for (int w = 0; w < NV; ++w) yv[w] = sO[t * L::LV + tx + 16 * w];
#pragma unroll
      for (int u = 0; u < NK; ++u) {
        const float qv = sg0 * sQ[t * L::LK + ty + 16 * u];
#pragma unroll
        for (int w = 0; w < NV; ++w) acc[u][w] += qv * yv[w];
      }
    }
    float* gX2 = a.dS + ch * DK * DV;
#pragma unroll
    for (int u = 0; u < NK; ++u)
#pragma unroll
      for (int w = 0; w < NV; ++w) gX2[(size_t)(ty + 16 * u) * DV + tx + 16 * w] = acc[u][w];
  }
}

// bwd_chain: chunks in reverse; dS1 of each chunk -> ws dS (after taking X2
// from there); dDelta = X1 + diag(b) K dS1 -> ws dD (in place of X1).  The
// dS slice lives in registers with the row mapping of fwd_chain.
template <int DK, int DV>
__global__ void __launch_bounds__(kNT, 2) bwd_bwd_chain_kernel(const BwdArgs a) {
  using L = ChainSmem<DK, DV>;
  using SL = Slice<DV>;
  constexpr int SW = SL::SW, NW = SL::NW, NK = DK / 16;
  extern __shared__ __align__(16) float smem[];
  float *sW = smem + L::oW, *sK = smem + L::oK, *sdS = smem + L::oS, *sdD = smem + L::oD,
        *sB = smem + L::oB, *sG = smem + L::oG;
  const int seq = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * SW;
  const int hq = h / (a.H_v / a.H_qk);
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const size_t st = ((size_t)seq * a.H_v + h) * DK * DV;
  float dr[NK][NW];  // rows NK ty + u, columns j0 + tx + 16 w
#pragma unroll
  for (int u = 0; u < NK; ++u)
#pragma unroll
    for (int w = 0; w < NW; ++w)
      dr[u][w] = a.d_final_state
                     ? __ldg(a.d_final_state + st + (size_t)(NK * ty + u) * DV + j0 + tx + 16 * w)
                     : 0.f;
  const int c_begin = a.seq_first[seq], c_end = a.seq_first[seq + 1];
  const ChunkEnt* ents = reinterpret_cast<const ChunkEnt*>(a.chunks);
  for (int c = c_end - 1; c >= c_begin; --c) {
    const ChunkEnt e = ents[c];
    const size_t ch = (size_t)c * a.H_v + h;
    __syncthreads();
    cp_tile(sW, L::LK, a.W + ch * kC * DK, DK, kC, kC, DK);
    cp_tile(sK, L::LK, a.kh + ((size_t)e.t0 * a.H_qk + hq) * DK, (size_t)a.H_qk * DK, kC, e.n, DK);
    cp_tile(sG, kC, a.G + ch * kC, kC, 1, 1, kC);
    cp_async_commit();
    float* gdS = a.dS + ch * DK * DV + j0;
    float x2[NK][NW];
#pragma unroll
    for (int u = 0; u < NK; ++u)
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const int i = NK * ty + u, j = tx + 16 * w;
        x2[u][w] = gdS[(size_t)i * DV + j];  // X2, then the same element gets dS1
        gdS[(size_t)i * DV + j] = dr[u][w];
        sdS[i * L::LS + j] = dr[u][w];
      }
    float* gdD = a.dD + ch * kC * DV + j0;
    float acc[4][NW];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < NW; ++w) acc[u][w] = gdD[(size_t)(ty + 16 * u) * DV + tx + 16 * w];
    cp_async_wait_all();
    __syncthreads();
    chunk_decay(sG, sB);
    if (c - 1 >= c_begin) {
      // the next (earlier) chunk's inputs into L2 while this one is computed
      const ChunkEnt e1 = ents[c - 1];
      const size_t ch1 = (size_t)(c - 1) * a.H_v + h;
      prefetch_rows(a.W + ch1 * kC * DK, 1, 0, kC * DK);
      prefetch_rows(a.kh + ((size_t)e1.t0 * a.H_qk + hq) * DK, e1.n, (size_t)a.H_qk * DK, DK);
      prefetch_rows(a.dS + ch1 * DK * DV + j0, DK, DV, SW);
      prefetch_rows(a.dD + ch1 * kC * DV + j0, kC, DV, SW);
      if (threadIdx.x == 0) sm100::prefetch_l2(a.G + ch1 * kC);
    }
    // dDelta = X1 + diag(b) K dS1  (zero on rows past the chunk's end)
    {
      float kacc[4][NW];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < NW; ++w) kacc[u][w] = 0.f;
#pragma unroll 8
      for (int i = 0; i < DK; ++i) {
        float sv[NW];
#pragma unroll
        for (int w = 0; w < NW; ++w) sv[w] = sdS[i * L::LS + tx + 16 * w];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float kv = sK[(ty + 16 * u) * L::LK + i];
#pragma unroll
          for (int w = 0; w < NW; ++w) kacc[u][w] += kv * sv[w];
        }
      }
      __syncthreads();  // sB ready
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = ty + 16 * u;
        const float bt = sB[t];
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          const int j = tx + 16 * w;
          const float v = t < e.n ? acc[u][w] + bt * kacc[u][w] : 0.f;
          sdD[t * L::LS + j] = v;
          gdD[(size_t)t * DV + j] = v;
        }
      }
    }
    __syncthreads();
    // dS <- gamma_C dS + X2 - W^T dDelta
    {
      const float gC = expf(sG[kC - 1]);
#pragma unroll
      for (int u = 0; u < NK; ++u)
#pragma unroll
        for (int w = 0; w < NW; ++w) dr[u][w] = gC * dr[u][w] + x2[u][w];
#pragma unroll 8
      for (int t = 0; t < kC; ++t) {
        float dv[NW], wv[NK];
#pragma unroll
        for (int w = 0; w < NW; ++w) dv[w] = sdD[t * L::LS + tx + 16 * w];
        lds_row<NK>(sW + t * L::LK + NK * ty, wv);
#pragma unroll
        for (int u = 0; u < NK; ++u)
#pragma unroll
          for (int w = 0; w < NW; ++w) dr[u][w] -= wv[u] * dv[w];
      }
    }
  }
  if (a.d_initial_state) {
#pragma unroll
    for (int u = 0; u < NK; ++u)
#pragma unroll
      for (int w = 0; w < NW; ++w)
        a.d_initial_state[st + (size_t)(NK * ty + u) * DV + j0 + tx + 16 * w] = dr[u][w];
  }
}

// ---------------------------------------------------------------------------
// chunk_a: per (chunk, value head).

template <int DV>
struct ChunkASmem {
  static constexpr int LV = DV + 4;
  static constexpr int oD = 0, odD = oD + kC * LV, odY = odD + kC * LV, oX = odY + kC * LV,
                       oT = oX + kC * LV, oKKE = oT + kC * kLC, oP = oKKE + kC * kLC,
                       oM1 = oP + kC * kLC, oM2 = oM1 + kC * kLC, oG = oM2 + kC * kLC,
                       oB = oG + kC, oR0 = oB + kC, oR1 = oR0 + kC, total = oR1 + kC;
  static constexpr size_t bytes = sizeof(float) * total;
};

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(kNT, 1) bwd_chunk_a_kernel(const BwdArgs a) {
  using L = ChunkASmem<DV>;
  constexpr int NV = DV / 16;
  extern __shared__ __align__(16) float smem[];
  const ChunkEnt* e;
  if (!chunk_of(a, &e)) return;
  const int h = blockIdx.y;
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const size_t ch = (size_t)blockIdx.x * a.H_v + h;
  const int n = e->n;
  float *sD = smem + L::oD, *sdD = smem + L::odD, *sdY = smem + L::odY, *sX = smem + L::oX,
        *sT = smem + L::oT, *sKKE = smem + L::oKKE, *sP = smem + L::oP, *sM1 = smem + L::oM1,
        *sM2 = smem + L::oM2, *sG = smem + L::oG, *sB = smem + L::oB, *sR0 = smem + L::oR0,
        *sR1 = smem + L::oR1;
  cp_tile(sD, L::LV, a.D + ch * kC * DV, DV, kC, kC, DV);
  cp_tile(sdD, L::LV, a.dD + ch * kC * DV, DV, kC, kC, DV);
  cp_tile(sdY, L::LV, a.dO + ((size_t)e->t0 * a.H_v + h) * DV, (size_t)a.H_v * DV, kC, n, DV);
  cp_tile(sT, kLC, a.T + ch * kC * kC, kC, kC, kC, kC);
  cp_tile(sKKE, kLC, a.KKE + ch * kC * kC, kC, kC, kC, kC);
  cp_tile(sP, kLC, a.P + ch * kC * kC, kC, kC, kC, kC);
  cp_tile(sG, kC, a.G + ch * kC, kC, 1, 1, kC);
  cp_async_commit();
  ld_rows_in(sX, L::LV, static_cast<const Tin*>(a.v) + ((size_t)e->t0 * a.H_v + h) * DV,
             (size_t)a.H_v * DV, kC, n, DV);
  if (tid < kC) sB[tid] = tid < n ? __ldg(a.beta + (size_t)(e->t0 + tid) * a.H_v + h) : 0.f;
  cp_async_wait_all();
  __syncthreads();

  // TdD = T^T dDelta -> global (reusing U's place); dV = diag(beta) TdD;
  // row term sum_j TdD_tj V_tj
  {
    float acc[4][NV];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < NV; ++w) acc[u][w] = 0.f;
    for (int i = 0; i < kC; ++i) {
      float dv[NV];
#pragma unroll
      for (int w = 0; w < NV; ++w) dv[w] = sdD[i * L::LV + tx + 16 * w];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float tv = sT[i * kLC + ty + 16 * u];  // T_{i,t}
#pragma unroll
        for (int w = 0; w < NV; ++w) acc[u][w] += tv * dv[w];
      }
    }
    float* gTdD = a.UT + ch * kC * DV;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = ty + 16 * u;
      float rv = 0.f;
#pragma unroll
      for (int w = 0; w < NV; ++w) {
        const int j = tx + 16 * w;
        gTdD[t * DV + j] = acc[u][w];
        rv += acc[u][w] * sX[t * L::LV + j];
        if (t < n) a.dv[((size_t)(e->t0 + t) * a.H_v + h) * DV + j] = sB[t] * acc[u][w];
      }
      rv = group_sum<16>(rv);
      if (tx == 0) sR0[t] = rv;
    }
  }
  __syncthreads();  // V no longer read
  // R = Delta + diag(beta) KKE Delta -> sX
  {
    float acc[4][NV];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < NV; ++w) acc[u][w] = 0.f;
    for (int i = 0; i < kC; ++i) {
      float dv[NV];
#pragma unroll
      for (int w = 0; w < NV; ++w) dv[w] = sD[i * L::LV + tx + 16 * w];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float kv = sKKE[(ty + 16 * u) * kLC + i];
#pragma unroll
        for (int w = 0; w < NV; ++w) acc[u][w] += kv * dv[w];
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = ty + 16 * u;
#pragma unroll
      for (int w = 0; w < NV; ++w) {
        const int j = tx + 16 * w;
        sX[t * L::LV + j] = sD[t * L::LV + j] + sB[t] * acc[u][w];
      }
    }
  }
  __syncthreads();
  // dT = dDelta R^T -> sM1; dP = (dO Delta^T)_lower-incl -> sM2
  {
    float tacc[4][4], pacc[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < 4; ++w) tacc[u][w] = pacc[u][w] = 0.f;
    for (int j = 0; j < DV; ++j) {
      float dd[4], yy[4], rr[4], dl[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        dd[u] = sdD[(ty + 16 * u) * L::LV + j];
        yy[u] = sdY[(ty + 16 * u) * L::LV + j];
        rr[u] = sX[(tx + 16 * u) * L::LV + j];
        dl[u] = sD[(tx + 16 * u) * L::LV + j];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          tacc[u][w] += dd[u] * rr[w];
          pacc[u][w] += yy[u] * dl[w];
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int t = ty + 16 * u, i = tx + 16 * w;
        sM1[t * kLC + i] = tacc[u][w];
        sM2[t * kLC + i] = i <= t ? pacc[u][w] : 0.f;
      }
  }
  __syncthreads();
  // Z = T^T dT (over s >= t), then dA = -(Z T^T)_strict
  {
    float z[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < 4; ++w) z[u][w] = 0.f;
    for (int s = 0; s < kC; ++s) {
      float tv[4], dv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        tv[u] = sT[s * kLC + ty + 16 * u];   // T_{s,t}
        dv[u] = sM1[s * kLC + tx + 16 * u];  // dT_{s,i}
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) z[u][w] += tv[u] * dv[w];
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < 4; ++w) sM1[(ty + 16 * u) * kLC + tx + 16 * w] = z[u][w];
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < 4; ++w) z[u][w] = 0.f;
    for (int s = 0; s < kC; ++s) {
      float zv[4], tv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        zv[u] = sM1[(ty + 16 * u) * kLC + s];  // Z_{t,s}
        tv[u] = sT[(tx + 16 * u) * kLC + s];   // T_{i,s}
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) z[u][w] += zv[u] * tv[w];
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int t = ty + 16 * u, i = tx + 16 * w;
        sM1[t * kLC + i] = i < t ? -z[u][w] : 0.f;
      }
  }
  __syncthreads();
  // row and column terms of the gates; dP o E and dA o E o beta -> global
  {
    float* gdPE = a.dPE + ch * kC * kC;
    float* gB = a.Bm + ch * kC * kC;
    for (int x = tid; x < kC * kC; x += kNT) {
      const int t = x / kC, i = x % kC;
      const float E = i <= t ? expf(sG[t] - sG[i]) : 0.f;
      gdPE[x] = sM2[t * kLC + i] * E;
      gB[x] = sM1[t * kLC + i] * E * sB[t];
    }
    if (tid < kC) {
      const int t = tid;
      float rP = 0.f, rA = 0.f, dbA = 0.f;
      for (int i = 0; i < kC; ++i) {
        rP += sM2[t * kLC + i] * sP[t * kLC + i];
        const float dk = sM1[t * kLC + i] * sKKE[t * kLC + i];
        rA += dk;
        dbA += dk;
      }
      float cP = 0.f, cA = 0.f;
      for (int s = 0; s < kC; ++s) {
        cP += sM2[s * kLC + t] * sP[s * kLC + t];
        cA += sM1[s * kLC + t] * sKKE[s * kLC + t] * sB[s];
      }
      a.row[ch * 2 * kC + t] = sR0[t] + dbA;                    // dbeta part
      a.row[ch * 2 * kC + kC + t] = rP - cP + sB[t] * rA - cA;  // dG part
    }
  }
}

// ---------------------------------------------------------------------------
// chunk_b: per (chunk, value head).

template <int DK, int DV>
struct ChunkBSmem {
  static constexpr int LK = DK + 4, LV = DV + 4;
  static constexpr int r1a = DK * LV, r1b = 2 * kC * LK;
  static constexpr int r2a = 2 * kC * LV, r2b = 2 * kC * kLC;
  static constexpr int oR1 = 0, oR2 = oR1 + (r1a > r1b ? r1a : r1b),
                       oG = oR2 + (r2a > r2b ? r2a : r2b), oB = oG + kC, oX = oB + kC,
                       oRed = oX + kC, total = oRed + kNT / 32;
  static constexpr size_t bytes = sizeof(float) * total;
};

template <int DK, int DV>
__global__ void __launch_bounds__(kNT, 1) bwd_chunk_b_kernel(const BwdArgs a) {
  using L = ChunkBSmem<DK, DV>;
  constexpr int NK = DK / 16;
  extern __shared__ __align__(16) float smem[];
  const ChunkEnt* e;
  if (!chunk_of(a, &e)) return;
  const int h = blockIdx.y, hq = h / (a.H_v / a.H_qk);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, ty = tid / 16, tx = tid % 16;
  const size_t ch = (size_t)blockIdx.x * a.H_v + h;
  const int n = e->n;
  float *sR1 = smem + L::oR1, *sR2 = smem + L::oR2, *sG = smem + L::oG, *sB = smem + L::oB,
        *sX = smem + L::oX, *sRed = smem + L::oRed;
  float L1[4][NK], L2[4][NK], L3[4][NK];
  // phase 1: L1 = dO S0^T, L2 = TdD S0^T
  {
    float* sS = sR1;
    float* sY = sR2;
    float* sTd = sR2 + kC * L::LV;
    cp_tile(sS, L::LV, a.S + ch * DK * DV, DV, DK, DK, DV);
    cp_tile(sY, L::LV, a.dO + ((size_t)e->t0 * a.H_v + h) * DV, (size_t)a.H_v * DV, kC, n, DV);
    cp_tile(sTd, L::LV, a.UT + ch * kC * DV, DV, kC, kC, DV);
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < NK; ++w) L1[u][w] = L2[u][w] = 0.f;
    for (int j = 0; j < DV; ++j) {
      float yv[4], tv[4], sv[NK];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        yv[u] = sY[(ty + 16 * u) * L::LV + j];
        tv[u] = sTd[(ty + 16 * u) * L::LV + j];
      }
#pragma unroll
      for (int w = 0; w < NK; ++w) sv[w] = sS[(tx + 16 * w) * L::LV + j];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < NK; ++w) {
          L1[u][w] += yv[u] * sv[w];
          L2[u][w] += tv[u] * sv[w];
        }
    }
    __syncthreads();
  }
  // phase 2: L3 = Delta dS1^T, and <S0, dS1>
  float sdot = 0.f;
  {
    float* sdS = sR1;
    float* sDl = sR2;
    cp_tile(sdS, L::LV, a.dS + ch * DK * DV, DV, DK, DK, DV);
    cp_tile(sDl, L::LV, a.D + ch * kC * DV, DV, kC, kC, DV);
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    const float* gS = a.S + ch * DK * DV;
    for (int x = tid; x < DK * DV; x += kNT) sdot += gS[x] * sdS[(x / DV) * L::LV + x % DV];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < NK; ++w) L3[u][w] = 0.f;
    for (int j = 0; j < DV; ++j) {
      float dv[4], sv[NK];
#pragma unroll
      for (int u = 0; u < 4; ++u) dv[u] = sDl[(ty + 16 * u) * L::LV + j];
#pragma unroll
      for (int w = 0; w < NK; ++w) sv[w] = sdS[(tx + 16 * w) * L::LV + j];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < NK; ++w) L3[u][w] += dv[u] * sv[w];
    }
    sdot = warp_sum(sdot);
    if (lane == 0) sRed[warp] = sdot;
    __syncthreads();
  }
  // phase 3: combine
  float* sK = sR1;
  float* sQ = sR1 + kC * L::LK;
  float* sdPE = sR2;
  float* sBm = sR2 + kC * kLC;
  float sd_total = 0.f;
  for (int w = 0; w < kNT / 32; ++w) sd_total += sRed[w];
  cp_tile(sK, L::LK, a.kh + ((size_t)e->t0 * a.H_qk + hq) * DK, (size_t)a.H_qk * DK, kC, n, DK);
  cp_tile(sQ, L::LK, a.qh + ((size_t)e->t0 * a.H_qk + hq) * DK, (size_t)a.H_qk * DK, kC, n, DK);
  cp_tile(sdPE, kLC, a.dPE + ch * kC * kC, kC, kC, kC, kC);
  cp_tile(sBm, kLC, a.Bm + ch * kC * kC, kC, kC, kC, kC);
  cp_tile(sG, kC, a.G + ch * kC, kC, 1, 1, kC);
  cp_async_commit();
  if (tid < kC) sB[tid] = tid < n ? __ldg(a.beta + (size_t)(e->t0 + tid) * a.H_v + h) : 0.f;
  cp_async_wait_all();
  __syncthreads();
  const float GC = sG[kC - 1];
  float dG6[4], db6[4], bk3[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int t = ty + 16 * u;
    float q1 = 0.f, k2 = 0.f, k3 = 0.f;
#pragma unroll
    for (int w = 0; w < NK; ++w) {
      const int c = tx + 16 * w;
      q1 += sQ[t * L::LK + c] * L1[u][w];
      k2 += sK[t * L::LK + c] * L2[u][w];
      k3 += sK[t * L::LK + c] * L3[u][w];
    }
    q1 = group_sum<16>(q1);
    k2 = group_sum<16>(k2);
    k3 = group_sum<16>(k3);
    const float gam = expf(sG[t]), bt = expf(GC - sG[t]), bet = sB[t];
    dG6[u] = gam * a.scale * q1 - bet * gam * k2 - bt * k3;
    db6[u] = -gam * k2;
    bk3[u] = bt * k3;
    // fold the diagonal factors into the accumulators
#pragma unroll
    for (int w = 0; w < NK; ++w) {
      L1[u][w] *= gam;
      L3[u][w] = bt * L3[u][w] - bet * gam * L2[u][w];
    }
  }
  // dQs += (dP o E) K ; dK += (dP o E)^T Qs + (B + B^T) K
  for (int i = 0; i < kC; ++i) {
    float kv[NK], qv[NK];
#pragma unroll
    for (int w = 0; w < NK; ++w) {
      kv[w] = sK[i * L::LK + tx + 16 * w];
      qv[w] = a.scale * sQ[i * L::LK + tx + 16 * w];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = ty + 16 * u;
      const float pe = sdPE[t * kLC + i];
      const float pt = sdPE[i * kLC + t];
      const float bb = sBm[t * kLC + i] + sBm[i * kLC + t];
#pragma unroll
      for (int w = 0; w < NK; ++w) {
        L1[u][w] += pe * kv[w];
        L3[u][w] += pt * qv[w] + bb * kv[w];
      }
    }
  }
  // write dq^ (per value head, times scale: Qs = scale q^) and dk^
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int t = ty + 16 * u;
    if (t < n) {
      const size_t off = ((size_t)(e->t0 + t) * a.H_v + h) * DK;
#pragma unroll
      for (int w = 0; w < NK; ++w) {
        a.dqh[off + tx + 16 * w] = a.scale * L1[u][w];
        a.dkh[off + tx + 16 * w] = L3[u][w];
      }
    }
  }
  // gates: dG per row, then dlog alpha = reverse cumsum within the chunk
  __syncthreads();  // sG/sB stay; reuse sX for the per-row dG
  if (tx == 0) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = ty + 16 * u;
      sX[t] = dG6[u] + a.row[ch * 2 * kC + kC + t];
      if (t < n) a.dbeta[(size_t)(e->t0 + t) * a.H_v + h] = db6[u] + a.row[ch * 2 * kC + t];
    }
  }
  // the last row also collects sum_t b_t (K L3^T)_tt and gamma_C <S0, dS1>
  float part = 0.f;
  if (tx == 0) {
#pragma unroll
    for (int u = 0; u < 4; ++u) part += bk3[u];
  }
  part = warp_sum(part);  // lanes 0 and 16 of each warp hold two rows' terms
  if (lane == 0) sRed[warp] = part;
  __syncthreads();
  if (warp == 0) {
    float tot = 0.f;
    for (int w = 0; w < kNT / 32; ++w) tot += sRed[w];
    // reverse inclusive scan over the 64 rows, two passes of 32 lanes
    float carry = 0.f;
    for (int base = kC - 32; base >= 0; base -= 32) {
      const int t = base + lane;
      float x = sX[t];
      if (t == kC - 1) x += tot + expf(GC) * sd_total;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float v = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += v;
      }
      x += carry;
      if (t < n) a.dlog_alpha[(size_t)(e->t0 + t) * a.H_v + h] = x;
      carry = __shfl_sync(0xffffffffu, x, 0);
    }
  }
}

// ---------------------------------------------------------------------------
// qk_final: one warp per (token, QK head): sum the value heads' dq^, dk^ and
// differentiate the L2 norm, dx = r (dx^ - x^ (x^ . dx^)).

template <int DK, typename Tin>
__global__ void __launch_bounds__(kNT) bwd_qk_final_kernel(const BwdArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (kNT / 32) + (threadIdx.x >> 5);
  if (row >= a.total_T * a.H_qk) return;
  const int64_t t = row / a.H_qk;
  const int hq = (int)(row % a.H_qk);
  const int G = a.H_v / a.H_qk;
  constexpr int M = (DK + 31) / 32;
#pragma unroll
  for (int which = 0; which < 2; ++which) {
    const Tin* X = static_cast<const Tin*>(which ? a.k : a.q) + row * DK;
    const float* part = which ? a.dkh : a.dqh;
    float* out = (which ? a.dk : a.dq) + row * DK;
    float gx[M], xv[M];
    float ss = 0.f;
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const int d = lane + 32 * m;
      gx[m] = xv[m] = 0.f;
      if (d < DK) {
        for (int g = 0; g < G; ++g) gx[m] += part[((size_t)t * a.H_v + hq * G + g) * DK + d];
        xv[m] = Elem<Tin>::load(X + d);
        ss += xv[m] * xv[m];
      }
    }
    if (a.l2norm) {
      ss = warp_sum(ss);
      const float r = rsqrtf(ss + a.eps_l2);
      float dot = 0.f;
#pragma unroll
      for (int m = 0; m < M; ++m) dot += xv[m] * r * gx[m];
      dot = warp_sum(dot);
#pragma unroll
      for (int m = 0; m < M; ++m) gx[m] = r * (gx[m] - xv[m] * r * dot);
    }
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const int d = lane + 32 * m;
      if (d < DK) out[d] = gx[m];
    }
  }
}

// dw_reduce: dnorm_w[j] = sum over every (chunk, value head) of its share.
template <int DV>
__global__ void __launch_bounds__(kNT) bwd_dw_reduce_kernel(const BwdArgs a) {
  __shared__ float red[kNT];
  const int per = kNT / DV > 0 ? kNT / DV : 1;  // threads per column
  const int j = threadIdx.x % DV, p = threadIdx.x / DV;
  const int64_t items = (int64_t)a.seq_first[a.n_seq] * a.H_v;
  float s = 0.f;
  if (p < per)
    for (int64_t x = p; x < items; x += per) s += a.dw[x * DV + j];
  red[threadIdx.x] = s;
  __syncthreads();
  if (threadIdx.x < DV) {
    float tot = 0.f;
    for (int q = 0; q < per; ++q) tot += red[q * DV + threadIdx.x];
    a.dnorm_w[threadIdx.x] = tot;
  }
}

// ---------------------------------------------------------------------------

template <typename K>
bool set_smem(K kern, size_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) ==
         cudaSuccess;
}

template <int DK, int DV, typename Tin>
gdn_status launch(const BwdArgs& a, cudaStream_t s) {
  const int64_t maxc = max_chunks_of(a.n_seq, a.total_T);
  const unsigned H = (unsigned)a.H_v;
  const dim3 per_chunk((unsigned)maxc, H), per_slice((unsigned)a.n_seq, H, Slice<DV>::NS);
  bwd_chunk_table_kernel<<<1, kNT, 0, s>>>(a);
  if (a.total_T > 0) {
    const unsigned rows = (unsigned)((a.total_T * a.H_qk + 7) / 8);
    bwd_normalise_kernel<DK, Tin><<<rows, kNT, 0, s>>>(a);
    auto k1 = bwd_prep_kernel<DK, DV, Tin>;
    if (!set_smem(k1, PrepSmem<DK, DV>::bytes)) return GDN_ERR_CUDA;
    k1<<<per_chunk, kNT, PrepSmem<DK, DV>::bytes, s>>>(a);
    auto k2 = bwd_fwd_chain_kernel<DK, DV>;
    if (!set_smem(k2, ChainSmem<DK, DV>::bytes)) return GDN_ERR_CUDA;
    k2<<<per_slice, kNT, ChainSmem<DK, DV>::bytes, s>>>(a);
    if (a.g != nullptr) {
      auto k3 = bwd_dout_kernel<DK, DV, Tin, true>;
      if (!set_smem(k3, DoutSmem<DK, DV, true>::bytes)) return GDN_ERR_CUDA;
      k3<<<per_chunk, kNT, DoutSmem<DK, DV, true>::bytes, s>>>(a);
    } else {
      auto k3 = bwd_dout_kernel<DK, DV, Tin, false>;
      if (!set_smem(k3, DoutSmem<DK, DV, false>::bytes)) return GDN_ERR_CUDA;
      k3<<<per_chunk, kNT, DoutSmem<DK, DV, false>::bytes, s>>>(a);
    }
  }
  auto k4 = bwd_bwd_chain_kernel<DK, DV>;
  if (!set_smem(k4, ChainSmem<DK, DV>::bytes)) return GDN_ERR_CUDA;
  k4<<<per_slice, kNT, ChainSmem<DK, DV>::bytes, s>>>(a);
  if (a.total_T > 0) {
    auto k5 = bwd_chunk_a_kernel<DK, DV, Tin>;
    if (!set_smem(k5, ChunkASmem<DV>::bytes)) return GDN_ERR_CUDA;
    k5<<<per_chunk, kNT, ChunkASmem<DV>::bytes, s>>>(a);
    auto k6 = bwd_chunk_b_kernel<DK, DV>;
    if (!set_smem(k6, ChunkBSmem<DK, DV>::bytes)) return GDN_ERR_CUDA;
    k6<<<per_chunk, kNT, ChunkBSmem<DK, DV>::bytes, s>>>(a);
    const unsigned rows = (unsigned)((a.total_T * a.H_qk + 7) / 8);
    bwd_qk_final_kernel<DK, Tin><<<rows, kNT, 0, s>>>(a);
  }
  if (a.g != nullptr && a.dnorm_w != nullptr) bwd_dw_reduce_kernel<DV><<<1, kNT, 0, s>>>(a);
  return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

template <typename Tin>
gdn_status dispatch(const BwdArgs& a, cudaStream_t s) {
#define GDN_DV_CASES(DK)                         \
  switch (a.d_v) {                               \
    case 16: return launch<DK, 16, Tin>(a, s);   \
    case 32: return launch<DK, 32, Tin>(a, s);   \
    case 64: return launch<DK, 64, Tin>(a, s);   \
    case 128: return launch<DK, 128, Tin>(a, s); \
    default: return GDN_ERR_UNSUPPORTED;         \
  }
  switch (a.d_k) {
    case 16: GDN_DV_CASES(16)
    case 32: GDN_DV_CASES(32)
    case 64: GDN_DV_CASES(64)
    case 128: GDN_DV_CASES(128)
    default: return GDN_ERR_UNSUPPORTED;
  }
#undef GDN_DV_CASES
}

}  // namespace

size_t chunk_bwd_workspace_bytes(int32_t n_seq, int64_t total_T, int32_t H_qk, int32_t H_v,
                                 int32_t d_k, int32_t d_v) {
  if (n_seq < 1 || total_T < 0 || H_qk < 1 || H_v < 1 || d_k < 1 || d_v < 1) return 0;
  const size_t maxc = (size_t)max_chunks_of(n_seq, total_T);
  const size_t nch = maxc * (size_t)H_v;
  const size_t f = sizeof(float);
  size_t b = 0;
  b += align256(maxc * sizeof(ChunkEnt));
  b += align256((size_t)(n_seq + 1) * sizeof(int32_t));
  b += 2 * align256(nch * d_k * d_v * f);            // S, dS
  b += 2 * align256(nch * kC * d_k * f);             // W, W^T
  b += 3 * align256(nch * kC * d_v * f);             // U / TdD, Delta, dDelta
  b += 5 * align256(nch * kC * kC * f);              // T, KKE, P, dPE, B
  b += align256(nch * kC * f);                       // G
  b += align256(nch * 2 * kC * f);                   // row terms
  b += align256(nch * d_v * f);                      // dw shares
  b += align256((size_t)total_T * H_v * d_v * f);    // dO
  b += 2 * align256((size_t)total_T * H_v * d_k * f);   // dq^, dk^ per value head
  b += 2 * align256((size_t)total_T * H_qk * d_k * f);  // q^, k^
  return b;
}

void chunk_bwd_workspace_layout(void* ws, BwdArgs* a) {
  const size_t maxc = (size_t)max_chunks_of(a->n_seq, a->total_T);
  const size_t nch = maxc * (size_t)a->H_v;
  const size_t f = sizeof(float);
  char* p = static_cast<char*>(ws);
  auto take = [&p](size_t bytes) {
    char* r = p;
    p += align256(bytes);
    return r;
  };
  a->chunks = take(maxc * sizeof(ChunkEnt));
  a->seq_first = reinterpret_cast<int32_t*>(take((size_t)(a->n_seq + 1) * sizeof(int32_t)));
  a->S = reinterpret_cast<float*>(take(nch * a->d_k * a->d_v * f));
  a->dS = reinterpret_cast<float*>(take(nch * a->d_k * a->d_v * f));
  a->W = reinterpret_cast<float*>(take(nch * kC * a->d_k * f));
  a->WT = reinterpret_cast<float*>(take(nch * kC * a->d_k * f));
  a->UT = reinterpret_cast<float*>(take(nch * kC * a->d_v * f));
  a->D = reinterpret_cast<float*>(take(nch * kC * a->d_v * f));
  a->dD = reinterpret_cast<float*>(take(nch * kC * a->d_v * f));
  a->T = reinterpret_cast<float*>(take(nch * kC * kC * f));
  a->KKE = reinterpret_cast<float*>(take(nch * kC * kC * f));
  a->P = reinterpret_cast<float*>(take(nch * kC * kC * f));
  a->dPE = reinterpret_cast<float*>(take(nch * kC * kC * f));
  a->Bm = reinterpret_cast<float*>(take(nch * kC * kC * f));
  a->G = reinterpret_cast<float*>(take(nch * kC * f));
  a->row = reinterpret_cast<float*>(take(nch * 2 * kC * f));
  a->dw = reinterpret_cast<float*>(take(nch * a->d_v * f));
  a->dO = reinterpret_cast<float*>(take((size_t)a->total_T * a->H_v * a->d_v * f));
  a->dqh = reinterpret_cast<float*>(take((size_t)a->total_T * a->H_v * a->d_k * f));
  a->dkh = reinterpret_cast<float*>(take((size_t)a->total_T * a->H_v * a->d_k * f));
  a->qh = reinterpret_cast<float*>(take((size_t)a->total_T * a->H_qk * a->d_k * f));
  a->kh = reinterpret_cast<float*>(take((size_t)a->total_T * a->H_qk * a->d_k * f));
}

gdn_status launch_chunk_bwd(const BwdArgs& a, cudaStream_t stream) {
  if (a.dtype == GDN_BF16) return dispatch<__nv_bfloat16>(a, stream);
  if (a.dtype == GDN_FP32) return dispatch<float>(a, stream);
  return GDN_ERR_UNSUPPORTED;
}

}  // namespace gdn
