// Backward of the chunked gated delta rule on CUDA cores, fp32 throughout.
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
//   prep         per chunk: G, T, K K^T o E, P, W, U
//   fwd_chain    per (sequence, 32 state columns): S entering each chunk, Delta
//   epilogue     per chunk: O, then dO from dy through the gate and RMS norm
//   bwd_chain    per (sequence, 32 state columns): dS1 of each chunk, dDelta
//   chunk_a      per chunk: TdD, dV, R, dT, dA, dP and their row terms
//   chunk_b      per chunk: L1..L3, dq^ and dk^ of this value head, dbeta, dlog alpha
//   qk_final     sum over the value heads of a QK head, then the L2 norm
//   dw_reduce    the norm weight's gradient, summed over chunks
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kC = 64;    // chunk length
constexpr int kNT = 256;  // threads per CTA; (ty, tx) = (tid / 16, tid % 16)
constexpr int kLC = kC + 1;

struct ChunkEnt {
  long long t0;  // first token
  int seq;
  int n;         // tokens in this chunk (1..64)
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

int64_t max_chunks_of(int32_t n_seq, int64_t total_T) { return (total_T + kC - 1) / kC + n_seq; }

// ---------------------------------------------------------------------------
// Shared-memory tiles are row-major with one float of padding per row.

__device__ __forceinline__ void ld_rows(float* s, int ld, const float* g, size_t gstride, int rows,
                                        int valid, int cols) {
  // rows x cols from global rows of stride gstride; rows >= valid are zero
  for (int e = threadIdx.x; e < rows * cols; e += kNT) {
    const int r = e / cols, c = e % cols;
    s[r * ld + c] = r < valid ? g[(size_t)r * gstride + c] : 0.f;
  }
}

template <typename Tin>
__device__ __forceinline__ void ld_rows_in(float* s, int ld, const Tin* g, size_t gstride, int rows,
                                           int valid, int cols) {
  for (int e = threadIdx.x; e < rows * cols; e += kNT) {
    const int r = e / cols, c = e % cols;
    s[r * ld + c] = r < valid ? Elem<Tin>::load(g + (size_t)r * gstride + c) : 0.f;
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
// prep: per (chunk, value head).

template <int DK, int DV>
struct PrepSmem {
  static constexpr int LK = DK + 1, LV = DV + 1;
  static constexpr int oK = 0, oQ = oK + kC * LK, oV = oQ + kC * LK, oA = oV + kC * LV,
                       oT = oA + kC * kLC, oG = oT + kC * kLC, oB = oG + kC, total = oB + kC;
  static constexpr size_t bytes = sizeof(float) * total;
};

// Inclusive cumsum of log alpha and beta over one chunk into sG / sB (warp 0).
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
    if (sB) sB[r] = b;
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
}

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(kNT, 1) bwd_prep_kernel(const BwdArgs a) {
  using L = PrepSmem<DK, DV>;
  extern __shared__ float smem[];
  const ChunkEnt* e;
  if (!chunk_of(a, &e)) return;
  const int h = blockIdx.y, hq = h / (a.H_v / a.H_qk);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, ty = tid / 16, tx = tid % 16;
  float *sK = smem + L::oK, *sQ = smem + L::oQ, *sV = smem + L::oV, *sA = smem + L::oA,
        *sT = smem + L::oT, *sG = smem + L::oG, *sB = smem + L::oB;
  const size_t ch = (size_t)blockIdx.x * a.H_v + h;
  const int n = e->n;
  ld_rows(sK, L::LK, a.kh + ((size_t)e->t0 * a.H_qk + hq) * DK, (size_t)a.H_qk * DK, kC, n, DK);
  ld_rows(sQ, L::LK, a.qh + ((size_t)e->t0 * a.H_qk + hq) * DK, (size_t)a.H_qk * DK, kC, n, DK);
  ld_rows_in(sV, L::LV, static_cast<const Tin*>(a.v) + ((size_t)e->t0 * a.H_v + h) * DV,
             (size_t)a.H_v * DV, kC, n, DV);
  load_gates(a, *e, h, sG, sB);
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
        qt[u] = sQ[(ty + 16 * u) * L::LK + d];
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
  __syncthreads();

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
  __syncthreads();

  // W = T diag(beta gamma) K, U = T diag(beta) V
  {
    constexpr int NK = DK / 16, NV = DV / 16;
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
        const float vv = bi * sV[i * L::LV + tx + 16 * w];
#pragma unroll
        for (int u = 0; u < 4; ++u) uacc[u][w] += tr[u] * vv;
      }
    }
    float* gW = a.W + ch * kC * DK;
    float* gU = a.UT + ch * kC * DV;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = ty + 16 * u;
#pragma unroll
      for (int w = 0; w < NK; ++w) gW[t * DK + tx + 16 * w] = wacc[u][w];
#pragma unroll
      for (int w = 0; w < NV; ++w) gU[t * DV + tx + 16 * w] = uacc[u][w];
    }
  }
  for (int x = tid; x < kC * kC; x += kNT) a.T[ch * kC * kC + x] = sT[(x / kC) * kLC + x % kC];
  if (tid < kC) a.G[ch * kC + tid] = sG[tid];
}

// ---------------------------------------------------------------------------
// fwd_chain: per (sequence, value head, slice of SW state columns).

template <int DV>
struct Slice {
  static constexpr int SW = DV < 32 ? DV : 32;
  static constexpr int NS = DV / SW;
  static constexpr int NW = SW / 16;  // column blocks per thread
};

template <int DK, int DV>
struct FwdChainSmem {
  static constexpr int LK = DK + 1, LS = Slice<DV>::SW + 1;
  static constexpr int oW = 0, oK = oW + kC * LK, oS = oK + kC * LK, oD = oS + DK * LS,
                       oG = oD + kC * LS, total = oG + kC;
  static constexpr size_t bytes = sizeof(float) * total;
};

template <int DK, int DV>
__global__ void __launch_bounds__(kNT, 1) bwd_fwd_chain_kernel(const BwdArgs a) {
  using L = FwdChainSmem<DK, DV>;
  using SL = Slice<DV>;
  constexpr int SW = SL::SW, NW = SL::NW, NK = DK / 16;
  extern __shared__ float smem[];
  float *sW = smem + L::oW, *sK = smem + L::oK, *sS = smem + L::oS, *sD = smem + L::oD,
        *sG = smem + L::oG;
  const int seq = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * SW;
  const int hq = h / (a.H_v / a.H_qk);
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const size_t st = ((size_t)seq * a.H_v + h) * DK * DV;
  for (int x = tid; x < DK * SW; x += kNT) {
    const int i = x / SW, j = x % SW;
    sS[i * L::LS + j] = a.initial_state ? __ldg(a.initial_state + st + (size_t)i * DV + j0 + j) : 0.f;
  }
  const int c_begin = a.seq_first[seq], c_end = a.seq_first[seq + 1];
  const ChunkEnt* ents = reinterpret_cast<const ChunkEnt*>(a.chunks);
  for (int c = c_begin; c < c_end; ++c) {
    const ChunkEnt e = ents[c];
    const size_t ch = (size_t)c * a.H_v + h;
    __syncthreads();  // previous chunk done with sW, sK, sD, sG; sS final
    float* gS = a.S + ch * DK * DV;
    for (int x = tid; x < DK * SW; x += kNT) {
      const int i = x / SW, j = x % SW;
      gS[(size_t)i * DV + j0 + j] = sS[i * L::LS + j];
    }
    ld_rows(sW, L::LK, a.W + ch * kC * DK, DK, kC, kC, DK);
    ld_rows(sK, L::LK, a.kh + ((size_t)e.t0 * a.H_qk + hq) * DK, (size_t)a.H_qk * DK, kC, e.n, DK);
    ld_rows(sD, L::LS, a.UT + ch * kC * DV + j0, DV, kC, kC, SW);
    if (tid < kC) sG[tid] = a.G[ch * kC + tid];
    __syncthreads();
    // Delta = U - W S
    {
      float acc[4][NW];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < NW; ++w) acc[u][w] = sD[(ty + 16 * u) * L::LS + tx + 16 * w];
      for (int i = 0; i < DK; ++i) {
        float sv[NW];
#pragma unroll
        for (int w = 0; w < NW; ++w) sv[w] = sS[i * L::LS + tx + 16 * w];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float wv = sW[(ty + 16 * u) * L::LK + i];
#pragma unroll
          for (int w = 0; w < NW; ++w) acc[u][w] -= wv * sv[w];
        }
      }
      __syncthreads();  // all reads of U done
      float* gD = a.D + ch * kC * DV + j0;
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          const int t = ty + 16 * u, j = tx + 16 * w;
          sD[t * L::LS + j] = acc[u][w];
          gD[(size_t)t * DV + j] = acc[u][w];
        }
    }
    __syncthreads();
    // S <- gamma_C S + (diag(b) K)^T Delta
    {
      const float GC = sG[kC - 1], gC = expf(GC);
      float acc[NK][NW];
#pragma unroll
      for (int u = 0; u < NK; ++u)
#pragma unroll
        for (int w = 0; w < NW; ++w) acc[u][w] = 0.f;
      for (int t = 0; t < kC; ++t) {
        const float bt = expf(GC - sG[t]);
        float dv[NW];
#pragma unroll
        for (int w = 0; w < NW; ++w) dv[w] = sD[t * L::LS + tx + 16 * w];
#pragma unroll
        for (int u = 0; u < NK; ++u) {
          const float kv = bt * sK[t * L::LK + ty + 16 * u];
#pragma unroll
          for (int w = 0; w < NW; ++w) acc[u][w] += kv * dv[w];
        }
      }
#pragma unroll
      for (int u = 0; u < NK; ++u)
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          float* p = sS + (ty + 16 * u) * L::LS + tx + 16 * w;
          *p = gC * *p + acc[u][w];  // each element owned by one thread
        }
    }
  }
}

// ---------------------------------------------------------------------------
// epilogue: per (chunk, value head).  dO = dy without the epilogue; with it,
// O is recomputed and dy is taken back through sigmoid(g), (1 + w) and the
// RMS norm.  Also writes dg and this chunk's share of dw.

template <int DK, int DV>
struct EpiSmem {
  static constexpr int LK = DK + 1, LV = DV + 1;
  static constexpr int oQ = 0, oS = oQ + kC * LK, oP = oS + DK * LV, oD = oP + kC * kLC,
                       oO = oD + kC * LV, oW = oO + kC * LV, oG = oW + (kNT / 32) * DV,
                       total = oG + kC;
  static constexpr size_t bytes = sizeof(float) * total;
};

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(kNT, 1) bwd_epilogue_kernel(const BwdArgs a) {
  using L = EpiSmem<DK, DV>;
  constexpr int NV = DV / 16;
  extern __shared__ float smem[];
  const ChunkEnt* e;
  if (!chunk_of(a, &e)) return;
  const int h = blockIdx.y, hq = h / (a.H_v / a.H_qk);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, ty = tid / 16, tx = tid % 16;
  const size_t ch = (size_t)blockIdx.x * a.H_v + h;
  const int n = e->n;
  const Tin* dY = static_cast<const Tin*>(a.dy);
  if (a.g == nullptr) {
    for (int x = tid; x < n * DV; x += kNT) {
      const size_t off = ((size_t)(e->t0 + x / DV) * a.H_v + h) * DV + x % DV;
      a.dO[off] = Elem<Tin>::load(dY + off);
    }
    return;
  }
  float *sQ = smem + L::oQ, *sS = smem + L::oS, *sP = smem + L::oP, *sD = smem + L::oD,
        *sO = smem + L::oO, *sWp = smem + L::oW, *sG = smem + L::oG;
  ld_rows(sQ, L::LK, a.qh + ((size_t)e->t0 * a.H_qk + hq) * DK, (size_t)a.H_qk * DK, kC, n, DK);
  ld_rows(sS, L::LV, a.S + ch * DK * DV, DV, DK, DK, DV);
  ld_rows(sP, kLC, a.P + ch * kC * kC, kC, kC, kC, kC);
  ld_rows(sD, L::LV, a.D + ch * kC * DV, DV, kC, kC, DV);
  if (tid < kC) sG[tid] = a.G[ch * kC + tid];
  __syncthreads();
  {
    float acc[4][NV], pacc[4][NV];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < NV; ++w) acc[u][w] = pacc[u][w] = 0.f;
    for (int i = 0; i < DK; ++i) {
      float sv[NV];
#pragma unroll
      for (int w = 0; w < NV; ++w) sv[w] = sS[i * L::LV + tx + 16 * w];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float qv = sQ[(ty + 16 * u) * L::LK + i];
#pragma unroll
        for (int w = 0; w < NV; ++w) acc[u][w] += qv * sv[w];
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
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = ty + 16 * u;
      const float sg = a.scale * expf(sG[t]);
#pragma unroll
      for (int w = 0; w < NV; ++w) sO[t * L::LV + tx + 16 * w] = sg * acc[u][w] + pacc[u][w];
    }
  }
  for (int x = tid; x < (kNT / 32) * DV; x += kNT) sWp[x] = 0.f;
  __syncthreads();
  const Tin* Gg = static_cast<const Tin*>(a.g);
  for (int r = warp; r < n; r += kNT / 32) {
    const size_t off = ((size_t)(e->t0 + r) * a.H_v + h) * DV;
    float ss = 0.f;
    for (int j = lane; j < DV; j += 32) ss += sO[r * L::LV + j] * sO[r * L::LV + j];
    ss = warp_sum(ss);
    const float rs = rsqrtf(ss / (float)DV + a.eps_norm);
    float dn[(DV + 31) / 32], nr[(DV + 31) / 32];
    float dot = 0.f;
#pragma unroll
    for (int m = 0; m < (DV + 31) / 32; ++m) {
      const int j = lane + 32 * m;
      dn[m] = nr[m] = 0.f;
      if (j < DV) {
        const float w = a.norm_w ? __ldg(a.norm_w + j) : 0.f;
        const float sg = sigmoidf_(Elem<Tin>::load(Gg + off + j));
        const float nv = sO[r * L::LV + j] * rs;
        const float dyj = Elem<Tin>::load(dY + off + j);
        a.dg[off + j] = dyj * nv * (1.f + w) * sg * (1.f - sg);
        sWp[warp * DV + j] += dyj * nv * sg;
        dn[m] = dyj * (1.f + w) * sg;
        nr[m] = nv;
        dot += dn[m] * nv;
      }
    }
    dot = warp_sum(dot) / (float)DV;
#pragma unroll
    for (int m = 0; m < (DV + 31) / 32; ++m) {
      const int j = lane + 32 * m;
      if (j < DV) a.dO[off + j] = rs * (dn[m] - nr[m] * dot);
    }
  }
  __syncthreads();
  for (int j = tid; j < DV; j += kNT) {
    float s = 0.f;
    for (int w = 0; w < kNT / 32; ++w) s += sWp[w * DV + j];
    a.dw[ch * DV + j] = s;
  }
}

// ---------------------------------------------------------------------------
// bwd_chain: per (sequence, value head, slice of SW state columns), chunks in
// reverse order.

template <int DK, int DV>
struct BwdChainSmem {
  static constexpr int LK = DK + 1, LS = Slice<DV>::SW + 1;
  static constexpr int oP = 0, oK = oP + kC * kLC, oW = oK + kC * LK, oQ = oW + kC * LK,
                       odS = oQ + kC * LK, odY = odS + DK * LS, odD = odY + kC * LS,
                       oG = odD + kC * LS, total = oG + kC;
  static constexpr size_t bytes = sizeof(float) * total;
};

template <int DK, int DV>
__global__ void __launch_bounds__(kNT, 1) bwd_bwd_chain_kernel(const BwdArgs a) {
  using L = BwdChainSmem<DK, DV>;
  using SL = Slice<DV>;
  constexpr int SW = SL::SW, NW = SL::NW, NK = DK / 16;
  extern __shared__ float smem[];
  float *sP = smem + L::oP, *sK = smem + L::oK, *sW = smem + L::oW, *sQ = smem + L::oQ,
        *sdS = smem + L::odS, *sdY = smem + L::odY, *sdD = smem + L::odD, *sG = smem + L::oG;
  const int seq = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * SW;
  const int hq = h / (a.H_v / a.H_qk);
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const size_t st = ((size_t)seq * a.H_v + h) * DK * DV;
  for (int x = tid; x < DK * SW; x += kNT) {
    const int i = x / SW, j = x % SW;
    sdS[i * L::LS + j] =
        a.d_final_state ? __ldg(a.d_final_state + st + (size_t)i * DV + j0 + j) : 0.f;
  }
  const int c_begin = a.seq_first[seq], c_end = a.seq_first[seq + 1];
  const ChunkEnt* ents = reinterpret_cast<const ChunkEnt*>(a.chunks);
  for (int c = c_end - 1; c >= c_begin; --c) {
    const ChunkEnt e = ents[c];
    const size_t ch = (size_t)c * a.H_v + h;
    __syncthreads();
    float* gdS = a.dS + ch * DK * DV;
    for (int x = tid; x < DK * SW; x += kNT) {
      const int i = x / SW, j = x % SW;
      gdS[(size_t)i * DV + j0 + j] = sdS[i * L::LS + j];
    }
    ld_rows(sP, kLC, a.P + ch * kC * kC, kC, kC, kC, kC);
    ld_rows(sK, L::LK, a.kh + ((size_t)e.t0 * a.H_qk + hq) * DK, (size_t)a.H_qk * DK, kC, e.n, DK);
    ld_rows(sW, L::LK, a.W + ch * kC * DK, DK, kC, kC, DK);
    ld_rows(sQ, L::LK, a.qh + ((size_t)e.t0 * a.H_qk + hq) * DK, (size_t)a.H_qk * DK, kC, e.n, DK);
    ld_rows(sdY, L::LS, a.dO + ((size_t)e.t0 * a.H_v + h) * DV + j0, (size_t)a.H_v * DV, kC, e.n,
            SW);
    if (tid < kC) sG[tid] = a.G[ch * kC + tid];
    __syncthreads();
    const float GC = sG[kC - 1];
    // dDelta = P^T dO + diag(b) K dS
    {
      float acc[4][NW], kacc[4][NW];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < NW; ++w) acc[u][w] = kacc[u][w] = 0.f;
      for (int s = 0; s < kC; ++s) {
        float yv[NW];
#pragma unroll
        for (int w = 0; w < NW; ++w) yv[w] = sdY[s * L::LS + tx + 16 * w];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float pv = sP[s * kLC + ty + 16 * u];  // P_{s,t}
#pragma unroll
          for (int w = 0; w < NW; ++w) acc[u][w] += pv * yv[w];
        }
      }
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
      float* gdD = a.dD + ch * kC * DV + j0;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = ty + 16 * u;
        const float bt = expf(GC - sG[t]);
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          const int j = tx + 16 * w;
          const float v = acc[u][w] + bt * kacc[u][w];
          sdD[t * L::LS + j] = v;
          gdD[(size_t)t * DV + j] = v;
        }
      }
    }
    __syncthreads();
    // dS <- gamma_C dS + (diag(gamma) Qs)^T dO - W^T dDelta
    {
      const float gC = expf(GC);
      float acc[NK][NW];
#pragma unroll
      for (int u = 0; u < NK; ++u)
#pragma unroll
        for (int w = 0; w < NW; ++w) acc[u][w] = gC * sdS[(ty + 16 * u) * L::LS + tx + 16 * w];
      for (int t = 0; t < kC; ++t) {
        const float sg = a.scale * expf(sG[t]);
        float yv[NW], dv[NW];
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          yv[w] = sdY[t * L::LS + tx + 16 * w];
          dv[w] = sdD[t * L::LS + tx + 16 * w];
        }
#pragma unroll
        for (int u = 0; u < NK; ++u) {
          const float qv = sg * sQ[t * L::LK + ty + 16 * u];
          const float wv = sW[t * L::LK + ty + 16 * u];
#pragma unroll
          for (int w = 0; w < NW; ++w) acc[u][w] += qv * yv[w] - wv * dv[w];
        }
      }
#pragma unroll
      for (int u = 0; u < NK; ++u)
#pragma unroll
        for (int w = 0; w < NW; ++w) sdS[(ty + 16 * u) * L::LS + tx + 16 * w] = acc[u][w];
    }
  }
  __syncthreads();
  if (a.d_initial_state) {
    for (int x = tid; x < DK * SW; x += kNT) {
      const int i = x / SW, j = x % SW;
      a.d_initial_state[st + (size_t)i * DV + j0 + j] = sdS[i * L::LS + j];
    }
  }
}

// ---------------------------------------------------------------------------
// chunk_a: per (chunk, value head).

template <int DV>
struct ChunkASmem {
  static constexpr int LV = DV + 1;
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
  extern __shared__ float smem[];
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
  ld_rows(sD, L::LV, a.D + ch * kC * DV, DV, kC, kC, DV);
  ld_rows(sdD, L::LV, a.dD + ch * kC * DV, DV, kC, kC, DV);
  ld_rows(sdY, L::LV, a.dO + ((size_t)e->t0 * a.H_v + h) * DV, (size_t)a.H_v * DV, kC, n, DV);
  ld_rows_in(sX, L::LV, static_cast<const Tin*>(a.v) + ((size_t)e->t0 * a.H_v + h) * DV,
             (size_t)a.H_v * DV, kC, n, DV);
  ld_rows(sT, kLC, a.T + ch * kC * kC, kC, kC, kC, kC);
  ld_rows(sKKE, kLC, a.KKE + ch * kC * kC, kC, kC, kC, kC);
  ld_rows(sP, kLC, a.P + ch * kC * kC, kC, kC, kC, kC);
  if (tid < kC) {
    sG[tid] = a.G[ch * kC + tid];
    sB[tid] = tid < n ? __ldg(a.beta + (size_t)(e->t0 + tid) * a.H_v + h) : 0.f;
  }
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
  static constexpr int LK = DK + 1, LV = DV + 1;
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
  extern __shared__ float smem[];
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
    ld_rows(sS, L::LV, a.S + ch * DK * DV, DV, DK, DK, DV);
    ld_rows(sY, L::LV, a.dO + ((size_t)e->t0 * a.H_v + h) * DV, (size_t)a.H_v * DV, kC, n, DV);
    ld_rows(sTd, L::LV, a.UT + ch * kC * DV, DV, kC, kC, DV);
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
    ld_rows(sdS, L::LV, a.dS + ch * DK * DV, DV, DK, DK, DV);
    ld_rows(sDl, L::LV, a.D + ch * kC * DV, DV, kC, kC, DV);
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
  ld_rows(sK, L::LK, a.kh + ((size_t)e->t0 * a.H_qk + hq) * DK, (size_t)a.H_qk * DK, kC, n, DK);
  ld_rows(sQ, L::LK, a.qh + ((size_t)e->t0 * a.H_qk + hq) * DK, (size_t)a.H_qk * DK, kC, n, DK);
  ld_rows(sdPE, kLC, a.dPE + ch * kC * kC, kC, kC, kC, kC);
  ld_rows(sBm, kLC, a.Bm + ch * kC * kC, kC, kC, kC, kC);
  if (tid < kC) {
    sG[tid] = a.G[ch * kC + tid];
    sB[tid] = tid < n ? __ldg(a.beta + (size_t)(e->t0 + tid) * a.H_v + h) : 0.f;
  }
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
  bwd_chunk_table_kernel<<<1, kNT, 0, s>>>(a);
  if (a.total_T > 0) {
    const unsigned rows = (unsigned)((a.total_T * a.H_qk + 7) / 8);
    bwd_normalise_kernel<DK, Tin><<<rows, kNT, 0, s>>>(a);
    auto k1 = bwd_prep_kernel<DK, DV, Tin>;
    if (!set_smem(k1, PrepSmem<DK, DV>::bytes)) return GDN_ERR_CUDA;
    k1<<<dim3((unsigned)maxc, H), kNT, PrepSmem<DK, DV>::bytes, s>>>(a);
    auto k2 = bwd_fwd_chain_kernel<DK, DV>;
    if (!set_smem(k2, FwdChainSmem<DK, DV>::bytes)) return GDN_ERR_CUDA;
    k2<<<dim3((unsigned)a.n_seq, H, Slice<DV>::NS), kNT, FwdChainSmem<DK, DV>::bytes, s>>>(a);
    auto k3 = bwd_epilogue_kernel<DK, DV, Tin>;
    if (!set_smem(k3, EpiSmem<DK, DV>::bytes)) return GDN_ERR_CUDA;
    k3<<<dim3((unsigned)maxc, H), kNT, EpiSmem<DK, DV>::bytes, s>>>(a);
  }
  auto k4 = bwd_bwd_chain_kernel<DK, DV>;
  if (!set_smem(k4, BwdChainSmem<DK, DV>::bytes)) return GDN_ERR_CUDA;
  k4<<<dim3((unsigned)a.n_seq, H, Slice<DV>::NS), kNT, BwdChainSmem<DK, DV>::bytes, s>>>(a);
  if (a.total_T > 0) {
    auto k5 = bwd_chunk_a_kernel<DK, DV, Tin>;
    if (!set_smem(k5, ChunkASmem<DV>::bytes)) return GDN_ERR_CUDA;
    k5<<<dim3((unsigned)maxc, H), kNT, ChunkASmem<DV>::bytes, s>>>(a);
    auto k6 = bwd_chunk_b_kernel<DK, DV>;
    if (!set_smem(k6, ChunkBSmem<DK, DV>::bytes)) return GDN_ERR_CUDA;
    k6<<<dim3((unsigned)maxc, H), kNT, ChunkBSmem<DK, DV>::bytes, s>>>(a);
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
  b += align256(nch * kC * d_k * f);                 // W
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
