// Portable chunked prefill of the gated delta rule on CUDA cores, fp32
// arithmetic throughout.  It serves every supported shape and dtype (the
// fp32-input mode in particular, whose tolerance bf16 tensor-core operands
// cannot meet) and is the kernel the tensor-core path is checked against.
//
// One CTA per (sequence, value head); the fp32 state S (d_k x d_v) lives in
// shared memory for the whole sequence.  Per chunk of C = 64 tokens, with the
// entering state S, G_t = sum_{s<=t} log alpha_s and gamma_t = exp(G_t):
//
//   A_ti  = beta_t exp(G_t - G_i) (k^_t . k^_i),  i < t       (strictly lower)
//   P_ti  = exp(G_t - G_i) (q^_t . k^_i),          i <= t
//   B     = diag(beta) (V - diag(gamma) K^ S)
//   Delta = (I + A)^{-1} B          (forward substitution, no explicit inverse)
//   Y     = scale (diag(gamma) Q^ S + P Delta)
//   S    <- gamma_C S + (diag(exp(G_C - G)) K^)^T Delta
//
// This is the recurrence of "Qwen3.8-Flash-Next: architecture, efficiency and
// technical lineage", section 03 "Gated DeltaNet" (update equations),
// regrouped: Delta_t is the value token t writes (beta_t times its error
// e_t), and the delta-rule coupling between tokens of one chunk is the unit
// lower-triangular system (I + A) Delta = B.  Only decay differences
// G_t - G_i <= 0 are exponentiated, so nothing overflows for any alpha.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kC = 64;     // chunk length
constexpr int kNT = 256;   // threads per CTA

template <int DK, int DV>
struct SimtSmem {
  static constexpr int LK = DK + 1;   // padded row lengths (bank spread)
  static constexpr int LV = DV + 1;
  static constexpr int LC = kC + 1;
  static constexpr int oK = 0;                    // K^  [C][LK]
  static constexpr int oQ = oK + kC * LK;         // Q^  [C][LK]
  static constexpr int oV = oQ + kC * LK;         // V -> B -> Delta [C][LV]
  static constexpr int oY = oV + kC * LV;         // Y   [C][LV]
  static constexpr int oS = oY + kC * LV;         // S   [DK][LV]
  static constexpr int oAP = oS + DK * LV;        // A (upper, transposed) + P (lower)
  static constexpr int oG = oAP + kC * LC;        // G_t
  static constexpr int oB = oG + kC;              // beta_t
  static constexpr int oCS = oB + kC;             // carried conv inputs [3][2 DK + DV]
  static constexpr int total = oCS + 3 * (2 * DK + DV);
  static constexpr size_t bytes = sizeof(float) * total;
};

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(kNT, 1) gdn_prefill_simt_kernel(const PrefillArgs a) {
  using L = SimtSmem<DK, DV>;
  extern __shared__ float smem[];
  float* sK = smem + L::oK;
  float* sQ = smem + L::oQ;
  float* sV = smem + L::oV;
  float* sY = smem + L::oY;
  float* sS = smem + L::oS;
  float* sAP = smem + L::oAP;
  float* sG = smem + L::oG;
  float* sB = smem + L::oB;
  float* sCS = smem + L::oCS;

  const int seq = blockIdx.x / a.H_v;
  const int h = blockIdx.x % a.H_v;
  const int hq = h / (a.H_v / a.H_qk);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int64_t t_begin, t_end;
  if (!seq_bounds(a.cu_seqlens, seq, a.total_T, &t_begin, &t_end, a.err)) return;

  const size_t st_off = ((size_t)seq * a.H_v + h) * (size_t)(DK * DV);
  for (int e = tid; e < DK * DV; e += kNT) {
    const int i = e / DV, j = e % DV;
    sS[i * L::LV + j] = a.initial_state ? __ldg(a.initial_state + st_off + e) : 0.f;
  }

  const Tin* Qg = static_cast<const Tin*>(a.q);
  const Tin* Kg = static_cast<const Tin*>(a.k);
  const Tin* Vg = static_cast<const Tin*>(a.v);
  const Tin* Gg = static_cast<const Tin*>(a.g);
  Tin* Yg = static_cast<Tin*>(a.y);
  const int ty = tid / 16, tx = tid % 16;
  // front end (optional): this value head's carried conv inputs
  constexpr int SROW = 2 * DK + DV;
  const bool conv = a.conv_w != nullptr;
  const size_t cs_off = ((size_t)seq * a.H_v + h) * 3 * SROW;
  if (conv)
    for (int e = tid; e < 3 * SROW; e += kNT)
      sCS[e] = a.conv_state_in ? __ldg(a.conv_state_in + cs_off + e) : 0.f;
  // The input x (raw, before the front end) of channel column `col` of the
  // carried-state row layout at token t, from the tensor (row stride `rs`,
  // column `c`), or from the carried inputs before the sequence's start.
  auto raw = [&](const Tin* X, size_t rs, int c, int col, int64_t t) -> float {
    return t >= t_begin ? Elem<Tin>::load(X + (size_t)t * rs + c)
                        : sCS[(3 - (int)(t_begin - t)) * SROW + col];
  };
  // conv of kernel 4 then SiLU: weights row `wrow` of conv_w
  auto front = [&](const Tin* X, size_t rs, int c, int col, int wrow, int64_t t) -> float {
    const float4 w = __ldg(reinterpret_cast<const float4*>(a.conv_w) + wrow);
    const float u = w.w * raw(X, rs, c, col, t) + w.z * raw(X, rs, c, col, t - 1) +
                    w.y * raw(X, rs, c, col, t - 2) + w.x * raw(X, rs, c, col, t - 3);
    return u / (1.f + __expf(-u));
  };
  if (conv) __syncthreads();  // sCS loaded

  for (int64_t c0 = t_begin; c0 < t_end; c0 += kC) {
    const int n = (t_end - c0) < kC ? (int)(t_end - c0) : kC;
    __syncthreads();  // previous chunk fully consumed
    // ---- 1. load, L2-normalise, gate cumsum -------------------------------
    for (int r = warp; r < kC; r += kNT / 32) {
      float nk = 0.f, nq = 0.f;
      for (int d = lane; d < DK; d += 32) {
        float kv = 0.f, qv = 0.f;
        if (r < n) {
          if (conv) {
            const size_t rs = (size_t)a.H_qk * DK;
            kv = front(Kg, rs, hq * DK + d, DK + d, (a.H_qk + hq) * DK + d, c0 + r);
            qv = front(Qg, rs, hq * DK + d, d, hq * DK + d, c0 + r);
          } else {
            const size_t off = ((size_t)(c0 + r) * a.H_qk + hq) * DK + d;
            kv = Elem<Tin>::load(Kg + off);
            qv = Elem<Tin>::load(Qg + off);
          }
        }
        sK[r * L::LK + d] = kv;
        sQ[r * L::LK + d] = qv;
        nk += kv * kv;
        nq += qv * qv;
      }
      nk = warp_sum(nk);
      nq = warp_sum(nq);
      const float rk = (a.l2norm && r < n) ? rsqrtf(nk + a.eps_l2) : 1.f;
      const float rq = (a.l2norm && r < n) ? rsqrtf(nq + a.eps_l2) : 1.f;
      for (int d = lane; d < DK; d += 32) {
        sK[r * L::LK + d] *= rk;
        sQ[r * L::LK + d] *= rq;
      }
      for (int j = lane; j < DV; j += 32)
        sV[r * L::LV + j] =
            r >= n ? 0.f
            : conv ? front(Vg, (size_t)a.H_v * DV, h * DV + j, 2 * DK + j,
                           2 * a.H_qk * DK + h * DV + j, c0 + r)
                   : Elem<Tin>::load(Vg + ((size_t)(c0 + r) * a.H_v + h) * DV + j);
    }
    if (warp == 0) {
      // inclusive cumsum of log alpha over the chunk (two 32-lane scans)
      float carry = 0.f;
      for (int base = 0; base < kC; base += 32) {
        const int r = base + lane;
        float x = r < n ? __ldg(a.log_alpha + (size_t)(c0 + r) * a.H_v + h) : 0.f;
        const float b = r < n ? __ldg(a.beta + (size_t)(c0 + r) * a.H_v + h) : 0.f;
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
    __syncthreads();

    // ---- 2. A (strictly lower, stored transposed in the upper triangle)
    //         and P (lower incl. diagonal) ------------------------------------
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
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int t = ty + 16 * u, i = tx + 16 * w;
          const float dec = expf(sG[t] - sG[i]);  // only used for i <= t
          if (i < t) sAP[i * L::LC + t] = sB[t] * dec * kk[u][w];
          if (i <= t) sAP[t * L::LC + i] = dec * qk[u][w];
        }
    }

    // ---- 3. B = beta (V - gamma K^ S) in place of V; Y0 = gamma Q^ S -------
    constexpr int NB = (DV + 15) / 16;  // column blocks per thread
    float yacc[4][NB];
    {
      float xs[4][NB];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < NB; ++w) xs[u][w] = yacc[u][w] = 0.f;
      for (int d = 0; d < DK; ++d) {
        float kr[4], qr[4], sv[NB];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          kr[u] = sK[(ty + 16 * u) * L::LK + d];
          qr[u] = sQ[(ty + 16 * u) * L::LK + d];
        }
#pragma unroll
        for (int w = 0; w < NB; ++w) {
          const int j = tx + 16 * w;
          sv[w] = j < DV ? sS[d * L::LV + j] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int w = 0; w < NB; ++w) {
            xs[u][w] += kr[u] * sv[w];
            yacc[u][w] += qr[u] * sv[w];
          }
      }
      __syncthreads();  // every read of V rows done before B overwrites them
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = ty + 16 * u;
        const float gam = expf(sG[t]);
#pragma unroll
        for (int w = 0; w < NB; ++w) {
          const int j = tx + 16 * w;
          if (j < DV) sV[t * L::LV + j] = sB[t] * (sV[t * L::LV + j] - gam * xs[u][w]);
          yacc[u][w] *= gam;
        }
      }
    }
    __syncthreads();

    // ---- 4. (I + A) Delta = B by forward substitution, in place ------------
    // Each warp owns DV/8 columns; LPC lanes share a column and split the
    // sum over earlier rows, so the sequential sweep needs only warp syncs.
    {
      constexpr int CPW = DV / 8 > 0 ? DV / 8 : 1;  // columns per warp
      constexpr int LPC = 32 / CPW;                  // lanes per column
      const int j = warp * CPW + lane / LPC;
      const int p = lane % LPC;
      for (int t = 1; t < kC; ++t) {
        float s = 0.f;
        for (int i = p; i < t; i += LPC) s += sAP[i * L::LC + t] * sV[i * L::LV + j];
#pragma unroll
        for (int o = LPC / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (p == 0) sV[t * L::LV + j] -= s;
        __syncwarp();
      }
    }
    __syncthreads();

    // ---- 5. Y = Y0 + P Delta -> sY -------------------------------------------
    {
      for (int i = 0; i < kC; ++i) {
        float pr[4], dv[NB];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int t = ty + 16 * u;
          pr[u] = i <= t ? sAP[t * L::LC + i] : 0.f;
        }
#pragma unroll
        for (int w = 0; w < NB; ++w) {
          const int j = tx + 16 * w;
          dv[w] = j < DV ? sV[i * L::LV + j] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int w = 0; w < NB; ++w) yacc[u][w] += pr[u] * dv[w];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < NB; ++w) {
          const int j = tx + 16 * w;
          if (j < DV) sY[(ty + 16 * u) * L::LV + j] = a.scale * yacc[u][w];
        }
    }

    // ---- 6. S <- gamma_C S + (diag(exp(G_C - G)) K^)^T Delta ----------------
    {
      const float GC = sG[kC - 1];
      const float gC = expf(GC);
      constexpr int RB = (DK + 15) / 16;
      for (int rb = 0; rb < RB; ++rb) {
        const int i = ty + 16 * rb;
        if (i >= DK) break;
        float acc[NB];
#pragma unroll
        for (int w = 0; w < NB; ++w) acc[w] = 0.f;
        for (int t = 0; t < kC; ++t) {
          const float kd = sK[t * L::LK + i] * expf(GC - sG[t]);
#pragma unroll
          for (int w = 0; w < NB; ++w) {
            const int j = tx + 16 * w;
            if (j < DV) acc[w] += kd * sV[t * L::LV + j];
          }
        }
#pragma unroll
        for (int w = 0; w < NB; ++w) {
          const int j = tx + 16 * w;
          if (j < DV) sS[i * L::LV + j] = gC * sS[i * L::LV + j] + acc[w];
        }
      }
    }
    __syncthreads();

    // ---- 7. epilogue and store y ----------------------------------------------
    for (int r = warp; r < n; r += kNT / 32) {
      const size_t yo = ((size_t)(c0 + r) * a.H_v + h) * DV;
      float rs = 1.f;
      if (Gg != nullptr) {
        float ss = 0.f;
        for (int j = lane; j < DV; j += 32) ss += sY[r * L::LV + j] * sY[r * L::LV + j];
        ss = warp_sum(ss);
        rs = rsqrtf(ss / (float)DV + a.eps_norm);
      }
      for (int j = lane; j < DV; j += 32) {
        float o = sY[r * L::LV + j];
        if (Gg != nullptr) {
          const float w = a.norm_w ? __ldg(a.norm_w + j) : 0.f;
          o = o * rs * (1.f + w) / (1.f + expf(-Elem<Tin>::load(Gg + yo + j)));
        }
        Elem<Tin>::store(Yg + yo + j, o);
      }
    }
  }
  __syncthreads();
  if (conv && a.conv_state_out) {
    // the sequence's last three raw inputs, oldest first (from the carried
    // ones for a sequence shorter than three)
    const int64_t len = t_end - t_begin;
    for (int e = tid; e < 3 * SROW; e += kNT) {
      const int m = e / SROW, col = e % SROW;
      const int64_t t = t_end - 3 + m;
      float x;
      if (t < t_begin) {
        x = sCS[(m + (int)len) * SROW + col];
      } else if (col < DK) {
        x = Elem<Tin>::load(Qg + ((size_t)t * a.H_qk + hq) * DK + col);
      } else if (col < 2 * DK) {
        x = Elem<Tin>::load(Kg + ((size_t)t * a.H_qk + hq) * DK + col - DK);
      } else {
        x = Elem<Tin>::load(Vg + ((size_t)t * a.H_v + h) * DV + col - 2 * DK);
      }
      a.conv_state_out[cs_off + e] = x;
    }
  }
  if (a.final_state) {
    for (int e = tid; e < DK * DV; e += kNT) {
      const int i = e / DV, j = e % DV;
      a.final_state[st_off + e] = sS[i * L::LV + j];
    }
  }
}

template <int DK, int DV, typename Tin>
gdn_status launch(const PrefillArgs& a, cudaStream_t stream) {
  using L = SimtSmem<DK, DV>;
  auto kern = gdn_prefill_simt_kernel<DK, DV, Tin>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes) !=
      cudaSuccess)
    return GDN_ERR_CUDA;
  const unsigned grid = (unsigned)a.n_seq * (unsigned)a.H_v;
  kern<<<grid, kNT, L::bytes, stream>>>(a);
  return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

template <typename Tin>
gdn_status dispatch(const PrefillArgs& a, cudaStream_t s) {
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

gdn_status launch_prefill_simt(const PrefillArgs& a, cudaStream_t stream) {
  if (a.dtype == GDN_BF16) return dispatch<__nv_bfloat16>(a, stream);
  if (a.dtype == GDN_FP32) return dispatch<float>(a, stream);
  return GDN_ERR_UNSUPPORTED;
}

}  // namespace gdn
