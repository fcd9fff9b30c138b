// Single-token decode step of the gated delta rule, one CTA per (sequence,
// value head).  The step is bound by HBM: the d_k x d_v fp32 state is read
// once and written once; everything else is a few KB.
//
// With S the state before the step, k^ and q^ the L2-normalised key/query,
// the error form of the rule ("Qwen3.8-Flash-Next: architecture, efficiency
// and technical lineage", section 03 "Gated DeltaNet", update equations)
// gives, with a = S^T k^ and b = S^T q^ (one pass over S for both):
//   e   = v - alpha a
//   S'  = alpha S + beta k^ e^T
//   y   = S'^T q^ = alpha b + beta (k^ . q^) e        (times `scale`)
// so the state is loaded into registers, reduced once over d_k, updated and
// stored back, with no second read.  Several tokens of one sequence (for
// speculative verification) run in one launch of the multi-token kernel,
// whose persistent CTAs loop over the (sequence, value head) items: the
// state stays in registers from token to token, is read once (streamed into
// shared memory while the previous item runs) and written once, and may be
// snapshotted after every token.
//
// Thread layout (d_k = d_v = 128, 256 threads): thread (rg, c4) owns columns
// 4*c4 .. 4*c4+3 (one float4) of rows rg, rg+8, ..., rg+120; a warp reads one
// whole 512-byte row per load instruction, so every access is a coalesced
// 128-bit load or store.
#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_sm100.cuh"

namespace gdn {
namespace {

template <int DK, int DV>
struct DecodeGeom {
  static constexpr int TPR = DV / 4;  // threads per state row (float4 each)
  static constexpr int NT_RAW = DK * DV / 16;
  static constexpr int NT = NT_RAW < 32 ? 32 : (NT_RAW > 256 ? 256 : NT_RAW);
  static constexpr int ROWG = NT / TPR;  // row groups
  static constexpr int RPT = DK / ROWG;  // rows per thread
  static_assert(NT % TPR == 0 && DK % ROWG == 0 && RPT >= 1, "bad decode geometry");
};

// The per-row arithmetic both kernels share (so that T_s steps of the
// multi-token kernel equal T_s single steps bit for bit), on column pairs
// with the packed fp32 instructions.
// a and b partial sums over one state row i: pa += S_i k^_i, pb += S_i q^_i.
__device__ __forceinline__ void row_partials(const float4& s, float ki, float qi, uint64_t* pa,
                                             uint64_t* pb) {
  const uint64_t s0 = f2_pack(s.x, s.y), s1 = f2_pack(s.z, s.w);
  const uint64_t k2 = f2_pack(ki, ki), q2 = f2_pack(qi, qi);
  pa[0] = f2_fma(s0, k2, pa[0]);
  pa[1] = f2_fma(s1, k2, pa[1]);
  pb[0] = f2_fma(s0, q2, pb[0]);
  pb[1] = f2_fma(s1, q2, pb[1]);
}
__device__ __forceinline__ float4 f2_to_float4(const uint64_t* p) {
  float4 r;
  f2_unpack(p[0], r.x, r.y);
  f2_unpack(p[1], r.z, r.w);
  return r;
}
// Sum over the row groups of one array of partial sums (in row-group order).
template <int ROWG, int TPR>
__device__ __forceinline__ float4 col_sum(const float4 (*red)[TPR], int c4) {
  uint64_t sa[2] = {0ull, 0ull};
#pragma unroll
  for (int g2 = 0; g2 < ROWG; ++g2) {
    const float4 x = red[g2][c4];
    sa[0] = f2_add(sa[0], f2_pack(x.x, x.y));
    sa[1] = f2_add(sa[1], f2_pack(x.z, x.w));
  }
  return f2_to_float4(sa);
}
// Sum over the row groups of their partial sums (in row-group order).
template <int ROWG, int TPR>
__device__ __forceinline__ void col_sums(const float4 (*red_a)[TPR], const float4 (*red_b)[TPR],
                                         int c4, float4* ta, float4* tb) {
  uint64_t sa[2] = {0ull, 0ull}, sb[2] = {0ull, 0ull};
#pragma unroll
  for (int g2 = 0; g2 < ROWG; ++g2) {
    const float4 x = red_a[g2][c4], z = red_b[g2][c4];
    sa[0] = f2_add(sa[0], f2_pack(x.x, x.y));
    sa[1] = f2_add(sa[1], f2_pack(x.z, x.w));
    sb[0] = f2_add(sb[0], f2_pack(z.x, z.y));
    sb[1] = f2_add(sb[1], f2_pack(z.z, z.w));
  }
  *ta = f2_to_float4(sa);
  *tb = f2_to_float4(sb);
}
// One state row after the step: alpha S_i + (beta k^_i) e, per column
// fma(beta k^_i, e, alpha S_i) with the product alpha S_i rounded first.
__device__ __forceinline__ float4 row_update(const float4& s, uint64_t alpha2, float bk,
                                             const uint64_t* e2) {
  const uint64_t b2 = f2_pack(bk, bk);
  uint64_t o[2];
  o[0] = f2_fma(b2, e2[0], f2_mul(alpha2, f2_pack(s.x, s.y)));
  o[1] = f2_fma(b2, e2[1], f2_mul(alpha2, f2_pack(s.z, s.w)));
  return f2_to_float4(o);
}

// e = v - alpha a, and y = scale (alpha b + (beta k^.q^) e), with every
// rounding written out, so that both kernels compute them alike wherever the
// code stands.
__device__ __forceinline__ float4 err4(const float4& v, float alpha, const float4& ta) {
  return make_float4(__fmaf_rn(-alpha, ta.x, v.x), __fmaf_rn(-alpha, ta.y, v.y),
                     __fmaf_rn(-alpha, ta.z, v.z), __fmaf_rn(-alpha, ta.w, v.w));
}
__device__ __forceinline__ float4 out4(float scale, float alpha, const float4& tb, float bkq,
                                       const float4& e) {
  return make_float4(__fmul_rn(scale, __fmaf_rn(alpha, tb.x, __fmul_rn(bkq, e.x))),
                     __fmul_rn(scale, __fmaf_rn(alpha, tb.y, __fmul_rn(bkq, e.y))),
                     __fmul_rn(scale, __fmaf_rn(alpha, tb.z, __fmul_rn(bkq, e.z))),
                     __fmul_rn(scale, __fmaf_rn(alpha, tb.w, __fmul_rn(bkq, e.w))));
}
// This thread's share of sum(y^2) over a row.
__device__ __forceinline__ float sq4(const float4& y) {
  return __fmaf_rn(y.w, y.w, __fmaf_rn(y.z, y.z, __fmaf_rn(y.y, y.y, __fmul_rn(y.x, y.x))));
}

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(DecodeGeom<DK, DV>::NT)
    gdn_decode_kernel(const DecodeArgs a) {
  using Geo = DecodeGeom<DK, DV>;
  constexpr int TPR = Geo::TPR, ROWG = Geo::ROWG, RPT = Geo::RPT;
  __shared__ float sq[DK], sk[DK];
  __shared__ float4 red_a[ROWG][TPR], red_b[ROWG][TPR];
  __shared__ float snorm[3];

  const int n = blockIdx.x / a.H_v;
  const int h = blockIdx.x % a.H_v;
  const int hq = h / (a.H_v / a.H_qk);
  const int tid = threadIdx.x;
  const int rg = tid / TPR, c4 = tid % TPR;

  // one token, state updated in place (state_out == state_in)
  float* S = a.state_out + ((size_t)n * a.H_v + h) * (size_t)(DK * DV);
  // issue every state load first: they are the whole cost of the step
  float4 s[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int i = rg + ROWG * r;
    s[r] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)i * DV) + c4);
  }
  const Tin* qp = static_cast<const Tin*>(a.q) + ((size_t)n * a.H_qk + hq) * DK;
  const Tin* kp = static_cast<const Tin*>(a.k) + ((size_t)n * a.H_qk + hq) * DK;
  for (int i = tid; i < DK; i += Geo::NT) {
    sq[i] = Elem<Tin>::load(qp + i);
    sk[i] = Elem<Tin>::load(kp + i);
  }
  const float4 v4 =
      Elem<Tin>::load4(static_cast<const Tin*>(a.v) + ((size_t)n * a.H_v + h) * DV + 4 * c4);
  const float alpha = __expf(__ldg(a.log_alpha + (size_t)n * a.H_v + h));
  const float beta = __ldg(a.beta + (size_t)n * a.H_v + h);
  __syncthreads();
  if (tid < 32) {
    float nq = 0.f, nk = 0.f, kq = 0.f;
    for (int i = tid; i < DK; i += 32) {
      nq += sq[i] * sq[i];
      nk += sk[i] * sk[i];
      kq += sk[i] * sq[i];
    }
    nq = warp_sum(nq);
    nk = warp_sum(nk);
    kq = warp_sum(kq);
    if (tid == 0) {
      const float rq = a.l2norm ? rsqrtf(nq + a.eps_l2) : 1.f;
      const float rk = a.l2norm ? rsqrtf(nk + a.eps_l2) : 1.f;
      snorm[0] = rq;
      snorm[1] = rk;
      snorm[2] = kq * rq * rk;
    }
  }
  __syncthreads();
  const float rq = snorm[0], rk = snorm[1], kq = snorm[2];

  // a = S^T k^, b = S^T q^ over this thread's rows, then across row groups
  uint64_t pa[2] = {0ull, 0ull}, pb[2] = {0ull, 0ull};
  float kk[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int i = rg + ROWG * r;
    const float ki = sk[i] * rk, qi = sq[i] * rq;
    kk[r] = ki;
    row_partials(s[r], ki, qi, pa, pb);
  }
  red_a[rg][c4] = f2_to_float4(pa);
  red_b[rg][c4] = f2_to_float4(pb);
  __syncthreads();
  float4 ta, tb;
  col_sums<ROWG, TPR>(red_a, red_b, c4, &ta, &tb);
  const float4 e = err4(v4, alpha, ta);

  // S' = alpha S + beta k^ e^T, stored in place (each thread rewrites
  // exactly the elements it loaded)
  const uint64_t alpha2 = f2_pack(alpha, alpha);
  const uint64_t e2[2] = {f2_pack(e.x, e.y), f2_pack(e.z, e.w)};
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int i = rg + ROWG * r;
    const float4 o = row_update(s[r], alpha2, beta * kk[r], e2);
    __stcs(reinterpret_cast<float4*>(S + (size_t)i * DV) + c4, o);
  }

  // y = scale (alpha b + beta (k^.q^) e), then the optional epilogue
  const float bkq = __fmul_rn(beta, kq);
  float4 y = out4(a.scale, alpha, tb, bkq, e);
  const size_t yo = ((size_t)n * a.H_v + h) * DV + 4 * c4;
  if (a.g != nullptr) {
    float ss = sq4(y);
    ss = group_sum<TPR>(ss);  // every row group holds the same y
    const float r = rsqrtf(__fadd_rn(__fmul_rn(ss, 1.f / (float)DV), a.eps_norm));
    const float4 g4 = Elem<Tin>::load4(static_cast<const Tin*>(a.g) + yo);
    float4 w4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (a.norm_w) w4 = __ldg(reinterpret_cast<const float4*>(a.norm_w + 4 * c4));
    y.x = y.x * r * (1.f + w4.x) * sigmoidf_(g4.x);
    y.y = y.y * r * (1.f + w4.y) * sigmoidf_(g4.y);
    y.z = y.z * r * (1.f + w4.z) * sigmoidf_(g4.z);
    y.w = y.w * r * (1.f + w4.w) * sigmoidf_(g4.w);
  }
  if (rg == 0) Elem<Tin>::store4(static_cast<Tin*>(a.y) + yo, y);
}

// a.T_s tokens per sequence, the state in registers from token to token,
// stored to state_out after the last token and optionally snapshotted after
// every token.  The CTAs are persistent: each takes (sequence, value head)
// items blockIdx.x, blockIdx.x + gridDim.x, ..., and while it runs the tokens
// of one item the state and the raw inputs of its next item are already on
// their way into shared memory (16-byte asynchronous copies; every thread
// copies exactly the state elements it will read, so no barrier guards that
// buffer).  All tokens' inputs (q, k, v, g, gates) are staged in shared
// memory per item, and the q/k norms and k^ . q^ of every token are taken
// once per item (one warp per token).  Per token there is then a single
// block barrier (the cross-warp reduction, double buffered by token parity);
// every thread sums the partials of a = S^T k^ (its update needs them),
// warp 0 alone those of b = S^T q^, from which it forms y and the epilogue.
template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(DecodeGeom<DK, DV>::NT, 2)
    gdn_decode_multi_kernel(const DecodeArgs a) {
  using Geo = DecodeGeom<DK, DV>;
  constexpr int TPR = Geo::TPR, ROWG = Geo::ROWG, RPT = Geo::RPT, NT = Geo::NT;
  extern __shared__ float4 dsm4[];
  __shared__ float4 red_a[2][ROWG][TPR], red_b[2][ROWG][TPR];

  const int tid = threadIdx.x, lane = tid & 31;
  const int rg = tid / TPR, c4 = tid % TPR;
  const bool has_g = a.g != nullptr;
  const int T_s = a.T_s;
  // the next item's state [DK][DV] (16-byte aligned at the start), then the
  // staged inputs, fp32: q, k [T_s][DK]; v, g [T_s][DV]; log alpha, beta,
  // k^ . q^ [T_s]
  float4* sst = dsm4;
  float* tq = reinterpret_cast<float*>(dsm4) + DK * DV;
  float* tk = tq + T_s * DK;
  float* tv = tk + T_s * DK;
  float* tg = tv + T_s * DV;
  float* tla = tg + (has_g ? T_s * DV : 0);
  float* tb = tla + T_s;
  float* tkq = tb + T_s;  // k^ . q^ per token
  // the next item's raw inputs as they are in memory (copied while the
  // current item runs): q, k [T_s][DK]; v, g [T_s][DV]; log alpha, beta [T_s]
  constexpr int VE = 16 / (int)sizeof(Tin);  // elements per 16-byte copy
  Tin* rq = reinterpret_cast<Tin*>(
      reinterpret_cast<uintptr_t>(tkq + T_s + 3) & ~(uintptr_t)15);  // 16-byte aligned
  Tin* rk = rq + T_s * DK;
  Tin* rv = rk + T_s * DK;
  Tin* rgt = rv + T_s * DV;
  float* rla = reinterpret_cast<float*>(rgt + (has_g ? T_s * DV : 0));
  float* rbe = rla + T_s;

  const int items = a.N * a.H_v;
  // this thread's elements of an item's state into the buffer
  auto prefetch_state = [&](int it) {
    const float* Sin = a.state_in + (size_t)it * (DK * DV);
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const int i = rg + ROWG * r;
      sm100::cp_async16(sm100::smem_u32(sst + i * TPR + c4), Sin + (size_t)i * DV + 4 * c4, true);
    }
    sm100::cp_async_commit();
  };
  auto prefetch_inputs = [&](int it) {
    const int n = it / a.H_v, h = it % a.H_v, hq = h / (a.H_v / a.H_qk);
    const Tin* Q = static_cast<const Tin*>(a.q);
    const Tin* K = static_cast<const Tin*>(a.k);
    const Tin* V = static_cast<const Tin*>(a.v);
    const Tin* G = static_cast<const Tin*>(a.g);
    for (int i = tid; i < T_s * (DK / VE); i += NT) {
      const int t = i / (DK / VE), col = (i % (DK / VE)) * VE;
      const size_t tok = (size_t)n * T_s + t;
      sm100::cp_async16(sm100::smem_u32(rq + t * DK + col), Q + (tok * a.H_qk + hq) * DK + col, true);
      sm100::cp_async16(sm100::smem_u32(rk + t * DK + col), K + (tok * a.H_qk + hq) * DK + col, true);
    }
    for (int i = tid; i < T_s * (DV / VE); i += NT) {
      const int t = i / (DV / VE), col = (i % (DV / VE)) * VE;
      const size_t tok = (size_t)n * T_s + t;
      sm100::cp_async16(sm100::smem_u32(rv + t * DV + col), V + (tok * a.H_v + h) * DV + col, true);
      if (has_g)
        sm100::cp_async16(sm100::smem_u32(rgt + t * DV + col), G + (tok * a.H_v + h) * DV + col,
                          true);
    }
    for (int i = tid; i < T_s; i += NT) {
      const size_t tok = (size_t)n * T_s + i;
      sm100::cp_async4(sm100::smem_u32(rla + i), a.log_alpha + tok * a.H_v + h, true);
      sm100::cp_async4(sm100::smem_u32(rbe + i), a.beta + tok * a.H_v + h, true);
    }
    sm100::cp_async_commit();
  };
  auto to_f = [](Tin x) -> float {
    if constexpr (sizeof(Tin) == 4) {
      return (float)x;
    } else {
      return __bfloat162float(x);
    }
  };
  if ((int)blockIdx.x < items) {
    prefetch_state(blockIdx.x);
    prefetch_inputs(blockIdx.x);
  }
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int n = item / a.H_v;
    const int h = item % a.H_v;
    const int hq = h / (a.H_v / a.H_qk);
    const size_t so = (size_t)item * (size_t)(DK * DV);
    // front end: this thread's channels' conv weights and carried inputs,
    // fetched together with the state
    constexpr int SROW = 2 * DK + DV;
    constexpr int CPT = (SROW + NT - 1) / NT;  // channels per thread
    float4 cwr[CPT];
    float cxr[CPT][3];
    float* cst = (a.conv_w && a.conv_state) ? a.conv_state + ((size_t)n * a.H_v + h) * 3 * SROW
                                            : nullptr;
    if (a.conv_w != nullptr) {
#pragma unroll
      for (int u = 0; u < CPT; ++u) {
        const int c = tid + u * NT;
        if (c < SROW) {
          const int wrow = c < DK ? hq * DK + c
                           : c < 2 * DK ? (a.H_qk + hq) * DK + (c - DK)
                                        : 2 * a.H_qk * DK + h * DV + (c - 2 * DK);
          cwr[u] = __ldg(reinterpret_cast<const float4*>(a.conv_w) + wrow);
#pragma unroll
          for (int r = 0; r < 3; ++r) cxr[u][r] = cst ? cst[r * SROW + c] : 0.f;
        }
      }
    }
    float4 w4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (has_g && a.norm_w) w4 = __ldg(reinterpret_cast<const float4*>(a.norm_w + 4 * c4));
    // this item's state and raw inputs (their copies have landed): the state
    // into registers, the inputs to fp32, then the next item's copies into
    // the same buffers
    sm100::cp_async_wait_all();
    __syncthreads();  // every thread's copies of the raw inputs have landed
    for (int i = tid; i < T_s * DK; i += NT) {
      tq[i] = to_f(rq[i]);
      tk[i] = to_f(rk[i]);
    }
    for (int i = tid; i < T_s * DV; i += NT) {
      tv[i] = to_f(rv[i]);
      if (has_g) tg[i] = to_f(rgt[i]);
    }
    for (int i = tid; i < T_s; i += NT) {
      tla[i] = rla[i];
      tb[i] = rbe[i];
    }
    __syncthreads();  // the raw buffers are read before the next item's copies
    float4 s[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) s[r] = sst[(rg + ROWG * r) * TPR + c4];
    if (item + (int)gridDim.x < items) {
      prefetch_state(item + gridDim.x);
      prefetch_inputs(item + gridDim.x);
    }
    if (a.conv_w != nullptr) {
      // front end: causal depthwise conv of kernel 4, then SiLU, over each
      // q / k / v channel of this (sequence, value head), in place on the
      // staged inputs; the three inputs before the first token come from this
      // value head's conv state, which is then rewritten with the last three
      __syncthreads();  // raw inputs staged
#pragma unroll
      for (int u = 0; u < CPT; ++u) {
        const int c = tid + u * NT;
        if (c >= SROW) break;
        float* col = c < DK ? tq + c : c < 2 * DK ? tk + (c - DK) : tv + (c - 2 * DK);
        const int stride = c < 2 * DK ? DK : DV;
        const float4 cw = cwr[u];
        float x3 = cxr[u][0], x2 = cxr[u][1], x1 = cxr[u][2];  // inputs 3, 2, 1 tokens back
        for (int t = 0; t < T_s; ++t) {
          const float x = col[t * stride];
          const float uu = cw.w * x + cw.z * x1 + cw.y * x2 + cw.x * x3;
          col[t * stride] = silu_approx(uu);
          x3 = x2;
          x2 = x1;
          x1 = x;
        }
        if (cst) {
          cst[c] = x3;
          cst[SROW + c] = x2;
          cst[2 * SROW + c] = x1;
        }
      }
    }
    __syncthreads();
    // once per token: the q/k norms and k^ . q^ (one warp per token, with the
    // single-token kernel's lane partition and order), then q and k
    // normalised in place
    for (int t = tid >> 5; t < T_s; t += NT / 32) {
      float* sq = tq + t * DK;
      float* sk = tk + t * DK;
      float nq = 0.f, nk = 0.f, kq = 0.f;
      for (int i = lane; i < DK; i += 32) {
        nq += sq[i] * sq[i];
        nk += sk[i] * sk[i];
        kq += sk[i] * sq[i];
      }
      nq = warp_sum(nq);
      nk = warp_sum(nk);
      kq = warp_sum(kq);
      const float rq = a.l2norm ? rsqrtf(nq + a.eps_l2) : 1.f;
      const float rk = a.l2norm ? rsqrtf(nk + a.eps_l2) : 1.f;
      if (lane == 0) tkq[t] = kq * rq * rk;  // the same association as the single-token kernel
      __syncwarp();
      for (int i = lane; i < DK; i += 32) {
        sq[i] *= rq;
        sk[i] *= rk;
      }
    }
    __syncthreads();

    for (int t = 0; t < T_s; ++t) {
      const int par = t & 1;
      const float* sq = tq + t * DK;  // q^
      const float* sk = tk + t * DK;  // k^
      const float alpha = __expf(tla[t]);
      const float beta = tb[t];
      const float kq = tkq[t];

      // a = S^T k^, b = S^T q^ over this thread's rows, then across row groups
      uint64_t pa[2] = {0ull, 0ull}, pb[2] = {0ull, 0ull};
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        const int i = rg + ROWG * r;
        row_partials(s[r], sk[i], sq[i], pa, pb);
      }
      red_a[par][rg][c4] = f2_to_float4(pa);
      red_b[par][rg][c4] = f2_to_float4(pb);
      __syncthreads();  // (the other parity's buffers were read before this barrier)
      // a for every thread (its rows' update); b only for warp 0, which forms y
      const float4 ta = col_sum<ROWG, TPR>(red_a[par], c4);
      const float4 v4 = *reinterpret_cast<const float4*>(tv + t * DV + 4 * c4);
      const float4 e = err4(v4, alpha, ta);

      // S' = alpha S + beta k^ e^T (each thread updates exactly the elements it
      // loaded), kept in registers, optionally snapshotted, stored to
      // state_out after the last token
      float* snap = a.snapshots ? a.snapshots + ((size_t)t * a.N * a.H_v) * (size_t)(DK * DV) + so
                                : nullptr;
      float* sout = (t + 1 == T_s && a.state_out) ? a.state_out + so : nullptr;
      const uint64_t alpha2 = f2_pack(alpha, alpha);
      const uint64_t e2[2] = {f2_pack(e.x, e.y), f2_pack(e.z, e.w)};
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        const int i = rg + ROWG * r;
        // k^_i again (not held across the reduction)
        const float4 o = row_update(s[r], alpha2, beta * sk[i], e2);
        s[r] = o;
        if (snap) __stcs(reinterpret_cast<float4*>(snap + (size_t)i * DV) + c4, o);
        if (sout) __stcs(reinterpret_cast<float4*>(sout + (size_t)i * DV) + c4, o);
      }

      // y = scale (alpha b + beta (k^.q^) e), then the optional epilogue: every
      // row group holds the same column sums, so warp 0 alone forms y (its row
      // groups in full, for the lane-group sum) and row group 0 stores it
      if (tid < 32) {
        const float4 tbv = col_sum<ROWG, TPR>(red_b[par], c4);
        const size_t tok = (size_t)n * T_s + t;
        const float bkq = __fmul_rn(beta, kq);
        float4 y = out4(a.scale, alpha, tbv, bkq, e);
        const size_t yo = (tok * a.H_v + h) * DV + 4 * c4;
        if (has_g) {
          float ss = sq4(y);
          ss = group_sum<TPR>(ss);
          const float r = rsqrtf(__fadd_rn(__fmul_rn(ss, 1.f / (float)DV), a.eps_norm));
          const float4 g4 = *reinterpret_cast<const float4*>(tg + t * DV + 4 * c4);
          y.x = y.x * r * (1.f + w4.x) * sigmoidf_(g4.x);
          y.y = y.y * r * (1.f + w4.y) * sigmoidf_(g4.y);
          y.z = y.z * r * (1.f + w4.z) * sigmoidf_(g4.z);
          y.w = y.w * r * (1.f + w4.w) * sigmoidf_(g4.w);
        }
        if (rg == 0) Elem<Tin>::store4(static_cast<Tin*>(a.y) + yo, y);
      }
    }  // tokens
    __syncthreads();  // the staged inputs and the reduction buffers are refilled for the next item
  }  // items
}

// Dynamic shared memory of the multi-token kernel for T_s tokens.
template <int DK, int DV>
size_t multi_smem_bytes(int T_s, bool has_g) {
  // state, fp32 inputs and scalars, then the raw next-item inputs (16-byte
  // aligned, at most 4 B of input per element) and their scalars
  return sizeof(float) * ((size_t)DK * DV + (size_t)T_s * (2 * DK + (has_g ? 2 : 1) * DV + 3) + 4) +
         (size_t)T_s * (2 * DK + (has_g ? 2 : 1) * DV) * 4 + (size_t)T_s * 8 + 16;
}

template <int DK, int DV, typename Tin>
gdn_status launch(const DecodeArgs& a, cudaStream_t stream) {
  const unsigned grid = (unsigned)a.N * (unsigned)a.H_v;
  const bool single = a.T_s == 1 && a.snapshots == nullptr && a.state_out == a.state_in &&
                      a.conv_w == nullptr;
  if (single)
    gdn_decode_kernel<DK, DV, Tin><<<grid, DecodeGeom<DK, DV>::NT, 0, stream>>>(a);
  else {
    const size_t smem = multi_smem_bytes<DK, DV>(a.T_s, a.g != nullptr);
    if (smem > 48 * 1024) {
      // more than the default allowance: opt in (per device, once)
      static bool opted[64] = {false};
      int dev = 0;
      if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
      if (dev < 0 || dev >= 64 || !opted[dev]) {
        if (cudaFuncSetAttribute(gdn_decode_multi_kernel<DK, DV, Tin>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)multi_smem_bytes<DK, DV>(kMaxDecodeTokens, true)) !=
            cudaSuccess)
          return GDN_ERR_CUDA;
        if (dev >= 0 && dev < 64) opted[dev] = true;
      }
    }
    // persistent CTAs: as many as can be resident at once (at most one per item)
    auto fn = gdn_decode_multi_kernel<DK, DV, Tin>;
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, DecodeGeom<DK, DV>::NT, smem) !=
            cudaSuccess)
      return GDN_ERR_CUDA;
    const unsigned cap = (unsigned)(per_sm > 0 ? per_sm : 1) * (unsigned)sms;
    fn<<<grid < cap ? grid : cap, DecodeGeom<DK, DV>::NT, smem, stream>>>(a);
  }
  return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

template <typename Tin>
gdn_status dispatch_dv(const DecodeArgs& a, cudaStream_t s) {
#define GDN_DV_CASES(DK)                                     \
  switch (a.d_v) {                                           \
    case 16: return launch<DK, 16, Tin>(a, s);               \
    case 32: return launch<DK, 32, Tin>(a, s);               \
    case 64: return launch<DK, 64, Tin>(a, s);               \
    case 128: return launch<DK, 128, Tin>(a, s);             \
    default: return GDN_ERR_UNSUPPORTED;                     \
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

gdn_status launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  if (a.N == 0 || a.T_s == 0) return GDN_OK;
  if (a.dtype == GDN_BF16) return dispatch_dv<__nv_bfloat16>(a, stream);
  if (a.dtype == GDN_FP32) return dispatch_dv<float>(a, stream);
  return GDN_ERR_UNSUPPORTED;
}

}  // namespace gdn
