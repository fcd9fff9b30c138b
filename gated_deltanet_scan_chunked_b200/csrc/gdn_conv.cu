// Front end of the mixer: short depthwise causal convolution over time
// (kernel 4) followed by SiLU, applied to the q, k and v projections before
// the gated delta rule ("Qwen3.8-Flash-Next: architecture, efficiency and
// technical lineage", section 02 module table, GDN row: Q/K/V pass a short
// causal conv of kernel 4; hyper.ai summary, "Method": projections followed
// by short depthwise causal convolutions; "On the Design of Qwen3.8-Next
// Architecture ... close reading", section 4.1: short conv + SiLU + L2).
//
// Per channel c with weights w[c][0..3] (w[c][3] on the current token):
//   u_t = w3 x_t + w2 x_{t-1} + w1 x_{t-2} + w0 x_{t-3},  out_t = u_t sigmoid(u_t)
// where inputs before a sequence's first token come from its carried conv
// state (or are zero).  Channels are numbered q | k | v: H_qk d_k channels of
// q, then those of k, then H_v d_v of v.
//
// The carried state is kept per value head, [n_seq, H_v, 3, 2 d_k + d_v]:
// value head h holds the last three inputs of its QK head's q and k channels
// and of its own v channels, oldest first.  The q/k part is therefore stored
// once per value head of a group (identical copies); a kernel that owns one
// value head can read and rewrite its own copy in place.
//
// This kernel is HBM-bound: each thread owns 8 consecutive channels over a
// run of 64 tokens, keeps the three previous inputs in registers, and reads
// and writes each element once with 16-byte (fp32: 2 x 16-byte) accesses.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kRun = 64;      // tokens per thread
constexpr int kCh = 8;        // channels per thread
constexpr int kThreads = 128;

template <typename Tin>
struct Vec8;
template <>
struct Vec8<float> {
  static __device__ __forceinline__ void load(const float* p, float* x) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
  static __device__ __forceinline__ void store(float* p, const float* x) {
    reinterpret_cast<float4*>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
  }
};
template <>
struct Vec8<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* x) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* x) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&b);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
};

// Where channel group `cg` (8 channels) lives: tensor, row stride, offset in
// the row, and its place in a value head's carried state.
struct ChanMap {
  int which;      // 0 q, 1 k, 2 v
  int col;        // first channel within the token row of that tensor
  int row_len;    // channels per token of that tensor
  int head;       // QK head (q, k) or value head (v)
  int st_off;     // offset within one value head's state row (2 d_k + d_v)
};

__device__ __forceinline__ ChanMap chan_map(const ConvArgs& a, int c) {
  const int cq = a.H_qk * a.d_k;
  ChanMap m;
  if (c < cq) {
    m.which = 0; m.col = c; m.row_len = cq; m.head = c / a.d_k; m.st_off = c % a.d_k;
  } else if (c < 2 * cq) {
    c -= cq;
    m.which = 1; m.col = c; m.row_len = cq; m.head = c / a.d_k; m.st_off = a.d_k + c % a.d_k;
  } else {
    c -= 2 * cq;
    m.which = 2; m.col = c; m.row_len = a.H_v * a.d_v; m.head = c / a.d_v;
    m.st_off = 2 * a.d_k + c % a.d_v;
  }
  return m;
}

// Sequence containing token t (cu_seqlens non-decreasing; NULL = one sequence).
__device__ __forceinline__ int seq_of(const int32_t* cu, int n_seq, int64_t t) {
  if (cu == nullptr) return 0;
  int lo = 0, hi = n_seq - 1;  // last s with cu[s] <= t, skipping empty sequences
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <typename Tin>
__global__ void __launch_bounds__(kThreads) gdn_conv_kernel(const ConvArgs a) {
  const int ctot = 2 * a.H_qk * a.d_k + a.H_v * a.d_v;
  const int c0 = (blockIdx.y * kThreads + threadIdx.x) * kCh;
  if (c0 >= ctot) return;
  const ChanMap m = chan_map(a, c0);
  const int G = a.H_v / a.H_qk;
  const int srow = 2 * a.d_k + a.d_v;
  const Tin* X = static_cast<const Tin*>(m.which == 0 ? a.q : m.which == 1 ? a.k : a.v);
  Tin* Y = static_cast<Tin*>(m.which == 0 ? a.q_out : m.which == 1 ? a.k_out : a.v_out);
  // the value head whose state copy is read (q/k: the group's first)
  const int hv_read = m.which == 2 ? m.head : m.head * G;
  const int hv_lo = m.which == 2 ? m.head : m.head * G;
  const int hv_hi = m.which == 2 ? m.head + 1 : (m.head + 1) * G;
  float w[4][kCh];
#pragma unroll
  for (int j = 0; j < kCh; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i][j] = __ldg(a.conv_w + (size_t)(c0 + j) * 4 + i);

  // empty sequences: carry the state through unchanged (block column 0 only)
  if (blockIdx.x == 0 && a.state_out != nullptr) {
    for (int s = 0; s < a.n_seq; ++s) {
      int64_t t0, t1;
      if (!seq_bounds(a.cu_seqlens, s, a.total_T, &t0, &t1, nullptr) || t1 != t0) continue;
      for (int hv = hv_lo; hv < hv_hi; ++hv)
        for (int r = 0; r < 3; ++r)
#pragma unroll
          for (int j = 0; j < kCh; ++j) {
            const float v =
                a.state_in ? a.state_in[(((size_t)s * a.H_v + hv_read) * 3 + r) * srow + m.st_off + j]
                           : 0.f;
            a.state_out[(((size_t)s * a.H_v + hv) * 3 + r) * srow + m.st_off + j] = v;
          }
    }
  }

  const int64_t ta = (int64_t)blockIdx.x * kRun;
  if (ta >= a.total_T) return;
  const int64_t tb = ta + kRun < a.total_T ? ta + kRun : a.total_T;
  int s = seq_of(a.cu_seqlens, a.n_seq, ta);
  int64_t s0, s1;
  if (!seq_bounds(a.cu_seqlens, s, a.total_T, &s0, &s1, a.err)) return;
  float xm[3][kCh];  // inputs 3, 2, 1 tokens back
  auto state_val = [&](int seq, int r, int j) -> float {
    return a.state_in
               ? a.state_in[(((size_t)seq * a.H_v + hv_read) * 3 + r) * srow + m.st_off + j]
               : 0.f;
  };
  auto load_window = [&](int64_t t) {
    // the three inputs before token t of sequence s (t in [s0, s1))
#pragma unroll
    for (int back = 3; back >= 1; --back) {
      const int64_t tt = t - back;
      float x[kCh];
      if (tt >= s0) {
        Vec8<Tin>::load(X + (size_t)tt * m.row_len + m.col, x);
      } else {
#pragma unroll
        for (int j = 0; j < kCh; ++j) x[j] = state_val(s, 3 - (int)(s0 - tt), j);
      }
#pragma unroll
      for (int j = 0; j < kCh; ++j) xm[3 - back][j] = x[j];
    }
  };
  load_window(ta);
  for (int64_t t = ta; t < tb; ++t) {
    while (t >= s1) {  // next non-empty sequence
      ++s;
      if (!seq_bounds(a.cu_seqlens, s, a.total_T, &s0, &s1, a.err)) return;
      if (t >= s0 && t < s1) load_window(t);
    }
    float x[kCh], y[kCh];
    Vec8<Tin>::load(X + (size_t)t * m.row_len + m.col, x);
#pragma unroll
    for (int j = 0; j < kCh; ++j) {
      const float u = w[3][j] * x[j] + w[2][j] * xm[2][j] + w[1][j] * xm[1][j] + w[0][j] * xm[0][j];
      y[j] = u / (1.f + __expf(-u));
    }
    Vec8<Tin>::store(Y + (size_t)t * m.row_len + m.col, y);
    if (a.state_out != nullptr) {
      // the last three inputs of the sequence; for a sequence shorter than
      // three, its first token's thread also writes the rows that still
      // come from the previous state
      const int64_t len = s1 - s0;
      if (t >= s1 - 3) {
        const int r = (int)(t - (s1 - 3));
        for (int hv = hv_lo; hv < hv_hi; ++hv)
#pragma unroll
          for (int j = 0; j < kCh; ++j)
            a.state_out[(((size_t)s * a.H_v + hv) * 3 + r) * srow + m.st_off + j] = x[j];
      }
      if (t == s0 && len < 3) {
        for (int r = 0; r < 3 - (int)len; ++r) {
          for (int hv = hv_lo; hv < hv_hi; ++hv)
#pragma unroll
            for (int j = 0; j < kCh; ++j)
              a.state_out[(((size_t)s * a.H_v + hv) * 3 + r) * srow + m.st_off + j] =
                  state_val(s, r + (int)len, j);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kCh; ++j) {
      xm[0][j] = xm[1][j];
      xm[1][j] = xm[2][j];
      xm[2][j] = x[j];
    }
  }
}

}  // namespace

gdn_status launch_conv(const ConvArgs& a, cudaStream_t stream) {
  const int ctot = 2 * a.H_qk * a.d_k + a.H_v * a.d_v;
  const unsigned gy = (unsigned)((ctot / kCh + kThreads - 1) / kThreads);
  const int64_t runs = (a.total_T + kRun - 1) / kRun;
  const unsigned gx = (unsigned)(runs > 0 ? runs : 1);  // one column also carries empty sequences
  if (a.dtype == GDN_BF16)
    gdn_conv_kernel<__nv_bfloat16><<<dim3(gx, gy), kThreads, 0, stream>>>(a);
  else if (a.dtype == GDN_FP32)
    gdn_conv_kernel<float><<<dim3(gx, gy), kThreads, 0, stream>>>(a);
  else
    return GDN_ERR_UNSUPPORTED;
  return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn
