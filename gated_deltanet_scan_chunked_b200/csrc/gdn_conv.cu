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
// This kernel is HBM-bound: a CTA stages the inputs of 256 channels x (64 + 3)
// tokens (bf16; 32 + 3 for fp32) in shared memory with 16-byte asynchronous
// copies, then each thread computes 8 consecutive channels of 8 (fp32: 4)
// consecutive tokens and writes them with 16-byte stores.
#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_sm100.cuh"

namespace gdn {
namespace {

constexpr int kCh = 8;        // channels per thread
constexpr int kLanes = 32;    // threads along the channels (256 channels)
constexpr int kTok = 8;       // thread rows per CTA
constexpr int kThreads = kLanes * kTok;
// consecutive tokens per thread (the CTA's input tile stays under 48 KB)
template <typename Tin>
struct Tpt { static constexpr int n = sizeof(Tin) == 2 ? 8 : 4; };

template <typename Tin>
struct Vec8;
template <>
struct Vec8<float> {
  static __device__ __forceinline__ void load_shared(const float* p, float* x) {
    const float4 a = reinterpret_cast<const float4*>(p)[0];
    const float4 b = reinterpret_cast<const float4*>(p)[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
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
  static __device__ __forceinline__ void load_shared(const __nv_bfloat16* p, float* x) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
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
__global__ void __launch_bounds__(kThreads, 3) gdn_conv_kernel(const ConvArgs a) {
  constexpr int kTPT = Tpt<Tin>::n;
  constexpr int kRows = kTok * kTPT + 3;                // the CTA's tokens and the 3 before
  constexpr int kChunks = kLanes * kCh * sizeof(Tin) / 16;  // 16-byte pieces per row
  constexpr int kPer = 16 / sizeof(Tin);                // channels per piece
  static_assert(kThreads % kChunks == 0, "a thread's pieces share one column");
  __shared__ float4 sw[kLanes * kCh];                   // weights (w0, w1, w2, w3)
  __shared__ __align__(16) Tin tile[kRows][kLanes * kCh];
  const int ctot = 2 * a.H_qk * a.d_k + a.H_v * a.d_v;
  const int cb = blockIdx.y * kLanes * kCh;
  const int64_t tb = (int64_t)blockIdx.x * kTok * kTPT;
  // every input the CTA needs, asynchronously (rows outside [0, total_T) and
  // channels past the end are zero); a thread copies one 16-byte column
  {
    const int q = threadIdx.x % kChunks;
    const int c = cb + q * kPer;
    const Tin* col = static_cast<const Tin*>(a.q);
    size_t rl = 0;
    if (c < ctot) {
      const ChanMap mm = chan_map(a, c);
      col = static_cast<const Tin*>(mm.which == 0 ? a.q : mm.which == 1 ? a.k : a.v) + mm.col;
      rl = (size_t)mm.row_len;
    }
    for (int r = threadIdx.x / kChunks; r < kRows; r += kThreads / kChunks) {
      const int64_t tt = tb - 3 + r;
      const bool ok = c < ctot && tt >= 0 && tt < a.total_T;
      sm100::cp_async16(sm100::smem_u32(&tile[r][q * kPer]), ok ? col + (size_t)tt * rl : col,
                        ok);
    }
  }
  sm100::cp_async_commit();
  for (int i = threadIdx.x; i < kLanes * kCh; i += kThreads)
    sw[i] = cb + i < ctot ? __ldg(reinterpret_cast<const float4*>(a.conv_w) + cb + i)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
  sm100::cp_async_wait_all();
  __syncthreads();

  const int lane = threadIdx.x % kLanes;
  const int c0 = cb + lane * kCh;
  if (c0 >= ctot) return;
  const ChanMap m = chan_map(a, c0);
  const int G = a.H_v / a.H_qk;
  const int srow = 2 * a.d_k + a.d_v;
  Tin* Y = static_cast<Tin*>(m.which == 0 ? a.q_out : m.which == 1 ? a.k_out : a.v_out);
  // the value head whose state copy is read (q/k: the group's first), and
  // the copies that are written
  const int hv_read = m.which == 2 ? m.head : m.head * G;
  const int hv_lo = hv_read;
  const int hv_hi = m.which == 2 ? m.head + 1 : (m.head + 1) * G;
  auto state_val = [&](int seq, int r, int j) -> float {
    return a.state_in
               ? a.state_in[(((size_t)seq * a.H_v + hv_read) * 3 + r) * srow + m.st_off + j]
               : 0.f;
  };
  auto put_state = [&](int seq, int r, const float* x) {
    for (int hv = hv_lo; hv < hv_hi; ++hv)
#pragma unroll
      for (int j = 0; j < kCh; ++j)
        a.state_out[(((size_t)seq * a.H_v + hv) * 3 + r) * srow + m.st_off + j] = x[j];
  };

  // empty sequences carry their state through unchanged (first token row only)
  if (blockIdx.x == 0 && threadIdx.x < kLanes && a.state_out != nullptr) {
    for (int s = 0; s < a.n_seq; ++s) {
      int64_t t0, t1;
      if (!seq_bounds(a.cu_seqlens, s, a.total_T, &t0, &t1, nullptr) || t1 != t0) continue;
      for (int r = 0; r < 3; ++r) {
        float x[kCh];
#pragma unroll
        for (int j = 0; j < kCh; ++j) x[j] = state_val(s, r, j);
        put_state(s, r, x);
      }
    }
  }

  float4 cw[kCh];  // this thread's channels' weights (read once; lane-strided shared reads conflict)
#pragma unroll
  for (int j = 0; j < kCh; ++j) cw[j] = sw[lane * kCh + j];
  const int row0 = (threadIdx.x / kLanes) * kTPT;  // tile row of this thread's first token - 3
  const int64_t tg = tb + row0;
  if (tg >= a.total_T) return;
  int s = seq_of(a.cu_seqlens, a.n_seq, tg);
  int64_t s0, s1;
  if (!seq_bounds(a.cu_seqlens, s, a.total_T, &s0, &s1, a.err)) return;
  if (tg - 3 >= s0 && tg + kTPT <= s1 - 3) {
    // common case: the thread's tokens and the three before them lie inside
    // one sequence, and none of them is among its last three (no state to
    // write): a sliding window over the tile, one shared load per token
    float xm3[kCh], xm2[kCh], xm1[kCh];
    Vec8<Tin>::load_shared(&tile[row0][lane * kCh], xm3);
    Vec8<Tin>::load_shared(&tile[row0 + 1][lane * kCh], xm2);
    Vec8<Tin>::load_shared(&tile[row0 + 2][lane * kCh], xm1);
    Tin* out = Y + (size_t)tg * m.row_len + m.col;
#pragma unroll
    for (int i = 0; i < kTPT; ++i) {
      float x[kCh], y[kCh];
      Vec8<Tin>::load_shared(&tile[row0 + 3 + i][lane * kCh], x);
#pragma unroll
      for (int j = 0; j < kCh; ++j) {
        const float u = cw[j].w * x[j] + cw[j].z * xm1[j] + cw[j].y * xm2[j] + cw[j].x * xm3[j];
        y[j] = __fdividef(u, 1.f + __expf(-u));
        xm3[j] = xm2[j];
        xm2[j] = xm1[j];
        xm1[j] = x[j];
      }
      Vec8<Tin>::store(out, y);
      out += m.row_len;
    }
    return;
  }
#pragma unroll 1
  for (int i = 0; i < kTPT; ++i) {
    const int64_t t = tg + i;
    if (t < a.total_T) {
      while (t >= s1) {  // the next non-empty sequence starts inside this thread's tokens
        ++s;
        if (!seq_bounds(a.cu_seqlens, s, a.total_T, &s0, &s1, a.err)) return;
      }
      float x[4][kCh];  // x[j] = input j tokens back (tile row row0 + i + 3 - j)
#pragma unroll
      for (int back = 0; back < 4; ++back)
        Vec8<Tin>::load_shared(&tile[row0 + i + 3 - back][lane * kCh], x[back]);
      if (t - 3 < s0) {  // inputs before the sequence's first token: the carried state
#pragma unroll
        for (int back = 1; back <= 3; ++back)
          if (t - back < s0)
#pragma unroll
            for (int j = 0; j < kCh; ++j) x[back][j] = state_val(s, 3 - (int)(s0 - (t - back)), j);
      }
      float y[kCh];
#pragma unroll
      for (int j = 0; j < kCh; ++j) {
        const float u = cw[j].w * x[0][j] + cw[j].z * x[1][j] + cw[j].y * x[2][j] +
                        cw[j].x * x[3][j];
        y[j] = __fdividef(u, 1.f + __expf(-u));
      }
      Vec8<Tin>::store(Y + (size_t)t * m.row_len + m.col, y);
      if (a.state_out != nullptr) {
        // the sequence's last three inputs, oldest first; for a sequence
        // shorter than three, its first token also carries over older rows
        if (t >= s1 - 3) put_state(s, (int)(t - (s1 - 3)), x[0]);
        const int64_t len = s1 - s0;
        if (t == s0 && len < 3) {
          for (int r = 0; r < 3 - (int)len; ++r) {
            float o[kCh];
#pragma unroll
            for (int j = 0; j < kCh; ++j) o[j] = state_val(s, r + (int)len, j);
            put_state(s, r, o);
          }
        }
      }
    }
  }
}

}  // namespace

gdn_status launch_conv(const ConvArgs& a, cudaStream_t stream) {
  const int ctot = 2 * a.H_qk * a.d_k + a.H_v * a.d_v;
  const unsigned gy = (unsigned)((ctot / kCh + kLanes - 1) / kLanes);
  const int tpt = a.dtype == GDN_BF16 ? Tpt<__nv_bfloat16>::n : Tpt<float>::n;
  const int64_t rows = (a.total_T + kTok * tpt - 1) / (kTok * tpt);
  const unsigned gx = (unsigned)(rows > 0 ? rows : 1);  // one row also carries empty sequences
  if (a.dtype == GDN_BF16)
    gdn_conv_kernel<__nv_bfloat16><<<dim3(gx, gy), kThreads, 0, stream>>>(a);
  else if (a.dtype == GDN_FP32)
    gdn_conv_kernel<float><<<dim3(gx, gy), kThreads, 0, stream>>>(a);
  else
    return GDN_ERR_UNSUPPORTED;
  return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn
