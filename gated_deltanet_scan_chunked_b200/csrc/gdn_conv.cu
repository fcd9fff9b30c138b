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
// This kernel is HBM-bound.  A CTA owns 256 channels and a run of
// consecutive token tiles (one wave of CTAs covers the whole input); it
// stages the inputs of a tile, 256 channels x (64 + 3) tokens (bf16; 32 + 3
// for fp32), in shared memory with 16-byte asynchronous copies, double-
// buffered so that the next tile's copies are in flight while this one is
// computed.  Each thread computes 4 consecutive channels of 16 (fp32: 8)
// consecutive tokens and writes them with 8-byte (fp32: 16-byte) stores.
#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_sm100.cuh"

namespace gdn {
namespace {

constexpr int kCh = 4;        // channels per thread
constexpr int kLanes = 64;    // threads along the channels (256 channels)
constexpr int kTok = 4;       // thread rows per CTA
constexpr int kThreads = kLanes * kTok;
constexpr int kMinCtas = 3;   // resident CTAs per SM the kernel is built for
// consecutive tokens per thread (a tile: 64 + 3 rows of 256 bf16 channels, 32 + 3 for fp32)
template <typename Tin>
struct Tpt { static constexpr int n = sizeof(Tin) == 2 ? 16 : 8; };

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// SiLU on a channel pair: per lane the operations of silu_approx
// (u / (1 + 2^(-u log2 e)), every step rounded in fp32, on the hardware 2^x
// and reciprocal approximations), with the multiplies and the add packed.
constexpr float kNegLog2e = -1.4426950408889634f;
__device__ __forceinline__ uint64_t silu2(uint64_t u) {
  float z0, z1;
  f2_unpack(f2_mul(u, f2_pack(kNegLog2e, kNegLog2e)), z0, z1);
  float d0, d1;
  f2_unpack(f2_add(f2_pack(sm100::ex2_approx(z0), sm100::ex2_approx(z1)), f2_pack(1.f, 1.f)), d0,
            d1);
  return f2_mul(u, f2_pack(rcp_approx(d0), rcp_approx(d1)));
}

// Four consecutive channels of one token: shared loads and global stores,
// as fp32 values or as two channel pairs.
template <typename Tin>
struct Vec4;
template <>
struct Vec4<float> {
  static __device__ __forceinline__ void load_shared(const float* p, float* x) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  }
  static __device__ __forceinline__ void store(float* p, const float* x) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
  static __device__ __forceinline__ void load_shared2(const float* p, uint64_t* x) {
    const ulonglong2 a = *reinterpret_cast<const ulonglong2*>(p);
    x[0] = a.x; x[1] = a.y;
  }
  static __device__ __forceinline__ void store2(float* p, const uint64_t* y) {
    *reinterpret_cast<ulonglong2*>(p) = make_ulonglong2(y[0], y[1]);
  }
};
template <>
struct Vec4<__nv_bfloat16> {
  // (a bf16 is the high half of its fp32 value)
  static __device__ __forceinline__ void load_shared(const __nv_bfloat16* p, float* x) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    x[0] = __uint_as_float(u.x << 16); x[1] = __uint_as_float(u.x & 0xffff0000u);
    x[2] = __uint_as_float(u.y << 16); x[3] = __uint_as_float(u.y & 0xffff0000u);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* x) {
    __nv_bfloat162 b0 = __floats2bfloat162_rn(x[0], x[1]);
    __nv_bfloat162 b1 = __floats2bfloat162_rn(x[2], x[3]);
    *reinterpret_cast<uint2*>(p) =
        make_uint2(*reinterpret_cast<uint32_t*>(&b0), *reinterpret_cast<uint32_t*>(&b1));
  }
  static __device__ __forceinline__ void load_shared2(const __nv_bfloat16* p, uint64_t* x) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    x[0] = f2_pack(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u));
    x[1] = f2_pack(__uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
  }
  static __device__ __forceinline__ void store2(__nv_bfloat16* p, const uint64_t* y) {
    float f[4];
    f2_unpack(y[0], f[0], f[1]);
    f2_unpack(y[1], f[2], f[3]);
    store(p, f);
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

// Shared memory of one CTA: two input tiles (dynamic; the weights are static).
template <typename Tin>
constexpr int conv_tile_rows() { return kTok * Tpt<Tin>::n + 3; }
template <typename Tin>
constexpr size_t conv_smem_bytes() {
  return 2 * (size_t)conv_tile_rows<Tin>() * kLanes * kCh * sizeof(Tin);
}

template <typename Tin>
__global__ void __launch_bounds__(kThreads, kMinCtas) gdn_conv_kernel(const ConvArgs a, int tiles_per_cta) {
  constexpr int kTPT = Tpt<Tin>::n;
  constexpr int kTileTok = kTok * kTPT;                 // tokens per tile
  constexpr int kRows = conv_tile_rows<Tin>();          // the tile's tokens and the 3 before
  constexpr int kW = kLanes * kCh;                      // channels per CTA
  constexpr int kChunks = kW * sizeof(Tin) / 16;        // 16-byte pieces per row
  constexpr int kPer = 16 / sizeof(Tin);                // channels per piece
  static_assert(kThreads % kChunks == 0, "a thread's pieces share one column");
  // weights (w0, w1, w2, w3) of channel cb + 8 l + j at sw[j][l]: a warp's
  // reads of one j are consecutive
  __shared__ float4 sw[kCh][kLanes];
  extern __shared__ __align__(16) unsigned char conv_smem[];
  Tin(*tiles)[kRows][kW] = reinterpret_cast<Tin(*)[kRows][kW]>(conv_smem);
  const int ctot = 2 * a.H_qk * a.d_k + a.H_v * a.d_v;
  const int cb = blockIdx.y * kW;
  const int64_t n_tiles = (a.total_T + kTileTok - 1) / kTileTok;
  const int64_t tile0 = (int64_t)blockIdx.x * tiles_per_cta;
  const int nt = (int)((n_tiles - tile0) < tiles_per_cta ? (n_tiles - tile0) : tiles_per_cta);

  // this thread's 16-byte input column (rows outside [0, total_T) and
  // channels past the end are zero filled)
  const int q = threadIdx.x % kChunks;
  const Tin* col = static_cast<const Tin*>(a.q);
  size_t rl = 0;
  bool col_ok = false;
  {
    const int c = cb + q * kPer;
    if (c < ctot) {
      const ChanMap mm = chan_map(a, c);
      col = static_cast<const Tin*>(mm.which == 0 ? a.q : mm.which == 1 ? a.k : a.v) + mm.col;
      rl = (size_t)mm.row_len;
      col_ok = true;
    }
  }
  auto load_tile = [&](int buf, int64_t tb) {
    for (int r = threadIdx.x / kChunks; r < kRows; r += kThreads / kChunks) {
      const int64_t tt = tb - 3 + r;
      const bool ok = col_ok && tt >= 0 && tt < a.total_T;
      sm100::cp_async16(sm100::smem_u32(&tiles[buf][r][q * kPer]),
                        ok ? col + (size_t)tt * rl : col, ok);
    }
  };
  if (nt > 0) load_tile(0, tile0 * kTileTok);
  sm100::cp_async_commit();
  for (int i = threadIdx.x; i < kW; i += kThreads)
    sw[i % kCh][i / kCh] = cb + i < ctot
                               ? __ldg(reinterpret_cast<const float4*>(a.conv_w) + cb + i)
                               : make_float4(0.f, 0.f, 0.f, 0.f);

  const int lane = threadIdx.x % kLanes;
  const int c0 = cb + lane * kCh;
  const bool chan_ok = c0 < ctot;
  const ChanMap m = chan_map(a, chan_ok ? c0 : 0);
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

  // empty sequences carry their state through unchanged (first token group only)
  if (chan_ok && blockIdx.x == 0 && threadIdx.x < kLanes && a.state_out != nullptr) {
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
  __syncthreads();  // weights staged

  const int row0 = (threadIdx.x / kLanes) * kTPT;  // tile row of this thread's first token - 3

  // One tile: outputs of this thread's kTPT tokens from the staged inputs.
  auto compute_tile = [&](const Tin (*tile)[kW], int64_t tb) {
    const int64_t tg = tb + row0;
    if (!chan_ok || tg >= a.total_T) return;
    int s = seq_of(a.cu_seqlens, a.n_seq, tg);
    int64_t s0, s1;
    if (!seq_bounds(a.cu_seqlens, s, a.total_T, &s0, &s1, a.err)) return;
    float4 cw[kCh];  // this thread's channels' weights
#pragma unroll
    for (int j = 0; j < kCh; ++j) cw[j] = sw[j][lane];
    if (tg - 3 >= s0 && tg + kTPT <= s1 - 3) {
      // common case: the thread's tokens and the three before them lie inside
      // one sequence, and none of them is among its last three (no state to
      // write): a sliding window over the tile, one shared load per token
      // (channel pairs: u = w3 x_t + w2 x_t-1 + w1 x_t-2 + w0 x_t-3, in
      // that order, as in the general path below)
      constexpr int kP = kCh / 2;
      uint64_t w0[kP], w1[kP], w2[kP], w3[kP];
#pragma unroll
      for (int p = 0; p < kP; ++p) {
        w0[p] = f2_pack(cw[2 * p].x, cw[2 * p + 1].x);
        w1[p] = f2_pack(cw[2 * p].y, cw[2 * p + 1].y);
        w2[p] = f2_pack(cw[2 * p].z, cw[2 * p + 1].z);
        w3[p] = f2_pack(cw[2 * p].w, cw[2 * p + 1].w);
      }
      uint64_t xm3[kP], xm2[kP], xm1[kP];
      Vec4<Tin>::load_shared2(&tile[row0][lane * kCh], xm3);
      Vec4<Tin>::load_shared2(&tile[row0 + 1][lane * kCh], xm2);
      Vec4<Tin>::load_shared2(&tile[row0 + 2][lane * kCh], xm1);
      Tin* out = Y + (size_t)tg * m.row_len + m.col;
#pragma unroll
      for (int i = 0; i < kTPT; ++i) {
        uint64_t x[kP], y[kP];
        Vec4<Tin>::load_shared2(&tile[row0 + 3 + i][lane * kCh], x);
#pragma unroll
        for (int p = 0; p < kP; ++p) {
          uint64_t u = f2_mul(w3[p], x[p]);
          u = f2_fma(w2[p], xm1[p], u);
          u = f2_fma(w1[p], xm2[p], u);
          u = f2_fma(w0[p], xm3[p], u);
          y[p] = silu2(u);
          xm3[p] = xm2[p];
          xm2[p] = xm1[p];
          xm1[p] = x[p];
        }
        Vec4<Tin>::store2(out, y);
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
        // u = sum over back = 0..3 of w[3 - back] x_(t - back); inputs before
        // the sequence's first token come from the carried state
        float x0[kCh], u[kCh];
        Vec4<Tin>::load_shared(&tile[row0 + i + 3][lane * kCh], x0);
#pragma unroll
        for (int j = 0; j < kCh; ++j) u[j] = __fmul_rn(cw[j].w, x0[j]);
#pragma unroll 1
        for (int back = 1; back <= 3; ++back) {
          float xb[kCh];
          if (t - back < s0) {
#pragma unroll
            for (int j = 0; j < kCh; ++j) xb[j] = state_val(s, 3 - (int)(s0 - (t - back)), j);
          } else {
            Vec4<Tin>::load_shared(&tile[row0 + i + 3 - back][lane * kCh], xb);
          }
#pragma unroll
          for (int j = 0; j < kCh; ++j) {
            const float wj = back == 1 ? cw[j].z : back == 2 ? cw[j].y : cw[j].x;
            u[j] = __fmaf_rn(wj, xb[j], u[j]);
          }
        }
        float y[kCh];
#pragma unroll
        for (int j = 0; j < kCh; ++j) y[j] = silu_approx(u[j]);
        Vec4<Tin>::store(Y + (size_t)t * m.row_len + m.col, y);
        if (a.state_out != nullptr) {
          // the sequence's last three inputs, oldest first; for a sequence
          // shorter than three, its first token also carries over older rows
          if (t >= s1 - 3) put_state(s, (int)(t - (s1 - 3)), x0);
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
  };

  for (int it = 0; it < nt; ++it) {
    // the next tile's copies go into the other buffer, read two tiles ago
    if (it + 1 < nt) load_tile((it + 1) & 1, (tile0 + it + 1) * kTileTok);
    sm100::cp_async_commit();
    sm100::cp_async_wait_group1();  // this tile's group has landed
    __syncthreads();
    compute_tile(tiles[it & 1], (tile0 + it) * kTileTok);
    __syncthreads();  // buffer it & 1 is refilled in the next iteration
  }
}

}  // namespace

gdn_status launch_conv(const ConvArgs& a, cudaStream_t stream) {
  const int ctot = 2 * a.H_qk * a.d_k + a.H_v * a.d_v;
  const unsigned gy = (unsigned)((ctot / kCh + kLanes - 1) / kLanes);
  const int tpt = a.dtype == GDN_BF16 ? Tpt<__nv_bfloat16>::n : Tpt<float>::n;
  int64_t n_tiles = (a.total_T + kTok * tpt - 1) / (kTok * tpt);
  if (n_tiles < 1) n_tiles = 1;  // one tile row also carries empty sequences
  // one wave: kMinCtas resident CTAs per SM, each taking a run of consecutive tiles
  static int sm_count[64] = {0};
  static bool attr_set[64][2] = {{false}};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GDN_ERR_CUDA;
  if (sm_count[dev] == 0 &&
      cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return GDN_ERR_CUDA;
  const int64_t slots = (int64_t)sm_count[dev] * kMinCtas;
  const int64_t per_col = (slots + gy - 1) / gy;  // CTAs along the tokens
  int64_t tiles_per_cta = (n_tiles + per_col - 1) / per_col;
  if (tiles_per_cta < 1) tiles_per_cta = 1;
  const unsigned gx = (unsigned)((n_tiles + tiles_per_cta - 1) / tiles_per_cta);
  if (a.dtype == GDN_BF16) {
    const size_t smem = conv_smem_bytes<__nv_bfloat16>();
    if (!attr_set[dev][0]) {
      if (cudaFuncSetAttribute(gdn_conv_kernel<__nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess)
        return GDN_ERR_CUDA;
      attr_set[dev][0] = true;
    }
    gdn_conv_kernel<__nv_bfloat16><<<dim3(gx, gy), kThreads, smem, stream>>>(a, (int)tiles_per_cta);
  } else if (a.dtype == GDN_FP32) {
    const size_t smem = conv_smem_bytes<float>();
    if (!attr_set[dev][1]) {
      if (cudaFuncSetAttribute(gdn_conv_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem) != cudaSuccess)
        return GDN_ERR_CUDA;
      attr_set[dev][1] = true;
    }
    gdn_conv_kernel<float><<<dim3(gx, gy), kThreads, smem, stream>>>(a, (int)tiles_per_cta);
  } else {
    return GDN_ERR_UNSUPPORTED;
  }
  return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn
