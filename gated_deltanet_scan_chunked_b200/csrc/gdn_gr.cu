// Gated Residual (GR) read and write over an FP8 residual state
// ("Qwen3.8-Flash-Next: architecture, efficiency and technical lineage",
// section 05 "Residual design", part 4 "GR" with its "Group RMSNorm",
// "Low-rank router" and "No Hres" boxes; the FP8 state and the fused
// read/write are in the inference paragraph of the same section):
//
//   R^_i = RMSNorm(R_i; gamma_i)
//   G    = unvec(sigmoid(W_u SiLU((1/n_r) W_d vec(R^))))
//   x    = (1/n_r) sum_i G_i o R^_i          (read: the block input)
//   s    = 2 sigmoid((1/n_r) W_w vec(R^))
//   R'_i = R_i + s_i y                         (write of the block output y)
//
// The state is E4M3 with one fp32 scale per (token, branch) row; a written
// row is requantised with scale max|R'| / 448 (1 for an all-zero row).
//
// Read = three kernels of this file around two bf16 GEMMs (gdn_gemm.cu:
// tcgen05 MMAs, fp32 accumulation) for the low-rank router:
//   gr_norm    codes -> R^ (bf16, group RMSNorm with gains), a warp per row
//   GEMM       H' = (1/n_r) R^ [W_d; W_w; 0]^T            [T, rank + 8]
//   gr_router  H = SiLU(H'[:, :rank]) in place; s = 2 sigmoid(H'[:, rank:rank+n_r])
//   GEMM       L = H W_u^T                                 [T, n_r d]
//   gr_gate    x = (1/n_r) sum_i sigmoid(L_i) o R^_i      [T, d] bf16
// Write = one kernel, one warp per (token, branch) row held in registers, in
// place.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kNT = 256;

__device__ __forceinline__ float e4m3_to_float(uint8_t c) {
  const __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
  return __half2float(__half(hr));
}

__device__ __forceinline__ void bf16x8_load(const __nv_bfloat16* p, float* x) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

__device__ __forceinline__ void bf16x8_store(__nv_bfloat16* p, const float* x) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&b);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// Two E4M3 codes (low byte first) -> their values as an fp32 pair (exact).
__device__ __forceinline__ uint64_t e4m3x2_to_f2(uint32_t c2) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((unsigned short)c2));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
  return f2_pack(f.x, f.y);
}
// An fp32 pair -> two E4M3 codes (low byte = first), round to nearest even,
// saturating to +-448.
__device__ __forceinline__ uint32_t f2_to_e4m3x2(uint64_t v) {
  float x0, x1;
  f2_unpack(v, x0, x1);
  unsigned short c;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "f"(x1), "f"(x0));
  return c;
}

// The write's codes are the E4M3 rounding of the exact quotient r / scale.
// With inv = fl(1 / scale), the kernel forms q- = r * fl(inv (1 - 2^-21)) and
// q+ = r * fl(inv (1 + 2^-21)), which bracket the exact quotient (each
// rounding moves the products by at most 2^-24 relative), and converts both
// (packed conversions): where the two codes agree, that is the exact
// quotient's code (rounding is monotone).  Where they differ -- the quotient
// lies within ~2^-20 (relative) of a rounding boundary, which is rare -- the
// boundary m between the two codes (exact in fp32) is compared with r / scale
// through the sign of |r| - m scale, which one fused multiply-add gives
// exactly; ties go to the even code.
__device__ __forceinline__ uint32_t e4m3_settle(float r, float scale, uint32_t clo,
                                                uint32_t chi) {
  const uint32_t sign = (__float_as_uint(r) >> 24) & 0x80u;
  clo &= 0x7fu;
  chi &= 0x7fu;
  if (clo > chi) {  // magnitudes in increasing order
    const uint32_t t = clo;
    clo = chi;
    chi = t;
  }
  float vlo, vhi;
  f2_unpack(e4m3x2_to_f2(clo | (chi << 8)), vlo, vhi);
  const float m = 0.5f * (vlo + vhi);
  const float t = __fmaf_rn(-m, scale, fabsf(r));
  const uint32_t c = t > 0.f ? chi : (t < 0.f ? clo : ((clo & 1u) ? chi : clo));
  return c | sign;
}

// gr_norm: one warp per (token, branch) row, the row's codes held in
// registers (GPL groups of 8 per lane): R^ = dequant / sqrt(mean sq + eps) *
// gamma, stored in bf16; the codes are decoded and scaled in pairs.
template <int GPL>
__global__ void __launch_bounds__(128) gr_norm_kernel(const GrArgs a) {
  const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= a.T * a.n_r) return;
  const int b = (int)(row % a.n_r);
  const int g8 = a.d / 8;
  const uint8_t* codes = a.codes + (size_t)row * a.d;
  const float sc = __ldg(a.scales + row);
  const uint64_t sc2 = f2_pack(sc, sc);
  uint2 raw[GPL];
#pragma unroll
  for (int k = 0; k < GPL; ++k) {
    const int j = lane + 32 * k;
    raw[k] = j < g8 ? __ldg(reinterpret_cast<const uint2*>(codes) + j) : make_uint2(0u, 0u);
  }
  uint64_t ss2 = 0ull;
#pragma unroll
  for (int k = 0; k < GPL; ++k) {
    const uint32_t cw[2] = {raw[k].x, raw[k].y};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint64_t x = f2_mul(e4m3x2_to_f2(cw[p / 2] >> (16 * (p % 2))), sc2);
      ss2 = f2_fma(x, x, ss2);
    }
  }
  float s0, s1;
  f2_unpack(ss2, s0, s1);
  const float ss = warp_sum(s0 + s1);
  const float r = rsqrtf(ss / (float)a.d + a.eps);
  __nv_bfloat16* out = a.rhat + (size_t)row * a.d;
  const float* gam = a.gamma + (size_t)b * a.d;
#pragma unroll
  for (int k = 0; k < GPL; ++k) {
    const int j = lane + 32 * k;
    if (j < g8) {
      const uint32_t cw[2] = {raw[k].x, raw[k].y};
      const float4 g0 = __ldg(reinterpret_cast<const float4*>(gam + 8 * j));
      const float4 g1 = __ldg(reinterpret_cast<const float4*>(gam + 8 * j) + 1);
      const uint64_t gm[4] = {f2_pack(g0.x * r, g0.y * r), f2_pack(g0.z * r, g0.w * r),
                              f2_pack(g1.x * r, g1.y * r), f2_pack(g1.z * r, g1.w * r)};
      float x[8];
#pragma unroll
      for (int p = 0; p < 4; ++p)
        f2_unpack(f2_mul(f2_mul(e4m3x2_to_f2(cw[p / 2] >> (16 * (p % 2))), sc2), gm[p]),
                  x[2 * p], x[2 * p + 1]);
      bf16x8_store(out + 8 * j, x);
    }
  }
}

// gr_router: on H' = (1/n_r) R^ [W_d; W_w]^T ([T, ldh], ldh = rank + 8):
// the first rank columns become SiLU(.) in place (bf16), the next n_r give
// the write scalars s = 2 sigmoid(.) (fp32).
__global__ void __launch_bounds__(kNT) gr_router_kernel(const GrArgs a, __nv_bfloat16* h,
                                                        int ldh) {
  const int64_t i = (int64_t)blockIdx.x * kNT + threadIdx.x;  // 8-column group
  const int gpr = ldh / 8;
  if (i >= a.T * gpr) return;
  const int64_t t = i / gpr;
  const int c = (int)(i % gpr) * 8;
  __nv_bfloat16* p = h + (size_t)t * ldh + c;
  float x[8];
  bf16x8_load(p, x);
  if (c < a.rank) {
#pragma unroll
    for (int k = 0; k < 8; ++k) x[k] = x[k] / (1.f + expf(-x[k]));
    bf16x8_store(p, x);
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (c + k - a.rank < a.n_r)
        a.s[(size_t)t * a.n_r + (c + k - a.rank)] = 2.f / (1.f + expf(-x[k]));
  }
}

// gr_gate: x[t, c] = (1/n_r) sum_i sigmoid(L[t, i d + c]) R^[t, i d + c]; the
// branches' loads are issued together.  sigmoid(l) = (1 + tanh(l / 2)) / 2
// with the hardware tanh (relative error about 2^-11, below the bf16
// rounding of L and R^), on channel pairs.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
template <int NR>  // branches (n_r)
__global__ void __launch_bounds__(kNT) gr_gate_kernel(const GrArgs a) {
  const int64_t idx = (int64_t)blockIdx.x * kNT + threadIdx.x;  // 8-channel group
  const int g8 = a.d / 8;
  if (idx >= a.T * g8) return;
  const int64_t t = idx / g8;
  const int c = (int)(idx % g8) * 8;
  const size_t base = (size_t)t * a.n_r * a.d + c;
  uint4 lr[NR], rr[NR];
#pragma unroll
  for (int b = 0; b < NR; ++b) {
    lr[b] = __ldg(reinterpret_cast<const uint4*>(a.logits + base + (size_t)b * a.d));
    rr[b] = __ldg(reinterpret_cast<const uint4*>(a.rhat + base + (size_t)b * a.d));
  }
  const uint64_t half2 = f2_pack(0.5f, 0.5f);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int b = 0; b < NR; ++b) {
    const uint32_t lw[4] = {lr[b].x, lr[b].y, lr[b].z, lr[b].w};
    const uint32_t rw[4] = {rr[b].x, rr[b].y, rr[b].z, rr[b].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // bf16 pairs: a bf16 is the high half of its fp32 value
      const uint64_t l2 = f2_pack(__uint_as_float(lw[i] << 16), __uint_as_float(lw[i] & 0xffff0000u));
      const uint64_t r2 = f2_pack(__uint_as_float(rw[i] << 16), __uint_as_float(rw[i] & 0xffff0000u));
      float h0, h1;
      f2_unpack(f2_mul(l2, half2), h0, h1);
      const uint64_t g = f2_fma(f2_pack(tanh_approx(h0), tanh_approx(h1)), half2, half2);
      acc[i] = f2_fma(g, r2, acc[i]);
    }
  }
  const float inv = 1.f / (float)NR;
  float o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f2_unpack(acc[i], o[2 * i], o[2 * i + 1]);
    o[2 * i] *= inv;
    o[2 * i + 1] *= inv;
  }
  bf16x8_store(static_cast<__nv_bfloat16*>(a.x) + (size_t)t * a.d + c, o);
}

// gr_write: one warp per (token, branch) row, in place, the row's values
// held in registers (GPL groups of 8 per lane, as fp32 pairs).  r = deq + s
// y with one rounding per operation; scale' = max|r| / 448 (1 if zero); code
// = the E4M3 rounding (nearest, ties to even, saturating) of the exact
// quotient r / scale', from r * fl(1 / scale') and the settlement above.
// Decoding and encoding work on channel pairs (packed conversions); the
// product and the sum stay scalar fp32 operations with explicit rounding, so
// that they are never fused into one.
template <int GPL>
__global__ void __launch_bounds__(128) gr_write_kernel(const GrWriteArgs a) {
  const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= a.T * a.n_r) return;
  const int64_t t = row / a.n_r;
  const int g8 = a.d / 8;
  uint8_t* codes = a.codes + (size_t)row * a.d;
  const __nv_bfloat16* y = static_cast<const __nv_bfloat16*>(a.y) + (size_t)t * a.d;
  const float sc = a.scales[row];
  const float sv = __ldg(a.s + row);
  uint2 raw[GPL];
  uint4 yr[GPL];
#pragma unroll
  for (int k = 0; k < GPL; ++k) {
    const int j = lane + 32 * k;
    raw[k] = j < g8 ? reinterpret_cast<const uint2*>(codes)[j] : make_uint2(0u, 0u);
    yr[k] = j < g8 ? __ldg(reinterpret_cast<const uint4*>(y) + j) : make_uint4(0u, 0u, 0u, 0u);
  }
  uint64_t r[GPL][4];  // element pairs (2p, 2p + 1) of group k
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < GPL; ++k) {
    const uint32_t cw[2] = {raw[k].x, raw[k].y};
    const uint32_t yw[4] = {yr[k].x, yr[k].y, yr[k].z, yr[k].w};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      float d0, d1;
      f2_unpack(e4m3x2_to_f2(cw[p / 2] >> (16 * (p % 2))), d0, d1);
      // product and sum rounded separately (never fused)
      const float r0 = __fadd_rn(__fmul_rn(d0, sc), __fmul_rn(sv, __uint_as_float(yw[p] << 16)));
      const float r1 =
          __fadd_rn(__fmul_rn(d1, sc), __fmul_rn(sv, __uint_as_float(yw[p] & 0xffff0000u)));
      r[k][p] = f2_pack(r0, r1);
      amax = fmaxf(amax, fmaxf(fabsf(r0), fabsf(r1)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float nsc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  const float inv = __fdiv_rn(1.f, nsc);
  const float inv_lo = inv * (1.f - 0x1p-21f), inv_hi = inv * (1.f + 0x1p-21f);
  const uint64_t inv2lo = f2_pack(inv_lo, inv_lo), inv2hi = f2_pack(inv_hi, inv_hi);
#pragma unroll
  for (int k = 0; k < GPL; ++k) {
    const int j = lane + 32 * k;
    if (j < g8) {
      // codes of q- (wl) and q+ (wh), element pairs packed
      uint32_t wl[2], wh[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint64_t ra = r[k][2 * h], rb = r[k][2 * h + 1];
        wl[h] = f2_to_e4m3x2(f2_mul(ra, inv2lo)) | (f2_to_e4m3x2(f2_mul(rb, inv2lo)) << 16);
        wh[h] = f2_to_e4m3x2(f2_mul(ra, inv2hi)) | (f2_to_e4m3x2(f2_mul(rb, inv2hi)) << 16);
      }
      if (((wl[0] ^ wh[0]) | (wl[1] ^ wh[1])) != 0u) {
        // rare: a code next to a rounding boundary, settled exactly
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int h = e >> 2, sh = 8 * (e & 3);
          const uint32_t cl = (wl[h] >> sh) & 0xffu, ch = (wh[h] >> sh) & 0xffu;
          if (cl != ch) {
            float r0, r1;
            f2_unpack(r[k][e >> 1], r0, r1);
            wl[h] = (wl[h] & ~(0xffu << sh)) | (e4m3_settle((e & 1) ? r1 : r0, nsc, cl, ch) << sh);
          }
        }
      }
      reinterpret_cast<uint2*>(codes)[j] = make_uint2(wl[0], wl[1]);
    }
  }
  if (lane == 0) a.scales[row] = nsc;
}

size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

size_t gr_read_workspace_bytes(int64_t T, int32_t n_r, int32_t d, int32_t rank) {
  const size_t nd = (size_t)n_r * d;
  return 2 * a256((size_t)T * nd * 2) + a256((size_t)T * (rank + 8) * 2) +
         a256((size_t)(rank + 8) * nd * 2) +
         a256(gemm_tn_workspace_bytes((int)T, rank + 8, (int)nd));
}

template <template <int> class K, typename Args>
gdn_status launch_rows(const Args& a, int64_t rows, int d, cudaStream_t stream) {
  const int gpl = (d / 8 + 31) / 32;
  const unsigned grid = (unsigned)((rows + 3) / 4);
  switch (gpl) {
#define GDN_GPL(n) case n: K<n>::launch(a, grid, stream); break;
    GDN_GPL(1) GDN_GPL(2) GDN_GPL(3) GDN_GPL(4) GDN_GPL(5) GDN_GPL(6) GDN_GPL(7) GDN_GPL(8)
    GDN_GPL(9) GDN_GPL(10) GDN_GPL(11) GDN_GPL(12) GDN_GPL(13) GDN_GPL(14) GDN_GPL(15)
    GDN_GPL(16)
#undef GDN_GPL
    default: return GDN_ERR_UNSUPPORTED;
  }
  return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

template <int GPL>
struct NormK {
  static void launch(const GrArgs& a, unsigned grid, cudaStream_t s) {
    gr_norm_kernel<GPL><<<grid, 128, 0, s>>>(a);
  }
};
template <int GPL>
struct WriteK {
  static void launch(const GrWriteArgs& a, unsigned grid, cudaStream_t s) {
    gr_write_kernel<GPL><<<grid, 128, 0, s>>>(a);
  }
};

gdn_status launch_gr_read(GrArgs a, void* ws, cudaStream_t stream) {
  char* p = static_cast<char*>(ws);
  const size_t nd = (size_t)a.n_r * a.d;
  const int ldh = a.rank + 8;
  a.rhat = reinterpret_cast<__nv_bfloat16*>(p);
  a.logits = reinterpret_cast<__nv_bfloat16*>(p + a256((size_t)a.T * nd * 2));
  __nv_bfloat16* H = reinterpret_cast<__nv_bfloat16*>(p + 2 * a256((size_t)a.T * nd * 2));
  char* Wdw = p + 2 * a256((size_t)a.T * nd * 2) + a256((size_t)a.T * ldh * 2);
  char* gws = Wdw + a256((size_t)ldh * nd * 2);  // the router GEMM's split-K partials
  const size_t gws_bytes = gemm_tn_workspace_bytes((int)a.T, ldh, (int)nd);
  if (a.T == 0) return GDN_OK;
  // [W_d; W_w; 0] in one operand, so that one GEMM gives the router and the
  // write scalars
  if (cudaMemcpyAsync(Wdw, a.W_d, (size_t)a.rank * nd * 2, cudaMemcpyDeviceToDevice, stream) !=
          cudaSuccess ||
      cudaMemcpyAsync(Wdw + (size_t)a.rank * nd * 2, a.W_w, (size_t)a.n_r * nd * 2,
                      cudaMemcpyDeviceToDevice, stream) != cudaSuccess ||
      cudaMemsetAsync(Wdw + (size_t)(a.rank + a.n_r) * nd * 2, 0,
                      (size_t)(8 - a.n_r) * nd * 2, stream) != cudaSuccess)
    return GDN_ERR_CUDA;
  gdn_status st = launch_rows<NormK>(a, a.T * a.n_r, a.d, stream);
  if (st != GDN_OK) return st;
  // H' [T][ldh] = (1/n_r) R^ [T][nd] [W_d; W_w; 0]^T
  st = gemm_tn_bf16((int)a.T, ldh, (int)nd, 1.f / (float)a.n_r, a.rhat, (int64_t)nd, Wdw,
                    (int64_t)nd, H, ldh, gws, gws_bytes, stream);
  if (st != GDN_OK) return st;
  const int64_t groups = a.T * (ldh / 8);
  gr_router_kernel<<<(unsigned)((groups + kNT - 1) / kNT), kNT, 0, stream>>>(a, H, ldh);
  // L [T][nd] = SiLU(H) [T][rank] W_u^T (W_u [nd][rank])
  st = gemm_tn_bf16((int)a.T, (int)nd, a.rank, 1.f, H, ldh, a.W_u, a.rank, a.logits,
                    (int64_t)nd, nullptr, 0, stream);
  if (st != GDN_OK) return st;
  const int64_t g2 = a.T * (a.d / 8);
  const unsigned gg = (unsigned)((g2 + kNT - 1) / kNT);
  switch (a.n_r) {
#define GDN_NR(n) \
  case n: gr_gate_kernel<n><<<gg, kNT, 0, stream>>>(a); break;
    GDN_NR(1) GDN_NR(2) GDN_NR(3) GDN_NR(4) GDN_NR(5) GDN_NR(6) GDN_NR(7) GDN_NR(8)
#undef GDN_NR
    default: return GDN_ERR_UNSUPPORTED;
  }
  return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status launch_gr_write(const GrWriteArgs& a, cudaStream_t stream) {
  const int64_t rows = a.T * a.n_r;
  if (rows == 0) return GDN_OK;
  return launch_rows<WriteK>(a, rows, a.d, stream);
}

}  // namespace gdn
