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
// Read = three kernels of this file around two bf16 GEMMs (cuBLASLt, fp32
// accumulation) for the low-rank router:
//   gr_norm    codes -> R^ (bf16, group RMSNorm with gains), a warp per row
//   GEMM       H' = (1/n_r) R^ [W_d; W_w; 0]^T            [T, rank + 8]
//   gr_router  H = SiLU(H'[:, :rank]) in place; s = 2 sigmoid(H'[:, rank:rank+n_r])
//   GEMM       L = H W_u^T                                 [T, n_r d]
//   gr_gate    x = (1/n_r) sum_i sigmoid(L_i) o R^_i      [T, d] bf16
// Write = one kernel, one warp per (token, branch) row held in registers, in
// place.
#include <cublasLt.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <mutex>

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

// gr_norm: one warp per (token, branch) row, the row's codes held in
// registers (GPL groups of 8 per lane): R^ = dequant / sqrt(mean sq + eps) *
// gamma, stored in bf16.
template <int GPL>
__global__ void __launch_bounds__(128) gr_norm_kernel(const GrArgs a) {
  const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= a.T * a.n_r) return;
  const int b = (int)(row % a.n_r);
  const int g8 = a.d / 8;
  const uint8_t* codes = a.codes + (size_t)row * a.d;
  const float sc = __ldg(a.scales + row);
  uint2 raw[GPL];
#pragma unroll
  for (int k = 0; k < GPL; ++k) {
    const int j = lane + 32 * k;
    raw[k] = j < g8 ? __ldg(reinterpret_cast<const uint2*>(codes) + j) : make_uint2(0u, 0u);
  }
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < GPL; ++k) {
    const uint32_t w[2] = {raw[k].x, raw[k].y};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float x = __fmul_rn(e4m3_to_float((w[i / 4] >> (8 * (i % 4))) & 0xFF), sc);
      ss += x * x;
    }
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)a.d + a.eps);
  __nv_bfloat16* out = a.rhat + (size_t)row * a.d;
  const float* gam = a.gamma + (size_t)b * a.d;
#pragma unroll
  for (int k = 0; k < GPL; ++k) {
    const int j = lane + 32 * k;
    if (j < g8) {
      const uint32_t w[2] = {raw[k].x, raw[k].y};
      const float4 g0 = __ldg(reinterpret_cast<const float4*>(gam + 8 * j));
      const float4 g1 = __ldg(reinterpret_cast<const float4*>(gam + 8 * j) + 1);
      const float gm[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      float x[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        x[i] = __fmul_rn(e4m3_to_float((w[i / 4] >> (8 * (i % 4))) & 0xFF), sc) * r * gm[i];
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
// branches' loads are issued together
__global__ void __launch_bounds__(kNT) gr_gate_kernel(const GrArgs a) {
  const int64_t idx = (int64_t)blockIdx.x * kNT + threadIdx.x;  // 8-channel group
  const int g8 = a.d / 8;
  if (idx >= a.T * g8) return;
  const int64_t t = idx / g8;
  const int c = (int)(idx % g8) * 8;
  const size_t base = (size_t)t * a.n_r * a.d + c;
  uint4 lr[kMaxGrBranches], rr[kMaxGrBranches];
#pragma unroll
  for (int b = 0; b < kMaxGrBranches; ++b) {
    if (b < a.n_r) {
      lr[b] = __ldg(reinterpret_cast<const uint4*>(a.logits + base + (size_t)b * a.d));
      rr[b] = __ldg(reinterpret_cast<const uint4*>(a.rhat + base + (size_t)b * a.d));
    }
  }
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
  for (int b = 0; b < kMaxGrBranches; ++b) {
    if (b < a.n_r) {
      const uint32_t lw[4] = {lr[b].x, lr[b].y, lr[b].z, lr[b].w};
      const uint32_t rw[4] = {rr[b].x, rr[b].y, rr[b].z, rr[b].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 l = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&lw[i]));
        const float2 r = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rw[i]));
        acc[2 * i] += __fdividef(r.x, 1.f + __expf(-l.x));
        acc[2 * i + 1] += __fdividef(r.y, 1.f + __expf(-l.y));
      }
    }
  }
  const float inv = 1.f / (float)a.n_r;
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] *= inv;
  bf16x8_store(static_cast<__nv_bfloat16*>(a.x) + (size_t)t * a.d + c, acc);
}

// gr_write: one warp per (token, branch) row, in place, the row's values
// held in registers (GPL groups of 8 per lane).  r = deq + s y with one
// rounding per operation; scale' = max|r| / 448 (1 if zero); inv = 1 /
// scale'; code = E4M3(r * inv) with round to nearest even and saturation.
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
  float r[GPL][8];
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < GPL; ++k) {
    const uint32_t yw[4] = {yr[k].x, yr[k].y, yr[k].z, yr[k].w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t w = i < 4 ? raw[k].x : raw[k].y;
      const float q = __fmul_rn(e4m3_to_float((w >> (8 * (i % 4))) & 0xFF), sc);
      const float yv = __bfloat162float(__ushort_as_bfloat16(
          (unsigned short)((i & 1) ? (yw[i / 2] >> 16) : (yw[i / 2] & 0xFFFFu))));
      r[k][i] = __fadd_rn(q, __fmul_rn(sv, yv));
      amax = fmaxf(amax, fabsf(r[k][i]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float nsc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  const float inv = __fdiv_rn(1.f, nsc);
#pragma unroll
  for (int k = 0; k < GPL; ++k) {
    const int j = lane + 32 * k;
    if (j < g8) {
      uint32_t w[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t c =
            __nv_cvt_float_to_fp8(__fmul_rn(r[k][i], inv), __NV_SATFINITE, __NV_E4M3);
        w[i / 4] |= (c & 0xFFu) << (8 * (i % 4));
      }
      reinterpret_cast<uint2*>(codes)[j] = make_uint2(w[0], w[1]);
    }
  }
  if (lane == 0) a.scales[row] = nsc;
}

// ---- cuBLASLt, one handle per device --------------------------------------

constexpr int kMaxDevices = 64;
std::mutex g_lt_mu;
cublasLtHandle_t g_lt[kMaxDevices] = {nullptr};

cublasLtHandle_t lt_handle() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_lt_mu);
  if (g_lt[dev] == nullptr && cublasLtCreate(&g_lt[dev]) != CUBLAS_STATUS_SUCCESS)
    g_lt[dev] = nullptr;
  return g_lt[dev];
}

// Column-major D[m x n] = alpha op(A) op(B), bf16 operands and result, fp32
// accumulation; A is stored k x m (ld lda) and transposed, B is k x n (ldb).
gdn_status lt_gemm(int m, int n, int k, float alpha, const void* A, int lda, const void* B,
                   int ldb, void* D, int ldd, void* ws, size_t ws_bytes, cudaStream_t stream) {
  cublasLtHandle_t h = lt_handle();
  if (h == nullptr) return GDN_ERR_CUDA;
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t Ad = nullptr, Bd = nullptr, Dd = nullptr;
  cublasLtMatmulPreference_t pref = nullptr;
  gdn_status st = GDN_ERR_CUDA;
  const cublasOperation_t ta = CUBLAS_OP_T, tb = CUBLAS_OP_N;
  const float beta = 0.f;
  cublasLtMatmulHeuristicResult_t res;
  int nres = 0;
  if (cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS)
    goto done;
  cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &ta, sizeof(ta));
  cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &tb, sizeof(tb));
  if (cublasLtMatrixLayoutCreate(&Ad, CUDA_R_16BF, k, m, lda) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatrixLayoutCreate(&Bd, CUDA_R_16BF, k, n, ldb) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatrixLayoutCreate(&Dd, CUDA_R_16BF, m, n, ldd) != CUBLAS_STATUS_SUCCESS)
    goto done;
  if (cublasLtMatmulPreferenceCreate(&pref) != CUBLAS_STATUS_SUCCESS) goto done;
  cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &ws_bytes,
                                       sizeof(ws_bytes));
  if (cublasLtMatmulAlgoGetHeuristic(h, op, Ad, Bd, Dd, Dd, pref, 1, &res, &nres) !=
          CUBLAS_STATUS_SUCCESS ||
      nres == 0) {
    st = GDN_ERR_UNSUPPORTED;
    goto done;
  }
  if (cublasLtMatmul(h, op, &alpha, A, Ad, B, Bd, &beta, D, Dd, D, Dd, &res.algo, ws, ws_bytes,
                     stream) == CUBLAS_STATUS_SUCCESS)
    st = GDN_OK;
done:
  if (pref) cublasLtMatmulPreferenceDestroy(pref);
  if (Dd) cublasLtMatrixLayoutDestroy(Dd);
  if (Bd) cublasLtMatrixLayoutDestroy(Bd);
  if (Ad) cublasLtMatrixLayoutDestroy(Ad);
  if (op) cublasLtMatmulDescDestroy(op);
  return st;
}

size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }
constexpr size_t kLtWorkspace = 32u << 20;

}  // namespace

size_t gr_read_workspace_bytes(int64_t T, int32_t n_r, int32_t d, int32_t rank) {
  const size_t nd = (size_t)n_r * d;
  return 2 * a256((size_t)T * nd * 2) + a256((size_t)T * (rank + 8) * 2) +
         a256((size_t)(rank + 8) * nd * 2) + kLtWorkspace;
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
  void* lt_ws = Wdw + a256((size_t)ldh * nd * 2);
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
  // H'^T (col-major ldh x T) = [W_d; W_w; 0] R^^T, alpha = 1/n_r
  st = lt_gemm(ldh, (int)a.T, (int)nd, 1.f / (float)a.n_r, Wdw, (int)nd, a.rhat, (int)nd, H, ldh,
               lt_ws, kLtWorkspace, stream);
  if (st != GDN_OK) return st;
  const int64_t groups = a.T * (ldh / 8);
  gr_router_kernel<<<(unsigned)((groups + kNT - 1) / kNT), kNT, 0, stream>>>(a, H, ldh);
  // L^T (col-major nd x T) = W_u (nd x rank) SiLU(H)^T
  st = lt_gemm((int)nd, (int)a.T, a.rank, 1.f, a.W_u, a.rank, H, ldh, a.logits, (int)nd, lt_ws,
               kLtWorkspace, stream);
  if (st != GDN_OK) return st;
  const int64_t g2 = a.T * (a.d / 8);
  gr_gate_kernel<<<(unsigned)((g2 + kNT - 1) / kNT), kNT, 0, stream>>>(a);
  return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status launch_gr_write(const GrWriteArgs& a, cudaStream_t stream) {
  const int64_t rows = a.T * a.n_r;
  if (rows == 0) return GDN_OK;
  return launch_rows<WriteK>(a, rows, a.d, stream);
}

}  // namespace gdn
