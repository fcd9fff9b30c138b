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
//   gr_norm   codes -> R^ (bf16, group RMSNorm with gains) and s (fp32)
//   GEMM      H = (1/n_r) R^ W_d^T                       [T, r]
//   gr_silu   H = SiLU(H)
//   GEMM      L = H W_u^T                                 [T, n_r d]
//   gr_gate   x = (1/n_r) sum_i sigmoid(L_i) o R^_i      [T, d] bf16
// Write = one kernel, one warp per (token, branch) row, in place.
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

// 8 codes -> 8 dequantised floats (one rounded product each)
__device__ __forceinline__ void dequant8(const uint8_t* p, float scale, float* x) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  const uint32_t w[2] = {u.x, u.y};
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = __fmul_rn(e4m3_to_float((w[i / 4] >> (8 * (i % 4))) & 0xFF), scale);
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

__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();  // red free
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kNT / 32; ++w) t += red[w];
  return t;
}

// gr_norm: one CTA per token.  R^ = dequant / sqrt(mean sq + eps) * gamma
// (bf16), s = 2 sigmoid((1/n_r) W_w vec(R^)) from the fp32 R^.
__global__ void __launch_bounds__(kNT) gr_norm_kernel(const GrArgs a) {
  __shared__ float red[kNT / 32];
  __shared__ float rs[kMaxGrBranches];
  __shared__ float sacc[kMaxGrBranches];
  const int64_t t = blockIdx.x;
  const int nd = a.n_r * a.d, g8 = a.d / 8;
  const uint8_t* row = a.codes + (size_t)t * nd;
  for (int b = 0; b < a.n_r; ++b) {
    const float sc = __ldg(a.scales + (size_t)t * a.n_r + b);
    float ss = 0.f;
    for (int j = threadIdx.x; j < g8; j += kNT) {
      float x[8];
      dequant8(row + (size_t)b * a.d + 8 * j, sc, x);
#pragma unroll
      for (int i = 0; i < 8; ++i) ss += x[i] * x[i];
    }
    ss = block_sum(ss, red);
    if (threadIdx.x == 0) rs[b] = rsqrtf(ss / (float)a.d + a.eps);
  }
  __syncthreads();
  float sp[kMaxGrBranches];
#pragma unroll
  for (int k = 0; k < kMaxGrBranches; ++k) sp[k] = 0.f;
  __nv_bfloat16* out = a.rhat + (size_t)t * nd;
  for (int b = 0; b < a.n_r; ++b) {
    const float sc = __ldg(a.scales + (size_t)t * a.n_r + b);
    const float r = rs[b];
    for (int j = threadIdx.x; j < g8; j += kNT) {
      const int e = b * a.d + 8 * j;
      float x[8], gm[8];
      dequant8(row + e, sc, x);
      const float4 g0 = __ldg(reinterpret_cast<const float4*>(a.gamma + e));
      const float4 g1 = __ldg(reinterpret_cast<const float4*>(a.gamma + e) + 1);
      gm[0] = g0.x; gm[1] = g0.y; gm[2] = g0.z; gm[3] = g0.w;
      gm[4] = g1.x; gm[5] = g1.y; gm[6] = g1.z; gm[7] = g1.w;
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = x[i] * r * gm[i];
      bf16x8_store(out + e, x);
#pragma unroll
      for (int k = 0; k < kMaxGrBranches; ++k) {
        if (k < a.n_r) {
          float w[8];
          bf16x8_load(static_cast<const __nv_bfloat16*>(a.W_w) + (size_t)k * nd + e, w);
#pragma unroll
          for (int i = 0; i < 8; ++i) sp[k] += w[i] * x[i];
        }
      }
    }
  }
  for (int k = 0; k < a.n_r; ++k) {
    const float v = block_sum(sp[k], red);
    if (threadIdx.x == 0) sacc[k] = v;
  }
  __syncthreads();
  if (threadIdx.x < a.n_r)
    a.s[(size_t)t * a.n_r + threadIdx.x] = 2.f / (1.f + expf(-sacc[threadIdx.x] / (float)a.n_r));
}

__global__ void __launch_bounds__(kNT) gr_silu_kernel(__nv_bfloat16* h, int64_t n8) {
  const int64_t i = (int64_t)blockIdx.x * kNT + threadIdx.x;
  if (i >= n8) return;
  float x[8];
  bf16x8_load(h + 8 * i, x);
#pragma unroll
  for (int k = 0; k < 8; ++k) x[k] = x[k] / (1.f + expf(-x[k]));
  bf16x8_store(h + 8 * i, x);
}

// gr_gate: x[t, c] = (1/n_r) sum_i sigmoid(L[t, i d + c]) R^[t, i d + c]
__global__ void __launch_bounds__(kNT) gr_gate_kernel(const GrArgs a) {
  const int64_t idx = (int64_t)blockIdx.x * kNT + threadIdx.x;  // 8-channel group
  const int g8 = a.d / 8;
  if (idx >= a.T * g8) return;
  const int64_t t = idx / g8;
  const int c = (int)(idx % g8) * 8;
  const size_t base = (size_t)t * a.n_r * a.d + c;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  for (int b = 0; b < a.n_r; ++b) {
    float l[8], r[8];
    bf16x8_load(a.logits + base + (size_t)b * a.d, l);
    bf16x8_load(a.rhat + base + (size_t)b * a.d, r);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += r[i] / (1.f + expf(-l[i]));
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] /= (float)a.n_r;
  bf16x8_store(static_cast<__nv_bfloat16*>(a.x) + (size_t)t * a.d + c, acc);
}

// gr_write: one warp per (token, branch) row, in place.  r = deq + s y with
// one rounding per operation; scale' = max|r| / 448 (1 if zero); code =
// E4M3(r / scale') with round to nearest even and saturation.  Two passes
// over the row (the second recomputes r from the same inputs).
__global__ void __launch_bounds__(128) gr_write_kernel(const GrWriteArgs a) {
  const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= a.T * a.n_r) return;
  const int64_t t = row / a.n_r;
  uint8_t* codes = a.codes + (size_t)row * a.d;
  const __nv_bfloat16* y = static_cast<const __nv_bfloat16*>(a.y) + (size_t)t * a.d;
  const float sc = a.scales[row];
  const float sv = __ldg(a.s + row);
  const int g8 = a.d / 8;
  float amax = 0.f;
  for (int j = lane; j < g8; j += 32) {
    float q[8], yv[8];
    dequant8(codes + 8 * j, sc, q);
    bf16x8_load(y + 8 * j, yv);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(__fadd_rn(q[i], __fmul_rn(sv, yv[i]))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float nsc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  // every lane has read its old codes in the first pass; the second pass
  // rereads them before overwriting (each lane touches only its own groups)
  for (int j = lane; j < g8; j += 32) {
    float q[8], yv[8];
    dequant8(codes + 8 * j, sc, q);
    bf16x8_load(y + 8 * j, yv);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float r = __fadd_rn(q[i], __fmul_rn(sv, yv[i]));
      const uint32_t c = __nv_cvt_float_to_fp8(__fdiv_rn(r, nsc), __NV_SATFINITE, __NV_E4M3);
      w[i / 4] |= (c & 0xFFu) << (8 * (i % 4));
    }
    *reinterpret_cast<uint2*>(codes + 8 * j) = make_uint2(w[0], w[1]);
  }
  __syncwarp();
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
  return 2 * a256((size_t)T * n_r * d * 2) + a256((size_t)T * rank * 2) + kLtWorkspace;
}

gdn_status launch_gr_read(GrArgs a, void* ws, cudaStream_t stream) {
  char* p = static_cast<char*>(ws);
  const size_t nrd = (size_t)a.T * a.n_r * a.d * 2;
  a.rhat = reinterpret_cast<__nv_bfloat16*>(p);
  a.logits = reinterpret_cast<__nv_bfloat16*>(p + a256(nrd));
  __nv_bfloat16* H = reinterpret_cast<__nv_bfloat16*>(p + 2 * a256(nrd));
  void* lt_ws = p + 2 * a256(nrd) + a256((size_t)a.T * a.rank * 2);
  if (a.T == 0) return GDN_OK;
  gr_norm_kernel<<<(unsigned)a.T, kNT, 0, stream>>>(a);
  if (cudaPeekAtLastError() != cudaSuccess) return GDN_ERR_CUDA;
  const int nd = a.n_r * a.d;
  // H^T (col-major r x T) = W_d (r x nd) R^^T, alpha = 1/n_r
  gdn_status st = lt_gemm(a.rank, (int)a.T, nd, 1.f / (float)a.n_r, a.W_d, nd, a.rhat, nd, H,
                          a.rank, lt_ws, kLtWorkspace, stream);
  if (st != GDN_OK) return st;
  const int64_t n8 = a.T * a.rank / 8;
  gr_silu_kernel<<<(unsigned)((n8 + kNT - 1) / kNT), kNT, 0, stream>>>(H, n8);
  // L^T (col-major nd x T) = W_u (nd x r) H^T
  st = lt_gemm(nd, (int)a.T, a.rank, 1.f, a.W_u, a.rank, H, a.rank, a.logits, nd, lt_ws,
               kLtWorkspace, stream);
  if (st != GDN_OK) return st;
  const int64_t groups = a.T * (a.d / 8);
  gr_gate_kernel<<<(unsigned)((groups + kNT - 1) / kNT), kNT, 0, stream>>>(a);
  return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status launch_gr_write(const GrWriteArgs& a, cudaStream_t stream) {
  const int64_t rows = a.T * a.n_r;
  if (rows == 0) return GDN_OK;
  gr_write_kernel<<<(unsigned)((rows + 3) / 4), 128, 0, stream>>>(a);
  return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn
