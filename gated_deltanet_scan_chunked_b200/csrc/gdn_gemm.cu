// bf16 "TN" GEMM on the 5th-generation tensor cores, for the Gated Residual
// read's low-rank router ("Qwen3.8-Flash-Next: architecture, efficiency and
// technical lineage", section 05 "Residual design", the "Low-rank router"
// box: G = sigmoid(W_u SiLU((1/n_r) W_d vec(R^))), and the write scalars
// s = 2 sigmoid((1/n_r) W_w vec(R^))):
//
//   D[M][N] = alpha * A[M][K] B[N][K]^T      (row-major, bf16 in and out,
//                                             fp32 accumulation)
//
// One CTA per 128 x BN tile of D:
//   - a producer thread streams 64-wide K slices of A and B into a ring of
//     shared-memory stages by TMA (2-D tensor maps, 128-byte swizzle; rows
//     and columns past the matrix read as zeros);
//   - an MMA thread issues tcgen05.mma (kind::f16, M = 128, N = BN, K = 16
//     per instruction, both operands K-major from shared memory) into an
//     fp32 accumulator in tensor memory and returns each stage with
//     tcgen05.commit;
//   - four epilogue warps read the accumulator back (tcgen05.ld, one warp per
//     32 TMEM lanes = 32 rows), scale by alpha, round to bf16 and store the
//     rows inside the matrix.
// Every wait is bounded; one that runs out sets the library's device error
// word and the CTA drains and frees its tensor memory.
#include <cuda.h>
#include <cuda_bf16.h>

#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kBM = 128;       // rows of a D tile (TMEM lanes)
constexpr int kBK = 64;        // K per stage (one 128-byte swizzle row of bf16)
constexpr int kEpiWarps = 4;   // warps 0-3: epilogue; warp 4: TMA; warp 5: MMA
constexpr int kThreads = 32 * (kEpiWarps + 2);
constexpr uint32_t kWait = 1u << 24;
constexpr uint32_t kDrain = 1u << 16;

template <int BN, int S>
struct GemmSmem {
  static constexpr uint32_t kA = kBM * kBK * 2;   // 16 KB
  static constexpr uint32_t kB = BN * kBK * 2;
  static constexpr uint32_t kStage = kA + kB;
  static constexpr uint32_t kBars = S * kStage;  // full[S], empty[S], done, TMEM slot
  static constexpr uint32_t kBytes = kBars + 8 * (2 * S + 1) + 16 + 1024;
};

struct GemmParams {
  CUtensorMap ta, tb;  // A [M][K], B [N][K] bf16, boxes 64 (K) x 128 / BN rows
  __nv_bfloat16* D;    // bf16 result (one K split)
  float* P;            // fp32 partial results [splits][M][N] (several K splits)
  int64_t ldd;
  int M, N, K;
  int kc;              // K per split (a multiple of 64)
  float alpha;
  int* err;
};

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Grid: (M tiles, N tiles, K splits).  With one split the epilogue writes
// alpha * acc in bf16 to D; with several, split z writes its fp32 partial
// product to P[z] and a second kernel sums the splits in order.
template <int BN, int kStages>
__global__ void __launch_bounds__(kThreads, 1) gemm_tn_kernel(const __grid_constant__ GemmParams p) {
  using L = GemmSmem<BN, kStages>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;  // 128-byte swizzle wants 1024-byte alignment
  uint8_t* gb = smem_raw + (sb - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(gb + L::kBars);
  uint64_t* empty = full + kStages;
  uint64_t* done = empty + kStages;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int m0 = blockIdx.x * kBM, n0 = blockIdx.y * BN;
  const int k_begin = blockIdx.z * p.kc;
  const int k_len = p.K - k_begin < p.kc ? p.K - k_begin : p.kc;
  const int kt_n = (k_len + kBK - 1) / kBK;

  if (warp == 0) tmem_alloc(tslot, BN);
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    fence_mbar_init();
  }
  if (tid == 32 * kEpiWarps) {
    prefetch_tmap(&p.ta);
    prefetch_tmap(&p.tb);
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tacc = *tslot;

  if (warp == kEpiWarps) {
    // ---- producer ----
    if ((tid & 31) == 0) {
      bool ok = true;
      int issued = 0;
      for (int kt = 0; kt < kt_n && ok; ++kt) {
        const int s = kt % kStages;
        if (kt >= kStages) ok = mbar_wait(&empty[s], (uint32_t)((kt / kStages) - 1) & 1u, kWait);
        if (!ok) break;
        const uint32_t st = sb + s * L::kStage;
        mbar_arrive_expect_tx(&full[s], L::kStage);
        tma_load_2d(st, &p.ta, k_begin + kt * kBK, m0, &full[s]);
        tma_load_2d(st + L::kA, &p.tb, k_begin + kt * kBK, n0, &full[s]);
        issued = kt + 1;
      }
      if (!ok) {
        atomicOr(p.err, kErrTimeout);
        // the copies of the last k steps issued get a short bounded chance to
        // land before the CTA exits (k step kt completes phase kt / S of its stage)
        for (int kt = issued - kStages < 0 ? 0 : issued - kStages; kt < issued; ++kt)
          mbar_wait(&full[kt % kStages], (uint32_t)(kt / kStages) & 1u, kDrain);
      }
    }
  } else if (warp == kEpiWarps + 1) {
    // ---- MMA issuer ----
    if ((tid & 31) == 0) {
      constexpr uint32_t idesc = idesc_f16(kBM, BN, false, false, false, false);
      bool ok = true;
      for (int kt = 0; kt < kt_n && ok; ++kt) {
        const int s = kt % kStages;
        ok = mbar_wait(&full[s], (uint32_t)(kt / kStages) & 1u, kWait);
        if (!ok) break;
        fence_after_sync();
        const uint32_t st = sb + s * L::kStage;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          mma_f16(tacc, sdesc(st + kk * 32, 16, 1024), sdesc(st + L::kA + kk * 32, 16, 1024),
                  idesc, (kt > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty[s]);  // the stage returns once its products are done
      }
      if (ok) {
        mma_commit(done);
      } else {
        atomicOr(p.err, kErrTimeout);
        mma_commit(done);  // the epilogue still gets its arrival (its result is discarded)
      }
    }
  } else {
    // ---- epilogue: warp w reads TMEM lanes (rows) 32 w .. 32 w + 31 ----
    const bool ok = mbar_wait(done, 0u, kWait);
    fence_after_sync();
    const int row = m0 + 32 * warp + (tid & 31);
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    if (!ok) {
      if ((tid & 31) == 0) atomicOr(p.err, kErrTimeout);
    } else {
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        float v[32];
        tmem_ld32(tacc + lane_off + c0, v);
        tmem_wait_ld();
        if (row < p.M && p.P != nullptr) {
          float* dst = p.P + ((size_t)blockIdx.z * p.M + row) * p.N + n0 + c0;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (n0 + c0 + 4 * q < p.N)
              *reinterpret_cast<float4*>(dst + 4 * q) =
                  make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        } else if (row < p.M) {
          __nv_bfloat16* dst = p.D + (size_t)row * p.ldd + n0 + c0;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            // 8 columns (16 bytes); N is a multiple of 8, so a chunk is
            // wholly inside or wholly outside the matrix
            if (n0 + c0 + 8 * q < p.N) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(p.alpha * v[8 * q + 2 * e],
                                                                 p.alpha * v[8 * q + 2 * e + 1]);
                w[e] = *reinterpret_cast<const uint32_t*>(&h2);
              }
              *reinterpret_cast<uint4*>(dst + 8 * q) = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tacc, BN);
}

// D = bf16(alpha * sum over the splits of P, in split order); one thread per
// 8 columns of a row.
__global__ void __launch_bounds__(256) gemm_splitk_reduce_kernel(const float* P, int splits, int M,
                                                                 int N, float alpha,
                                                                 __nv_bfloat16* D, int64_t ldd) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int per_row = N / 8;
  if (g >= (int64_t)M * per_row) return;
  const int row = (int)(g / per_row), c = (int)(g % per_row) * 8;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int z = 0; z < splits; ++z) {
    const float* src = P + ((size_t)z * M + row) * N + c;
    const float4 a = *reinterpret_cast<const float4*>(src);
    const float4 b = *reinterpret_cast<const float4*>(src + 4);
    acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
    acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
  }
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat162 h2 = __floats2bfloat162_rn(alpha * acc[2 * e], alpha * acc[2 * e + 1]);
    w[e] = *reinterpret_cast<const uint32_t*>(&h2);
  }
  *reinterpret_cast<uint4*>(D + (size_t)row * ldd + c) = make_uint4(w[0], w[1], w[2], w[3]);
}

// ---- host ---------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn gemm_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// [rows][cols] bf16 with row stride `ld` elements; boxes of 64 columns x `box_rows`
bool make_tmap_2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld,
                  int box_rows) {
  EncodeTiledFn fn = gemm_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int gemm_bn(int N) { return N <= 64 ? 64 : 128; }

// K splits: enough CTAs for two per SM on a 148-SM part when the tile grid
// alone gives fewer, each split keeping at least eight 64-wide K steps.
int gemm_splits(int M, int N, int K) {
  const int tiles = ((M + kBM - 1) / kBM) * ((N + gemm_bn(N) - 1) / gemm_bn(N));
  int s = 1;
  while (s < 8 && tiles * s < 296 && K / (kBK * (s * 2)) >= 8) s *= 2;
  return s;
}

template <int BN, int S>
gdn_status launch_bn(const GemmParams& prm, int splits, cudaStream_t stream) {
  using L = GemmSmem<BN, S>;
  static bool attr_set[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    if (cudaFuncSetAttribute(gemm_tn_kernel<BN, S>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)L::kBytes) != cudaSuccess)
      return GDN_ERR_CUDA;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const dim3 grid((unsigned)((prm.M + kBM - 1) / kBM), (unsigned)((prm.N + BN - 1) / BN),
                  (unsigned)splits);
  gemm_tn_kernel<BN, S><<<grid, kThreads, L::kBytes, stream>>>(prm);
  return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace

// D[M][N] = alpha A[M][K] B[N][K]^T, bf16 row-major with leading dimensions
// lda / ldb / ldd (elements).  Requirements (else GDN_ERR_UNSUPPORTED): K and
// N multiples of 8, leading dimensions multiples of 8, 16-byte aligned
// pointers.  Products with at most 64 columns take 64-column tiles.
size_t gemm_tn_workspace_bytes(int M, int N, int K) {
  return (size_t)gemm_splits(M, N, K) * (size_t)M * (size_t)N * sizeof(float);
}

gdn_status gemm_tn_bf16(int M, int N, int K, float alpha, const void* A, int64_t lda,
                        const void* B, int64_t ldb, void* D, int64_t ldd, void* ws,
                        size_t ws_bytes, cudaStream_t stream) {
  if (M <= 0 || N <= 0) return GDN_OK;
  if (K <= 0 || K % 8 || N % 8 || lda % 8 || ldb % 8 || ldd % 8 || lda < K || ldb < K ||
      ldd < N)
    return GDN_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B) |
       reinterpret_cast<uintptr_t>(D)) & 15u)
    return GDN_ERR_UNSUPPORTED;
  GemmParams prm;
  const int bn = gemm_bn(N);
  int splits = gemm_splits(M, N, K);
  if (splits > 1 && (ws == nullptr || ws_bytes < gemm_tn_workspace_bytes(M, N, K) ||
                     (reinterpret_cast<uintptr_t>(ws) & 15u)))
    splits = 1;  // no room for the partial products: one split
  if (!make_tmap_2d(&prm.ta, A, M, K, lda, kBM) || !make_tmap_2d(&prm.tb, B, N, K, ldb, bn))
    return GDN_ERR_CUDA;
  prm.D = static_cast<__nv_bfloat16*>(D);
  prm.P = splits > 1 ? static_cast<float*>(ws) : nullptr;
  prm.ldd = ldd;
  prm.M = M;
  prm.N = N;
  prm.K = K;
  prm.kc = ((K + splits * kBK - 1) / (splits * kBK)) * kBK;
  prm.alpha = alpha;
  prm.err = device_error_word();
  if (prm.err == nullptr) return GDN_ERR_CUDA;
  // short K loops (two stages suffice) leave room for more CTAs per SM, whose
  // epilogues then overlap each other's loads
  const bool short_k = prm.kc <= 8 * kBK;
  gdn_status st = bn == 64 ? (short_k ? launch_bn<64, 2>(prm, splits, stream)
                                      : launch_bn<64, 4>(prm, splits, stream))
                           : (short_k ? launch_bn<128, 2>(prm, splits, stream)
                                      : launch_bn<128, 4>(prm, splits, stream));
  if (st != GDN_OK || splits == 1) return st;
  const int64_t threads = (int64_t)M * (N / 8);
  gemm_splitk_reduce_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, stream>>>(
      prm.P, splits, M, N, alpha, prm.D, ldd);
  return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn
