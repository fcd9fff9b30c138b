// Internal interface between the host entry points (gdn_api.cu) and the
// kernel translation units.  Not installed; not part of the C ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn.h"

namespace gdn {

// Bits of the device-side error word.
enum : int {
  kErrTimeout = 1,      // a bounded wait ran out
  kErrBadSeqlens = 2,   // cu_seqlens not monotone / out of range
};

struct PrefillArgs {
  const void* q;
  const void* k;
  const void* v;
  const float* log_alpha;
  const float* beta;
  const void* g;           // nullptr: no epilogue
  const float* norm_w;     // nullptr: zeros
  const float* initial_state;  // nullptr: zeros
  const int32_t* cu_seqlens;   // nullptr: one sequence of total_T tokens
  float* final_state;      // nullptr: not written
  void* y;
  int32_t n_seq;
  int64_t total_T;
  int32_t H_qk, H_v, d_k, d_v;
  gdn_dtype dtype;
  int32_t l2norm;
  float eps_l2, eps_norm, scale;
  int* err;                // device error word
  int tc_variant;          // tensor kernel: 0 auto, 1 CTA pairs, 2 one CTA per head, 3 scan layout
  // Scan-layout workspace (nullptr: none): hand-off ring slots and their
  // flags, placed by prefill_tc_workspace_layout (sizes: scan_ws_bytes).
  void* ring = nullptr;
  unsigned long long* ring_flags = nullptr;
  // Larger batches with a workspace: the order in which the one-CTA layout
  // takes the sequences, longest first (nullptr: in index order).
  int32_t* seq_order = nullptr;
  // Front end fused into the portable kernel (nullptr: q, k, v are used as
  // given): conv weights [2 H_qk d_k + H_v d_v, 4] and the per-value-head conv
  // states [n_seq, H_v, 3, 2 d_k + d_v] before / after each sequence.
  const float* conv_w = nullptr;
  const float* conv_state_in = nullptr;
  float* conv_state_out = nullptr;
};

// Tokens per launch of the multi-token decode (its inputs are staged in
// shared memory: ~4.1 KB per token at d_k = d_v = 128).
constexpr int kMaxDecodeTokens = 32;

struct DecodeArgs {
  const void* q;           // [N, T_s, H_qk, d_k]
  const void* k;
  const void* v;           // [N, T_s, H_v, d_v]
  const float* log_alpha;  // [N, T_s, H_v]
  const float* beta;
  const void* g;           // [N, T_s, H_v, d_v] or nullptr
  const float* norm_w;
  const float* state_in;   // [N, H_v, d_k, d_v]
  float* state_out;        // same shape, may be state_in; nullptr: not written
  float* snapshots;        // [T_s, N, H_v, d_k, d_v] or nullptr: state after each token
  void* y;                 // [N, T_s, H_v, d_v]
  const float* conv_w = nullptr;  // [2 H_qk d_k + H_v d_v, 4]: q, k, v pass the front end
  float* conv_state = nullptr;    // [N, H_v, 3, 2 d_k + d_v], read and rewritten; nullptr: zeros
  int32_t N, T_s, H_qk, H_v, d_k, d_v;
  gdn_dtype dtype;
  int32_t l2norm;
  float eps_l2, eps_norm, scale;
};

struct BwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const float* log_alpha;
  const float* beta;
  const void* g;               // nullptr: no epilogue
  const float* norm_w;         // nullptr: zeros
  const float* initial_state;  // nullptr: zeros
  const int32_t* cu_seqlens;   // nullptr: one sequence
  const void* dy;              // [total_T, H_v, d_v], input dtype
  const float* d_final_state;  // nullptr: zeros
  float* dq;                   // [total_T, H_qk, d_k]
  float* dk;
  float* dv;                   // [total_T, H_v, d_v]
  float* dlog_alpha;           // [total_T, H_v]
  float* dbeta;
  float* dg;                   // [total_T, H_v, d_v] (with g)
  float* dnorm_w;              // [d_v] (with g) or nullptr
  float* d_initial_state;      // [n_seq, H_v, d_k, d_v] or nullptr
  int32_t n_seq;
  int64_t total_T;
  int32_t H_qk, H_v, d_k, d_v;
  gdn_dtype dtype;
  int32_t l2norm;
  float eps_l2, eps_norm, scale;
  int* err;
  // workspace parts, placed by chunk_bwd_workspace_layout
  void* chunks;
  int32_t* seq_first;
  float *S, *dS, *W, *WT, *UT, *D, *dD, *T, *KKE, *P, *dPE, *Bm, *G, *row, *dw, *dO, *dqh,
      *dkh, *qh, *kh;
};

struct ConvArgs {
  const void* q;               // [total_T, H_qk, d_k] input dtype (before the front end)
  const void* k;
  const void* v;               // [total_T, H_v, d_v]
  const float* conv_w;         // [2 H_qk d_k + H_v d_v, 4]
  const float* state_in;       // [n_seq, H_v, 3, 2 d_k + d_v] or nullptr (zeros)
  float* state_out;            // same shape or nullptr; must not overlap state_in
  const int32_t* cu_seqlens;   // nullptr: one sequence
  int32_t n_seq;
  int64_t total_T;
  int32_t H_qk, H_v, d_k, d_v;
  gdn_dtype dtype;
  void* q_out;                 // outputs, input dtype, shapes of q, k, v
  void* k_out;
  void* v_out;
  int* err;
};

gdn_status launch_conv(const ConvArgs& a, cudaStream_t stream);

// Gated Residual read / write over an E4M3 residual state.
constexpr int kMaxGrBranches = 8;

struct GrArgs {
  const uint8_t* codes;   // [T, n_r, d] E4M3
  const float* scales;    // [T, n_r]
  const float* gamma;     // [n_r, d]
  const void* W_d;        // [rank, n_r d] bf16
  const void* W_u;        // [n_r d, rank] bf16
  const void* W_w;        // [n_r, n_r d] bf16
  int64_t T;
  int32_t n_r, d, rank;
  float eps;
  void* x;                // [T, d] bf16
  float* s;               // [T, n_r]
  __nv_bfloat16* rhat = nullptr;    // workspace: [T, n_r d]
  __nv_bfloat16* logits = nullptr;  // workspace: [T, n_r d]
};

struct GrWriteArgs {
  uint8_t* codes;         // [T, n_r, d], rewritten
  float* scales;          // [T, n_r], rewritten
  const void* y;          // [T, d] bf16
  const float* s;         // [T, n_r]
  int64_t T;
  int32_t n_r, d;
};

size_t gr_read_workspace_bytes(int64_t T, int32_t n_r, int32_t d, int32_t rank);

// The library's device error word on the current device (nullptr on failure).
int* device_error_word();

// D[M][N] = alpha A[M][K] B[N][K]^T: bf16 row-major operands with leading
// dimensions in elements, fp32 accumulation on the tensor cores
// (gdn_gemm.cu).  K, N and the leading dimensions multiples of 8, pointers
// 16-byte aligned, else GDN_ERR_UNSUPPORTED.  Products with few output tiles
// split K over several CTAs; their fp32 partials need `ws` (16-byte aligned,
// gemm_tn_workspace_bytes), without which K is not split.
size_t gemm_tn_workspace_bytes(int M, int N, int K);
gdn_status gemm_tn_bf16(int M, int N, int K, float alpha, const void* A, int64_t lda,
                        const void* B, int64_t ldb, void* D, int64_t ldd, void* ws,
                        size_t ws_bytes, cudaStream_t stream);
gdn_status launch_gr_read(GrArgs a, void* ws, cudaStream_t stream);
gdn_status launch_gr_write(const GrWriteArgs& a, cudaStream_t stream);

size_t chunk_bwd_workspace_bytes(int32_t n_seq, int64_t total_T, int32_t H_qk, int32_t H_v,
                                 int32_t d_k, int32_t d_v);
void chunk_bwd_workspace_layout(void* ws, BwdArgs* a);
gdn_status launch_chunk_bwd(const BwdArgs& a, cudaStream_t stream);

// Argument checks shared by the entry points: head counts and grouping, dims
// and epsilons (GDN_ERR_INVALID_ARG), then dtype and compiled dims
// (GDN_ERR_UNSUPPORTED).
gdn_status check_common(int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v, gdn_dtype dt,
                        float eps_l2, float eps_norm);

// Each launcher returns GDN_OK, GDN_ERR_UNSUPPORTED (shape not compiled) or
// GDN_ERR_CUDA (launch failed).
gdn_status launch_decode(const DecodeArgs& a, cudaStream_t stream);
gdn_status launch_prefill_simt(const PrefillArgs& a, cudaStream_t stream);
gdn_status launch_prefill_tc(const PrefillArgs& a, cudaStream_t stream);
bool prefill_tc_supports(const PrefillArgs& a);
// Workspace bytes the tensor kernel can use for n_seq x H_v items (the scan
// layout's ring for small batches, the one-CTA layout's sequence order for
// larger ones; 0 when neither applies), and the placement of its parts
// within a 256-byte aligned workspace.
size_t prefill_tc_workspace_bytes(int32_t n_seq, int32_t H_v, int32_t d_k, int32_t d_v,
                                  gdn_dtype dtype);

// Workspace of the tensor-core prefill's scan layout (small batches) for
// `items` (sequence, value head) items: per item kScanRing "ready" and
// kScanRing "consumed" flags (64-bit), the whole flag block padded to 256
// bytes, then per item kScanRing hand-off slots of kScanSlotBytes (a
// multiple of 256).
constexpr int kScanRing = 8;
constexpr size_t kScanSlotBytes = 73984;
constexpr long long kScanMaxItems = 64;
constexpr size_t scan_flag_bytes(long long items) {
  return ((size_t)items * 2 * kScanRing * sizeof(unsigned long long) + 255) & ~(size_t)255;
}
constexpr size_t scan_ws_bytes(long long items) {
  return scan_flag_bytes(items) + (size_t)items * kScanRing * kScanSlotBytes;
}
// Co-resident items of the scan layout on this device (0: unavailable), and
// its launch (needs the workspace placed in a.ring / a.ring_flags).
int prefill_scan_capacity();
gdn_status launch_prefill_scan(const PrefillArgs& a, cudaStream_t stream);
void prefill_tc_workspace_layout(void* ws, int32_t n_seq, int32_t H_v, PrefillArgs* a);

}  // namespace gdn
