// Host entry points of libgdn: argument validation, kernel selection and the
// device-side error word.  See include/gdn.h for the contract of each call.
#include <cuda_runtime.h>

#include <mutex>

#include "gdn_internal.h"
#include "gdn_sm100.cuh"

namespace gdn {
namespace {

// A hand-off flag that nothing ever sets, for the bounded-wait self-test.
__device__ unsigned long long g_never_set = 0;

// One CTA waits on g_never_set with the library's bounded wait (the one the
// scan-layout prefill uses for its hand-off flags), gives up after `iters` polls,
// records the timeout in the error word and returns.
__global__ void selftest_wait_kernel(int* err, uint32_t iters) {
  if (threadIdx.x != 0) return;
  if (!sm100::wait_flag_ge(&g_never_set, 1ull, iters)) atomicOr(err, kErrTimeout);
}

// One error word per device.  Kernels OR bits into it (a bounded wait that
// ran out, a malformed cu_seqlens); gdn_check_device_error reads and clears.
__device__ int g_error_word = 0;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int* g_err_ptr[kMaxDevices] = {nullptr};

int* error_word_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_err_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<int*>(p);
  }
  return g_err_ptr[dev];
}

bool dim_ok(int32_t d) { return d == 16 || d == 32 || d == 64 || d == 128; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

int* device_error_word() { return error_word_ptr(); }

gdn_status check_common(int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v, gdn_dtype dt,
                        float eps_l2, float eps_norm) {
  if (H_qk <= 0 || H_v <= 0 || H_v % H_qk != 0) return GDN_ERR_INVALID_ARG;
  if (d_k <= 0 || d_v <= 0) return GDN_ERR_INVALID_ARG;
  if (!(eps_l2 >= 0.f) || !(eps_norm >= 0.f)) return GDN_ERR_INVALID_ARG;
  if (dt != GDN_BF16 && dt != GDN_FP32) return GDN_ERR_UNSUPPORTED;
  if (!dim_ok(d_k) || !dim_ok(d_v)) return GDN_ERR_UNSUPPORTED;
  return GDN_OK;
}

}  // namespace gdn

using namespace gdn;

namespace {

// gdn_chunk_fwd_ws, optionally with the front end fused into the portable
// kernel (conv_w non-null: only the portable path takes it).
gdn_status chunk_fwd_impl(
    const void* q, const void* k, const void* v, const float* log_alpha, const float* beta,
    const void* g, const float* norm_w, const float* initial_state, const int32_t* cu_seqlens,
    int32_t n_seq, int64_t total_T, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
    gdn_dtype in_dtype, int32_t l2norm_qk, float eps_l2, float eps_norm, float scale, void* y,
    float* final_state, gdn_prefill_path path, void* workspace, size_t workspace_bytes,
    gdn_stream_t stream, const float* conv_w, const float* conv_state_in,
    float* conv_state_out) {
  gdn_status st = check_common(H_qk, H_v, d_k, d_v, in_dtype, eps_l2, eps_norm);
  if (st != GDN_OK) return st;
  if (n_seq < 1 || total_T < 0) return GDN_ERR_INVALID_ARG;
  if (cu_seqlens == nullptr && n_seq != 1) return GDN_ERR_INVALID_ARG;
  if ((int64_t)n_seq * H_v > 0x7fffffffLL) return GDN_ERR_INVALID_ARG;
  if (total_T > 0 && (!q || !k || !v || !log_alpha || !beta || !y)) return GDN_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, log_alpha, beta, g, norm_w, initial_state, y, final_state};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return GDN_ERR_INVALID_ARG;
  if (initial_state && final_state && initial_state != final_state) {
    // exact aliasing is allowed; partial overlap is not
    const char* a0 = reinterpret_cast<const char*>(initial_state);
    const char* b0 = reinterpret_cast<const char*>(final_state);
    const size_t bytes = (size_t)n_seq * H_v * d_k * d_v * sizeof(float);
    if (a0 < b0 + bytes && b0 < a0 + bytes) return GDN_ERR_INVALID_ARG;
  }
  if (path != GDN_PATH_AUTO && path != GDN_PATH_TENSOR && path != GDN_PATH_SIMT &&
      path != GDN_PATH_TENSOR_PAIR && path != GDN_PATH_TENSOR_SINGLE &&
      path != GDN_PATH_TENSOR_SPLIT)
    return GDN_ERR_INVALID_ARG;
  const size_t ws_need = prefill_tc_workspace_bytes(n_seq, H_v, d_k, d_v, in_dtype);
  if (workspace != nullptr) {
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDN_ERR_INVALID_ARG;
    if (workspace_bytes < ws_need) return GDN_ERR_INVALID_ARG;
  }
  if (path == GDN_PATH_TENSOR_SPLIT && (workspace == nullptr || ws_need == 0))
    return workspace == nullptr && ws_need != 0 ? GDN_ERR_INVALID_ARG : GDN_ERR_UNSUPPORTED;

  PrefillArgs a;
  a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
  a.g = g; a.norm_w = g ? norm_w : nullptr;
  a.initial_state = initial_state; a.cu_seqlens = cu_seqlens; a.final_state = final_state;
  a.y = y; a.n_seq = n_seq; a.total_T = total_T;
  a.H_qk = H_qk; a.H_v = H_v; a.d_k = d_k; a.d_v = d_v; a.dtype = in_dtype;
  a.l2norm = l2norm_qk ? 1 : 0; a.eps_l2 = eps_l2; a.eps_norm = eps_norm; a.scale = scale;
  a.tc_variant = path == GDN_PATH_TENSOR_PAIR     ? 1
                 : path == GDN_PATH_TENSOR_SINGLE ? 2
                 : path == GDN_PATH_TENSOR_SPLIT  ? 3
                                                  : 0;
  if (workspace != nullptr && ws_need != 0) prefill_tc_workspace_layout(workspace, n_seq, H_v, &a);

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool tc_ok = prefill_tc_supports(a);
  const bool want_tc = path == GDN_PATH_TENSOR || path == GDN_PATH_TENSOR_PAIR ||
                       path == GDN_PATH_TENSOR_SINGLE || path == GDN_PATH_TENSOR_SPLIT;
  if (want_tc && !tc_ok) return GDN_ERR_UNSUPPORTED;
  a.err = error_word_ptr();
  if (a.err == nullptr) return GDN_ERR_CUDA;
  if (conv_w != nullptr) {
    if (path != GDN_PATH_SIMT) return GDN_ERR_UNSUPPORTED;
    a.conv_w = conv_w; a.conv_state_in = conv_state_in; a.conv_state_out = conv_state_out;
    return launch_prefill_simt(a, s);
  }
  if (want_tc || (path == GDN_PATH_AUTO && tc_ok)) return launch_prefill_tc(a, s);
  return launch_prefill_simt(a, s);
}

}  // namespace

extern "C" gdn_status gdn_chunk_fwd_ws(
    const void* q, const void* k, const void* v, const float* log_alpha, const float* beta,
    const void* g, const float* norm_w, const float* initial_state, const int32_t* cu_seqlens,
    int32_t n_seq, int64_t total_T, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
    gdn_dtype in_dtype, int32_t l2norm_qk, float eps_l2, float eps_norm, float scale, void* y,
    float* final_state, gdn_prefill_path path, void* workspace, size_t workspace_bytes,
    gdn_stream_t stream) {
  return chunk_fwd_impl(q, k, v, log_alpha, beta, g, norm_w, initial_state, cu_seqlens, n_seq,
                        total_T, H_qk, H_v, d_k, d_v, in_dtype, l2norm_qk, eps_l2, eps_norm, scale,
                        y, final_state, path, workspace, workspace_bytes, stream, nullptr,
                        nullptr, nullptr);
}

extern "C" gdn_status gdn_chunk_fwd_path(
    const void* q, const void* k, const void* v, const float* log_alpha, const float* beta,
    const void* g, const float* norm_w, const float* initial_state, const int32_t* cu_seqlens,
    int32_t n_seq, int64_t total_T, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
    gdn_dtype in_dtype, int32_t l2norm_qk, float eps_l2, float eps_norm, float scale, void* y,
    float* final_state, gdn_prefill_path path, gdn_stream_t stream) {
  return gdn_chunk_fwd_ws(q, k, v, log_alpha, beta, g, norm_w, initial_state, cu_seqlens, n_seq,
                          total_T, H_qk, H_v, d_k, d_v, in_dtype, l2norm_qk, eps_l2, eps_norm,
                          scale, y, final_state, path, nullptr, 0, stream);
}

extern "C" size_t gdn_chunk_fwd_workspace_size(int32_t n_seq, int32_t H_v, int32_t d_k,
                                               int32_t d_v, gdn_dtype in_dtype) {
  if (n_seq < 1 || H_v < 1) return 0;
  return prefill_tc_workspace_bytes(n_seq, H_v, d_k, d_v, in_dtype);
}

extern "C" gdn_status gdn_chunk_fwd(
    const void* q, const void* k, const void* v, const float* log_alpha, const float* beta,
    const void* g, const float* norm_w, const float* initial_state, const int32_t* cu_seqlens,
    int32_t n_seq, int64_t total_T, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
    gdn_dtype in_dtype, int32_t l2norm_qk, float eps_l2, float eps_norm, float scale, void* y,
    float* final_state, gdn_stream_t stream) {
  return gdn_chunk_fwd_path(q, k, v, log_alpha, beta, g, norm_w, initial_state, cu_seqlens,
                            n_seq, total_T, H_qk, H_v, d_k, d_v, in_dtype, l2norm_qk, eps_l2,
                            eps_norm, scale, y, final_state, GDN_PATH_AUTO, stream);
}

namespace {

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b) return false;
  const char* x = static_cast<const char*>(a);
  const char* y = static_cast<const char*>(b);
  return x < y + nb && y < x + na;
}

gdn_status decode_impl(const void* q, const void* k, const void* v, const float* log_alpha,
                       const float* beta, const void* g, const float* norm_w,
                       const float* conv_w, float* conv_state, const float* state_in,
                       float* state_out, float* snapshots, int32_t N, int32_t T_s, int32_t H_qk,
                       int32_t H_v, int32_t d_k, int32_t d_v, gdn_dtype in_dtype,
                       int32_t l2norm_qk, float eps_l2, float eps_norm, float scale, void* y,
                       gdn_stream_t stream) {
  gdn_status st = check_common(H_qk, H_v, d_k, d_v, in_dtype, eps_l2, eps_norm);
  if (st != GDN_OK) return st;
  if (N < 0 || T_s < 0 || (int64_t)N * H_v > 0x7fffffffLL) return GDN_ERR_INVALID_ARG;
  if (T_s > kMaxDecodeTokens) return GDN_ERR_UNSUPPORTED;
  if (N == 0 || T_s == 0) return GDN_OK;
  if (!q || !k || !v || !log_alpha || !beta || !state_in || !y) return GDN_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, log_alpha, beta, g, norm_w, state_in, state_out, snapshots, y};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  const size_t sbytes = (size_t)N * H_v * d_k * d_v * sizeof(float);
  if (state_out && state_out != state_in) {
    // exact aliasing is allowed; partial overlap is not
    const char* a0 = reinterpret_cast<const char*>(state_in);
    const char* b0 = reinterpret_cast<const char*>(state_out);
    if (a0 < b0 + sbytes && b0 < a0 + sbytes) return GDN_ERR_INVALID_ARG;
  }
  if (snapshots) {
    // snapshots may not overlap either state
    const char* s0 = reinterpret_cast<const char*>(snapshots);
    const size_t nb = sbytes * (size_t)T_s;
    const float* states[] = {state_in, state_out};
    for (const float* x : states) {
      const char* x0 = reinterpret_cast<const char*>(x);
      if (x && x0 < s0 + nb && s0 < x0 + sbytes) return GDN_ERR_INVALID_ARG;
    }
  }
  DecodeArgs a;
  a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
  a.g = g; a.norm_w = g ? norm_w : nullptr;
  a.state_in = state_in; a.state_out = state_out; a.snapshots = snapshots; a.y = y;
  a.N = N; a.T_s = T_s; a.H_qk = H_qk; a.H_v = H_v; a.d_k = d_k; a.d_v = d_v;
  a.dtype = in_dtype;
  a.l2norm = l2norm_qk ? 1 : 0; a.eps_l2 = eps_l2; a.eps_norm = eps_norm; a.scale = scale;
  a.conv_w = conv_w; a.conv_state = conv_state;
  return launch_decode(a, reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" gdn_status gdn_decode_multi(
    const void* q, const void* k, const void* v, const float* log_alpha, const float* beta,
    const void* g, const float* norm_w, const float* state_in, float* state_out,
    float* snapshots, int32_t N, int32_t T_s, int32_t H_qk, int32_t H_v, int32_t d_k,
    int32_t d_v, gdn_dtype in_dtype, int32_t l2norm_qk, float eps_l2, float eps_norm,
    float scale, void* y, gdn_stream_t stream) {
  return decode_impl(q, k, v, log_alpha, beta, g, norm_w, nullptr, nullptr, state_in, state_out,
                     snapshots, N, T_s, H_qk, H_v, d_k, d_v, in_dtype, l2norm_qk, eps_l2,
                     eps_norm, scale, y, stream);
}

extern "C" gdn_status gdn_decode_conv(
    const void* q, const void* k, const void* v, const float* conv_w, float* conv_state,
    const float* log_alpha, const float* beta, const void* g, const float* norm_w,
    const float* state_in, float* state_out, float* snapshots, int32_t N, int32_t T_s,
    int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v, gdn_dtype in_dtype, int32_t l2norm_qk,
    float eps_l2, float eps_norm, float scale, void* y, gdn_stream_t stream) {
  if (N > 0 && T_s > 0 && conv_w == nullptr) return GDN_ERR_INVALID_ARG;
  if ((conv_w && !aligned16(conv_w)) || (conv_state && !aligned16(conv_state)))
    return GDN_ERR_INVALID_ARG;
  if (conv_state) {
    // the conv state may not overlap the recurrent states or the snapshots
    const size_t cb = (size_t)N * H_v * 3 * (2 * d_k + d_v) * sizeof(float);
    const size_t sb = (size_t)N * H_v * d_k * d_v * sizeof(float);
    if (overlaps(conv_state, cb, state_in, sb) || overlaps(conv_state, cb, state_out, sb) ||
        overlaps(conv_state, cb, snapshots, sb * (size_t)(T_s > 0 ? T_s : 0)))
      return GDN_ERR_INVALID_ARG;
  }
  return decode_impl(q, k, v, log_alpha, beta, g, norm_w, conv_w, conv_state, state_in,
                     state_out, snapshots, N, T_s, H_qk, H_v, d_k, d_v, in_dtype, l2norm_qk,
                     eps_l2, eps_norm, scale, y, stream);
}

namespace {

size_t conv_buffers_bytes(int64_t total_T, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
                          gdn_dtype dt) {
  const size_t e = dt == GDN_BF16 ? 2 : 4;
  auto a256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return 2 * a256((size_t)total_T * H_qk * d_k * e) + a256((size_t)total_T * H_v * d_v * e);
}

gdn_status conv_impl(const void* q, const void* k, const void* v, const float* conv_w,
                     const float* conv_state_in, float* conv_state_out,
                     const int32_t* cu_seqlens, int32_t n_seq, int64_t total_T, int32_t H_qk,
                     int32_t H_v, int32_t d_k, int32_t d_v, gdn_dtype in_dtype, void* q_out,
                     void* k_out, void* v_out, gdn_stream_t stream) {
  gdn_status st = check_common(H_qk, H_v, d_k, d_v, in_dtype, 0.f, 0.f);
  if (st != GDN_OK) return st;
  if (n_seq < 1 || total_T < 0) return GDN_ERR_INVALID_ARG;
  if (cu_seqlens == nullptr && n_seq != 1) return GDN_ERR_INVALID_ARG;
  if ((int64_t)n_seq * H_v > 0x7fffffffLL) return GDN_ERR_INVALID_ARG;
  if (!conv_w) return GDN_ERR_INVALID_ARG;
  if (total_T > 0 && (!q || !k || !v || !q_out || !k_out || !v_out)) return GDN_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, conv_w, conv_state_in, conv_state_out, q_out, k_out, v_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return GDN_ERR_INVALID_ARG;
  const size_t e = in_dtype == GDN_BF16 ? 2 : 4;
  const size_t nqk = (size_t)total_T * H_qk * d_k * e, nv = (size_t)total_T * H_v * d_v * e;
  const size_t ns = (size_t)n_seq * H_v * 3 * (2 * d_k + d_v) * sizeof(float);
  if (overlaps(conv_state_in, ns, conv_state_out, ns)) return GDN_ERR_INVALID_ARG;
  const void* ins[] = {q, k, v};
  const size_t in_n[] = {nqk, nqk, nv};
  void* outs[] = {q_out, k_out, v_out};
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j)
      if (overlaps(outs[i], in_n[i], ins[j], in_n[j])) return GDN_ERR_INVALID_ARG;
  ConvArgs a;
  a.q = q; a.k = k; a.v = v; a.conv_w = conv_w; a.state_in = conv_state_in;
  a.state_out = conv_state_out; a.cu_seqlens = cu_seqlens; a.n_seq = n_seq; a.total_T = total_T;
  a.H_qk = H_qk; a.H_v = H_v; a.d_k = d_k; a.d_v = d_v; a.dtype = in_dtype;
  a.q_out = q_out; a.k_out = k_out; a.v_out = v_out;
  a.err = error_word_ptr();
  if (a.err == nullptr) return GDN_ERR_CUDA;
  return launch_conv(a, reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" gdn_status gdn_conv_frontend(
    const void* q, const void* k, const void* v, const float* conv_w,
    const float* conv_state_in, float* conv_state_out, const int32_t* cu_seqlens, int32_t n_seq,
    int64_t total_T, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v, gdn_dtype in_dtype,
    void* q_out, void* k_out, void* v_out, gdn_stream_t stream) {
  return conv_impl(q, k, v, conv_w, conv_state_in, conv_state_out, cu_seqlens, n_seq, total_T,
                   H_qk, H_v, d_k, d_v, in_dtype, q_out, k_out, v_out, stream);
}

extern "C" size_t gdn_chunk_fwd_conv_workspace_size(int32_t n_seq, int64_t total_T,
                                                    int32_t H_qk, int32_t H_v, int32_t d_k,
                                                    int32_t d_v, gdn_dtype in_dtype) {
  if (n_seq < 1 || total_T < 0 || H_qk < 1 || H_v < 1 || H_v % H_qk != 0) return 0;
  if (!dim_ok(d_k) || !dim_ok(d_v) || (in_dtype != GDN_BF16 && in_dtype != GDN_FP32)) return 0;
  return conv_buffers_bytes(total_T, H_qk, H_v, d_k, d_v, in_dtype) +
         prefill_tc_workspace_bytes(n_seq, H_v, d_k, d_v, in_dtype);
}

extern "C" gdn_status gdn_chunk_fwd_conv(
    const void* q, const void* k, const void* v, const float* conv_w,
    const float* conv_state_in, float* conv_state_out, const float* log_alpha,
    const float* beta, const void* g, const float* norm_w, const float* initial_state,
    const int32_t* cu_seqlens, int32_t n_seq, int64_t total_T, int32_t H_qk, int32_t H_v,
    int32_t d_k, int32_t d_v, gdn_dtype in_dtype, int32_t l2norm_qk, float eps_l2,
    float eps_norm, float scale, void* y, float* final_state, gdn_prefill_path path,
    void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
  gdn_status st = check_common(H_qk, H_v, d_k, d_v, in_dtype, eps_l2, eps_norm);
  if (st != GDN_OK) return st;
  if (n_seq < 1 || total_T < 0) return GDN_ERR_INVALID_ARG;
  const size_t need = gdn_chunk_fwd_conv_workspace_size(n_seq, total_T, H_qk, H_v, d_k, d_v,
                                                        in_dtype);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < need)
    return GDN_ERR_INVALID_ARG;
  // the portable kernel takes the front end fused (no activation round trip)
  const bool tc_shape = in_dtype == GDN_BF16 && d_k == 128 && d_v == 128;
  if (path == GDN_PATH_SIMT || (path == GDN_PATH_AUTO && !tc_shape)) {
    if (!conv_w || !aligned16(conv_w)) return GDN_ERR_INVALID_ARG;
    if ((conv_state_in && !aligned16(conv_state_in)) ||
        (conv_state_out && !aligned16(conv_state_out)))
      return GDN_ERR_INVALID_ARG;
    const size_t ns = (size_t)n_seq * H_v * 3 * (2 * d_k + d_v) * sizeof(float);
    if (overlaps(conv_state_in, ns, conv_state_out, ns)) return GDN_ERR_INVALID_ARG;
    return chunk_fwd_impl(q, k, v, log_alpha, beta, g, norm_w, initial_state, cu_seqlens, n_seq,
                          total_T, H_qk, H_v, d_k, d_v, in_dtype, l2norm_qk, eps_l2, eps_norm,
                          scale, y, final_state, GDN_PATH_SIMT, nullptr, 0, stream, conv_w,
                          conv_state_in, conv_state_out);
  }
  // the front end's outputs first in the workspace, the prefill's part after
  const size_t e = in_dtype == GDN_BF16 ? 2 : 4;
  auto a256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
  char* p = static_cast<char*>(workspace);
  void* qc = p;
  void* kc = p + a256((size_t)total_T * H_qk * d_k * e);
  void* vc = p + 2 * a256((size_t)total_T * H_qk * d_k * e);
  const size_t cbytes = conv_buffers_bytes(total_T, H_qk, H_v, d_k, d_v, in_dtype);
  const size_t pbytes = prefill_tc_workspace_bytes(n_seq, H_v, d_k, d_v, in_dtype);
  st = conv_impl(q, k, v, conv_w, conv_state_in, conv_state_out, cu_seqlens, n_seq, total_T,
                 H_qk, H_v, d_k, d_v, in_dtype, total_T > 0 ? qc : nullptr,
                 total_T > 0 ? kc : nullptr, total_T > 0 ? vc : nullptr, stream);
  if (st != GDN_OK) return st;
  return gdn_chunk_fwd_ws(qc, kc, vc, log_alpha, beta, g, norm_w, initial_state, cu_seqlens,
                          n_seq, total_T, H_qk, H_v, d_k, d_v, in_dtype, l2norm_qk, eps_l2,
                          eps_norm, scale, y, final_state, path,
                          pbytes > 0 ? p + cbytes : nullptr, pbytes, stream);
}

extern "C" gdn_status gdn_decode_step(const void* q, const void* k, const void* v,
                                      const float* log_alpha, const float* beta, const void* g,
                                      const float* norm_w, float* state, int32_t N, int32_t H_qk,
                                      int32_t H_v, int32_t d_k, int32_t d_v, gdn_dtype in_dtype,
                                      int32_t l2norm_qk, float eps_l2, float eps_norm,
                                      float scale, void* y, gdn_stream_t stream) {
  if (N > 0 && !state) return GDN_ERR_INVALID_ARG;
  return gdn_decode_multi(q, k, v, log_alpha, beta, g, norm_w, state, state, nullptr, N, 1,
                          H_qk, H_v, d_k, d_v, in_dtype, l2norm_qk, eps_l2, eps_norm, scale, y,
                          stream);
}

extern "C" size_t gdn_chunk_bwd_workspace_size(int32_t n_seq, int64_t total_T, int32_t H_qk,
                                               int32_t H_v, int32_t d_k, int32_t d_v) {
  if (!dim_ok(d_k) || !dim_ok(d_v) || H_qk < 1 || H_v % H_qk != 0) return 0;
  return chunk_bwd_workspace_bytes(n_seq, total_T, H_qk, H_v, d_k, d_v);
}

extern "C" gdn_status gdn_chunk_bwd(
    const void* q, const void* k, const void* v, const float* log_alpha, const float* beta,
    const void* g, const float* norm_w, const float* initial_state, const int32_t* cu_seqlens,
    int32_t n_seq, int64_t total_T, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
    gdn_dtype in_dtype, int32_t l2norm_qk, float eps_l2, float eps_norm, float scale,
    const void* dy, const float* d_final_state, float* dq, float* dk, float* dv,
    float* dlog_alpha, float* dbeta, float* dg, float* dnorm_w, float* d_initial_state,
    void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
  gdn_status st = check_common(H_qk, H_v, d_k, d_v, in_dtype, eps_l2, eps_norm);
  if (st != GDN_OK) return st;
  if (n_seq < 1 || total_T < 0) return GDN_ERR_INVALID_ARG;
  if (cu_seqlens == nullptr && n_seq != 1) return GDN_ERR_INVALID_ARG;
  if ((int64_t)n_seq * H_v > 0x7fffffffLL) return GDN_ERR_INVALID_ARG;
  if (total_T > 0 && (!q || !k || !v || !log_alpha || !beta || !dy || !dq || !dk || !dv ||
                      !dlog_alpha || !dbeta))
    return GDN_ERR_INVALID_ARG;
  if ((g != nullptr) != (dg != nullptr) || (g == nullptr && dnorm_w != nullptr))
    return GDN_ERR_INVALID_ARG;
  const void* ptrs[] = {q,  k,  v,  log_alpha, beta,  g,  norm_w,  initial_state,  dy,
                        d_final_state, dq, dk, dv, dlog_alpha, dbeta, dg, dnorm_w,
                        d_initial_state};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return GDN_ERR_INVALID_ARG;
  const size_t need = chunk_bwd_workspace_bytes(n_seq, total_T, H_qk, H_v, d_k, d_v);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < need)
    return GDN_ERR_INVALID_ARG;
  BwdArgs a;
  a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
  a.g = g; a.norm_w = g ? norm_w : nullptr;
  a.initial_state = initial_state; a.cu_seqlens = cu_seqlens;
  a.dy = dy; a.d_final_state = d_final_state;
  a.dq = dq; a.dk = dk; a.dv = dv; a.dlog_alpha = dlog_alpha; a.dbeta = dbeta;
  a.dg = dg; a.dnorm_w = dnorm_w; a.d_initial_state = d_initial_state;
  a.n_seq = n_seq; a.total_T = total_T;
  a.H_qk = H_qk; a.H_v = H_v; a.d_k = d_k; a.d_v = d_v; a.dtype = in_dtype;
  a.l2norm = l2norm_qk ? 1 : 0; a.eps_l2 = eps_l2; a.eps_norm = eps_norm; a.scale = scale;
  a.err = error_word_ptr();
  if (a.err == nullptr) return GDN_ERR_CUDA;
  chunk_bwd_workspace_layout(workspace, &a);
  return launch_chunk_bwd(a, reinterpret_cast<cudaStream_t>(stream));
}

namespace {

gdn_status gr_check(int64_t T, int32_t n_r, int32_t d) {
  if (T < 0 || n_r < 1 || n_r > kMaxGrBranches || d < 8 || d % 8 != 0) return GDN_ERR_INVALID_ARG;
  if ((int64_t)n_r * d > (1 << 24)) return GDN_ERR_UNSUPPORTED;
  return GDN_OK;
}

}  // namespace

extern "C" size_t gdn_gr_read_workspace_size(int64_t T, int32_t n_r, int32_t d, int32_t rank) {
  if (gr_check(T, n_r, d) != GDN_OK || rank < 8 || rank % 8 != 0) return 0;
  return gr_read_workspace_bytes(T, n_r, d, rank);
}

extern "C" gdn_status gdn_gr_read(const uint8_t* codes, const float* scales, const float* gamma,
                                  const void* W_d, const void* W_u, const void* W_w, int64_t T,
                                  int32_t n_r, int32_t d, int32_t rank, float eps, void* x,
                                  float* s, void* workspace, size_t workspace_bytes,
                                  gdn_stream_t stream) {
  gdn_status st = gr_check(T, n_r, d);
  if (st != GDN_OK) return st;
  if (rank < 8 || rank % 8 != 0 || !(eps >= 0.f)) return GDN_ERR_INVALID_ARG;
  if (T > 0 && (!codes || !scales || !gamma || !W_d || !W_u || !W_w || !x || !s))
    return GDN_ERR_INVALID_ARG;
  const void* ptrs[] = {codes, scales, gamma, W_d, W_u, W_w, x, s};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < gr_read_workspace_bytes(T, n_r, d, rank))
    return GDN_ERR_INVALID_ARG;
  GrArgs a;
  a.codes = codes; a.scales = scales; a.gamma = gamma; a.W_d = W_d; a.W_u = W_u; a.W_w = W_w;
  a.T = T; a.n_r = n_r; a.d = d; a.rank = rank; a.eps = eps; a.x = x; a.s = s;
  return launch_gr_read(a, workspace, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" gdn_status gdn_gr_write(uint8_t* codes, float* scales, const void* y, const float* s,
                                   int64_t T, int32_t n_r, int32_t d, gdn_stream_t stream) {
  gdn_status st = gr_check(T, n_r, d);
  if (st != GDN_OK) return st;
  if (T > 0 && (!codes || !scales || !y || !s)) return GDN_ERR_INVALID_ARG;
  const void* ptrs[] = {codes, scales, y, s};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  GrWriteArgs a;
  a.codes = codes; a.scales = scales; a.y = y; a.s = s; a.T = T; a.n_r = n_r; a.d = d;
  return launch_gr_write(a, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" gdn_status gdn_selftest_bounded_wait(int32_t iterations, gdn_stream_t stream) {
  if (iterations < 1) return GDN_ERR_INVALID_ARG;
  int* err = error_word_ptr();
  if (err == nullptr) return GDN_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      err, (uint32_t)iterations);
  return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

extern "C" gdn_status gdn_check_device_error(gdn_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return GDN_ERR_CUDA;
  int* p = error_word_ptr();
  if (p == nullptr) return GDN_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return GDN_ERR_CUDA;
  if (word != 0) {
    const int zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return GDN_ERR_CUDA;
  }
  if (word & kErrTimeout) return GDN_ERR_TIMEOUT;
  if (word & kErrBadSeqlens) return GDN_ERR_INVALID_ARG;
  return GDN_OK;
}

extern "C" const char* gdn_status_string(gdn_status s) {
  switch (s) {
    case GDN_OK: return "ok";
    case GDN_ERR_INVALID_ARG: return "invalid argument";
    case GDN_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case GDN_ERR_CUDA: return "CUDA error";
    case GDN_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

extern "C" int32_t gdn_version(void) { return 100; }
