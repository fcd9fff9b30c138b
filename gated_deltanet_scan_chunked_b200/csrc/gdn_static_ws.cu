// gdn_chunk_fwd_static_ws: the split-layout prefill (GDN_PATH_TENSOR_SPLIT:
// the scan layout of gdn_prefill_scan.cu) with its hand-off
// workspace in a fixed device array of this library, for callers that cannot
// hand the library any memory.  Nothing here allocates: the array is part of
// the module image, its address comes from cudaGetSymbolAddress (looked up
// once per device and kept; not valid across a device reset), and the call
// forwards to gdn_chunk_fwd_ws.
#include <cuda_runtime.h>

#include <mutex>

#include "gdn_internal.h"

namespace gdn {
namespace {

// Capacity: 48 (sequence, value head) items -- one sequence of a 48-value-head
// layer -- sized from the scan layout's own workspace formula.
constexpr int kStaticItems = 48;
constexpr size_t kStaticBytes = scan_ws_bytes(kStaticItems);
static_assert(kStaticItems <= kScanMaxItems, "static workspace holds a scan-layout batch");

static __device__ __align__(256) unsigned char g_static_ws[kStaticBytes];

constexpr int kMaxDevices = 64;
std::mutex g_ws_mu;
void* g_ws_ptr[kMaxDevices] = {nullptr};

void* static_ws_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_ws_mu);
  if (g_ws_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess) return nullptr;
    g_ws_ptr[dev] = p;
  }
  return g_ws_ptr[dev];
}

}  // namespace
}  // namespace gdn

extern "C" gdn_status gdn_chunk_fwd_static_ws(
    const void* q, const void* k, const void* v, const float* log_alpha, const float* beta,
    const void* g, const float* norm_w, const float* initial_state, const int32_t* cu_seqlens,
    int32_t n_seq, int64_t total_T, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
    gdn_dtype in_dtype, int32_t l2norm_qk, float eps_l2, float eps_norm, float scale, void* y,
    float* final_state, gdn_stream_t stream) {
  // the same argument errors as gdn_chunk_fwd_ws, before the capacity check
  const gdn_status st = gdn::check_common(H_qk, H_v, d_k, d_v, in_dtype, eps_l2, eps_norm);
  if (st != GDN_OK) return st;
  if (n_seq < 1 || total_T < 0) return GDN_ERR_INVALID_ARG;
  const size_t need = gdn_chunk_fwd_workspace_size(n_seq, H_v, d_k, d_v, in_dtype);
  // a shape the split layout does not serve, or more items than the array holds
  if ((long long)n_seq * H_v > gdn::kStaticItems || need == 0 || need > gdn::kStaticBytes)
    return GDN_ERR_UNSUPPORTED;
  void* ws = gdn::static_ws_ptr();
  if (ws == nullptr) return GDN_ERR_CUDA;
  // the scan launch clears the array's flags on `stream` before its kernel
  return gdn_chunk_fwd_ws(q, k, v, log_alpha, beta, g, norm_w, initial_state, cu_seqlens, n_seq,
                          total_T, H_qk, H_v, d_k, d_v, in_dtype, l2norm_qk, eps_l2, eps_norm,
                          scale, y, final_state, GDN_PATH_TENSOR_SPLIT, ws, gdn::kStaticBytes,
                          stream);
}
