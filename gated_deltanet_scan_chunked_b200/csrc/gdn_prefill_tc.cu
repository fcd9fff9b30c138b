// placeholder, replaced by the tensor-core kernel
#include "gdn_internal.h"
namespace gdn {
bool prefill_tc_supports(const PrefillArgs&) { return false; }
gdn_status launch_prefill_tc(const PrefillArgs&, cudaStream_t) { return GDN_ERR_UNSUPPORTED; }
}  // namespace gdn
