// kmip_fwd_tc.cu -- tcgen05 tensor-core forward (bf16).  Not yet enabled.
#include "kmip_internal.h"

namespace kmip {

bool fwd_tc_supported(int, int) { return false; }

cudaError_t launch_fwd_tc(const FwdArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace kmip
