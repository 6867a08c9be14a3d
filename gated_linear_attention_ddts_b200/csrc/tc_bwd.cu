// tc_bwd.cu -- tensor-core chunked backward (placeholder until the kernel lands).
#include "launch.h"

namespace rdm {
bool tc_bwd_supported(const BwdParams&) { return false; }
size_t tc_bwd_workspace(const BwdParams&) { return 0; }
cudaError_t launch_tc_bwd(const BwdParams&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace rdm
