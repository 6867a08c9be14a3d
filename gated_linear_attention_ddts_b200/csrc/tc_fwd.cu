// tc_fwd.cu -- tensor-core chunked forward (placeholder until the kernel lands).
#include "launch.h"

namespace rdm {
bool tc_fwd_supported(const SeqParams&) { return false; }
cudaError_t launch_tc_fwd(const SeqParams&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace rdm
