// conv_launch.h -- host launchers of the ShortConv kernels (shortconv.cu) for
// several independent problems in one launch (the q, k and v convolutions of
// a layer, say): their tiles form one index space that the persistent blocks
// share, so the launch pays one ramp and one tail for all of them.
#pragma once

#include <cuda_runtime.h>

#include "launch.h"

namespace rdm {

constexpr int kMaxConvBatch = 4;

// n in [1, kMaxConvBatch] problems with the same element type, width W and
// SiLU switch (the caller checks); each may have its own B, H, T, D.
cudaError_t launch_conv_fwd_many(const ConvParams* ps, int n, cudaStream_t s);
cudaError_t launch_conv_bwd_many(const ConvParams* ps, int n, cudaStream_t s);

}  // namespace rdm
