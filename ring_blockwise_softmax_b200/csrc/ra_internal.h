// ra_internal.h - declarations shared between the host translation units of the library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "ra_common.cuh"

namespace ra {

cudaError_t launch_fmha_dp32(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const AttnWork& w,
                             int n_steps, int epi, int sms, cudaStream_t stream);
cudaError_t launch_fmha_dp64(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const AttnWork& w,
                             int n_steps, int epi, int sms, cudaStream_t stream);
cudaError_t launch_fmha_dp128(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const AttnWork& w,
                              int n_steps, int epi, int sms, cudaStream_t stream);

}  // namespace ra
