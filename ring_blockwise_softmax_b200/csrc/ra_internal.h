// ra_internal.h - declarations shared between the host translation units of the library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "ra_common.cuh"

namespace ra {
struct BwdTcWork;
}

namespace ra {

// Identifier of the calling thread's current CUDA context (cuCtxGetId), or 0 when there is none
// yet or the driver cannot say.  Device addresses of the library's __device__ variables are cached
// per context: a context torn down and created again (cudaDeviceReset) reloads the module, and
// the variables may then sit at other addresses.
unsigned long long current_context_id();

cudaError_t launch_fmha_dp32(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const AttnWork& w,
                             int n_steps, int epi, int sms, cudaStream_t stream, bool dependent);
cudaError_t launch_fmha_dp64(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const AttnWork& w,
                             int n_steps, int epi, int sms, cudaStream_t stream, bool dependent);
cudaError_t launch_fmha_dp128(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const AttnWork& w,
                              int n_steps, int epi, int sms, cudaStream_t stream, bool dependent);

// Tensor maps of the tensor-core backward: 128-row boxes for the fixed operands of a CTA,
// 64-row boxes for the streamed tiles.
struct BwdMaps {
  CUtensorMap q128, k128, v128, do128;
  CUtensorMap q64, k64, v64, do64, o64;
};
cudaError_t launch_bwd_dp32(const BwdMaps& m, const BwdTcWork& wq, const BwdTcWork& wkv, cudaStream_t stream);
cudaError_t launch_bwd_dp64(const BwdMaps& m, const BwdTcWork& wq, const BwdTcWork& wkv, cudaStream_t stream);
cudaError_t launch_bwd_dp128(const BwdMaps& m, const BwdTcWork& wq, const BwdTcWork& wkv, cudaStream_t stream);

}  // namespace ra
