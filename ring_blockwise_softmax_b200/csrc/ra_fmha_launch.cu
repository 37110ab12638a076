// ra_fmha_launch.cu - instantiates the tensor-core attention kernel for one padded head dim
// (RA_FMHA_DP = 32, 64 or 128; the file is compiled once per value) and launches it.
#include "ra_fmha_sm100.cuh"
#include "ra_internal.h"

#ifndef RA_FMHA_DP
#error "compile with -DRA_FMHA_DP=32|64|128"
#endif

namespace ra {

template <int EPI, bool WIN>
static cudaError_t launch_epi(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const AttnWork& w,
                              int n_steps, int sms, cudaStream_t stream, bool dependent) {
  using C = FmhaCfg<RA_FMHA_DP>;
  auto kern = fmha_fwd_sm100<RA_FMHA_DP, EPI, WIN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  // The warpgroups' setmaxnreg shares must fit in the registers the block is launched with, or a
  // setmaxnreg.inc would never be granted: refuse the launch if the compiled kernel has fewer.
  cudaFuncAttributes attr;
  e = cudaFuncGetAttributes(&attr, kern);
  if (e != cudaSuccess) return e;
  if (attr.numRegs * C::THREADS < RegSplit<RA_FMHA_DP, EPI>::kTotal || attr.maxThreadsPerBlock < C::THREADS)
    return cudaErrorInvalidConfiguration;
  // Persistent grid: one CTA per SM (at most one per work item of 256 query rows).
  const long long n_items = static_cast<long long>((w.n_q + C::ROWS - 1) / C::ROWS) * w.n_r * w.H * w.B;
  if (n_items > 2147483647LL) return cudaErrorInvalidValue;
  const int grid = static_cast<int>(n_items < sms ? n_items : sms);
  if (!dependent) {
    kern<<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, w, n_steps, static_cast<int>(n_items));
    return cudaGetLastError();
  }
  // Programmatic dependent launch: this grid may start while the previous kernel on the stream
  // (the previous ring step, which signals at its start) is finishing; its epilogue waits for it.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, w, n_steps, static_cast<int>(n_items));
}

#define RA_CAT2(a, b) a##b
#define RA_CAT(a, b) RA_CAT2(a, b)

cudaError_t RA_CAT(launch_fmha_dp, RA_FMHA_DP)(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                                               const AttnWork& w, int n_steps, int epi, int sms,
                                               cudaStream_t stream, bool dependent) {
  // Launches with a sliding window use their own instantiation (WIN = true).
  const bool win = w.window > 0;
  switch (epi) {
    case kEpiOut:
      return win ? launch_epi<kEpiOut, true>(mq, mk, mv, w, n_steps, sms, stream, dependent)
                 : launch_epi<kEpiOut, false>(mq, mk, mv, w, n_steps, sms, stream, dependent);
    case kEpiPart:
      return win ? launch_epi<kEpiPart, true>(mq, mk, mv, w, n_steps, sms, stream, dependent)
                 : launch_epi<kEpiPart, false>(mq, mk, mv, w, n_steps, sms, stream, dependent);
    case kEpiAcc:
      return win ? launch_epi<kEpiAcc, true>(mq, mk, mv, w, n_steps, sms, stream, dependent)
                 : launch_epi<kEpiAcc, false>(mq, mk, mv, w, n_steps, sms, stream, dependent);
    case kEpiAccOut:
      return win ? launch_epi<kEpiAccOut, true>(mq, mk, mv, w, n_steps, sms, stream, dependent)
                 : launch_epi<kEpiAccOut, false>(mq, mk, mv, w, n_steps, sms, stream, dependent);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace ra
