// ra_bwd_launch.cu - instantiates the tensor-core backward kernels (dQ and dK/dV instances) for
// one padded head dim (RA_BWD_DP = 32, 64 or 128; the file is compiled once per value) and
// launches them.
#include "ra_bwd_sm100.cuh"
#include "ra_internal.h"

#ifndef RA_BWD_DP
#error "compile with -DRA_BWD_DP=32|64|128"
#endif

namespace ra {

#ifndef RA_PDL
#define RA_PDL 1
#endif

// kv (the dK/dV instance, launched after the dQ one): as a programmatic dependent of the dQ launch.
template <class C, class K>
static cudaError_t launch_kernel(K kern, bool kv, const CUtensorMap& a1, const CUtensorMap& a2, const CUtensorMap& b1,
                                 const CUtensorMap& b2, const CUtensorMap& b3, const BwdTcWork& w,
                                 cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  // The kernel's warpgroups rebalance registers with setmaxnreg; an increase beyond the pool the
  // block was launched with would never complete, so such a build is refused here.
  cudaFuncAttributes attr;
  e = cudaFuncGetAttributes(&attr, kern);
  if (e != cudaSuccess) return e;
  if (attr.numRegs * C::THREADS < C::REG_TOTAL || attr.maxThreadsPerBlock < C::THREADS)
    return cudaErrorInvalidConfiguration;
  const int rows = kv ? w.n_kv : w.n_q;
  const dim3 grid((rows + C::BM - 1) / C::BM, kv ? w.H_kv : w.H, w.B);
  if (!(kv && RA_PDL)) {
    kern<<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(a1, a2, b1, b2, b3, w);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a1, a2, b1, b2, b3, w);
}

// The warpgroup ping-pong kernel wherever each warpgroup's (S, dP) buffer and P, dS columns fit
// beside the accumulators; the column-split kernel for the dK/dV instance at DP = 128, where they
// do not (writing P, dS over S, dP instead measured slower there).
template <bool KV>
static cudaError_t launch_bwd_one(const CUtensorMap& a1, const CUtensorMap& a2, const CUtensorMap& b1,
                                  const CUtensorMap& b2, const CUtensorMap& b3, const BwdTcWork& w,
                                  cudaStream_t stream) {
  if constexpr (KV && RA_BWD_DP == 128)
    return launch_kernel<BwdCfgSplit<RA_BWD_DP, KV>>(attn_bwd_sm100_split<RA_BWD_DP, KV>, KV, a1, a2, b1, b2, b3, w,
                                                     stream);
  else
    return launch_kernel<BwdCfg<RA_BWD_DP, KV>>(attn_bwd_sm100<RA_BWD_DP, KV>, KV, a1, a2, b1, b2, b3, w, stream);
}

#define RA_CAT2(a, b) a##b
#define RA_CAT(a, b) RA_CAT2(a, b)

// Maps: q128/k128/v128/do128 with 128-row boxes (fixed operands), q64/k64/v64/do64/o64 with
// 64-row boxes (streamed tiles).  dQ first, then dK/dV; both on `stream`.
cudaError_t RA_CAT(launch_bwd_dp, RA_BWD_DP)(const BwdMaps& m, const BwdTcWork& wq, const BwdTcWork& wkv,
                                             cudaStream_t stream) {
  cudaError_t e = launch_bwd_one<false>(m.q128, m.do128, m.k64, m.v64, m.k64, wq, stream);
  if (e != cudaSuccess) return e;
  return launch_bwd_one<true>(m.k128, m.v128, m.q64, m.do64, m.o64, wkv, stream);
}

}  // namespace ra
