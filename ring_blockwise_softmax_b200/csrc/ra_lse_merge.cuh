// ra_lse_merge.cuh - LSE merge of partial attention results, bound by HBM bandwidth.
//
// Two partials (O_a, LSE_a), (O_b, LSE_b) of the same query rows over disjoint key sets combine
// as LSE = max(a,b) + log1p(e^{-|a-b|}), O = e^{a-LSE} O_a + e^{b-LSE} O_b (blog.gitcode.com
// "分布式注意力机制突破…" §2.2 phase 3, exponent sign corrected); M partials combine in one pass
// through the aligned-maximum form of §3.4: m = max_i LSE_i, s = sum_i e^{LSE_i - m},
// LSE = m + ln s, O = sum_i e^{LSE_i - m} O_i / s.
//
// Layout: O [rows, d] fp32 row-major, LSE [rows] fp32.  A group of G lanes (G = the power of two
// >= d/VEC, at most 32) owns one row; lane g of the group moves VEC-wide vectors g, g+G, ...
// Every lane of the group reads the row's LSE values itself (broadcast through L1) before the
// group synchronises, and only then does lane 0 write the output LSE, so the outputs may alias
// the first input in place.  Grid-stride over row groups; the grid is sized to fill the SMs.
#pragma once

#include "ra_common.cuh"

namespace ra {

template <int VEC>
struct VecT;
template <>
struct VecT<4> {
  using T = float4;
};
template <>
struct VecT<1> {
  using T = float;
};

__device__ __forceinline__ float4 axpby(float a, float4 x, float b, float4 y) {
  return make_float4(fmaf(a, x.x, b * y.x), fmaf(a, x.y, b * y.y), fmaf(a, x.z, b * y.z), fmaf(a, x.w, b * y.w));
}
__device__ __forceinline__ float axpby(float a, float x, float b, float y) { return fmaf(a, x, b * y); }
__device__ __forceinline__ float4 fma4(float a, float4 x, float4 acc) {
  return make_float4(fmaf(a, x.x, acc.x), fmaf(a, x.y, acc.y), fmaf(a, x.z, acc.z), fmaf(a, x.w, acc.w));
}
__device__ __forceinline__ float fma4(float a, float x, float acc) { return fmaf(a, x, acc); }
__device__ __forceinline__ float4 zero_v(float4*) { return make_float4(0.f, 0.f, 0.f, 0.f); }
__device__ __forceinline__ float zero_v(float*) { return 0.f; }
__device__ __forceinline__ float4 scale_v(float4 x, float a) { return make_float4(x.x * a, x.y * a, x.z * a, x.w * a); }
__device__ __forceinline__ float scale_v(float x, float a) { return x * a; }

template <int VEC, int G>
__global__ void __launch_bounds__(256) lse_merge2_kernel(const float* o_a, const float* lse_a,
                                                         const float* o_b, const float* lse_b,
                                                         float* o_out, float* lse_out, long long rows, int d) {
  using V = typename VecT<VEC>::T;
  constexpr int R = 2;  // rows per group and iteration: 2 x 2 loads in flight per lane
  const int nv = d / VEC;
  const int lane = threadIdx.x & 31;
  const int g = lane % G;
  const long long groups_per_block = blockDim.x / G;
  const long long first = static_cast<long long>(blockIdx.x) * groups_per_block + threadIdx.x / G;
  const long long stride = static_cast<long long>(gridDim.x) * groups_per_block;
  const long long n_iter = (rows + R * stride - 1) / (R * stride);  // same trip count in a warp
  for (long long it = 0; it < n_iter; ++it) {
    long long row[R];
    bool active[R];
    V va[R], vb[R];
#pragma unroll
    for (int rr = 0; rr < R; ++rr) {
      row[rr] = first + (it * R + rr) * stride;
      active[rr] = row[rr] < rows;
      // The first column group's O loads go out before the LSE arithmetic (latencies overlap).
      if (active[rr] && g < nv) {
        va[rr] = __ldcs(reinterpret_cast<const V*>(o_a + row[rr] * d) + g);
        vb[rr] = __ldcs(reinterpret_cast<const V*>(o_b + row[rr] * d) + g);
      }
    }
    float L[R], wa[R], wb[R];
#pragma unroll
    for (int rr = 0; rr < R; ++rr) {
      L[rr] = 0.f;
      wa[rr] = 0.f;
      wb[rr] = 0.f;
      if (active[rr]) lse_merge_weights(lse_a[row[rr]], lse_b[row[rr]], L[rr], wa[rr], wb[rr]);
    }
#pragma unroll
    for (int rr = 0; rr < R; ++rr) {
      if (!active[rr]) continue;
      const V* pa = reinterpret_cast<const V*>(o_a + row[rr] * d);
      const V* pb = reinterpret_cast<const V*>(o_b + row[rr] * d);
      V* po = reinterpret_cast<V*>(o_out + row[rr] * d);
      for (int c = g; c < nv; c += G) {
        if (c != g) {
          va[rr] = __ldcs(pa + c);
          vb[rr] = __ldcs(pb + c);
        }
        __stcs(po + c, axpby(wa[rr], va[rr], wb[rr], vb[rr]));
      }
    }
    __syncwarp();
#pragma unroll
    for (int rr = 0; rr < R; ++rr)
      if (active[rr] && g == 0) lse_out[row[rr]] = L[rr];
  }
}

struct MergeParts {
  const float* o[32];
  const float* l[32];
};

// KMAX >= k: the part loops are unrolled KMAX times and predicated on i < k, so the weights stay
// in registers and the k loads of one vector are issued back to back.
template <int VEC, int G, int KMAX>
__global__ void __launch_bounds__(256) lse_merge_n_kernel(const MergeParts parts, int k, float* o_out,
                                                          float* lse_out, long long rows, int d) {
  using V = typename VecT<VEC>::T;
  const int nv = d / VEC;
  const int lane = threadIdx.x & 31;
  const int g = lane % G;
  const long long groups_per_block = blockDim.x / G;
  const long long first = static_cast<long long>(blockIdx.x) * groups_per_block + threadIdx.x / G;
  const long long stride = static_cast<long long>(gridDim.x) * groups_per_block;
  const long long n_iter = (rows + stride - 1) / stride;
  for (long long it = 0; it < n_iter; ++it) {
    const long long row = first + it * stride;
    const bool active = row < rows;
    float L = -INFINITY;
    if (active) {
      // Issue this row's O loads for the first column group before the LSE arithmetic, so the
      // two memory latencies overlap instead of adding up.
      V ov[KMAX];
      const bool first_ok = g < nv;
#pragma unroll
      for (int i = 0; i < KMAX; ++i)
        if (i < k && first_ok) ov[i] = __ldcs(reinterpret_cast<const V*>(parts.o[i] + row * d) + g);
      float wgt[KMAX];
      float m = -INFINITY;
#pragma unroll
      for (int i = 0; i < KMAX; ++i) {
        wgt[i] = (i < k) ? parts.l[i][row] : -INFINITY;
        m = fmaxf(m, wgt[i]);
      }
      float ssum = 0.f;
      const float m_safe = (m == -INFINITY) ? 0.f : m;
#pragma unroll
      for (int i = 0; i < KMAX; ++i) {
        wgt[i] = expf(wgt[i] - m_safe);  // e^{-inf} = 0 for empty partials and unused slots
        ssum += wgt[i];
      }
      if (m != -INFINITY) L = m + logf(ssum);
      const float inv = ssum > 0.f ? 1.f / ssum : 0.f;
      V* po = reinterpret_cast<V*>(o_out + row * d);
      for (int c = g; c < nv; c += G) {
        if (c != g) {
#pragma unroll
          for (int i = 0; i < KMAX; ++i)
            if (i < k) ov[i] = __ldcs(reinterpret_cast<const V*>(parts.o[i] + row * d) + c);
        }
        V acc = zero_v(static_cast<V*>(nullptr));
#pragma unroll
        for (int i = 0; i < KMAX; ++i)
          if (i < k) acc = fma4(wgt[i], ov[i], acc);
        __stcs(po + c, scale_v(acc, inv));
      }
    }
    __syncwarp();
    if (active && g == 0) lse_out[row] = L;
  }
}

}  // namespace ra
