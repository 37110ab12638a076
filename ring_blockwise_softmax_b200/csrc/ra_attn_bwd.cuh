// ra_attn_bwd.cuh - backward pass of softmax attention (fp32 arithmetic on fp32 or bf16 inputs).
//
// What it computes: the gradients of L = sum(dO * O) with respect to Q, K and V for O =
// softmax(scale Q K^T) V, given the forward's saved O and LSE.  The attention weights are
// recomputed from LSE instead of being stored (intelliparadigm.com "深度学习注意力机制优化与
// FlashAttention实践" §3.3 and §4.1, item 3):
//   P = e^{S - LSE} on visible entries (S = scale Q K^T),  D_i = sum_c dO_ic O_ic,
//   dV = P^T dO,   dS = P * (dO V^T - D),   dQ = scale dS K,   dK = scale dS^T Q.
// Visibility is the forward's: all keys, causal (key index <= query index), or a causal sliding
// window of `window` positions.  K and V may have fewer heads than Q (grouped-query attention:
// query head h uses K/V head h / (H / H_kv)); dK and dV then sum over the group.
//
// Two kernels, each over 64-row (or 64-key) blocks with TPR = DP / 16 threads per row, so a
// thread holds 16 elements of each d-vector: thread p of a row owns elements p, p + TPR, ...,
// which keeps the row's threads on different shared-memory banks:
//   attn_bwd_dq  - a block of query rows walks the visible key tiles: dQ (and D, from dO and O);
//   attn_bwd_dkv - a block of keys walks the query rows of every head of its group: dK, dV.
// No atomics: every output element is owned by one thread.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace ra {

struct BwdWork {
  int B, H, H_kv, n_q, n_kv, d;
  int causal;
  long long window;  // 0 = none (causal only)
  float scale;
  // strides in elements, [b, h, t, c]
  const void* q;
  long long q_sb, q_sh, q_st;
  const void* k;
  long long k_sb, k_sh, k_st;
  const void* v;
  long long v_sb, v_sh, v_st;
  const void* o;
  long long o_sb, o_sh, o_st;
  const void* d_o;
  long long do_sb, do_sh, do_st;
  const float* lse;  // [B, H, n_q] contiguous
  float* dq;
  long long dq_sb, dq_sh, dq_st;
  float* dk;
  long long dk_sb, dk_sh, dk_st;
  float* dv;
  long long dv_sb, dv_sh, dv_st;
};

constexpr int kBwdRows = 64;  // query rows (dQ kernel) or keys (dK/dV kernel) per block
constexpr int kBwdTile = 32;  // keys (dQ kernel) or query rows (dK/dV kernel) per shared-memory tile
constexpr int kBwdDH = 16;    // d-elements per thread (16: 2x the occupancy of 32, measured 20 % faster)

template <typename T>
__device__ __forceinline__ float ld_elem(const void* base, long long off) {
  return static_cast<float>(static_cast<const T*>(base)[off]);
}
template <>
__device__ __forceinline__ float ld_elem<__nv_bfloat16>(const void* base, long long off) {
  return __bfloat162float(static_cast<const __nv_bfloat16*>(base)[off]);
}

// Query i may see key j (both local indices = positions of a single pass).
__device__ __forceinline__ bool bwd_visible(const BwdWork& w, int i, int j) {
  if (!w.causal) return true;
  if (j > i) return false;
  return w.window <= 0 || static_cast<long long>(j) > static_cast<long long>(i) - w.window;
}

// Sum over the TPR consecutive lanes that share one row.
template <int TPR>
__device__ __forceinline__ float row_sum(float x) {
#pragma unroll
  for (int m = 1; m < TPR; m <<= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

template <typename T, int DP>
__global__ void __launch_bounds__(kBwdRows * (DP / kBwdDH))
    attn_bwd_dq(const BwdWork w) {
  constexpr int TPR = DP / kBwdDH;
  __shared__ float sk[kBwdTile][DP + 1];
  __shared__ float sv[kBwdTile][DP + 1];
  const int b = blockIdx.z, h = blockIdx.y;
  const int hk = h / (w.H / w.H_kv);
  const int row = threadIdx.x / TPR, part = threadIdx.x % TPR;
  const int i = blockIdx.x * kBwdRows + row;
  const bool row_ok = i < w.n_q;

  float qv[kBwdDH], dov[kBwdDH], acc[kBwdDH];
  float dsum = 0.f;
#pragma unroll
  for (int e = 0; e < kBwdDH; ++e) {
    const int c = e * TPR + part;
    const bool in = row_ok && c < w.d;
    qv[e] = in ? ld_elem<T>(w.q, b * w.q_sb + h * w.q_sh + i * w.q_st + c) : 0.f;
    dov[e] = in ? ld_elem<T>(w.d_o, b * w.do_sb + h * w.do_sh + i * w.do_st + c) : 0.f;
    const float ov = in ? ld_elem<T>(w.o, b * w.o_sb + h * w.o_sh + i * w.o_st + c) : 0.f;
    dsum = fmaf(dov[e], ov, dsum);
    acc[e] = 0.f;
  }
  const float D = row_sum<TPR>(dsum);
  const float L = row_ok ? w.lse[(static_cast<long long>(b) * w.H + h) * w.n_q + i] : -INFINITY;
  const bool any = row_ok && L != -INFINITY;

  // Keys any row of the block can see.
  const int i_last = min(w.n_q, static_cast<int>(blockIdx.x) * kBwdRows + kBwdRows) - 1;
  const int i_first = blockIdx.x * kBwdRows;
  int j_end = w.n_kv, j_begin = 0;
  if (w.causal) {
    j_end = min(w.n_kv, i_last + 1);
    if (w.window > 0) j_begin = static_cast<int>(max(0LL, static_cast<long long>(i_first) - w.window + 1));
  }
  j_begin -= j_begin % kBwdTile;
  for (int j0 = j_begin; j0 < j_end; j0 += kBwdTile) {
    __syncthreads();
    for (int e = threadIdx.x; e < kBwdTile * DP; e += blockDim.x) {
      const int kr = e / DP, c = e % DP;
      const int j = j0 + kr;
      const bool in = j < w.n_kv && c < w.d;
      sk[kr][c] = in ? ld_elem<T>(w.k, b * w.k_sb + hk * w.k_sh + j * w.k_st + c) : 0.f;
      sv[kr][c] = in ? ld_elem<T>(w.v, b * w.v_sb + hk * w.v_sh + j * w.v_st + c) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int kr = 0; kr < kBwdTile; ++kr) {
      const int j = j0 + kr;
      float s_part = 0.f, dp_part = 0.f;
#pragma unroll
      for (int e = 0; e < kBwdDH; ++e) {
        s_part = fmaf(qv[e], sk[kr][e * TPR + part], s_part);
        dp_part = fmaf(dov[e], sv[kr][e * TPR + part], dp_part);
      }
      const float s = row_sum<TPR>(s_part) * w.scale;
      const float dp = row_sum<TPR>(dp_part);
      const bool vis = any && j < w.n_kv && bwd_visible(w, i, j);
      const float p = vis ? expf(s - L) : 0.f;
      const float ds = p * (dp - D);
#pragma unroll
      for (int e = 0; e < kBwdDH; ++e) acc[e] = fmaf(ds, sk[kr][e * TPR + part], acc[e]);
    }
  }
  if (!row_ok) return;
#pragma unroll
  for (int e = 0; e < kBwdDH; ++e) {
    const int c = e * TPR + part;
    if (c < w.d) w.dq[b * w.dq_sb + h * w.dq_sh + i * w.dq_st + c] = w.scale * acc[e];
  }
}

template <typename T, int DP>
__global__ void __launch_bounds__(kBwdRows * (DP / kBwdDH))
    attn_bwd_dkv(const BwdWork w) {
  constexpr int TPR = DP / kBwdDH;
  __shared__ float sq[kBwdTile][DP + 1];
  __shared__ float sdo[kBwdTile][DP + 1];
  __shared__ float s_lse[kBwdTile];
  __shared__ float s_d[kBwdTile];
  const int b = blockIdx.z, hk = blockIdx.y;
  const int qpk = w.H / w.H_kv;
  const int key = threadIdx.x / TPR, part = threadIdx.x % TPR;
  const int j = blockIdx.x * kBwdRows + key;
  const bool key_ok = j < w.n_kv;

  float kv[kBwdDH], vv[kBwdDH], dk[kBwdDH], dv[kBwdDH];
#pragma unroll
  for (int e = 0; e < kBwdDH; ++e) {
    const int c = e * TPR + part;
    const bool in = key_ok && c < w.d;
    kv[e] = in ? ld_elem<T>(w.k, b * w.k_sb + hk * w.k_sh + j * w.k_st + c) : 0.f;
    vv[e] = in ? ld_elem<T>(w.v, b * w.v_sb + hk * w.v_sh + j * w.v_st + c) : 0.f;
    dk[e] = 0.f;
    dv[e] = 0.f;
  }
  // Query rows any key of the block can be seen by.
  const int j_first = blockIdx.x * kBwdRows;
  const int j_last = min(w.n_kv, j_first + kBwdRows) - 1;
  int i_begin = 0, i_end = w.n_q;
  if (w.causal) {
    i_begin = j_first;
    if (w.window > 0) i_end = static_cast<int>(min(static_cast<long long>(w.n_q), j_last + w.window));
  }
  i_begin -= i_begin % kBwdTile;
  for (int g = 0; g < qpk; ++g) {
    const int h = hk * qpk + g;
    for (int i0 = i_begin; i0 < i_end; i0 += kBwdTile) {
      // D_i = dO_i . O_i of the tile's rows, from O staged (coalesced) in the Q buffer.
      __syncthreads();
      for (int e = threadIdx.x; e < kBwdTile * DP; e += blockDim.x) {
        const int r = e / DP, c = e % DP;
        const int i = i0 + r;
        const bool in = i < w.n_q && c < w.d;
        sq[r][c] = in ? ld_elem<T>(w.o, b * w.o_sb + h * w.o_sh + i * w.o_st + c) : 0.f;
        sdo[r][c] = in ? ld_elem<T>(w.d_o, b * w.do_sb + h * w.do_sh + i * w.do_st + c) : 0.f;
      }
      __syncthreads();
      if (threadIdx.x < kBwdTile) {
        const int r = threadIdx.x;
        const int i = i0 + r;
        float dsum = 0.f;
        for (int c = 0; c < DP; ++c) dsum = fmaf(sdo[r][c], sq[r][c], dsum);
        s_d[r] = dsum;
        s_lse[r] = i < w.n_q ? w.lse[(static_cast<long long>(b) * w.H + h) * w.n_q + i] : -INFINITY;
      }
      __syncthreads();
      for (int e = threadIdx.x; e < kBwdTile * DP; e += blockDim.x) {
        const int r = e / DP, c = e % DP;
        const int i = i0 + r;
        sq[r][c] = (i < w.n_q && c < w.d) ? ld_elem<T>(w.q, b * w.q_sb + h * w.q_sh + i * w.q_st + c) : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int r = 0; r < kBwdTile; ++r) {
        const int i = i0 + r;
        float s_part = 0.f, dp_part = 0.f;
#pragma unroll
        for (int e = 0; e < kBwdDH; ++e) {
          s_part = fmaf(sq[r][e * TPR + part], kv[e], s_part);
          dp_part = fmaf(sdo[r][e * TPR + part], vv[e], dp_part);
        }
        const float s = row_sum<TPR>(s_part) * w.scale;
        const float dp = row_sum<TPR>(dp_part);
        const float L = s_lse[r];
        const bool vis = key_ok && i < w.n_q && L != -INFINITY && bwd_visible(w, i, j);
        const float p = vis ? expf(s - L) : 0.f;
        const float ds = p * (dp - s_d[r]);
#pragma unroll
        for (int e = 0; e < kBwdDH; ++e) {
          dv[e] = fmaf(p, sdo[r][e * TPR + part], dv[e]);
          dk[e] = fmaf(ds, sq[r][e * TPR + part], dk[e]);
        }
      }
    }
  }
  if (!key_ok) return;
#pragma unroll
  for (int e = 0; e < kBwdDH; ++e) {
    const int c = e * TPR + part;
    if (c >= w.d) continue;
    w.dk[b * w.dk_sb + hk * w.dk_sh + j * w.dk_st + c] = w.scale * dk[e];
    w.dv[b * w.dv_sb + hk * w.dv_sh + j * w.dv_st + c] = dv[e];
  }
}

}  // namespace ra
