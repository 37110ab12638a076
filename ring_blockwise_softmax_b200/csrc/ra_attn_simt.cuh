// ra_attn_simt.cuh - fp32 blockwise attention on the CUDA cores (no tensor cores).
//
// Same method and same work description as the tensor-core kernel (online softmax over K/V
// tiles streamed through shared memory, intelliparadigm.com "深度学习注意力机制优化与
// FlashAttention实践" §4.2 with the output rescaled at every max update; ring walk over KV shards
// with positions for the causal mask), for fp32 inputs.  Arithmetic: fp32 dot products and
// exponentials (expf, full accuracy), running max in fp32, the running sum of exponentials and
// the LSE in fp64 so that the natural-log LSE stays within ~1 ulp of fp32 (the pages ask for
// fp32 or better in the log/exp statistics, §5.1).
//
// CTA = 128 threads = 64 query rows; two threads share a row, each owning half of the head
// dimension for q and the output accumulator; the two half dot products are combined with one
// shuffle.  K/V tiles of 32 keys are staged in shared memory.
#pragma once

#include "ra_common.cuh"

namespace ra {

constexpr int kSimtRows = 64;
constexpr int kSimtKeys = 32;

template <int DP>
__global__ void __launch_bounds__(128)
    attn_fwd_simt_f32(const AttnWork w, int n_steps, int epi) {
  constexpr int DH = DP / 2;  // elements per thread
  __shared__ float sk[kSimtKeys][DP + 1];
  __shared__ float sv[kSimtKeys][DP + 1];

  const int tile = blockIdx.x % w.n_q_tiles;
  const int r = w.r_first + (blockIdx.x / w.n_q_tiles) * w.r_step;
  const int h = blockIdx.y;
  const int hk = h / (w.H / w.H_kv);  // K/V head of this query head
  const int b = blockIdx.z;
  const int row = threadIdx.x >> 1;
  const int half = threadIdx.x & 1;
  const int tq = tile * kSimtRows + row;
  const bool row_ok = tq < w.n_q;
  const int rows_valid = min(kSimtRows, w.n_q - tile * kSimtRows);
  const long long q_pos0 = w.q_off + static_cast<long long>(r) * w.q_rstep;
  const long long pos_q = q_pos0 + static_cast<long long>(tq) * w.q_tstride;
  const long long pos_last = q_pos0 + static_cast<long long>(tile * kSimtRows + rows_valid - 1) * w.q_tstride;
  const long long pos_first = q_pos0 + static_cast<long long>(tile * kSimtRows) * w.q_tstride;

  const float* qg = static_cast<const float*>(w.q);
  const float* kg = static_cast<const float*>(w.k);
  const float* vg = static_cast<const float*>(w.v);

  float qv[DH];
  float ov[DH];
#pragma unroll
  for (int i = 0; i < DH; ++i) {
    const int c = half * DH + i;
    qv[i] = (row_ok && c < w.d) ? qg[b * w.q_sb + h * w.q_sh + r * w.q_rs + static_cast<long long>(tq) * w.q_ts + c]
                                : 0.f;
    ov[i] = 0.f;
  }
  float m = -INFINITY;  // running max of scaled scores
  double l = 0.0;       // running sum of e^{x - m}

  for (int step = 0; step < n_steps; ++step) {
    int s = (r - (w.ring_step + step)) % w.P;
    if (s < 0) s += w.P;
    const int kv_lim = visible_key_limit(w, pos_last, s);
    const int kv_start = visible_key_start(w, pos_first, s);  // keys before it: outside every row's window
    const int row_lim = row_ok ? visible_key_limit(w, pos_q, s) : 0;
    const int row_lo = row_ok ? visible_key_start(w, pos_q, s) : 0;
    for (int u0 = kv_start - kv_start % kSimtKeys; u0 < kv_lim; u0 += kSimtKeys) {
      __syncthreads();
      for (int e = threadIdx.x; e < kSimtKeys * DP; e += blockDim.x) {
        const int kr = e / DP, c = e % DP;
        const int u = u0 + kr;
        const bool in = (u < w.n_kv) && (c < w.d);
        sk[kr][c] = in ? kg[b * w.k_sb + hk * w.k_sh + s * w.k_rs + static_cast<long long>(u) * w.k_ts + c] : 0.f;
        sv[kr][c] = in ? vg[b * w.v_sb + hk * w.v_sh + s * w.v_rs + static_cast<long long>(u) * w.v_ts + c] : 0.f;
      }
      __syncthreads();
      float sc[kSimtKeys];
      float mt = -INFINITY;
#pragma unroll
      for (int kr = 0; kr < kSimtKeys; ++kr) {
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < DH; ++i) part = fmaf(qv[i], sk[kr][half * DH + i], part);
        const float full = part + __shfl_xor_sync(0xffffffffu, part, 1);
        const float x = (u0 + kr < row_lim && u0 + kr >= row_lo) ? full * w.scale : -INFINITY;
        sc[kr] = x;
        mt = fmaxf(mt, x);
      }
      if (mt == -INFINITY) continue;  // no visible key for this row in this tile
      const float m_new = fmaxf(m, mt);
      const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
      double tile_sum = 0.0;
#pragma unroll
      for (int i = 0; i < DH; ++i) ov[i] *= alpha;
#pragma unroll
      for (int kr = 0; kr < kSimtKeys; ++kr) {
        const float p = expf(sc[kr] - m_new);
        tile_sum += static_cast<double>(p);
#pragma unroll
        for (int i = 0; i < DH; ++i) ov[i] = fmaf(p, sv[kr][half * DH + i], ov[i]);
      }
      l = l * static_cast<double>(alpha) + tile_sum;
      m = m_new;
    }
  }

  if (!row_ok) return;
  const bool has = l > 0.0;
  if (epi == kEpiAcc && !has) return;  // merging with an empty partial is the identity
  const double lse_part = has ? static_cast<double>(m) + log(l) : -INFINITY;
  const double inv_l = has ? 1.0 / l : 0.0;
  double L = lse_part, w_acc = 0.0, w_part = 1.0;
  float* acc_row = nullptr;
  float* accl = nullptr;
  if (epi != kEpiOut) {
    acc_row = w.acc_o + b * w.a_sb + h * w.a_sh + r * w.a_rs + static_cast<long long>(tq) * w.a_ts;
    accl = w.acc_l + b * w.al_sb + h * w.al_sh + r * w.al_rs + static_cast<long long>(tq) * w.al_ts;
  }
  if (epi == kEpiAcc || epi == kEpiAccOut) lse_merge_weights(static_cast<double>(*accl), lse_part, L, w_acc, w_part);
  const double wp = w_part * inv_l;
  float* out_row = nullptr;
  if (epi == kEpiOut || epi == kEpiAccOut)
    out_row = static_cast<float*>(w.o) + b * w.o_sb + h * w.o_sh + r * w.o_rs + static_cast<long long>(tq) * w.o_ts;
#pragma unroll
  for (int i = 0; i < DH; ++i) {
    const int c = half * DH + i;
    if (c >= w.d) continue;
    double val = static_cast<double>(ov[i]) * wp;
    if (epi == kEpiAcc || epi == kEpiAccOut) val += w_acc * static_cast<double>(acc_row[c]);
    if (epi == kEpiPart || epi == kEpiAcc)
      acc_row[c] = static_cast<float>(val);
    else
      out_row[c] = static_cast<float>(val);
  }
  if (half == 0) {
    if (epi == kEpiPart || epi == kEpiAcc)
      *accl = static_cast<float>(L);
    else if (w.lse != nullptr)
      w.lse[b * w.l_sb + h * w.l_sh + r * w.l_rs + static_cast<long long>(tq) * w.l_ts] = static_cast<float>(L);
  }
}

}  // namespace ra
