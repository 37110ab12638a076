// ra_fmha_sm100.cuh - fused blockwise attention forward on the sm_100a tensor cores.
//
// Computes, for one 128-row query tile, the online softmax of intelliparadigm.com
// "深度学习注意力机制优化与FlashAttention实践" §4.2 (with the output rescaled whenever the running
// max moves, which the printed listing omits): K/V tiles of 128 keys stream through shared
// memory; S = Q K^T and O += P V run as tcgen05 MMAs with fp32 accumulators in tensor memory;
// a per-row running max m and sum s are kept in fp32 registers.  One launch may walk several
// KV shards of a ring in ring order (query shard r meets KV shard (r - t) mod P at step t,
// vibe-research.pages.dev "Ring Attention" diagram); a shard boundary needs no extra work
// because the running (m, s, O) already is the merged state of every shard seen so far
// (blog.gitcode.com "分布式注意力机制突破…" §3.4: align maxima, rescale sums).
//
// CTA = 192 threads, one 128-row query tile:
//   warps 0-3  softmax: thread i owns query row i = tensor-memory lane i.  Loads its S row,
//              masks, updates (m, s), writes P (bf16) back over S in tensor memory, rescales
//              its O row when m moved by more than 2^8 (lazy rescale; exact because the final
//              division uses the same stale m), and runs the epilogue.
//   warp 4     TMA producer: Q once, then K_j / V_j into a STAGES-deep ring.
//   warp 5     MMA issuer (one thread): S_j = Q K_j^T (SS form, both K-major),
//              O += P_j V_j (TS form: P from tensor memory, V MN-major from shared memory).
// Tensor memory (512 columns): three S slots of 128 columns (tile j uses slot j % 3; P_j is
// packed bf16x2 into the first 64 columns of the same slot) and O at column 384 (DP columns).
//
// Every wait is bounded (ra_common.cuh); on a timeout all roles stop, tensor memory is freed and
// the kernel returns with the device status word set.
#pragma once

#include "ra_common.cuh"

namespace ra {

template <int DP>
struct FmhaCfg {
  static_assert(DP == 32 || DP == 64 || DP == 128, "padded head dim must be 32, 64 or 128");
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int CB = (DP == 32) ? 32 : 64;  // columns per TMA box / swizzle span
  static constexpr int NCB = DP / CB;              // column blocks per tile
  static constexpr int ROW_BYTES = CB * 2;         // bytes of one row inside a column block
  static constexpr uint32_t SWZ = (DP == 32) ? kSwizzle64B : kSwizzle128B;
  static constexpr int ATOM_BYTES = 8 * ROW_BYTES;     // 8-row swizzle atom
  static constexpr int BLOCK_BYTES = 128 * ROW_BYTES;  // one column block of a 128-row tile
  static constexpr int TILE_BYTES = 128 * DP * 2;      // a whole Q, K or V tile (bf16)
  static constexpr int STAGES = (DP == 128) ? 2 : (DP == 64 ? 4 : 8);  // >= 114 KB smem: one CTA per SM
  static constexpr int NSLOT = 3;                      // S slots in tensor memory
  static constexpr int O_COL = 384;
  static constexpr int SMEM_TILES = TILE_BYTES * (1 + 2 * STAGES);
  static constexpr int NBAR = 2 + 3 * STAGES + 3 * NSLOT;
  static constexpr int SMEM_BYTES = 1024 /*alignment slack*/ + SMEM_TILES + NBAR * 8 + 16 + 64 * 8;
  static constexpr int THREADS = 192;
  static constexpr int MAX_STEPS = 64;  // shards one launch may walk
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x (low 16 bits) = lo
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void reg_dep(uint32_t (&r)[32]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

// Bounded wait that ignores the abort flag (used to drain in-flight TMA before exit).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) break;
  }
}

template <int DP, int EPI>
__global__ void __launch_bounds__(192, 1)
    fmha_fwd_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnWork w, int n_steps) {
  using C = FmhaCfg<DP>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);

  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::TILE_BYTES;
  uint8_t* sV = sK + C::STAGES * C::TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + C::STAGES * C::TILE_BYTES);
  uint64_t* bar_q = bars;
  uint64_t* bar_kfull = bars + 1;
  uint64_t* bar_vfull = bar_kfull + C::STAGES;
  uint64_t* bar_kvempty = bar_vfull + C::STAGES;
  uint64_t* bar_sfull = bar_kvempty + C::STAGES;
  uint64_t* bar_pfull = bar_sfull + C::NSLOT;
  uint64_t* bar_pvdone = bar_pfull + C::NSLOT;
  uint64_t* bar_mma_done = bar_pvdone + C::NSLOT;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* walk_n = reinterpret_cast<int*>(tmem_slot + 2);
  int* walk_shard = reinterpret_cast<int*>(tmem_slot + 4);
  int* walk_end = walk_shard + C::MAX_STEPS;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int tile = blockIdx.x % w.n_q_tiles;
  const int r = w.r_first + (blockIdx.x / w.n_q_tiles) * w.r_step;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int t0 = tile * C::BM;
  const int rows_valid = min(C::BM, w.n_q - t0);
  const long long q_pos0 = w.q_off + static_cast<long long>(r) * w.q_rstep;
  const long long pos_last = q_pos0 + static_cast<long long>(t0 + rows_valid - 1) * w.q_tstride;

  WaitCtl ctl{abort_flag, w.wait_limit_ns, w.dev_status};

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(bar_kfull + i, 1);
      mbar_init(bar_vfull + i, 1);
      mbar_init(bar_kvempty + i, 1);
    }
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(bar_sfull + i, 1);
      mbar_init(bar_pfull + i, 128);
      mbar_init(bar_pvdone + i, 1);
    }
    mbar_init(bar_mma_done, 1);
    *abort_flag = 0;
    // The KV shards this tile visits, in ring order, and how many key tiles of each are not
    // entirely in the causal future of the tile's last row.
    int total = 0, n = 0;
    for (int i = 0; i < n_steps; ++i) {
      int s = (r - (w.ring_step + i)) % w.P;
      if (s < 0) s += w.P;
      const int lim = visible_key_limit(w, pos_last, s);
      const int nt = (lim + C::BN - 1) / C::BN;
      if (nt > 0) {
        total += nt;
        walk_shard[n] = s;
        walk_end[n] = total;
        ++n;
      }
    }
    *walk_n = n;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_map(&tm_q);
    tma_prefetch_map(&tm_k);
    tma_prefetch_map(&tm_v);
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_walk = *walk_n;
  const int n_tiles = n_walk > 0 ? walk_end[n_walk - 1] : 0;

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && n_tiles > 0) {
      int issued = 0;
      mbar_arrive_expect_tx(bar_q, C::TILE_BYTES);
#pragma unroll
      for (int cb = 0; cb < C::NCB; ++cb)
        tma_load_5d(sQ + cb * C::BLOCK_BYTES, &tm_q, bar_q, cb * C::CB, t0, r, h, b);
      int wi = 0, tile_base = 0;
      for (int j = 0; j < n_tiles; ++j) {
        while (j >= walk_end[wi]) tile_base = walk_end[wi++];
        const int s = walk_shard[wi];
        const int u0 = (j - tile_base) * C::BN;
        const int st = j % C::STAGES;
        if (j >= C::STAGES && !mbar_wait(bar_kvempty + st, ((j / C::STAGES) - 1) & 1, ctl, 0x101)) break;
        mbar_arrive_expect_tx(bar_kfull + st, C::TILE_BYTES);
#pragma unroll
        for (int cb = 0; cb < C::NCB; ++cb)
          tma_load_5d(sK + st * C::TILE_BYTES + cb * C::BLOCK_BYTES, &tm_k, bar_kfull + st, cb * C::CB, u0, s, h, b);
        mbar_arrive_expect_tx(bar_vfull + st, C::TILE_BYTES);
#pragma unroll
        for (int cb = 0; cb < C::NCB; ++cb)
          tma_load_5d(sV + st * C::TILE_BYTES + cb * C::BLOCK_BYTES, &tm_v, bar_vfull + st, cb * C::CB, u0, s, h, b);
        issued = j + 1;
      }
      // Make sure no TMA write to shared memory is still in flight when the CTA exits.
      mbar_drain(bar_q, 0, w.wait_limit_ns);
      for (int j = max(0, issued - C::STAGES); j < issued; ++j) {
        mbar_drain(bar_kfull + j % C::STAGES, (j / C::STAGES) & 1, w.wait_limit_ns);
        mbar_drain(bar_vfull + j % C::STAGES, (j / C::STAGES) & 1, w.wait_limit_ns);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t idesc_qk = make_idesc_bf16(128, C::BN, 0, 0);
      constexpr uint32_t idesc_pv = make_idesc_bf16(128, DP, 0, 1);
      const uint32_t q_base = smem_addr(sQ);
      const uint32_t k_base = smem_addr(sK);
      const uint32_t v_base = smem_addr(sV);
      bool ok = mbar_wait(bar_q, 0, ctl, 0x201);
      for (int j = 0; ok && j <= n_tiles; ++j) {
        if (j < n_tiles) {
          const int st = j % C::STAGES;
          const int slot = j % C::NSLOT;
          ok = mbar_wait(bar_kfull + st, (j / C::STAGES) & 1, ctl, 0x202);
          if (ok && j >= C::NSLOT) ok = mbar_wait(bar_pvdone + slot, ((j - C::NSLOT) / C::NSLOT) & 1, ctl, 0x203);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d_s = tmem + slot * 128;
#pragma unroll
          for (int kk = 0; kk < DP / 16; ++kk) {
            const int cb = (kk * 16) / C::CB;
            const uint32_t koff = ((kk * 16) % C::CB) * 2;
            const uint64_t a = make_smem_desc(q_base + cb * C::BLOCK_BYTES + koff, 16, C::ATOM_BYTES, C::SWZ);
            const uint64_t bd =
                make_smem_desc(k_base + st * C::TILE_BYTES + cb * C::BLOCK_BYTES + koff, 16, C::ATOM_BYTES, C::SWZ);
            mma_ss(d_s, a, bd, idesc_qk, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar_sfull + slot);
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int st = jj % C::STAGES;
          const int slot = jj % C::NSLOT;
          ok = mbar_wait(bar_pfull + slot, (jj / C::NSLOT) & 1, ctl, 0x204);
          if (ok) ok = mbar_wait(bar_vfull + st, (jj / C::STAGES) & 1, ctl, 0x205);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < C::BN / 16; ++kk) {
            const uint32_t a_tmem = tmem + slot * 128 + kk * 8;
            const uint64_t bd = make_smem_desc(v_base + st * C::TILE_BYTES + kk * 16 * C::ROW_BYTES, C::BLOCK_BYTES,
                                               C::ATOM_BYTES, C::SWZ);
            mma_ts(tmem + C::O_COL, a_tmem, bd, idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar_pvdone + slot);
          mma_commit(bar_kvempty + st);
        }
      }
      // Tensor memory is freed below only after every MMA issued here has completed.
      mma_commit(bar_mma_done);
      mbar_drain(bar_mma_done, 0, w.wait_limit_ns);
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int row = threadIdx.x;  // 0..127 == tensor-memory lane
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const bool row_ok = row < rows_valid;
    const long long pos_q = q_pos0 + static_cast<long long>(t0 + row) * w.q_tstride;
    const float sl2 = w.scale_log2;
    float m_used = -INFINITY;  // running max of scaled scores, log2 units
    float l_sum = 0.f;         // running sum of 2^(x - m_used)
    bool ok = true;
    int wi = 0, tile_base = 0;
    int row_lim = (n_tiles > 0 && row_ok) ? visible_key_limit(w, pos_q, walk_shard[0]) : w.n_kv;
    for (int j = 0; j < n_tiles; ++j) {
      if (j >= walk_end[wi]) {
        tile_base = walk_end[wi++];
        row_lim = row_ok ? visible_key_limit(w, pos_q, walk_shard[wi]) : w.n_kv;
      }
      const int slot = j % C::NSLOT;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_sfull + slot, (j / C::NSLOT) & 1, ctl, 0x301));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lane_addr + slot * 128 + c * 32, sr[c]);
      tmem_ld_wait(sr[0]);
      reg_dep(sr[1]);
      reg_dep(sr[2]);
      reg_dep(sr[3]);

      const int lim = row_lim - (j - tile_base) * C::BN;  // keys [0, lim) of this tile are visible
      if (lim < C::BN) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= lim) sr[c >> 5][c & 31] = __float_as_uint(-INFINITY);
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) mx = fmaxf(mx, __uint_as_float(sr[c >> 5][c & 31]));
      const float m_tile = mx * sl2;
      float m_new = m_used;
      float alpha = 1.f;
      bool rescale = false;
      if (m_tile > m_used) {
        if (m_used == -INFINITY) {
          m_new = m_tile;  // nothing accumulated yet: this row of O is still zero
        } else if (m_tile > m_used + 8.f) {
          m_new = m_tile;
          alpha = ex2_approx(m_used - m_new);
          rescale = true;
        }
      }
      const float base = (m_new == -INFINITY) ? 0.f : m_new;
      float rs = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = ex2_approx(fmaf(__uint_as_float(sr[(2 * c) >> 5][(2 * c) & 31]), sl2, -base));
        const float p1 = ex2_approx(fmaf(__uint_as_float(sr[(2 * c + 1) >> 5][(2 * c + 1) & 31]), sl2, -base));
        rs += p0 + p1;
        pk[c] = pack_bf16x2(p0, p1);
      }
      if (__any_sync(0xffffffffu, rescale)) {
        // O holds sum_{i<j} P_i V_i only once PV_{j-1} has completed.
        const int jp = j - 1;
        ok = __all_sync(0xffffffffu, mbar_wait(bar_pvdone + jp % C::NSLOT, (jp / C::NSLOT) & 1, ctl, 0x302));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < DP / 32; ++c) {
          uint32_t orow[32];
          tmem_ld32(lane_addr + C::O_COL + c * 32, orow);
          tmem_ld_wait(orow);
#pragma unroll
          for (int e = 0; e < 32; ++e) orow[e] = __float_as_uint(__uint_as_float(orow[e]) * alpha);
          tmem_st32(lane_addr + C::O_COL + c * 32, orow);
        }
      }
      l_sum = l_sum * alpha + rs;
      m_used = m_new;
      tmem_st16(lane_addr + slot * 128, pk);
      tmem_st16(lane_addr + slot * 128 + 16, pk + 16);
      tmem_st16(lane_addr + slot * 128 + 32, pk + 32);
      tmem_st16(lane_addr + slot * 128 + 48, pk + 48);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_pfull + slot);
    }

    // ---------------------------------------------------------------- epilogue
    // Merging with an empty partial is the identity: nothing to read or write.
    if (EPI == kEpiAcc && n_tiles == 0) ok = false;
    if (ok && n_tiles > 0) {
      const int jl = n_tiles - 1;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_pvdone + jl % C::NSLOT, (jl / C::NSLOT) & 1, ctl, 0x303));
      if (ok) tc_fence_after();
    }
    if (ok) {
      const bool has = l_sum > 0.f;
      const float inv_l = has ? 1.f / l_sum : 0.f;
      // LSE in natural log: sum_j e^{scale q.k_j} = 2^{m_used} * l_sum.
      const float lse_part = has ? (m_used * 0.69314718055994531f + logf(l_sum)) : -INFINITY;
      float L = lse_part, w_part = 1.f, w_acc = 0.f;
      float* acc_row = nullptr;
      if (EPI == kEpiPart || EPI == kEpiAcc || EPI == kEpiAccOut) {
        acc_row = w.acc_o + b * w.a_sb + h * w.a_sh + r * w.a_rs + static_cast<long long>(t0 + row) * w.a_ts;
      }
      float* accl_ptr = nullptr;
      if (EPI != kEpiOut)
        accl_ptr = w.acc_l + b * w.al_sb + h * w.al_sh + r * w.al_rs + static_cast<long long>(t0 + row) * w.al_ts;
      if ((EPI == kEpiAcc || EPI == kEpiAccOut) && row_ok) {
        const float la = *accl_ptr;
        lse_merge_weights(la, lse_part, L, w_acc, w_part);
      }
      __nv_bfloat16* out_row = nullptr;
      if (EPI == kEpiOut || EPI == kEpiAccOut)
        out_row = static_cast<__nv_bfloat16*>(w.o) + b * w.o_sb + h * w.o_sh + r * w.o_rs +
                  static_cast<long long>(t0 + row) * w.o_ts;
      const float wp = w_part * inv_l;
#pragma unroll
      for (int c = 0; c < DP / 32; ++c) {
        uint32_t orow[32];
        if (n_tiles > 0) {
          tmem_ld32(lane_addr + C::O_COL + c * 32, orow);
          tmem_ld_wait(orow);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) orow[e] = 0u;
        }
        if (row_ok) {
          float vals[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) vals[e] = __uint_as_float(orow[e]) * wp;
          if (EPI == kEpiAcc || EPI == kEpiAccOut) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              if (c * 32 + e < w.d) {
                const float4 a = *reinterpret_cast<const float4*>(acc_row + c * 32 + e);
                vals[e] = fmaf(w_acc, a.x, vals[e]);
                vals[e + 1] = fmaf(w_acc, a.y, vals[e + 1]);
                vals[e + 2] = fmaf(w_acc, a.z, vals[e + 2]);
                vals[e + 3] = fmaf(w_acc, a.w, vals[e + 3]);
              }
            }
          }
          if (EPI == kEpiPart || EPI == kEpiAcc) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              if (c * 32 + e < w.d)
                *reinterpret_cast<float4*>(acc_row + c * 32 + e) =
                    make_float4(vals[e], vals[e + 1], vals[e + 2], vals[e + 3]);
          } else {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              if (c * 32 + e < w.d) {
                uint4 pkt;
                pkt.x = pack_bf16x2(vals[e], vals[e + 1]);
                pkt.y = pack_bf16x2(vals[e + 2], vals[e + 3]);
                pkt.z = pack_bf16x2(vals[e + 4], vals[e + 5]);
                pkt.w = pack_bf16x2(vals[e + 6], vals[e + 7]);
                *reinterpret_cast<uint4*>(out_row + c * 32 + e) = pkt;
              }
            }
          }
        }
      }
      if (row_ok) {
        if (EPI == kEpiPart || EPI == kEpiAcc) {
          *accl_ptr = L;
        } else if (w.lse != nullptr) {
          w.lse[b * w.l_sb + h * w.l_sh + r * w.l_rs + static_cast<long long>(t0 + row) * w.l_ts] = L;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace ra
