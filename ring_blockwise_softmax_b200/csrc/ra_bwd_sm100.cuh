// ra_bwd_sm100.cuh - backward pass of softmax attention on the sm_100a tensor cores (bf16 inputs,
// fp32 accumulation, fp32 gradients).
//
// What it computes: the gradients of L = sum(dO * O) with respect to Q, K and V for O =
// softmax(scale Q K^T) V, with the attention weights recomputed from the forward's saved LSE
// instead of being stored (intelliparadigm.com "深度学习注意力机制优化与FlashAttention实践" §3.3
// and §4.1, item 3):
//   P = e^{S - LSE} on visible entries (S = scale Q K^T),  D_i = sum_c dO_ic O_ic,
//   dV = P^T dO,   dS = P * (dO V^T - D),   dQ = scale dS K,   dK = scale dS^T Q.
// Visibility is the forward's: all keys, causal (key index <= query index), or a causal sliding
// window of `window` positions; K and V may have fewer heads than Q (query head h uses K/V head
// h / (H / H_kv)), and dK, dV then sum over the heads of the group.
//
// One kernel template serves both halves.  A CTA holds a FIXED block of 128 rows of two
// operands (A1, A2) in shared memory and streams 64-row tiles of two or three others (B1, B2,
// B3) through a STAGES-deep ring; per tile, with the fixed rows on the 128 tensor-memory lanes:
//   S  = A1 B1^T,  dP = A2 B2^T             (tcgen05 SS form, fp32 in tensor memory)
//   P  = exp2(S log2(e) - LSE log2(e)),  dS = P (dP - D)      (fp32 registers, stored as bf16
//                                                             pairs into tensor memory)
//   ACC1 += dS B1,  ACC2 += P B2            (TS form: A from tensor memory, B MN-major)
// KV = true:  A1 = K, A2 = V of a block of keys, B1 = Q, B2 = dO, B3 = O of 64 query rows of
//             every query head of the K/V head's group: ACC1 = dK / scale, ACC2 = dV.  The
//             query rows' LSE and D (= dO . O, from the staged O tile) go through shared memory.
// KV = false: A1 = Q, A2 = dO of a block of query rows, B1 = K, B2 = V of 64 keys:
//             ACC1 = dQ / scale.  The rows' LSE and D sit in registers.
// S and dP here are the transposes of each other's roles in the two instances, so both use the
// forward's operand forms unchanged.  No atomics: every gradient element has one owner.
//
// Roles: two element-wise warpgroups (warps 0-3 and 4-7) take alternate streamed tiles, thread =
// tensor-memory lane (warp % 4) * 32 + lane, all 64 columns of its row; each warpgroup has its
// own (S, dP) buffer and P, dS columns in tensor memory, so one computes while the other waits on
// its loads, stores and barriers.  (The dK/dV instance at DP = 128 lacks the tensor memory for
// that and runs attn_bwd_sm100_split, further below.)  Warp 8 is the TMA producer (and allocates
// tensor memory); warps 9, 10 and 11 issue the MMAs: S and dP of tile j + 2 (warps 9, 10) as soon
// as warpgroup j % 2 holds tile j in registers, the products of each tile (warp 11) once its P
// and dS are stored.  The dK/dV instance adds warps 12-15, which compute the streamed rows' LSE
// and D a few tiles ahead into shared-memory slots.  Registers are rebalanced with setmaxnreg
// (BwdCfg::REG_*).  At the end the eight element-wise warps run the epilogue.  Every wait is
// bounded.
#pragma once

#include "ra_common.cuh"

namespace ra {

struct BwdTcWork {
  int B, H, H_kv, n_q, n_kv, d;
  int qpk;  // H / H_kv
  int causal;
  long long window;  // 0 = none (causal only)
  float scale;
  float scale_log2;  // scale * log2(e)
  const float* lse;  // [B, H, n_q] contiguous (natural log)
  // O and dO, read directly for the per-row D of the dQ instance.
  const __nv_bfloat16* o;
  long long o_sb, o_sh, o_st;
  const __nv_bfloat16* d_o;
  long long do_sb, do_sh, do_st;
  // Outputs: out1 = dQ (KV = false) or dK (KV = true); out2 = dV (KV = true).  fp32.
  float* out1;
  long long o1_sb, o1_sh, o1_st;
  float* out2;
  long long o2_sb, o2_sh, o2_st;
  unsigned long long wait_limit_ns;
  unsigned int* dev_status;
  int global_order;  // remap CTAs to one heavy-first order over all heads (see bwd_range)
};

template <int DP, bool KV>
struct BwdCfg {
  static_assert(DP == 32 || DP == 64 || DP == 128, "padded head dim must be 32, 64 or 128");
  static constexpr int BM = 128;  // fixed rows (tensor-memory lanes)
  static constexpr int BN = 64;   // rows of a streamed tile (tensor-memory columns of S, dP)
  static constexpr int CB = (DP == 32) ? 32 : 64;  // columns per TMA box / swizzle span
  static constexpr int NCB = DP / CB;
  static constexpr int ROW_BYTES = CB * 2;
  static constexpr uint32_t SWZ = (DP == 32) ? kSwizzle64B : kSwizzle128B;
  static constexpr int ATOM_BYTES = 8 * ROW_BYTES;
  static constexpr int BLK_M = BM * ROW_BYTES;  // one column block of a fixed operand
  static constexpr int BLK_N = BN * ROW_BYTES;  // one column block of a streamed operand
  static constexpr int FIX_BYTES = BM * DP * 2;
  static constexpr int TILE_BYTES = BN * DP * 2;
  static constexpr int NSTREAM = KV ? 3 : 2;
  static constexpr int STAGE_BYTES = NSTREAM * TILE_BYTES;
  static constexpr int STAGES_FIT = (220 * 1024 - 2 * FIX_BYTES) / STAGE_BYTES;  // of 227 KB
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  static_assert(STAGES >= 2, "shared memory holds fewer than two stages");
  static constexpr int NACC = KV ? 2 : 1;
  // Tensor-memory columns (512 allocated).  Warpgroup g: (S, dP) buffer at g * 128 (S in its
  // first 64 columns, dP in the next 64) and P, dS (bf16 pairs, 32 columns each) at
  // P_COL(g), DS_COL(g); ACC1, ACC2 (DP columns each) from ACC_COL.  This leaves room for
  // NACC * DP <= 128: every instance but dK/dV at DP = 128, which runs the column-split kernel
  // (BwdCfgSplit) instead.
  static constexpr int SB_STRIDE = 128;
  static constexpr int S_COL = 0;
  static constexpr int DP_COL = 64;
  static constexpr int ACC_COL = 384;
  __host__ __device__ static constexpr int P_COL(int g) { return 256 + g * 64; }
  __host__ __device__ static constexpr int DS_COL(int g) { return 256 + g * 64 + 32; }
  static_assert(ACC_COL + NACC * DP <= 512, "tensor memory overflow: use the column-split kernel");
  // The issuer starts S(j + 2) before the products of tile j, which needs the stage of tile j + 2
  // loaded while tile j's is still held: three stages.
  static_assert(STAGES >= 3, "the look-ahead needs a third stage");
  // Barriers: fixed_full, stage_full[S], stage_empty[S], s_full[2], s_free[2], p_full[2],
  // pv_done[2], acc_done, stats_ready[4], stats_free[4] (per statistics slot).
  static constexpr int NSLOT = 4;  // statistics slots: tile j uses slot j % NSLOT
  static constexpr int NBAR = 1 + 2 * STAGES + 8 + 1 + 2 * NSLOT;
  static constexpr int BAR_BYTES = (NBAR * 8 + 15) / 16 * 16;
  // + tensor-memory slot and abort flag (16 B) + statistics [NSLOT][BN] float2.
  static constexpr int SMEM_BYTES = 1024 + 2 * FIX_BYTES + STAGES * STAGE_BYTES + BAR_BYTES + 16 + NSLOT * BN * 8;
  // The dK/dV instance has a fourth warpgroup (warps 12-15) that computes the streamed rows'
  // statistics (LSE, D) ahead of the element-wise warps.
  static constexpr bool STATS_WG = KV;
  static constexpr int THREADS = STATS_WG ? 512 : 384;
  // Registers: at launch 65536 / THREADS (rounded down to 8) for every thread; the control
  // warpgroup (producer and issuers) keeps REG_CTL, the statistics warpgroup REG_ST, and the
  // element-wise warpgroups take the rest.
  static constexpr int REG_LAUNCH = (65536 / THREADS) / 8 * 8;
  static constexpr int REG_CTL = 96;
  static constexpr int REG_ST = 40;
  static constexpr int REG_EW = ((REG_LAUNCH * THREADS - 128 * REG_CTL - (STATS_WG ? 128 * REG_ST : 0)) / 256) / 8 * 8;
  static constexpr int REG_TOTAL = 256 * REG_EW + 128 * REG_CTL + (STATS_WG ? 128 * REG_ST : 0);
  static_assert(REG_TOTAL <= REG_LAUNCH * THREADS, "register split exceeds the launch");
};

// The streamed tiles of one CTA: tiles tb .. te-1 (of BN rows) of each of `heads` streamed heads.
struct BwdRange {
  int b, hf;     // batch, head of the fixed operands
  int m0;        // first fixed row
  int tb, te;    // streamed tile range
  int heads;     // streamed heads (query heads of the group, or 1)
  int n;         // heads * (te - tb), or 0
};

template <bool KV>
__device__ __forceinline__ BwdRange bwd_range(const BwdTcWork& w) {
  BwdRange r;
  // CTAs start in linear block order (x fastest), heavy-first within each head.  With
  // w.global_order the linear index is remapped so that the heaviest blocks of every head come
  // first, then the next heaviest of every head, and so on: one global heavy-first order, which
  // balances causal work over the SMs better (B=2 H=16 N=8192 d=64: +4 %) but spreads the CTAs
  // running at one time over every head, which costs L2 locality (B=1 H=32 N=32768 d=128: -4 %).
  // The host sets it for causal launches of few waves of CTAs, where the balance matters.
  int level;  // 0 = heaviest
  if (w.global_order) {
    const int lin = static_cast<int>(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z));
    const int nhb = static_cast<int>(gridDim.y * gridDim.z);
    level = lin / nhb;
    const int hb = lin - level * nhb;
    r.b = hb / static_cast<int>(gridDim.y);
    r.hf = hb - r.b * static_cast<int>(gridDim.y);
  } else {
    level = static_cast<int>(blockIdx.x);
    r.b = static_cast<int>(blockIdx.z);
    r.hf = static_cast<int>(blockIdx.y);
  }
  constexpr int BM = 128, BN = 64;
  if (KV) {
    // Key blocks: the first ones are seen by the most query rows (causal).
    r.m0 = level * BM;
    const int m_last = min(r.m0 + BM, w.n_kv) - 1;
    const int lo = w.causal ? r.m0 : 0;
    int hi = w.n_q;
    if (w.causal && w.window > 0) hi = static_cast<int>(min(static_cast<long long>(w.n_q), m_last + w.window));
    r.heads = w.qpk;
    r.tb = lo / BN;
    r.te = lo < hi ? (hi + BN - 1) / BN : r.tb;
  } else {
    // Query blocks last-first: under a causal mask the last rows see the most keys.
    r.m0 = (static_cast<int>(gridDim.x) - 1 - level) * BM;
    const int m_last = min(r.m0 + BM, w.n_q) - 1;
    const int hi = w.causal ? min(w.n_kv, m_last + 1) : w.n_kv;
    int lo = 0;
    if (w.causal && w.window > 0) lo = static_cast<int>(max(0LL, r.m0 - w.window + 1));
    r.heads = 1;
    r.tb = lo / BN;
    r.te = lo < hi ? (hi + BN - 1) / BN : r.tb;
  }
  r.n = r.heads * (r.te - r.tb);
  return r;
}

// Warpgroup-wide register reallocation (every warp of the warpgroup executes it).  An increase
// waits until the block's register pool, fixed at launch, has the registers free: the host checks
// the compiled kernel's pool against the split before every launch.
template <int N>
__device__ __forceinline__ void bwd_setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void bwd_setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // low 16 bits = lo
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bwd_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Keep the compiler from using `r` before an earlier tcgen05.wait::ld (a second register array
// loaded before the same wait).
__device__ __forceinline__ void reg_pin32(uint32_t (&r)[32]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

// Waits use the suspending try_wait (mbar_wait): spinning on the non-blocking test measured slower
// here, both for the issuer and for the element-wise warps.
__device__ __forceinline__ bool bwd_wait2(uint64_t* b0, uint32_t p0, uint64_t* b1, uint32_t p1, const WaitCtl& ctl,
                                          unsigned site) {
  return mbar_wait(b0, p0, ctl, site) && (b1 == nullptr || mbar_wait(b1, p1, ctl, site + 1));
}

__device__ __forceinline__ bool bwd_wait(uint64_t* bar, uint32_t parity, const WaitCtl& ctl, unsigned site) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, ctl, site));
}

__device__ __forceinline__ void bwd_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) break;
  }
}

template <int DP, bool KV>
__global__ void __launch_bounds__(BwdCfg<DP, KV>::THREADS, 1)
    attn_bwd_sm100(const __grid_constant__ CUtensorMap tm_a1, const __grid_constant__ CUtensorMap tm_a2,
                   const __grid_constant__ CUtensorMap tm_b1, const __grid_constant__ CUtensorMap tm_b2,
                   const __grid_constant__ CUtensorMap tm_b3, const BwdTcWork w) {
  using C = BwdCfg<DP, KV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sFix = smem;                        // A1 | A2
  uint8_t* sStage = smem + 2 * C::FIX_BYTES;   // STAGES x (B1 | B2 [| B3])
  uint64_t* bars = reinterpret_cast<uint64_t*>(sStage + C::STAGES * C::STAGE_BYTES);
  uint64_t* bar_fixed = bars;
  uint64_t* bar_stage_full = bars + 1;
  uint64_t* bar_stage_empty = bar_stage_full + C::STAGES;
  uint64_t* bar_s_full = bar_stage_empty + C::STAGES;  // [2] per warpgroup
  uint64_t* bar_s_free = bar_s_full + 2;               // [2]
  uint64_t* bar_p_full = bar_s_free + 2;               // [2]
  uint64_t* bar_pv_done = bar_p_full + 2;              // [2]
  uint64_t* bar_acc_done = bar_pv_done + 2;
  uint64_t* bar_stats = bar_acc_done + 1;          // [NSLOT] statistics of the slot's tile written
  uint64_t* bar_stats_free = bar_stats + C::NSLOT;  // [NSLOT] the slot's tile read by its warpgroup
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(bars) + C::BAR_BYTES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // [NSLOT][BN] (LSE log2(e), D) of streamed rows (dK/dV instance); 16-byte aligned.
  float2* s_st = reinterpret_cast<float2*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WaitCtl ctl{abort_flag, w.wait_limit_ns, w.dev_status};
  const BwdRange rg = bwd_range<KV>(w);

  if (threadIdx.x == 0) {
    mbar_init(bar_fixed, 1);
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(bar_stage_full + i, 1);
      mbar_init(bar_stage_empty + i, KV ? 1 + 4 : 1);  // MMA commit (+ the 4 warps reading O)
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_s_full + i, 2);  // the S and the dP issuer
      mbar_init(bar_s_free + i, 4);  // one arrival per warp of the warpgroup
      mbar_init(bar_p_full + i, 4);
      mbar_init(bar_pv_done + i, 1);
    }
    mbar_init(bar_acc_done, 3);  // one commit per issuer
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(bar_stats + i, 4);       // the statistics warpgroup's warps
      mbar_init(bar_stats_free + i, 4);  // the warps of the element-wise warpgroup that read it
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    if (lane == 0) {
      tma_prefetch_map(&tm_a1);
      tma_prefetch_map(&tm_a2);
      tma_prefetch_map(&tm_b1);
      tma_prefetch_map(&tm_b2);
      if (KV) tma_prefetch_map(&tm_b3);
    }
    __syncwarp();
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The dK/dV launch follows the dQ launch as a programmatic dependent (the two read the same
  // inputs and write different outputs), so its CTAs may fill SMs the dQ grid leaves idle at its
  // end.  Every CTA waits for any such prerequisite grid before it exits (below), so neither
  // launch completes before the one ahead of it on the stream.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // Register split (warpgroup-wide): the control warpgroup (warps 8-11) shrinks, and the
  // element-wise warpgroups grow into what it released.
  if (C::STATS_WG && warp >= 12) {
    bwd_setmaxnreg_dec<C::REG_ST>();
    // ============================================================ statistics (dK/dV instance)
    // D = dO . O and LSE log2(e) of the 64 query rows of every streamed tile j, into slot
    // j % NSLOT once the element-wise warpgroup that used the slot's previous tile has read it.
    // Two threads per row, each half of the row's 16-byte chunks of the staged O and dO tiles
    // (both tiles share one swizzled layout, so the same physical chunks pair the same elements).
    // A row's LSE is loaded one tile ahead.
    const int tid = threadIdx.x - 384;
    const int sc = tid >> 1, part = tid & 1;
    auto lse_of = [&](int gg, int tt) -> float {
      const int qi = tt * C::BN + sc;
      const int hq = rg.hf * w.qpk + gg;
      return qi < w.n_q ? w.lse[(static_cast<long long>(rg.b) * w.H + hq) * w.n_q + qi] : -INFINITY;
    };
    int g = 0, t = rg.tb;  // head and tile of tile j
    float lse_next = (part == 0 && rg.n > 0) ? lse_of(g, t) : 0.f;
    bool ok = true;
    for (int j = 0; ok && j < rg.n; ++j) {
      const int slot = j % C::NSLOT, st = j % C::STAGES;
      const float L = lse_next;
      int gn = g, tn = t + 1;
      if (tn == rg.te) {
        tn = rg.tb;
        ++gn;
      }
      if (part == 0 && j + 1 < rg.n) lse_next = lse_of(gn, tn);
      if (j >= C::NSLOT && !(ok = bwd_wait(bar_stats_free + slot, ((j / C::NSLOT) - 1) & 1, ctl, 0x726))) break;
      if (!(ok = bwd_wait(bar_stage_full + st, (j / C::STAGES) & 1, ctl, 0x721))) break;
      constexpr int NCH = DP / 16;    // chunks per thread
      constexpr int CPR = C::CB / 8;  // chunks per row of one column block
      const uint8_t* sdo = sStage + st * C::STAGE_BYTES + C::TILE_BYTES;
      const uint8_t* so = sdo + C::TILE_BYTES;
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
        const int kc = part * NCH + i;
        const int off = (kc / CPR) * C::BLK_N + sc * C::ROW_BYTES + (kc % CPR) * 16;
        const uint4 a = *reinterpret_cast<const uint4*>(so + off);
        const uint4 bb = *reinterpret_cast<const uint4*>(sdo + off);
        const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* y = reinterpret_cast<const __nv_bfloat162*>(&bb);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 fx = __bfloat1622float2(x[e]), fy = __bfloat1622float2(y[e]);
          acc = fmaf(fx.x, fy.x, acc);
          acc = fmaf(fx.y, fy.y, acc);
        }
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      // Rows past the end (LSE -inf here) and empty rows get LSE log2(e) = +inf, so P = 0.
      if (part == 0)
        s_st[slot * C::BN + sc] = make_float2(L == -INFINITY ? INFINITY : L * 1.4426950408889634f, acc);
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar_stage_empty + st);  // this warp is done with the stage's O tile
        mbar_arrive(bar_stats + slot);
      }
      g = gn;
      t = tn;
    }
  } else if (warp >= 8) {
   bwd_setmaxnreg_dec<C::REG_CTL>();
   if (warp == 8) {
    if (lane == 0 && rg.n > 0) {
      // ================================================================ TMA producer
      mbar_arrive_expect_tx(bar_fixed, 2 * C::FIX_BYTES);
#pragma unroll
      for (int cb = 0; cb < C::NCB; ++cb) {
        tma_load_5d(sFix + cb * C::BLK_M, &tm_a1, bar_fixed, cb * C::CB, rg.m0, 0, rg.hf, rg.b);
        tma_load_5d(sFix + C::FIX_BYTES + cb * C::BLK_M, &tm_a2, bar_fixed, cb * C::CB, rg.m0, 0, rg.hf, rg.b);
      }
      int g = 0, t = rg.tb, j = 0;
      for (; j < rg.n; ++j) {
        const int st = j % C::STAGES;
        if (j >= C::STAGES && !mbar_wait(bar_stage_empty + st, ((j / C::STAGES) - 1) & 1, ctl, 0x701)) break;
        const int hs = KV ? rg.hf * w.qpk + g : rg.hf / w.qpk;  // streamed head
        uint8_t* dst = sStage + st * C::STAGE_BYTES;
        mbar_arrive_expect_tx(bar_stage_full + st, C::STAGE_BYTES);
#pragma unroll
        for (int cb = 0; cb < C::NCB; ++cb) {
          tma_load_5d(dst + cb * C::BLK_N, &tm_b1, bar_stage_full + st, cb * C::CB, t * C::BN, 0, hs, rg.b);
          tma_load_5d(dst + C::TILE_BYTES + cb * C::BLK_N, &tm_b2, bar_stage_full + st, cb * C::CB, t * C::BN, 0,
                      hs, rg.b);
          if (KV)
            tma_load_5d(dst + 2 * C::TILE_BYTES + cb * C::BLK_N, &tm_b3, bar_stage_full + st, cb * C::CB,
                        t * C::BN, 0, hs, rg.b);
        }
        if (++t == rg.te) {
          t = rg.tb;
          ++g;
        }
      }
      // No TMA write may still be in flight when the CTA exits.
      bwd_drain(bar_fixed, 0, w.wait_limit_ns);
      for (int i = (j > C::STAGES ? j - C::STAGES : 0); i < j; ++i)
        bwd_drain(bar_stage_full + i % C::STAGES, (i / C::STAGES) & 1, w.wait_limit_ns);
    }
   } else {
    if (lane == 0) {
      // ================================================================ MMA issuers
      // Three issuing threads (warp 9: S, warp 10: dP, warp 11: the gradient products): one
      // thread issues a tcgen05.mma about every 115 cycles whatever its size, far below the tensor
      // core's rate for these 128 x 64 x 16 and 128 x d x 16 shapes, so the MMA rate grows with
      // the number of issuing threads.
      constexpr uint32_t idesc_s = make_idesc_bf16(128, C::BN, 0, 0);
      constexpr uint32_t idesc_acc = make_idesc_bf16(128, DP, 0, 1);
      const uint64_t kmaj = make_smem_desc(0, 16, C::ATOM_BYTES, C::SWZ);
      const uint64_t mn = make_smem_desc(0, C::BLK_N, C::ATOM_BYTES, C::SWZ);
      const uint32_t a1 = smem_addr(sFix), a2 = a1 + C::FIX_BYTES;
      const uint32_t stage0 = smem_addr(sStage);
      // S, dP of tile jj into the buffer of warpgroup jj % 2, once the tile's stage has landed and
      // the warpgroup holds its previous tile (jj - 2) in registers.
      auto issue_s = [&](int jj) -> bool {
        const int st = jj % C::STAGES, b = jj & 1;
        if (!bwd_wait2(bar_stage_full + st, (jj / C::STAGES) & 1, jj >= 2 ? bar_s_free + b : nullptr,
                       ((jj >> 1) - 1) & 1, ctl, 0x712))
          return false;
        tc_fence_after();
        // S = A1 B1^T (warp 9) or dP = A2 B2^T (warp 10); s_full completes on both commits.
        const uint32_t bx = stage0 + st * C::STAGE_BYTES + (warp == 9 ? 0 : C::TILE_BYTES);
        const uint32_t ax = warp == 9 ? a1 : a2;
        const uint64_t da = kmaj | ((ax >> 4) & 0x3FFFu), dbx = kmaj | ((bx >> 4) & 0x3FFFu);
        const uint32_t col = tmem + b * C::SB_STRIDE + (warp == 9 ? C::S_COL : C::DP_COL);
#pragma unroll
        for (int kk = 0; kk < DP / 16; ++kk) {
          const int cb = (kk * 16) / C::CB;
          const uint32_t in = ((kk * 16) % C::CB) * 2;
          const uint32_t offa = (cb * C::BLK_M + in) >> 4, offb = (cb * C::BLK_N + in) >> 4;
          mma_ss(col, da + offa, dbx + offb, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_s_full + b);
        return true;
      };
      // ACC1 += dS B1 (and ACC2 += P B2) of tile jj, once its P and dS are in tensor memory; then
      // its stage and the warpgroup's P, dS columns are released.
      auto issue_acc = [&](int jj) -> bool {
        const int b = jj & 1;
        if (!mbar_wait(bar_p_full + b, (jj >> 1) & 1, ctl, 0x714)) return false;
        tc_fence_after();
        const int sp = jj % C::STAGES;
        const uint32_t b1 = stage0 + sp * C::STAGE_BYTES, b2 = b1 + C::TILE_BYTES;
        const uint64_t mb1 = mn | ((b1 >> 4) & 0x3FFFu), mb2 = mn | ((b2 >> 4) & 0x3FFFu);
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          const uint32_t off = (kk * 16 * C::ROW_BYTES) >> 4;
          const uint32_t acc = (jj > 0 || kk > 0) ? 1u : 0u;
          mma_ts(tmem + C::ACC_COL, tmem + C::DS_COL(b) + kk * 8, mb1 + off, idesc_acc, acc);
          if (KV) mma_ts(tmem + C::ACC_COL + DP, tmem + C::P_COL(b) + kk * 8, mb2 + off, idesc_acc, acc);
        }
        mma_commit(bar_pv_done + b);
        mma_commit(bar_stage_empty + sp);
        return true;
      };
      if (warp == 9 || warp == 10) {
        // S (dP) of every tile, each as soon as its stage has landed and its warpgroup holds the
        // tile two before it in registers.
        bool ok = rg.n > 0 && mbar_wait(bar_fixed, 0, ctl, 0x711);
        for (int j = 0; ok && j < rg.n; ++j) ok = issue_s(j);
      } else {
        // The products of every tile, as soon as its P and dS are in tensor memory.
        bool ok = rg.n > 0;
        for (int j = 0; ok && j < rg.n; ++j) ok = issue_acc(j);
      }
      // The epilogue waits on acc_done: every MMA either issuer issued has completed (also after
      // an abort).
      if (rg.n > 0)
        mma_commit(bar_acc_done);
      else
        mbar_arrive(bar_acc_done);
      bwd_drain(bar_acc_done, 0, w.wait_limit_ns);
    }
   }
  } else {
    bwd_setmaxnreg_inc<C::REG_EW>();
    // ==================================================================== element-wise (warps 0-7)
    const int grp = warp >> 2;  // warpgroup: streamed tiles j with j % 2 == grp
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t sbuf = lane_addr + grp * C::SB_STRIDE;
    const int fixed_pos = rg.m0 + row;
    const long long win = w.causal ? w.window : 0;
    // Per-row statistics of the fixed rows (dQ instance): LSE log2(e) and D = dO . O.
    float row_l2 = INFINITY, row_d = 0.f;
    if (!KV && fixed_pos < w.n_q) {
      const float L = w.lse[(static_cast<long long>(rg.b) * w.H + rg.hf) * w.n_q + fixed_pos];
      row_l2 = (L == -INFINITY) ? INFINITY : L * 1.4426950408889634f;
      const uint4* po = reinterpret_cast<const uint4*>(w.o + rg.b * w.o_sb + rg.hf * w.o_sh + fixed_pos * w.o_st);
      const uint4* pd = reinterpret_cast<const uint4*>(w.d_o + rg.b * w.do_sb + rg.hf * w.do_sh + fixed_pos * w.do_st);
      float acc = 0.f;
      for (int c = 0; c < w.d / 8; ++c) {
        const uint4 a = po[c], bb = pd[c];
        const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* y = reinterpret_cast<const __nv_bfloat162*>(&bb);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 fx = __bfloat1622float2(x[e]), fy = __bfloat1622float2(y[e]);
          acc = fmaf(fx.x, fy.x, acc);
          acc = fmaf(fx.y, fy.y, acc);
        }
      }
      row_d = acc;
    }
    auto advance = [&](int& gg, int& tt) {
      if (++tt == rg.te) {
        tt = rg.tb;
        ++gg;
      }
    };
    bool ok = true;
    int g = 0, t = rg.tb;  // head and tile of tile j
    if (grp == 1) advance(g, t);
    int k = 0;  // tiles of this warpgroup so far
    for (int j = grp; ok && j < rg.n; j += 2, ++k) {
      const int t0 = t * C::BN;  // first streamed row of the tile
      if (!(ok = bwd_wait(bar_s_full + grp, k & 1, ctl, 0x722))) break;
      if (KV && !(ok = bwd_wait(bar_stats + j % C::NSLOT, (j / C::NSLOT) & 1, ctl, 0x723))) break;
      tc_fence_after();
      const float4* stv = reinterpret_cast<const float4*>(s_st + (j % C::NSLOT) * C::BN);
      uint32_t pp[32], dd[32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t sv[32], pv[32];
        tmem_ld32(sbuf + C::S_COL + 32 * h, sv);
        tmem_ld32(sbuf + C::DP_COL + 32 * h, pv);
        tmem_ld_wait(sv);
        reg_pin32(pv);
        if (h == 1) {
          // The whole tile is in registers: the issuer may refill this warpgroup's buffer.
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_s_free + grp);
        }
        // Visible columns i (0..31 of this half) satisfy lo <= i < hi.
        const int base = t0 + 32 * h;
        int lo = 0, hi = 32;
        bool masked;
        if (KV) {
          // fixed row = key at fixed_pos; column = query at base + i.
          masked = w.causal && (t0 < rg.m0 + C::BM - 1 || (win > 0 && t0 + C::BN - 1 - rg.m0 >= win));
          if (masked) {
            lo = fixed_pos - base;                                                  // query >= key
            if (win > 0) hi = static_cast<int>(min(32LL, fixed_pos - base + win));  // query < key + win
          }
        } else {
          // fixed row = query at fixed_pos; column = key at base + i.
          masked = (t0 + C::BN > w.n_kv) ||
                   (w.causal && (t0 + C::BN - 1 > rg.m0 || (win > 0 && rg.m0 + C::BM - 1 - t0 >= win)));
          if (masked) {
            hi = min(32, w.n_kv - base);
            if (w.causal) {
              hi = min(hi, fixed_pos - base + 1);                                        // key <= query
              if (win > 0) lo = static_cast<int>(max(0LL, fixed_pos - win + 1 - base));  // key > query - win
            }
          }
        }
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float4 cs = make_float4(row_l2, row_d, row_l2, row_d);  // (LSE log2(e), D) of columns i, i + 1
          if (KV) cs = stv[16 * h + i / 2];
          float e0 = bwd_ex2(fmaf(__uint_as_float(sv[i]), w.scale_log2, -cs.x));
          float e1 = bwd_ex2(fmaf(__uint_as_float(sv[i + 1]), w.scale_log2, -cs.z));
          if (masked) {
            if (i < lo || i >= hi) e0 = 0.f;
            if (i + 1 < lo || i + 1 >= hi) e1 = 0.f;
          }
          pp[16 * h + i / 2] = bf16x2_bits(e0, e1);
          dd[16 * h + i / 2] = bf16x2_bits(e0 * (__uint_as_float(pv[i]) - cs.y), e1 * (__uint_as_float(pv[i + 1]) - cs.w));
        }
      }
      if (KV) {
        // The tile's statistics are in registers: its slot may take the tile NSLOT further on.
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_stats_free + j % C::NSLOT);
      }
      // The warpgroup's P, dS columns are free once the products of its previous tile are done.
      if (k > 0 && !(ok = bwd_wait(bar_pv_done + grp, (k - 1) & 1, ctl, 0x724))) break;
      tc_fence_after();
      if (KV) tmem_st32(lane_addr + C::P_COL(grp), pp);
      tmem_st32(lane_addr + C::DS_COL(grp), dd);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p_full + grp);
      advance(g, t);
      advance(g, t);
    }
    // ================================================================== epilogue
    const bool have = ok && rg.n > 0 && bwd_wait(bar_acc_done, 0, ctl, 0x725);
    if (rg.n == 0 || have) {
      tc_fence_after();
      const int n_rows = KV ? w.n_kv : w.n_q;
      const bool row_ok = fixed_pos < n_rows;
      constexpr int CH = DP / 32;  // 32-column chunks per accumulator
#pragma unroll 1
      for (int q = grp; q < C::NACC * CH; q += 2) {
        const int a = q / CH, ch = q % CH;
        uint32_t v[32];
        if (rg.n > 0) {
          tmem_ld32(lane_addr + C::ACC_COL + a * DP + ch * 32, v);
          tmem_ld_wait(v);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0u;
        }
        if (!row_ok) continue;
        const float f = (a == 0) ? w.scale : 1.f;
        float* dst = (a == 0) ? w.out1 + rg.b * w.o1_sb + rg.hf * w.o1_sh + fixed_pos * w.o1_st
                              : w.out2 + rg.b * w.o2_sb + rg.hf * w.o2_sh + fixed_pos * w.o2_st;
        const int c0 = ch * 32;
        const int nc = min(32, w.d - c0);
        if (nc == 32 && (reinterpret_cast<uintptr_t>(dst + c0) & 15) == 0) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + c0 + i) =
                make_float4(f * __uint_as_float(v[i]), f * __uint_as_float(v[i + 1]),
                            f * __uint_as_float(v[i + 2]), f * __uint_as_float(v[i + 3]));
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < nc) dst[c0 + i] = f * __uint_as_float(v[i]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------------------------------------
// Column-split variant, used where the two warpgroups' P and dS do not fit beside their (S, dP)
// buffers and the accumulators (the dK/dV instance at DP = 128): both warpgroups work on the same
// tile, warps 0-3 on its columns 0-31 and warps 4-7 on columns 32-63, with one (S, dP) buffer
// that the issuer refills as soon as every warp holds the current tile in registers.  Same
// arithmetic, operands and products as attn_bwd_sm100.
// ---------------------------------------------------------------------------------------------
template <int DP, bool KV>
struct BwdCfgSplit {
  static_assert(DP == 32 || DP == 64 || DP == 128, "padded head dim must be 32, 64 or 128");
  static constexpr int BM = 128;  // fixed rows (tensor-memory lanes)
  static constexpr int BN = 64;   // rows of a streamed tile (tensor-memory columns of S, dP)
  static constexpr int CB = (DP == 32) ? 32 : 64;  // columns per TMA box / swizzle span
  static constexpr int NCB = DP / CB;
  static constexpr int ROW_BYTES = CB * 2;
  static constexpr uint32_t SWZ = (DP == 32) ? kSwizzle64B : kSwizzle128B;
  static constexpr int ATOM_BYTES = 8 * ROW_BYTES;
  static constexpr int BLK_M = BM * ROW_BYTES;  // one column block of a fixed operand
  static constexpr int BLK_N = BN * ROW_BYTES;  // one column block of a streamed operand
  static constexpr int FIX_BYTES = BM * DP * 2;
  static constexpr int TILE_BYTES = BN * DP * 2;
  static constexpr int NSTREAM = KV ? 3 : 2;
  static constexpr int STAGE_BYTES = NSTREAM * TILE_BYTES;
  static constexpr int STAGES_FIT = (192 * 1024 - 2 * FIX_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  static_assert(STAGES >= 2, "shared memory holds fewer than two stages");
  static constexpr int NACC = KV ? 2 : 1;
  // Tensor-memory columns (512 allocated): NSB buffers of (S, dP) (fp32, 64 columns each), P and
  // dS (bf16 pairs, 32 columns each), ACC1 and ACC2 (DP columns each).  Two (S, dP) buffers let
  // the issuer compute the tile after next while the element-wise warps work; the dK/dV instance
  // at DP = 128 has room for one.
  static constexpr int NSB = (NACC * DP + 384 <= 512) ? 2 : 1;
  static constexpr int SB_STRIDE = 128;  // columns between (S, dP) buffers
  static constexpr int S_COL = 0;
  static constexpr int DP_COL = 64;
  static constexpr int P_COL = NSB * SB_STRIDE;
  static constexpr int DS_COL = P_COL + 32;
  static constexpr int ACC_COL = NSB == 2 ? 384 : 256;
  static_assert(ACC_COL + NACC * DP <= 512, "tensor memory overflow");
  static_assert(NSB == 1 || STAGES >= 3, "a second (S, dP) buffer needs a third stage in flight");
  // Barriers: fixed_full, stage_full[S], stage_empty[S], s_full[2], s_free[2], p_full, pv_done,
  // acc_done, stats_ready[2].
  static constexpr int NBAR = 1 + 2 * STAGES + 7 + 2;
  static_assert((NBAR * 8) % 16 == 0, "statistics buffer must stay 16-byte aligned");
  static constexpr int SMEM_BYTES = 1024 + 2 * FIX_BYTES + STAGES * STAGE_BYTES + NBAR * 8 + 16 + 4 * BN * 4;
  static constexpr int THREADS = 384;
  // Registers: at launch 65536 / THREADS (rounded down to 8) for every thread; the control
  // warpgroup (producer and issuers) gives up all but REG_CTL to the element-wise warpgroups.
  static constexpr int REG_LAUNCH = (65536 / THREADS) / 8 * 8;
  static constexpr int REG_CTL = 96;
  static constexpr int REG_EW = ((REG_LAUNCH * THREADS - 128 * REG_CTL) / 256) / 8 * 8;
  static constexpr int REG_TOTAL = 256 * REG_EW + 128 * REG_CTL;
  static_assert(REG_TOTAL <= REG_LAUNCH * THREADS, "register split exceeds the launch");
};

template <int DP, bool KV>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_sm100_split(const __grid_constant__ CUtensorMap tm_a1, const __grid_constant__ CUtensorMap tm_a2,
                   const __grid_constant__ CUtensorMap tm_b1, const __grid_constant__ CUtensorMap tm_b2,
                   const __grid_constant__ CUtensorMap tm_b3, const BwdTcWork w) {
  using C = BwdCfgSplit<DP, KV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sFix = smem;                        // A1 | A2
  uint8_t* sStage = smem + 2 * C::FIX_BYTES;   // STAGES x (B1 | B2 [| B3])
  uint64_t* bars = reinterpret_cast<uint64_t*>(sStage + C::STAGES * C::STAGE_BYTES);
  uint64_t* bar_fixed = bars;
  uint64_t* bar_stage_full = bars + 1;
  uint64_t* bar_stage_empty = bar_stage_full + C::STAGES;
  uint64_t* bar_s_full = bar_stage_empty + C::STAGES;  // [2], one per (S, dP) buffer
  uint64_t* bar_s_free = bar_s_full + 2;               // [2]
  uint64_t* bar_p_full = bar_s_free + 2;
  uint64_t* bar_pv_done = bar_p_full + 1;
  uint64_t* bar_acc_done = bar_pv_done + 1;
  uint64_t* bar_stats = bar_acc_done + 1;  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_stats + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // [2][BN] (LSE log2(e), D) of streamed rows (dK/dV instance); 16-byte aligned.
  float2* s_st = reinterpret_cast<float2*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WaitCtl ctl{abort_flag, w.wait_limit_ns, w.dev_status};
  const BwdRange rg = bwd_range<KV>(w);

  if (threadIdx.x == 0) {
    mbar_init(bar_fixed, 1);
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(bar_stage_full + i, 1);
      mbar_init(bar_stage_empty + i, KV ? 1 + 8 : 1);  // MMA commit (+ the 8 warps reading O)
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_s_full + i, 2);  // the S and the dP issuer
      mbar_init(bar_s_free + i, 8);  // one arrival per element-wise warp
    }
    mbar_init(bar_p_full, 8);
    mbar_init(bar_pv_done, 1);
    mbar_init(bar_acc_done, 3);  // one commit per issuer
    mbar_init(bar_stats + 0, 8);
    mbar_init(bar_stats + 1, 8);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    if (lane == 0) {
      tma_prefetch_map(&tm_a1);
      tma_prefetch_map(&tm_a2);
      tma_prefetch_map(&tm_b1);
      tma_prefetch_map(&tm_b2);
      if (KV) tma_prefetch_map(&tm_b3);
    }
    __syncwarp();
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The dK/dV launch follows the dQ launch as a programmatic dependent (the two read the same
  // inputs and write different outputs), so its CTAs may fill SMs the dQ grid leaves idle at its
  // end.  Every CTA waits for any such prerequisite grid before it exits (below), so neither
  // launch completes before the one ahead of it on the stream.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // Register split (warpgroup-wide): the control warpgroup (warps 8-11) shrinks, and the
  // element-wise warpgroups grow into what it released.
  if (warp >= 8) {
   bwd_setmaxnreg_dec<C::REG_CTL>();
   if (warp == 8) {
    if (lane == 0 && rg.n > 0) {
      // ================================================================ TMA producer
      mbar_arrive_expect_tx(bar_fixed, 2 * C::FIX_BYTES);
#pragma unroll
      for (int cb = 0; cb < C::NCB; ++cb) {
        tma_load_5d(sFix + cb * C::BLK_M, &tm_a1, bar_fixed, cb * C::CB, rg.m0, 0, rg.hf, rg.b);
        tma_load_5d(sFix + C::FIX_BYTES + cb * C::BLK_M, &tm_a2, bar_fixed, cb * C::CB, rg.m0, 0, rg.hf, rg.b);
      }
      int g = 0, t = rg.tb, j = 0;
      for (; j < rg.n; ++j) {
        const int st = j % C::STAGES;
        if (j >= C::STAGES && !mbar_wait(bar_stage_empty + st, ((j / C::STAGES) - 1) & 1, ctl, 0x701)) break;
        const int hs = KV ? rg.hf * w.qpk + g : rg.hf / w.qpk;  // streamed head
        uint8_t* dst = sStage + st * C::STAGE_BYTES;
        mbar_arrive_expect_tx(bar_stage_full + st, C::STAGE_BYTES);
#pragma unroll
        for (int cb = 0; cb < C::NCB; ++cb) {
          tma_load_5d(dst + cb * C::BLK_N, &tm_b1, bar_stage_full + st, cb * C::CB, t * C::BN, 0, hs, rg.b);
          tma_load_5d(dst + C::TILE_BYTES + cb * C::BLK_N, &tm_b2, bar_stage_full + st, cb * C::CB, t * C::BN, 0,
                      hs, rg.b);
          if (KV)
            tma_load_5d(dst + 2 * C::TILE_BYTES + cb * C::BLK_N, &tm_b3, bar_stage_full + st, cb * C::CB,
                        t * C::BN, 0, hs, rg.b);
        }
        if (++t == rg.te) {
          t = rg.tb;
          ++g;
        }
      }
      // No TMA write may still be in flight when the CTA exits.
      bwd_drain(bar_fixed, 0, w.wait_limit_ns);
      for (int i = (j > C::STAGES ? j - C::STAGES : 0); i < j; ++i)
        bwd_drain(bar_stage_full + i % C::STAGES, (i / C::STAGES) & 1, w.wait_limit_ns);
    }
   } else {
    if (lane == 0) {
      // ================================================================ MMA issuers
      // Three issuing threads (warp 9: S, warp 10: dP, warp 11: the gradient products): one
      // thread issues a tcgen05.mma about every 115 cycles whatever its size, far below the tensor
      // core's rate for these 128 x 64 x 16 and 128 x d x 16 shapes, so the MMA rate grows with
      // the number of issuing threads.
      constexpr uint32_t idesc_s = make_idesc_bf16(128, C::BN, 0, 0);
      constexpr uint32_t idesc_acc = make_idesc_bf16(128, DP, 0, 1);
      const uint64_t kmaj = make_smem_desc(0, 16, C::ATOM_BYTES, C::SWZ);
      const uint64_t mn = make_smem_desc(0, C::BLK_N, C::ATOM_BYTES, C::SWZ);
      const uint32_t a1 = smem_addr(sFix), a2 = a1 + C::FIX_BYTES;
      const uint32_t stage0 = smem_addr(sStage);
      // S, dP of tile jj into buffer jj % NSB, once its stage has landed and the element-wise
      // warps hold the buffer's previous tile in registers.
      auto issue_s = [&](int jj) -> bool {
        const int st = jj % C::STAGES, b = jj % C::NSB;
        if (!bwd_wait2(bar_stage_full + st, (jj / C::STAGES) & 1, jj >= C::NSB ? bar_s_free + b : nullptr,
                       ((jj / C::NSB) - 1) & 1, ctl, 0x712))
          return false;
        tc_fence_after();
        // S = A1 B1^T (warp 9) or dP = A2 B2^T (warp 10); s_full completes on both commits.
        const uint32_t bx = stage0 + st * C::STAGE_BYTES + (warp == 9 ? 0 : C::TILE_BYTES);
        const uint32_t ax = warp == 9 ? a1 : a2;
        const uint64_t da = kmaj | ((ax >> 4) & 0x3FFFu), dbx = kmaj | ((bx >> 4) & 0x3FFFu);
        const uint32_t col = tmem + b * C::SB_STRIDE + (warp == 9 ? C::S_COL : C::DP_COL);
#pragma unroll
        for (int kk = 0; kk < DP / 16; ++kk) {
          const int cb = (kk * 16) / C::CB;
          const uint32_t in = ((kk * 16) % C::CB) * 2;
          const uint32_t offa = (cb * C::BLK_M + in) >> 4, offb = (cb * C::BLK_N + in) >> 4;
          mma_ss(col, da + offa, dbx + offb, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_s_full + b);
        return true;
      };
      // ACC1 += dS B1 (and ACC2 += P B2) of tile jj, once its P and dS are in tensor memory; then
      // its stage and the P, dS columns are released.
      auto issue_acc = [&](int jj) -> bool {
        if (!mbar_wait(bar_p_full, jj & 1, ctl, 0x714)) return false;
        tc_fence_after();
        const int sp = jj % C::STAGES;
        const uint32_t b1 = stage0 + sp * C::STAGE_BYTES, b2 = b1 + C::TILE_BYTES;
        const uint64_t mb1 = mn | ((b1 >> 4) & 0x3FFFu), mb2 = mn | ((b2 >> 4) & 0x3FFFu);
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          const uint32_t off = (kk * 16 * C::ROW_BYTES) >> 4;
          const uint32_t acc = (jj > 0 || kk > 0) ? 1u : 0u;
          mma_ts(tmem + C::ACC_COL, tmem + C::DS_COL + kk * 8, mb1 + off, idesc_acc, acc);
          if (KV) mma_ts(tmem + C::ACC_COL + DP, tmem + C::P_COL + kk * 8, mb2 + off, idesc_acc, acc);
        }
        mma_commit(bar_pv_done);
        mma_commit(bar_stage_empty + sp);
        return true;
      };
      if (warp == 9 || warp == 10) {
        // S (dP) of every tile, each as soon as its stage has landed and the element-wise warps
        // hold the previous tile of its buffer in registers.
        bool ok = rg.n > 0 && mbar_wait(bar_fixed, 0, ctl, 0x711);
        for (int j = 0; ok && j < rg.n; ++j) ok = issue_s(j);
      } else {
        // The products of every tile, as soon as its P and dS are in tensor memory.
        bool ok = rg.n > 0;
        for (int j = 0; ok && j < rg.n; ++j) ok = issue_acc(j);
      }
      // The epilogue waits on acc_done: every MMA either issuer issued has completed (also after
      // an abort).
      if (rg.n > 0)
        mma_commit(bar_acc_done);
      else
        mbar_arrive(bar_acc_done);
      bwd_drain(bar_acc_done, 0, w.wait_limit_ns);
    }
   }
  } else {
    bwd_setmaxnreg_inc<C::REG_EW>();
    // ==================================================================== element-wise (warps 0-7)
    const int grp = warp >> 2;           // 0: columns 0-31, 1: columns 32-63
    const int row = (warp & 3) * 32 + lane;
    const int tid = threadIdx.x;         // 0..255
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int fixed_pos = rg.m0 + row;
    const long long win = w.causal ? w.window : 0;
    // Per-row statistics of the fixed rows (dQ instance): LSE log2(e) and D = dO . O.
    float row_l2 = INFINITY, row_d = 0.f;
    if (!KV && fixed_pos < w.n_q) {
      const float L = w.lse[(static_cast<long long>(rg.b) * w.H + rg.hf) * w.n_q + fixed_pos];
      row_l2 = (L == -INFINITY) ? INFINITY : L * 1.4426950408889634f;
      const uint4* po = reinterpret_cast<const uint4*>(w.o + rg.b * w.o_sb + rg.hf * w.o_sh + fixed_pos * w.o_st);
      const uint4* pd = reinterpret_cast<const uint4*>(w.d_o + rg.b * w.do_sb + rg.hf * w.do_sh + fixed_pos * w.do_st);
      float acc = 0.f;
      for (int c = 0; c < w.d / 8; ++c) {
        const uint4 a = po[c], bb = pd[c];
        const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* y = reinterpret_cast<const __nv_bfloat162*>(&bb);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 fx = __bfloat1622float2(x[e]), fy = __bfloat1622float2(y[e]);
          acc = fmaf(fx.x, fy.x, acc);
          acc = fmaf(fx.y, fy.y, acc);
        }
      }
      row_d = acc;
    }
    // Statistics of streamed query rows (dK/dV instance), one tile ahead of their use: D and
    // LSE log2(e) of tile jj's 64 rows go to buffer jj & 1 as interleaved pairs.  Four threads per
    // row, each a quarter of the row's 16-byte chunks of the staged O and dO tiles (both tiles
    // share one swizzled layout, so the same physical chunks pair the same elements); the row's
    // LSE is loaded one tile before it is needed.
    const int sc = tid >> 2, part = tid & 3;
    auto lse_of = [&](int gg, int tt) -> float {
      const int qi = tt * C::BN + sc;
      const int hq = rg.hf * w.qpk + gg;
      return qi < w.n_q ? w.lse[(static_cast<long long>(rg.b) * w.H + hq) * w.n_q + qi] : -INFINITY;
    };
    auto stats = [&](int jj, float L) -> bool {
      const int st = jj % C::STAGES;
      if (!bwd_wait(bar_stage_full + st, (jj / C::STAGES) & 1, ctl, 0x721)) return false;
      constexpr int NCH = DP / 32;    // chunks per thread
      constexpr int CPR = C::CB / 8;  // chunks per row of one column block
      const uint8_t* sdo = sStage + st * C::STAGE_BYTES + C::TILE_BYTES;
      const uint8_t* so = sdo + C::TILE_BYTES;
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
        const int k = part * NCH + i;
        const int off = (k / CPR) * C::BLK_N + sc * C::ROW_BYTES + (k % CPR) * 16;
        const uint4 a = *reinterpret_cast<const uint4*>(so + off);
        const uint4 bb = *reinterpret_cast<const uint4*>(sdo + off);
        const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* y = reinterpret_cast<const __nv_bfloat162*>(&bb);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 fx = __bfloat1622float2(x[e]), fy = __bfloat1622float2(y[e]);
          acc = fmaf(fx.x, fy.x, acc);
          acc = fmaf(fx.y, fy.y, acc);
        }
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      // Rows past the end (LSE -inf here) and empty rows get LSE log2(e) = +inf, so P = 0.
      if (part == 0) s_st[(jj & 1) * C::BN + sc] = make_float2(L == -INFINITY ? INFINITY : L * 1.4426950408889634f, acc);
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar_stage_empty + st);  // this warp is done with the stage's O tile
        mbar_arrive(bar_stats + (jj & 1));
      }
      return true;
    };
    bool ok = true;
    int g = 0, t = rg.tb;    // head and tile of tile j
    int gn = 0, tn = rg.tb;  // head and tile of the next tile whose statistics are due
    auto advance = [&](int& gg, int& tt) {
      if (++tt == rg.te) {
        tt = rg.tb;
        ++gg;
      }
    };
    if (KV && rg.n > 0) {
      ok = stats(0, part == 0 ? lse_of(0, rg.tb) : 0.f);
      advance(gn, tn);
    }
    for (int j = 0; ok && j < rg.n; ++j) {
      const int t0 = t * C::BN;  // first streamed row of the tile
      float lse_next = 0.f;
      if (KV && part == 0 && j + 1 < rg.n) lse_next = lse_of(gn, tn);
      // S and dP of this tile's 32 columns of the thread's row.
      const int sb = j % C::NSB;
      if (!(ok = bwd_wait(bar_s_full + sb, (j / C::NSB) & 1, ctl, 0x722))) break;
      tc_fence_after();
      uint32_t sv[32], pv[32];
      tmem_ld32(lane_addr + sb * C::SB_STRIDE + C::S_COL + 32 * grp, sv);
      tmem_ld32(lane_addr + sb * C::SB_STRIDE + C::DP_COL + 32 * grp, pv);
      tmem_ld_wait(sv);
      reg_pin32(pv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_s_free + sb);
      // Visible columns i (0..31 of this half) satisfy lo <= i < hi.
      const int base = t0 + 32 * grp;
      int lo = 0, hi = 32;
      bool masked;
      if (KV) {
        // fixed row = key at fixed_pos; column = query at base + i.
        masked = w.causal && (t0 < rg.m0 + C::BM - 1 || (win > 0 && t0 + C::BN - 1 - rg.m0 >= win));
        if (masked) {
          lo = fixed_pos - base;                                                  // query >= key
          if (win > 0) hi = static_cast<int>(min(32LL, fixed_pos - base + win));  // query < key + win
        }
      } else {
        // fixed row = query at fixed_pos; column = key at base + i.
        masked = (t0 + C::BN > w.n_kv) ||
                 (w.causal && (t0 + C::BN - 1 > rg.m0 || (win > 0 && rg.m0 + C::BM - 1 - t0 >= win)));
        if (masked) {
          hi = min(32, w.n_kv - base);
          if (w.causal) {
            hi = min(hi, fixed_pos - base + 1);                                        // key <= query
            if (win > 0) lo = static_cast<int>(max(0LL, fixed_pos - win + 1 - base));  // key > query - win
          }
        }
      }
      if (KV && !(ok = bwd_wait(bar_stats + (j & 1), (j >> 1) & 1, ctl, 0x723))) break;
      const float4* stv = reinterpret_cast<const float4*>(s_st + (j & 1) * C::BN + 32 * grp);
      uint32_t pp[16], dd[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        float4 cs = make_float4(row_l2, row_d, row_l2, row_d);  // (LSE log2(e), D) of columns i, i + 1
        if (KV) cs = stv[i / 2];
        float e0 = bwd_ex2(fmaf(__uint_as_float(sv[i]), w.scale_log2, -cs.x));
        float e1 = bwd_ex2(fmaf(__uint_as_float(sv[i + 1]), w.scale_log2, -cs.z));
        if (masked) {
          if (i < lo || i >= hi) e0 = 0.f;
          if (i + 1 < lo || i + 1 >= hi) e1 = 0.f;
        }
        pp[i / 2] = bf16x2_bits(e0, e1);
        dd[i / 2] = bf16x2_bits(e0 * (__uint_as_float(pv[i]) - cs.y), e1 * (__uint_as_float(pv[i + 1]) - cs.w));
      }
      if (j > 0 && !(ok = bwd_wait(bar_pv_done, (j - 1) & 1, ctl, 0x724))) break;
      tc_fence_after();
      if (KV) tmem_st16(lane_addr + C::P_COL + 16 * grp, pp);
      tmem_st16(lane_addr + C::DS_COL + 16 * grp, dd);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p_full);
      advance(g, t);
      if (KV && j + 1 < rg.n) {
        if (!(ok = stats(j + 1, lse_next))) break;
        advance(gn, tn);
      }
    }
    // ================================================================== epilogue
    const bool have = ok && rg.n > 0 && bwd_wait(bar_acc_done, 0, ctl, 0x725);
    if (rg.n == 0 || have) {
      tc_fence_after();
      const int n_rows = KV ? w.n_kv : w.n_q;
      const bool row_ok = fixed_pos < n_rows;
      constexpr int CH = DP / 32;  // 32-column chunks per accumulator
#pragma unroll 1
      for (int q = grp; q < C::NACC * CH; q += 2) {
        const int a = q / CH, ch = q % CH;
        uint32_t v[32];
        if (rg.n > 0) {
          tmem_ld32(lane_addr + C::ACC_COL + a * DP + ch * 32, v);
          tmem_ld_wait(v);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0u;
        }
        if (!row_ok) continue;
        const float f = (a == 0) ? w.scale : 1.f;
        float* dst = (a == 0) ? w.out1 + rg.b * w.o1_sb + rg.hf * w.o1_sh + fixed_pos * w.o1_st
                              : w.out2 + rg.b * w.o2_sb + rg.hf * w.o2_sh + fixed_pos * w.o2_st;
        const int c0 = ch * 32;
        const int nc = min(32, w.d - c0);
        if (nc == 32 && (reinterpret_cast<uintptr_t>(dst + c0) & 15) == 0) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + c0 + i) =
                make_float4(f * __uint_as_float(v[i]), f * __uint_as_float(v[i + 1]),
                            f * __uint_as_float(v[i + 2]), f * __uint_as_float(v[i + 3]));
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < nc) dst[c0 + i] = f * __uint_as_float(v[i]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace ra
