// ra_fmha_sm100.cuh - fused blockwise attention forward on the sm_100a tensor cores.
//
// What it computes: the online softmax of intelliparadigm.com "深度学习注意力机制优化与
// FlashAttention实践" §4.2 (with the output rescaled when the running max moves, which the
// printed listing omits): K/V tiles stream through shared memory, S = Q K^T and O += P V run as
// tcgen05 MMAs with fp32 accumulators in tensor memory, and a per-row running max m and sum s
// are kept in fp32 registers.  One launch may walk several KV shards of a ring in ring order
// (query shard r meets KV shard (r - t) mod P at step t, vibe-research.pages.dev "Ring
// Attention" diagram); a shard boundary needs no extra work because the running (m, s, O)
// already is the merged state of every shard seen so far (blog.gitcode.com "分布式注意力机制突破…"
// §3.4: align the maxima, rescale the sums).
//
// Structure (persistent: one CTA per SM walks work items; an item is 256 query rows = two
// 128-row query tiles of one (batch, head, query shard); items are numbered longest first and
// dealt to the CTAs in a snake order):
//   warps 0-3   softmax of query tile 0, thread i = row i = tensor-memory lane i
//   warps 4-7   softmax of query tile 1
//   warps 8-11  epilogue: normalise O, write O / LSE or LSE-merge into the accumulator
//   warp 12     TMA producer: Q (two tiles) per item, then K_j / V_j into a STAGES-deep ring; it
//               also publishes each item's decoded plan (ItemPlan) to the other roles
//   warps 13,14 MMA issuers, one thread per query tile: S_q = Q_q K_j^T (SS form), O_q += P_q V_j
//               (TS form, P from tensor memory)
// Both query tiles share every K/V tile (loaded once per 256 rows).  K/V tiles are 128 keys for
// DP <= 64 and 64 keys for DP = 128, so that P always has its own tensor-memory columns: the
// next QK_q starts as soon as the softmax holds S_q in registers, overlapping this tile's
// softmax.  Tensor memory (512 columns): S_0, S_1 (BN fp32 columns each), P_0, P_1 (BN/2 columns
// of bf16 pairs each), O_0, O_1 (DP columns each).  (With FmhaCfg's RA_D128_BN64 = 0, DP = 128
// uses 128-key tiles with P written over S and one issuer in the fixed order PV_0(j), QK_0(j+1),
// PV_1(j), QK_1(j+1); both layouts measure within 2 %.)
// Registers are rebalanced with setmaxnreg (RegSplit) per instance, without spills in every
// instance without a sliding window.
// Hand-offs: an issuer polls every barrier an MMA group needs in one loop, the softmax tests its
// next barriers while its exponentials run (at DP = 128 the two softmax warpgroups take turns at
// the exponential loop), and work-item index arithmetic uses launch-time multiply-shift dividers
// (an integer divide would queue behind the exponentials on the MUFU).  The softmax arithmetic
// uses packed fp32x2 instructions and three-input max.  A polynomial exp2 on the FMA pipe
// (exp2_poly3) can take 1 in kEmuEvery column pairs of unmasked tiles; it is off by default
// (measured slower).  A column-split softmax (RA_SOFTMAX_SPLIT) is off by default (measured
// slower).
// Programmatic dependent launch: each CTA signals dependents once set up; the epilogue waits for
// any prerequisite grid before it touches memory (the next ring step's accumulator).
// Every wait is bounded; on a timeout all roles stop, tensor memory is freed and the kernel
// returns with the device status word set.
#pragma once

#include "ra_common.cuh"

namespace ra {

#ifndef RA_D128_BN64
#define RA_D128_BN64 1
#endif
#ifndef RA_SOFTMAX_SPLIT
#define RA_SOFTMAX_SPLIT 0
#endif

template <int DP>
struct FmhaCfg {
  static_assert(DP == 32 || DP == 64 || DP == 128, "padded head dim must be 32, 64 or 128");
  static constexpr int BM = 128;    // rows of one query tile
  // Keys of one K/V tile.  At DP = 128 the two O accumulators take half of tensor memory, so
  // 64-key tiles are what leaves room for S and P in separate columns (see P_SEP).
  static constexpr int BN = (DP == 128 && RA_D128_BN64) ? 64 : 128;
  static constexpr int ROWS = 256;  // query rows of one work item (two tiles)
  static constexpr int CB = (DP == 32) ? 32 : 64;  // columns per TMA box / swizzle span
  static constexpr int NCB = DP / CB;
  static constexpr int ROW_BYTES = CB * 2;
  static constexpr uint32_t SWZ = (DP == 32) ? kSwizzle64B : kSwizzle128B;
  static constexpr int ATOM_BYTES = 8 * ROW_BYTES;
  static constexpr int Q_BLOCK_BYTES = BM * ROW_BYTES;   // one CB-column block of a Q tile
  static constexpr int KV_BLOCK_BYTES = BN * ROW_BYTES;  // one CB-column block of a K or V tile
  static constexpr int Q_TILE_BYTES = BM * DP * 2;
  static constexpr int KV_TILE_BYTES = BN * DP * 2;
  static constexpr int STAGES = (DP == 128) ? (BN == 64 ? 4 : 2) : (DP == 64 ? 5 : 8);
  // P in its own tensor-memory columns, so S_q may be overwritten as soon as the softmax holds it
  // in registers: one MMA issuer per query tile.  P over S (DP = 128 with 128-key tiles): one
  // issuer in a fixed PV_0, QK_0, PV_1, QK_1 order, which staggers the two tiles.
  static constexpr bool P_SEP = DP <= 64 || BN == 64;
  static constexpr int ISSUERS = P_SEP ? 2 : 1;
  static constexpr int S_COL0 = 0;
  static constexpr int S_STRIDE = BN;
  static constexpr int O_COL0 = 256;
  static constexpr int O_STRIDE = (DP == 128) ? 128 : 64;
  static constexpr int P_COL0 = P_SEP ? (DP == 128 ? 2 * BN : 384) : 0;
  static constexpr int P_STRIDE = P_SEP ? BN / 2 : 128;
  static_assert(!P_SEP || P_COL0 + 2 * P_STRIDE <= (DP == 128 ? O_COL0 : 512), "tensor memory columns overlap");
  static constexpr int NSC = BN / 32;  // 32-column chunks of one S row
  // Column-split softmax: two warpgroups per query tile, each taking half of every S row (and
  // half of the O columns in rescales and the epilogue), so four softmax warps share each SM
  // sub-partition instead of two and hide one another's barrier / tensor-memory latencies.  The
  // halves exchange row maxima per tile and row sums per item through shared memory.  The
  // epilogue runs in the softmax warps (no registers are left for a separate warpgroup).
  static constexpr bool SPLIT = RA_SOFTMAX_SPLIT != 0 && P_SEP;
  static constexpr int HCOLS = SPLIT ? BN / 2 : BN;  // S columns per softmax thread
  static constexpr int SM_WARPS = SPLIT ? 16 : 8;     // softmax warps
  static constexpr int PROD_WARP = SPLIT ? 16 : 12;   // TMA producer; MMA issuers follow it
  static constexpr int SMEM_TILES = 2 * Q_TILE_BYTES + 2 * STAGES * KV_TILE_BYTES;
  static constexpr int NBAR = 3 + 3 * STAGES + 11 * 2;
  static constexpr int STATS_BYTES = 2 * 128 * 8;
  static constexpr int PLAN_BYTES = 2 * 64;
  static constexpr int XCH_BYTES = SPLIT ? 2 * (2 * 2 * 2 * 128 * 4) : 0;  // row max and row sum exchange
  static constexpr int SMEM_BYTES = 1024 + SMEM_TILES + NBAR * 8 + 16 + STATS_BYTES + PLAN_BYTES + XCH_BYTES;
  static constexpr int THREADS = SPLIT ? 640 : 512;
  static constexpr int D = DP;
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

// Per-thread register budgets after setmaxnreg (softmax, epilogue, producer/MMA warpgroups).  The
// merging epilogues (accumulate modes) need more registers than the plain output one.
template <int DP, int EPI>
struct RegSplit {
  static constexpr bool kSplit = FmhaCfg<DP>::SPLIT;
  static constexpr bool kAcc = (EPI == 2 || EPI == 3);
  // Registers per thread at launch: 65536 / threads rounded down to a multiple of 8 (the host
  // checks the compiled kernel's count against this before launching).
  static constexpr int kLaunch = (65536 / FmhaCfg<DP>::THREADS) / 8 * 8;
  // Producer / MMA-issuer warpgroup: 64 registers leave the softmax of the d = 64 instances and of
  // the merging d = 32 instances enough to compile without spills; the d = 32 output and partial
  // instances measured 10 % faster with 80 (and do not spill with it), and at d = 128 (64-key
  // tiles) the softmax needs fewer registers, so 80 there too.
  static constexpr int kProd = kSplit ? 64 : ((DP == 64 || (DP == 32 && kAcc)) ? 64 : 80);
  static constexpr int kEpi = kSplit ? 0 : (kAcc ? 80 : (DP <= 64 ? 48 : 64));
  static constexpr int kSoftmaxWGs = kSplit ? 4 : 2;
  static constexpr int kSoftmax =
      ((kLaunch * FmhaCfg<DP>::THREADS / 128 - kProd - kEpi) / kSoftmaxWGs) / 8 * 8;
  // Every warpgroup's share, added up, must fit in what the block was launched with, or a
  // setmaxnreg.inc would wait forever.
  static_assert(kSoftmaxWGs * 128 * kSoftmax + 128 * kEpi + 128 * kProd <= kLaunch * FmhaCfg<DP>::THREADS,
                "register split exceeds the launch");
  static constexpr int kTotal = kSoftmaxWGs * 128 * kSoftmax + 128 * kEpi + 128 * kProd;
};

#ifndef RA_EMU_EVERY
#define RA_EMU_EVERY 0
#endif
constexpr int kEmuEvery = RA_EMU_EVERY;  // 1 in kEmuEvery column pairs of unmasked tiles use the FMA-pipe exp2

#ifndef RA_EXP_ALTERNATE
#define RA_EXP_ALTERNATE 1
#endif
// The two softmax warpgroups take turns at their exponential loops (see the softmax role).  With
// 64-key tiles (DP = 128) one warpgroup's exponentials take less time than its per-tile hand-offs,
// so the turns hide them (measured +2-4 %); with 128-key tiles (DP <= 64) they lose 10-15 %.
template <int DP>
struct AlternateExps {
  static constexpr bool value = RA_EXP_ALTERNATE != 0 && FmhaCfg<DP>::BN == 64;
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipe: x = n + f with n = round(x) (added to the exponent field), f in
// [-1/2, 1/2], and 2^f from a degree-3 polynomial fitted minimax in relative error by the Remez
// exchange algorithm (max relative error 7.5e-5; coefficients from csrc/gen_exp2_poly.py).
// Inputs below -126 are clamped, so the result is never exactly zero: callers use it only where
// no score is masked.
__device__ __forceinline__ float exp2_poly3(float x) {
  x = fmaxf(x, -126.f);
  const float t = x + 12582912.f;  // 1.5 * 2^23: round(x) lands in the low mantissa bits of t
  const float n = t - 12582912.f;
  const float f = x - n;
  float p = fmaf(0.0551716685295105f, f, 0.2426111251115799f);
  p = fmaf(p, f, 0.6932609677314758f);
  p = fmaf(p, f, 0.9999280571937561f);
  // (bits(t) << 23) == n << 23 (mod 2^32): the constant part of bits(t) shifts out.
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// Two lanes of exp2_poly3 with packed fp32x2 arithmetic (same polynomial and range reduction).
__device__ __forceinline__ float2 exp2_poly3_x2(float2 x) {
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 magic = make_float2(12582912.f, 12582912.f);
  const float2 t = __fadd2_rn(x, magic);
  const float2 n = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));  // round(x), exact
  const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);                // x - round(x), exact
  float2 p = __ffma2_rn(make_float2(0.0551716685295105f, 0.0551716685295105f), f,
                        make_float2(0.2426111251115799f, 0.2426111251115799f));
  p = __ffma2_rn(p, f, make_float2(0.6932609677314758f, 0.6932609677314758f));
  p = __ffma2_rn(p, f, make_float2(0.9999280571937561f, 0.9999280571937561f));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
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

// Bounded wait that ignores the abort flag (used to drain in-flight copies / MMAs before exit).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) break;
  }
}

#ifndef RA_ISSUER_SPIN
#define RA_ISSUER_SPIN 1
#endif
#ifndef RA_ISSUER_BACKOFF_NS
#define RA_ISSUER_BACKOFF_NS 0
#endif
// Wait used by the single-thread MMA issuers: spin on the non-blocking test (a sleeping try_wait
// wakes up late, and each issuer hop sits on the critical path of a query tile), bounded like
// mbar_wait.
__device__ __forceinline__ bool mbar_wait_issuer(uint64_t* bar, uint32_t parity, const WaitCtl& ctl, unsigned site) {
  if (!RA_ISSUER_SPIN) return mbar_wait(bar, parity, ctl, site);
  if (mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 256; ++i) {
      if (mbar_test_wait(bar, parity)) return true;
      if (RA_ISSUER_BACKOFF_NS > 0) __nanosleep(RA_ISSUER_BACKOFF_NS);
    }
    if (*ctl.abort) return false;
    if (globaltimer_ns() - t0 > ctl.limit_ns) {
      atomicOr(ctl.status, kDevStatusTimeout);
      atomicCAS(ctl.status + 1, 0u, site);
      *ctl.abort = 1;
      __threadfence_block();
      return false;
    }
  }
}

// Wait used by the MMA issuers for everything one MMA group needs: up to three (barrier, parity)
// pairs (nullptr = none).  Each poll tests every pair not yet seen complete back to back, so the
// latencies of the tests (a few hundred cycles even on a completed phase) overlap instead of
// adding up.  Bounded like mbar_wait.
__device__ __forceinline__ bool mbar_wait_all_issuer(uint64_t* b0, uint32_t p0, uint64_t* b1, uint32_t p1, uint64_t* b2,
                                                     uint32_t p2, const WaitCtl& ctl, unsigned site) {
  if (!RA_ISSUER_SPIN)
    return (b0 == nullptr || mbar_wait(b0, p0, ctl, site)) && (b1 == nullptr || mbar_wait(b1, p1, ctl, site)) &&
           (b2 == nullptr || mbar_wait(b2, p2, ctl, site));
  bool d0 = b0 == nullptr, d1 = b1 == nullptr, d2 = b2 == nullptr;
  auto poll = [&]() -> bool {
    const bool t0 = d0 || mbar_test_wait(b0, p0);
    const bool t1 = d1 || mbar_test_wait(b1, p1);
    const bool t2 = d2 || mbar_test_wait(b2, p2);
    d0 = t0;
    d1 = t1;
    d2 = t2;
    if (RA_ISSUER_BACKOFF_NS > 0 && !(t0 && t1 && t2)) __nanosleep(RA_ISSUER_BACKOFF_NS);
    return t0 && t1 && t2;
  };
  if (poll()) return true;
  const uint64_t start = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 256; ++i)
      if (poll()) return true;
    if (*ctl.abort) return false;
    if (globaltimer_ns() - start > ctl.limit_ns) {
      atomicOr(ctl.status, kDevStatusTimeout);
      atomicCAS(ctl.status + 1, 0u, site);
      *ctl.abort = 1;
      __threadfence_block();
      return false;
    }
  }
}

template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ---------------------------------------------------------------------------------------------
// Work items and the walk over KV tiles
// ---------------------------------------------------------------------------------------------
// Items are numbered longest first; CTA c takes item c in its first sweep, G-1-c in its second,
// G+c in its third, ... (a snake over the G persistent CTAs), which pairs long with short items.
__device__ __forceinline__ int item_of_cta(int k) {
  const int G = static_cast<int>(gridDim.x);
  const int c = static_cast<int>(blockIdx.x);
  return k * G + ((k & 1) ? (G - 1 - c) : c);
}

struct Item {
  int b, h, r, t0;
  int hk;  // K/V head of query head h
  int rows_valid[2];
  long long pos0;       // global position of local query token 0 of shard r
  long long pos_last;   // position of the item's last valid query row
  long long pos_first;  // position of the item's first query row
};

// A work item as the TMA producer publishes it to the other roles (decoded once per CTA).  Used
// with P in its own tensor-memory columns (d <= 64), where item set-up sat on the critical path of
// short causal items; the d = 128 roles decode items themselves (measured faster there).
struct ItemPlan {
  Item it;
  int n;  // K/V tiles the item walks
  int pad;
};
static_assert(sizeof(ItemPlan) == 64, "plan slot size");

// Items come in head groups of w.hgroup (batch, head) pairs, so the K/V the concurrently running
// CTAs read stays in L2; inside a group the order is longest first with heads innermost.
__device__ __forceinline__ void decode_item(const AttnWork& w, int idx, Item& it) {
  // Index arithmetic with launch-time fast dividers only (no divide instructions).
  const int n_blk = (w.n_q + 255) >> 8;
  const int bh_count = w.B * w.H;
  const int per_head = n_blk * w.n_r;
  const int hg = w.hgroup;
  const int grp = fdiv(idx, w.fd_grp);  // items per group = hg * per_head
  const int local = idx - grp * hg * per_head;
  const bool last_grp = bh_count - grp * hg < hg;
  const FastDiv& fh = last_grp ? w.fd_hg_last : w.fd_hg;
  const int rest = fdiv(local, fh);
  const int bh = grp * hg + (local - rest * static_cast<int>(fh.d));
  int ri, blk;
  if (w.r_major) {  // positions grow with the shard first (contiguous shards): longest first
    const int a = fdiv(rest, w.fd_nblk);
    ri = w.n_r - 1 - a;
    blk = n_blk - 1 - (rest - a * n_blk);
  } else {
    const int a = fdiv(rest, w.fd_nr);
    blk = n_blk - 1 - a;
    ri = w.n_r - 1 - (rest - a * w.n_r);
  }
  it.b = fdiv(bh, w.fd_H);
  it.h = bh - it.b * w.H;
  it.hk = fdiv(it.h, w.fd_qpk);
  it.r = w.r_first + ri * w.r_step;
  it.t0 = blk * 256;
  it.rows_valid[0] = max(0, min(128, w.n_q - it.t0));
  it.rows_valid[1] = max(0, min(128, w.n_q - it.t0 - 128));
  it.pos0 = w.q_off + static_cast<long long>(it.r) * w.q_rstep;
  const int last = it.t0 + it.rows_valid[0] + it.rows_valid[1] - 1;
  it.pos_last = it.pos0 + static_cast<long long>(last) * w.q_tstride;
  it.pos_first = it.pos0 + static_cast<long long>(it.t0) * w.q_tstride;
}

// Striped shards (shard s holds the keys at positions u * P + s): for a position D = a * P + b
// (0 <= b < P), the keys of shard s at or before D are u <= a - (s > b), and the keys at or after
// D are u >= a + (b > s).  Launches with a tile-major walk have exactly this geometry, so their
// per-tile bounds need no division.
struct StripedPos {
  int a, b;  // b = -1: a position before the first key (every key is at or after it)
};
__device__ __forceinline__ StripedPos striped_pos(const AttnWork& w, long long pos) {
  if (pos < 0) return {0, -1};
  const int a = pos < 0x7fffffffLL ? fdiv(static_cast<int>(pos), w.fd_P) : static_cast<int>(pos / w.P);
  return {a, static_cast<int>(pos - static_cast<long long>(a) * w.P)};
}
// visible_key_limit for a query at p (causal bound; all keys otherwise).
__device__ __forceinline__ int striped_lim(const AttnWork& w, StripedPos p, int s) {
  if (!w.causal) return w.n_kv;
  return min(w.n_kv, p.a + 1 - (s > p.b ? 1 : 0));
}
// visible_key_start for a window whose first position is p.
__device__ __forceinline__ int striped_start(const AttnWork& w, StripedPos p, int s) {
  return min(w.n_kv, p.a + (p.b > s ? 1 : 0));
}

struct Walk {
  int step;  // ring step offset within this launch
  int s;     // KV shard
  int u0;    // first key of the current tile
  int lim;   // keys of shard s visible to the item's last row
  // Tile-major walk: the largest lim over the launch's shards, the shard of step 0, and the
  // item's last position and first window position.
  int umax, s0;
  StripedPos last, first;
};

// Keys [start, lim) of shard s are visible to some row of the item: lim from its last row (the
// causal bound), start from its first row (the sliding-window bound; 0 without a window).  The
// walk covers the 128-key tiles that meet that range.  WIN: the launch has a sliding window
// (compiled separately so that the plain path carries none of its arithmetic).
template <bool WIN, int BN>
__device__ __forceinline__ bool walk_seek(Walk& k, const AttnWork& w, const Item& it, int n_steps) {
  for (; k.step < n_steps; ++k.step) {
    const int s = ring_shard(w, it.r, w.ring_step + k.step);
    const int lim = visible_key_limit(w, it.pos_last, s);
    const int start = WIN ? visible_key_start(w, it.pos_first, s) : 0;
    if (lim > start) {
      k.s = s;
      k.lim = lim;
      k.u0 = start & ~(BN - 1);
      return true;
    }
  }
  return false;
}

// The tile-major walk is compiled into the 64-key-tile (d = 128) kernels only: the 128-key-tile
// kernels keep their registers for the softmax (their ring workloads use contiguous shards).
template <int BN>
constexpr bool kTileWalk = BN == 64;

// Tile-major order (w.tile_major, striped shards): tile u0 of every shard that has it, then tile
// u0 + BN, ...  Striped shards interleave their keys in memory, so this order reads each stretch
// of K/V once per item instead of once per shard.  Same tiles as the shard-major walk.
template <bool WIN, int BN>
__device__ __forceinline__ bool walk_seek_tiles(Walk& k, const AttnWork& w, const Item& it, int n_steps) {
  while (k.u0 < k.umax) {
    for (; k.step < n_steps; ++k.step) {
      int s = k.s0 - k.step;
      while (s < 0) s += w.P;
      const int lim = striped_lim(w, k.last, s);
      const int start = WIN ? striped_start(w, k.first, s) : 0;
      if (lim > start && k.u0 < lim && k.u0 + BN > start) {
        k.s = s;
        k.lim = lim;
        return true;
      }
    }
    k.step = 0;
    k.u0 += BN;
  }
  return false;
}

template <bool WIN, int BN>
__device__ __forceinline__ bool walk_begin(Walk& k, const AttnWork& w, const Item& it, int n_steps) {
  k.step = 0;
  if (kTileWalk<BN> && w.tile_major) {
    k.s0 = ring_shard(w, it.r, w.ring_step);
    k.last = striped_pos(w, it.pos_last);
    k.first = (WIN && w.window > 0) ? striped_pos(w, it.pos_first - w.window + 1) : StripedPos{0, -1};
    int umax = 0, ulo = 0x7fffffff;
    for (int step = 0; step < n_steps; ++step) {
      int s = k.s0 - step;
      while (s < 0) s += w.P;
      const int lim = striped_lim(w, k.last, s);
      const int start = WIN ? striped_start(w, k.first, s) : 0;
      if (lim > start) {
        umax = max(umax, lim);
        ulo = min(ulo, start & ~(BN - 1));
      }
    }
    k.umax = umax;
    k.u0 = umax > 0 ? ulo : 0;
    return walk_seek_tiles<WIN, BN>(k, w, it, n_steps);
  }
  return walk_seek<WIN, BN>(k, w, it, n_steps);
}

template <bool WIN, int BN>
__device__ __forceinline__ bool walk_next(Walk& k, const AttnWork& w, const Item& it, int n_steps) {
  if (kTileWalk<BN> && w.tile_major) {
    ++k.step;
    return walk_seek_tiles<WIN, BN>(k, w, it, n_steps);
  }
  k.u0 += BN;
  if (k.u0 < k.lim) return true;
  ++k.step;
  return walk_seek<WIN, BN>(k, w, it, n_steps);
}


// Number of K/V tiles the item walks (what the MMA issuer needs; it never reads the keys).
template <bool WIN, int BN>
__device__ __forceinline__ int walk_count(const AttnWork& w, const Item& it, int n_steps) {
  int n = 0;
  for (int step = 0; step < n_steps; ++step) {
    const int s = ring_shard(w, it.r, w.ring_step + step);
    const int lim = visible_key_limit(w, it.pos_last, s);
    const int start = WIN ? visible_key_start(w, it.pos_first, s) : 0;
    if (lim > start) n += (lim + BN - 1) / BN - start / BN;
  }
  return n;
}

// ---------------------------------------------------------------------------------------------
// MMA issue (single thread) and the per-row epilogue
// ---------------------------------------------------------------------------------------------
// Shared-memory descriptors differ only in their start-address field (bits 0-13, address >> 4),
// so each MMA adds a small offset to a base descriptor built once.
template <class C>
struct DescBase {
  uint64_t kmaj;  // K-major operand (Q, K): leading 16 B, stride = one 8-row swizzle atom
  uint64_t vmn;   // MN-major V: leading = next 64-column block, stride = one 8-row swizzle atom
  __device__ __forceinline__ DescBase() {
    kmaj = make_smem_desc(0, 16, C::ATOM_BYTES, C::SWZ);
    vmn = make_smem_desc(0, C::KV_BLOCK_BYTES, C::ATOM_BYTES, C::SWZ);
  }
};

__device__ __forceinline__ uint64_t desc_at(uint64_t base, uint32_t saddr) {
  return base | static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
}

// S[tmem d_s] = Q (K-major, swizzled, at q_addr) * K^T (K-major at k_addr), K = D in steps of 16.
template <class C>
__device__ __forceinline__ void fmha_issue_qk(const DescBase<C>& db, uint32_t d_s, uint32_t q_addr, uint32_t k_addr,
                                              uint32_t idesc) {
  const uint64_t a0 = desc_at(db.kmaj, q_addr);
  const uint64_t b0 = desc_at(db.kmaj, k_addr);
#pragma unroll
  for (int kk = 0; kk < C::D / 16; ++kk) {
    const int cb = (kk * 16) / C::CB;
    const uint32_t off_a = (cb * C::Q_BLOCK_BYTES + ((kk * 16) % C::CB) * 2) >> 4;  // compile-time
    const uint32_t off_b = (cb * C::KV_BLOCK_BYTES + ((kk * 16) % C::CB) * 2) >> 4;
    mma_ss(d_s, a0 + off_a, b0 + off_b, idesc, kk > 0 ? 1u : 0u);
  }
}

// O[tmem d_o] (+)= P (bf16 pairs in tensor memory at p_tmem) * V (MN-major at v_addr): 16 keys
// per MMA; the next 64-column block of V sits one KV_BLOCK_BYTES further (leading byte offset).
template <class C>
__device__ __forceinline__ void fmha_issue_pv(const DescBase<C>& db, uint32_t d_o, uint32_t p_tmem, uint32_t v_addr,
                                              uint32_t idesc, bool accumulate) {
  const uint64_t b0 = desc_at(db.vmn, v_addr);
#pragma unroll
  for (int kk = 0; kk < C::BN / 16; ++kk) {
    const uint32_t off = (kk * 16 * C::ROW_BYTES) >> 4;  // compile-time
    mma_ts(d_o, p_tmem + kk * 8, b0 + off, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// One query row: O = O_acc / l and LSE = m ln 2 + ln l (natural log; sum_j e^{scale q.k_j} =
// 2^m * l), then by mode: write (O bf16, LSE), write the fp32 partial, or LSE-merge it into the
// fp32 accumulator (gitcode page §2.2 phase 3).  Warp-collective (tensor-memory loads).
template <class C, int EPI>
__device__ __forceinline__ void fmha_epilogue_row(const AttnWork& w, const Item& it, int t, bool row_ok,
                                                  bool has_o, float2 ml, uint32_t o_addr) {
  const bool has = ml.y > 0.f;
  const float inv_l = has ? 1.f / ml.y : 0.f;
  const float lse_part = has ? (ml.x * 0.69314718055994531f + logf(ml.y)) : -INFINITY;
  const bool skip = (EPI == kEpiAcc) && !has;  // merging an empty partial is the identity
  float L = lse_part, w_part = 1.f, w_acc = 0.f;
  float* acc_row = nullptr;
  float* accl_ptr = nullptr;
  if (EPI != kEpiOut) {
    acc_row = w.acc_o + it.b * w.a_sb + it.h * w.a_sh + it.r * w.a_rs + static_cast<long long>(t) * w.a_ts;
    accl_ptr = w.acc_l + it.b * w.al_sb + it.h * w.al_sh + it.r * w.al_rs + static_cast<long long>(t) * w.al_ts;
  }
  if ((EPI == kEpiAcc || EPI == kEpiAccOut) && row_ok && !skip) {
    const float la = *accl_ptr;
    lse_merge_weights(la, lse_part, L, w_acc, w_part);
  }
  __nv_bfloat16* out_row = nullptr;
  if (EPI == kEpiOut || EPI == kEpiAccOut)
    out_row = static_cast<__nv_bfloat16*>(w.o) + it.b * w.o_sb + it.h * w.o_sh + it.r * w.o_rs +
              static_cast<long long>(t) * w.o_ts;
  const float wp = w_part * inv_l;
#pragma unroll
  for (int cc = 0; cc < C::D / 32; ++cc) {
    uint32_t orow[32];
    if (has_o) {
      tmem_ld32(o_addr + cc * 32, orow);
      tmem_ld_wait(orow);
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) orow[e] = 0u;
    }
    if (row_ok && !skip) {
      float vals[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) vals[e] = __uint_as_float(orow[e]) * wp;
      if (EPI == kEpiAcc || EPI == kEpiAccOut) {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          if (cc * 32 + e < w.d) {
            const float4 a = *reinterpret_cast<const float4*>(acc_row + cc * 32 + e);
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
          if (cc * 32 + e < w.d)
            *reinterpret_cast<float4*>(acc_row + cc * 32 + e) = make_float4(vals[e], vals[e + 1], vals[e + 2], vals[e + 3]);
      } else {
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          if (cc * 32 + e < w.d) {
            uint4 pkt;
            pkt.x = pack_bf16x2(vals[e], vals[e + 1]);
            pkt.y = pack_bf16x2(vals[e + 2], vals[e + 3]);
            pkt.z = pack_bf16x2(vals[e + 4], vals[e + 5]);
            pkt.w = pack_bf16x2(vals[e + 6], vals[e + 7]);
            *reinterpret_cast<uint4*>(out_row + cc * 32 + e) = pkt;
          }
        }
      }
    }
  }
  if (row_ok && !skip) {
    if (EPI == kEpiPart || EPI == kEpiAcc) {
      *accl_ptr = L;
    } else if (w.lse != nullptr) {
      w.lse[it.b * w.l_sb + it.h * w.l_sh + it.r * w.l_rs + static_cast<long long>(t) * w.l_ts] = L;
    }
  }
}

#ifndef RA_SPLIT_WARP_ARRIVE
#define RA_SPLIT_WARP_ARRIVE 0
#endif
// Column-split softmax: arrivals on the per-tile barriers (S consumed, P written) one per warp
// instead of one per thread.
constexpr bool kSplitWarpArrive = RA_SPLIT_WARP_ARRIVE != 0;

// The 8 warps of one query tile's two column-split softmax warpgroups meet on `bar` (an mbarrier
// counting one arrival per warp, after the warp's own lanes have synchronised; n counts this
// thread's meetings so far).  Bounded like every wait: returns false if it ran out or the CTA is
// aborting.
__device__ __forceinline__ bool pair_meet(uint64_t* bar, int& n, const WaitCtl& ctl) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  const bool ok = mbar_wait(bar, static_cast<uint32_t>(n) & 1, ctl, 0x307);
  ++n;
  return ok;
}

// fmha_epilogue_row for the column-split softmax: this thread's half of the row, O columns
// [half * D/2, (half + 1) * D/2).  Both halves hold the same (m, l); half 0 writes the LSE.  In
// the in-place accumulate mode the pair meets between reading the stored LSE and overwriting it.
template <class C, int EPI>
__device__ __forceinline__ void fmha_epilogue_row_half(const AttnWork& w, const Item& it, int t, bool row_ok,
                                                       bool has_o, float2 ml, uint32_t o_addr, int half,
                                                       uint64_t* pair_bar, int& pair_n, const WaitCtl& ctl) {
  constexpr int HD = C::D / 2;           // O columns of this half
  constexpr int CH = HD < 32 ? HD : 32;  // columns per tensor-memory load
  const bool has = ml.y > 0.f;
  const float inv_l = has ? 1.f / ml.y : 0.f;
  const float lse_part = has ? (ml.x * 0.69314718055994531f + logf(ml.y)) : -INFINITY;
  const bool skip = (EPI == kEpiAcc) && !has;  // merging an empty partial is the identity
  float L = lse_part, w_part = 1.f, w_acc = 0.f;
  float* acc_row = nullptr;
  float* accl_ptr = nullptr;
  if (EPI != kEpiOut) {
    acc_row = w.acc_o + it.b * w.a_sb + it.h * w.a_sh + it.r * w.a_rs + static_cast<long long>(t) * w.a_ts;
    accl_ptr = w.acc_l + it.b * w.al_sb + it.h * w.al_sh + it.r * w.al_rs + static_cast<long long>(t) * w.al_ts;
  }
  if ((EPI == kEpiAcc || EPI == kEpiAccOut) && row_ok && !skip) {
    const float la = *accl_ptr;
    lse_merge_weights(la, lse_part, L, w_acc, w_part);
  }
  if (EPI == kEpiAcc) (void)pair_meet(pair_bar, pair_n, ctl);  // both halves have read the stored LSE
  __nv_bfloat16* out_row = nullptr;
  if (EPI == kEpiOut || EPI == kEpiAccOut)
    out_row = static_cast<__nv_bfloat16*>(w.o) + it.b * w.o_sb + it.h * w.o_sh + it.r * w.o_rs +
              static_cast<long long>(t) * w.o_ts;
  const float wp = w_part * inv_l;
#pragma unroll
  for (int cc = 0; cc < HD / CH; ++cc) {
    const int col0 = half * HD + cc * CH;
    uint32_t orow[CH];
    if (has_o) {
      if constexpr (CH == 32)
        tmem_ld32(o_addr + col0, orow);
      else
        tmem_ld16(o_addr + col0, orow);
      tmem_ld_wait(orow);
    } else {
#pragma unroll
      for (int e = 0; e < CH; ++e) orow[e] = 0u;
    }
    if (row_ok && !skip) {
      float vals[CH];
#pragma unroll
      for (int e = 0; e < CH; ++e) vals[e] = __uint_as_float(orow[e]) * wp;
      if (EPI == kEpiAcc || EPI == kEpiAccOut) {
#pragma unroll
        for (int e = 0; e < CH; e += 4) {
          if (col0 + e < w.d) {
            const float4 a = *reinterpret_cast<const float4*>(acc_row + col0 + e);
            vals[e] = fmaf(w_acc, a.x, vals[e]);
            vals[e + 1] = fmaf(w_acc, a.y, vals[e + 1]);
            vals[e + 2] = fmaf(w_acc, a.z, vals[e + 2]);
            vals[e + 3] = fmaf(w_acc, a.w, vals[e + 3]);
          }
        }
      }
      if (EPI == kEpiPart || EPI == kEpiAcc) {
#pragma unroll
        for (int e = 0; e < CH; e += 4)
          if (col0 + e < w.d)
            *reinterpret_cast<float4*>(acc_row + col0 + e) = make_float4(vals[e], vals[e + 1], vals[e + 2], vals[e + 3]);
      } else {
#pragma unroll
        for (int e = 0; e < CH; e += 8) {
          if (col0 + e < w.d) {
            uint4 pkt;
            pkt.x = pack_bf16x2(vals[e], vals[e + 1]);
            pkt.y = pack_bf16x2(vals[e + 2], vals[e + 3]);
            pkt.z = pack_bf16x2(vals[e + 4], vals[e + 5]);
            pkt.w = pack_bf16x2(vals[e + 6], vals[e + 7]);
            *reinterpret_cast<uint4*>(out_row + col0 + e) = pkt;
          }
        }
      }
    }
  }
  if (row_ok && !skip && half == 0) {
    if (EPI == kEpiPart || EPI == kEpiAcc) {
      *accl_ptr = L;
    } else if (w.lse != nullptr) {
      w.lse[it.b * w.l_sb + it.h * w.l_sh + it.r * w.l_rs + static_cast<long long>(t) * w.l_ts] = L;
    }
  }
}

// p = 2^(s * scale_log2 - base) for the scores of column pairs [E0, E1) of this row, packed to
// bf16 pairs in pk (the row of P_q); row sums accumulated in two packed fp32x2 chains.  EVERY > 0: one column pair in
// EVERY goes to the FMA-pipe polynomial instead of the MUFU (only for tiles without masked
// scores, see exp2_poly3).
template <int EVERY, int E0, int E1, int NSC>
__device__ __forceinline__ void softmax_exp(const uint32_t (&sr)[NSC][32], float sl2, float base,
                                            uint32_t (&pk)[NSC * 16], float2 (&rs)[2]) {
  const float2 sc = make_float2(sl2, sl2);
  const float2 nb = make_float2(-base, -base);
#pragma unroll
  for (int e = E0; e < E1; ++e) {
    const float2 x = __ffma2_rn(
        make_float2(__uint_as_float(sr[e >> 4][(2 * e) & 31]), __uint_as_float(sr[e >> 4][(2 * e + 1) & 31])), sc, nb);
    float2 p;
    if (EVERY > 0 && (e % (EVERY > 0 ? EVERY : 1)) == (EVERY > 0 ? EVERY : 1) - 1) {
      p = exp2_poly3_x2(x);
    } else {
      p.x = ex2_approx(x.x);
      p.y = ex2_approx(x.y);
    }
    rs[e & 1] = __fadd2_rn(rs[e & 1], p);
    pk[e] = pack_bf16x2(p.x, p.y);
  }
}

// As softmax_exp, but each 16-pair chunk of P_q goes to tensor memory as soon as it is computed
// (fewer live registers; used where P_q's columns are known to be free before the exponentials).
template <int EVERY, int NSC>
__device__ __forceinline__ void softmax_exp_store(const uint32_t (&sr)[NSC][32], float sl2, float base,
                                                  uint32_t p_addr, float2 (&rs)[2]) {
  const float2 sc = make_float2(sl2, sl2);
  const float2 nb = make_float2(-base, -base);
#pragma unroll
  for (int cc = 0; cc < NSC; ++cc) {
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[cc][2 * e]), __uint_as_float(sr[cc][2 * e + 1])), sc, nb);
      float2 p;
      if (EVERY > 0 && (e % (EVERY > 0 ? EVERY : 1)) == (EVERY > 0 ? EVERY : 1) - 1) {
        p = exp2_poly3_x2(x);
      } else {
        p.x = ex2_approx(x.x);
        p.y = ex2_approx(x.y);
      }
      rs[e & 1] = __fadd2_rn(rs[e & 1], p);
      pk[e] = pack_bf16x2(p.x, p.y);
    }
    tmem_st16(p_addr + cc * 16, pk);
  }
}

// ---------------------------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------------------------
template <int DP, int EPI, bool WIN>
__global__ void __launch_bounds__(FmhaCfg<DP>::THREADS, 1)
    fmha_fwd_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnWork w, int n_steps, int n_items) {
  using C = FmhaCfg<DP>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);

  uint8_t* sQ = smem;  // two tiles
  uint8_t* sK = sQ + 2 * C::Q_TILE_BYTES;
  uint8_t* sV = sK + C::STAGES * C::KV_TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + C::STAGES * C::KV_TILE_BYTES);
  uint64_t* bar_q_full = bars;
  uint64_t* bar_q_empty = bars + 1;
  uint64_t* bar_mma_done = bars + 2;
  uint64_t* bar_k_full = bars + 3;
  uint64_t* bar_v_full = bar_k_full + C::STAGES;
  uint64_t* bar_kv_empty = bar_v_full + C::STAGES;
  uint64_t* bar_s_full = bar_kv_empty + C::STAGES;  // [2]
  uint64_t* bar_p_full = bar_s_full + 2;            // [2]
  uint64_t* bar_pv_done = bar_p_full + 2;           // [2]
  uint64_t* bar_o_full = bar_pv_done + 2;           // [2]
  uint64_t* bar_o_empty = bar_o_full + 2;           // [2]
  uint64_t* bar_stats = bar_o_empty + 2;            // [2]
  uint64_t* bar_s_free = bar_stats + 2;             // [2] softmax has loaded S_q into registers
  uint64_t* bar_plan_full = bar_s_free + 2;         // [2] item plan slot written
  uint64_t* bar_plan_empty = bar_plan_full + 2;     // [2] item plan slot read by every consumer
  uint64_t* bar_exp_done = bar_plan_empty + 2;      // [2] softmax warpgroup q finished an exponential phase
  uint64_t* bar_pair = bar_exp_done + 2;            // [2] column-split halves of tile q meet (256 threads)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_pair + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float2* stats = reinterpret_cast<float2*>(tmem_slot + 4);  // [2][128] (m_used, l_sum)
  ItemPlan* plan = reinterpret_cast<ItemPlan*>(stats + 2 * 128);  // [2], slot = item sequence & 1
  // Column-split softmax: row maxima [2 tile parity][2 q][2 half][128] and row sums [2 item
  // parity][2 q][2 half][128] of the two halves of each row.
  float* xch = reinterpret_cast<float*>(plan + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WaitCtl ctl{abort_flag, w.wait_limit_ns, w.dev_status};

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    mbar_init(bar_q_empty, C::ISSUERS);   // one arrival per MMA issuer
    mbar_init(bar_mma_done, C::ISSUERS);
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(bar_k_full + i, 1);
      mbar_init(bar_v_full + i, 1);
      mbar_init(bar_kv_empty + i, C::ISSUERS);  // one arrival per MMA issuer
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(bar_s_full + q, 1);
      constexpr int kHalves = C::SPLIT ? 2 : 1;
      mbar_init(bar_p_full + q, C::SPLIT && kSplitWarpArrive ? 8 : 128 * kHalves);
      mbar_init(bar_pv_done + q, 1);
      mbar_init(bar_o_full + q, 1);
      mbar_init(bar_o_empty + q, 128 * kHalves);
      mbar_init(bar_stats + q, 128);
      mbar_init(bar_s_free + q, C::SPLIT && kSplitWarpArrive ? 8 : 128 * kHalves);
      // Readers of a plan slot: each MMA issuer thread, every softmax warp, the 4 epilogue warps.
      mbar_init(bar_plan_full + q, 1);
      mbar_init(bar_plan_empty + q, C::ISSUERS + C::SM_WARPS + (C::SPLIT ? 0 : 4));
      mbar_init(bar_exp_done + q, 4);  // one arrival per softmax warp
      mbar_init(bar_pair + q, 8);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::PROD_WARP && lane == 0) {
    tma_prefetch_map(&tm_q);
    tma_prefetch_map(&tm_k);
    tma_prefetch_map(&tm_v);
  }
  if (warp == 13) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // A launch that follows this one on the stream with programmatic dependent launch (the next
  // step of the stepwise ring) may be scheduled now: it takes SMs only as this grid's CTAs exit,
  // and waits for this grid to finish before its epilogue touches memory this grid writes.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp >= C::PROD_WARP) {
    setmaxnreg_dec<RegSplit<DP, EPI>::kProd>();
    if (warp == C::PROD_WARP && lane == 0) {
      // ================================================================ TMA producer
      int it_q = 0, it_seq = 0;
      long long g = 0;
      bool ok = true;
      for (int k = 0; ok && k * static_cast<int>(gridDim.x) < n_items; ++k) {
        const int idx = item_of_cta(k);
        if (idx >= n_items) continue;
        // Publish the item's plan (decoded item and tile count) to the other roles.  The
        // producer runs ahead of them, so this set-up leaves their critical path.
        Item it;
        decode_item(w, idx, it);
        if (C::P_SEP) {
          const int slot = it_seq & 1;
          if (it_seq >= 2 && !mbar_wait(bar_plan_empty + slot, ((it_seq >> 1) - 1) & 1, ctl, 0x103)) break;
          plan[slot].it = it;
          plan[slot].n = walk_count<WIN, C::BN>(w, it, n_steps);
          mbar_arrive(bar_plan_full + slot);
          ++it_seq;
        }
        Walk wk;
        bool has = walk_begin<WIN, C::BN>(wk, w, it, n_steps);
        if (!has) continue;
        if (it_q > 0 && !mbar_wait(bar_q_empty, (it_q - 1) & 1, ctl, 0x101)) break;
        mbar_arrive_expect_tx(bar_q_full, 2 * C::Q_TILE_BYTES);
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int cb = 0; cb < C::NCB; ++cb)
            tma_load_5d(sQ + q * C::Q_TILE_BYTES + cb * C::Q_BLOCK_BYTES, &tm_q, bar_q_full, cb * C::CB,
                        it.t0 + 128 * q, it.r, it.h, it.b);
        ++it_q;
        for (; has; has = walk_next<WIN, C::BN>(wk, w, it, n_steps)) {
          const int st = static_cast<int>(g % C::STAGES);
          if (g >= C::STAGES &&
              !mbar_wait(bar_kv_empty + st, static_cast<uint32_t>((g / C::STAGES) - 1) & 1, ctl, 0x102)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar_k_full + st, C::KV_TILE_BYTES);
#pragma unroll
          for (int cb = 0; cb < C::NCB; ++cb)
            tma_load_5d(sK + st * C::KV_TILE_BYTES + cb * C::KV_BLOCK_BYTES, &tm_k, bar_k_full + st, cb * C::CB, wk.u0,
                        wk.s, it.hk, it.b);
          mbar_arrive_expect_tx(bar_v_full + st, C::KV_TILE_BYTES);
#pragma unroll
          for (int cb = 0; cb < C::NCB; ++cb)
            tma_load_5d(sV + st * C::KV_TILE_BYTES + cb * C::KV_BLOCK_BYTES, &tm_v, bar_v_full + st, cb * C::CB, wk.u0,
                        wk.s, it.hk, it.b);
          ++g;
        }
      }
      // No TMA write may still be in flight when the CTA exits.
      if (it_q > 0) mbar_drain(bar_q_full, (it_q - 1) & 1, w.wait_limit_ns);
      for (long long j = (g > C::STAGES ? g - C::STAGES : 0); j < g; ++j) {
        mbar_drain(bar_k_full + j % C::STAGES, static_cast<uint32_t>(j / C::STAGES) & 1, w.wait_limit_ns);
        mbar_drain(bar_v_full + j % C::STAGES, static_cast<uint32_t>(j / C::STAGES) & 1, w.wait_limit_ns);
      }
    } else if (!C::P_SEP && warp == C::PROD_WARP + 1 && lane == 0) {
      // ================================================================ MMA issuer (P over S)
      // One thread, fixed order per key tile j: PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1).  QK_q(j+1)
      // rewrites S_q, which holds P_q(j), so it waits for PV_q(j) to complete; meanwhile the
      // tensor core runs the other tile's work, and the two query tiles stay staggered.
      constexpr uint32_t idesc_qk = make_idesc_bf16(128, C::BN, 0, 0);
      constexpr uint32_t idesc_pv = make_idesc_bf16(128, DP, 0, 1);
      const uint32_t q_base = smem_addr(sQ);
      const uint32_t k_base = smem_addr(sK);
      const uint32_t v_base = smem_addr(sV);
      const DescBase<C> db;
      int it_all = 0, it_q = 0;
      long long g = 0;
      // Every query tile processes every K/V tile, so the per-tile barrier phases all follow the
      // CTA's running K/V tile index g + j.
      bool ok = true;
      for (int k = 0; ok && k * static_cast<int>(gridDim.x) < n_items; ++k) {
        const int idx = item_of_cta(k);
        if (idx >= n_items) continue;
        Item it;
        decode_item(w, idx, it);
        const int n = walk_count<WIN, C::BN>(w, it, n_steps);
        if (n == 0) {
          for (int q = 0; q < 2 && ok && it_all > 0; ++q)
            ok = mbar_wait_issuer(bar_o_empty + q, (it_all - 1) & 1, ctl, 0x208);
          if (!ok) break;
          mma_commit(bar_o_full + 0);
          mma_commit(bar_o_full + 1);
          ++it_all;
          continue;
        }
        ok = mbar_wait_issuer(bar_q_full, it_q & 1, ctl, 0x201) &&
             mbar_wait_issuer(bar_k_full + g % C::STAGES, static_cast<uint32_t>(g / C::STAGES) & 1, ctl, 0x204);
        for (int q = 0; q < 2 && ok; ++q) {
          if (g > 0 && !(ok = mbar_wait_issuer(bar_pv_done + q, static_cast<uint32_t>(g - 1) & 1, ctl, 0x203))) break;
          tc_fence_after();
          fmha_issue_qk<C>(db, tmem + C::S_COL0 + C::S_STRIDE * q, q_base + q * C::Q_TILE_BYTES,
                           k_base + static_cast<int>(g % C::STAGES) * C::KV_TILE_BYTES, idesc_qk);
          mma_commit(bar_s_full + q);
        }
        if (!ok) break;
        if (n == 1) mma_commit(bar_q_empty);
        for (int j = 0; ok && j < n; ++j) {
          const long long gj = g + j;
          const bool has_next = j + 1 < n;
          for (int q = 0; q < 2 && ok; ++q) {
            ok = mbar_wait_all_issuer(bar_p_full + q, static_cast<uint32_t>(gj) & 1,
                                      q == 1 ? nullptr : bar_v_full + gj % C::STAGES, static_cast<uint32_t>(gj / C::STAGES) & 1,
                                      (j > 0 || it_all == 0) ? nullptr : bar_o_empty + q, (it_all - 1) & 1, ctl, 0x205);
            if (!ok) break;
            tc_fence_after();
            fmha_issue_pv<C>(db, tmem + C::O_COL0 + C::O_STRIDE * q, tmem + C::P_COL0 + C::P_STRIDE * q,
                             v_base + static_cast<int>(gj % C::STAGES) * C::KV_TILE_BYTES, idesc_pv, j > 0);
            mma_commit(bar_pv_done + q);
            if (has_next) {
              const long long gn = gj + 1;
              ok = mbar_wait_all_issuer(bar_pv_done + q, static_cast<uint32_t>(gj) & 1,
                                        q == 1 ? nullptr : bar_k_full + gn % C::STAGES,
                                        static_cast<uint32_t>(gn / C::STAGES) & 1, nullptr, 0, ctl, 0x209);
              if (!ok) break;
              tc_fence_after();
              fmha_issue_qk<C>(db, tmem + C::S_COL0 + C::S_STRIDE * q, q_base + q * C::Q_TILE_BYTES,
                               k_base + static_cast<int>(gn % C::STAGES) * C::KV_TILE_BYTES, idesc_qk);
              mma_commit(bar_s_full + q);
              if (q == 1 && j + 2 == n) mma_commit(bar_q_empty);  // last QKs of the item issued
            }
          }
          if (!ok) break;
          mma_commit(bar_kv_empty + gj % C::STAGES);
        }
        if (!ok) break;
        mma_commit(bar_o_full + 0);
        mma_commit(bar_o_full + 1);
        g += n;
        ++it_q;
        ++it_all;
      }
      // Tensor memory is freed only after every MMA issued here has completed.
      mma_commit(bar_mma_done);
      mbar_drain(bar_mma_done, 0, w.wait_limit_ns);
    } else if (C::P_SEP && (warp == C::PROD_WARP + 1 || warp == C::PROD_WARP + 2) && lane == 0) {
      // ================================================================ MMA issuers
      // One thread per query tile q (warp 13: q = 0, warp 14: q = 1).  Each blocks on its own next
      // event and issues, per key tile j:
      //   QK_q(j+1) once K_{j+1} is loaded and S_q is free: with P in its own columns, as soon as
      //             the softmax has loaded S_q(j) into registers (s_free); with P over S, once
      //             PV_q(j) has completed (pv_done);
      //   PV_q(j)   once P_q(j) is written (p_full), V_j is loaded and, for the first tile of an
      //             item, the epilogue is done with O_q of the previous item (o_empty).
      // A K/V stage is released when both issuers have committed it (kv_empty counts 2), and Q
      // when both have issued their last QK of the item (q_empty counts 2).  The issuer that is
      // behind never waits on the one ahead, so the two cannot deadlock.
      const int q = warp - (C::PROD_WARP + 1);
      constexpr uint32_t idesc_qk = make_idesc_bf16(128, C::BN, 0, 0);
      constexpr uint32_t idesc_pv = make_idesc_bf16(128, DP, 0, 1);
      const uint32_t q_addr = smem_addr(sQ) + q * C::Q_TILE_BYTES;
      const uint32_t k_base = smem_addr(sK);
      const uint32_t v_base = smem_addr(sV);
      const uint32_t d_s = tmem + C::S_COL0 + C::S_STRIDE * q;
      const uint32_t d_o = tmem + C::O_COL0 + C::O_STRIDE * q;
      const uint32_t p_t = tmem + C::P_COL0 + C::P_STRIDE * q;
      const DescBase<C> db;
      int it_all = 0, it_q = 0;
      long long g = 0;
      int cq = 0;   // QKs issued for this query tile (all items)
      int cpv = 0;  // PVs issued for this query tile (all items)
      bool ok = true;
      auto qk = [&](long long gk, bool last_of_item) -> bool {
        // S_q must be free: the previous QK's S consumed (own P columns) or its PV done (P over S).
        if (!mbar_wait_all_issuer(cq > 0 ? (C::P_SEP ? bar_s_free + q : bar_pv_done + q) : nullptr, (cq - 1) & 1,
                                  bar_k_full + gk % C::STAGES, static_cast<uint32_t>(gk / C::STAGES) & 1, nullptr, 0,
                                  ctl, 0x202))
          return false;
        tc_fence_after();
        fmha_issue_qk<C>(db, d_s, q_addr, k_base + static_cast<int>(gk % C::STAGES) * C::KV_TILE_BYTES, idesc_qk);
        mma_commit(bar_s_full + q);
        ++cq;
        if (last_of_item) mma_commit(bar_q_empty);
        return true;
      };
      for (int k = 0; ok && k * static_cast<int>(gridDim.x) < n_items; ++k) {
        const int idx = item_of_cta(k);
        if (idx >= n_items) continue;
        if (!(ok = mbar_wait_issuer(bar_plan_full + (it_all & 1), (it_all >> 1) & 1, ctl, 0x20b))) break;
        const int n = plan[it_all & 1].n;
        mbar_arrive(bar_plan_empty + (it_all & 1));
        if (n > 0) {
          ok = mbar_wait_issuer(bar_q_full, it_q & 1, ctl, 0x201) && qk(g, n == 1);
          for (int j = 0; ok && j < n; ++j) {
            const long long gj = g + j;
            if (C::P_SEP && j + 1 < n && !(ok = qk(gj + 1, j + 2 == n))) break;
            ok = mbar_wait_all_issuer(bar_p_full + q, cpv & 1, bar_v_full + gj % C::STAGES,
                                      static_cast<uint32_t>(gj / C::STAGES) & 1,
                                      (j > 0 || it_all == 0) ? nullptr : bar_o_empty + q, (it_all - 1) & 1, ctl, 0x206);
            if (!ok) break;
            tc_fence_after();
            fmha_issue_pv<C>(db, d_o, p_t, v_base + static_cast<int>(gj % C::STAGES) * C::KV_TILE_BYTES, idesc_pv,
                             j > 0);
            mma_commit(bar_pv_done + q);
            ++cpv;
            mma_commit(bar_kv_empty + gj % C::STAGES);
            if (!C::P_SEP && j + 1 < n && !(ok = qk(gj + 1, j + 2 == n))) break;
          }
          if (!ok) break;
          mma_commit(bar_o_full + q);  // O_q of this item is final once these MMAs land
          g += n;
          ++it_q;
        } else {
          // No PV in this item; still keep o_full at most one phase ahead of the epilogue.
          if (it_all > 0 && !(ok = mbar_wait_issuer(bar_o_empty + q, (it_all - 1) & 1, ctl, 0x208))) break;
          mma_commit(bar_o_full + q);
        }
        ++it_all;
      }
      // Tensor memory is freed only after every MMA issued here has completed.
      mma_commit(bar_mma_done);
      mbar_drain(bar_mma_done, 0, w.wait_limit_ns);
    }
  } else if (C::SPLIT) {
    if constexpr (C::SPLIT) {
      setmaxnreg_inc<RegSplit<DP, EPI>::kSoftmax>();
      asm volatile("griddepcontrol.wait;" ::: "memory");  // runs the epilogue (see the epilogue role)
      // ============================================================ softmax, column-split
      // Warps 0-3 / 4-7: query tile 0 / 1, S columns [0, BN/2); warps 8-11 / 12-15: the same tiles,
      // columns [BN/2, BN).  Thread = row = tensor-memory lane, as in the unsplit softmax.
      const int q = (warp >> 2) & 1;
      const int half = warp >> 3;
      const int row = threadIdx.x & 127;
      const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
      const uint32_t s_addr = lane_addr + C::S_COL0 + C::S_STRIDE * q + half * C::HCOLS;
      const uint32_t p_addr = lane_addr + C::P_COL0 + C::P_STRIDE * q + half * (C::HCOLS / 2);
      const uint32_t o_addr = lane_addr + C::O_COL0 + C::O_STRIDE * q;
      float* xmax = xch;                  // [2][2][2][128]
      float* xsum = xch + 2 * 2 * 2 * 128;  // [2][2][2][128]
      const float sl2 = w.scale_log2;
      constexpr int NH = C::HCOLS / 32;   // 32-column chunks of this half of an S row
      constexpr int HD = C::D / 2;        // O columns of this half
      constexpr int OCH = HD < 32 ? HD : 32;
      int it_all = 0, c = 0, meets = 0;
      bool ok = true;
      bool s_seen = false;  // S_q of tile c already seen complete
      for (int k = 0; ok && k * static_cast<int>(gridDim.x) < n_items; ++k) {
        const int idx = item_of_cta(k);
        if (idx >= n_items) continue;
        ok = __all_sync(0xffffffffu, mbar_wait(bar_plan_full + (it_all & 1), (it_all >> 1) & 1, ctl, 0x305));
        if (!ok) break;
        const Item it = plan[it_all & 1].it;
        const bool has_o = plan[it_all & 1].n > 0;
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_plan_empty + (it_all & 1));
        const bool row_ok = row < it.rows_valid[q];
        const long long pos_q = it.pos0 + static_cast<long long>(it.t0 + 128 * q + row) * w.q_tstride;
        float m_used = -INFINITY;  // running max of scaled scores, log2 units (same in both halves)
        float l_sum = 0.f;         // running sum of 2^(x - m_used) over this half's columns
        Walk wk;
        int cur_s = -1, row_lim = 0, row_lo = 0;
        for (bool has = walk_begin<WIN, C::BN>(wk, w, it, n_steps); has; has = walk_next<WIN, C::BN>(wk, w, it, n_steps)) {
          if (wk.s != cur_s) {
            cur_s = wk.s;
            row_lim = row_ok ? visible_key_limit(w, pos_q, wk.s) : w.n_kv;
            if (WIN) row_lo = row_ok ? visible_key_start(w, pos_q, wk.s) : 0;
          }
          if (!__all_sync(0xffffffffu, s_seen)) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar_s_full + q, c & 1, ctl, 0x301));
            if (!ok) break;
          }
          s_seen = false;
          tc_fence_after();
          uint32_t sr[NH][32];
#pragma unroll
          for (int cc = 0; cc < NH; ++cc) tmem_ld32(s_addr + cc * 32, sr[cc]);
          tmem_ld_wait(sr[0]);
#pragma unroll
          for (int cc = 1; cc < NH; ++cc) reg_dep(sr[cc]);
          tc_fence_before();
          if (kSplitWarpArrive) {  // the next QK_q may overwrite S_q once both halves hold it
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_s_free + q);
          } else {
            mbar_arrive(bar_s_free + q);
          }
          const int c0 = wk.u0 + half * C::HCOLS;  // key of this half's first column
          const int lim = row_lim - c0;            // columns [lo, lim) of this half are visible
          const int lo = WIN ? row_lo - c0 : 0;
          const bool cut = WIN ? (lim < C::HCOLS || lo > 0) : lim < C::HCOLS;
          const bool masked = __any_sync(0xffffffffu, cut);
          if (cut) {
#pragma unroll
            for (int e = 0; e < C::HCOLS; ++e)
              if (e >= lim || (WIN && e < lo)) sr[e >> 5][e & 31] = __float_as_uint(-INFINITY);
          }
          float mxp[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) mxp[i] = __uint_as_float(sr[0][i]);
#pragma unroll
          for (int e = 8; e < C::HCOLS; e += 2)
            mxp[(e >> 1) & 7] = fmax3(mxp[(e >> 1) & 7], __uint_as_float(sr[e >> 5][e & 31]),
                                      __uint_as_float(sr[(e + 1) >> 5][(e + 1) & 31]));
          const float mx_half =
              fmax3(fmax3(mxp[0], mxp[1], mxp[2]), fmax3(mxp[3], mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7]));
          // Row max over both halves: exchange through shared memory (slot by tile parity).
          float* xm = xmax + ((c & 1) * 4 + q * 2) * 128;
          xm[half * 128 + row] = mx_half;
          ok = __all_sync(0xffffffffu, pair_meet(bar_pair + q, meets, ctl));
          if (!ok) break;
          const float mx = fmaxf(mx_half, xm[(half ^ 1) * 128 + row]);
          const float m_tile = mx * sl2;
          float m_new = m_used;
          float alpha = 1.f;
          bool rescale = false;
          if (m_tile > m_used) {
            if (m_used == -INFINITY) {
              m_new = m_tile;  // nothing accumulated yet in this item: this row of O is zero
            } else if (m_tile > m_used + 8.f) {
              m_new = m_tile;
              alpha = ex2_approx(m_used - m_new);
              rescale = true;
            }
          }
          const float base = (m_new == -INFINITY) ? 0.f : m_new;
          const bool any_rescale = __any_sync(0xffffffffu, rescale);
          float2 rsp[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};  // packed row sums
          constexpr int HALF = NH * 8;  // column pairs in half of this half-row
          uint32_t pk[NH * 16];
          bool pv_seen;
          if (masked || kEmuEvery == 0) {
            softmax_exp<0, 0, HALF>(sr, sl2, base, pk, rsp);
            pv_seen = c == 0 || mbar_test_wait(bar_pv_done + q, (c - 1) & 1);
            softmax_exp<0, HALF, 2 * HALF>(sr, sl2, base, pk, rsp);
          } else {
            softmax_exp<kEmuEvery, 0, HALF>(sr, sl2, base, pk, rsp);
            pv_seen = c == 0 || mbar_test_wait(bar_pv_done + q, (c - 1) & 1);
            softmax_exp<kEmuEvery, HALF, 2 * HALF>(sr, sl2, base, pk, rsp);
          }
          s_seen = mbar_test_wait(bar_s_full + q, (c + 1) & 1);  // the next QK_q, issued at s_free
          if (!__all_sync(0xffffffffu, pv_seen)) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar_pv_done + q, (c - 1) & 1, ctl, 0x302));
            if (!ok) break;
          }
          tc_fence_after();
          if constexpr (NH == 2)
            tmem_st32(p_addr, pk);
          else
            tmem_st16(p_addr, pk);
          if (any_rescale) {
            // This half's columns of O (the previous PV_q has landed: its wait is above).
#pragma unroll
            for (int cc = 0; cc < HD / OCH; ++cc) {
              const uint32_t a = o_addr + half * HD + cc * OCH;
              uint32_t orow[OCH];
              if constexpr (OCH == 32)
                tmem_ld32(a, orow);
              else
                tmem_ld16(a, orow);
              tmem_ld_wait(orow);
#pragma unroll
              for (int e = 0; e < OCH; e += 2) {
                const float2 v = __fmul2_rn(make_float2(__uint_as_float(orow[e]), __uint_as_float(orow[e + 1])),
                                            make_float2(alpha, alpha));
                orow[e] = __float_as_uint(v.x);
                orow[e + 1] = __float_as_uint(v.y);
              }
              if constexpr (OCH == 32)
                tmem_st32(a, orow);
              else
                tmem_st16(a, orow);
            }
          }
          l_sum = l_sum * alpha + ((rsp[0].x + rsp[0].y) + (rsp[1].x + rsp[1].y));
          m_used = m_new;
          tmem_st_wait();
          tc_fence_before();
          if (kSplitWarpArrive) {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_p_full + q);
          } else {
            mbar_arrive(bar_p_full + q);
          }
          ++c;
        }
        if (!ok) break;
        // Epilogue of this item's tile q: the row sum over both halves, then O / l and the LSE.
        float* xs = xsum + ((it_all & 1) * 4 + q * 2) * 128;
        xs[half * 128 + row] = l_sum;
        ok = __all_sync(0xffffffffu, pair_meet(bar_pair + q, meets, ctl));
        if (!ok) break;
        const float l_row = l_sum + xs[(half ^ 1) * 128 + row];
        ok = __all_sync(0xffffffffu, mbar_wait(bar_o_full + q, it_all & 1, ctl, 0x401));
        if (!ok) break;
        tc_fence_after();
        fmha_epilogue_row_half<C, EPI>(w, it, it.t0 + 128 * q + row, row_ok, has_o, make_float2(m_used, l_row),
                                       o_addr, half, bar_pair + q, meets, ctl);
        tc_fence_before();
        mbar_arrive(bar_o_empty + q);
        ++it_all;
      }
    }
  } else if (warp < 8) {
   if constexpr (!C::SPLIT) {
    setmaxnreg_inc<RegSplit<DP, EPI>::kSoftmax>();
    // ================================================================ softmax (query tile q)
    const int q = warp >> 2;
    const int row = threadIdx.x & 127;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t s_addr = lane_addr + C::S_COL0 + C::S_STRIDE * q;
    const uint32_t p_addr = lane_addr + C::P_COL0 + C::P_STRIDE * q;
    const uint32_t o_addr = lane_addr + C::O_COL0 + C::O_STRIDE * q;
    const float sl2 = w.scale_log2;
    int it_all = 0, c = 0;
    bool ok = true;
    // Barrier tests issued ahead of their use: a test costs a few hundred cycles even when the
    // phase is complete, so it is issued while the exponentials run and its result read later.
    bool s_seen = false;  // S_q of tile c already seen complete
    for (int k = 0; ok && k * static_cast<int>(gridDim.x) < n_items; ++k) {
        const int idx = item_of_cta(k);
        if (idx >= n_items) continue;
      Item it;
      if (C::P_SEP) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_plan_full + (it_all & 1), (it_all >> 1) & 1, ctl, 0x305));
        if (!ok) break;
        it = plan[it_all & 1].it;
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_plan_empty + (it_all & 1));
      } else {
        decode_item(w, idx, it);
      }
      const bool row_ok = row < it.rows_valid[q];
      const long long pos_q = it.pos0 + static_cast<long long>(it.t0 + 128 * q + row) * w.q_tstride;
      float m_used = -INFINITY;  // running max of scaled scores, log2 units
      float l_sum = 0.f;         // running sum of 2^(x - m_used)
      Walk wk;
      int cur_s = -1, row_lim = 0, row_lo = 0;
      StripedPos row_last{0, -1}, row_first{0, -1};  // tile-major launches: this row's position and window start
      if (kTileWalk<C::BN> && w.tile_major) {
        row_last = striped_pos(w, pos_q);
        if (WIN && w.window > 0) row_first = striped_pos(w, pos_q - w.window + 1);
      }
      for (bool has = walk_begin<WIN, C::BN>(wk, w, it, n_steps); has; has = walk_next<WIN, C::BN>(wk, w, it, n_steps)) {
        if (wk.s != cur_s) {
          cur_s = wk.s;
          if (kTileWalk<C::BN> && w.tile_major) {
            row_lim = row_ok ? striped_lim(w, row_last, wk.s) : w.n_kv;
            if (WIN) row_lo = row_ok ? striped_start(w, row_first, wk.s) : 0;
          } else {
            row_lim = row_ok ? visible_key_limit(w, pos_q, wk.s) : w.n_kv;
            if (WIN) row_lo = row_ok ? visible_key_start(w, pos_q, wk.s) : 0;
          }
        }
        if (!__all_sync(0xffffffffu, s_seen)) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar_s_full + q, c & 1, ctl, 0x301));
          if (!ok) break;
        }
        s_seen = false;
        tc_fence_after();
        constexpr int NSC = C::NSC;
        uint32_t sr[NSC][32];
#pragma unroll
        for (int cc = 0; cc < NSC; ++cc) tmem_ld32(s_addr + cc * 32, sr[cc]);
        tmem_ld_wait(sr[0]);
#pragma unroll
        for (int cc = 1; cc < NSC; ++cc) reg_dep(sr[cc]);
        if (C::P_SEP) {
          // S_q is in registers: the next QK_q may overwrite it while this tile's softmax runs.
          tc_fence_before();
          mbar_arrive(bar_s_free + q);
        }
        const int lim = row_lim - wk.u0;  // keys [lo, lim) of this tile are visible to this row
        const int lo = WIN ? row_lo - wk.u0 : 0;
        const bool cut = WIN ? (lim < C::BN || lo > 0) : lim < C::BN;
        const bool masked = __any_sync(0xffffffffu, cut);
        if (cut) {
#pragma unroll
          for (int e = 0; e < C::BN; ++e)
            if (e >= lim || (WIN && e < lo)) sr[e >> 5][e & 31] = __float_as_uint(-INFINITY);
        }
        // Row max as 8 independent chains (a single chain of BN dependent max operations would
        // be latency-bound).
        float mxp[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mxp[i] = __uint_as_float(sr[0][i]);
#pragma unroll
        for (int e = 8; e < C::BN; e += 2)
          mxp[(e >> 1) & 7] = fmax3(mxp[(e >> 1) & 7], __uint_as_float(sr[e >> 5][e & 31]),
                                    __uint_as_float(sr[(e + 1) >> 5][(e + 1) & 31]));
        const float mx = fmax3(fmax3(mxp[0], mxp[1], mxp[2]), fmax3(mxp[3], mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7]));
        const float m_tile = mx * sl2;
        float m_new = m_used;
        float alpha = 1.f;
        bool rescale = false;
        if (m_tile > m_used) {
          if (m_used == -INFINITY) {
            m_new = m_tile;  // nothing accumulated yet in this item: this row of O is zero
          } else if (m_tile > m_used + 8.f) {
            m_new = m_tile;
            alpha = ex2_approx(m_used - m_new);
            rescale = true;
          }
        }
        const float base = (m_new == -INFINITY) ? 0.f : m_new;
        const bool any_rescale = __any_sync(0xffffffffu, rescale);
        float2 rsp[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};  // packed row sums
        if (C::P_SEP) {
          // P_q has its own columns, which the previous PV_q may still be reading.  The
          // exponentials are computed into registers first, so by the time of this wait that PV
          // has almost always landed.
          constexpr int HALF = NSC * 8;  // column pairs in half a row
          uint32_t pk[NSC * 16];
          bool pv_seen;
          if (AlternateExps<DP>::value) {
            // Exponential phases alternate between the two warpgroups: tile c of warpgroup 0
            // waits for phase c - 1 of warpgroup 1, which waits for phase c of warpgroup 0.
            const bool first = q == 0 && c == 0;
            if (!first) {
              const uint32_t par = q == 0 ? static_cast<uint32_t>(c - 1) & 1 : static_cast<uint32_t>(c) & 1;
              ok = __all_sync(0xffffffffu, mbar_wait(bar_exp_done + (q ^ 1), par, ctl, 0x306));
              if (!ok) break;
            }
          }
          if (masked || kEmuEvery == 0) {
            softmax_exp<0, 0, HALF>(sr, sl2, base, pk, rsp);
            pv_seen = c == 0 || mbar_test_wait(bar_pv_done + q, (c - 1) & 1);
            softmax_exp<0, HALF, 2 * HALF>(sr, sl2, base, pk, rsp);
          } else {
            softmax_exp<kEmuEvery, 0, HALF>(sr, sl2, base, pk, rsp);
            pv_seen = c == 0 || mbar_test_wait(bar_pv_done + q, (c - 1) & 1);
            softmax_exp<kEmuEvery, HALF, 2 * HALF>(sr, sl2, base, pk, rsp);
          }
          if (AlternateExps<DP>::value) {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_exp_done + q);
          }
          s_seen = mbar_test_wait(bar_s_full + q, (c + 1) & 1);  // the next QK_q, issued at s_free
          if (!__all_sync(0xffffffffu, pv_seen)) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar_pv_done + q, (c - 1) & 1, ctl, 0x302));
            if (!ok) break;
          }
          tc_fence_after();
          if constexpr (NSC == 4)
            tmem_st64(p_addr, pk);
          else
            tmem_st32(p_addr, pk);
        } else {
          // P_q over S_q: those columns are free once S_q is loaded (the next QK_q waits for this
          // PV_q); only the O rescale needs the previous PV_q to have landed.
          if (any_rescale && c > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar_pv_done + q, (c - 1) & 1, ctl, 0x302));
            if (!ok) break;
            tc_fence_after();
          }
          if (masked || kEmuEvery == 0)
            softmax_exp_store<0, NSC>(sr, sl2, base, p_addr, rsp);
          else
            softmax_exp_store<kEmuEvery, NSC>(sr, sl2, base, p_addr, rsp);
        }
        if (any_rescale) {
#pragma unroll
          for (int cc = 0; cc < DP / 32; ++cc) {
            uint32_t orow[32];
            tmem_ld32(o_addr + cc * 32, orow);
            tmem_ld_wait(orow);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 v = __fmul2_rn(make_float2(__uint_as_float(orow[e]), __uint_as_float(orow[e + 1])),
                                          make_float2(alpha, alpha));
              orow[e] = __float_as_uint(v.x);
              orow[e + 1] = __float_as_uint(v.y);
            }
            tmem_st32(o_addr + cc * 32, orow);
          }
        }
        l_sum = l_sum * alpha + ((rsp[0].x + rsp[0].y) + (rsp[1].x + rsp[1].y));
        m_used = m_new;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar_p_full + q);
        ++c;
      }
      if (!ok) break;
      // Hand (m, l) of this item to the epilogue warps once they are done with the previous item.
      if (it_all > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_o_empty + q, (it_all - 1) & 1, ctl, 0x303));
        if (!ok) break;
      }
      stats[q * 128 + row] = make_float2(m_used, l_sum);
      mbar_arrive(bar_stats + q);
      ++it_all;
    }
   }
  } else {
   if constexpr (!C::SPLIT) {
    setmaxnreg_dec<RegSplit<DP, EPI>::kEpi>();
    // ================================================================ epilogue (both tiles)
    // The only role that touches global memory other than Q, K, V: when launched as a dependent of
    // the previous ring step, wait here for that grid to complete (returns at once otherwise).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int row = threadIdx.x & 127;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    int it_all = 0;
    bool ok = true;
    for (int k = 0; ok && k * static_cast<int>(gridDim.x) < n_items; ++k) {
        const int idx = item_of_cta(k);
        if (idx >= n_items) continue;
      Item it;
      bool has_o;
      if (C::P_SEP) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_plan_full + (it_all & 1), (it_all >> 1) & 1, ctl, 0x403));
        if (!ok) break;
        it = plan[it_all & 1].it;
        has_o = plan[it_all & 1].n > 0;
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_plan_empty + (it_all & 1));
      } else {
        decode_item(w, idx, it);
        Walk wk;
        has_o = walk_begin<WIN, C::BN>(wk, w, it, n_steps);
      }
      for (int q = 0; q < 2; ++q) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_o_full + q, it_all & 1, ctl, 0x401) &&
                                         mbar_wait(bar_stats + q, it_all & 1, ctl, 0x402));
        if (!ok) break;
        tc_fence_after();
        const float2 ml = stats[q * 128 + row];
        const bool row_ok = row < it.rows_valid[q];
        const int t = it.t0 + 128 * q + row;
        fmha_epilogue_row<C, EPI>(w, it, t, row_ok, has_o, ml, lane_addr + C::O_COL0 + C::O_STRIDE * q);
        tc_fence_before();
        mbar_arrive(bar_o_empty + q);
      }
      ++it_all;
    }
   }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace ra
