// ra_common.cuh - device-side building blocks shared by the kernels of the library:
// shared-memory barriers with bounded waits, TMA tile loads, tcgen05 (5th-generation tensor
// core) issue / commit / tensor-memory access, and the LSE merge arithmetic.
//
// All PTX below is written for sm_100a from the PTX ISA's descriptions of mbarrier,
// cp.async.bulk.tensor and tcgen05.  Nothing here spins without a limit: every wait on a
// barrier gives up after a globaltimer deadline, latches an error in the device status word,
// and raises the CTA's abort flag so the other roles stop too.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ra {

// ---------------------------------------------------------------------------------------------
// Device status word (read and cleared by ra_get_device_status)
// ---------------------------------------------------------------------------------------------
enum : unsigned {
  kDevStatusTimeout = 1u,
};
// The word lives in the library's main translation unit; kernels receive its address
// (word 0: OR of kDevStatus* flags, word 1: site id of the first wait that gave up).

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of the phase with `parity`.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Per-CTA control block for bounded waits.
struct WaitCtl {
  volatile int* abort;   // shared-memory flag: some wait in this CTA gave up
  uint64_t limit_ns;     // per-wait limit
  unsigned int* status;  // device status word (2 x u32)
};

// Wait until the phase with `parity` of `bar` has completed.  Returns false (and raises the
// CTA abort flag) if the wait ran out or another role already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtl& ctl, unsigned site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
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

// ---------------------------------------------------------------------------------------------
// TMA (tensor copies global -> shared, completion counted in bytes on an mbarrier)
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 5-D tiled load; coordinates innermost first.  Out-of-range elements are filled with zero.
__device__ __forceinline__ void tma_load_5d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_addr(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(smem_addr(bar))
      : "memory");
}

// ---------------------------------------------------------------------------------------------
// tcgen05: tensor memory allocation, MMA issue, commit, loads/stores, fences
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(smem_result)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// Warp-collective: thread i of the warp reads 32 consecutive 32-bit columns of TMEM lane
// (lane field of taddr) + i.  The values are valid only after tmem_ld_wait().
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// Wait for this thread's outstanding tcgen05.ld, and make `r` depend on the wait so that no use
// of the loaded registers can be scheduled before it.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

// As tmem_ld32 for 16 consecutive columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15])
               :
               : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
      "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]),
      "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// 64 consecutive 32-bit columns of the thread's lane in one instruction.
__device__ __forceinline__ void tmem_st64(uint32_t taddr, const uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]), "r"(r[32]), "r"(r[33]), "r"(r[34]), "r"(r[35]), "r"(r[36]), "r"(r[37]), "r"(r[38]), "r"(r[39]), "r"(r[40]), "r"(r[41]), "r"(r[42]), "r"(r[43]), "r"(r[44]), "r"(r[45]), "r"(r[46]), "r"(r[47]), "r"(r[48]), "r"(r[49]), "r"(r[50]), "r"(r[51]), "r"(r[52]), "r"(r[53]), "r"(r[54]), "r"(r[55]), "r"(r[56]), "r"(r[57]), "r"(r[58]), "r"(r[59]), "r"(r[60]), "r"(r[61]), "r"(r[62]), "r"(r[63])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------------------------
// Descriptors (bit layouts from the PTX ISA, "Shared memory descriptor" / "Instruction
// descriptor" of tcgen05.mma)
// ---------------------------------------------------------------------------------------------
enum SwizzleMode : uint32_t { kSwizzleNone = 0, kSwizzle128B = 2, kSwizzle64B = 4, kSwizzle32B = 6 };

// Shared-memory matrix descriptor: start address, leading / stride byte offsets (all >> 4),
// descriptor version 1 (bits 46-47), base offset 0, swizzle mode in bits 61-63.
__device__ __forceinline__ uint64_t make_smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                                   uint32_t swizzle) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(swizzle & 7u) << 61;
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 D.
// a_mn_major / b_mn_major: 0 = K-major, 1 = MN-major.
__host__ __device__ constexpr uint32_t make_idesc_bf16(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4)                                     // D format: f32
         | (1u << 7)                                   // A format: bf16
         | (1u << 10)                                  // B format: bf16
         | (static_cast<uint32_t>(a_mn_major) << 15)   // A major
         | (static_cast<uint32_t>(b_mn_major) << 16)   // B major
         | (static_cast<uint32_t>(N >> 3) << 17)       // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);      // M / 16
}

// ---------------------------------------------------------------------------------------------
// LSE merge arithmetic (gitcode page, §2.2 phase 3; exponent sign corrected)
// ---------------------------------------------------------------------------------------------
// L = max(a,b) + log1p(e^{-|a-b|}); w_a = e^{a-L}, w_b = e^{b-L}.  -inf is the empty partial.
__device__ __forceinline__ void lse_merge_weights(float la, float lb, float& L, float& wa, float& wb) {
  const float hi = fmaxf(la, lb);
  const float lo = fminf(la, lb);
  if (hi == -INFINITY) {
    L = -INFINITY;
    wa = 0.f;
    wb = 0.f;
    return;
  }
  L = hi + log1pf(expf(lo - hi));
  wa = expf(la - L);
  wb = expf(lb - L);
}

__device__ __forceinline__ void lse_merge_weights(double la, double lb, double& L, double& wa, double& wb) {
  const double hi = fmax(la, lb);
  const double lo = fmin(la, lb);
  if (hi == -INFINITY) {
    L = -INFINITY;
    wa = 0.0;
    wb = 0.0;
    return;
  }
  L = hi + log1p(exp(lo - hi));
  wa = exp(la - L);
  wb = exp(lb - L);
}

// ---------------------------------------------------------------------------------------------
// Work description shared by the attention kernels
// ---------------------------------------------------------------------------------------------
// A launch covers query shards r = r_first + i * r_step (i < n_r) of B*H heads.  For query shard
// r at ring step t the KV shard is s = (r - t) mod P (P = 1 for a single pass or one explicit
// partial).  Local query token t_q of shard r sits at global position
//   q_off + r * q_rstep + t_q * q_tstride
// and local key u of shard s at k_off + s * k_sstep + u * k_ustride.
enum EpilogueMode : int {
  kEpiOut = 0,     // write O (input dtype) and LSE to the output
  kEpiPart = 1,    // write the fp32 partial (O, LSE) to the accumulator
  kEpiAcc = 2,     // merge into the fp32 accumulator in place
  kEpiAccOut = 3,  // merge with the fp32 accumulator and write the result to the output
};

// Division by a divisor fixed for the launch, as a multiply and shift (Granlund and Montgomery,
// "Division by invariant integers using multiplication", 1994): with s = ceil(log2 d) and
// m = ceil(2^(32+s) / d), floor(n / d) = (n * m) >> (32 + s) exactly for 0 <= n < 2^31 (the
// rounding error n * (m * d - 2^(32+s)) / (d * 2^(32+s)) stays below 1/d).  The kernel's
// per-item index arithmetic uses it because the hardware integer divide sequence goes through
// the MUFU unit, which the softmax keeps saturated with exponentials.
struct FastDiv {
  unsigned long long m;
  unsigned int d;
  unsigned int s;
};

inline FastDiv make_fastdiv(unsigned int d) {  // host side; d >= 1
  FastDiv f;
  f.d = d;
  f.s = 0;
  while ((1ull << f.s) < d) ++f.s;
  f.m = ((1ull << (32 + f.s)) + d - 1) / d;
  return f;
}

__host__ __device__ __forceinline__ int fdiv(int n, const FastDiv& f) {  // 0 <= n < 2^31
  return static_cast<int>((static_cast<unsigned long long>(n) * f.m) >> (32 + f.s));
}
__host__ __device__ __forceinline__ int fmod_(int n, const FastDiv& f) {
  return n - fdiv(n, f) * static_cast<int>(f.d);
}

struct AttnWork {
  int B;          // batch
  int r_major;    // work-item order: 1 = query shards outermost (contiguous shards), 0 = blocks
  int tile_major; // K/V walk of a multi-step launch: 1 = tile index outermost, the shards inside
  int hgroup;     // heads per item group (the group's K/V is sized to stay resident in L2)
  int n_q;        // query tokens per shard
  int n_kv;       // key tokens per shard
  int H;          // heads (of Q, O and LSE)
  int H_kv;       // heads of K and V: query head h reads K/V head h / (H / H_kv) (GQA; MQA: 1)
  int d;          // head dim
  int P;          // shards in the ring (1 for a single pass / explicit partial)
  int n_q_tiles;  // ceil(n_q / 128) (tensor-core path) or ceil(n_q / rows per CTA)
  int r_first, r_step, n_r;
  int ring_step;  // t
  int causal;
  long long window;  // sliding window (causal only): keys at positions > pos_q - window; 0 = none
  long long q_off, q_rstep, q_tstride;
  long long k_off, k_sstep, k_ustride;
  float scale;       // softmax scale applied to q.k
  float scale_log2;  // scale * log2(e)
  // Raw pointers / strides (elements) of the operands, used by the SIMT path (the tensor-core
  // path reads through TMA maps).  Shard r's token t_q is row (r * x_rs + t_q * x_ts).
  const void* q;
  const void* k;
  const void* v;
  long long q_sb, q_sh, q_rs, q_ts;
  long long k_sb, k_sh, k_rs, k_ts;
  long long v_sb, v_sh, v_rs, v_ts;
  // Output (dtype of the inputs) and LSE output; row (b, h, r, t_q).
  void* o;
  long long o_sb, o_sh, o_rs, o_ts;
  float* lse;  // may be null
  long long l_sb, l_sh, l_rs, l_ts;
  // fp32 accumulator (partial / accumulate modes).
  float* acc_o;
  long long a_sb, a_sh, a_rs, a_ts;
  float* acc_l;
  long long al_sb, al_sh, al_rs, al_ts;
  unsigned long long wait_limit_ns;
  unsigned int* dev_status;
  // Fast dividers (set at launch): items per head group, heads per group, heads of the last group,
  // 256-row blocks per shard, query shards, heads, ring size, key position stride.
  FastDiv fd_grp, fd_hg, fd_hg_last, fd_nblk, fd_nr, fd_H, fd_P, fd_kus;
  FastDiv fd_qpk;  // query heads per K/V head (H / H_kv)
};

// Number of keys u in [0, n_kv) of shard s that are visible to a query at global position
// pos_q: all of them if not causal, else those with k_off + s*k_sstep + u*k_ustride <= pos_q.
// (k_ustride >= 1.)  The quotient avoids the divide instruction sequence whenever the operands
// fit: every role of the attention kernel evaluates this at each work item's start, on the item's
// critical path.
__host__ __device__ __forceinline__ int visible_key_limit(const AttnWork& w, long long pos_q, int s) {
  if (!w.causal) return w.n_kv;
  const long long base = w.k_off + static_cast<long long>(s) * w.k_sstep;
  if (pos_q < base) return 0;
  const unsigned long long diff = static_cast<unsigned long long>(pos_q - base);
  const unsigned long long stride = static_cast<unsigned long long>(w.k_ustride);
  unsigned long long quot;
  if (stride == 1)
    quot = diff;
  else if ((diff >> 31) == 0 && stride == w.fd_kus.d)
    quot = static_cast<unsigned long long>(fdiv(static_cast<int>(diff), w.fd_kus));
  else
    quot = diff / stride;
  return quot < static_cast<unsigned long long>(w.n_kv) ? static_cast<int>(quot) + 1 : w.n_kv;
}

// First key u of shard s inside the sliding window of a query at global position pos_q: the keys
// at positions pos_q - window + 1 ... pos_q (the window's most recent positions, the query's own
// included; vibe-research page, "Sliding Window Attention": each token attends to the w most
// recent tokens).  0 without a window.  (k_ustride >= 1.)
__host__ __device__ __forceinline__ int visible_key_start(const AttnWork& w, long long pos_q, int s) {
  if (w.window <= 0) return 0;
  const long long base = w.k_off + static_cast<long long>(s) * w.k_sstep;
  const long long first = pos_q - w.window + 1;  // first visible position
  if (first <= base) return 0;
  const unsigned long long diff = static_cast<unsigned long long>(first - base);  // > 0
  const unsigned long long stride = static_cast<unsigned long long>(w.k_ustride);
  unsigned long long quot;  // ceil(diff / stride)
  if (stride == 1)
    quot = diff;
  else if (((diff + stride - 1) >> 31) == 0 && stride == w.fd_kus.d)
    quot = static_cast<unsigned long long>(fdiv(static_cast<int>(diff + stride - 1), w.fd_kus));
  else
    quot = (diff + stride - 1) / stride;
  return quot < static_cast<unsigned long long>(w.n_kv) ? static_cast<int>(quot) : w.n_kv;
}

// (r - t) mod P for 0 <= r < P, 0 <= t < 2P (the launch keeps ring_step + steps <= 2P).
__host__ __device__ __forceinline__ int ring_shard(const AttnWork& w, int r, int t) {
  return fmod_(r - t + 2 * w.P, w.fd_P);
}

}  // namespace ra
