/*
 * ra_attn.h - C ABI of the B200 (sm_100a) blockwise / ring softmax attention library.
 *
 * What is computed (all entry points): exact softmax attention of one or more heads,
 *
 *     O = softmax(scale * Q K^T) V,      LSE_i = ln sum_j exp(scale * q_i . k_j),
 *
 * over tensors laid out as [B, H, N, d] (intelliparadigm.com, "Mosaic多轴注意力分片：突破
 * Transformer长序列处理瓶颈", §2.1: Attention(Q,K,V) = softmax(QK^T/sqrt(d))V; intelliparadigm.com,
 * "深度学习注意力机制优化与FlashAttention实践", §2.1).  It is computed blockwise with an online
 * softmax: per query tile, K/V tiles stream past and a running per-row max m and sum s are
 * updated (same FlashAttention page, §4.2; vibe-research.pages.dev, "架构层解决方案 - Sparse
 * Attention与Ring Attention", section "Ring Attention", the blockwise identity).  A ring shard's
 * partial result is the pair (O_partial, LSE), and two partials over disjoint key sets combine by
 * the log-sum-exp rule LSE(a,b) = max(a,b) + log(1 + e^{-|a-b|}) (blog.gitcode.com,
 * "分布式注意力机制突破：长序列处理的全景技术架构与实践指南", §2.2 phase 3 - printed there with
 * the sign of the exponent wrong - and §3.4 for the M-way form).
 *
 * Conventions shared by every call
 *  - Natural-log LSE of the *scaled* scores.  A query row with no visible key gets O = 0 and
 *    LSE = -inf; merging with such a partial is the identity.
 *  - Causal masking uses global token positions: key j is visible to query i iff
 *    pos(j) <= pos(i).  A shard's local token t sits at global position offset + t * stride
 *    (ra_pos_t), which covers both ring layouts: contiguous shard r = tokens [r*n, (r+1)*n);
 *    striped shard r = tokens r, r+P, r+2P, ... (Striped Attention, git.kang-kang.com,
 *    "注意力机制演进", timeline).
 *  - Ownership: the caller allocates every buffer (device memory for tensor data, LSE and the
 *    ring workspace) and every stream.  No entry point allocates device memory.
 *  - Asynchrony: every compute call only enqueues work on the given stream(s) and returns.  The
 *    return value reports argument and launch errors.  Faults detected on the device (a bounded
 *    wait that ran out) are latched in a device status word read by ra_get_device_status().
 *  - Errors never abort the process, and ra_last_error() returns a message for the calling thread.
 *    On a non-RA_OK return no kernel has been enqueued: every argument, shape and index limit is
 *    checked before the first launch.  The one exception is RA_ERR_CUDA from the CUDA runtime
 *    refusing a kernel launch in the middle of a multi-launch ring call (ra_ring_fwd and its
 *    variants): the launches before it stay queued, and streams[0] is still ordered after them.
 *  - Device pointers must belong to the current CUDA device.
 *  - Stream order holds as usual: work enqueued after a call, with an ordinary launch or copy,
 *    starts after all of the call's work.  Inside a call, later steps of the stepwise ring and the
 *    dK/dV half of the backward are launched as programmatic dependents of the kernel before them
 *    (they start on SMs that kernel leaves idle and wait for it before touching its outputs); the
 *    library's kernels signal dependents at their start, so a kernel of the caller's that is itself
 *    launched as a programmatic dependent of a library call must wait for its grid dependency
 *    before reading the call's outputs, as with any such launch.
 *
 * Supported inputs
 *  - dtype RA_BF16 (tensor-core path, fp32 accumulation, bf16 output): head dim d a multiple of 8
 *    with d <= 128; every stride except stride[3] a multiple of 8 elements (16 bytes, TMA);
 *    data pointer 16-byte aligned; stride[3] == 1.
 *  - dtype RA_F32 (SIMT path, fp32 arithmetic, row sums in fp64): d <= 128, stride[3] == 1.
 *  - B, H, N < 2^31; N of every tensor >= 1.
 */
#ifndef RA_ATTN_H
#define RA_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Binary-compatible with cudaStream_t / CUstream (NULL = the legacy default stream). */
typedef struct CUstream_st* ra_stream_t;

typedef enum {
  RA_OK = 0,
  RA_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, mismatched tensors, bad enum value */
  RA_ERR_UNSUPPORTED = 2,  /* valid request the library cannot run (dtype, head dim, no sm_100) */
  RA_ERR_ALIGNMENT = 3,    /* pointer or stride violates the 16-byte rule of the bf16 path */
  RA_ERR_WORKSPACE = 4,    /* ring workspace missing or smaller than ra_ring_workspace_size */
  RA_ERR_CUDA = 5,         /* a CUDA runtime/driver call failed (message in ra_last_error) */
  RA_ERR_TIMEOUT = 6       /* a device-side bounded wait ran out (from ra_get_device_status) */
} ra_status_t;

typedef enum { RA_F32 = 0, RA_BF16 = 1 } ra_dtype_t;

typedef enum { RA_CONTIGUOUS = 0, RA_STRIPED = 1 } ra_layout_t;

/* Ring schedules of ra_ring_fwd.
 *  RA_RING_STEPWISE: P ring steps; at step t every query shard r meets KV shard (r - t) mod P in
 *    one launch per (step, stream), and the step's partial is merged into an fp32 (O, LSE)
 *    accumulator held in the caller's workspace by the LSE rule (the single-GPU image of P
 *    devices each doing step t).  Pairs whose keys are all in the causal future are skipped.
 *  RA_RING_FUSED: one launch; each query tile walks the KV shards in the same ring order and
 *    merges each shard's partial into an on-chip accumulator with the same (m, s) rule, so no
 *    partial result goes through HBM.  Needs no workspace. */
typedef enum { RA_RING_STEPWISE = 0, RA_RING_FUSED = 1 } ra_ring_schedule_t;

/* A strided 4-D tensor [B, H, N, d] in device memory.  stride[] is in elements (not bytes);
 * stride[3] must be 1.  Any other strides are allowed (e.g. a head-split view of
 * [batch, rows, features, embed] with stride[1] = head_dim and stride[2] = features*embed). */
typedef struct {
  void* data;
  int32_t dtype; /* ra_dtype_t */
  int32_t reserved;
  int64_t shape[4];
  int64_t stride[4];
} ra_tensor_t;

/* Grouped-query / multi-query attention: in every call below, k and v may have H_kv heads
 * instead of H (shape[1] = H_kv for both, H_kv dividing the query heads H of q).  Query head h
 * then attends with K/V head h / (H / H_kv): consecutive groups of H / H_kv query heads share one
 * K/V pair (vibe-research page, "MQA与GQA" section; H_kv = H is multi-head attention, H_kv = 1
 * multi-query attention).  o and lse always have the H heads of q.  k and v with different head
 * counts, or an H_kv that does not divide H, return RA_ERR_INVALID_ARG. */

/* Global position of local token t: offset + t * stride (stride >= 1). */
typedef struct {
  int64_t offset;
  int64_t stride;
} ra_pos_t;

/* Single full pass (ring with P = 1).
 * q [B,H,Nq,d]; k, v [B,H,Nk,d] (or [B,H_kv,Nk,d], see above); o [B,H,Nq,d] with
 * o->dtype == q->dtype (bf16 in -> bf16 out, fp32 in -> fp32 out); lse: fp32 [B,H,Nq] contiguous, may be NULL.  scale <= 0 selects
 * 1/sqrt(d).  causal != 0: query i and key j both sit at position = index (0-based), key j is
 * visible iff j <= i.  o must not overlap q, k or v. */
ra_status_t ra_attn_fwd(const ra_tensor_t* q, const ra_tensor_t* k, const ra_tensor_t* v,
                        const ra_tensor_t* o, float* lse, float scale, int causal,
                        ra_stream_t stream);

/* Sliding-window attention (vibe-research page, "Sliding Window Attention": each token attends
 * only to the w most recent tokens; only the mask changes).  As ra_attn_fwd with causal = 1, and
 * key j is visible to query i iff i - window < j <= i: the window's most recent positions, the
 * query's own included (window = 1: each token attends to itself only; window >= Nk: plain
 * causal).  window < 1 returns RA_ERR_INVALID_ARG.  (Extension beyond the calls the pages' ring
 * method needs.) */
ra_status_t ra_attn_fwd_window(const ra_tensor_t* q, const ra_tensor_t* k, const ra_tensor_t* v,
                               const ra_tensor_t* o, float* lse, float scale, int64_t window,
                               ra_stream_t stream);

/* One ring step: the partial attention of a query shard against one KV shard.
 * k_shard, v_shard hold the shard's keys/values (any strided view, e.g. every P-th row of the
 * full K for the striped layout).  q_pos / kv_pos give the global positions used by the causal
 * mask (ignored when causal == 0).
 * Output: o_part, an fp32 tensor [B,H,Nq,d] (stride[3] == 1), and lse_part, fp32 [B,H,Nq]
 * contiguous.  O_part is normalised over the shard's visible keys.
 * accumulate == 0: (o_part, lse_part) are overwritten with this shard's partial.
 * accumulate != 0: (o_part, lse_part) must hold a previous partial of the same query rows over
 *   disjoint keys; it is replaced by the LSE merge of the two (gitcode page, §2.2 phase 3).
 * Rows whose keys are all in the future get O = 0, LSE = -inf (or are left unchanged when
 * accumulating, since merging with an empty partial is the identity). */
ra_status_t ra_attn_partial(const ra_tensor_t* q, const ra_tensor_t* k_shard,
                            const ra_tensor_t* v_shard, ra_pos_t q_pos, ra_pos_t kv_pos,
                            int causal, float scale, const ra_tensor_t* o_part, float* lse_part,
                            int accumulate, ra_stream_t stream);

/* Pairwise LSE merge of two partials of the same rows (gitcode page, §2.2 phase 3):
 *   LSE = max(la, lb) + log1p(exp(-|la - lb|)),  O = e^{la - LSE} O_a + e^{lb - LSE} O_b.
 * o_a, o_b, o_out: fp32 [rows, d] row-major contiguous; lse_*: fp32 [rows].  The outputs may
 * alias either input exactly (in-place accumulate); partial overlap is not allowed.
 * rows >= 0 (0 is a no-op), 1 <= d <= 4096.  Bound by HBM bandwidth. */
ra_status_t ra_lse_merge(const float* o_a, const float* lse_a, const float* o_b,
                         const float* lse_b, float* o_out, float* lse_out, int64_t rows, int d,
                         ra_stream_t stream);

/* M-way merge in one pass (gitcode page, §3.4): m = max_i LSE_i, s = sum_i e^{LSE_i - m},
 * LSE = m + ln s, O = sum_i e^{LSE_i - m} O_i / s.
 * o_parts, lse_parts: HOST arrays of k DEVICE pointers (read during the call only), each
 * [rows, d] / [rows] fp32 contiguous.  1 <= k <= RA_MERGE_MAX_PARTS.  The outputs may alias
 * o_parts[0] / lse_parts[0] exactly. */
#define RA_MERGE_MAX_PARTS 32
ra_status_t ra_lse_merge_n(const float* const* o_parts, const float* const* lse_parts, int k,
                           float* o_out, float* lse_out, int64_t rows, int d,
                           ra_stream_t stream);

/* Backward pass (extension beyond the forward path the pages' ring method needs): gradients of
 * L = sum(d_o * O) with respect to q, k, v for O = ra_attn_fwd(q, k, v, ..., scale, causal) (or
 * ra_attn_fwd_window with window > 0), with the attention weights recomputed from the forward's
 * saved lse instead of stored (intelliparadigm.com "深度学习注意力机制优化与FlashAttention实践",
 * §3.3 and §4.1 item 3).  With P = e^{scale q k^T - lse} on visible entries:
 *   dv = P^T d_o,  dS = P * (d_o v^T - rowsum(d_o * o)),  dq = scale dS k,  dk = scale dS^T q.
 * q [B,H,Nq,d], k, v [B,H_kv,Nk,d] (grouped-query K/V: dk, dv sum over each group), o and d_o
 * [B,H,Nq,d] of q's dtype (o the forward's output), lse fp32 [B,H,Nq] contiguous (the forward's),
 * dq fp32 [B,H,Nq,d], dk, dv fp32 [B,H_kv,Nk,d]; all overwritten.  scale <= 0 selects 1/sqrt(d).
 * window: 0, or with causal the forward's sliding window.  The backward of ra_ring_fwd (either
 * layout or schedule) is this call on the same full tensors: the ring computes the same function
 * of global positions.
 * bf16 inputs whose q, k, v, o, d_o satisfy the forward's TMA rules (16-byte aligned base,
 * strides multiples of 8 elements, d % 8 == 0) run on the tensor cores: P and dS are rounded to
 * bf16 before the products dv = P^T d_o, dk = dS^T q, dq = dS k (fp32 accumulation), so each
 * gradient element errs by at most ~2^-8 times the same sums taken over absolute values.
 * fp32 inputs (and bf16 tensors outside those rules) use fp32 SIMT kernels.  Two launches on
 * `stream`, no workspace.  Errors: RA_ERR_INVALID_ARG for shape / dtype / window mismatches. */
ra_status_t ra_attn_bwd(const ra_tensor_t* q, const ra_tensor_t* k, const ra_tensor_t* v,
                        const ra_tensor_t* o, const float* lse, const ra_tensor_t* d_o,
                        const ra_tensor_t* dq, const ra_tensor_t* dk, const ra_tensor_t* dv,
                        float scale, int causal, int64_t window, ra_stream_t stream);

/* Workspace bytes ra_ring_fwd needs for (q, P, schedule): 0 for RA_RING_FUSED; for
 * RA_RING_STEPWISE an fp32 accumulator of B*H*N*(d+1)*4 bytes (plus alignment). */
ra_status_t ra_ring_workspace_size(const ra_tensor_t* q, int P, int schedule, size_t* bytes);

/* Ring attention over P virtual sequence shards on one GPU (vibe-research page, "Ring
 * Attention" sequence diagram; intelliparadigm.com "Mosaic…", §3.2: KV blocks rotate, Q stays,
 * GPU r at step t uses the KV shard that started on GPU (r - t) mod P).
 * q, k, v [B,H,N,d] (k, v may have H_kv heads) of one dtype with N % P == 0; the shards are
 * views, nothing is copied:
 *   layout RA_CONTIGUOUS: shard r = tokens [r*N/P, (r+1)*N/P);
 *   layout RA_STRIPED:    shard r = tokens r, r+P, r+2P, ... (token i on shard i mod P).
 * o [B,H,N,d] (dtype of q), lse fp32 [B,H,N] contiguous (may be NULL).  Positions are the
 * global token indices, so the result equals ra_attn_fwd(q, k, v, o, lse, scale, causal) up to
 * rounding, for either layout.
 * streams: n_streams >= 1 caller-owned streams (query shards are dealt round-robin over them;
 * work for one shard stays on one stream).  The call orders itself after work already queued on
 * streams[0] and, on return, all its work is ordered before later work on streams[0].
 * workspace: device memory of at least ra_ring_workspace_size() bytes, 256-byte aligned (may be
 * NULL when that size is 0).  It must not be used by other work until the call's work is done. */
ra_status_t ra_ring_fwd(const ra_tensor_t* q, const ra_tensor_t* k, const ra_tensor_t* v, int P,
                        int layout, int causal, float scale, int schedule,
                        const ra_tensor_t* o, float* lse, const ra_stream_t* streams,
                        int n_streams, void* workspace, size_t workspace_bytes);

/* ra_ring_fwd with a causal sliding window of `window` positions (as ra_attn_fwd_window, on
 * global token positions, either layout, either schedule).  window < 1 returns
 * RA_ERR_INVALID_ARG.  Shard pairs and key tiles wholly outside every row's window are skipped. */
ra_status_t ra_ring_fwd_window(const ra_tensor_t* q, const ra_tensor_t* k, const ra_tensor_t* v, int P,
                               int layout, int64_t window, float scale, int schedule,
                               const ra_tensor_t* o, float* lse, const ra_stream_t* streams,
                               int n_streams, void* workspace, size_t workspace_bytes);

/* ra_ring_fwd for inputs and outputs that live in host memory, with the transfers overlapped with
 * the computation.  There is no counterpart on the source pages: this is an interface convenience
 * of this library, for callers whose tensors are host-resident (and, on the pages' multi-device
 * ring, for a rank that receives its shards from the host).
 * The flattened B*H_kv heads are split into n_chunks chunks (fewer when there are fewer heads);
 * chunk c's query, key and value heads go host -> device on streams[0], its ring runs (fused
 * schedule) on streams[1] as soon as they have landed, and its O and LSE go device -> host on
 * streams[2] as soon as it is done, so chunk c+1's copies in and chunk c-1's copies out overlap
 * chunk c's kernels.  Attention is independent per head, so the result equals ra_ring_fwd on the
 * whole tensors.
 * q_host, k_host, v_host, o_host: contiguous [B,H,N,d] (k, v: [B,H_kv,N,d]) tensors in host memory;
 * page-locked memory is needed for the copies to overlap (pageable memory gives the same result,
 * without the overlap).  q_dev .. o_dev: device tensors of the same shapes and dtypes, contiguous
 * (caller-allocated staging; every chunk has its own region, nothing is reused within the call).
 * lse_host, lse_dev: fp32 [B,H,N], both given or both NULL.  streams: three distinct caller-owned
 * streams (copy in, compute, copy out).  The call orders itself after work already queued on
 * streams[1]; on return every part of it, the copies out included, is ordered before later work
 * on streams[1], so synchronising streams[1] makes o_host and lse_host valid.  Every check runs
 * before anything is enqueued; RA_ERR_CUDA from a failed copy or launch in the middle leaves the
 * earlier chunks queued.  Other arguments and errors as for ra_ring_fwd. */
ra_status_t ra_ring_fwd_host(const ra_tensor_t* q_host, const ra_tensor_t* k_host, const ra_tensor_t* v_host, int P,
                             int layout, int causal, float scale, const ra_tensor_t* o_host, float* lse_host,
                             const ra_tensor_t* q_dev, const ra_tensor_t* k_dev, const ra_tensor_t* v_dev,
                             const ra_tensor_t* o_dev, float* lse_dev, int n_chunks, const ra_stream_t* streams);

/* ra_ring_fwd with the RA_RING_STEPWISE schedule for callers that cannot allocate device memory
 * at the point of the call: code inside a host application whose caching allocator already holds
 * all device memory and offers no scratch interface, services that fix their memory budget at
 * start-up and allow no allocation afterwards, and latency-critical paths that must not pay for
 * the implicit device-wide synchronisation of cudaMalloc / cudaFree.  There is no counterpart on
 * the source pages: this is an interface convenience of this library.
 * The fp32 (O, LSE) accumulator lives in a fixed array of RA_NOALLOC_SCRATCH_BYTES inside the
 * library (held on every device that loads the library, until the process exits); nothing is
 * allocated.  Problems whose accumulator (ra_ring_workspace_size with RA_RING_STEPWISE) exceeds
 * that size are rejected with RA_ERR_WORKSPACE and a message naming both sizes.
 * Set-up: the first call on each device (and again the first call after the device's context has
 * been torn down and recreated, e.g. by cudaDeviceReset) looks up the array's device address with
 * that device current; make that first call before any stream capture.  All calls on a device
 * share the one array: calls whose work overlaps on the GPU (different streams, or interleaved
 * with ra_ring_fwd_noalloc calls on other threads) race on it, so order them on one stream.  The
 * array keeps the last call's contents; no clearing is needed because ring step 0 overwrites
 * every element the later steps read.  Other arguments and errors as for ra_ring_fwd (one
 * stream). */
#define RA_NOALLOC_SCRATCH_BYTES (32u << 20)
ra_status_t ra_ring_fwd_noalloc(const ra_tensor_t* q, const ra_tensor_t* k, const ra_tensor_t* v, int P,
                                int layout, int causal, float scale, const ra_tensor_t* o, float* lse,
                                ra_stream_t stream);

/* Synchronises `stream`, then reads and clears the device status word that kernels set when a
 * bounded wait runs out (each wait gives up after ra_set_wait_timeout_ns(); the kernel then
 * stops its work, frees its tensor memory and returns, leaving its outputs undefined).
 * Returns RA_OK, RA_ERR_TIMEOUT, or RA_ERR_CUDA if the synchronisation itself failed. */
ra_status_t ra_get_device_status(ra_stream_t stream);

/* Limit of every device-side wait, in nanoseconds (default 2e9).  Applies to later launches. */
ra_status_t ra_set_wait_timeout_ns(uint64_t ns);

/* Order in which a launch that covers several ring steps (the fused schedule) walks the key/value
 * tiles of STRIPED shards, for head dims padded to 128 (the 64-key-tile kernels):
 *   RA_WALK_SHARD_MAJOR (0, default): every tile of one shard, then the next shard;
 *   RA_WALK_TILE_MAJOR  (1): tile u of every shard, then tile u + 1.
 * Striped shards interleave their keys in memory (key u of shard s sits at position u * P + s),
 * so the tile-major order reads each stretch of K/V once per work item instead of once per shard:
 * on one B200, B=1 H=32 N=32768 d=128 P=8 causal reads 1.8 instead of 6.7 GB of DRAM per launch,
 * but runs 2-3 % slower.  Either order visits the same tiles (results equal within
 * rounding).  Contiguous shards, other head dims and one-step launches ignore the setting.
 * Process-wide; applies to later calls.  Returns RA_ERR_INVALID_ARG for any other value. */
#define RA_WALK_SHARD_MAJOR 0
#define RA_WALK_TILE_MAJOR 1
ra_status_t ra_set_striped_walk(int order);

/* Diagnostic: enqueue one single-CTA kernel whose threads wait on a shared-memory barrier that
 * nothing ever arrives at, with the given limit.  The wait must give up and latch
 * RA_ERR_TIMEOUT in the device status word; the kernel then returns normally.  Used to test the
 * failure path without faulting or hanging the device. */
ra_status_t ra_debug_unarrived_wait(uint64_t timeout_ns, ra_stream_t stream);

/* Diagnostic: evaluate the two device exp2 routines of the attention kernel on n inputs (device
 * arrays): y_poly[i] = the FMA-pipe polynomial 2^x (range reduction to [-1/2, 1/2] plus a degree-3
 * minimax polynomial, max relative error 7.5e-5, inputs clamped at -126) and y_mufu[i] = the
 * hardware ex2.approx.  Either output may be NULL.  Lets a test check both against their error
 * bounds. */
ra_status_t ra_debug_exp2(const float* x, float* y_poly, float* y_mufu, int64_t n, ra_stream_t stream);

const char* ra_status_string(ra_status_t status);

/* Message describing the last non-RA_OK return on the calling thread ("" if none). */
const char* ra_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
int ra_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RA_ATTN_H */
