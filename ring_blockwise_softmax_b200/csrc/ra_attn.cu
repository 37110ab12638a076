// ra_attn.cu - the C ABI declared in include/ra_attn.h: argument checks, TMA descriptor
// encoding, kernel launches, the ring driver, and the device status word.
//
// Host code only marshals work to the kernels; every arithmetic step of the method runs on the
// GPU.  Nothing here allocates device memory: buffers and streams come from the caller.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>
#include <vector>

#include "ra_attn.h"
#include "ra_attn_simt.cuh"
#include "ra_fmha_sm100.cuh"
#include "ra_internal.h"
#include "ra_lse_merge.cuh"
#include "ra_attn_bwd.cuh"
#include "ra_bwd_sm100.cuh"

namespace ra {
// Device status word: [0] OR of kDevStatus* flags, [1] site of the first wait that gave up.
__device__ unsigned int g_dev_status[2];

// A shared-memory barrier that nothing arrives at: the bounded wait must give up.
__global__ void unarrived_wait_kernel(unsigned long long limit_ns, unsigned int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  WaitCtl ctl{&abort_flag, limit_ns, status};
  (void)mbar_wait(&bar, 0, ctl, 0x901);
}
__global__ void exp2_probe_kernel(const float* x, float* y_poly, float* y_mufu, long long n) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float v = x[i];
    if (y_poly) y_poly[i] = exp2_poly3(v);
    if (y_mufu) y_mufu[i] = ex2_approx(v);
  }
}
}  // namespace ra

namespace {

constexpr int kVersion = 10000;  // 1.0.0
constexpr double kLog2e = 1.4426950408889634;
// Walk order of multi-step launches over striped shards (ra_set_striped_walk): 1 = K/V tile
// index first, the shards inside.  That order reads 3.4x fewer DRAM bytes on a striped d = 128
// ring (1.8 instead of 6.7 GB at B=1 H=32 N=32768 P=8) but runs 2.7 % slower under the power cap,
// so the shard-major walk is the default.
std::atomic<int> g_striped_walk{RA_WALK_SHARD_MAJOR};

thread_local std::string t_last_error;
std::atomic<unsigned long long> g_wait_limit_ns{2000000000ull};

ra_status_t fail(ra_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return st;
}

ra_status_t ok() {
  t_last_error.clear();
  return RA_OK;
}

ra_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(RA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// ------------------------------------------------------------------------------------------
// Device / argument checks
// ------------------------------------------------------------------------------------------
struct DevInfo {
  int major = -1, minor = -1, sms = 0;
  unsigned int* status = nullptr;  // device address of ra::g_dev_status in the context below
  unsigned long long ctx = 0;      // context the address was looked up in
};
std::mutex g_dev_mu;
DevInfo g_dev[64];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;
std::once_flag g_ctx_once;

ra_status_t current_device(DevInfo* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(RA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_dev[dev].major < 0) {
    cudaDeviceProp p;
    e = cudaGetDeviceProperties(&p, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
    g_dev[dev].major = p.major;
    g_dev[dev].minor = p.minor;
    g_dev[dev].sms = p.multiProcessorCount;
  }
  if (g_dev[dev].major == 10 && g_dev[dev].minor == 0) {
    // The status word's address, looked up again whenever the current context is not the one it
    // was found in (or the context cannot be identified).
    const unsigned long long ctx = ra::current_context_id();
    if (g_dev[dev].status == nullptr || ctx == 0 || ctx != g_dev[dev].ctx) {
      void* addr = nullptr;
      e = cudaGetSymbolAddress(&addr, ra::g_dev_status);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status word)");
      g_dev[dev].status = static_cast<unsigned int*>(addr);
      g_dev[dev].ctx = ra::current_context_id();
    }
  }
  *out = g_dev[dev];
  if (out->major != 10 || out->minor != 0)
    return fail(RA_ERR_UNSUPPORTED, "this library is built for sm_100a (B200); device %d is sm_%d%d", dev,
                out->major, out->minor);
  return RA_OK;
}

const int64_t kMax32 = (int64_t(1) << 31) - 1;

ra_status_t check_tensor(const ra_tensor_t* t, const char* name) {
  if (t == nullptr) return fail(RA_ERR_INVALID_ARG, "%s is NULL", name);
  if (t->data == nullptr) return fail(RA_ERR_INVALID_ARG, "%s->data is NULL", name);
  if (t->dtype != RA_F32 && t->dtype != RA_BF16) return fail(RA_ERR_INVALID_ARG, "%s->dtype %d unknown", name, t->dtype);
  for (int i = 0; i < 4; ++i) {
    if (t->shape[i] < 1 || t->shape[i] > kMax32)
      return fail(RA_ERR_INVALID_ARG, "%s->shape[%d] = %lld out of range [1, 2^31)", name, i, (long long)t->shape[i]);
    if (t->stride[i] < 0) return fail(RA_ERR_INVALID_ARG, "%s->stride[%d] is negative", name, i);
  }
  if (t->stride[3] != 1) return fail(RA_ERR_INVALID_ARG, "%s->stride[3] must be 1 (head dim contiguous)", name);
  return RA_OK;
}

// The bf16 tensor-core path reads through TMA: base 16-byte aligned, strides multiples of 16 B.
ra_status_t check_tma_tensor(const ra_tensor_t* t, const char* name) {
  if (reinterpret_cast<uintptr_t>(t->data) % 16 != 0)
    return fail(RA_ERR_ALIGNMENT, "%s->data must be 16-byte aligned for the bf16 path", name);
  for (int i = 0; i < 3; ++i)
    if (t->shape[i] > 1 && t->stride[i] % 8 != 0)
      return fail(RA_ERR_ALIGNMENT, "%s->stride[%d] = %lld must be a multiple of 8 elements (16 bytes)", name, i,
                  (long long)t->stride[i]);
  return RA_OK;
}

ra_status_t check_f32_vec_tensor(const ra_tensor_t* t, const char* name) {
  if (reinterpret_cast<uintptr_t>(t->data) % 16 != 0)
    return fail(RA_ERR_ALIGNMENT, "%s->data must be 16-byte aligned", name);
  for (int i = 0; i < 3; ++i)
    if (t->shape[i] > 1 && t->stride[i] % 4 != 0)
      return fail(RA_ERR_ALIGNMENT, "%s->stride[%d] must be a multiple of 4 elements", name, i);
  return RA_OK;
}

ra_status_t check_head_dim(int d, int dtype) {
  if (d < 1 || d > 128) return fail(RA_ERR_UNSUPPORTED, "head dim %d not in [1, 128]", d);
  if (dtype == RA_BF16 && d % 8 != 0) return fail(RA_ERR_UNSUPPORTED, "bf16 path needs head dim %% 8 == 0 (got %d)", d);
  return RA_OK;
}

int padded_dim(int d) { return d <= 32 ? 32 : (d <= 64 ? 64 : 128); }

// Rows of one K/V tile of the tensor-core forward kernel (the TMA box height of K and V).
int kv_box_rows(int dp) {
  return dp == 32 ? ra::FmhaCfg<32>::BN : (dp == 64 ? ra::FmhaCfg<64>::BN : ra::FmhaCfg<128>::BN);
}

float resolve_scale(float scale, int d) { return scale > 0.f ? scale : static_cast<float>(1.0 / std::sqrt((double)d)); }

// ------------------------------------------------------------------------------------------
// TMA descriptors
// ------------------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
cudaError_t g_encode_err = cudaSuccess;

ra_status_t get_encode(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::call_once(g_encode_once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    g_encode_err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (g_encode_err == cudaSuccess && q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  if (g_encode == nullptr) return fail(RA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorName(g_encode_err));
  *fn = g_encode;
  return RA_OK;
}

// 5-D view (d, token, shard, head, batch) of a bf16 tensor; strides in elements.
struct View5 {
  const void* base;
  int64_t dim[5];
  int64_t stride[5];  // stride[0] == 1
};

ra_status_t encode_view(CUtensorMap* map, const View5& v, int dp, int box_rows = 128) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  ra_status_t st = get_encode(&enc);
  if (st != RA_OK) return st;
  cuuint64_t dims[5];
  cuuint64_t strides[4];
  for (int i = 0; i < 5; ++i) dims[i] = static_cast<cuuint64_t>(v.dim[i]);
  for (int i = 1; i < 5; ++i) {
    int64_t s = v.stride[i];
    if (v.dim[i] == 1 || s == 0) s = 8;  // unused dimension: any valid stride
    if (s % 8 != 0) return fail(RA_ERR_ALIGNMENT, "TMA stride %lld elements is not a multiple of 16 bytes", (long long)s);
    strides[i - 1] = static_cast<cuuint64_t>(s) * 2;
  }
  const cuuint32_t box0 = dp == 32 ? 32 : 64;
  cuuint32_t box[5] = {box0, static_cast<cuuint32_t>(box_rows), 1, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUtensorMapSwizzle swz = dp == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(v.base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(RA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return RA_OK;
}

// Shard view of a [B, H, N, d] tensor: token t of shard s is row s * shard_rows + t * tok_rows.
View5 shard_view(const ra_tensor_t* t, int64_t n_local, int64_t P, int64_t shard_rows, int64_t tok_rows) {
  View5 v;
  v.base = t->data;
  v.dim[0] = t->shape[3];
  v.dim[1] = n_local;
  v.dim[2] = P;
  v.dim[3] = t->shape[1];
  v.dim[4] = t->shape[0];
  v.stride[0] = 1;
  v.stride[1] = tok_rows * t->stride[2];
  v.stride[2] = shard_rows * t->stride[2];
  v.stride[3] = t->stride[1];
  v.stride[4] = t->stride[0];
  return v;
}

// ------------------------------------------------------------------------------------------
// Launch helpers
// ------------------------------------------------------------------------------------------
struct Maps {
  CUtensorMap q, k, v;
};

// Heads per work-item group: the largest divisor of B*H (equal groups keep the longest-first
// balance inside each group) whose K and V, all shards, fit in an L2 budget.  When every head's
// K/V fits in 80 MiB of the 126 MB L2, all heads form one group, so the whole launch keeps one
// longest-first order (causal items differ in length).  Otherwise groups are sized to 40 MiB: the
// L2 is split over the GPU's two dies, and the CTAs running at one time then share K/V that fits
// one half (measured on the B=1 H=32 N=32768 d=128 causal ring: 0.99 -> 1.03 PFLOP/s; splitting
// a problem that fits one group costs 10 %).
int heads_per_group(const ra::AttnWork& w, int elem_bytes) {
  // K and V bytes per query head (query heads that share a K/V head share its bytes in L2).
  const int qpk = (w.H_kv > 0 && w.H % w.H_kv == 0) ? w.H / w.H_kv : 1;
  const double kv_bytes = 2.0 * static_cast<double>(w.n_kv) * w.P * w.d * elem_bytes / qpk;
  const long long bh = static_cast<long long>(w.B) * w.H;
  const double whole = 80.0 * 1024 * 1024;
  if (kv_bytes * static_cast<double>(bh) <= whole) return static_cast<int>(bh);
#ifndef RA_L2_GROUP_MIB
#define RA_L2_GROUP_MIB 40
#endif
  const double budget = static_cast<double>(RA_L2_GROUP_MIB) * 1024 * 1024;
  long long hg_max = static_cast<long long>(budget / (kv_bytes > 1.0 ? kv_bytes : 1.0));
  if (hg_max < 1) hg_max = 1;
  if (hg_max >= bh) return static_cast<int>(bh);
  for (long long hg = hg_max; hg > 1; --hg)
    if (bh % hg == 0) return static_cast<int>(hg);
  return 1;
}

ra_status_t prepare_attention(const ra_tensor_t* q, const ra::AttnWork& w_in, int n_steps, ra::AttnWork* out) {
  if (w_in.B > 65535 || w_in.H > 65535) return fail(RA_ERR_UNSUPPORTED, "B and H must be <= 65535");
  ra::AttnWork w = w_in;
  if (w.H_kv == 0) w.H_kv = w.H;
  w.hgroup = heads_per_group(w, q->dtype == RA_BF16 ? 2 : 4);
  {
    // Launch-time fast dividers for the kernels' index arithmetic (all operands stay below 2^31).
    const long long n_blk = (static_cast<long long>(w.n_q) + 255) / 256;
    const long long per_group = static_cast<long long>(w.hgroup) * n_blk * w.n_r;
    const long long bh = static_cast<long long>(w.B) * w.H;
    if (per_group * ((bh + w.hgroup - 1) / w.hgroup) > 2147483647LL || w.k_ustride > 2147483647LL ||
        w.ring_step < 0 || w.ring_step + n_steps > 2 * w.P)
      return fail(RA_ERR_UNSUPPORTED, "problem too large for 32-bit work-item indices");
    const long long hg_last = bh - (bh - 1) / w.hgroup * w.hgroup;
    w.fd_grp = ra::make_fastdiv(static_cast<unsigned>(per_group));
    w.fd_hg = ra::make_fastdiv(static_cast<unsigned>(w.hgroup));
    w.fd_hg_last = ra::make_fastdiv(static_cast<unsigned>(hg_last));
    w.fd_nblk = ra::make_fastdiv(static_cast<unsigned>(n_blk));
    w.fd_nr = ra::make_fastdiv(static_cast<unsigned>(w.n_r));
    w.fd_H = ra::make_fastdiv(static_cast<unsigned>(w.H));
    w.fd_P = ra::make_fastdiv(static_cast<unsigned>(w.P));
    w.fd_kus = ra::make_fastdiv(static_cast<unsigned>(w.k_ustride));
    if (w.H_kv < 1 || w.H % w.H_kv != 0) return fail(RA_ERR_INVALID_ARG, "H_kv must divide H");
    w.fd_qpk = ra::make_fastdiv(static_cast<unsigned>(w.H / w.H_kv));
  }
  if (q->dtype != RA_BF16 && static_cast<long long>(w.n_q_tiles) * w.n_r > 2147483647LL)
    return fail(RA_ERR_UNSUPPORTED, "grid too large");
  *out = w;
  return RA_OK;
}

// Launches a work description completed by prepare_attention.
ra_status_t launch_prepared(const ra_tensor_t* q, const Maps* maps, const ra::AttnWork& w, int n_steps, int epi,
                            int sms, cudaStream_t stream, bool dependent = false) {
  cudaError_t e;
  if (q->dtype == RA_BF16) {
    const int dp = padded_dim(w.d);
    if (dp == 32)
      e = ra::launch_fmha_dp32(maps->q, maps->k, maps->v, w, n_steps, epi, sms, stream, dependent);
    else if (dp == 64)
      e = ra::launch_fmha_dp64(maps->q, maps->k, maps->v, w, n_steps, epi, sms, stream, dependent);
    else
      e = ra::launch_fmha_dp128(maps->q, maps->k, maps->v, w, n_steps, epi, sms, stream, dependent);
  } else {
    const long long gx = static_cast<long long>(w.n_q_tiles) * w.n_r;
    dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(w.H), static_cast<unsigned>(w.B));
    const int dp = padded_dim(w.d);
    if (dp == 32)
      ra::attn_fwd_simt_f32<32><<<grid, 128, 0, stream>>>(w, n_steps, epi);
    else if (dp == 64)
      ra::attn_fwd_simt_f32<64><<<grid, 128, 0, stream>>>(w, n_steps, epi);
    else
      ra::attn_fwd_simt_f32<128><<<grid, 128, 0, stream>>>(w, n_steps, epi);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return RA_OK;
}

ra_status_t launch_attention(const ra_tensor_t* q, const Maps* maps, const ra::AttnWork& w_in, int n_steps, int epi,
                             int sms, cudaStream_t stream) {
  ra::AttnWork w;
  ra_status_t st = prepare_attention(q, w_in, n_steps, &w);
  if (st != RA_OK) return st;
  return launch_prepared(q, maps, w, n_steps, epi, sms, stream);
}

void set_operand_ptrs(ra::AttnWork& w, const ra_tensor_t* q, const ra_tensor_t* k, const ra_tensor_t* v,
                      int64_t shard_rows, int64_t tok_rows) {
  w.q = q->data;
  w.k = k->data;
  w.v = v->data;
  w.H_kv = static_cast<int>(k->shape[1]);
  w.q_sb = q->stride[0];
  w.q_sh = q->stride[1];
  w.q_rs = shard_rows * q->stride[2];
  w.q_ts = tok_rows * q->stride[2];
  w.k_sb = k->stride[0];
  w.k_sh = k->stride[1];
  w.k_rs = shard_rows * k->stride[2];
  w.k_ts = tok_rows * k->stride[2];
  w.v_sb = v->stride[0];
  w.v_sh = v->stride[1];
  w.v_rs = shard_rows * v->stride[2];
  w.v_ts = tok_rows * v->stride[2];
}

ra_status_t check_qkv(const ra_tensor_t* q, const ra_tensor_t* k, const ra_tensor_t* v) {
  ra_status_t st;
  if ((st = check_tensor(q, "q")) != RA_OK) return st;
  if ((st = check_tensor(k, "k")) != RA_OK) return st;
  if ((st = check_tensor(v, "v")) != RA_OK) return st;
  if (k->dtype != q->dtype || v->dtype != q->dtype) return fail(RA_ERR_INVALID_ARG, "q, k, v must share one dtype");
  if (k->shape[0] != q->shape[0] || v->shape[0] != q->shape[0])
    return fail(RA_ERR_INVALID_ARG, "q, k, v must agree on B");
  if (v->shape[1] != k->shape[1] || k->shape[1] < 1 || q->shape[1] % k->shape[1] != 0)
    return fail(RA_ERR_INVALID_ARG, "k and v must have the same number of heads H_kv, and H_kv must divide the "
                                    "query heads H (H_kv = H: multi-head, 1: multi-query, else grouped-query)");
  if (k->shape[3] != q->shape[3] || v->shape[3] != q->shape[3])
    return fail(RA_ERR_INVALID_ARG, "q, k, v must share the head dim");
  if (v->shape[2] != k->shape[2]) return fail(RA_ERR_INVALID_ARG, "k and v must have the same number of keys");
  if ((st = check_head_dim(static_cast<int>(q->shape[3]), q->dtype)) != RA_OK) return st;
  if (q->dtype == RA_BF16) {
    if ((st = check_tma_tensor(q, "q")) != RA_OK) return st;
    if ((st = check_tma_tensor(k, "k")) != RA_OK) return st;
    if ((st = check_tma_tensor(v, "v")) != RA_OK) return st;
  }
  return RA_OK;
}

ra_status_t check_out(const ra_tensor_t* o, const ra_tensor_t* q, const char* name, int want_dtype) {
  ra_status_t st = check_tensor(o, name);
  if (st != RA_OK) return st;
  if (o->dtype != want_dtype) return fail(RA_ERR_INVALID_ARG, "%s has the wrong dtype", name);
  for (int i = 0; i < 4; ++i)
    if (o->shape[i] != q->shape[i]) return fail(RA_ERR_INVALID_ARG, "%s must have the shape of q", name);
  if (o->dtype == RA_BF16) return check_tma_tensor(o, name);
  return RA_OK;
}

ra::AttnWork base_work(const ra_tensor_t* q, float scale, int causal, const DevInfo& dev) {
  ra::AttnWork w{};
  w.dev_status = dev.status;
  w.B = static_cast<int>(q->shape[0]);
  w.r_major = 0;
  w.H = static_cast<int>(q->shape[1]);
  w.d = static_cast<int>(q->shape[3]);
  w.causal = causal ? 1 : 0;
  w.scale = resolve_scale(scale, w.d);
  w.scale_log2 = static_cast<float>(static_cast<double>(w.scale) * kLog2e);
  w.r_first = 0;
  w.r_step = 1;
  w.n_r = 1;
  w.ring_step = 0;
  w.P = 1;
  w.wait_limit_ns = g_wait_limit_ns.load();
  return w;
}

int q_rows_per_cta(int dtype) { return dtype == RA_BF16 ? 128 : ra::kSimtRows; }

}  // namespace

namespace {
// Launchers for the runtime lane-group size G (a power of two <= 32).
template <int VEC>
static void launch_merge2(int G, dim3 grid, cudaStream_t st, const float* o_a, const float* lse_a, const float* o_b,
                          const float* lse_b, float* o_out, float* lse_out, long long rows, int d) {
  switch (G) {
    case 1: ra::lse_merge2_kernel<VEC, 1><<<grid, 256, 0, st>>>(o_a, lse_a, o_b, lse_b, o_out, lse_out, rows, d); break;
    case 2: ra::lse_merge2_kernel<VEC, 2><<<grid, 256, 0, st>>>(o_a, lse_a, o_b, lse_b, o_out, lse_out, rows, d); break;
    case 4: ra::lse_merge2_kernel<VEC, 4><<<grid, 256, 0, st>>>(o_a, lse_a, o_b, lse_b, o_out, lse_out, rows, d); break;
    case 8: ra::lse_merge2_kernel<VEC, 8><<<grid, 256, 0, st>>>(o_a, lse_a, o_b, lse_b, o_out, lse_out, rows, d); break;
    case 16: ra::lse_merge2_kernel<VEC, 16><<<grid, 256, 0, st>>>(o_a, lse_a, o_b, lse_b, o_out, lse_out, rows, d); break;
    default: ra::lse_merge2_kernel<VEC, 32><<<grid, 256, 0, st>>>(o_a, lse_a, o_b, lse_b, o_out, lse_out, rows, d); break;
  }
}

template <int VEC, int KMAX>
static void launch_merge_n(int G, dim3 grid, cudaStream_t st, const ra::MergeParts& parts, int k, float* o_out,
                           float* lse_out, long long rows, int d) {
  switch (G) {
    case 1: ra::lse_merge_n_kernel<VEC, 1, KMAX><<<grid, 256, 0, st>>>(parts, k, o_out, lse_out, rows, d); break;
    case 2: ra::lse_merge_n_kernel<VEC, 2, KMAX><<<grid, 256, 0, st>>>(parts, k, o_out, lse_out, rows, d); break;
    case 4: ra::lse_merge_n_kernel<VEC, 4, KMAX><<<grid, 256, 0, st>>>(parts, k, o_out, lse_out, rows, d); break;
    case 8: ra::lse_merge_n_kernel<VEC, 8, KMAX><<<grid, 256, 0, st>>>(parts, k, o_out, lse_out, rows, d); break;
    case 16: ra::lse_merge_n_kernel<VEC, 16, KMAX><<<grid, 256, 0, st>>>(parts, k, o_out, lse_out, rows, d); break;
    default: ra::lse_merge_n_kernel<VEC, 32, KMAX><<<grid, 256, 0, st>>>(parts, k, o_out, lse_out, rows, d); break;
  }
}

}  // namespace

namespace ra {
unsigned long long current_context_id() {
  std::call_once(g_ctx_once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult r;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (g_ctx_get_current == nullptr || g_ctx_get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (g_ctx_get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Lets the library's other translation units report through ra_last_error().
ra_status_t set_last_error(ra_status_t status, const char* message) { return fail(status, "%s", message); }
}  // namespace ra

// ==============================================================================================
// Entry points
// ==============================================================================================
extern "C" {

static ra_status_t attn_fwd_impl(const ra_tensor_t* q, const ra_tensor_t* k, const ra_tensor_t* v,
                                 const ra_tensor_t* o, float* lse, float scale, int causal, int64_t window,
                                 ra_stream_t stream) {
  ra_status_t st = check_qkv(q, k, v);
  if (st != RA_OK) return st;
  if ((st = check_out(o, q, "o", q->dtype)) != RA_OK) return st;
  DevInfo dev;
  if ((st = current_device(&dev)) != RA_OK) return st;
  ra::AttnWork w = base_work(q, scale, causal, dev);
  w.window = window;
  w.n_q = static_cast<int>(q->shape[2]);
  w.n_kv = static_cast<int>(k->shape[2]);
  w.n_q_tiles = (w.n_q + q_rows_per_cta(q->dtype) - 1) / q_rows_per_cta(q->dtype);
  w.q_off = 0;
  w.q_rstep = 0;
  w.q_tstride = 1;
  w.k_off = 0;
  w.k_sstep = 0;
  w.k_ustride = 1;
  set_operand_ptrs(w, q, k, v, 0, 1);
  w.o = o->data;
  w.o_sb = o->stride[0];
  w.o_sh = o->stride[1];
  w.o_rs = 0;
  w.o_ts = o->stride[2];
  w.lse = lse;
  w.l_sb = q->shape[1] * q->shape[2];
  w.l_sh = q->shape[2];
  w.l_rs = 0;
  w.l_ts = 1;

  Maps maps;
  if (q->dtype == RA_BF16) {
    const int dp = padded_dim(w.d);
    if ((st = encode_view(&maps.q, shard_view(q, w.n_q, 1, 0, 1), dp)) != RA_OK) return st;
    if ((st = encode_view(&maps.k, shard_view(k, w.n_kv, 1, 0, 1), dp, kv_box_rows(dp))) != RA_OK) return st;
    if ((st = encode_view(&maps.v, shard_view(v, w.n_kv, 1, 0, 1), dp, kv_box_rows(dp))) != RA_OK) return st;
  }
  st = launch_attention(q, &maps, w, 1, ra::kEpiOut, dev.sms, reinterpret_cast<cudaStream_t>(stream));
  return st == RA_OK ? ok() : st;
}

ra_status_t ra_attn_partial(const ra_tensor_t* q, const ra_tensor_t* k_shard, const ra_tensor_t* v_shard,
                            ra_pos_t q_pos, ra_pos_t kv_pos, int causal, float scale, const ra_tensor_t* o_part,
                            float* lse_part, int accumulate, ra_stream_t stream) {
  ra_status_t st = check_qkv(q, k_shard, v_shard);
  if (st != RA_OK) return st;
  if ((st = check_out(o_part, q, "o_part", RA_F32)) != RA_OK) return st;
  if (lse_part == nullptr) return fail(RA_ERR_INVALID_ARG, "lse_part is NULL");
  if (q->dtype == RA_BF16 && (st = check_f32_vec_tensor(o_part, "o_part")) != RA_OK) return st;
  if (causal && (q_pos.stride < 1 || kv_pos.stride < 1))
    return fail(RA_ERR_INVALID_ARG, "position strides must be >= 1");
  DevInfo dev;
  if ((st = current_device(&dev)) != RA_OK) return st;
  ra::AttnWork w = base_work(q, scale, causal, dev);
  w.n_q = static_cast<int>(q->shape[2]);
  w.n_kv = static_cast<int>(k_shard->shape[2]);
  w.n_q_tiles = (w.n_q + q_rows_per_cta(q->dtype) - 1) / q_rows_per_cta(q->dtype);
  w.q_off = q_pos.offset;
  w.q_rstep = 0;
  w.q_tstride = causal ? q_pos.stride : 1;
  w.k_off = kv_pos.offset;
  w.k_sstep = 0;
  w.k_ustride = causal ? kv_pos.stride : 1;
  set_operand_ptrs(w, q, k_shard, v_shard, 0, 1);
  w.acc_o = static_cast<float*>(o_part->data);
  w.a_sb = o_part->stride[0];
  w.a_sh = o_part->stride[1];
  w.a_rs = 0;
  w.a_ts = o_part->stride[2];
  w.acc_l = lse_part;
  w.al_sb = q->shape[1] * q->shape[2];
  w.al_sh = q->shape[2];
  w.al_rs = 0;
  w.al_ts = 1;

  Maps maps;
  if (q->dtype == RA_BF16) {
    const int dp = padded_dim(w.d);
    if ((st = encode_view(&maps.q, shard_view(q, w.n_q, 1, 0, 1), dp)) != RA_OK) return st;
    if ((st = encode_view(&maps.k, shard_view(k_shard, w.n_kv, 1, 0, 1), dp, kv_box_rows(dp))) != RA_OK) return st;
    if ((st = encode_view(&maps.v, shard_view(v_shard, w.n_kv, 1, 0, 1), dp, kv_box_rows(dp))) != RA_OK) return st;
  }
  st = launch_attention(q, &maps, w, 1, accumulate ? ra::kEpiAcc : ra::kEpiPart, dev.sms,
                        reinterpret_cast<cudaStream_t>(stream));
  return st == RA_OK ? ok() : st;
}

static int merge_group(int nv) {
  int g = 1;
  while (g < nv && g < 32) g *= 2;
  return g;
}

static unsigned merge_grid(long long rows, int G, int sms) {
  const long long groups_per_block = 256 / G;
  long long blocks = (rows + groups_per_block - 1) / groups_per_block;
  const long long cap = static_cast<long long>(sms) * 8;  // 8 blocks of 256 threads fill an SM
  if (blocks > cap) blocks = cap;
  return static_cast<unsigned>(blocks < 1 ? 1 : blocks);
}

static bool aligned16(const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; }

ra_status_t ra_lse_merge(const float* o_a, const float* lse_a, const float* o_b, const float* lse_b, float* o_out,
                         float* lse_out, int64_t rows, int d, ra_stream_t stream) {
  if (rows < 0) return fail(RA_ERR_INVALID_ARG, "rows < 0");
  if (d < 1 || d > 4096) return fail(RA_ERR_INVALID_ARG, "d must be in [1, 4096]");
  if (rows == 0) return ok();
  if (!o_a || !lse_a || !o_b || !lse_b || !o_out || !lse_out) return fail(RA_ERR_INVALID_ARG, "NULL pointer");
  DevInfo dev;
  ra_status_t s0 = current_device(&dev);
  if (s0 != RA_OK) return s0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool vec = d % 4 == 0 && aligned16(o_a) && aligned16(o_b) && aligned16(o_out);
  const int G = merge_group(vec ? d / 4 : d);
  dim3 grid(merge_grid(rows, G, dev.sms));
  if (vec)
    launch_merge2<4>(G, grid, st, o_a, lse_a, o_b, lse_b, o_out, lse_out, (long long)rows, d);
  else
    launch_merge2<1>(G, grid, st, o_a, lse_a, o_b, lse_b, o_out, lse_out, (long long)rows, d);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "lse merge launch");
  return ok();
}

ra_status_t ra_lse_merge_n(const float* const* o_parts, const float* const* lse_parts, int k, float* o_out,
                           float* lse_out, int64_t rows, int d, ra_stream_t stream) {
  if (k < 1 || k > RA_MERGE_MAX_PARTS) return fail(RA_ERR_INVALID_ARG, "k must be in [1, %d]", RA_MERGE_MAX_PARTS);
  if (rows < 0) return fail(RA_ERR_INVALID_ARG, "rows < 0");
  if (d < 1 || d > 4096) return fail(RA_ERR_INVALID_ARG, "d must be in [1, 4096]");
  if (rows == 0) return ok();
  if (!o_parts || !lse_parts || !o_out || !lse_out) return fail(RA_ERR_INVALID_ARG, "NULL pointer");
  ra::MergeParts parts{};
  bool vec = d % 4 == 0 && aligned16(o_out);
  for (int i = 0; i < k; ++i) {
    if (!o_parts[i] || !lse_parts[i]) return fail(RA_ERR_INVALID_ARG, "NULL partial %d", i);
    parts.o[i] = o_parts[i];
    parts.l[i] = lse_parts[i];
    vec = vec && aligned16(o_parts[i]);
  }
  DevInfo dev;
  ra_status_t s0 = current_device(&dev);
  if (s0 != RA_OK) return s0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int G = merge_group(vec ? d / 4 : d);
  dim3 grid(merge_grid(rows, G, dev.sms));
  if (vec) {
    if (k <= 4)
      launch_merge_n<4, 4>(G, grid, st, parts, k, o_out, lse_out, (long long)rows, d);
    else if (k <= 8)
      launch_merge_n<4, 8>(G, grid, st, parts, k, o_out, lse_out, (long long)rows, d);
    else if (k <= 16)
      launch_merge_n<4, 16>(G, grid, st, parts, k, o_out, lse_out, (long long)rows, d);
    else
      launch_merge_n<4, 32>(G, grid, st, parts, k, o_out, lse_out, (long long)rows, d);
  } else {
    if (k <= 8)
      launch_merge_n<1, 8>(G, grid, st, parts, k, o_out, lse_out, (long long)rows, d);
    else
      launch_merge_n<1, 32>(G, grid, st, parts, k, o_out, lse_out, (long long)rows, d);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "lse merge launch");
  return ok();
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

ra_status_t ra_ring_workspace_size(const ra_tensor_t* q, int P, int schedule, size_t* bytes) {
  if (bytes == nullptr) return fail(RA_ERR_INVALID_ARG, "bytes is NULL");
  ra_status_t st = check_tensor(q, "q");
  if (st != RA_OK) return st;
  if (P < 1 || q->shape[2] % P != 0) return fail(RA_ERR_INVALID_ARG, "P must be >= 1 and divide N");
  if (schedule != RA_RING_STEPWISE && schedule != RA_RING_FUSED) return fail(RA_ERR_INVALID_ARG, "unknown schedule");
  if (schedule == RA_RING_FUSED || P == 1) {
    *bytes = 0;
    return ok();
  }
  const size_t rows = static_cast<size_t>(q->shape[0]) * q->shape[1] * q->shape[2];
  *bytes = align256(rows * q->shape[3] * sizeof(float)) + align256(rows * sizeof(float));
  return ok();
}

// dry_run: every check of the call, encoding and launch preparation included, and nothing enqueued.
static ra_status_t ring_fwd_impl(const ra_tensor_t* q, const ra_tensor_t* k, const ra_tensor_t* v, int P,
                                 int layout, int causal, int64_t window, float scale, int schedule,
                                 const ra_tensor_t* o, float* lse, const ra_stream_t* streams, int n_streams,
                                 void* workspace, size_t workspace_bytes, bool dry_run = false) {
  ra_status_t st = check_qkv(q, k, v);
  if (st != RA_OK) return st;
  if ((st = check_out(o, q, "o", q->dtype)) != RA_OK) return st;
  if (k->shape[2] != q->shape[2]) return fail(RA_ERR_INVALID_ARG, "ring attention needs as many keys as queries");
  if (P < 1 || P > 64) return fail(RA_ERR_INVALID_ARG, "P must be in [1, 64]");
  if (q->shape[2] % P != 0) return fail(RA_ERR_INVALID_ARG, "N = %lld is not a multiple of P = %d", (long long)q->shape[2], P);
  if (layout != RA_CONTIGUOUS && layout != RA_STRIPED) return fail(RA_ERR_INVALID_ARG, "unknown layout %d", layout);
  if (schedule != RA_RING_STEPWISE && schedule != RA_RING_FUSED) return fail(RA_ERR_INVALID_ARG, "unknown schedule");
  if (streams == nullptr || n_streams < 1) return fail(RA_ERR_INVALID_ARG, "need at least one stream");
  if (n_streams > P) n_streams = P;
  size_t need = 0;
  if ((st = ra_ring_workspace_size(q, P, schedule, &need)) != RA_OK) return st;
  if (need > 0 && (workspace == nullptr || workspace_bytes < need))
    return fail(RA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
  if (need > 0 && reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
    return fail(RA_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  DevInfo dev;
  if ((st = current_device(&dev)) != RA_OK) return st;

  const int64_t N = q->shape[2];
  const int64_t n_local = N / P;
  const bool striped = layout == RA_STRIPED;
  // Rows of shard r / local token t in the full [.., N, ..] tensors.
  const int64_t shard_rows = striped ? 1 : n_local;
  const int64_t tok_rows = striped ? P : 1;

  ra::AttnWork w = base_work(q, scale, causal, dev);
  w.window = window;
  w.P = P;
  w.n_q = static_cast<int>(n_local);
  w.n_kv = static_cast<int>(n_local);
  w.n_q_tiles = static_cast<int>((n_local + q_rows_per_cta(q->dtype) - 1) / q_rows_per_cta(q->dtype));
  w.q_off = 0;
  w.q_rstep = shard_rows;
  w.q_tstride = tok_rows;
  w.k_off = 0;
  w.k_sstep = shard_rows;
  w.k_ustride = tok_rows;
  w.r_major = striped ? 0 : 1;
  w.tile_major = striped && g_striped_walk.load() == RA_WALK_TILE_MAJOR ? 1 : 0;
  set_operand_ptrs(w, q, k, v, shard_rows, tok_rows);
  w.o = o->data;
  w.o_sb = o->stride[0];
  w.o_sh = o->stride[1];
  w.o_rs = shard_rows * o->stride[2];
  w.o_ts = tok_rows * o->stride[2];
  w.lse = lse;
  w.l_sb = q->shape[1] * N;
  w.l_sh = N;
  w.l_rs = shard_rows;
  w.l_ts = tok_rows;
  if (need > 0) {
    const int64_t d = q->shape[3];
    w.acc_o = static_cast<float*>(workspace);
    w.a_ts = d;
    w.a_rs = n_local * d;
    w.a_sh = P * n_local * d;
    w.a_sb = q->shape[1] * P * n_local * d;
    const size_t o_bytes = align256(static_cast<size_t>(q->shape[0]) * q->shape[1] * N * d * sizeof(float));
    w.acc_l = reinterpret_cast<float*>(static_cast<char*>(workspace) + o_bytes);
    w.al_ts = 1;
    w.al_rs = n_local;
    w.al_sh = P * n_local;
    w.al_sb = q->shape[1] * P * n_local;
  }

  Maps maps;
  if (q->dtype == RA_BF16) {
    const int dp = padded_dim(w.d);
    if ((st = encode_view(&maps.q, shard_view(q, n_local, P, shard_rows, tok_rows), dp)) != RA_OK) return st;
    if ((st = encode_view(&maps.k, shard_view(k, n_local, P, shard_rows, tok_rows), dp, kv_box_rows(dp))) != RA_OK) return st;
    if ((st = encode_view(&maps.v, shard_view(v, n_local, P, shard_rows, tok_rows), dp, kv_box_rows(dp))) != RA_OK) return st;
  }

  // Every launch of the call is described and checked before the first one is enqueued.
  struct Launch {
    ra::AttnWork w;
    int stream, n_steps, epi;
    bool dependent;  // a later step of the stepwise ring on the same stream (tensor-core path)
  };
  std::vector<Launch> launches;
  for (int i = 0; i < n_streams; ++i) {
    ra::AttnWork wi = w;
    wi.r_first = i;
    wi.r_step = n_streams;
    wi.n_r = (P - i + n_streams - 1) / n_streams;
    if (schedule == RA_RING_FUSED || P == 1) {
      wi.ring_step = 0;
      launches.push_back({wi, i, P, ra::kEpiOut, false});
    } else {
      for (int t = 0; t < P; ++t) {
        wi.ring_step = t;
#ifndef RA_PDL
#define RA_PDL 1
#endif
        launches.push_back({wi, i, 1, t == 0 ? ra::kEpiPart : (t == P - 1 ? ra::kEpiAccOut : ra::kEpiAcc),
                            RA_PDL && t > 0 && q->dtype == RA_BF16});
      }
    }
  }
  for (Launch& l : launches)
    if ((st = prepare_attention(q, l.w, l.n_steps, &l.w)) != RA_OK) return st;
  if (dry_run) return ok();

  // Events that fork the extra streams off streams[0] (so the call is ordered after work already
  // queued there) and join them back, created before anything is enqueued.
  cudaStream_t s0 = reinterpret_cast<cudaStream_t>(streams[0]);
  std::vector<cudaEvent_t> events;
  auto destroy_events = [&events] {
    for (cudaEvent_t ev : events) cudaEventDestroy(ev);
  };
  cudaError_t e;
  for (int i = 0; i < (n_streams > 1 ? n_streams : 0); ++i) {
    cudaEvent_t ev = nullptr;
    if ((e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming)) != cudaSuccess) {
      destroy_events();
      return cuda_fail(e, "event");
    }
    events.push_back(ev);  // events[0]: fork; events[i >= 1]: join of streams[i]
  }
  if (n_streams > 1) {
    e = cudaEventRecord(events[0], s0);
    for (int i = 1; i < n_streams && e == cudaSuccess; ++i)
      e = cudaStreamWaitEvent(reinterpret_cast<cudaStream_t>(streams[i]), events[0], 0);
    if (e != cudaSuccess) {
      destroy_events();
      return cuda_fail(e, "stream fork");
    }
  }

  // A launch can still fail here only through the CUDA runtime; the streams that already hold
  // work of this call are joined to streams[0] all the same, and the error is returned.
  st = RA_OK;
  std::string launch_error;
  for (const Launch& l : launches) {
    st = launch_prepared(q, &maps, l.w, l.n_steps, l.epi, dev.sms, reinterpret_cast<cudaStream_t>(streams[l.stream]),
                         l.dependent);
    if (st != RA_OK) {
      launch_error = t_last_error;
      break;
    }
  }
  for (int i = 1; i < n_streams; ++i) {
    e = cudaEventRecord(events[i], reinterpret_cast<cudaStream_t>(streams[i]));
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s0, events[i], 0);
    if (e != cudaSuccess) {
      destroy_events();
      return cuda_fail(e, "stream join (kernels of this call may be queued)");
    }
  }
  destroy_events();
  if (st != RA_OK)
    return fail(st, "%s (earlier launches of this ring call stay queued, ordered before later work on streams[0])",
                launch_error.c_str());
  return ok();
}

ra_status_t ra_attn_fwd(const ra_tensor_t* q, const ra_tensor_t* k, const ra_tensor_t* v, const ra_tensor_t* o,
                        float* lse, float scale, int causal, ra_stream_t stream) {
  return attn_fwd_impl(q, k, v, o, lse, scale, causal, 0, stream);
}

ra_status_t ra_attn_fwd_window(const ra_tensor_t* q, const ra_tensor_t* k, const ra_tensor_t* v,
                               const ra_tensor_t* o, float* lse, float scale, int64_t window, ra_stream_t stream) {
  if (window < 1) return fail(RA_ERR_INVALID_ARG, "window must be >= 1 (got %lld)", (long long)window);
  return attn_fwd_impl(q, k, v, o, lse, scale, 1, window, stream);
}

ra_status_t ra_ring_fwd(const ra_tensor_t* q, const ra_tensor_t* k, const ra_tensor_t* v, int P, int layout,
                        int causal, float scale, int schedule, const ra_tensor_t* o, float* lse,
                        const ra_stream_t* streams, int n_streams, void* workspace, size_t workspace_bytes) {
  return ring_fwd_impl(q, k, v, P, layout, causal, 0, scale, schedule, o, lse, streams, n_streams, workspace,
                       workspace_bytes);
}

ra_status_t ra_ring_fwd_window(const ra_tensor_t* q, const ra_tensor_t* k, const ra_tensor_t* v, int P, int layout,
                               int64_t window, float scale, int schedule, const ra_tensor_t* o, float* lse,
                               const ra_stream_t* streams, int n_streams, void* workspace, size_t workspace_bytes) {
  if (window < 1) return fail(RA_ERR_INVALID_ARG, "window must be >= 1 (got %lld)", (long long)window);
  return ring_fwd_impl(q, k, v, P, layout, 1, window, scale, schedule, o, lse, streams, n_streams, workspace,
                       workspace_bytes);
}

// A contiguous [B, H, N, d] tensor: stride = (H*N*d, N*d, d, 1).
static bool packed_4d(const ra_tensor_t* t) {
  return t->stride[3] == 1 && t->stride[2] == t->shape[3] && t->stride[1] == t->shape[2] * t->shape[3] &&
         (t->shape[0] == 1 || t->stride[0] == t->shape[1] * t->shape[2] * t->shape[3]);
}

// Heads [h0, h0 + nh) of the flattened B*H heads of a contiguous tensor, as a [1, nh, N, d] view.
static ra_tensor_t head_chunk(const ra_tensor_t* t, int64_t h0, int64_t nh) {
  ra_tensor_t c = *t;
  const int64_t per_head = t->shape[2] * t->shape[3];
  const size_t elem = t->dtype == RA_BF16 ? 2 : 4;
  c.data = static_cast<char*>(t->data) + static_cast<size_t>(h0 * per_head) * elem;
  c.shape[0] = 1;
  c.shape[1] = nh;
  c.stride[0] = nh * per_head;
  c.stride[1] = per_head;
  return c;
}

ra_status_t ra_ring_fwd_host(const ra_tensor_t* q_host, const ra_tensor_t* k_host, const ra_tensor_t* v_host, int P,
                             int layout, int causal, float scale, const ra_tensor_t* o_host, float* lse_host,
                             const ra_tensor_t* q_dev, const ra_tensor_t* k_dev, const ra_tensor_t* v_dev,
                             const ra_tensor_t* o_dev, float* lse_dev, int n_chunks, const ra_stream_t* streams) {
  const ra_tensor_t* hosts[4] = {q_host, k_host, v_host, o_host};
  const ra_tensor_t* devs[4] = {q_dev, k_dev, v_dev, o_dev};
  const char* names[4] = {"q", "k", "v", "o"};
  ra_status_t st;
  for (int i = 0; i < 4; ++i) {
    if ((st = check_tensor(hosts[i], names[i])) != RA_OK) return st;
    if ((st = check_tensor(devs[i], names[i])) != RA_OK) return st;
    if (!packed_4d(hosts[i]) || !packed_4d(devs[i]))
      return fail(RA_ERR_UNSUPPORTED, "%s: host and device tensors must be contiguous [B, H, N, d]", names[i]);
    if (hosts[i]->dtype != devs[i]->dtype)
      return fail(RA_ERR_INVALID_ARG, "%s: host and device tensors differ in dtype", names[i]);
    for (int a = 0; a < 4; ++a)
      if (hosts[i]->shape[a] != devs[i]->shape[a])
        return fail(RA_ERR_INVALID_ARG, "%s: host and device tensors differ in shape", names[i]);
  }
  if ((lse_host == nullptr) != (lse_dev == nullptr))
    return fail(RA_ERR_INVALID_ARG, "lse_host and lse_dev must both be given or both be NULL");
  if (streams == nullptr || streams[0] == streams[1] || streams[1] == streams[2] || streams[0] == streams[2])
    return fail(RA_ERR_INVALID_ARG, "three distinct streams are needed (copy in, compute, copy out)");
  if (n_chunks < 1) return fail(RA_ERR_INVALID_ARG, "n_chunks must be >= 1");
  const int64_t kv_heads = k_dev->shape[0] * k_dev->shape[1];  // flattened K/V heads
  if (k_dev->shape[1] < 1 || q_dev->shape[1] % k_dev->shape[1] != 0)
    return fail(RA_ERR_INVALID_ARG, "H_kv must divide H");
  const int64_t qpk = q_dev->shape[1] / k_dev->shape[1];
  const int64_t chunks = n_chunks < kv_heads ? n_chunks : kv_heads;
  // Chunk c: K/V heads [c*G/n, (c+1)*G/n) of the flattened B*H_kv, and their qpk query heads each.
  auto bounds = [&](int64_t c, int64_t* k0, int64_t* nk) {
    *k0 = c * kv_heads / chunks;
    *nk = (c + 1) * kv_heads / chunks - *k0;
  };
  // Every check of the per-chunk ring call before anything is enqueued (chunks differ only in
  // their head count, so the first and the largest one cover them all).
  const ra_stream_t compute[1] = {streams[1]};
  for (int64_t c : {int64_t(0), chunks - 1}) {
    int64_t k0, nk;
    bounds(c, &k0, &nk);
    ra_tensor_t qc = head_chunk(q_dev, k0 * qpk, nk * qpk), kc = head_chunk(k_dev, k0, nk),
                vc = head_chunk(v_dev, k0, nk), oc = head_chunk(o_dev, k0 * qpk, nk * qpk);
    if ((st = ring_fwd_impl(&qc, &kc, &vc, P, layout, causal, 0, scale, RA_RING_FUSED, &oc,
                            lse_dev ? lse_dev + k0 * qpk * q_dev->shape[2] : nullptr, compute, 1, nullptr, 0,
                            true)) != RA_OK)
      return st;
  }
  const cudaStream_t s_in = reinterpret_cast<cudaStream_t>(streams[0]);
  const cudaStream_t s_cmp = reinterpret_cast<cudaStream_t>(streams[1]);
  const cudaStream_t s_out = reinterpret_cast<cudaStream_t>(streams[2]);
  std::vector<cudaEvent_t> ev(2 * chunks + 2, nullptr);
  cudaError_t e = cudaSuccess;
  for (auto& x : ev)
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming);
  auto destroy = [&ev] {
    for (cudaEvent_t x : ev)
      if (x) cudaEventDestroy(x);
  };
  if (e != cudaSuccess) {
    destroy();
    return cuda_fail(e, "event");
  }
  // The copies wait for work already queued on the compute stream (which may still use the
  // device buffers).
  e = cudaEventRecord(ev[2 * chunks], s_cmp);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s_in, ev[2 * chunks], 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev[2 * chunks], 0);
  if (e != cudaSuccess) {
    destroy();
    return cuda_fail(e, "stream fork");
  }
  const size_t lse_row = static_cast<size_t>(q_dev->shape[2]) * sizeof(float);
  for (int64_t c = 0; c < chunks && st == RA_OK; ++c) {
    int64_t k0, nk;
    bounds(c, &k0, &nk);
    const ra_tensor_t qh = head_chunk(q_host, k0 * qpk, nk * qpk), kh = head_chunk(k_host, k0, nk),
                      vh = head_chunk(v_host, k0, nk), oh = head_chunk(o_host, k0 * qpk, nk * qpk);
    ra_tensor_t qc = head_chunk(q_dev, k0 * qpk, nk * qpk), kc = head_chunk(k_dev, k0, nk),
                vc = head_chunk(v_dev, k0, nk), oc = head_chunk(o_dev, k0 * qpk, nk * qpk);
    const size_t elem = q_dev->dtype == RA_BF16 ? 2 : 4;
    const size_t qbytes = static_cast<size_t>(nk * qpk * q_dev->shape[2] * q_dev->shape[3]) * elem;
    const size_t kbytes = static_cast<size_t>(nk * k_dev->shape[2] * k_dev->shape[3]) * elem;
    e = cudaMemcpyAsync(qc.data, qh.data, qbytes, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess) e = cudaMemcpyAsync(kc.data, kh.data, kbytes, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess) e = cudaMemcpyAsync(vc.data, vh.data, kbytes, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess) e = cudaEventRecord(ev[2 * c], s_in);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_cmp, ev[2 * c], 0);
    if (e != cudaSuccess) {
      st = cuda_fail(e, "host-to-device copy");
      break;
    }
    float* lc = lse_dev ? lse_dev + k0 * qpk * q_dev->shape[2] : nullptr;
    if ((st = ring_fwd_impl(&qc, &kc, &vc, P, layout, causal, 0, scale, RA_RING_FUSED, &oc, lc, compute, 1, nullptr,
                            0)) != RA_OK)
      break;
    e = cudaEventRecord(ev[2 * c + 1], s_cmp);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev[2 * c + 1], 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(oh.data, oc.data, qbytes, cudaMemcpyDeviceToHost, s_out);
    if (e == cudaSuccess && lse_host)
      e = cudaMemcpyAsync(lse_host + k0 * qpk * q_dev->shape[2], lc, static_cast<size_t>(nk * qpk) * lse_row,
                          cudaMemcpyDeviceToHost, s_out);
    if (e != cudaSuccess) st = cuda_fail(e, "device-to-host copy");
  }
  // Later work on the compute stream is ordered after the whole call, the copies out included.
  e = cudaEventRecord(ev[2 * chunks + 1], s_out);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s_cmp, ev[2 * chunks + 1], 0);
  destroy();
  if (st != RA_OK) return st;
  if (e != cudaSuccess) return cuda_fail(e, "stream join");
  return ok();
}

ra_status_t ra_attn_bwd(const ra_tensor_t* q, const ra_tensor_t* k, const ra_tensor_t* v, const ra_tensor_t* o,
                        const float* lse, const ra_tensor_t* d_o, const ra_tensor_t* dq, const ra_tensor_t* dk,
                        const ra_tensor_t* dv, float scale, int causal, int64_t window, ra_stream_t stream) {
  ra_status_t st = check_qkv(q, k, v);
  if (st != RA_OK) return st;
  if ((st = check_tensor(o, "o")) != RA_OK) return st;
  if ((st = check_tensor(d_o, "d_o")) != RA_OK) return st;
  if ((st = check_tensor(dq, "dq")) != RA_OK) return st;
  if ((st = check_tensor(dk, "dk")) != RA_OK) return st;
  if ((st = check_tensor(dv, "dv")) != RA_OK) return st;
  if (lse == nullptr) return fail(RA_ERR_INVALID_ARG, "lse is NULL (the forward's saved log-sum-exp is required)");
  if (o->dtype != q->dtype || d_o->dtype != q->dtype) return fail(RA_ERR_INVALID_ARG, "o and d_o must have q's dtype");
  if (dq->dtype != RA_F32 || dk->dtype != RA_F32 || dv->dtype != RA_F32)
    return fail(RA_ERR_INVALID_ARG, "dq, dk, dv must be fp32");
  for (int i = 0; i < 4; ++i) {
    if (o->shape[i] != q->shape[i] || d_o->shape[i] != q->shape[i] || dq->shape[i] != q->shape[i])
      return fail(RA_ERR_INVALID_ARG, "o, d_o and dq must have the shape of q");
    if (dk->shape[i] != k->shape[i] || dv->shape[i] != k->shape[i])
      return fail(RA_ERR_INVALID_ARG, "dk and dv must have the shape of k");
  }
  if (window < 0 || (window > 0 && !causal)) return fail(RA_ERR_INVALID_ARG, "window must be 0 or, with causal, >= 1");
  DevInfo dev;
  if ((st = current_device(&dev)) != RA_OK) return st;
  ra::BwdWork w{};
  w.B = static_cast<int>(q->shape[0]);
  w.H = static_cast<int>(q->shape[1]);
  w.H_kv = static_cast<int>(k->shape[1]);
  w.n_q = static_cast<int>(q->shape[2]);
  w.n_kv = static_cast<int>(k->shape[2]);
  w.d = static_cast<int>(q->shape[3]);
  w.causal = causal != 0;
  w.window = window;
  w.scale = scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(w.d));
  auto set = [](const ra_tensor_t* t, long long& sb, long long& sh, long long& st) {
    sb = t->stride[0];
    sh = t->stride[1];
    st = t->stride[2];
  };
  w.q = q->data;
  set(q, w.q_sb, w.q_sh, w.q_st);
  w.k = k->data;
  set(k, w.k_sb, w.k_sh, w.k_st);
  w.v = v->data;
  set(v, w.v_sb, w.v_sh, w.v_st);
  w.o = o->data;
  set(o, w.o_sb, w.o_sh, w.o_st);
  w.d_o = d_o->data;
  set(d_o, w.do_sb, w.do_sh, w.do_st);
  w.lse = lse;
  w.dq = static_cast<float*>(dq->data);
  set(dq, w.dq_sb, w.dq_sh, w.dq_st);
  w.dk = static_cast<float*>(dk->data);
  set(dk, w.dk_sb, w.dk_sh, w.dk_st);
  w.dv = static_cast<float*>(dv->data);
  set(dv, w.dv_sb, w.dv_sh, w.dv_st);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int dp = padded_dim(w.d);
  if (q->dtype == RA_BF16 && w.H % w.H_kv == 0 && check_head_dim(w.d, RA_BF16) == RA_OK &&
      check_tma_tensor(q, "q") == RA_OK && check_tma_tensor(k, "k") == RA_OK && check_tma_tensor(v, "v") == RA_OK &&
      check_tma_tensor(o, "o") == RA_OK && check_tma_tensor(d_o, "d_o") == RA_OK) {
    // Tensor-core path: dQ over blocks of 128 query rows, dK/dV over blocks of 128 keys.
    ra::BwdMaps m;
    struct {
      CUtensorMap* map;
      const ra_tensor_t* t;
      int rows;
    } maps[] = {{&m.q128, q, 128}, {&m.k128, k, 128}, {&m.v128, v, 128}, {&m.do128, d_o, 128}, {&m.q64, q, 64},
                {&m.k64, k, 64},   {&m.v64, v, 64},   {&m.do64, d_o, 64}, {&m.o64, o, 64}};
    for (auto& e : maps)
      if ((st = encode_view(e.map, shard_view(e.t, e.t->shape[2], 1, 0, 1), dp, e.rows)) != RA_OK) return st;
    ra::BwdTcWork tw{};
    tw.B = w.B;
    tw.H = w.H;
    tw.H_kv = w.H_kv;
    tw.n_q = w.n_q;
    tw.n_kv = w.n_kv;
    tw.d = w.d;
    tw.qpk = w.H / w.H_kv;
    tw.causal = w.causal;
    tw.window = w.window;
    tw.scale = w.scale;
    tw.scale_log2 = static_cast<float>(w.scale * kLog2e);
    tw.lse = lse;
    tw.o = static_cast<const __nv_bfloat16*>(o->data);
    tw.o_sb = w.o_sb;
    tw.o_sh = w.o_sh;
    tw.o_st = w.o_st;
    tw.d_o = static_cast<const __nv_bfloat16*>(d_o->data);
    tw.do_sb = w.do_sb;
    tw.do_sh = w.do_sh;
    tw.do_st = w.do_st;
    tw.wait_limit_ns = g_wait_limit_ns.load();
    tw.dev_status = dev.status;
    ra::BwdTcWork wq = tw, wkv = tw;
    // One heavy-first order over all heads for causal launches of at most 32 waves of CTAs (load
    // balance matters there; longer launches balance anyway and keep each head's CTAs together).
    {
      const long long waves = 32LL * (dev.sms > 0 ? dev.sms : 148);
      const long long cq = static_cast<long long>((w.n_q + 127) / 128) * w.H * w.B;
      const long long ckv = static_cast<long long>((w.n_kv + 127) / 128) * w.H_kv * w.B;
      wq.global_order = w.causal && cq <= waves;
      wkv.global_order = w.causal && ckv <= waves;
    }
    wq.out1 = w.dq;
    wq.o1_sb = w.dq_sb;
    wq.o1_sh = w.dq_sh;
    wq.o1_st = w.dq_st;
    wkv.out1 = w.dk;
    wkv.o1_sb = w.dk_sb;
    wkv.o1_sh = w.dk_sh;
    wkv.o1_st = w.dk_st;
    wkv.out2 = w.dv;
    wkv.o2_sb = w.dv_sb;
    wkv.o2_sh = w.dv_sh;
    wkv.o2_st = w.dv_st;
    cudaError_t e = dp == 32 ? ra::launch_bwd_dp32(m, wq, wkv, s)
                    : dp == 64 ? ra::launch_bwd_dp64(m, wq, wkv, s)
                               : ra::launch_bwd_dp128(m, wq, wkv, s);
    if (e != cudaSuccess) return cuda_fail(e, "backward kernel launch");
    return ok();
  }
  const dim3 gq((w.n_q + ra::kBwdRows - 1) / ra::kBwdRows, w.H, w.B);
  const dim3 gk((w.n_kv + ra::kBwdRows - 1) / ra::kBwdRows, w.H_kv, w.B);
  const unsigned threads = static_cast<unsigned>(ra::kBwdRows * (dp / ra::kBwdDH));
#define RA_BWD_LAUNCH(T, DPV)                                  \
  do {                                                         \
    ra::attn_bwd_dq<T, DPV><<<gq, threads, 0, s>>>(w);         \
    ra::attn_bwd_dkv<T, DPV><<<gk, threads, 0, s>>>(w);        \
  } while (0)
  if (q->dtype == RA_BF16) {
    if (dp == 32) RA_BWD_LAUNCH(__nv_bfloat16, 32);
    else if (dp == 64) RA_BWD_LAUNCH(__nv_bfloat16, 64);
    else RA_BWD_LAUNCH(__nv_bfloat16, 128);
  } else {
    if (dp == 32) RA_BWD_LAUNCH(float, 32);
    else if (dp == 64) RA_BWD_LAUNCH(float, 64);
    else RA_BWD_LAUNCH(float, 128);
  }
#undef RA_BWD_LAUNCH
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "backward kernel launch");
  return ok();
}

ra_status_t ra_get_device_status(ra_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned int words[2] = {0, 0};
  const unsigned int zero[2] = {0, 0};
  if ((e = cudaMemcpyFromSymbol(words, ra::g_dev_status, sizeof(words))) != cudaSuccess)
    return cuda_fail(e, "read status");
  if (words[0] != 0) {
    if ((e = cudaMemcpyToSymbol(ra::g_dev_status, zero, sizeof(zero))) != cudaSuccess) return cuda_fail(e, "clear");
    if (words[0] & ra::kDevStatusTimeout)
      return fail(RA_ERR_TIMEOUT, "a device-side wait ran out (site 0x%x)", words[1]);
  }
  return ok();
}

ra_status_t ra_set_wait_timeout_ns(uint64_t ns) {
  if (ns < 1000 || ns > 60ull * 1000000000ull) return fail(RA_ERR_INVALID_ARG, "timeout must be in [1 us, 60 s]");
  g_wait_limit_ns.store(ns);
  return ok();
}

ra_status_t ra_set_striped_walk(int order) {
  if (order != RA_WALK_SHARD_MAJOR && order != RA_WALK_TILE_MAJOR)
    return fail(RA_ERR_INVALID_ARG, "walk order must be RA_WALK_SHARD_MAJOR or RA_WALK_TILE_MAJOR");
  g_striped_walk.store(order);
  return ok();
}

ra_status_t ra_debug_unarrived_wait(uint64_t timeout_ns, ra_stream_t stream) {
  if (timeout_ns < 1000 || timeout_ns > 10ull * 1000000000ull)
    return fail(RA_ERR_INVALID_ARG, "timeout must be in [1 us, 10 s]");
  DevInfo dev;
  ra_status_t st = current_device(&dev);
  if (st != RA_OK) return st;
  ra::unarrived_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(timeout_ns, dev.status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch");
  return ok();
}

ra_status_t ra_debug_exp2(const float* x, float* y_poly, float* y_mufu, int64_t n, ra_stream_t stream) {
  if (n < 0) return fail(RA_ERR_INVALID_ARG, "n < 0");
  if (n == 0) return ok();
  if (x == nullptr) return fail(RA_ERR_INVALID_ARG, "x is NULL");
  DevInfo dev;
  ra_status_t st = current_device(&dev);
  if (st != RA_OK) return st;
  long long blocks = (n + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  ra::exp2_probe_kernel<<<static_cast<unsigned>(blocks), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      x, y_poly, y_mufu, static_cast<long long>(n));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch");
  return ok();
}

const char* ra_status_string(ra_status_t s) {
  switch (s) {
    case RA_OK: return "RA_OK";
    case RA_ERR_INVALID_ARG: return "RA_ERR_INVALID_ARG";
    case RA_ERR_UNSUPPORTED: return "RA_ERR_UNSUPPORTED";
    case RA_ERR_ALIGNMENT: return "RA_ERR_ALIGNMENT";
    case RA_ERR_WORKSPACE: return "RA_ERR_WORKSPACE";
    case RA_ERR_CUDA: return "RA_ERR_CUDA";
    case RA_ERR_TIMEOUT: return "RA_ERR_TIMEOUT";
  }
  return "RA_ERR_UNKNOWN";
}

const char* ra_last_error(void) { return t_last_error.c_str(); }

int ra_version(void) { return kVersion; }

}  // extern "C"
