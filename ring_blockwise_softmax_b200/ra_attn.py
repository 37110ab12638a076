"""ctypes binding of the C ABI in ``include/ra_attn.h`` (``libra_attn.so``, built in-tree).

Argument marshalling only: every step of the computation runs in the library's CUDA kernels.
Tensors are torch CUDA tensors, used for their device memory; streams are torch streams (or
raw ``cudaStream_t`` integers).  Importing this module loads the library and raises
``ImportError`` if it has not been built (``python -m ring_blockwise_softmax_b200.build``);
there is no fallback path.
"""

from __future__ import annotations

import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libra_attn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m ring_blockwise_softmax_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

RA_OK = 0
RA_ERR_INVALID_ARG = 1
RA_ERR_UNSUPPORTED = 2
RA_ERR_ALIGNMENT = 3
RA_ERR_WORKSPACE = 4
RA_ERR_CUDA = 5
RA_ERR_TIMEOUT = 6

RA_F32 = 0
RA_BF16 = 1
RA_CONTIGUOUS = 0
RA_STRIPED = 1
RA_RING_STEPWISE = 0
RA_RING_FUSED = 1
RA_MERGE_MAX_PARTS = 32

LAYOUTS = {"contiguous": RA_CONTIGUOUS, "striped": RA_STRIPED}
SCHEDULES = {"stepwise": RA_RING_STEPWISE, "fused": RA_RING_FUSED}

# Exported symbols of the library, in header order (the CPU test checks each one is present).
SYMBOLS = (
    "ra_attn_fwd", "ra_attn_fwd_window", "ra_attn_bwd", "ra_attn_partial", "ra_lse_merge", "ra_lse_merge_n", "ra_ring_workspace_size",
    "ra_ring_fwd", "ra_ring_fwd_window", "ra_ring_fwd_host", "ra_ring_fwd_noalloc", "ra_get_device_status", "ra_set_wait_timeout_ns", "ra_set_striped_walk", "ra_debug_unarrived_wait",
    "ra_debug_exp2", "ra_status_string", "ra_last_error", "ra_version",
)


class RaTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class RaPos(ctypes.Structure):
    _fields_ = [("offset", ctypes.c_int64), ("stride", ctypes.c_int64)]


_T = ctypes.POINTER(RaTensor)
_F = ctypes.c_void_p  # float* (device)
_S = ctypes.c_void_p  # cudaStream_t

_lib.ra_attn_fwd.argtypes = [_T, _T, _T, _T, _F, ctypes.c_float, ctypes.c_int, _S]
_lib.ra_attn_fwd_window.argtypes = [_T, _T, _T, _T, _F, ctypes.c_float, ctypes.c_int64, _S]
_lib.ra_attn_bwd.argtypes = [_T, _T, _T, _T, _F, _T, _T, _T, _T, ctypes.c_float, ctypes.c_int, ctypes.c_int64, _S]
_lib.ra_attn_partial.argtypes = [_T, _T, _T, RaPos, RaPos, ctypes.c_int, ctypes.c_float, _T, _F, ctypes.c_int, _S]
_lib.ra_lse_merge.argtypes = [_F, _F, _F, _F, _F, _F, ctypes.c_int64, ctypes.c_int, _S]
_lib.ra_lse_merge_n.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_void_p), ctypes.c_int, _F,
                                _F, ctypes.c_int64, ctypes.c_int, _S]
_lib.ra_ring_workspace_size.argtypes = [_T, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)]
_lib.ra_ring_fwd.argtypes = [_T, _T, _T, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int, _T,
                             _F, ctypes.POINTER(ctypes.c_void_p), ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t]
_lib.ra_ring_fwd_window.argtypes = [_T, _T, _T, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_int,
                                    _T, _F, ctypes.POINTER(ctypes.c_void_p), ctypes.c_int, ctypes.c_void_p,
                                    ctypes.c_size_t]
_lib.ra_ring_fwd_host.argtypes = [_T, _T, _T, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, _T, _F, _T, _T,
                                  _T, _T, _F, ctypes.c_int, ctypes.POINTER(ctypes.c_void_p)]
_lib.ra_ring_fwd_noalloc.argtypes = [_T, _T, _T, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, _T, _F,
                                     _S]
_lib.ra_get_device_status.argtypes = [_S]
_lib.ra_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
_lib.ra_set_striped_walk.argtypes = [ctypes.c_int]
_lib.ra_debug_unarrived_wait.argtypes = [ctypes.c_uint64, _S]
_lib.ra_debug_exp2.argtypes = [_F, _F, _F, ctypes.c_int64, _S]
_lib.ra_status_string.argtypes = [ctypes.c_int]
_lib.ra_status_string.restype = ctypes.c_char_p
_lib.ra_last_error.argtypes = []
_lib.ra_last_error.restype = ctypes.c_char_p
_lib.ra_version.argtypes = []
for _name in SYMBOLS:
    if _name not in ("ra_status_string", "ra_last_error"):
        getattr(_lib, _name).restype = ctypes.c_int


class RaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.ra_last_error().decode(errors="replace")
        super().__init__(f"{where}: {status_string(status)}: {msg}")


def _check(status: int, where: str):
    if status != RA_OK:
        raise RaError(status, where)


def status_string(status: int) -> str:
    return _lib.ra_status_string(int(status)).decode()


def version() -> int:
    return int(_lib.ra_version())


def lib_handle():
    return _lib


# ---------------------------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------------------------

def _dtype_code(t) -> int:
    import torch

    if t.dtype == torch.float32:
        return RA_F32
    if t.dtype == torch.bfloat16:
        return RA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def tensor_desc(t) -> RaTensor:
    """Describe a 4-D torch tensor [B, H, N, d] (any strides) for the C ABI."""
    if t.dim() != 4:
        raise ValueError("expected a 4-D tensor [B, H, N, d]")
    d = RaTensor()
    d.data = t.data_ptr()
    d.dtype = _dtype_code(t)
    d.reserved = 0
    for i in range(4):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return d


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch

        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


# ---------------------------------------------------------------------------------------------
# entry points (same names as the C ABI, without the ra_ prefix)
# ---------------------------------------------------------------------------------------------

def attn_fwd(q, k, v, o, lse=None, scale: float = 0.0, causal: bool = False, stream=None, window: int = 0):
    """ra_attn_fwd: O (and LSE, natural log) of softmax(scale*QK^T)V into the given buffers.
    window > 0: ra_attn_fwd_window (causal sliding window of that many positions)."""
    tq, tk, tv, to = (tensor_desc(x) for x in (q, k, v, o))
    if window:
        _check(_lib.ra_attn_fwd_window(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), ctypes.byref(to),
                                       _ptr(lse), float(scale), int(window), _stream(stream)), "ra_attn_fwd_window")
        return
    _check(_lib.ra_attn_fwd(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), ctypes.byref(to), _ptr(lse),
                            float(scale), int(bool(causal)), _stream(stream)), "ra_attn_fwd")


def attn_bwd(q, k, v, o, lse, d_o, dq, dk, dv, scale: float = 0.0, causal: bool = False, window: int = 0,
             stream=None):
    """ra_attn_bwd: fp32 dq, dk, dv of sum(d_o * O) from the forward's O and LSE (overwritten)."""
    tq, tk, tv, to, tdo, tdq, tdk, tdv = (tensor_desc(x) for x in (q, k, v, o, d_o, dq, dk, dv))
    _check(_lib.ra_attn_bwd(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), ctypes.byref(to), _ptr(lse),
                            ctypes.byref(tdo), ctypes.byref(tdq), ctypes.byref(tdk), ctypes.byref(tdv), float(scale),
                            int(bool(causal)), int(window), _stream(stream)), "ra_attn_bwd")


def attention_backward(q, k, v, o, lse, d_o, causal: bool = False, scale: float = 0.0, window: int = 0, stream=None):
    """Allocate fp32 dq, dk, dv, run ra_attn_bwd, return (dq, dk, dv)."""
    import torch

    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty(k.shape, dtype=torch.float32, device=q.device)
    dv = torch.empty(v.shape, dtype=torch.float32, device=q.device)
    attn_bwd(q, k, v, o, lse, d_o, dq, dk, dv, scale, causal, window, stream)
    return dq, dk, dv


def attn_partial(q, k_shard, v_shard, o_part, lse_part, q_pos=(0, 1), kv_pos=(0, 1), causal: bool = False,
                 scale: float = 0.0, accumulate: bool = False, stream=None):
    """ra_attn_partial: fp32 (O_part, LSE_part) of q against one KV shard, written or LSE-merged."""
    tq, tk, tv, to = (tensor_desc(x) for x in (q, k_shard, v_shard, o_part))
    _check(_lib.ra_attn_partial(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), RaPos(*q_pos), RaPos(*kv_pos),
                                int(bool(causal)), float(scale), ctypes.byref(to), _ptr(lse_part),
                                int(bool(accumulate)), _stream(stream)), "ra_attn_partial")


def lse_merge(o_a, lse_a, o_b, lse_b, o_out, lse_out, stream=None):
    """ra_lse_merge over rows of contiguous fp32 [rows, d] / [rows] tensors."""
    d = o_a.shape[-1]
    rows = o_a.numel() // d
    _check(_lib.ra_lse_merge(_ptr(o_a), _ptr(lse_a), _ptr(o_b), _ptr(lse_b), _ptr(o_out), _ptr(lse_out), rows, d,
                             _stream(stream)), "ra_lse_merge")


def lse_merge_n(o_parts, lse_parts, o_out, lse_out, stream=None):
    """ra_lse_merge_n of k partials (lists of contiguous fp32 tensors) in one pass."""
    k = len(o_parts)
    d = o_parts[0].shape[-1]
    rows = o_parts[0].numel() // d
    op = (ctypes.c_void_p * max(k, 1))(*[x.data_ptr() for x in o_parts])
    lp = (ctypes.c_void_p * max(k, 1))(*[x.data_ptr() for x in lse_parts])
    _check(_lib.ra_lse_merge_n(op, lp, k, _ptr(o_out), _ptr(lse_out), rows, d, _stream(stream)), "ra_lse_merge_n")


def ring_workspace_size(q, P: int, schedule: str = "stepwise") -> int:
    tq = tensor_desc(q)
    out = ctypes.c_size_t(0)
    _check(_lib.ra_ring_workspace_size(ctypes.byref(tq), int(P), SCHEDULES[schedule], ctypes.byref(out)),
           "ra_ring_workspace_size")
    return int(out.value)


def ring_fwd(q, k, v, P: int, layout: str, causal: bool, o, lse=None, scale: float = 0.0,
             schedule: str = "stepwise", streams=None, workspace=None, window: int = 0):
    """ra_ring_fwd: ring attention over P virtual shards (contiguous or striped) on one GPU.
    window > 0: ra_ring_fwd_window (causal sliding window of that many positions)."""
    import torch

    if streams is None:
        streams = [torch.cuda.current_stream()]
    arr = (ctypes.c_void_p * len(streams))(*[(s if isinstance(s, int) else s.cuda_stream) for s in streams])
    tq, tk, tv, to = (tensor_desc(x) for x in (q, k, v, o))
    ws_ptr = None if workspace is None else ctypes.c_void_p(workspace.data_ptr())
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if window:
        _check(_lib.ra_ring_fwd_window(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), int(P), LAYOUTS[layout],
                                       int(window), float(scale), SCHEDULES[schedule], ctypes.byref(to), _ptr(lse),
                                       arr, len(streams), ws_ptr, ws_bytes), "ra_ring_fwd_window")
        return
    _check(_lib.ra_ring_fwd(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), int(P), LAYOUTS[layout],
                            int(bool(causal)), float(scale), SCHEDULES[schedule], ctypes.byref(to), _ptr(lse), arr,
                            len(streams), ws_ptr, ws_bytes), "ra_ring_fwd")


def ring_fwd_host(q_host, k_host, v_host, P: int, layout: str, causal: bool, o_host, lse_host, q_dev, k_dev, v_dev,
                  o_dev, lse_dev, scale: float = 0.0, n_chunks: int = 8, streams=None):
    """ra_ring_fwd_host: host-resident inputs and outputs (pinned for overlap), device staging
    tensors of the same shapes, three streams (copy in, compute, copy out; default: new ones)."""
    import torch

    if streams is None:
        streams = [torch.cuda.Stream(device=q_dev.device) for _ in range(3)]
    arr = (ctypes.c_void_p * 3)(*[(s if isinstance(s, int) else s.cuda_stream) for s in streams])
    ts = [tensor_desc(x) for x in (q_host, k_host, v_host, o_host, q_dev, k_dev, v_dev, o_dev)]
    _check(_lib.ra_ring_fwd_host(ctypes.byref(ts[0]), ctypes.byref(ts[1]), ctypes.byref(ts[2]), int(P), LAYOUTS[layout],
                                 int(bool(causal)), float(scale), ctypes.byref(ts[3]), _ptr(lse_host),
                                 ctypes.byref(ts[4]), ctypes.byref(ts[5]), ctypes.byref(ts[6]), ctypes.byref(ts[7]),
                                 _ptr(lse_dev), int(n_chunks), arr), "ra_ring_fwd_host")
    return streams


NOALLOC_SCRATCH_BYTES = 32 << 20


def ring_fwd_noalloc(q, k, v, P: int, layout: str, causal: bool, o, lse=None, scale: float = 0.0, stream=None):
    """ra_ring_fwd_noalloc: the stepwise ring with the library's fixed scratch (no workspace)."""
    tq, tk, tv, to = (tensor_desc(x) for x in (q, k, v, o))
    _check(_lib.ra_ring_fwd_noalloc(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), int(P), LAYOUTS[layout],
                                    int(bool(causal)), float(scale), ctypes.byref(to), _ptr(lse), _stream(stream)),
           "ra_ring_fwd_noalloc")


def get_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status (RA_OK or RA_ERR_TIMEOUT)."""
    return int(_lib.ra_get_device_status(_stream(stream)))


def set_wait_timeout_ns(ns: int):
    _check(_lib.ra_set_wait_timeout_ns(int(ns)), "ra_set_wait_timeout_ns")


WALKS = {"shard": 0, "tile": 1}  # RA_WALK_SHARD_MAJOR, RA_WALK_TILE_MAJOR


def set_striped_walk(order: str):
    """ra_set_striped_walk: "shard" (default) or "tile", the K/V walk of fused rings over striped shards."""
    _check(_lib.ra_set_striped_walk(WALKS[order]), "ra_set_striped_walk")


def debug_unarrived_wait(timeout_ns: int, stream=None):
    _check(_lib.ra_debug_unarrived_wait(int(timeout_ns), _stream(stream)), "ra_debug_unarrived_wait")


def debug_exp2(x, y_poly=None, y_mufu=None, stream=None):
    """ra_debug_exp2 on contiguous fp32 device tensors."""
    _check(_lib.ra_debug_exp2(_ptr(x), _ptr(y_poly), _ptr(y_mufu), x.numel(), _stream(stream)), "ra_debug_exp2")


# ---------------------------------------------------------------------------------------------
# conveniences that allocate outputs with torch (device memory only; compute stays in the lib)
# ---------------------------------------------------------------------------------------------

def attention(q, k, v, causal: bool = False, scale: float = 0.0, stream=None, window: int = 0):
    """Allocate O (dtype of q) and fp32 LSE, run ra_attn_fwd (ra_attn_fwd_window when window > 0),
    return (O, LSE)."""
    import torch

    B, H, N, d = q.shape
    o = torch.empty((B, H, N, d), dtype=q.dtype, device=q.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    attn_fwd(q, k, v, o, lse, scale, causal, stream, window)
    return o, lse


def ring_attention(q, k, v, P: int, layout: str = "contiguous", causal: bool = False, scale: float = 0.0,
                   schedule: str = "stepwise", streams=None, window: int = 0):
    """Allocate O, LSE and the workspace, run ra_ring_fwd (ra_ring_fwd_window when window > 0),
    return (O, LSE)."""
    import torch

    B, H, N, d = q.shape
    o = torch.empty((B, H, N, d), dtype=q.dtype, device=q.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    nbytes = ring_workspace_size(q, P, schedule)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device) if nbytes > 0 else None
    ring_fwd(q, k, v, P, layout, causal, o, lse, scale, schedule, streams, ws, window)
    return o, lse


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
