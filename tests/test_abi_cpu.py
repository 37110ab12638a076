"""CPU checks of the C ABI: the library builds, loads, exports every declared entry point, and
rejects bad arguments on the host before touching a device.  No kernel is launched here."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ra():
    from ring_blockwise_softmax_b200 import build

    build.build()
    from ring_blockwise_softmax_b200 import ra_attn

    return ra_attn


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            with open(os.path.join(ROOT, "include", fn), encoding="utf-8") as f:
                src = f.read()
            names.update(re.findall(r"^\s*(?:ra_status_t|const char\*|int)\s+(ra_\w+)\s*\(", src, re.M))
    return sorted(names)


def test_header_declares_the_boundary():
    names = _declared_symbols()
    for want in ("ra_attn_fwd", "ra_attn_partial", "ra_lse_merge", "ra_lse_merge_n", "ra_ring_fwd",
                 "ra_ring_workspace_size", "ra_get_device_status", "ra_status_string"):
        assert want in names


def test_library_exports_every_declared_symbol(ra):
    lib = ctypes.CDLL(ra.LIB_PATH)
    for name in _declared_symbols():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert set(ra.SYMBOLS) == set(_declared_symbols())


def test_status_strings_and_version(ra):
    assert ra.status_string(ra.RA_OK) == "RA_OK"
    assert ra.status_string(ra.RA_ERR_TIMEOUT) == "RA_ERR_TIMEOUT"
    assert ra.version() >= 10000


def test_host_validation_without_a_device(ra):
    import torch

    lib = ra.lib_handle()
    # NULL tensors are rejected before any CUDA call.
    st = lib.ra_attn_fwd(None, None, None, None, None, ctypes.c_float(0.0), 0, None)
    assert st == ra.RA_ERR_INVALID_ARG
    assert b"q is NULL" in lib.ra_last_error()
    # A CPU tensor is described like any other; shape errors are found on the host.
    q = torch.zeros(1, 2, 16, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 3, 16, 64, dtype=torch.bfloat16)
    tq, tk = ra.tensor_desc(q), ra.tensor_desc(k)
    st = lib.ra_attn_fwd(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tk), ctypes.byref(tq), None,
                         ctypes.c_float(0.0), 0, None)
    assert st == ra.RA_ERR_INVALID_ARG and b"H_kv must divide" in lib.ra_last_error()
    # grouped-query K/V: H_kv must divide H, and k, v must agree on it; B must agree
    q4 = torch.zeros(1, 4, 16, 64, dtype=torch.bfloat16)
    k2 = torch.zeros(1, 2, 16, 64, dtype=torch.bfloat16)
    v1 = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16)
    kb = torch.zeros(2, 2, 16, 64, dtype=torch.bfloat16)
    tq4, tk2, tv1, tkb = (ra.tensor_desc(x) for x in (q4, k2, v1, kb))
    st = lib.ra_attn_fwd(ctypes.byref(tq4), ctypes.byref(tk2), ctypes.byref(tv1), ctypes.byref(tq4), None,
                         ctypes.c_float(0.0), 0, None)
    assert st == ra.RA_ERR_INVALID_ARG and b"same number of heads" in lib.ra_last_error()
    st = lib.ra_attn_fwd(ctypes.byref(tq4), ctypes.byref(tkb), ctypes.byref(tkb), ctypes.byref(tq4), None,
                         ctypes.c_float(0.0), 0, None)
    assert st == ra.RA_ERR_INVALID_ARG and b"agree on B" in lib.ra_last_error()
    # a sliding window must cover at least the query's own position
    st = lib.ra_attn_fwd_window(ctypes.byref(tq4), ctypes.byref(tq4), ctypes.byref(tq4), ctypes.byref(tq4), None,
                                ctypes.c_float(0.0), 0, None)
    assert st == ra.RA_ERR_INVALID_ARG and b"window" in lib.ra_last_error()
    # bf16 head dim must be a multiple of 8 and <= 128
    q2 = torch.zeros(1, 1, 16, 136, dtype=torch.bfloat16)
    t2 = ra.tensor_desc(q2)
    st = lib.ra_attn_fwd(ctypes.byref(t2), ctypes.byref(t2), ctypes.byref(t2), ctypes.byref(t2), None,
                         ctypes.c_float(0.0), 0, None)
    assert st == ra.RA_ERR_UNSUPPORTED
    # unaligned token stride for the TMA path
    q3 = torch.zeros(1, 1, 16, 68, dtype=torch.bfloat16)[..., :64]
    t3 = ra.tensor_desc(q3)
    st = lib.ra_attn_fwd(ctypes.byref(t3), ctypes.byref(t3), ctypes.byref(t3), ctypes.byref(t3), None,
                         ctypes.c_float(0.0), 0, None)
    assert st == ra.RA_ERR_ALIGNMENT
    # merge with zero rows is a no-op; bad d is rejected
    assert lib.ra_lse_merge(None, None, None, None, None, None, 0, 64, None) == ra.RA_OK
    assert lib.ra_lse_merge(None, None, None, None, None, None, 10, 0, None) == ra.RA_ERR_INVALID_ARG
    assert lib.ra_lse_merge_n(None, None, 0, None, None, 10, 64, None) == ra.RA_ERR_INVALID_ARG
    assert lib.ra_lse_merge_n(None, None, 33, None, None, 10, 64, None) == ra.RA_ERR_INVALID_ARG
    # timeout limits
    assert lib.ra_set_wait_timeout_ns(10) == ra.RA_ERR_INVALID_ARG
    # walk order over striped shards: the two named orders only (a process-wide setting, restored)
    assert lib.ra_set_striped_walk(2) == ra.RA_ERR_INVALID_ARG
    assert lib.ra_set_striped_walk(-1) == ra.RA_ERR_INVALID_ARG
    assert lib.ra_set_striped_walk(1) == ra.RA_OK
    assert lib.ra_set_striped_walk(0) == ra.RA_OK


def test_ring_workspace_size(ra):
    import torch

    q = torch.zeros(2, 16, 8192, 64, dtype=torch.bfloat16)
    assert ra.ring_workspace_size(q, 8, "fused") == 0
    assert ra.ring_workspace_size(q, 1, "stepwise") == 0
    rows = 2 * 16 * 8192
    assert ra.ring_workspace_size(q, 8, "stepwise") == rows * 64 * 4 + rows * 4
    with pytest.raises(ra.RaError):
        ra.ring_workspace_size(q, 3, "stepwise")  # 8192 % 3 != 0


def test_backward_host_validation(ra):
    """ra_attn_bwd rejects bad arguments before any CUDA call."""
    import torch

    lib = ra.lib_handle()
    q = torch.zeros(1, 4, 32, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 2, 32, 64, dtype=torch.bfloat16)
    g32 = torch.zeros(1, 4, 32, 64, dtype=torch.float32)
    gk = torch.zeros(1, 2, 32, 64, dtype=torch.float32)
    lse = torch.zeros(1, 4, 32, dtype=torch.float32)
    tq, tk, tg, tgk = (ra.tensor_desc(x) for x in (q, k, g32, gk))
    lse_p = ctypes.c_void_p(lse.data_ptr())

    def call(dq=tg, dk=tgk, dv=tgk, lse_ptr=lse_p, causal=1, window=0, o=tq, d_o=tq, kk=tk):
        return lib.ra_attn_bwd(ctypes.byref(tq), ctypes.byref(kk), ctypes.byref(kk), ctypes.byref(o), lse_ptr,
                               ctypes.byref(d_o), ctypes.byref(dq), ctypes.byref(dk), ctypes.byref(dv),
                               ctypes.c_float(0.0), causal, ctypes.c_int64(window), None)

    assert call(lse_ptr=None) == ra.RA_ERR_INVALID_ARG and b"lse is NULL" in lib.ra_last_error()
    tbad = ra.tensor_desc(torch.zeros(1, 4, 32, 64, dtype=torch.bfloat16))
    assert call(dq=tbad) == ra.RA_ERR_INVALID_ARG and b"fp32" in lib.ra_last_error()
    assert call(dq=tgk) == ra.RA_ERR_INVALID_ARG and b"shape of q" in lib.ra_last_error()
    assert call(dk=tg) == ra.RA_ERR_INVALID_ARG and b"shape of k" in lib.ra_last_error()
    assert call(causal=0, window=16) == ra.RA_ERR_INVALID_ARG and b"window" in lib.ra_last_error()
    assert call(window=-1) == ra.RA_ERR_INVALID_ARG
    to32 = ra.tensor_desc(torch.zeros(1, 4, 32, 64, dtype=torch.float32))
    assert call(o=to32) == ra.RA_ERR_INVALID_ARG and b"q's dtype" in lib.ra_last_error()
    k3 = ra.tensor_desc(torch.zeros(1, 3, 32, 64, dtype=torch.bfloat16))
    assert call(kk=k3) == ra.RA_ERR_INVALID_ARG


def test_host_pipeline_validation(ra):
    """ra_ring_fwd_host rejects bad arguments before anything reaches a device."""
    import torch

    lib = ra.lib_handle()
    q = torch.zeros(1, 4, 64, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16)
    t = {n: ra.tensor_desc(x) for n, x in (("q", q), ("k", k), ("v", k), ("o", q))}
    strided = ra.tensor_desc(q.transpose(1, 2).contiguous().transpose(1, 2))  # [B,H,N,d] view, not packed
    f32 = ra.tensor_desc(q.float())
    small = ra.tensor_desc(q[:, :2])
    streams = (ctypes.c_void_p * 3)(1, 2, 3)
    same = (ctypes.c_void_p * 3)(1, 1, 3)
    lse = ctypes.c_void_p(16)

    def call(qh=None, qd=None, lse_h=lse, lse_d=lse, chunks=2, st=streams):
        qh = qh or t["q"]
        qd = qd or t["q"]
        return lib.ra_ring_fwd_host(ctypes.byref(qh), ctypes.byref(t["k"]), ctypes.byref(t["v"]), 4, 0, 1,
                                    ctypes.c_float(0), ctypes.byref(t["o"]), lse_h, ctypes.byref(qd),
                                    ctypes.byref(t["k"]), ctypes.byref(t["v"]), ctypes.byref(t["o"]), lse_d, chunks, st)

    assert call(qh=strided) == ra.RA_ERR_UNSUPPORTED and b"contiguous" in lib.ra_last_error()
    assert call(qd=f32) == ra.RA_ERR_INVALID_ARG and b"dtype" in lib.ra_last_error()
    assert call(qd=small) == ra.RA_ERR_INVALID_ARG and b"shape" in lib.ra_last_error()
    assert call(lse_d=None) == ra.RA_ERR_INVALID_ARG and b"both" in lib.ra_last_error()
    assert call(st=same) == ra.RA_ERR_INVALID_ARG and b"distinct streams" in lib.ra_last_error()
    assert call(chunks=0) == ra.RA_ERR_INVALID_ARG and b"n_chunks" in lib.ra_last_error()


def test_header_compiles_and_links_from_c(ra, tmp_path):
    """The boundary as a C caller sees it: the header compiles as C and as C++, and a C program
    that takes the address of every declared entry point links against the library and runs
    (ra_version and ra_status_string need no device)."""
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    inc = os.path.join(ROOT, "include")
    names = _declared_symbols()
    src = tmp_path / "abi.c"
    body = "\n".join(f"  fns[{i}] = (void (*)(void))&{n};" for i, n in enumerate(names))
    src.write_text(
        "#include <stdio.h>\n#include \"ra_attn.h\"\n"
        f"int main(void) {{\n  void (*fns[{len(names)}])(void);\n{body}\n"
        "  for (unsigned i = 0; i < sizeof(fns) / sizeof(fns[0]); ++i) if (!fns[i]) return 2;\n"
        "  printf(\"%d %s\\n\", ra_version(), ra_status_string(RA_ERR_WORKSPACE));\n  return 0;\n}\n")
    for lang, comp in (("c", gcc), ("c++", shutil.which("g++") or gcc)):
        r = subprocess.run([comp, "-fsyntax-only", "-Wall", "-Werror", "-x", lang, os.path.join(inc, "ra_attn.h")],
                           capture_output=True, text=True)
        assert r.returncode == 0, (lang, r.stderr)
    libdir = os.path.dirname(ra.LIB_PATH)
    exe = tmp_path / "abi"
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", inc, str(src), "-L", libdir, "-lra_attn",
                        f"-Wl,-rpath,{libdir}", "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert r.stdout.split() == [str(ra.version()), "RA_ERR_WORKSPACE"]
