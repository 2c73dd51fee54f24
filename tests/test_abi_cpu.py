"""C-ABI checks that need no GPU: the library loads, exports every function
include/*.h declares, and its host-side logic (counts, workspace sizing,
argument validation before any launch) behaves as documented."""
import ctypes
import glob
import os
import re

import pytest

import oracle
from sparse_attention_context_b200 import _lib
from sparse_attention_context_b200._lib import IsaShape

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names.update(re.findall(r"\b(isa_\w+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(_lib.LIB_PATH):
        from sparse_attention_context_b200 import build

        build.build()
    return _lib.lib()


def test_exports_every_declared_function(L):
    names = declared_functions()
    assert "isa_attn_fwd" in names and "isa_dense_attn_fwd" in names
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(_lib.SIGNATURES), "binding signatures and header disagree"


def shape(**kw):
    base = dict(B=1, H=24, N_src=20280, N_ctx=20280, d=128, block=128, keep=0.25, rho=0.2, scale=0.0)
    base.update(kw)
    return IsaShape(**base)


@pytest.mark.parametrize("keep,rho,N_src,N_ctx,blk", [
    (0.25, 0.2, 20280, 20280, 128), (0.5, 0.25, 256, 256, 64), (0.3, 0.2, 4096, 4096, 128),
    (0.2, 0.15, 75600, 75600, 128), (0.0, 0.0, 100, 0, 64), (1.0, 1.0, 77, 300, 64), (0.1, 0.5, 32768, 32768, 128),
    # the guard's cap: 0.200002 * 10^6 is an exact count at N >= 10^6
    (0.5, 0.200002, 600000, 400000, 128), (0.5, 1.0, 1900000, 100000, 128)])
def test_counts_match_oracle(L, keep, rho, N_src, N_ctx, blk):
    s = shape(N_src=N_src, N_ctx=N_ctx, block=blk, keep=keep, rho=rho)
    nCB = -(-N_ctx // blk)
    assert L.isa_n_keep(ctypes.byref(s)) == oracle.n_keep_of(keep, nCB)
    assert L.isa_n_route(ctypes.byref(s)) == oracle.n_route_of(rho, N_src + N_ctx)
    nB = -(-N_src // blk) + nCB
    assert L.isa_n_route_blocks(ctypes.byref(s)) == oracle.n_route_blocks_of(rho, nB)


def test_workspace_size(L):
    s = shape()
    n = L.isa_workspace_size(ctypes.byref(s))
    # block means (3 x fp32) + gathered bf16 operands + sharpness + index sets
    BH, N, nB, d = 24, 40560, 318, 128
    assert n >= 3 * BH * nB * d * 4 + BH * N * 4 + BH * N * 4
    assert n < 64 * 2**20
    assert L.isa_workspace_size(ctypes.byref(shape(d=96))) == 0
    assert L.isa_dense_workspace_size(128) >= 256 + 148 * 256 * 128 * 4
    assert L.isa_dense_workspace_size(96) == 0


@pytest.mark.parametrize("bad,code", [
    (dict(d=96), 2), (dict(block=32), 2), (dict(keep=1.5), 1), (dict(rho=-0.1), 1), (dict(N_src=0), 1),
    (dict(B=0), 1), (dict(N_ctx=-1), 1), (dict(H=70000), 2), (dict(N_ctx=4097 * 64, block=64), 2)])
def test_invalid_shapes_rejected_before_launch(L, bad, code):
    s = shape(**bad)
    buf = (ctypes.c_uint8 * 1024)()
    p = ctypes.addressof(buf)
    assert L.isa_preselect_ctx(ctypes.byref(s), p, p, p, p, None, p, 1024, None) == code
    assert L.isa_forward(ctypes.byref(s), p, p, p, p, p, 1024, None) == code
    assert L.isa_n_keep(ctypes.byref(s)) == -1


def test_bad_pointers_and_workspace_rejected(L):
    s = shape(H=2, N_src=256, N_ctx=256, d=64, block=64)
    need = L.isa_workspace_size(ctypes.byref(s))
    buf = (ctypes.c_uint8 * 4096)()
    p = (ctypes.addressof(buf) + 255) // 256 * 256
    assert L.isa_preselect_ctx(ctypes.byref(s), None, p, p, p, None, p, need, None) == 1       # null q
    assert L.isa_preselect_ctx(ctypes.byref(s), p + 2, p, p, p, None, p, need, None) == 1      # misaligned
    assert L.isa_preselect_ctx(ctypes.byref(s), p, p, p, p, None, p, need - 1, None) == 3      # small ws
    assert L.isa_preselect_ctx(ctypes.byref(s), p, p, p, None, None, p, need, None) == 1       # kept missing
    assert L.isa_route_queries(ctypes.byref(s), p, p, None, p, None, p, need, None) == 1       # routed missing
    assert L.isa_attn_fwd(ctypes.byref(s), p, p, p, p, p, p, None, p, need, None) == 1         # out missing
    assert L.isa_full_attn_rows_fwd(ctypes.byref(s), p, p, p, p, p, -1, p, p, need, None) == 1  # negative rows
    assert L.isa_full_attn_rows_fwd(ctypes.byref(s), p, p, p, p, None, 4, p, p, need, None) == 1  # rows missing
    assert L.isa_route_blocks_taylor_fwd(ctypes.byref(s), p, p, None, p, None, None, p, p, need, None) == 1
    assert L.isa_forward_blocks(ctypes.byref(s), p, p, p, p, p, need - 1, None) == 3             # small ws
    assert L.isa_dense_attn_fwd(1, 1, 128, 80, 0.0, p, p, p, p, p, 256, None) == 2
    assert L.isa_dense_attn_fwd(1, 1, 128, 64, 0.0, p, p, p, p, p, 8, None) == 3
    assert L.isa_dense_attn_fwd(1, 1, 0, 64, 0.0, p, p, p, p, p, 256, None) == 1


def test_status_strings(L):
    assert L.isa_status_string(0) == b"ok"
    assert b"timed out" in L.isa_status_string(5)
    assert L.isa_status_string(99) == b"unknown status"


def test_nvtx_ranges_opt_in():
    """With ISA_NVTX=1 every entry point opens and closes an NVTX range (a
    no-op without a profiler attached); argument validation still returns
    its status.  Run in a fresh process, since the variable is read once."""
    import subprocess
    import sys

    code = (
        "import ctypes\n"
        "from sparse_attention_context_b200 import _lib\n"
        "L = _lib.lib()\n"
        "s = _lib.IsaShape(1, 2, 256, 256, 96, 64, 0.5, 0.25, 0.0)\n"
        "buf = (ctypes.c_uint8 * 1024)(); p = ctypes.addressof(buf)\n"
        "assert L.isa_forward(ctypes.byref(s), p, p, p, p, p, 1024, None) == 2\n"
        "assert L.isa_dense_attn_fwd(1, 1, 0, 64, 0.0, p, p, p, p, p, 256, None) == 1\n"
        "print('ok')\n")
    for flag in ("1", "0"):
        r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=120,
                           env=dict(os.environ, ISA_NVTX=flag))
        assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr


def test_host_staging_size_and_validation(L):
    """isa_host_staging_size: a slice workspace plus a ring of up to three
    slices of q, k, v, out; isa_forward_host rejects bad arguments before
    enqueuing anything."""
    s = shape()  # 480p: 24 heads
    ws2 = L.isa_workspace_size(ctypes.byref(shape(H=2)))
    head = 40560 * 128 * 2
    n_default = L.isa_host_staging_size(ctypes.byref(s), 0)   # 12 slices of 2 heads
    assert n_default >= ws2 + 3 * 4 * 2 * head
    assert n_default < ws2 + 3 * 4 * 2 * head + 64 * 1024
    n1 = L.isa_host_staging_size(ctypes.byref(s), 1)          # one slice of all 24 heads
    assert n1 >= L.isa_workspace_size(ctypes.byref(s)) + 4 * 24 * head
    assert L.isa_host_staging_size(ctypes.byref(s), 100) == L.isa_host_staging_size(ctypes.byref(s), 24)
    assert L.isa_host_staging_size(ctypes.byref(shape(d=96)), 0) == 0
    buf = (ctypes.c_uint8 * 4096)()
    p = (ctypes.addressof(buf) + 255) // 256 * 256
    t = shape(H=2, N_src=256, N_ctx=256, d=64, block=64)
    need = L.isa_host_staging_size(ctypes.byref(t), 0)
    assert L.isa_forward_host(ctypes.byref(shape(d=96)), p, p, p, p, p, need, 0, None, None, None) == 2
    assert L.isa_forward_host(ctypes.byref(shape(keep=2.0)), p, p, p, p, p, need, 0, None, None, None) == 1
    assert L.isa_forward_host(ctypes.byref(t), None, p, p, p, p, need, 0, None, None, None) == 1
    assert L.isa_forward_host(ctypes.byref(t), p, p, p, None, p, need, 0, None, None, None) == 1
    assert L.isa_forward_host(ctypes.byref(t), p, p, p, p, p + 8, need, 0, None, None, None) == 1
    assert L.isa_forward_host(ctypes.byref(t), p, p, p, p, p, need - 1, 0, None, None, None) == 3
