"""Python binding of libisa.so: argument marshalling only.

Every function takes torch tensors for device memory and the current torch
CUDA stream, and calls the C entry point of the same name (include/isa.h);
no step of the ISA path runs in Python or torch.
"""
from __future__ import annotations

import ctypes

import torch

from ._lib import IsaShape, check, lib


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _check_qkv(*ts):
    for t in ts:
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and t.dim() == 4):
            raise ValueError("q, k, v, out must be contiguous CUDA bf16 tensors [B, H, N, d]")


def make_shape(q: torch.Tensor, N_src: int, block: int, keep: float, rho: float, scale: float = 0.0) -> IsaShape:
    B, H, N, d = q.shape
    return IsaShape(B, H, int(N_src), int(N - N_src), d, int(block), float(keep), float(rho), float(scale))


def isa_n_keep(shape: IsaShape) -> int:
    return lib().isa_n_keep(ctypes.byref(shape))


def isa_n_route(shape: IsaShape) -> int:
    return lib().isa_n_route(ctypes.byref(shape))


def isa_n_route_blocks(shape: IsaShape) -> int:
    return lib().isa_n_route_blocks(ctypes.byref(shape))


def isa_workspace_size(shape: IsaShape) -> int:
    return lib().isa_workspace_size(ctypes.byref(shape))


def new_workspace(shape: IsaShape, device="cuda") -> torch.Tensor:
    """Zeroed workspace (control block included) for every call on `shape`."""
    n = isa_workspace_size(shape)
    if n == 0:
        raise ValueError("invalid or unsupported shape")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def isa_preselect_ctx(q, k, v, shape: IsaShape, ws, kept=None, saliency=None, want_saliency=True, stream=None):
    """Stage 1.  Returns (kept_ctx_idx [B,H,n_keep] int32, saliency [B,H,nCB] or None)."""
    _check_qkv(q, k, v)
    B, H = shape.B, shape.H
    nk = isa_n_keep(shape)
    nCB = -(-shape.N_ctx // shape.block)
    if kept is None:
        kept = torch.empty((B, H, nk), dtype=torch.int32, device=q.device)
    if saliency is None and want_saliency:
        saliency = torch.empty((B, H, nCB), dtype=torch.float32, device=q.device)
    rc = lib().isa_preselect_ctx(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                 _ptr(kept) if nk > 0 else None, _ptr(saliency), ws.data_ptr(), ws.numel(),
                                 _stream(stream))
    check("isa_preselect_ctx", rc)
    return kept, saliency


def isa_route_queries(q, kept, shape: IsaShape, ws, routed=None, taylor=None, sharpness=None, want_sharpness=True,
                      stream=None):
    """Stage 2.  Returns (routed_idx [B,H,n_route], taylor_idx [B,H,N-n_route], sharpness [B,H,N] or None)."""
    _check_qkv(q)
    B, H, N = shape.B, shape.H, shape.N_src + shape.N_ctx
    nr = isa_n_route(shape)
    if routed is None:
        routed = torch.empty((B, H, nr), dtype=torch.int32, device=q.device)
    if taylor is None:
        taylor = torch.empty((B, H, N - nr), dtype=torch.int32, device=q.device)
    if sharpness is None and want_sharpness:
        sharpness = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    rc = lib().isa_route_queries(ctypes.byref(shape), q.data_ptr(), _ptr(kept) if kept.numel() else None,
                                 _ptr(routed) if nr > 0 else None, _ptr(taylor) if N - nr > 0 else None,
                                 _ptr(sharpness), ws.data_ptr(), ws.numel(), _stream(stream))
    check("isa_route_queries", rc)
    return routed, taylor, sharpness


def isa_route_taylor_fwd(q, kept, shape: IsaShape, ws, out, routed=None, taylor=None, sharpness=None,
                         want_sharpness=True, stream=None):
    """Stages 2 + 4 fused: sharpness, routing, and the Taylor output of every
    row of `out`.  Returns (routed_idx, taylor_idx, sharpness or None)."""
    _check_qkv(q, out)
    B, H, N = shape.B, shape.H, shape.N_src + shape.N_ctx
    nr = isa_n_route(shape)
    if routed is None:
        routed = torch.empty((B, H, nr), dtype=torch.int32, device=q.device)
    if taylor is None:
        taylor = torch.empty((B, H, N - nr), dtype=torch.int32, device=q.device)
    if sharpness is None and want_sharpness:
        sharpness = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    rc = lib().isa_route_taylor_fwd(ctypes.byref(shape), q.data_ptr(), _ptr(kept) if kept.numel() else None,
                                    _ptr(routed) if nr > 0 else None, _ptr(taylor) if N - nr > 0 else None,
                                    _ptr(sharpness), out.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
    check("isa_route_taylor_fwd", rc)
    return routed, taylor, sharpness


def isa_attn_fwd(q, k, v, kept, routed, taylor, shape: IsaShape, ws, out=None, stream=None):
    """Stages 3 and 4.  Returns out [B,H,N,d] bf16."""
    if out is None:
        out = torch.empty_like(q)
    _check_qkv(q, k, v, out)
    rc = lib().isa_attn_fwd(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                            _ptr(kept) if kept.numel() else None, _ptr(routed) if routed.numel() else None,
                            _ptr(taylor) if taylor.numel() else None, out.data_ptr(), ws.data_ptr(), ws.numel(),
                            _stream(stream))
    check("isa_attn_fwd", rc)
    return out


def isa_full_attn_fwd(q, k, v, kept, routed, shape: IsaShape, ws, out, stream=None):
    """Stage 3 only: full attention for the routed rows of `out`."""
    _check_qkv(q, k, v, out)
    rc = lib().isa_full_attn_fwd(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                 _ptr(kept) if kept.numel() else None, _ptr(routed) if routed.numel() else None,
                                 out.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
    check("isa_full_attn_fwd", rc)
    return out


def isa_taylor_attn_fwd(q, kept, taylor, shape: IsaShape, ws, out, stream=None):
    """Stage 4 only: 0-th order Taylor attention for the taylor rows of `out`."""
    _check_qkv(q, out)
    rc = lib().isa_taylor_attn_fwd(ctypes.byref(shape), q.data_ptr(), _ptr(kept) if kept.numel() else None,
                                   _ptr(taylor) if taylor.numel() else None, out.data_ptr(), ws.data_ptr(),
                                   ws.numel(), _stream(stream))
    check("isa_taylor_attn_fwd", rc)
    return out


def isa_full_attn_rows_fwd(q, k, v, kept, rows, shape: IsaShape, ws, out, stream=None):
    """Stage 3 for an explicit row list rows [B,H,n_rows] (-1 entries are padding)."""
    _check_qkv(q, k, v, out)
    n_rows = rows.shape[-1]
    rc = lib().isa_full_attn_rows_fwd(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                      _ptr(kept) if kept.numel() else None, _ptr(rows) if rows.numel() else None,
                                      int(n_rows), out.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
    check("isa_full_attn_rows_fwd", rc)
    return out


def isa_route_blocks_taylor_fwd(q, kept, shape: IsaShape, ws, out, want_scores=True, want_sharpness=True,
                                stream=None):
    """Stages 2 + 4 with whole query blocks routed.  Returns (routed block
    indices [B,H,n_rb], routed rows [B,H,n_rb*block] with -1 pads, block
    scores [B,H,nB] or None, sharpness [B,H,N] or None)."""
    _check_qkv(q, out)
    B, H, N = shape.B, shape.H, shape.N_src + shape.N_ctx
    nB = -(-shape.N_src // shape.block) + -(-shape.N_ctx // shape.block)
    nrb = isa_n_route_blocks(shape)
    rblk = torch.empty((B, H, nrb), dtype=torch.int32, device=q.device)
    rows = torch.empty((B, H, nrb * shape.block), dtype=torch.int32, device=q.device)
    score = torch.empty((B, H, nB), dtype=torch.float32, device=q.device) if want_scores else None
    sharp = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if want_sharpness else None
    rc = lib().isa_route_blocks_taylor_fwd(ctypes.byref(shape), q.data_ptr(), _ptr(kept) if kept.numel() else None,
                                           _ptr(rblk) if nrb else None, _ptr(rows) if nrb else None, _ptr(score),
                                           _ptr(sharp), out.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
    check("isa_route_blocks_taylor_fwd", rc)
    return rblk, rows, score, sharp


def isa_forward_blocks(q, k, v, N_src: int, block: int, keep: float, rho: float, scale: float = 0.0, ws=None,
                       out=None, stream=None):
    """The ISA forward with block-granular query grouping (CUDA tensors)."""
    shape = make_shape(q, N_src, block, keep, rho, scale)
    if ws is None:
        ws = new_workspace(shape, q.device)
    o = torch.empty_like(q) if out is None else out
    _check_qkv(q, k, v, o)
    rc = lib().isa_forward_blocks(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                  ws.data_ptr(), ws.numel(), _stream(stream))
    check("isa_forward_blocks", rc)
    return o


def taylor1_workspace(shape: IsaShape, device="cuda") -> torch.Tensor:
    """Buffer for the correction matrices of the first-order Taylor variant."""
    n = lib().isa_taylor1_workspace_size(ctypes.byref(shape))
    if n == 0:
        raise ValueError("invalid or unsupported shape")
    return torch.empty(n, dtype=torch.uint8, device=device)


def isa_taylor1_attn_fwd(q, k, v, kept, taylor, shape: IsaShape, ws, cws, out, stream=None):
    """First-order Taylor output for the taylor rows of `out` (C_b land in cws)."""
    _check_qkv(q, k, v, out)
    rc = lib().isa_taylor1_attn_fwd(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                    _ptr(kept) if kept.numel() else None, _ptr(taylor) if taylor.numel() else None,
                                    out.data_ptr(), ws.data_ptr(), ws.numel(), cws.data_ptr(), cws.numel(),
                                    _stream(stream))
    check("isa_taylor1_attn_fwd", rc)
    return out


def isa_forward_taylor1(q, k, v, N_src: int, block: int, keep: float, rho: float, scale: float = 0.0, ws=None,
                        cws=None, out=None, stream=None):
    """The ISA forward with first-order Taylor attention for the rows that are not routed."""
    shape = make_shape(q, N_src, block, keep, rho, scale)
    if ws is None:
        ws = new_workspace(shape, q.device)
    if cws is None:
        cws = taylor1_workspace(shape, q.device)
    o = torch.empty_like(q) if out is None else out
    _check_qkv(q, k, v, o)
    rc = lib().isa_forward_taylor1(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   ws.data_ptr(), ws.numel(), cws.data_ptr(), cws.numel(), _stream(stream))
    check("isa_forward_taylor1", rc)
    return o


def isa_forward(q, k, v, N_src: int, block: int, keep: float, rho: float, scale: float = 0.0, ws=None, out=None,
                stream=None, groups=None):
    """All ISA stages in one call.

    CUDA inputs: runs on the current stream and returns a CUDA tensor.
    CPU inputs (the host-buffer path): copies q, k, v to the GPU, runs, and
    copies the output back into a pinned CPU tensor (returned).  Every
    (b, h) is an independent unit, so the heads are taken in `groups`
    consecutive slices (default: two heads a slice from 8 heads on): the
    host-to-device copy of a slice, the forward of the previous slice and the
    device-to-host copy of the one before run on three streams at once, and
    PCIe transfers in both directions overlap the GPU work.  Pass pinned
    host tensors for the copies to be asynchronous.
    """
    if q.is_cuda:
        shape = make_shape(q, N_src, block, keep, rho, scale)
        if ws is None:
            ws = new_workspace(shape, q.device)
        o = torch.empty_like(q) if out is None else out
        _check_qkv(q, k, v, o)
        rc = lib().isa_forward(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                               ws.data_ptr(), ws.numel(), _stream(stream))
        check("isa_forward", rc)
        return o
    return _isa_forward_host(q, k, v, N_src, block, keep, rho, scale, ws, out, groups)


def _isa_forward_host(q, k, v, N_src, block, keep, rho, scale, ws, out, groups):
    """Host-buffer path of isa_forward: head slices pipelined over a copy-in
    stream, the caller's current stream (compute) and a copy-out stream."""
    dev = torch.device("cuda")
    B, H, N, d = q.shape
    BH = B * H
    G = groups if groups is not None else (BH // 2 if BH >= 8 else 1)  # two heads a slice (measured best at 480p)
    G = max(1, min(int(G), BH))
    bounds = [BH * i // G for i in range(G + 1)]
    qf, kf, vf = (t.reshape(BH, N, d) for t in (q, k, v))
    dq, dk, dv = (torch.empty((BH, N, d), dtype=q.dtype, device=dev) for _ in range(3))
    do = torch.empty((BH, N, d), dtype=q.dtype, device=dev)
    dst = out if out is not None else torch.empty((B, H, N, d), dtype=q.dtype, pin_memory=True)
    dstf = dst.reshape(BH, N, d)
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    start = torch.cuda.Event()
    start.record(comp)
    s_in.wait_event(start)
    s_out.wait_event(start)
    big = max(bounds[i + 1] - bounds[i] for i in range(G))
    shape_big = make_shape(torch.empty((1, big, N, d), device="meta"), N_src, block, keep, rho, scale)
    if ws is None or ws.numel() < lib().isa_workspace_size(ctypes.byref(shape_big)):
        ws = new_workspace(shape_big, dev)
    done_in, done_comp = [], []
    for g in range(G):
        a, b = bounds[g], bounds[g + 1]
        with torch.cuda.stream(s_in):
            for src, buf in ((qf, dq), (kf, dk), (vf, dv)):
                buf[a:b].copy_(src[a:b], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(s_in)
            done_in.append(ev)
    for g in range(G):
        a, b = bounds[g], bounds[g + 1]
        comp.wait_event(done_in[g])
        shape = make_shape(torch.empty((1, b - a, N, d), device="meta"), N_src, block, keep, rho, scale)
        rc = lib().isa_forward(ctypes.byref(shape), dq[a].data_ptr(), dk[a].data_ptr(), dv[a].data_ptr(),
                               do[a].data_ptr(), ws.data_ptr(), ws.numel(), _stream(None))
        check("isa_forward", rc)
        ev = torch.cuda.Event()
        ev.record(comp)
        done_comp.append(ev)
    with torch.cuda.stream(s_out):
        for g in range(G):
            a, b = bounds[g], bounds[g + 1]
            s_out.wait_event(done_comp[g])
            dstf[a:b].copy_(do[a:b], non_blocking=True)
    fin = torch.cuda.Event()
    fin.record(s_out)
    comp.wait_event(fin)
    comp.synchronize()
    for t in (dq, dk, dv, do, ws):  # keep the caching allocator from reusing them early
        t.record_stream(s_in)
        t.record_stream(s_out)
    return dst


def isa_forward_static(q, k, v, N_src: int, block: int, keep: float, rho: float, scale: float = 0.0, out=None,
                       stream=None):
    """All ISA stages with the library's fixed device scratch (no workspace,
    nothing allocated by the library).  CUDA tensors only; returns out."""
    if out is None:
        out = torch.empty_like(q)
    _check_qkv(q, k, v, out)
    shape = make_shape(q, N_src, block, keep, rho, scale)
    rc = lib().isa_forward_static(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                  _stream(stream))
    check("isa_forward_static", rc)
    return out


def dense_workspace(d: int = 128, device="cuda") -> torch.Tensor:
    n = lib().isa_dense_workspace_size(int(d))
    if n == 0:
        raise ValueError("unsupported head dimension")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def isa_dense_attn_fwd(q, k, v, scale: float = 0.0, out=None, ws=None, stream=None):
    """In-house dense flash attention (the baseline).  Returns out [B,H,N,d] bf16."""
    if out is None:
        out = torch.empty_like(q)
    _check_qkv(q, k, v, out)
    B, H, N, d = q.shape
    if ws is None:
        ws = dense_workspace(d, q.device)
    rc = lib().isa_dense_attn_fwd(B, H, N, d, float(scale), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                  out.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
    check("isa_dense_attn_fwd", rc)
    return out


def isa_read_device_status(ws, stream=None) -> int:
    """Synchronise, return the device status word of `ws` and reset it."""
    return lib().isa_read_device_status(ws.data_ptr(), _stream(stream))


def isa_selftest_umma(A, B, P, V, ws, stream=None):
    """Test-only: one-tile UMMA products S = A B^T, O = P V (P in shared
    memory) and O2 = P V (P in tensor memory), all fp32."""
    d, bn = A.shape[1], B.shape[0]
    S = torch.empty((128, bn), dtype=torch.float32, device=A.device)
    O = torch.empty((128, d), dtype=torch.float32, device=A.device)
    O2 = torch.empty((128, d), dtype=torch.float32, device=A.device)
    rc = lib().isa_selftest_umma(d, bn, A.data_ptr(), B.data_ptr(), P.data_ptr(), V.data_ptr(), S.data_ptr(),
                                 O.data_ptr(), O2.data_ptr(), ws.data_ptr(), _stream(stream))
    check("isa_selftest_umma", rc)
    return S, O, O2


def isa_selftest_ex2(x, stream=None):
    """Test-only: (FMA-pipe 2^x of the softmax, MUFU ex2, exp2f) of the fp32
    CUDA tensor x, each a tensor like x."""
    if not (x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()):
        raise ValueError("x must be a contiguous CUDA float32 tensor")
    yp, ym, yr = (torch.empty_like(x) for _ in range(3))
    rc = lib().isa_selftest_ex2(x.data_ptr(), yp.data_ptr(), ym.data_ptr(), yr.data_ptr(), x.numel(), _stream(stream))
    check("isa_selftest_ex2", rc)
    return yp, ym, yr
