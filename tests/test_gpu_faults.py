"""Failure detection without a GPU fault: the test sets the workspace's
fault-injection word, the attention kernels then take their timeout path
(as if a bounded mbarrier wait had expired) without waiting, record
ISA_ERR_DEVICE_TIMEOUT in the status word, release TMEM and exit; the
context stays usable and the next call is correct."""
import pytest
import torch

from sparse_attention_context_b200 import api
from workloads import CONFIGS

from _parity import check_out, inputs

pytestmark = pytest.mark.gpu


def test_injected_timeout_is_reported_and_recovered(cuda_ok):
    cfg = CONFIGS["tiny"]
    _, (q, k, v) = inputs(cfg)
    shape = api.make_shape(q, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    ws = api.new_workspace(shape)
    good = api.isa_forward(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, ws=ws).clone()
    assert api.isa_read_device_status(ws) == 0
    ws[4:8].view(torch.int32).fill_(1)
    api.isa_forward(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, ws=ws)
    assert api.isa_read_device_status(ws) == 5
    ws[4:8].view(torch.int32).fill_(0)
    again = api.isa_forward(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, ws=ws)
    assert api.isa_read_device_status(ws) == 0
    assert torch.equal(again.view(torch.int16), good.view(torch.int16))


def test_injected_timeout_dense(cuda_ok):
    cfg = CONFIGS["tiny"]
    _, (q, k, v) = inputs(cfg)
    ws = api.dense_workspace(q.shape[-1])
    ws[4:8].view(torch.int32).fill_(1)
    api.isa_dense_attn_fwd(q, k, v, ws=ws)
    assert api.isa_read_device_status(ws) == 5
    ws[4:8].view(torch.int32).fill_(0)
    out = api.isa_dense_attn_fwd(q, k, v, ws=ws)
    assert api.isa_read_device_status(ws) == 0
    ref = torch.nn.functional.scaled_dot_product_attention(q.float(), k.float(), v.float())
    check_out(out.double().cpu().numpy(), ref.double().cpu().numpy(), "dense after fault")


def test_bad_route_index_is_flagged_not_faulted(cuda_ok):
    """An out-of-range query index is skipped and reported, never dereferenced."""
    cfg = CONFIGS["tiny"]
    _, (q, k, v) = inputs(cfg)
    shape = api.make_shape(q, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    ws = api.new_workspace(shape)
    kept, _ = api.isa_preselect_ctx(q, k, v, shape, ws)
    routed, taylor, _ = api.isa_route_queries(q, kept, shape, ws)
    routed[0, 0, 0] = cfg.N + 5
    api.isa_attn_fwd(q, k, v, kept, routed, taylor, shape, ws)
    assert api.isa_read_device_status(ws) == 1


def test_timed_out_key_split_writes_no_rows(cuda_ok):
    """A full-attention launch whose items run split along the keys: after
    an (injected) timeout no piece writes partials, so the merge must leave
    the rows unwritten instead of combining stale partial buffers."""
    cfg = CONFIGS["tiny"].replace(H=1, d=128, N_src=3000, N_ctx=2900, block=128, keep=0.35, rho=0.25)
    _, (q, k, v) = inputs(cfg)
    shape = api.make_shape(q, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    ws = api.new_workspace(shape)
    out = torch.empty_like(q)
    kept, _ = api.isa_preselect_ctx(q, k, v, shape, ws)
    routed, taylor, _ = api.isa_route_queries(q, kept, shape, ws)
    api.isa_full_attn_fwd(q, k, v, kept, routed, shape, ws, out)  # fills the partial buffers
    assert api.isa_read_device_status(ws) == 0
    good = out.clone()
    sentinel = torch.full_like(q, 7.0)
    ws[4:8].view(torch.int32).fill_(1)
    api.isa_full_attn_fwd(q, k, v, kept, routed, shape, ws, sentinel)
    assert api.isa_read_device_status(ws) == 5
    assert bool((sentinel == 7.0).all()), "rows written after a timeout"
    ws[4:8].view(torch.int32).fill_(0)
    api.isa_full_attn_fwd(q, k, v, kept, routed, shape, ws, sentinel)
    assert api.isa_read_device_status(ws) == 0
    r = routed[0, 0].long()
    assert torch.equal(sentinel[0, 0, r].view(torch.int16), good[0, 0, r].view(torch.int16))
