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
