"""A wait that runs out: the kernel records a status, finishes, and the
workspace and context stay usable.

Every wait inside the kernels is bounded (about one second). The one-kernel
decode layer's grid barrier counts arrivals in the workspace's control words
(word 3: arrivals, counted up through a launch, barrier j opening at j times
the grid; word 4: CTAs past their last barrier), compared as wrap-around
differences. With the arrival count started 2^20 below zero, no barrier's
target is ever reached: each CTA's wait gives up, records the grid-wait status
and the kernel returns. Nothing faults and nothing hangs; the host reads the
status (which clears it and the counters) and the next call is normal. A
launch that finds the status word already set does nothing at all.
"""

import numpy as np
import pytest
import torch

import sparse_moe_transformer_route_b200 as M
from oracle import moe_oracle as O
from sparse_moe_transformer_route_b200 import synthetic as S
from tests._parity import LazyF64, assert_close, f64, require_gpu

pytestmark = pytest.mark.gpu

GRID_WAIT_TIMEOUT = 0x105


@pytest.fixture(autouse=True, scope="module")
def _gpu():
    require_gpu()


def test_grid_barrier_wait_runs_out_and_reports():
    sh = S.LayerShape(T=1, d_model=256, n_experts=16, top_k=4, d_ff=256)
    inp = S.layer_inputs(sh, seed=90)
    cfg = M.config(sh.T, sh.d_model, sh.n_experts, sh.top_k, sh.d_ff)
    ws = M.workspace(cfg)
    x, wr, wgu, wd = (t.cuda() for t in (inp.x, inp.w_router, inp.w_gate_up, inp.w_down))
    y = torch.zeros_like(x)
    ws.view(torch.int32)[3] = -(1 << 20)  # an arrival count no barrier can complete from
    M.moe_forward_decode(cfg, x, wr, None, wgu, wd, y, None, None, None, ws)
    torch.cuda.synchronize()  # returns: the waits gave up
    assert M.moe_get_device_status(ws) == GRID_WAIT_TIMEOUT
    # the status read cleared the counters: the same workspace works again
    M.moe_forward_decode(cfg, x, wr, None, wgu, wd, y, None, None, None, ws)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 0
    ref = O.moe_forward(f64(inp.x), f64(inp.w_router), LazyF64(inp.w_gate_up), LazyF64(inp.w_down), sh.top_k)
    assert_close(y.cpu(), ref["y"], "y after recovery")
    assert np.isfinite(y.cpu().float().numpy()).all()


def test_decode_does_nothing_while_a_failure_is_recorded():
    sh = S.LayerShape(T=2, d_model=256, n_experts=16, top_k=4, d_ff=256)
    inp = S.layer_inputs(sh, seed=91)
    cfg = M.config(sh.T, sh.d_model, sh.n_experts, sh.top_k, sh.d_ff)
    ws = M.workspace(cfg)
    x, wr, wgu, wd = (t.cuda() for t in (inp.x, inp.w_router, inp.w_gate_up, inp.w_down))
    y = torch.full_like(x, 7.0)
    ws.view(torch.int32)[0] = GRID_WAIT_TIMEOUT  # as a launch that gave up leaves it
    ws.view(torch.int32)[3] = 5  # and a stale arrival count
    M.moe_forward_decode(cfg, x, wr, None, wgu, wd, y, None, None, None, ws)
    torch.cuda.synchronize()
    assert torch.all(y == 7.0), "the kernel ran although a failure was recorded"
    assert M.moe_get_device_status(ws) == GRID_WAIT_TIMEOUT
    M.moe_forward_decode(cfg, x, wr, None, wgu, wd, y, None, None, None, ws)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 0
    ref = O.moe_forward(f64(inp.x), f64(inp.w_router), LazyF64(inp.w_gate_up), LazyF64(inp.w_down), sh.top_k)
    assert_close(y.cpu(), ref["y"], "y after the status was read")
