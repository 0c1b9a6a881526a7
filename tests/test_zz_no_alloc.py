"""moe_route_static, the router entry point that allocates nothing.

Some callers cannot give the library device memory: their device memory is
planned and owned by a host framework or a serving runtime, or they run a loop
that must not call cudaMalloc (it synchronises the device). moe_route_static
serves them with the router's scratch in a fixed array inside the library.
These tests call it through the C ABI and compare it with moe_route, which
uses a caller-provided workspace, on two calls in a row (the second call finds
the first one's contents in the shared array). This file is collected last.
"""

import pytest
import torch

import sparse_moe_transformer_route_b200 as M
from sparse_moe_transformer_route_b200 import synthetic as S
from tests._parity import assert_close, assert_loss_close, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _outputs(cfg):
    T, E, k = cfg.T, cfg.n_experts, cfg.top_k
    return dict(idx=torch.full((T, k), -7, dtype=torch.int32, device="cuda"),
                w=torch.full((T, k), float("nan"), device="cuda"),
                counts=torch.full((E,), -7, dtype=torch.int32, device="cuda"),
                losses=torch.full((2,), float("nan"), device="cuda"))


def test_static_router_matches_workspace_router_on_two_calls():
    calls = [
        (S.PREFILL_4096, 1, None),                                        # the OLMoE layer
        (S.LayerShape(300, 512, 64, 8, 256), 2, S.zipf_router_offset(64)),  # smaller, skewed
    ]
    for shape, seed, bias in calls:
        inp = S.layer_inputs(shape, seed=seed)
        x, wr = inp.x.cuda(), inp.w_router.cuda()
        b = bias.cuda() if bias is not None else None
        cfg = M.config(shape.T, shape.d_model, shape.n_experts, shape.top_k, shape.d_ff)
        ref = _outputs(cfg)
        ws = M.workspace(cfg)
        M.moe_route(cfg, x, wr, b, ref["idx"], ref["w"], ref["counts"], ref["losses"], ws)
        got = _outputs(cfg)
        M.moe_route_static(cfg, x, wr, b, got["idx"], got["w"], got["counts"], got["losses"])
        torch.cuda.synchronize()
        assert torch.equal(got["idx"], ref["idx"])
        assert torch.equal(got["counts"], ref["counts"])
        assert_close(got["w"], ref["w"].cpu().double().numpy(), "router weights")
        for i in range(2):
            assert_loss_close(got["losses"][i].item(), ref["losses"][i].item(), f"loss {i}")


def test_static_router_rejects_calls_beyond_its_scratch():
    cfg = M.config(S.TRAIN_16384.T, 2048, 64, 8, 1024)
    x = torch.zeros(cfg.T, 2048, dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros(64, 2048, dtype=torch.bfloat16, device="cuda")
    out = _outputs(cfg)
    with pytest.raises(M.MoeError) as ei:
        M.moe_route_static(cfg, x, wr, None, out["idx"], out["w"], out["counts"], out["losses"])
    assert ei.value.status == 3  # MOE_ERR_WORKSPACE_TOO_SMALL
    assert torch.all(out["idx"] == -7)  # nothing was launched
