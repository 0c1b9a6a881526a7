"""moe_route_static, the router entry point that allocates nothing.

Some callers cannot give the library device memory: their device memory is
planned and owned by a host framework or a serving runtime, or they run a loop
that must not call cudaMalloc (it synchronises the device). moe_route_static
serves them with the router's scratch in a fixed array inside the library.
These tests call it through the C ABI: against the oracle's routing, and
against moe_route (which uses a caller-provided workspace) on two calls in a row
(the second call finds the first one's contents in the shared array); at the
largest batch the array holds and one token beyond. This file is collected last.
"""

import numpy as np
import pytest
import torch

import sparse_moe_transformer_route_b200 as M
from oracle import moe_oracle as O
from sparse_moe_transformer_route_b200 import synthetic as S
from tests._parity import assert_close, assert_loss_close, f64, index_parity, require_gpu

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


def _route_static(shape, seed, dtype=torch.bfloat16, bias=None, normalised=True):
    inp = S.layer_inputs(shape, seed=seed, dtype=dtype, normalised=normalised)
    cfg = M.config(shape.T, shape.d_model, shape.n_experts, shape.top_k, shape.d_ff, dtype)
    got = _outputs(cfg)
    b = bias.cuda() if bias is not None else None
    M.moe_route_static(cfg, inp.x.cuda(), inp.w_router.cuda(), b, got["idx"], got["w"], got["counts"],
                       got["losses"])
    torch.cuda.synchronize()
    return inp, {n: t.cpu() for n, t in got.items()}


def _check_routing_against_oracle(inp, got, bias=None):
    """The chosen experts bit-exact except near-ties, their weights to 1e-5, the
    counts, and both losses to 1e-4 relative."""
    k, E = inp.shape.top_k, inp.shape.n_experts
    p, lse = O.softmax_lse(O.router_logits(f64(inp.x), f64(inp.w_router), f64(bias) if bias is not None else None))
    idx, w = O.topk_no_renorm(p, k)
    bad, _, diff = index_parity(got["idx"].numpy(), idx, O.near_tie_tokens(p, k))
    assert bad.size == 0, f"{bad.size} tokens routed differently from the oracle"
    same = ~diff
    assert_close(got["w"][torch.from_numpy(same)], w[same], "router weights", max_abs=1e-5, rel_l2=1e-5)
    assert np.array_equal(got["counts"].numpy(), np.bincount(got["idx"].numpy().reshape(-1), minlength=E))
    if not diff.any():
        assert np.array_equal(got["counts"].numpy(), np.bincount(idx.reshape(-1), minlength=E))
    L_lb, _ = O.load_balance_loss(idx, p, E)
    assert_loss_close(got["losses"][0].item(), L_lb, "L_lb")
    assert_loss_close(got["losses"][1].item(), O.router_z_loss(lse), "L_z")


def test_static_router_matches_oracle():
    """The OLMoE prefill layer (bf16), the small fp32 layer, a skewed bf16 layer."""
    inp, got = _route_static(S.PREFILL_4096, seed=3)
    _check_routing_against_oracle(inp, got)
    inp, got = _route_static(S.SMALL_FP32, seed=0, dtype=torch.float32, normalised=False)
    _check_routing_against_oracle(inp, got)
    bias = S.zipf_router_offset(64)
    inp, got = _route_static(S.LayerShape(300, 512, 64, 8, 256), seed=5, bias=bias)
    _check_routing_against_oracle(inp, got, bias)


def test_static_router_at_its_size_limit():
    """7,167 tokens of 64 experts fill the array (T (4.5 E + 4.5) bytes plus
    alignment); 7,168 do not and are refused before anything is launched."""
    inp, got = _route_static(S.LayerShape(7167), seed=9)
    _check_routing_against_oracle(inp, got)
    cfg = M.config(7168, 2048, 64, 8, 1024)
    x = torch.zeros(cfg.T, 2048, dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros(64, 2048, dtype=torch.bfloat16, device="cuda")
    out = _outputs(cfg)
    with pytest.raises(M.MoeError) as ei:
        M.moe_route_static(cfg, x, wr, None, out["idx"], out["w"], out["counts"], out["losses"])
    assert ei.value.status == 3  # MOE_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
    assert torch.all(out["idx"] == -7)  # nothing was launched


def test_static_router_rejects_calls_beyond_its_scratch():
    cfg = M.config(S.TRAIN_16384.T, 2048, 64, 8, 1024)
    x = torch.zeros(cfg.T, 2048, dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros(64, 2048, dtype=torch.bfloat16, device="cuda")
    out = _outputs(cfg)
    with pytest.raises(M.MoeError) as ei:
        M.moe_route_static(cfg, x, wr, None, out["idx"], out["w"], out["counts"], out["losses"])
    assert ei.value.status == 3  # MOE_ERR_WORKSPACE_TOO_SMALL
    assert torch.all(out["idx"] == -7)  # nothing was launched
