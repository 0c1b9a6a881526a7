"""The one-kernel decode layer (T <= 8) against the oracle.

moe_forward takes this path by itself for batches of up to 6 tokens when
nothing is saved for the backward, and moe_stack_forward runs each layer of
such a batch as one launch with the RMSNorm and the residual add fused;
moe_forward_decode calls it explicitly for up to 8 tokens. Its router sums
exact products in fp64, so the chosen experts are checked bit for bit on every
token (no near-tie allowance) and the weights to 1e-6; outputs at the usual bars (max-abs 2e-2, relative L2 1e-2);
losses to 1e-4 relative.
"""

import numpy as np
import pytest
import torch

import sparse_moe_transformer_route_b200 as M
from oracle import moe_oracle as O
from sparse_moe_transformer_route_b200 import synthetic as S
from tests._parity import LazyF64, assert_close, assert_loss_close, f64, require_gpu
from tests.test_gpu_workloads import _check_stack_per_layer, _gpu_stack_layers

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


@pytest.fixture(scope="module")
def olmoe_layer():
    return S.make_weights(S.PREFILL_4096, seed=78)


def _decode(sh, x, wr, wgu, wd, bias=None, renorm=False, explicit=True):
    cfg = M.config(sh.T, sh.d_model, sh.n_experts, sh.top_k, sh.d_ff, renorm=renorm)
    ws = M.workspace(cfg)
    dev = [t.cuda() for t in (x, wr, wgu, wd)]
    b = bias.cuda() if bias is not None else None
    y = torch.full_like(dev[0], float("nan"))
    losses = torch.empty(2, device="cuda")
    idx = torch.full((sh.T, sh.top_k), -1, dtype=torch.int32, device="cuda")
    w = torch.empty(sh.T, sh.top_k, device="cuda")
    if explicit:
        M.moe_forward_decode(cfg, dev[0], dev[1], b, dev[2], dev[3], y, losses, idx, w, ws)
    else:
        M.moe_forward(cfg, dev[0], dev[1], b, dev[2], dev[3], y, losses, idx, w, False, ws)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 0
    return dict(y=y.cpu(), losses=losses.cpu(), idx=idx.cpu().numpy(), w=w.cpu())


def _check(sh, x, wr, wgu, wd, out, bias=None, renorm=False):
    xx = f64(x)
    b = f64(bias) if bias is not None else None
    p, lse = O.softmax_lse(O.router_logits(xx, f64(wr), b))
    ref_idx, ref_w = O.topk_renorm(p, sh.top_k) if renorm else O.topk_no_renorm(p, sh.top_k)
    assert np.array_equal(out["idx"], ref_idx), "chosen experts differ from the exact ones"
    assert_close(out["w"], ref_w, "weights", max_abs=1e-6, rel_l2=1e-6)
    y_ref = O.experts_grouped(xx, ref_idx, ref_w, LazyF64(wgu), LazyF64(wd))
    assert_close(out["y"], y_ref, "y")
    L_lb, _ = O.load_balance_loss(ref_idx, p, sh.n_experts)
    assert_loss_close(out["losses"][0].item(), L_lb, "L_lb")
    assert_loss_close(out["losses"][1].item(), O.router_z_loss(lse), "L_z")


@pytest.mark.parametrize("T", [1, 2, 3, 5, 8])
def test_olmoe_shapes(olmoe_layer, T):
    sh = S.LayerShape(T=T)
    x = S.make_tokens(sh, seed=600 + T)
    out = _decode(sh, x, *olmoe_layer)
    _check(sh, x, *olmoe_layer, out)


@pytest.mark.parametrize("T", [1, 4, 6, 8])
def test_fused_and_layered_paths_agree(olmoe_layer, T):
    """moe_forward without save_for_backward runs the one-kernel layer up to 4
    tokens (bit-identical to moe_forward_decode there); with save_for_backward
    it runs the layered kernels. Both choose the same experts; weights and
    outputs agree."""
    sh = S.LayerShape(T=T)
    x = S.make_tokens(sh, seed=700 + T)
    fused = _decode(sh, x, *olmoe_layer, explicit=True)
    auto = _decode(sh, x, *olmoe_layer, explicit=False)
    assert np.array_equal(auto["idx"], fused["idx"])
    if T <= 4:
        assert torch.equal(auto["y"], fused["y"])
    cfg = M.config(T, sh.d_model, sh.n_experts, sh.top_k, sh.d_ff)
    ws = M.workspace(cfg, True)
    dev = [t.cuda() for t in (x, *olmoe_layer)]
    y = torch.empty_like(dev[0])
    idx = torch.empty(T, 8, dtype=torch.int32, device="cuda")
    w = torch.empty(T, 8, device="cuda")
    M.moe_forward(cfg, dev[0], dev[1], None, dev[2], dev[3], y, None, idx, w, True, ws)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 0
    assert np.array_equal(idx.cpu().numpy(), fused["idx"])
    assert_close(w.cpu(), f64(fused["w"]), "weights, layered vs fused", max_abs=1e-5, rel_l2=1e-5)
    assert_close(y.cpu(), f64(fused["y"]), "y, layered vs fused")


@pytest.mark.parametrize("T,d,E,k,f,bias,renorm", [
    (2, 2048, 64, 8, 1024, True, False),    # OLMoE with the Zipf router offset
    (3, 2048, 64, 8, 1024, False, True),    # renormalised weights
    (5, 256, 1, 1, 128, False, False),      # one expert: every token takes it
    (8, 4096, 16, 4, 512, False, False),    # wide model, 64 KB of staged tokens
    (7, 128, 64, 16, 2048, False, False),   # k = 16, 7*16 (token, slot) rows of h, 448 KB
    (4, 512, 40, 5, 256, True, False),      # E not a multiple of 32
])
def test_shapes_and_options(T, d, E, k, f, bias, renorm):
    sh = S.LayerShape(T=T, d_model=d, n_experts=E, top_k=k, d_ff=f)
    inp = S.layer_inputs(sh, seed=T * 31 + E)
    b = S.zipf_router_offset(E) if bias else None
    cfg = M.config(T, d, E, k, f, renorm=renorm)
    fits = f <= 2 * d and max(T * d, T * k * f) * 2 + 8 * d <= 192 * 1024
    if not fits:  # beyond the kernel's staging: moe_forward_decode refuses, moe_forward runs the layered path
        with pytest.raises(M.MoeError) as e:
            _decode(sh, inp.x, inp.w_router, inp.w_gate_up, inp.w_down, b, renorm)
        assert e.value.status == 2
        out = _decode(sh, inp.x, inp.w_router, inp.w_gate_up, inp.w_down, b, renorm, explicit=False)
        y_ref = O.moe_forward(f64(inp.x), f64(inp.w_router), LazyF64(inp.w_gate_up), LazyF64(inp.w_down), k,
                              f64(b) if b is not None else None, renorm=renorm)["y"]
        assert_close(out["y"], y_ref, "y (layered)")
        return
    out = _decode(sh, inp.x, inp.w_router, inp.w_gate_up, inp.w_down, b, renorm)
    _check(sh, inp.x, inp.w_router, inp.w_gate_up, inp.w_down, out, b, renorm)


def test_stack_of_decode_layers():
    """Four skewed layers at T = 4 (one fused launch per layer, RMSNorm and the
    residual add inside): every token of every layer against the oracle fed
    that layer's input; the whole stack in one call equals its trace variant
    and its single-layer calls, with consistent per-layer counts."""
    sh = S.LayerShape(T=4, d_model=512, n_experts=64, top_k=8, d_ff=256)
    n = 4
    x0, layers = S.stack_inputs(sh, n, seed=13)
    _check_stack_per_layer(sh, x0, layers)
    r1, _ = _gpu_stack_layers(sh, x0, layers, trace=False)
    r2, tr = _gpu_stack_layers(sh, x0, layers)
    assert torch.equal(r1, r2)
    r = x0
    for L in layers:
        r, _ = _gpu_stack_layers(sh, r, [L], trace=False)
    assert torch.equal(r1, r)
    for l in range(n):
        assert np.array_equal(np.bincount(tr["idx"][l].reshape(-1), minlength=sh.n_experts), tr["counts"][l])


def test_deterministic_and_refusals(olmoe_layer):
    sh = S.LayerShape(T=6)
    x = S.make_tokens(sh, seed=800)
    a = _decode(sh, x, *olmoe_layer)
    b = _decode(sh, x, *olmoe_layer)
    assert torch.equal(a["y"], b["y"]) and torch.equal(a["losses"], b["losses"])
    big = S.LayerShape(T=9)
    with pytest.raises(M.MoeError) as e:
        _decode(big, S.make_tokens(big, seed=801), *olmoe_layer)
    assert e.value.status == 2


@pytest.fixture(scope="module")
def olmoe_stack_weights():
    """Sixteen OLMoE-shape layers (the skewed stack's weights and Zipf offset)."""
    _, layers = S.stack_inputs(S.LayerShape(T=1), S.STACK_LAYERS, seed=8)
    return layers


@pytest.mark.parametrize("T", [1, 4])
def test_sixteen_layer_decode_stack_in_one_launch(olmoe_stack_weights, T):
    """The whole 16-layer stack of decode blocks as one persistent launch: every
    layer on the oracle's residual at its depth, and the one-launch stack equal
    bit for bit to its sixteen single-layer launches."""
    sh = S.LayerShape(T=T)
    x0 = S.make_tokens(sh, seed=90 + T, dtype=torch.float32, normalised=False)
    layers = olmoe_stack_weights
    _check_stack_per_layer(sh, x0, layers)
    one, tr = _gpu_stack_layers(sh, x0, layers)
    r = x0
    for L in layers:
        r, _ = _gpu_stack_layers(sh, r, [L], trace=False)
    assert torch.equal(one, r)
    for l in range(len(layers)):
        assert np.array_equal(np.bincount(tr["idx"][l].reshape(-1), minlength=sh.n_experts), tr["counts"][l])
