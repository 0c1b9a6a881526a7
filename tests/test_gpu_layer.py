"""The whole layer through the C ABI against the oracle, on seeded inputs.

Indices: bit-exact on every token that is not a near-tie (two neighbours among
the k+1 largest probabilities closer than 1e-6 relative); near-ties are
counted. Outputs and gradients: max-abs 2e-2 and relative L2 1e-2. Losses:
1e-4 relative.
"""

import numpy as np
import pytest
import torch

import sparse_moe_transformer_route_b200 as M
from oracle import moe_oracle as O
from sparse_moe_transformer_route_b200 import synthetic as S
from tests._layer import check_forward, run_forward
from tests._parity import LazyF64, assert_close, bf16_round, f64, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def test_small_fp32_layer():
    """T=128, d=512, E=64, k=8, f=256 in fp32, seed 0, x ~ N(0, 1)."""
    inp = S.layer_inputs(S.SMALL_FP32, seed=0, dtype=torch.float32, normalised=False)
    out = run_forward(inp)
    check_forward(inp, out)


@pytest.mark.parametrize("T,d,E,k,f", [(300, 256, 16, 4, 256), (1000, 512, 64, 8, 256), (1, 2048, 64, 8, 1024),
                                       (77, 384, 32, 3, 128)])
def test_bf16_layers_with_ragged_groups(T, d, E, k, f):
    inp = S.layer_inputs(S.LayerShape(T, d, E, k, f), seed=T + d)
    out = run_forward(inp)
    check_forward(inp, out)


def test_eight_experts_take_every_token():
    """A large router offset on experts 0..7: they receive all T rows (several
    tiles each) and the other 56 experts none."""
    sh = S.LayerShape(600, 256, 64, 8, 256)
    inp = S.layer_inputs(sh, seed=4)
    bias = torch.zeros(64)
    bias[:8] = 30.0
    out = run_forward(inp, bias=bias)
    assert set(np.unique(out["idx"].cpu().numpy())) == set(range(8))
    check_forward(inp, out, bias=bias)


def _route_gpu_and_oracle(inp, bias=None):
    out = run_forward(inp, bias=bias)
    h = O.router_logits(f64(inp.x), f64(inp.w_router), None if bias is None else f64(bias))
    p, _ = O.softmax_lse(h)
    ref_idx, _ = O.topk_no_renorm(p, inp.shape.top_k)
    return out["idx"].cpu().numpy(), ref_idx


def test_router_breaks_exact_ties_by_lower_index():
    """Experts 0..15 share one router row, so their logits are equal for every
    token: the choice among them must go to the lower indices, on every token."""
    sh = S.LayerShape(333, 512, 64, 8, 256)
    inp = S.layer_inputs(sh, seed=31)
    wr = inp.w_router.clone()
    wr[1:16] = wr[0]
    inp.w_router = wr
    got, ref = _route_gpu_and_oracle(inp)
    assert np.array_equal(got, ref)


def test_router_orders_logits_one_ulp_apart():
    """Odd experts copy the even expert's router row with one weight moved by one
    bf16 ulp: their logits differ by ~1e-4, inside the fp32 uncertainty band the
    router re-ranks with exact arithmetic, and the order must match on every token."""
    sh = S.LayerShape(1000, 2048, 64, 8, 1024)
    inp = S.layer_inputs(sh, seed=32)
    wr = inp.w_router.clone()
    g = torch.Generator().manual_seed(3)
    for e in range(0, 64, 2):
        row = wr[e].clone()
        i = int(torch.randint(0, 2048, (1,), generator=g))
        row.view(torch.int16)[i] += 1  # the next bf16 value (one ulp in magnitude)
        wr[e + 1] = row
    inp.w_router = wr
    got, ref = _route_gpu_and_oracle(inp)
    assert np.array_equal(got, ref)


def test_olmoe_prefill_4096():
    """The OLMoE-shape layer: T=4096, d=2048, E=64, k=8, f=1024, bf16. Routing of
    every token; outputs on a sample of tokens (the first, the last, and 46 drawn)."""
    inp = S.layer_inputs(S.PREFILL_4096, seed=1)
    out = run_forward(inp)
    r = np.random.default_rng(0)
    sample = np.unique(np.concatenate([[0, 4095], r.choice(4096, 46, replace=False)]))
    check_forward(inp, out, sample=sample)


def test_forward_is_deterministic_and_stages_compose():
    sh = S.LayerShape(700, 512, 64, 8, 256)
    inp = S.layer_inputs(sh, seed=12)
    a = run_forward(inp)
    b = run_forward(inp)
    assert torch.equal(a["y"], b["y"]) and torch.equal(a["losses"], b["losses"])
    # the stage entry points reproduce moe_forward bit for bit
    x, wr, wgu, wd, _ = a["dev"]
    cfg = a["cfg"]
    T, E, k = sh.T, sh.n_experts, sh.top_k
    P = M.moe_padded_rows(cfg)
    ws = M.workspace(cfg)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    losses = torch.empty(2, device="cuda")
    M.moe_route(cfg, x, wr, None, idx, w, counts, losses, ws)
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    gs = torch.empty_like(off)
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty_like(perm)
    xp = torch.empty(P, sh.d_model, dtype=x.dtype, device="cuda")
    M.moe_dispatch(cfg, idx, x, off, perm, inv, gs, xp, ws)
    h = torch.empty(P, sh.d_ff, dtype=x.dtype, device="cuda")
    op = torch.empty(P, sh.d_model, dtype=x.dtype, device="cuda")
    M.moe_expert_ffn(cfg, xp, gs, off, wgu, wd, h, op, ws)
    y = torch.empty_like(x)
    M.moe_combine(cfg, op, inv, w, y)
    torch.cuda.synchronize()
    assert torch.equal(y, a["y"]) and torch.equal(losses, a["losses"]) and torch.equal(idx, a["idx"])
    assert int(counts.sum()) == T * k
    assert np.array_equal(counts.cpu().numpy(), np.bincount(idx.cpu().numpy().reshape(-1), minlength=E))


def test_host_buffer_entry_point_matches_device():
    sh = S.LayerShape(256, 512, 64, 8, 256)
    inp = S.layer_inputs(sh, seed=13)
    a = run_forward(inp)
    x, wr, wgu, wd, _ = a["dev"]
    cfg = a["cfg"]
    ws = M.workspace(cfg)
    xh = inp.x.clone().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    lh = torch.empty(2).pin_memory()
    M.moe_forward_host(cfg, xh, wr, None, wgu, wd, yh, lh, ws)
    assert torch.equal(yh, a["y"].cpu()) and torch.equal(lh, a["losses"].cpu())


def test_async_host_entry_point_with_two_calls_in_flight():
    """moe_forward_host_async on two streams, each with its own workspace and
    output buffers, three rounds: every call's result equals the device-buffer
    forward of its own tokens."""
    sh = S.LayerShape(1024, 512, 64, 8, 256)
    inps = [S.layer_inputs(sh, seed=40)]
    inps.append(S.LayerInputs(sh, S.make_tokens(sh, seed=41), inps[0].w_router, inps[0].w_gate_up, inps[0].w_down))
    refs = [run_forward(i) for i in inps]
    x, wr, wgu, wd, _ = refs[0]["dev"]
    cfg = refs[0]["cfg"]
    streams = [torch.cuda.Stream() for _ in range(2)]
    wss = [M.workspace(cfg) for _ in range(2)]
    xh = [i.x.clone().pin_memory() for i in inps]
    yh = [torch.empty_like(xh[0]).pin_memory() for _ in range(2)]
    lh = [torch.empty(2).pin_memory() for _ in range(2)]
    for _ in range(3):
        for j in range(2):
            yh[j].fill_(float("nan"))
        torch.cuda.synchronize()
        for j in range(2):
            M.moe_forward_host_async(cfg, xh[j], wr, None, wgu, wd, yh[j], lh[j], wss[j], stream=streams[j])
        for st in streams:
            st.synchronize()
        for j in range(2):
            assert torch.equal(yh[j], refs[j]["y"].cpu()) and torch.equal(lh[j], refs[j]["losses"].cpu())
    for ws in wss:
        assert M.moe_get_device_status(ws) == 0


def check_backward(inp, alpha=0.01, beta=0.001, experts=None, tol_scale=1.0, renorm=False):
    sh = inp.shape
    x, wr, wgu, wd, dy = (t.cuda() for t in (inp.x, inp.w_router, inp.w_gate_up, inp.w_down, inp.dy))
    cfg = M.config(sh.T, sh.d_model, sh.n_experts, sh.top_k, sh.d_ff, x.dtype, alpha, beta, renorm=renorm)
    ws = M.workspace(cfg, True)
    y = torch.empty_like(x)
    losses = torch.empty(2, device="cuda")
    idx = torch.empty(sh.T, sh.top_k, dtype=torch.int32, device="cuda")
    M.moe_forward(cfg, x, wr, None, wgu, wd, y, losses, idx, None, True, ws)
    g = dict(dx=torch.empty_like(x), dw_router=torch.empty_like(wr), dw_gate_up=torch.empty_like(wgu),
             dw_down=torch.empty_like(wd))
    M.moe_backward(cfg, dy, x, wr, wgu, wd, g["dx"], g["dw_router"], g["dw_gate_up"], g["dw_down"], ws)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 0
    args = (f64(inp.x), f64(inp.w_router), LazyF64(inp.w_gate_up), LazyF64(inp.w_down), sh.top_k, f64(inp.dy),
            alpha, beta)
    # the reference rounds the contraction operands (h, do, [da; db]) to bf16, as
    # bf16 inputs are; at these sizes the unrounded oracle is met at both bars too
    refs = (("", O.moe_backward(*args, experts=experts, renorm=renorm, store=bf16_round)),
            (" (unrounded oracle)", O.moe_backward(*args, experts=experts, renorm=renorm)))
    # gradients sum over tokens, so the routing must agree on every token (near-ties
    # included: the router decides on logits accumulated in fp64 from exact products)
    assert np.array_equal(idx.cpu().numpy(), refs[0][1]["fwd"]["idx"]), "routing differs from the oracle"
    es = range(sh.n_experts) if experts is None else experts
    for tag, ref in refs:
        assert_close(g["dx"], ref["dx"], "dx" + tag)
        assert_close(g["dw_router"], ref["dw_router"], "dW_router" + tag)
        for e in es:
            assert_close(g["dw_gate_up"][e], ref["dw_gate_up"][e], f"dW_gate_up[{e}]" + tag)
            assert_close(g["dw_down"][e], ref["dw_down"][e], f"dW_down[{e}]" + tag)
    return g


def test_backward_small_layer_bf16():
    """The small layer's shapes (T=128, d=512, E=64, k=8, f=256) in bf16."""
    inp = S.layer_inputs(S.SMALL_FP32, seed=0, dtype=torch.bfloat16, normalised=False, with_grad=True)
    check_backward(inp)


def test_backward_rejects_fp32():
    sh = S.SMALL_FP32
    cfg = M.config(sh.T, sh.d_model, sh.n_experts, sh.top_k, sh.d_ff, torch.float32)
    ws = M.workspace(cfg, True)
    t = torch.zeros(sh.T, sh.d_model, device="cuda")
    wr = torch.zeros(sh.n_experts, sh.d_model, device="cuda")
    wgu = torch.zeros(sh.n_experts, 2 * sh.d_ff, sh.d_model, device="cuda")
    wd = torch.zeros(sh.n_experts, sh.d_model, sh.d_ff, device="cuda")
    with pytest.raises(M.MoeError) as ei:
        M.moe_backward(cfg, t, t, wr, wgu, wd, t.clone(), wr.clone(), wgu.clone(), wd.clone(), ws)
    assert ei.value.status == 2


@pytest.mark.parametrize("T,d,E,k,f", [(512, 256, 16, 4, 256), (300, 384, 8, 2, 128)])
def test_backward_bf16(T, d, E, k, f):
    inp = S.layer_inputs(S.LayerShape(T, d, E, k, f), seed=T, with_grad=True)
    check_backward(inp)


def test_backward_loss_terms_alone():
    """dy = 0: only alpha * L_lb + beta * L_z drive the router gradient."""
    sh = S.LayerShape(256, 256, 16, 4, 128)
    inp = S.layer_inputs(sh, seed=21, dtype=torch.bfloat16, with_grad=True)
    inp.dy = torch.zeros_like(inp.dy)
    check_backward(inp, alpha=0.5, beta=0.25)


# ------------------------------------------------------------------ renormalised router


@pytest.mark.parametrize("T,d,E,k,f,dtype", [(128, 512, 64, 8, 256, torch.float32),   # SIMT router
                                             (1000, 512, 64, 8, 256, torch.bfloat16),  # tensor-core router
                                             (5000, 256, 16, 4, 128, torch.bfloat16)])  # split router
def test_renormalised_router_forward(T, d, E, k, f, dtype):
    """Router mode 1: the same experts, weights summing to one per token."""
    inp = S.layer_inputs(S.LayerShape(T, d, E, k, f), seed=T + 7, dtype=dtype, normalised=dtype != torch.float32)
    out = run_forward(inp, renorm=True)
    sample = None if T <= 1000 else np.arange(0, T, 97)
    check_forward(inp, out, sample=sample, renorm=True)
    assert torch.allclose(out["w"].sum(dim=1), torch.ones(T, device="cuda"), atol=1e-5)


def test_renormalised_router_backward():
    inp = S.layer_inputs(S.LayerShape(384, 256, 16, 4, 256), seed=44, with_grad=True)
    check_backward(inp, alpha=0.3, beta=0.2, renorm=True)


# ------------------------------------------------------------------ edge cases


@pytest.mark.parametrize("T,d,E,k,f", [
    (100, 128, 1, 1, 128),     # one expert: p = w = 1, the layer is a plain SwiGLU MLP
    (50, 256, 2, 2, 128),      # every expert chosen by every token
    (3, 128, 64, 16, 128),     # the largest k, fewer tokens than one tile
    (33, 4096, 16, 4, 4096),   # the largest d and f (bf16)
    (260, 256, 256, 16, 128),  # the most experts (SIMT router) with the largest k
    (257, 512, 40, 5, 256),    # E not a multiple of 16, ragged last tile
])
def test_edge_shapes(T, d, E, k, f):
    inp = S.layer_inputs(S.LayerShape(T, d, E, k, f), seed=T + E)
    out = run_forward(inp)
    check_forward(inp, out)
    if E == 1:
        assert torch.all(out["w"] == 1) and torch.all(out["idx"] == 0)
