"""Expert-choice routing on the GPU against the oracle.

Each expert keeps the C tokens with the largest router probability for it
("OLMoE: Open Mixture-of-Experts Language Models", section 4.1.4, read as the
oracle's module notes state). The kernel re-ranks the tokens near each
expert's C-th value by exact keys, so its choice is compared directly with the
oracle's choice on fp64 probabilities: a token chosen by one side only must
sit within 1e-6 (relative) of the expert's C-th value (a near-tie, counted).
The probabilities themselves, the z-loss and the layer output are compared with
the oracle at the usual bars.
"""

import numpy as np
import pytest
import torch

import sparse_moe_transformer_route_b200 as M
from oracle import moe_oracle as O
from sparse_moe_transformer_route_b200 import synthetic as S
from tests._parity import LazyF64, assert_close, assert_loss_close, f64, require_gpu

pytestmark = pytest.mark.gpu

BOUNDARY_REL = 1e-6


@pytest.fixture(autouse=True, scope="module")
def _gpu():
    require_gpu()


def _route(inp, capacity=0, bias=None):
    sh = inp.shape
    x, wr = inp.x.cuda(), inp.w_router.cuda()
    cfg = M.config(sh.T, sh.d_model, sh.n_experts, sh.top_k, sh.d_ff, x.dtype)
    C = capacity if capacity > 0 else M.moe_expert_choice_capacity(cfg)
    ws = M.workspace(cfg)
    sel = torch.full((sh.n_experts, C), -7, dtype=torch.int32, device="cuda")
    gates = torch.empty(sh.n_experts, C, device="cuda")
    probs = torch.empty(sh.T, sh.n_experts, device="cuda")
    counts = torch.empty(sh.n_experts, dtype=torch.int32, device="cuda")
    losses = torch.empty(2, device="cuda")
    b = bias.cuda() if bias is not None else None
    M.moe_route_expert_choice(cfg, x, wr, b, sel, gates, probs, counts, losses, ws, capacity=capacity)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 0
    return dict(cfg=cfg, C=C, default=capacity <= 0, sel=sel.cpu().numpy(), gates=gates.cpu(), probs=probs.cpu(),
                counts=counts.cpu(), losses=losses.cpu())


def _forward(inp, capacity=0):
    sh = inp.shape
    x, wr, wgu, wd = (t.cuda() for t in (inp.x, inp.w_router, inp.w_gate_up, inp.w_down))
    cfg = M.config(sh.T, sh.d_model, sh.n_experts, sh.top_k, sh.d_ff, x.dtype)
    C = capacity if capacity > 0 else M.moe_expert_choice_capacity(cfg)
    ws = M.workspace(cfg)
    y = torch.full_like(x, float("nan"))
    losses = torch.empty(2, device="cuda")
    sel = torch.empty(sh.n_experts, C, dtype=torch.int32, device="cuda")
    gates = torch.empty(sh.n_experts, C, device="cuda")
    M.moe_forward_expert_choice(cfg, x, wr, None, wgu, wd, y, losses, sel, gates, ws, capacity=capacity)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 0
    return dict(C=C, y=y.cpu(), losses=losses.cpu(), sel=sel.cpu().numpy(), gates=gates.cpu())


def _check_routing(inp, r):
    """Selection, weights, probabilities, counts and losses against the oracle."""
    x = f64(inp.x)
    h = O.router_logits(x, f64(inp.w_router))
    p, lse = O.softmax_lse(h)
    C = r["C"]
    E = inp.shape.n_experts
    if r["default"]:
        assert C == O.ec_capacity(inp.shape.T, inp.shape.top_k, E)
    # probabilities (fp32 from fp32 tensor-core logits)
    assert_close(r["probs"], p, "probabilities", max_abs=1e-5, rel_l2=1e-5)
    # the weights are the kernel's probabilities of its chosen tokens, bit for bit
    kp = f64(r["probs"])
    want = torch.from_numpy(np.take_along_axis(kp.T, r["sel"].astype(np.int64), axis=1)).float()
    assert torch.equal(r["gates"], want)
    # the choice against the oracle's on fp64 probabilities: only near-ties may differ
    sel64, _ = O.expert_choice(p, C)
    n_boundary = 0
    for e in range(E):
        a, b = set(r["sel"][e].tolist()), set(sel64[e].tolist())
        if a == b:
            continue
        kth = np.sort(p[:, e])[::-1][C - 1]
        for t in a ^ b:
            assert abs(p[t, e] - kth) <= BOUNDARY_REL * kth, f"expert {e} token {t} is not a boundary tie"
        n_boundary += 1
    assert (r["counts"] == C).all()
    assert r["losses"][0].item() == 0.0
    assert_loss_close(r["losses"][1].item(), O.router_z_loss(lse), "L_z")
    return p, n_boundary


def _check_output(inp, out, p, tokens=None):
    """y on `tokens` (all when None) from the oracle's experts on the kernel's
    choice, weighted by the oracle's probabilities."""
    T = inp.shape.T
    E = inp.shape.n_experts
    sel = out["sel"]
    toks = np.arange(T) if tokens is None else np.unique(np.asarray(tokens))
    x = f64(inp.x)
    wgu = LazyF64(inp.w_gate_up)
    wd = LazyF64(inp.w_down)
    y_ref = np.zeros((toks.size, inp.shape.d_model))
    row = {t: i for i, t in enumerate(toks.tolist())}
    for e in range(E):
        hit = [t for t in sel[e].tolist() if t in row]
        if not hit:
            continue
        o = O.swiglu_expert(x[hit], wgu[e], wd[e])
        for j, t in enumerate(hit):
            y_ref[row[t]] += p[t, e] * o[j]
    got = out["y"][torch.from_numpy(toks)]
    assert_close(got, y_ref, "y")
    fan = np.bincount(sel.reshape(-1), minlength=T)
    dropped = toks[fan[toks] == 0]
    assert torch.all(out["y"][torch.from_numpy(dropped)] == 0)
    return int((fan == 0).sum())


@pytest.mark.parametrize("T,d,E,k,f", [(300, 256, 16, 4, 128), (257, 512, 64, 8, 256), (1000, 128, 8, 2, 128)])
def test_small_layers_every_token(T, d, E, k, f):
    inp = S.layer_inputs(S.LayerShape(T=T, d_model=d, n_experts=E, top_k=k, d_ff=f), seed=T + E)
    r = _route(inp)
    p, _ = _check_routing(inp, r)
    out = _forward(inp)
    # the forward makes the same choice as the routing call
    assert np.array_equal(out["sel"], r["sel"])
    assert torch.equal(out["gates"], r["gates"])
    assert torch.equal(out["losses"], r["losses"])
    _check_output(inp, out, p)


def test_olmoe_prefill_4096_tokens():
    """OLMoE's shapes at T=4096: C = 512 rows per expert, no padding rows; all
    routing checked, the output on 96 sampled tokens (first, last, dropped)."""
    inp = S.layer_inputs(S.PREFILL_4096, seed=41)
    r = _route(inp)
    assert r["C"] == 512
    p, _ = _check_routing(inp, r)
    out = _forward(inp)
    assert np.array_equal(out["sel"], r["sel"])
    fan = np.bincount(out["sel"].reshape(-1), minlength=4096)
    rng = np.random.default_rng(5)
    toks = np.concatenate([[0, 4095], np.nonzero(fan == 0)[0][:8], np.argsort(-fan)[:6], rng.choice(4096, 80)])
    _check_output(inp, out, p, toks)


def test_long_column_read_from_l2():
    """T past the shared-memory staging limit (40,960 tokens): the select reads its
    column from the probabilities in L2 on every pass."""
    sh = S.LayerShape(T=49152, d_model=128, n_experts=64, top_k=8, d_ff=128)
    inp = S.layer_inputs(sh, seed=43)
    r = _route(inp)
    assert r["C"] == 6144
    p, _ = _check_routing(inp, r)
    out = _forward(inp)
    rng = np.random.default_rng(6)
    _check_output(inp, out, p, np.concatenate([[0, 49151], rng.choice(49152, 64)]))


def test_exact_ties_go_to_the_lower_token():
    """Repeated token rows inside one 32-token router tile get bit-identical
    probabilities (rows of different tiles may differ in the last bits: each
    tile's CTA starts its walk over K at a different step), so every expert meets
    exact ties; the lower token indices must win."""
    sh = S.LayerShape(T=32, d_model=256, n_experts=16, top_k=2, d_ff=128)
    inp = S.layer_inputs(sh, seed=44)
    inp.x = inp.x[:4].clone().repeat(8, 1)  # token t equals token t mod 4
    r = _route(inp)
    assert r["C"] == 4
    kp = f64(r["probs"])
    assert np.array_equal(kp, np.tile(kp[:4], (8, 1)))
    p, _ = _check_routing(inp, r)
    # each expert takes the first four copies of its best distinct row
    for e in range(sh.n_experts):
        vals = kp[:4, e]
        best = int(np.argmax(vals))
        if np.sum(vals == vals[best]) == 1:
            assert r["sel"][e].tolist() == [best, best + 4, best + 8, best + 12]
    out = _forward(inp)
    _check_output(inp, out, p)


def test_exact_ties_across_router_tiles_go_to_the_lower_token():
    """Repeated rows spread over four 32-token router tiles: their fp32
    probabilities may differ in the last bits between tiles, but their exact
    keys are equal, so each expert takes the lowest-index copies of its best
    row (32 copies, C = 16 of them: the first 16)."""
    sh = S.LayerShape(T=128, d_model=256, n_experts=16, top_k=2, d_ff=128)
    inp = S.layer_inputs(sh, seed=48)
    inp.x = inp.x[:4].clone().repeat(32, 1)
    r = _route(inp)
    assert r["C"] == 16
    p, _ = _check_routing(inp, r)
    for e in range(sh.n_experts):
        vals = p[:4, e]
        best = int(np.argmax(vals))
        if np.sum(vals == vals[best]) == 1:
            assert r["sel"][e].tolist() == [best + 4 * i for i in range(16)]


@pytest.mark.parametrize("capacity", [1, 37, 200])
def test_explicit_capacities(capacity):
    """C = 1 (most tokens dropped: zero output), an odd C, and C = T (every expert
    takes every token: the dense softmax-weighted layer). k = E here, so the
    padded row count leaves room for C = T."""
    sh = S.LayerShape(T=200, d_model=256, n_experts=8, top_k=8, d_ff=128)
    inp = S.layer_inputs(sh, seed=45)
    r = _route(inp, capacity=capacity)
    assert r["C"] == capacity
    p, _ = _check_routing(inp, r)
    out = _forward(inp, capacity=capacity)
    n_dropped = _check_output(inp, out, p)
    if capacity == 200:
        assert n_dropped == 0 and (np.sort(out["sel"], axis=1) == np.arange(200)).all()
    if capacity == 1:
        assert n_dropped >= 200 - 8


def test_one_token_goes_to_every_expert():
    """T = 1: C = ceil(k / E) = 1, so each of the 64 experts takes the token."""
    inp = S.layer_inputs(S.LayerShape(T=1), seed=46)
    r = _route(inp)
    assert r["C"] == 1 and (r["sel"] == 0).all()
    p, _ = _check_routing(inp, r)
    out = _forward(inp)
    _check_output(inp, out, p)


def test_deterministic():
    inp = S.layer_inputs(S.LayerShape(T=2048, d_model=512, n_experts=64, top_k=8, d_ff=256), seed=47)
    a = _forward(inp)
    b = _forward(inp)
    assert torch.equal(a["y"], b["y"]) and np.array_equal(a["sel"], b["sel"])


def _outs(E, C):
    return torch.empty(E, C, dtype=torch.int32, device="cuda"), torch.empty(E, C, device="cuda")


def test_rejected_configs():
    x = torch.zeros(64, 256, dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros(8, 256, dtype=torch.bfloat16, device="cuda")
    cfg = M.config(64, 256, 8, 2, 128)
    ws = M.workspace(cfg)
    for cap in (65, 200):  # C > T; E groups of C rows do not fit the padded rows
        with pytest.raises(M.MoeError) as e:
            M.moe_route_expert_choice(cfg, x, wr, None, *_outs(8, cap), None, None, None, ws, capacity=cap)
        assert e.value.status == 1
    renorm = M.config(64, 256, 8, 2, 128, renorm=True)  # expert choice has no renormalised variant
    with pytest.raises(M.MoeError) as e:
        M.moe_route_expert_choice(renorm, x, wr, None, *_outs(8, 16), None, None, None, M.workspace(renorm))
    assert e.value.status == 2
    fp = M.config(64, 256, 8, 2, 128, torch.float32)  # the tensor-core router is bf16 only
    with pytest.raises(M.MoeError) as e:
        M.moe_route_expert_choice(fp, x.float(), wr.float(), None, *_outs(8, 16), None, None, None,
                                  M.workspace(fp))
    assert e.value.status == 2
