"""Pins for the CPU oracle: each checks it against something other than itself.

Sources of truth, by kind:
  * values printed on the pages (tests/golden/*.txt, each file cites its page);
  * closed forms (uniform routing gives L_lb = 1, zero router gives L_z = ln(E)^2,
    RMSNorm of a constant row);
  * special cases that reduce to a textbook routine (one expert, k = 1 is a
    plain SwiGLU MLP, checked against torch.nn.functional.silu);
  * brute force on tiny inputs (dispatch order by explicit loops, the
    every-expert-on-every-token layer);
  * central finite differences of the scalar objective for every gradient.
"""

import math
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_moe_transformer_route_b200 import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _small_layer(seed, T=24, d=32, E=16, k=4, f=8, std=0.2):
    r = _rng(seed)
    return dict(
        x=r.standard_normal((T, d)),
        w_router=r.standard_normal((E, d)) * std,
        w_gate_up=r.standard_normal((E, 2 * f, d)) * std,
        w_down=r.standard_normal((E, d, f)) * std,
        k=k,
    )


def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ------------------------------------------------------------------ router pins


def test_router_variants_worked_example():
    """The page's router table: with softmax then top-8 and no renormalisation the
    weights average 0.744 and differ from top-k-then-softmax by up to 2.23e-01."""
    table = {r[0]: r[1:] for r in _read_table("router_variants_seed0.txt")}
    torch.manual_seed(0)
    s = (torch.randn(1000, 64) * 2).double().numpy()
    p, _ = O.softmax_lse(s)
    idx, w = O.topk_no_renorm(p, 8)
    # top-k then softmax, written from the page's formula for that variant
    top_idx = np.argpartition(-s, 8, axis=1)[:, :8]
    top = np.take_along_axis(s, top_idx, axis=1)
    ref = np.exp(top - top.max(axis=1, keepdims=True))
    ref /= ref.sum(axis=1, keepdims=True)
    # same experts, compared as sets
    assert all(set(a) == set(b) for a, b in zip(idx.tolist(), top_idx.tolist()))
    # map the reference weights into the oracle's slot order
    ref_by_expert = [dict(zip(a, b)) for a, b in zip(top_idx.tolist(), ref.tolist())]
    ref_w = np.array([[m[e] for e in row] for m, row in zip(ref_by_expert, idx.tolist())])
    assert f"{np.abs(w - ref_w).max():.2e}" == table["softmax_topk"][1]
    assert f"{w.sum(axis=1).mean():.3f}" == table["softmax_topk"][2]
    idx_r, renorm = O.topk_renorm(p, 8)
    assert np.array_equal(idx_r, idx)
    # exact identity in real arithmetic; the page's 1.79e-07 is its fp32 rounding
    assert np.abs(renorm - ref_w).max() < 1e-12
    assert np.allclose(renorm.sum(axis=1), 1.0, atol=1e-14, rtol=0)
    assert float(table["softmax_topk_renorm"][1]) < 1e-6


def test_softmax_sums_to_one_and_topk_is_valid():
    r = _rng(1)
    h = r.standard_normal((300, 64)) * 3
    p, lse = O.softmax_lse(h)
    assert np.allclose(p.sum(axis=1), 1.0, atol=1e-14, rtol=0)
    assert np.allclose(lse, np.log(np.exp(h).sum(axis=1)), atol=1e-12, rtol=0)
    idx, w = O.topk_no_renorm(p, 8)
    assert idx.min() >= 0 and idx.max() < 64
    assert all(len(set(row)) == 8 for row in idx.tolist())
    # descending weights, every unchosen probability at most the smallest chosen
    assert np.all(np.diff(w, axis=1) <= 0)
    for t in range(300):
        rest = np.delete(p[t], idx[t])
        assert rest.max() <= w[t, -1]


def test_topk_ties_go_to_lower_index():
    p = np.full((1, 8), 1.0 / 8)
    idx, _ = O.topk_no_renorm(p, 3)
    assert idx.tolist() == [[0, 1, 2]]
    p = np.array([[0.1, 0.3, 0.2, 0.3, 0.1]])
    idx, w = O.topk_no_renorm(p, 3)
    assert idx.tolist() == [[1, 3, 2]]
    assert O.near_tie_tokens(p, 3).tolist() == [True]
    assert O.near_tie_tokens(np.array([[0.5, 0.3, 0.15, 0.05]]), 2).tolist() == [False]


def test_router_bias_is_an_additive_logit_offset():
    L = _small_layer(2)
    b = np.linspace(-1, 1, 16)
    h0 = O.router_logits(L["x"], L["w_router"])
    h1 = O.router_logits(L["x"], L["w_router"], b)
    assert np.allclose(h1 - h0, b[None, :], atol=1e-14)
    # a -inf offset removes an expert (the keep-mask of the pruning section)
    b2 = np.zeros(16)
    b2[[3, 5]] = -np.inf
    p, _ = O.softmax_lse(O.router_logits(L["x"], L["w_router"], b2))
    idx, _ = O.topk_no_renorm(p, 4)
    assert not np.isin(idx, [3, 5]).any()


def test_expected_experts_touched_under_uniform_routing():
    """E(1 - (1 - k/E)^B) experts per batch of B tokens under uniform routing
    (the formula of the section on experts in and out of GPU memory)."""
    r = _rng(3)
    E, k = 64, 8
    for B, trials in ((8, 3000), (32, 1500)):
        touched = []
        for _ in range(trials):
            p, _ = O.softmax_lse(r.standard_normal((B, E)))
            idx, _ = O.topk_no_renorm(p, k)
            touched.append(len(np.unique(idx)))
        expect = E * (1 - (1 - k / E) ** B)
        assert abs(np.mean(touched) - expect) < 0.01 * expect


# ------------------------------------------------------------------ losses


def test_load_balance_loss_is_one_when_probabilities_are_uniform():
    r = _rng(4)
    T, d, E, k = 50, 16, 64, 8
    x = r.standard_normal((T, d))
    p, lse = O.softmax_lse(O.router_logits(x, np.zeros((E, d))))
    # any selection at all: sum_i f_i = 1 and P_i = 1/E
    idx = np.stack([r.choice(E, k, replace=False) for _ in range(T)])
    L, counts = O.load_balance_loss(idx, p, E)
    assert abs(L - 1.0) < 1e-14
    assert counts.sum() == T * k
    assert abs(O.router_z_loss(lse) - math.log(64) ** 2) < 1e-12


def test_load_balance_loss_is_one_when_assignments_are_uniform():
    r = _rng(5)
    E, k, m = 64, 8, 3
    T = (E // k) * m
    h = r.standard_normal((T, E)) * 0.1  # arbitrary P
    for t in range(T):
        g = t % (E // k)
        h[t, g * k:(g + 1) * k] += 20.0  # token t selects experts 8g..8g+7
    p, _ = O.softmax_lse(h)
    idx, _ = O.topk_no_renorm(p, k)
    L, counts = O.load_balance_loss(idx, p, E)
    assert np.all(counts == T * k // E)
    assert abs(L - 1.0) < 1e-12


def test_load_balance_loss_hand_case():
    # T=2, E=4, k=1: token 0 -> expert 0, token 1 -> expert 0.
    p = np.array([[0.7, 0.1, 0.1, 0.1], [0.4, 0.3, 0.2, 0.1]])
    idx = np.array([[0], [0]])
    L, _ = O.load_balance_loss(idx, p, 4)
    # f = (1, 0, 0, 0); P_0 = 0.55; L = 4 * 0.55
    assert abs(L - 2.2) < 1e-14


def test_z_loss_closed_form():
    h = np.array([[0.0, 0.0], [math.log(3.0), 0.0]])
    _, lse = O.softmax_lse(h)
    expect = (math.log(2.0) ** 2 + math.log(4.0) ** 2) / 2
    assert abs(O.router_z_loss(lse) - expect) < 1e-15


# ------------------------------------------------------------------ dispatch


def test_dispatch_order_brute_force():
    r = _rng(6)
    T, E, k = 37, 16, 4
    idx = np.stack([r.choice(E, k, replace=False) for _ in range(T)])
    perm, counts, offsets = O.dispatch_order(idx, E)
    brute = []
    for e in range(E):
        for t in range(T):
            for j in range(k):
                if idx[t, j] == e:
                    brute.append(t * k + j)
    assert perm.tolist() == brute
    assert sorted(perm.tolist()) == list(range(T * k))  # bijection
    assert counts.sum() == T * k
    assert offsets[0] == 0 and offsets[-1] == T * k and np.all(np.diff(offsets) >= 0)
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(idx.reshape(-1)[seg] == e)
        assert np.all(np.diff(seg // k) > 0)  # ascending tokens inside a group


def test_dispatch_with_empty_and_full_experts():
    T, E, k = 10, 8, 2
    idx = np.tile(np.array([[3, 5]]), (T, 1))
    perm, counts, offsets = O.dispatch_order(idx, E)
    assert counts.tolist() == [0, 0, 0, T, 0, T, 0, 0]
    assert perm[:T].tolist() == [t * k for t in range(T)]
    assert perm[T:].tolist() == [t * k + 1 for t in range(T)]


# ------------------------------------------------------------------ experts


def test_single_expert_is_a_plain_swiglu_mlp():
    """E = 1, k = 1: the weight is p = 1 and the layer is SwiGLU(x)."""
    r = _rng(7)
    T, d, f = 20, 16, 12
    x = r.standard_normal((T, d))
    wgu = r.standard_normal((1, 2 * f, d)) * 0.3
    wd = r.standard_normal((1, d, f)) * 0.3
    out = O.moe_forward(x, np.zeros((1, d)), wgu, wd, k=1)
    assert np.all(out["w"] == 1.0)
    xt = torch.from_numpy(x)
    gate = torch.from_numpy(wgu[0, :f])
    up = torch.from_numpy(wgu[0, f:])
    down = torch.from_numpy(wd[0])
    ref = (torch.nn.functional.silu(xt @ gate.T) * (xt @ up.T)) @ down.T
    assert np.abs(out["y"] - ref.numpy()).max() < 1e-13


def test_grouped_equals_dense_on_the_pages_toy():
    vals = {r[0]: r[1] for r in _read_table("toy_dispatch.txt")}
    T, d, f, E, k = (int(vals[n]) for n in ("T", "d", "f", "E", "k"))
    torch.manual_seed(0)
    gate_up = torch.empty(E, 2 * f, d).normal_(std=0.05)
    down = torch.empty(E, d, f).normal_(std=0.05)
    x = torch.randn(T, d)
    router = torch.randn(d, E) * 0.1
    s = (x.double() @ router.double()).numpy()
    p, _ = O.softmax_lse(s)
    idx, w = O.topk_no_renorm(p, k)
    args = (x.double().numpy(), idx, w, gate_up.double().numpy(), down.double().numpy())
    yg = O.experts_grouped(*args)
    yd = O.experts_dense(*args)
    # fp64: far below the page's fp32 figure
    assert np.abs(yg - yd).max() < 1e-12
    assert np.abs(yg - yd).max() < float(vals["fp32_max_difference"])
    assert np.abs(yg).max() > 1e-3


def test_grouped_equals_dense_random():
    L = _small_layer(8, T=40, E=16, k=4)
    out = O.moe_forward(**L)
    yd = O.experts_dense(L["x"], out["idx"], out["w"], L["w_gate_up"], L["w_down"])
    assert np.abs(out["y"] - yd).max() < 1e-12


def test_olmoe_parameter_counts():
    """Shapes: 16 layers x 64 experts x 3*d*f, and 8 active experts per token,
    reproduce the page's active/total counts given its non-expert remainder."""
    vals = {r[0]: int(r[1]) for r in _read_table("olmoe_param_counts.txt")}
    per_expert = 3 * S.OLMOE_D_MODEL * S.OLMOE_D_FF
    experts = S.OLMOE_N_LAYERS * S.OLMOE_N_EXPERTS * per_expert
    rest = vals["total"] - experts
    active = rest + S.OLMOE_N_LAYERS * S.OLMOE_TOP_K * per_expert
    assert active == vals["active"]
    assert experts == 6_442_450_944


# ------------------------------------------------------------------ gradients


def _fd_check(L, dy, alpha, beta, name, seed, eps=1e-6, renorm=False):
    g = O.moe_backward(dy=dy, alpha=alpha, beta=beta, renorm=renorm, **L)
    assert not g["fwd"]["near_tie"].any()
    r = _rng(seed)
    key = {"x": "dx", "w_router": "dw_router", "w_gate_up": "dw_gate_up",
           "w_down": "dw_down"}[name]
    for _ in range(3):
        v = r.standard_normal(L[name].shape)
        Lp = dict(L)
        Lp[name] = L[name] + eps * v
        Lm = dict(L)
        Lm[name] = L[name] - eps * v
        jp = O.moe_objective(dy=dy, alpha=alpha, beta=beta, renorm=renorm, **Lp)
        jm = O.moe_objective(dy=dy, alpha=alpha, beta=beta, renorm=renorm, **Lm)
        # the choice must not change inside the step, or the difference is meaningless
        ip = O.moe_forward(**Lp)["idx"]
        im = O.moe_forward(**Lm)["idx"]
        assert np.array_equal(ip, im)
        fd = (jp - jm) / (2 * eps)
        an = float(np.sum(g[key] * v))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


@pytest.mark.parametrize("name", ["x", "w_router", "w_gate_up", "w_down"])
def test_gradients_by_finite_differences(name):
    L = _small_layer(9, T=12, d=16, E=8, k=3, f=6, std=0.4)
    dy = _rng(10).standard_normal((12, 16))
    # alpha, beta far above OLMoE's so the loss terms are visible in the check
    _fd_check(L, dy, alpha=0.7, beta=0.3, name=name, seed=11)


@pytest.mark.parametrize("name", ["x", "w_router", "w_gate_up"])
def test_renormalised_router_gradients_by_finite_differences(name):
    L = _small_layer(26, T=12, d=16, E=8, k=3, f=6, std=0.4)
    dy = _rng(27).standard_normal((12, 16))
    _fd_check(L, dy, alpha=0.7, beta=0.3, name=name, seed=28, renorm=True)


def test_loss_gradients_alone_by_finite_differences():
    """dy = 0 isolates alpha*L_lb + beta*L_z, so a dropped loss term shows up."""
    L = _small_layer(12, T=10, d=12, E=8, k=2, f=4, std=0.5)
    dy = np.zeros((10, 12))
    _fd_check(L, dy, alpha=1.0, beta=1.0, name="w_router", seed=13)
    _fd_check(L, dy, alpha=1.0, beta=0.0, name="x", seed=14)
    _fd_check(L, dy, alpha=0.0, beta=1.0, name="x", seed=15)


def test_backward_expert_subset_matches_full():
    L = _small_layer(16, T=12, d=16, E=8, k=3, f=6)
    dy = _rng(17).standard_normal((12, 16))
    full = O.moe_backward(dy=dy, alpha=0.01, beta=0.001, **L)
    part = O.moe_backward(dy=dy, alpha=0.01, beta=0.001, experts=[2, 5], **L)
    assert np.array_equal(part["dw_down"][[2, 5]], full["dw_down"][[2, 5]])
    assert np.all(part["dw_down"][[0, 1, 3, 4, 6, 7]] == 0)
    assert np.array_equal(part["dx"], full["dx"])


def test_token_subset_input_grads_match_the_batch():
    """dx of a few tokens, given only the batch's counts and size, equals those
    rows of the batch backward (itself pinned by finite differences above); a
    dropped load-balance or z term, or the wrong T, would show here."""
    L = _small_layer(20, T=14, d=16, E=8, k=3, f=6, std=0.4)
    dy = _rng(21).standard_normal((14, 16))
    full = O.moe_backward(dy=dy, alpha=0.7, beta=0.3, **L)
    rows = [0, 5, 13]
    dx = O.token_input_grads(L["x"][rows], L["w_router"], L["w_gate_up"], L["w_down"], L["k"], dy[rows],
                             0.7, 0.3, full["fwd"]["counts"], 14)
    assert np.abs(dx - full["dx"][rows]).max() < 1e-12


def test_expert_weight_grad_slices_match_the_batch():
    L = _small_layer(22, T=20, d=16, E=8, k=3, f=6)
    dy = _rng(23).standard_normal((20, 16))
    full = O.moe_backward(dy=dy, alpha=0.01, beta=0.001, **L)
    fw = full["fwd"]
    for e in (0, 3):
        rows, cols = O.expert_weight_grad_slices(L["x"], fw["idx"], fw["w"], dy, L["w_gate_up"][e],
                                                 L["w_down"][e], e, gate_up_rows=[0, 4, 6, 11], down_cols=[1, 5])
        assert np.abs(rows - full["dw_gate_up"][e][[0, 4, 6, 11]]).max() < 1e-12
        assert np.abs(cols - full["dw_down"][e][:, [1, 5]]).max() < 1e-12


# ------------------------------------------------------------------ storage rounding


def test_store_identity_changes_nothing_and_zero_store_removes_the_experts():
    L = _small_layer(24, T=12, d=16, E=8, k=3, f=6, std=0.4)
    dy = _rng(25).standard_normal((12, 16))
    plain = O.moe_backward(dy=dy, alpha=0.3, beta=0.2, **L)
    ident = O.moe_backward(dy=dy, alpha=0.3, beta=0.2, store=lambda v: v, **L)
    for key in ("dx", "dw_router", "dw_gate_up", "dw_down"):
        assert np.array_equal(plain[key], ident[key]), key
    assert np.array_equal(plain["fwd"]["y"], ident["fwd"]["y"])
    # a store that zeroes every activation silences the experts: y = 0, and the
    # gradient is that of the two losses alone (the same as dy = 0)
    zero = O.moe_backward(dy=dy, alpha=0.3, beta=0.2, store=lambda v: 0.0 * v, **L)
    loss_only = O.moe_backward(dy=np.zeros_like(dy), alpha=0.3, beta=0.2, **L)
    assert np.all(zero["fwd"]["y"] == 0)
    assert np.allclose(zero["dx"], loss_only["dx"], atol=1e-15, rtol=0)
    assert np.allclose(zero["dw_router"], loss_only["dw_router"], atol=1e-15, rtol=0)
    assert np.all(zero["dw_gate_up"] == 0) and np.all(zero["dw_down"] == 0)


def test_store_rounding_on_a_two_expert_scalar_layer():
    """d = f = 1, two experts, k = 1, rounding to multiples of 1/8; only the
    contraction operands h, do and [da; db] are rounded. By hand: logits
    h = [0.3, -0.2], so expert 0 wins with p0 = 1 / (1 + e^-0.5) = 0.6225; the
    pre-activations a = 0.7, b = 1.3 stay as they are; the hidden
    silu(0.7) * 1.3 = 0.4677 * 1.3 = 0.6081 is rounded to 0.625 before the down
    projection; the output o = 0.9 * 0.625 = 0.5625 is NOT rounded (it would
    become 0.5), so y = 0.5625 p0. With dy = 1 and no loss terms dw = <dy, o> =
    0.5625, dh = [0.5625 p0 p1, -0.5625 p0 p1] and dW_r = dh x with x = 1. do =
    p0 is rounded to 0.625, so dW_down = 0.625 * 0.625 and dg = 0.625 * 0.9 =
    0.5625; da = dg b silu'(a) = 0.6021 rounds to 0.625 and db = dg silu(a) =
    0.2631 rounds to 0.25, which are dW_gate_up (x = 1)."""
    R = lambda v: np.round(np.asarray(v) * 8.0) / 8.0
    x = np.array([[1.0]])
    w_router = np.array([[0.3], [-0.2]])
    w_gate_up = np.array([[[0.7], [1.3]], [[0.5], [0.5]]])
    w_down = np.array([[[0.9]], [[0.5]]])
    g = O.moe_backward(x, w_router, w_gate_up, w_down, 1, np.array([[1.0]]), 0.0, 0.0, store=R)
    p0 = 1.0 / (1.0 + math.exp(-0.5))
    p1 = 1.0 - p0
    assert g["fwd"]["idx"][0, 0] == 0
    assert abs(g["fwd"]["y"][0, 0] - p0 * 0.5625) < 1e-15
    assert abs(g["dw"][0, 0] - 0.5625) < 1e-15
    assert np.allclose(g["dw_router"][:, 0], [0.5625 * p0 * p1, -0.5625 * p0 * p1], atol=1e-15, rtol=0)
    assert abs(g["dw_down"][0, 0, 0] - 0.625 * 0.625) < 1e-15
    assert abs(g["dw_gate_up"][0, 0, 0] - 0.625) < 1e-15 and abs(g["dw_gate_up"][0, 1, 0] - 0.25) < 1e-15
    assert np.all(g["dw_gate_up"][1] == 0) and np.all(g["dw_down"][1] == 0)
    # the unrounded values the rounding acted on, by hand
    s = 1.0 / (1.0 + math.exp(-0.7))
    assert abs(0.7 * s * 1.3 - 0.6081) < 1e-4
    assert abs(0.5625 * 1.3 * s * (1.0 + 0.7 * (1.0 - s)) - 0.6021) < 1e-4
    assert abs(0.5625 * 0.7 * s - 0.2631) < 1e-4


def test_operand_rounding_alone_moves_olmoe_router_gradient_past_the_max_abs_bar():
    """Why weight gradients are compared with the operand-rounded oracle: on a
    1024-token layer of OLMoE's shapes, rounding only the contraction operands
    to bf16 (what any bf16-input implementation must do) moves dW_router by
    more than 2e-2 max-abs from the unrounded fp64 gradient, while its relative
    L2 change stays near 2e-3 and dx stays far inside both bars."""
    sh = S.LayerShape(T=1024)
    inp = S.layer_inputs(sh, seed=4, with_grad=True)
    f = lambda t: t.to(torch.float64).numpy()
    args = (f(inp.x), f(inp.w_router), f(inp.w_gate_up), f(inp.w_down), sh.top_k, f(inp.dy), 0.01, 0.001)
    bf16 = lambda a: torch.from_numpy(np.ascontiguousarray(a)).float().bfloat16().double().numpy()
    plain = O.moe_backward(*args, experts=[])
    rounded = O.moe_backward(*args, experts=[], store=bf16)
    d = rounded["dw_router"] - plain["dw_router"]
    assert np.abs(d).max() > 2e-2
    assert np.linalg.norm(d) / np.linalg.norm(plain["dw_router"]) < 5e-3
    assert np.abs(rounded["dx"] - plain["dx"]).max() < 5e-3


# ------------------------------------------------------------------ stack


def test_rms_norm_closed_form():
    c = 3.0
    x = np.full((2, 10), c)
    y = O.rms_norm(x, eps=1e-5)
    assert np.allclose(y, c / math.sqrt(c * c + 1e-5), atol=1e-15)
    w = np.arange(10.0)
    assert np.allclose(O.rms_norm(x, w), y * w, atol=1e-14)


def test_stack_with_zero_experts_is_identity_and_one_layer_is_one_block():
    L = _small_layer(18, T=8, d=16, E=8, k=2, f=4)
    x0 = _rng(19).standard_normal((8, 16)) * 2
    zero = dict(w_router=L["w_router"], w_gate_up=np.zeros_like(L["w_gate_up"]),
                w_down=L["w_down"])
    r, _ = O.stack_forward(x0, [zero, zero], k=2)
    assert np.array_equal(r, x0)
    one = dict(w_router=L["w_router"], w_gate_up=L["w_gate_up"], w_down=L["w_down"])
    r, _ = O.stack_forward(x0, [one], k=2)
    ref = x0 + O.moe_forward(O.rms_norm(x0), L["w_router"], L["w_gate_up"], L["w_down"], 2)["y"]
    assert np.allclose(r, ref, atol=1e-14, rtol=0)


def test_zipf_offset_matches_its_calibration():
    """The skewed stack's router offset gives the 8 most favoured experts half of
    the assignments on layer 0's input (calibrated by tests/golden/calibrate_zipf.py)."""
    vals = {r[0]: float(r[1]) for r in _read_table("zipf_lambda.txt")}
    assert S.ZIPF_LAMBDA == vals["lambda"]
    import importlib.util
    spec = importlib.util.spec_from_file_location("calibrate_zipf", os.path.join(GOLDEN, "calibrate_zipf.py"))
    cal = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(cal)
    x, wr = cal.layer0_inputs()
    assert abs(cal.top8_share(S.ZIPF_LAMBDA, x, wr) - 0.5) <= 0.01


# ------------------------------------------------------------------ expert-choice pins


def test_expert_choice_hand_case():
    """Four tokens, two experts, capacity 2, worked by hand. Expert 0's column
    (0.5, 0.2, 0.9, 0.5): token 2, then the tie at 0.5 goes to token 0. Expert 1's
    column (0.5, 0.8, 0.1, 0.5): token 1, then token 0 over token 3."""
    p = np.array([[0.5, 0.5], [0.2, 0.8], [0.9, 0.1], [0.5, 0.5]])
    sel, gates = O.expert_choice(p, 2)
    assert sel.tolist() == [[0, 2], [0, 1]]
    assert gates.tolist() == [[0.5, 0.9], [0.5, 0.8]]


def test_expert_choice_selection_by_brute_force():
    """Every chosen token beats every unchosen one in the expert's column (or ties
    it with a lower index), checked pair by pair; the list is in token order and
    holds exactly C distinct tokens. Equal values are planted so ties occur."""
    r = _rng(21)
    for T, E, C in [(9, 3, 4), (13, 5, 1), (16, 4, 16), (11, 2, 7)]:
        p = r.integers(0, 4, size=(T, E)) / 4.0  # many exact ties
        sel, gates = O.expert_choice(p, C)
        for e in range(E):
            chosen = [int(t) for t in sel[e]]
            assert len(chosen) == C == len(set(chosen))
            assert chosen == sorted(chosen)
            for t in chosen:
                assert gates[e][chosen.index(t)] == p[t, e]
                for u in range(T):
                    if u in chosen:
                        continue
                    assert p[t, e] > p[u, e] or (p[t, e] == p[u, e] and t < u)


def test_expert_choice_capacity():
    """ceil(T k / E), capped at T: OLMoE's shapes give T/8 tokens per expert."""
    assert O.ec_capacity(4096, 8, 64) == 512
    assert O.ec_capacity(16384, 8, 64) == 2048
    assert O.ec_capacity(1, 8, 64) == 1
    assert O.ec_capacity(100, 3, 7) == 43  # 300 / 7 = 42.86
    assert O.ec_capacity(5, 8, 4) == 5  # 10 would exceed T


def test_expert_choice_full_capacity_is_the_dense_softmax_layer():
    """With C = T every expert takes every token, so y = sum_e p[t, e] Expert_e(x_t):
    the page's every-expert-on-every-token layer with the full softmax as gate."""
    L = _small_layer(22, T=10, E=6, k=6)
    out = O.moe_forward_expert_choice(**L)
    assert out["capacity"] == 10
    assert np.all(out["fanout"] == 6)
    T, E = out["p"].shape
    idx = np.tile(np.arange(E), (T, 1))
    yd = O.experts_dense(L["x"], idx, out["p"], L["w_gate_up"], L["w_down"])
    assert np.abs(out["y"] - yd).max() < 1e-12


def test_expert_choice_single_expert_is_a_plain_swiglu_mlp():
    """E = 1: p = 1 and the one expert takes all T tokens: y = SwiGLU(x)."""
    r = _rng(23)
    T, d, f = 12, 16, 8
    x = r.standard_normal((T, d))
    wgu = r.standard_normal((1, 2 * f, d)) * 0.3
    wd = r.standard_normal((1, d, f)) * 0.3
    out = O.moe_forward_expert_choice(x, np.zeros((1, d)), wgu, wd, k=1)
    assert out["sel"].tolist() == [list(range(T))]
    xt = torch.from_numpy(x)
    ref = (torch.nn.functional.silu(xt @ torch.from_numpy(wgu[0, :f]).T) * (xt @ torch.from_numpy(wgu[0, f:]).T)) @ \
        torch.from_numpy(wd[0]).T
    assert np.abs(out["y"] - ref.numpy()).max() < 1e-13


def test_expert_choice_dropped_tokens_get_zero_and_z_loss_is_unchanged():
    """With C = 1 most tokens are chosen by no expert; their rows are zero. The
    chosen ones equal the dense layer restricted to the (token, expert) pairs
    picked. L_z is the token-choice z-loss of the same logits."""
    L = _small_layer(24, T=30, E=4, k=1)
    out = O.moe_forward_expert_choice(**L, capacity=1)
    gate = np.zeros_like(out["p"])
    for e in range(4):
        t = int(out["sel"][e, 0])
        assert t == int(np.argmax(out["p"][:, e]))  # the column's largest (no ties here)
        gate[t, e] = out["p"][t, e]
    idx = np.tile(np.arange(4), (30, 1))
    yd = O.experts_dense(L["x"], idx, gate, L["w_gate_up"], L["w_down"])
    assert np.abs(out["y"] - yd).max() < 1e-12
    assert np.all(out["y"][out["fanout"] == 0] == 0.0)
    assert out["L_z"] == O.moe_forward(**L)["L_z"]
    assert out["L_lb"] == 0.0


@pytest.mark.parametrize("name", ["x", "w_router", "w_gate_up", "w_down"])
def test_expert_choice_gradients_by_finite_differences(name):
    """Central differences of <dy, y> + beta L_z under expert choice, with the
    choice held fixed inside the step (checked)."""
    L = _small_layer(31, T=12, d=16, E=6, k=2, f=6, std=0.4)
    dy = _rng(32).standard_normal((12, 16))
    beta, eps = 0.3, 1e-6
    g = O.moe_backward_expert_choice(dy=dy, beta=beta, **L)
    key = {"x": "dx", "w_router": "dw_router", "w_gate_up": "dw_gate_up", "w_down": "dw_down"}[name]
    r = _rng(33)
    for _ in range(3):
        v = r.standard_normal(L[name].shape)
        Lp = dict(L)
        Lp[name] = L[name] + eps * v
        Lm = dict(L)
        Lm[name] = L[name] - eps * v
        assert np.array_equal(O.moe_forward_expert_choice(**Lp)["sel"], O.moe_forward_expert_choice(**Lm)["sel"])
        fd = (O.moe_objective_expert_choice(dy=dy, beta=beta, **Lp)
              - O.moe_objective_expert_choice(dy=dy, beta=beta, **Lm)) / (2 * eps)
        an = float(np.sum(g[key] * v))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_expert_choice_backward_at_full_capacity_is_the_dense_layers():
    """With C = T every token meets every expert with weight p[t, e], which is
    token choice with k = E (all experts chosen, weights p): with no loss terms
    the two objectives are the same function, so every gradient agrees, and
    dp is <dy_t, Expert_e(x_t)> for every pair."""
    L = _small_layer(34, T=7, d=12, E=4, k=4, f=5, std=0.4)
    dy = _rng(35).standard_normal((7, 12))
    ec = O.moe_backward_expert_choice(dy=dy, beta=0.0, **L)
    assert ec["fwd"]["capacity"] == 7
    tc = O.moe_backward(dy=dy, alpha=0.0, beta=0.0, **L)
    for name in ("dx", "dw_router", "dw_gate_up", "dw_down"):
        assert np.abs(ec[name] - tc[name]).max() < 1e-12, name
    for e in range(4):
        o = O.swiglu_expert(L["x"], L["w_gate_up"][e], L["w_down"][e])
        assert np.abs(ec["dp"][:, e] - np.sum(dy * o, axis=1)).max() < 1e-12
