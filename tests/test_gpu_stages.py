"""Each stage of the CUDA path against the oracle on seeded stage inputs.

The stage inputs (expert choices, group sizes, permuted rows) are drawn from
seeded generators here, never taken from another CUDA stage, so every stage is
checked on its own, including the awkward group sizes: empty experts, a single
row, exactly one tile, one row past a tile, many tiles.
"""

import numpy as np
import pytest
import torch

import sparse_moe_transformer_route_b200 as M
from oracle import moe_oracle as O
from tests._parity import assert_close, bf16_round, f64, padded_group_starts, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def seeded_choices(T, E, k, seed, mode="uniform"):
    r = np.random.default_rng(seed)
    if mode == "uniform":
        return np.stack([r.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    if mode == "same":  # every token picks the same k experts, in a shuffled slot order
        base = r.choice(E, k, replace=False)
        return np.stack([r.permutation(base) for _ in range(T)]).astype(np.int32)
    if mode == "skewed":  # low expert ids much more likely
        p = 1.0 / np.arange(1, E + 1) ** 1.2
        p /= p.sum()
        return np.stack([r.choice(E, k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    raise ValueError(mode)


DISPATCH_CASES = [
    (1, 64, 8, "uniform"),
    (300, 16, 4, "uniform"),
    (1000, 64, 8, "uniform"),
    (700, 8, 8, "uniform"),      # k = E: every token takes every expert
    (513, 64, 8, "same"),        # eight experts get everything, 56 get nothing
    (5000, 64, 8, "skewed"),     # many dispatch chunks, skewed groups
]


@pytest.mark.parametrize("T,E,k,mode", DISPATCH_CASES)
def test_dispatch_matches_oracle(T, E, k, mode):
    d = 256
    idx = seeded_choices(T, E, k, seed=T + E, mode=mode)
    cfg = M.config(T, d, E, k, 128)
    P = M.moe_padded_rows(cfg)
    g = torch.Generator().manual_seed(7)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16).cuda()
    idx_t = torch.from_numpy(idx).cuda()
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    group_start = torch.empty_like(offsets)
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv_perm = torch.empty_like(perm)
    x_perm = torch.full((P, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = M.workspace(cfg)
    M.moe_dispatch(cfg, idx_t, x, offsets, perm, inv_perm, group_start, x_perm, ws)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 0

    ref_perm, counts, ref_off = O.dispatch_order(idx, E)
    assert np.array_equal(perm.cpu().numpy(), ref_perm)
    assert np.array_equal(offsets.cpu().numpy(), ref_off)
    gs = padded_group_starts(counts)
    assert np.array_equal(group_start.cpu().numpy(), gs)
    # inverse permutation: pair at sorted position s lives at padded row gs[e] + (s - offsets[e])
    flat = idx.reshape(-1)
    s = np.arange(T * k)
    e_of = flat[ref_perm]
    rows = gs[e_of] + (s - ref_off[e_of])
    want_inv = np.empty(T * k, dtype=np.int64)
    want_inv[ref_perm] = rows
    inv = inv_perm.cpu().numpy()
    assert np.array_equal(inv, want_inv)
    xp = x_perm.cpu()
    xc = x.cpu()
    assert torch.equal(xp[torch.from_numpy(want_inv)], xc[torch.from_numpy(np.arange(T * k) // k)])
    # padding rows are zero
    valid = np.zeros(P, dtype=bool)
    valid[want_inv] = True
    pad = np.zeros(P, dtype=bool)
    pad[: gs[-1]] = True
    pad &= ~valid
    assert torch.all(xp[torch.from_numpy(pad)] == 0)


def test_dispatch_reports_bad_expert_index():
    T, E, k, d = 64, 16, 4, 128
    idx = seeded_choices(T, E, k, seed=3)
    idx[5, 2] = E + 3
    idx[9, 0] = -1
    cfg = M.config(T, d, E, k, 128)
    P = M.moe_padded_rows(cfg)
    x = torch.ones(T, d, dtype=torch.bfloat16, device="cuda")
    out = [torch.empty(E + 1, dtype=torch.int32, device="cuda") for _ in range(2)]
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty_like(perm)
    x_perm = torch.empty(P, d, dtype=torch.bfloat16, device="cuda")
    ws = M.workspace(cfg)
    M.moe_dispatch(cfg, torch.from_numpy(idx).cuda(), x, out[0], perm, inv, out[1], x_perm, ws)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 0x201
    assert M.moe_get_device_status(ws) == 0  # reading clears it
    inv = inv.cpu().numpy()
    assert inv[5 * k + 2] == -1 and inv[9 * k + 0] == -1


def _bar(ref):
    return 2e-2 * max(1.0, float(np.abs(ref).max()))


GEMM_COUNTS = [
    [0, 1, 127, 128, 129, 300, 0, 5],
    [513, 0, 0, 2, 255, 256, 1, 64],
    [700, 129, 384, 0, 255, 1, 513, 128],
    # >= 384 rows per expert on average: 256-row tiles on CTA pairs, some whose
    # second half lies in the next expert's group (and must not be written)
    [700, 129, 385, 0, 900, 1, 513, 640],
]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("counts", GEMM_COUNTS)
@pytest.mark.parametrize("d,f", [(256, 256), (384, 128)])
def test_expert_gemms_match_oracle(counts, dtype, d, f):
    E = len(counts)
    k = 1
    T = int(sum(counts))
    cfg = M.config(T, d, E, k, f, dtype)
    P = M.moe_padded_rows(cfg)
    gs = padded_group_starts(counts)
    assert gs[-1] <= P
    off = np.zeros(E + 1, dtype=np.int64)
    off[1:] = np.cumsum(counts)
    g = torch.Generator().manual_seed(sum(counts) + d)
    x_perm = torch.randn(P, d, generator=g).to(dtype)  # padding rows hold junk on purpose
    w_gate_up = (torch.randn(E, 2 * f, d, generator=g) * 0.05).to(dtype)
    w_down = (torch.randn(E, d, f, generator=g) * 0.05).to(dtype)
    dev = lambda t: t.cuda()
    h = torch.full((P, f), float("nan"), dtype=dtype, device="cuda")
    pre = torch.full((P, 2 * f), float("nan"), dtype=torch.float32, device="cuda")  # kept unrounded
    o = torch.full((P, d), float("nan"), dtype=dtype, device="cuda")
    gs_t = torch.from_numpy(gs.astype(np.int32)).cuda()
    off_t = torch.from_numpy(off.astype(np.int32)).cuda()
    ws = M.workspace(cfg)
    M.moe_expert_gate_up(cfg, dev(x_perm), gs_t, off_t, dev(w_gate_up), h, pre, ws)
    M.moe_expert_down(cfg, h, gs_t, off_t, dev(w_down), o, ws)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 0
    hc, pc, oc = h.cpu(), pre.cpu(), o.cpu()
    xp = f64(x_perm)
    for e in range(E):
        r0, c = int(gs[e]), counts[e]
        rows = slice(r0, r0 + c)
        pad = slice(r0 + c, int(gs[e + 1]))
        if c:
            # these stage inputs are not unit-scale, so the absolute bar scales with
            # the output's magnitude (bf16 keeps 8 significant bits)
            a, b = O.gate_up_preact(xp[rows], f64(w_gate_up[e]))
            assert_close(pc[rows, :f], a, f"preact gate e={e}", max_abs=_bar(a))
            assert_close(pc[rows, f:], b, f"preact up e={e}", max_abs=_bar(b))
            href = O.swiglu_hidden(xp[rows], f64(w_gate_up[e]))
            assert_close(hc[rows], href, f"h e={e}", max_abs=_bar(href))
            oref = O.expert_down(href, f64(w_down[e]))
            assert_close(oc[rows], oref, f"o e={e}", max_abs=_bar(oref))
        assert torch.all(hc[pad] == 0) and torch.all(oc[pad] == 0) and torch.all(pc[pad] == 0)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_combine_matches_oracle(dtype):
    T, E, k, d = 333, 16, 4, 256
    idx = seeded_choices(T, E, k, seed=11)
    perm, counts, off = O.dispatch_order(idx, E)
    gs = padded_group_starts(counts)
    cfg = M.config(T, d, E, k, 128, dtype)
    P = M.moe_padded_rows(cfg)
    flat = idx.reshape(-1)
    s = np.arange(T * k)
    inv = np.empty(T * k, dtype=np.int64)
    inv[perm] = gs[flat[perm]] + (s - off[flat[perm]])
    g = torch.Generator().manual_seed(5)
    o_perm = torch.randn(P, d, generator=g).to(dtype)
    w = torch.rand(T, k, generator=g, dtype=torch.float32)
    y = torch.empty(T, d, dtype=dtype, device="cuda")
    M.moe_combine(cfg, o_perm.cuda(), torch.from_numpy(inv.astype(np.int32)).cuda(), w.cuda(), y)
    torch.cuda.synchronize()
    ref = np.einsum("tk,tkd->td", f64(w), f64(o_perm)[inv.reshape(T, k)])
    assert_close(y, ref, "combine", max_abs=2e-2, rel_l2=4e-3)
    # residual form adds into fp32
    resid = torch.randn(T, d, generator=g)
    r = resid.clone().cuda()
    M.moe_combine_residual(cfg, o_perm.cuda(), torch.from_numpy(inv.astype(np.int32)).cuda(), w.cuda(), r)
    torch.cuda.synchronize()
    assert_close(r, f64(resid) + ref, "combine residual", max_abs=1e-5, rel_l2=1e-6)


def test_rmsnorm_matches_oracle():
    T, d = 77, 384
    cfg = M.config(T, d, 8, 2, 128)
    g = torch.Generator().manual_seed(9)
    r = torch.randn(T, d, generator=g) * 3
    w = torch.rand(d, generator=g) + 0.5
    out = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    M.moe_rmsnorm(cfg, r.cuda(), w.cuda(), 1e-5, out)
    torch.cuda.synchronize()
    # the kernel forms the value in fp64 and rounds it (to fp32, then bf16) as the
    # oracle's value is rounded here, so the two agree bit for bit (eps is the
    # fp32 value the call passes)
    ref = bf16_round(O.rms_norm(f64(r), f64(w), eps=float(np.float32(1e-5))))
    assert np.array_equal(f64(out), ref)
