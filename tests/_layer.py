"""Whole-layer helpers shared by the GPU parity tests: one forward through the C
ABI, and its check against the oracle."""

import numpy as np
import torch

import sparse_moe_transformer_route_b200 as M
from oracle import moe_oracle as O
from tests._parity import LazyF64, assert_close, assert_loss_close, f64, index_parity


def run_forward(inp, train=False, bias=None, renorm=False):
    x, wr, wgu, wd = (t.cuda() for t in (inp.x, inp.w_router, inp.w_gate_up, inp.w_down))
    sh = inp.shape
    cfg = M.config(sh.T, sh.d_model, sh.n_experts, sh.top_k, sh.d_ff, x.dtype, renorm=renorm)
    ws = M.workspace(cfg, train)
    y = torch.empty_like(x)
    losses = torch.empty(2, device="cuda")
    idx = torch.empty(sh.T, sh.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(sh.T, sh.top_k, device="cuda")
    b = bias.cuda() if bias is not None else None
    M.moe_forward(cfg, x, wr, b, wgu, wd, y, losses, idx, w, train, ws)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 0
    return dict(cfg=cfg, ws=ws, y=y, losses=losses, idx=idx, w=w, dev=(x, wr, wgu, wd, b))


def check_forward(inp, out, bias=None, sample=None, renorm=False):
    """Routing for every token; outputs on `sample` tokens (all when None)."""
    x = f64(inp.x)
    wr = f64(inp.w_router)
    k = inp.shape.top_k
    E = inp.shape.n_experts
    b = f64(bias) if bias is not None else None
    h = O.router_logits(x, wr, b)
    p, lse = O.softmax_lse(h)
    ref_idx, ref_w = O.topk_renorm(p, k) if renorm else O.topk_no_renorm(p, k)
    near = O.near_tie_tokens(p, k)
    gidx = out["idx"].cpu().numpy()
    bad, n_near, diff = index_parity(gidx, ref_idx, near)
    assert bad.size == 0, f"{bad.size} non-near-tie tokens routed differently, e.g. {bad[:5]}"
    same = ~diff
    assert_close(out["w"].cpu()[torch.from_numpy(same)], ref_w[same], "router weights", max_abs=1e-5, rel_l2=1e-5)
    L_lb, _ = O.load_balance_loss(ref_idx, p, E)
    assert_loss_close(out["losses"][0].item(), L_lb, "L_lb")
    assert_loss_close(out["losses"][1].item(), O.router_z_loss(lse), "L_z")
    toks = np.arange(inp.shape.T) if sample is None else np.asarray(sample)
    toks = toks[same[toks]]
    wgu = LazyF64(inp.w_gate_up)
    wd = LazyF64(inp.w_down)
    y_ref = O.experts_grouped(x[toks], ref_idx[toks], ref_w[toks], wgu, wd)
    assert_close(out["y"].cpu()[torch.from_numpy(toks)], y_ref, "y")
    return n_near
