"""fp64 CPU oracle for the OLMoE mixture-of-experts FFN layer.

TEST INFRASTRUCTURE. Only the tests, the smoke check and the CPU-baseline leg of
the benchmark may import this module. The product path (the CUDA library and its
Python binding) never calls it, and this module imports nothing from the product.

Everything here is plain numpy in float64, written to be read against the pages
it cites, not to be fast. Inputs are taken as already-rounded values (bf16 or
fp32 tensors converted to float64), so the oracle and the GPU see identical
numbers. Pages cited:

  [OLMoE-Guide]  "OLMoE Guide: 64-Expert Fine-Grained Open MoE Architecture",
                 section "Router Mechanics & Loss Formulations" (routing formula,
                 auxiliary load-balancing loss, router z-loss) and "Hands-On
                 Implementation" (the PyTorch layer).
  [MoE-scratch]  "Mixture-of-experts LLMs from scratch with OLMoE",
                 section 2 "The router and the experts" (softmax_topk, Experts,
                 dispatch, dense_run) and section 3 "OLMoE in PyTorch" (the config
                 dump with norm_topk_prob False, RMSNorm, the fp32 residual).
  [OLMoE-paper]  "OLMoE: Open Mixture-of-Experts Language Models" (summary page),
                 "Pretraining architecture" (dropless token choice, loss weights
                 alpha and beta), sections 4.1.6 and 4.1.7.

Readings taken where the pages are silent or disagree (each is also listed in
the design notes):
  * Routing: softmax over all E experts, then the k largest probabilities are
    both the choice and the weights, with no renormalisation ([MoE-scratch] §2
    and §3, norm_topk_prob False). [OLMoE-Guide]'s top-k-then-softmax formula
    contradicts this and is not used.
  * Ties in the top-k: the lower expert index wins; slots are ordered by
    descending probability.
  * L_lb is reported unscaled, E * sum_i f_i * P_i with f_i = count_i / (T*k);
    L_z is reported unscaled, mean_t lse_t^2. alpha and beta weight them only in
    the backward objective  <dy, y> + alpha * L_lb + beta * L_z.
  * No gradient flows through the expert choice or through f ([OLMoE-Guide]
    computes f with bincount, a count).
  * Expert choice (the alternative the paper summary compares in section
    4.1.4, "Expert Choice vs. Token Choice": experts pick tokens instead of
    tokens picking experts). The pages give no formula; the plain reading
    taken: the same router probabilities p = softmax(h) over experts; each
    expert e takes the C tokens with the largest p[t, e] (ties to the lower
    token index); C = ceil(T*k/E) capped at T, so the expert work equals token
    choice's; the weight of (t, e) is p[t, e]; a token sums over the experts
    that took it in ascending expert order and gets zero when none did; the
    z-loss is unchanged and there is no load-balancing loss (every expert
    holds exactly C tokens).
  * Operand precision (optional `store` argument of the expert functions,
    moe_forward and moe_backward). The agreement bar is stated for "bf16
    inputs with fp32 accumulation": every contraction of the layer takes bf16
    operands. By default nothing is rounded. Given a rounding function, the
    operands of the contractions that are not layer inputs already are passed
    through it: the SwiGLU output h (the down projection's input and dW_down's
    right factor), do = w dy (the input of dg = do W_down and dW_down's left
    factor) and [da; db] (the input of the gate/up data gradient and dW_gate_up's
    left factor). Values no contraction reads (the expert output o, the
    pre-activations a and b that the SwiGLU derivative uses) are never
    rounded, and all arithmetic stays fp64. A gradient that sums many
    products of rounded operands (dW_router sums T terms <dy_t, o_tj> x_t with
    o computed from a bf16 h) can then be compared at the bar it should meet.

Parity pins for every function live in tests/test_oracle_pins.py.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "router_logits",
    "softmax_lse",
    "topk_no_renorm",
    "topk_renorm",
    "near_tie_tokens",
    "load_balance_loss",
    "router_z_loss",
    "dispatch_order",
    "silu",
    "gate_up_preact",
    "swiglu_hidden",
    "expert_down",
    "swiglu_expert",
    "experts_grouped",
    "experts_dense",
    "moe_forward",
    "moe_objective",
    "moe_backward",
    "token_input_grads",
    "expert_weight_grad_slices",
    "rms_norm",
    "stack_forward",
    "ec_capacity",
    "expert_choice",
    "experts_expert_choice",
    "moe_forward_expert_choice",
    "moe_objective_expert_choice",
    "moe_backward_expert_choice",
]


def _f64(a):
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------- router


def router_logits(x, w_router, router_bias=None):
    """Router scores h_t = W_r x_t (+ b), for every token and every expert.

    [OLMoE-Guide] "Top-8 Softmax Routing Formulation": h(x) = W_g x with W_g of
    shape (E, d). [MoE-scratch] §2: the router is one matrix with a row per
    expert, s = W_r x; §3 MoE.forward: scores are taken in 32-bit floats and an
    optional per-expert offset (the keep-mask) is applied before the softmax.
    `router_bias` is that per-expert additive offset, shape (E,), or None.
    Returns h of shape (T, E), float64.
    """
    h = _f64(x) @ _f64(w_router).T
    if router_bias is not None:
        h = h + _f64(router_bias)[None, :]
    return h


def softmax_lse(h):
    """Softmax over all experts and its log-normaliser.

    p_{t,i} = exp(h_{t,i}) / sum_j exp(h_{t,j}),  lse_t = log sum_j exp(h_{t,j}).
    [MoE-scratch] §2 softmax_topk takes the softmax over all experts first;
    [OLMoE-Guide] "Router Z-Loss Regularization" defines the log-sum-exp.
    The maximum is subtracted first so exp never overflows.
    """
    h = _f64(h)
    m = h.max(axis=1, keepdims=True)
    e = np.exp(h - m)
    s = e.sum(axis=1, keepdims=True)
    return e / s, (m + np.log(s))[:, 0]


def topk_no_renorm(p, k):
    """The k largest probabilities per token, without renormalisation.

    [MoE-scratch] §2 softmax_topk (OLMoE's router) and §3 (norm_topk_prob False):
    the chosen experts are the k largest softmax probabilities and their weights
    are those probabilities unchanged, so they sum to less than one.
    Ties are broken towards the lower expert index (a stable sort of -p).
    Returns (idx [T,k] int64, w [T,k] float64), slots in descending p.
    """
    p = _f64(p)
    order = np.argsort(-p, axis=1, kind="stable")[:, :k]
    return order.astype(np.int64), np.take_along_axis(p, order, axis=1)


def topk_renorm(p, k):
    """The same choice as topk_no_renorm, with the k weights renormalised to sum
    to one: w_tj = p_tj / sum_j' p_tj'.

    [OLMoE-Guide] "Top-8 Softmax Routing Formulation" writes the router as a
    softmax over the k largest logits; dividing the k chosen probabilities by
    their sum is the same thing ([MoE-scratch] §2, the router-variants table:
    "softmax, top-k, renormalise" and "top-k, softmax" agree). OLMoE itself does
    not renormalise; this is the variant behind the library's router mode 1.
    """
    idx, w = topk_no_renorm(p, k)
    return idx, w / w.sum(axis=1, keepdims=True)


def near_tie_tokens(p, k, rel=1e-6):
    """Tokens whose selection or slot order is decided by a near-tie.

    A token is flagged when two neighbours among its k+1 largest probabilities
    differ by less than `rel` relative to the larger one. For such tokens a
    different rounding order may legitimately pick or order experts
    differently, so parity on indices is counted separately for them.
    """
    p = _f64(p)
    s = -np.sort(-p, axis=1)[:, : min(k + 1, p.shape[1])]
    gaps = s[:, :-1] - s[:, 1:]
    return np.any(gaps < rel * s[:, :-1], axis=1)


def load_balance_loss(idx, p, n_experts):
    """Switch-style load-balancing loss, unscaled: E * sum_i f_i * P_i.

    [OLMoE-Guide] "Auxiliary Load Balancing Loss": f_i is the fraction of the
    T*k token-slot assignments that went to expert i (a bincount, no gradient),
    P_i is the mean over tokens of the full softmax probability of expert i.
    Returns (L_lb, counts [E] int64).
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    counts = np.bincount(idx.reshape(-1), minlength=n_experts)
    f = counts / float(T * k)
    P = _f64(p).mean(axis=0)
    return float(n_experts * np.sum(f * P)), counts


def router_z_loss(lse):
    """Router z-loss, unscaled: (1/T) * sum_t lse_t^2 ([OLMoE-Guide] "Router Z-Loss")."""
    lse = _f64(lse)
    return float(np.mean(lse * lse))


# --------------------------------------------------------------------------- dispatch


def dispatch_order(idx, n_experts):
    """Grouping of (token, slot) pairs by expert, as in [MoE-scratch] §2 `dispatch`.

    The pairs are the flattened [T, k] choice matrix (pair id = t*k + j). They are
    sorted stably by expert, so inside one expert the pairs keep token order.
    Returns
      perm    [T*k]  pair id at each sorted position,
      counts  [E]    pairs per expert (bincount),
      offsets [E+1]  exclusive prefix sum of counts (start of each expert's group).
    """
    pairs = np.asarray(idx).reshape(-1)
    perm = np.argsort(pairs, kind="stable").astype(np.int64)
    counts = np.bincount(pairs, minlength=n_experts).astype(np.int64)
    offsets = np.zeros(n_experts + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    return perm, counts, offsets


# --------------------------------------------------------------------------- experts


def silu(z):
    """SiLU / Swish: z * sigmoid(z) = z / (1 + exp(-z))."""
    z = _f64(z)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def gate_up_preact(x_rows, w_gate_up_e):
    """The two pre-activations (x W_gate^T, x W_up^T) of one expert, each [n, f]."""
    w_gate_up_e = _f64(w_gate_up_e)
    f = w_gate_up_e.shape[0] // 2
    x_rows = _f64(x_rows)
    return x_rows @ w_gate_up_e[:f].T, x_rows @ w_gate_up_e[f:].T


def swiglu_hidden(x_rows, w_gate_up_e):
    """The expert's hidden activation Swish(x W_gate) * (x W_up), rows [n, f].

    [MoE-scratch] §2 `Experts.run`: the (2f, d) gate_up matrix holds the gate
    rows first, then the up rows; the product is split in two halves.
    """
    w_gate_up_e = _f64(w_gate_up_e)
    f = w_gate_up_e.shape[0] // 2
    x_rows = _f64(x_rows)
    a = x_rows @ w_gate_up_e[:f].T
    b = x_rows @ w_gate_up_e[f:].T
    return silu(a) * b


def expert_down(g_rows, w_down_e):
    """The expert's down projection g W_down^T with W_down of shape (d, f)."""
    return _f64(g_rows) @ _f64(w_down_e).T


def _store(store):
    return (lambda v: v) if store is None else (lambda v: _f64(store(v)))


def swiglu_expert(x_rows, w_gate_up_e, w_down_e, store=None):
    """One SwiGLU expert on a block of rows.

    [OLMoE-Guide] "Top-8 Softmax Routing Formulation": Expert_i(x) =
    (Swish(x W_gate) * (x W_up)) W_down. [MoE-scratch] §2 `Experts` stores the
    gate rows first, then the up rows, in one (2f, d) matrix, and the down
    projection as (d, f). `store` (see the module notes) rounds h, the down
    projection's operand; the output o is not rounded.
    """
    S = _store(store)
    return expert_down(S(swiglu_hidden(x_rows, w_gate_up_e)), w_down_e)


def experts_grouped(x, idx, w, w_gate_up, w_down, store=None):
    """y_t = sum_j w_tj * Expert_{S_tj}(x_t), computed group by group.

    [MoE-scratch] §2 `dispatch`: sort the pairs by expert, run each expert once on
    the rows that chose it, add the weighted results back to their tokens.
    """
    x = _f64(x)
    idx = np.asarray(idx)
    w = _f64(w)
    T, k = idx.shape
    n_experts = w_gate_up.shape[0]
    perm, counts, offsets = dispatch_order(idx, n_experts)
    y = np.zeros_like(x)
    for e in range(n_experts):
        sel = perm[offsets[e] : offsets[e + 1]]
        if sel.size == 0:
            continue
        tok = sel // k
        out = swiglu_expert(x[tok], w_gate_up[e], w_down[e], store)
        # Each token chooses an expert at most once, so `tok` has no repeats.
        y[tok] += w.reshape(-1)[sel][:, None] * out
    return y


def experts_dense(x, idx, w, w_gate_up, w_down):
    """The same layer computed the wasteful way: every expert on every token.

    [MoE-scratch] §2 `dense_run`: scatter the k weights into a T x E gate that is
    zero elsewhere, run all E experts on all tokens and sum gate * output.
    """
    x = _f64(x)
    idx = np.asarray(idx)
    T, k = idx.shape
    n_experts = w_gate_up.shape[0]
    gate = np.zeros((T, n_experts))
    gate[np.arange(T)[:, None], idx] = _f64(w)
    y = np.zeros_like(x)
    for e in range(n_experts):
        y += gate[:, e : e + 1] * swiglu_expert(x, w_gate_up[e], w_down[e])
    return y


# --------------------------------------------------------------------------- layer


def moe_forward(x, w_router, w_gate_up, w_down, k, router_bias=None, store=None, renorm=False):
    """The whole layer: route, dispatch, experts, combine, and the two losses.
    `renorm` selects topk_renorm's weights (the choice and both losses are unchanged).

    Returns a dict with
      y [T,d], idx [T,k], w [T,k], p [T,E], lse [T], h [T,E],
      counts [E], offsets [E+1], perm [T*k], L_lb, L_z, near_tie [T] (bool).
    """
    n_experts = _f64(w_router).shape[0]
    h = router_logits(x, w_router, router_bias)
    p, lse = softmax_lse(h)
    idx, w = topk_renorm(p, k) if renorm else topk_no_renorm(p, k)
    y = experts_grouped(x, idx, w, w_gate_up, w_down, store)
    L_lb, counts = load_balance_loss(idx, p, n_experts)
    perm, _, offsets = dispatch_order(idx, n_experts)
    return {
        "y": y,
        "idx": idx,
        "w": w,
        "p": p,
        "lse": lse,
        "h": h,
        "counts": counts,
        "offsets": offsets,
        "perm": perm,
        "L_lb": L_lb,
        "L_z": router_z_loss(lse),
        "near_tie": near_tie_tokens(p, k),
    }


def moe_objective(x, w_router, w_gate_up, w_down, k, dy, alpha, beta, router_bias=None, renorm=False):
    """The scalar whose gradient the backward returns: <dy, y> + alpha*L_lb + beta*L_z.

    [OLMoE-Guide] "Router Mechanics & Loss Formulations": L = L_LM + alpha*L_balance
    + beta*L_router_z; [OLMoE-paper] 4.1.6 and 4.1.7 fix alpha = 0.01, beta = 0.001.
    The upstream gradient dy stands in for dL_LM/dy.
    """
    out = moe_forward(x, w_router, w_gate_up, w_down, k, router_bias, renorm=renorm)
    return float(np.sum(_f64(dy) * out["y"])) + alpha * out["L_lb"] + beta * out["L_z"]


def moe_backward(x, w_router, w_gate_up, w_down, k, dy, alpha, beta, router_bias=None,
                 experts=None, store=None, renorm=False):
    """Gradients of moe_objective with respect to x and the three weights.

    Chain rule through each step of moe_forward (f and the choice carry none):
      expert rows   o_tj = W_down,e g_tj,  g = silu(a) * b,  [a; b] = W_gate_up,e x_t
      combine       dw_tj = <dy_t, o_tj>,  do_tj = w_tj dy_t
      down          dW_down,e = sum_rows do g^T,   dg = W_down,e^T do
      SwiGLU        da = dg * b * silu'(a),  db = dg * silu(a)
      gate/up       dW_gate_up,e = sum_rows [da; db] x^T,  dx_t += W_gate_up,e^T [da; db]
      softmax       dp_ti = sum_j [S_tj = i] dw_tj + alpha * E * f_i / T
                    dh_t  = p_t * (dp_t - <dp_t, p_t>) + beta * (2 lse_t / T) * p_t
      router        dW_r = sum_t dh_t x_t^T,   dx_t += W_r^T dh_t
    `experts` optionally restricts which experts' weight gradients are formed
    (the rest are left zero); dx and dW_r always use every expert. `store`
    (see the module notes) rounds the contraction operands h, do and [da; db].
    With `renorm` the weights are w_tj = p_tj / s_t (s_t the sum of the chosen
    p), so the chosen probabilities receive dp_ti = (dw_tj - sum_j' dw_tj' w_tj') / s_t
    for i = S_tj instead of dw_tj.
    Returns dict dx [T,d], dw_router [E,d], dw_gate_up [E,2f,d], dw_down [E,d,f],
    plus the forward dict under "fwd" and dw [T,k].
    """
    x = _f64(x)
    dy = _f64(dy)
    S = _store(store)
    fwd = moe_forward(x, w_router, w_gate_up, w_down, k, router_bias, store, renorm)
    idx, w, p, lse = fwd["idx"], fwd["w"], fwd["p"], fwd["lse"]
    T, d = x.shape
    n_experts = _f64(w_router).shape[0]
    f = _f64(w_down[0]).shape[1]
    want = set(range(n_experts)) if experts is None else set(int(e) for e in experts)

    dx = np.zeros_like(x)
    dw = np.zeros((T, k))
    dw_gate_up = np.zeros((n_experts, 2 * f, d))
    dw_down = np.zeros((n_experts, d, f))
    perm, counts, offsets = dispatch_order(idx, n_experts)
    for e in range(n_experts):
        sel = perm[offsets[e] : offsets[e + 1]]
        if sel.size == 0:
            continue
        tok = sel // k
        wgu = _f64(w_gate_up[e])
        wd = _f64(w_down[e])
        xr = x[tok]
        a = xr @ wgu[:f].T
        b = xr @ wgu[f:].T
        with np.errstate(over="ignore"):
            sig = 1.0 / (1.0 + np.exp(-a))
        g = S(a * sig * b)
        o = g @ wd.T
        dw.reshape(-1)[sel] = np.sum(dy[tok] * o, axis=1)
        do = S(w.reshape(-1)[sel][:, None] * dy[tok])
        dg = do @ wd
        da = S(dg * b * (sig * (1.0 + a * (1.0 - sig))))
        db = S(dg * (a * sig))
        if e in want:
            dw_down[e] = do.T @ g
            dw_gate_up[e, :f] = da.T @ xr
            dw_gate_up[e, f:] = db.T @ xr
        dx[tok] += da @ wgu[:f] + db @ wgu[f:]

    dp = np.zeros((T, n_experts))
    if renorm:
        s_chosen = np.take_along_axis(p, idx, axis=1).sum(axis=1, keepdims=True)
        dsel = (dw - np.sum(dw * w, axis=1, keepdims=True)) / s_chosen
        np.add.at(dp, (np.arange(T)[:, None].repeat(k, axis=1), idx), dsel)
    else:
        np.add.at(dp, (np.arange(T)[:, None].repeat(k, axis=1), idx), dw)
    frac = counts / float(T * k)
    dp += alpha * n_experts * frac[None, :] / T
    dh = p * (dp - np.sum(dp * p, axis=1, keepdims=True))
    dh += beta * (2.0 * lse / T)[:, None] * p
    w_r = _f64(w_router)
    dx += dh @ w_r
    return {
        "dx": dx,
        "dw_router": dh.T @ x,
        "dw_gate_up": dw_gate_up,
        "dw_down": dw_down,
        "dw": dw,
        "dh": dh,
        "fwd": fwd,
    }


def token_input_grads(x_rows, w_router, w_gate_up, w_down, k, dy_rows, alpha, beta, counts, n_tokens,
                      router_bias=None):
    """dx for some of the tokens of a batch, one token at a time.

    Every step of the chain rule in moe_backward acts on one token alone except
    the load-balance term, whose derivative with respect to p_ti is
    alpha * E * f_i / T: it needs only the batch's counts (f_i = count_i / (T k))
    and its size T = `n_tokens`. Given those, the rows `x_rows` (any subset of
    the batch, with their upstream gradients `dy_rows`) get exactly the dx rows
    moe_backward gives them. Returns dx [n, d].
    """
    x = _f64(x_rows)
    dy = _f64(dy_rows)
    w_r = _f64(w_router)
    n_experts = w_r.shape[0]
    f = _f64(w_down[0]).shape[1]
    h = router_logits(x, w_r, router_bias)
    p, lse = softmax_lse(h)
    idx, w = topk_no_renorm(p, k)
    n = x.shape[0]
    dx = np.zeros_like(x)
    dp = np.zeros((n, n_experts))
    for t in range(n):
        for j in range(k):
            e = int(idx[t, j])
            wgu = _f64(w_gate_up[e])
            wd = _f64(w_down[e])
            a = wgu[:f] @ x[t]
            b = wgu[f:] @ x[t]
            sig = 1.0 / (1.0 + np.exp(-a))
            g = a * sig * b
            dp[t, e] += dy[t] @ (wd @ g)        # dw_tj = <dy_t, o_tj>
            dg = wd.T @ (w[t, j] * dy[t])       # do_tj = w_tj dy_t
            da = dg * b * (sig * (1.0 + a * (1.0 - sig)))
            db = dg * (a * sig)
            dx[t] += wgu[:f].T @ da + wgu[f:].T @ db
    frac = np.asarray(counts, dtype=np.float64) / float(n_tokens * k)
    dp += alpha * n_experts * frac[None, :] / n_tokens
    dh = p * (dp - np.sum(dp * p, axis=1, keepdims=True))
    dh += beta * (2.0 * lse / n_tokens)[:, None] * p
    return dx + dh @ w_r


def expert_weight_grad_slices(x, idx, w, dy, w_gate_up_e, w_down_e, e, gate_up_rows, down_cols):
    """Chosen rows of dW_gate_up,e and chosen columns of dW_down,e.

    Same formulas as moe_backward (dW_gate_up,e = sum over e's rows of [da; db] x^T,
    dW_down,e = sum over e's rows of do g^T), restricted so that only the named
    hidden units are evaluated: row j < f of dW_gate_up needs a_j, b_j and dg_j of
    every row routed to e; row f + j the same; column c of dW_down needs g_c.
    `x`, `idx`, `w`, `dy` are the whole batch's. Returns (rows [len, d], cols [d, len]).
    """
    x = _f64(x)
    dy = _f64(dy)
    idx = np.asarray(idx)
    w = _f64(w)
    wgu = _f64(w_gate_up_e)
    wd = _f64(w_down_e)
    f = wd.shape[1]
    tok, slot = np.nonzero(idx == e)
    xr = x[tok]
    do = w[tok, slot][:, None] * dy[tok]

    def unit(j):
        a = xr @ wgu[j]
        b = xr @ wgu[f + j]
        sig = 1.0 / (1.0 + np.exp(-a))
        return a, b, sig

    rows = []
    for r in gate_up_rows:
        j = int(r) % f
        a, b, sig = unit(j)
        dg = do @ wd[:, j]
        coef = dg * b * (sig * (1.0 + a * (1.0 - sig))) if int(r) < f else dg * (a * sig)
        rows.append(coef @ xr)
    cols = []
    for c in down_cols:
        a, b, sig = unit(int(c))
        cols.append(do.T @ (a * sig * b))
    return np.array(rows).reshape(len(rows), x.shape[1]), np.array(cols).T.reshape(wd.shape[0], len(cols))


# --------------------------------------------------------------------------- stack


def rms_norm(x, weight=None, eps=1e-5):
    """RMSNorm: x / sqrt(mean(x^2) + eps) * weight.

    [MoE-scratch] §3 `RMSNorm` (eps 1e-5, the library default noted beside the
    config; weight initialised to one).
    """
    x = _f64(x)
    y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return y if weight is None else y * _f64(weight)


def stack_forward(x0, layers, k, eps=1e-5, round_input=None):
    """A stack of MoE blocks with a residual stream: r <- r + MoE_l(RMSNorm(r)).

    [MoE-scratch] §3 `Block.forward`: pre-norm, and the residual stream is kept in
    32-bit floats between layers. `layers` is a list of dicts with keys
    w_router, w_gate_up, w_down and optionally router_bias. `round_input`, if
    given, is applied to the normalised activations before each layer (the
    GPU feeds the experts bf16 activations, so the oracle can be handed the
    same rounding). Returns the final residual [T, d] and the per-layer
    forward dicts.
    """
    r = _f64(x0).copy()
    outs = []
    for L in layers:
        xn = rms_norm(r, eps=eps)
        if round_input is not None:
            xn = _f64(round_input(xn))
        out = moe_forward(xn, L["w_router"], L["w_gate_up"], L["w_down"], k,
                          L.get("router_bias"))
        r = r + out["y"]
        outs.append(out)
    return r, outs


# --------------------------------------------------------------------------- expert choice


def ec_capacity(n_tokens, k, n_experts):
    """Tokens per expert under expert choice: ceil(T*k/E), at most T.

    With this capacity the E experts process about T*k rows in total, the same
    expert work as top-k token choice ([OLMoE-paper] section 4.1.4 compares the
    two at equal compute).
    """
    return min(int(n_tokens), -(-int(n_tokens) * int(k) // int(n_experts)))


def expert_choice(p, capacity):
    """Each expert picks its `capacity` highest-probability tokens.

    [OLMoE-paper] section 4.1.4 "Expert Choice vs. Token Choice": the experts
    choose the tokens. For expert e the candidates are the column p[:, e] of
    the softmax over experts; the C largest are kept, equal values going to the
    lower token index (a stable sort of -p[:, e]). The chosen tokens are listed
    in ascending token order (the order of the expert's rows).
    Returns (sel [E, C] int64 token indices, gates [E, C] float64 = p[sel, e]).
    """
    p = _f64(p)
    T, E = p.shape
    C = int(capacity)
    sel = np.zeros((E, C), dtype=np.int64)
    gates = np.zeros((E, C))
    for e in range(E):
        top = np.argsort(-p[:, e], kind="stable")[:C]
        top = np.sort(top)
        sel[e] = top
        gates[e] = p[top, e]
    return sel, gates


def experts_expert_choice(x, sel, gates, w_gate_up, w_down, store=None):
    """y_t = sum over experts e that chose t (ascending e) of p[t, e] * Expert_e(x_t).

    Each expert runs once on its C rows (as in [MoE-scratch] section 2
    `dispatch`, with the rows given by the expert's choice); a token that no
    expert chose gets y_t = 0.
    """
    x = _f64(x)
    sel = np.asarray(sel)
    gates = _f64(gates)
    y = np.zeros_like(x)
    for e in range(sel.shape[0]):
        if sel.shape[1] == 0:
            continue
        out = swiglu_expert(x[sel[e]], w_gate_up[e], w_down[e], store)
        # an expert picks a token at most once, so sel[e] has no repeats
        y[sel[e]] += gates[e][:, None] * out
    return y


def moe_forward_expert_choice(x, w_router, w_gate_up, w_down, k, router_bias=None, capacity=None,
                              store=None):
    """The layer with expert-choice routing (see the module notes for the reading).

    Returns a dict with y [T,d], sel [E,C], gates [E,C], p [T,E], lse [T], h [T,E],
    capacity C, fanout [T] (experts per token), L_lb (0: no balance loss), L_z.
    """
    x = _f64(x)
    T = x.shape[0]
    E = _f64(w_router).shape[0]
    C = ec_capacity(T, k, E) if capacity is None else int(capacity)
    h = router_logits(x, w_router, router_bias)
    p, lse = softmax_lse(h)
    sel, gates = expert_choice(p, C)
    y = experts_expert_choice(x, sel, gates, w_gate_up, w_down, store)
    fanout = np.bincount(sel.reshape(-1), minlength=T)
    return {
        "y": y,
        "sel": sel,
        "gates": gates,
        "p": p,
        "lse": lse,
        "h": h,
        "capacity": C,
        "fanout": fanout,
        "L_lb": 0.0,
        "L_z": router_z_loss(lse),
    }


def moe_objective_expert_choice(x, w_router, w_gate_up, w_down, k, dy, beta, router_bias=None, capacity=None):
    """<dy, y> + beta * L_z for the expert-choice layer (it has no balance loss)."""
    out = moe_forward_expert_choice(x, w_router, w_gate_up, w_down, k, router_bias, capacity)
    return float(np.sum(_f64(dy) * out["y"])) + beta * out["L_z"]


def moe_backward_expert_choice(x, w_router, w_gate_up, w_down, k, dy, beta, router_bias=None, capacity=None):
    """Gradients of moe_objective_expert_choice with respect to x and the weights.

    The same chain rule as moe_backward, with the expert's chosen tokens as its
    rows and p[t, e] as the weight of (t, e); the choice carries no gradient:
      expert rows   o_te = W_down,e g_te,  g = silu(a) * b,  [a; b] = W_gate_up,e x_t
      combine       dp_te = <dy_t, o_te> for t chosen by e (zero elsewhere),
                    do_te = p_te dy_t
      experts       as in moe_backward
      softmax       dh_t = p_t * (dp_t - <dp_t, p_t>) + beta * (2 lse_t / T) * p_t
      router        dW_r = sum_t dh_t x_t^T,   dx_t += W_r^T dh_t
    Returns dict dx, dw_router, dw_gate_up, dw_down, dp [T,E], and "fwd".
    """
    x = _f64(x)
    dy = _f64(dy)
    fwd = moe_forward_expert_choice(x, w_router, w_gate_up, w_down, k, router_bias, capacity)
    sel, p, lse = fwd["sel"], fwd["p"], fwd["lse"]
    T, d = x.shape
    n_experts = p.shape[1]
    f = _f64(w_down[0]).shape[1]
    dx = np.zeros_like(x)
    dp = np.zeros((T, n_experts))
    dw_gate_up = np.zeros((n_experts, 2 * f, d))
    dw_down = np.zeros((n_experts, d, f))
    for e in range(n_experts):
        tok = sel[e]
        if tok.size == 0:
            continue
        wgu = _f64(w_gate_up[e])
        wd = _f64(w_down[e])
        xr = x[tok]
        a = xr @ wgu[:f].T
        b = xr @ wgu[f:].T
        with np.errstate(over="ignore"):
            sig = 1.0 / (1.0 + np.exp(-a))
        g = a * sig * b
        o = g @ wd.T
        dp[tok, e] = np.sum(dy[tok] * o, axis=1)
        do = p[tok, e][:, None] * dy[tok]
        dg = do @ wd
        da = dg * b * (sig * (1.0 + a * (1.0 - sig)))
        db = dg * (a * sig)
        dw_down[e] = do.T @ g
        dw_gate_up[e, :f] = da.T @ xr
        dw_gate_up[e, f:] = db.T @ xr
        dx[tok] += da @ wgu[:f] + db @ wgu[f:]
    dh = p * (dp - np.sum(dp * p, axis=1, keepdims=True))
    dh += beta * (2.0 * lse / T)[:, None] * p
    dx += dh @ _f64(w_router)
    return {"dx": dx, "dw_router": dh.T @ x, "dw_gate_up": dw_gate_up, "dw_down": dw_down, "dp": dp, "fwd": fwd}
