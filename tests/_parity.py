"""Shared helpers for the GPU parity tests: tolerances, conversions, and a lazy
fp64 view of large expert weights for the oracle."""

import os

import numpy as np
import pytest
import torch

# Agreement bars: outputs and gradients within max-abs 2e-2 AND relative L2
# 1e-2 (bf16 inputs, fp32 accumulation); losses within 1e-4 relative; indices
# and the dispatch permutation bit-exact except counted near-ties.
MAX_ABS = 2e-2
REL_L2 = 1e-2
LOSS_REL = 1e-4


def f64(t):
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to("cpu", torch.float64).numpy()


def bf16_round(a):
    """fp64 values rounded to bf16 the way the kernels round an fp32 result: to
    fp32 first, then to bf16 (both round to nearest even); returned as fp64."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    return t.to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


def f32_round(a):
    return np.asarray(a, dtype=np.float64).astype(np.float32).astype(np.float64)


def errors(got, ref):
    got = f64(got)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    diff = got - ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(diff)) / denom if denom > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_close(got, ref, name, max_abs=MAX_ABS, rel_l2=REL_L2):
    ma, rl = errors(got, ref)
    assert ma <= max_abs and rl <= rel_l2, f"{name}: max abs {ma:.3e} (bar {max_abs}), rel L2 {rl:.3e} (bar {rel_l2})"
    return ma, rl


def assert_loss_close(got, ref, name):
    got = float(got)
    rel = abs(got - ref) / max(abs(ref), 1e-30)
    assert rel <= LOSS_REL, f"{name}: {got!r} vs {ref!r} (rel {rel:.2e})"


class LazyF64:
    """Indexable fp64 view of a [E, ...] torch tensor, converted one expert at a time."""

    def __init__(self, t):
        self.t = t.detach().cpu()
        self.shape = tuple(self.t.shape)

    def __getitem__(self, e):
        return self.t[e].to(torch.float64).numpy()


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_moe_transformer_route_b200 import binding as B
    if not os.path.exists(B.LIB_PATH):
        from sparse_moe_transformer_route_b200 import build
        build.build()
    major, minor = torch.cuda.get_device_capability()
    assert (major, minor) == (10, 0), "these kernels are built for sm_100a (B200)"


def padded_group_starts(counts, align=128):
    gs = np.zeros(len(counts) + 1, dtype=np.int64)
    gs[1:] = np.cumsum([(c + align - 1) // align * align for c in counts])
    return gs


def index_parity(gpu_idx, ref_idx, near_tie):
    """Bit-exact agreement of the chosen experts (and their slot order) on every
    token that is not a near-tie; returns (mismatching tokens, near-tie count)."""
    g = np.asarray(gpu_idx)
    r = np.asarray(ref_idx)
    diff = np.any(g != r, axis=1)
    bad = np.nonzero(diff & ~near_tie)[0]
    return bad, int(near_tie.sum()), diff
