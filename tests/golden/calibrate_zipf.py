"""Finds the Zipf router-offset strength for the skewed 16-layer stack.

The stack workload biases every layer's router logits by b_e = lam * ln(z_e),
z_e = (e + 1)^-1.2, so that the 8 most favoured experts receive about half of
all top-8 assignments. This script finds lam by bisection with the CPU oracle
on layer 0's seeded input (the RMS-normalised residual stream entering the
stack) and writes it to tests/golden/zipf_lambda.txt. The synthetic-input
module carries the same constant; a test checks that they agree and that the
share measured with the oracle is 0.50 +- 0.01.

    python tests/golden/calibrate_zipf.py
"""

import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import moe_oracle as O  # noqa: E402
from sparse_moe_transformer_route_b200 import synthetic as S  # noqa: E402


def top8_share(lam, x, w_router, k=8):
    E = w_router.shape[0]
    b = S.zipf_router_offset(E, lam).double().numpy()
    p, _ = O.softmax_lse(O.router_logits(x, w_router, b))
    idx, _ = O.topk_no_renorm(p, k)
    counts = np.bincount(idx.reshape(-1), minlength=E)
    return float(np.sort(counts)[::-1][:8].sum() / counts.sum())


def layer0_inputs(T=S.STACK_8192.T):
    x0, layers = S.stack_inputs(S.STACK_8192, 1, seed=5, zipf=False)
    x = O.rms_norm(x0[:T].double().numpy())
    x = x.astype(np.float32)
    x = torch.from_numpy(x).to(torch.bfloat16).double().numpy()  # the layer's bf16 input
    return x, layers[0]["w_router"].double().numpy()


def calibrate(target=0.5, tol=1e-4):
    x, wr = layer0_inputs()
    lo, hi = 0.0, 4.0
    while hi - lo > tol:
        mid = 0.5 * (lo + hi)
        if top8_share(mid, x, wr) < target:
            lo = mid
        else:
            hi = mid
    lam = round(0.5 * (lo + hi), 4)
    return lam, top8_share(lam, x, wr)


if __name__ == "__main__":
    lam, share = calibrate()
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "zipf_lambda.txt")
    with open(out, "w") as fh:
        fh.write("# Zipf router-offset strength for the skewed stack, written by calibrate_zipf.py\n")
        fh.write("# (bisection with the CPU oracle on layer 0 of the seeded stack input).\n")
        fh.write(f"lambda {lam}\n")
        fh.write(f"top8_share {share:.4f}\n")
    print(lam, share)
