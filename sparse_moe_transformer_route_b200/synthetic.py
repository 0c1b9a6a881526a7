"""Seeded synthetic inputs with OLMoE's shapes.

This module only draws random numbers and shapes them; it holds none of the
layer's arithmetic. Both the CUDA path (through its tests and the benchmark)
and the CPU oracle are fed from here.

Recipe (all drawn with a CPU torch.Generator in float32, then cast once):
  * tokens x: rows of N(0, 1), each row divided by its root-mean-square
    (sqrt(mean(x^2) + 1e-5)), i.e. activations as they leave a pre-norm with
    unit weight, which is what an OLMoE MoE block receives; the small fp32
    layer uses plain N(0, 1) rows.
  * router W_r [E, d], expert W_gate_up [E, 2f, d] (gate rows then up rows),
    W_down [E, d, f]: N(0, 0.02^2).
  * upstream gradient dy [T, d]: N(0, 1).
  * skewed stack: a per-expert router offset b_e = lam * ln(z_e) with
    z_e = (e + 1)^-1.2 (a Zipf law over expert ids); lam is the fixed constant
    ZIPF_LAMBDA, chosen so that the 8 most favoured experts take about half of
    all assignments on these inputs (the tests measure the share).
"""

from __future__ import annotations

import dataclasses
import math

import torch

# OLMoE-1B-7B layer shapes ("Mixture-of-experts LLMs from scratch with OLMoE",
# section 3, the config dump: hidden 2048, 64 experts, 8 per token, expert width
# 1024, 16 layers).
OLMOE_D_MODEL = 2048
OLMOE_N_EXPERTS = 64
OLMOE_TOP_K = 8
OLMOE_D_FF = 1024
OLMOE_N_LAYERS = 16
INIT_STD = 0.02
ALPHA_LB = 0.01
BETA_Z = 0.001
ZIPF_S = 1.2
ZIPF_LAMBDA = 0.5599  # the 8 most favoured experts then take half the assignments
RMS_EPS = 1e-5


@dataclasses.dataclass(frozen=True)
class LayerShape:
    T: int
    d_model: int = OLMOE_D_MODEL
    n_experts: int = OLMOE_N_EXPERTS
    top_k: int = OLMOE_TOP_K
    d_ff: int = OLMOE_D_FF


# The five workloads, by what they are.
SMALL_FP32 = LayerShape(T=128, d_model=512, n_experts=64, top_k=8, d_ff=256)
PREFILL_4096 = LayerShape(T=4096)
DECODE_TOKENS = (1, 8, 32, 64)
TRAIN_16384 = LayerShape(T=16384)
STACK_8192 = LayerShape(T=8192)
STACK_LAYERS = OLMOE_N_LAYERS


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def unit_rms_rows(T: int, d: int, g: torch.Generator) -> torch.Tensor:
    x = torch.randn(T, d, generator=g, dtype=torch.float32)
    return x * torch.rsqrt(x.pow(2).mean(dim=-1, keepdim=True) + RMS_EPS)


def make_tokens(shape: LayerShape, seed: int, dtype=torch.bfloat16, normalised=True):
    g = _gen(seed)
    if normalised:
        x = unit_rms_rows(shape.T, shape.d_model, g)
    else:
        x = torch.randn(shape.T, shape.d_model, generator=g, dtype=torch.float32)
    return x.to(dtype)


def make_weights(shape: LayerShape, seed: int, dtype=torch.bfloat16, std=INIT_STD):
    """Router and expert weights of one layer: (w_router, w_gate_up, w_down)."""
    g = _gen(seed)
    E, d, f = shape.n_experts, shape.d_model, shape.d_ff
    w_router = torch.randn(E, d, generator=g, dtype=torch.float32) * std
    w_gate_up = torch.randn(E, 2 * f, d, generator=g, dtype=torch.float32) * std
    w_down = torch.randn(E, d, f, generator=g, dtype=torch.float32) * std
    return w_router.to(dtype), w_gate_up.to(dtype), w_down.to(dtype)


def make_upstream_grad(shape: LayerShape, seed: int, dtype=torch.bfloat16):
    g = _gen(seed)
    return torch.randn(shape.T, shape.d_model, generator=g, dtype=torch.float32).to(dtype)


def zipf_router_offset(n_experts: int, lam: float | None = None, s: float = ZIPF_S):
    """b_e = lam * ln((e + 1)^-s), float32 [E]: favours low expert ids."""
    lam = ZIPF_LAMBDA if lam is None else lam
    return torch.tensor([lam * (-s) * math.log(e + 1) for e in range(n_experts)],
                        dtype=torch.float32)


@dataclasses.dataclass
class LayerInputs:
    shape: LayerShape
    x: torch.Tensor
    w_router: torch.Tensor
    w_gate_up: torch.Tensor
    w_down: torch.Tensor
    dy: torch.Tensor | None = None
    router_bias: torch.Tensor | None = None


def layer_inputs(shape: LayerShape, seed: int, dtype=torch.bfloat16, normalised=True,
                 with_grad=False) -> LayerInputs:
    """All inputs of one layer from one seed (weights, tokens, upstream gradient)."""
    w_router, w_gate_up, w_down = make_weights(shape, 1000003 * seed + 11, dtype)
    x = make_tokens(shape, 1000003 * seed + 23, dtype, normalised)
    dy = make_upstream_grad(shape, 1000003 * seed + 37, dtype) if with_grad else None
    return LayerInputs(shape, x, w_router, w_gate_up, w_down, dy)


def stack_inputs(shape: LayerShape, n_layers: int, seed: int, dtype=torch.bfloat16,
                 zipf=True):
    """Residual-stream input and independently seeded weights for each layer."""
    x0 = make_tokens(shape, 1000003 * seed + 23, torch.float32, normalised=False)
    layers = []
    for l in range(n_layers):
        w_router, w_gate_up, w_down = make_weights(shape, 7919 * (seed + 1) + 104729 * l, dtype)
        bias = zipf_router_offset(shape.n_experts) if zipf else None
        layers.append(dict(w_router=w_router, w_gate_up=w_gate_up, w_down=w_down,
                           router_bias=bias))
    return x0, layers
