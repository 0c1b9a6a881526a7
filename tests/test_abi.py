"""The C-ABI library loads on a machine without a GPU and exports every entry
point include/moe.h declares. Only host-side functions are called here (shape
validation, sizes, status strings); nothing that launches work."""

import ctypes
import os
import re

import pytest
import torch

import sparse_moe_transformer_route_b200 as M
from sparse_moe_transformer_route_b200 import binding as B
from sparse_moe_transformer_route_b200 import synthetic as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module", autouse=True)
def built_library():
    if not os.path.exists(B.LIB_PATH):
        from sparse_moe_transformer_route_b200 import build
        build.build()
    return B.LIB_PATH


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert _declared() == sorted(B.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(B.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name


def test_library_has_no_gpu_only_load_dependencies():
    # static CUDA runtime: the .so must load here, where there is no driver
    lib = M.lib()
    assert lib.moe_abi_version() == B.ABI_VERSION == 6


def test_status_strings():
    for code, name in B.STATUS_NAMES.items():
        assert M.status_string(code).startswith(name)
    assert M.status_string(99) == "unknown moe_status"


def test_config_validation():
    ok = M.config(4096, 2048, 64, 8, 1024)
    assert M.moe_check_config(ok) == 0
    bad = [
        M.config(0, 2048, 64, 8, 1024),            # no tokens
        M.config(16, 2000, 64, 8, 1024),           # d not a multiple of 128
        M.config(16, 2048, 64, 8, 1000),           # f not a multiple of 128
        M.config(16, 2048, 64, 17, 1024),          # k > 16
        M.config(16, 2048, 4, 8, 1024),            # k > E
        M.config(16, 2048, 300, 8, 1024),          # E > 256
        M.config(16, 4096, 64, 8, 1024, torch.float32),  # fp32 router tile limit
    ]
    odd = M.config(16, 2048, 64, 8, 1024)
    odd.router_mode = 2                            # no such router mode
    bad.append(odd)
    for cfg in bad:
        assert M.moe_check_config(cfg) == 2
        assert M.moe_workspace_bytes(cfg) == 0
        assert M.moe_padded_rows(cfg) == -1
    assert M.moe_check_config(M.config(16, 2048, 64, 8, 1024, renorm=True)) == 0


@pytest.mark.parametrize("T,E,k", [(1, 64, 8), (128, 64, 8), (4096, 64, 8), (300, 16, 4)])
def test_padded_rows_bound(T, E, k):
    cfg = M.config(T, 512, E, k, 256)
    P = M.moe_padded_rows(cfg)
    assert P % B.ROW_ALIGN == 0
    # every expert's group is padded to a multiple of 128: sum_e roundup(c_e) <= T*k + E*127
    assert P >= T * k + E * (B.ROW_ALIGN - 1)
    assert P < T * k + E * (B.ROW_ALIGN - 1) + B.ROW_ALIGN


@pytest.mark.parametrize("T,E,k", [(1, 64, 8), (7, 64, 8), (4096, 64, 8), (16384, 64, 8), (300, 16, 4),
                                   (129, 64, 1), (5, 4, 4)])
def test_expert_choice_capacity_and_groups_fit(T, E, k):
    """The default capacity is ceil(T k / E) capped at T (the oracle's ec_capacity),
    and E groups of it, each padded to 128 rows, fit in the padded row count."""
    cfg = M.config(T, 512, E, k, 256)
    C = M.moe_expert_choice_capacity(cfg)
    assert C == min(T, -(-T * k // E))
    cpad = -(-C // B.ROW_ALIGN) * B.ROW_ALIGN
    assert E * cpad <= M.moe_padded_rows(cfg)


def test_expert_choice_capacity_rejects_a_bad_config():
    bad = M.config(4, 128, 8, 2, 128)
    bad.d_model = 100
    with pytest.raises(M.MoeError):
        M.moe_expert_choice_capacity(bad)


def test_workspace_sizes_grow_with_training():
    cfg = M.config(S.PREFILL_4096.T, 2048, 64, 8, 1024)
    fwd = M.moe_workspace_bytes(cfg, False)
    bwd = M.moe_workspace_bytes(cfg, True)
    P = M.moe_padded_rows(cfg)
    assert fwd >= P * 2048 * 2 * 2 + P * 1024 * 2  # x_perm, o_perm, h
    # + the saved fp32 pre-activations and fp32 expert outputs
    assert bwd > fwd + P * 2 * 1024 * 4 + P * 2048 * 4


def test_binding_rejects_wrong_tensors_before_calling():
    cfg = M.config(4, 128, 8, 2, 128)
    x = torch.zeros(4, 128, dtype=torch.float32)
    with pytest.raises(TypeError):
        M.moe_combine(cfg, x, x, x, x)
    with pytest.raises(ValueError):
        B._ptr(torch.zeros(4, 128, dtype=torch.bfloat16), torch.bfloat16, (4, 128), "x")  # host tensor


def test_binding_checks_the_new_entry_points_before_calling():
    """Wrong dtypes, shapes and host tensors are refused in Python, before the
    library is called (no GPU needed, so each case fails on the first argument
    the binding examines)."""
    cfg = M.config(4, 128, 8, 2, 128)
    C = M.moe_expert_choice_capacity(cfg)  # ceil(4 * 2 / 8) = 1
    assert C == 1
    bf = torch.bfloat16
    x = torch.zeros(4, 128, dtype=bf)
    wr = torch.zeros(8, 128, dtype=bf)
    wgu = torch.zeros(8, 256, 128, dtype=bf)
    wd = torch.zeros(8, 128, 128, dtype=bf)
    ws = torch.zeros(1024, dtype=torch.uint8)
    sel = torch.zeros(8, C, dtype=torch.int32)
    gates = torch.zeros(8, C)
    with pytest.raises(TypeError, match="x must be torch.bfloat16"):
        M.moe_forward_decode(cfg, x.float(), wr, None, wgu, wd, x, None, None, None, ws)
    with pytest.raises(ValueError, match="x must have shape"):
        M.moe_forward_decode(cfg, x[:3], wr, None, wgu, wd, x, None, None, None, ws)
    with pytest.raises(ValueError, match="x must be a CUDA tensor"):
        M.moe_forward_decode(cfg, x, wr, None, wgu, wd, x, None, None, None, ws)
    with pytest.raises(TypeError, match="x must be torch.bfloat16"):
        M.moe_route_expert_choice(cfg, x.float(), wr, None, sel, gates, None, None, None, ws)
    with pytest.raises(ValueError, match="x must be a CUDA tensor"):
        M.moe_route_expert_choice(cfg, x, wr, None, sel, gates, None, None, None, ws)
    with pytest.raises(ValueError, match="x must have shape"):
        M.moe_forward_expert_choice(cfg, torch.zeros(4, 256, dtype=bf), wr, None, wgu, wd, x, None, sel, gates, ws)
    with pytest.raises(ValueError, match="x_host must be a host tensor"):
        M.moe_forward_host_async(cfg, x.cuda() if torch.cuda.is_available() else _FakeCuda(x), wr, None, wgu, wd,
                                 x, None, ws)
    with pytest.raises(TypeError, match="x_host must be torch.bfloat16"):
        M.moe_forward_host_async(cfg, x.float(), wr, None, wgu, wd, x, None, ws)
    with pytest.raises(ValueError, match="w_router must be a CUDA tensor"):
        M.moe_forward_host_async(cfg, x, wr, None, wgu, wd, x, None, ws)


class _FakeCuda(torch.Tensor):
    """A host tensor that reports itself as a CUDA tensor (for the binding's
    host-or-device check on a machine without a GPU)."""

    @staticmethod
    def __new__(cls, t):
        return torch.Tensor._make_subclass(cls, t)

    @property
    def is_cuda(self):
        return True
