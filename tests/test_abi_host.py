"""Host-only checks of the C ABI (no GPU needed): the library loads, exports every
entry point include/bitmoe.h declares, and rejects bad arguments before any launch.
Also checks that the oracle and the CUDA package do not import each other."""
import ast
import ctypes
import os
import re

import pytest

import bit_moe_routed_b200 as bm
from bit_moe_routed_b200 import build as bm_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitmoe.h")


@pytest.fixture(scope="module")
def L():
    bm_build.build()
    return bm.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("moe_route_topk", "moe_dispatch", "moe_expert_ffn", "moe_combine"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    names = declared_functions()
    assert set(names) == set(bm.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def test_workspace_size_host(L):
    assert bm.workspace_size(0, 6, 256, 4096, 2048) > 0
    assert bm.workspace_size(1, 6, 256, 4096, 2048) > 7 * 4096
    assert bm.workspace_size(4, 2, 8, 100, 128) == 0  # d not a multiple of 128


def test_invalid_arguments_rejected_on_host(L):
    P = ctypes.c_void_p
    dummy = P(256)
    assert L.moe_route_topk(dummy, 4, 8, 9, dummy, dummy, None) == bm.MOE_ERR_INVALID_ARG
    assert b"k=9" in L.moe_last_error()
    assert L.moe_route_topk(dummy, -1, 8, 2, dummy, dummy, None) == bm.MOE_ERR_INVALID_ARG
    assert L.moe_route_topk(P(2), 4, 8, 2, dummy, dummy, None) == bm.MOE_ERR_INVALID_ARG  # align
    assert L.moe_act_quant(dummy, 4, 100, dummy, dummy, None) == bm.MOE_ERR_INVALID_ARG
    assert L.moe_combine(dummy, dummy, dummy, dummy, 4, 0, 64, dummy, None) == \
        bm.MOE_ERR_INVALID_ARG
    w = bm._Weights(256, 256, 256, 256, 256, 256, 8, 256, 100)  # f not a multiple of 128
    assert L.moe_expert_ffn(dummy, 4, 2, ctypes.byref(w), dummy, dummy, dummy, dummy, dummy,
                            1 << 30, None) == bm.MOE_ERR_INVALID_ARG
    w = bm._Weights(16, 256, 256, 256, 256, 256, 8, 256, 128)  # codes not 32-byte aligned
    assert L.moe_expert_ffn(dummy, 4, 2, ctypes.byref(w), dummy, dummy, dummy, dummy, dummy,
                            1 << 30, None) == bm.MOE_ERR_INVALID_ARG
    # T == 0 is a valid no-op for route / quant / combine
    assert L.moe_route_topk(None, 0, 8, 2, None, None, None) == bm.MOE_OK
    assert L.moe_combine(None, None, None, None, 0, 2, 64, None, None) == bm.MOE_OK


def _imports(path):
    mods = set()
    for dirpath, _, files in os.walk(path):
        for fn in files:
            if fn.endswith(".py"):
                tree = ast.parse(open(os.path.join(dirpath, fn)).read())
                for node in ast.walk(tree):
                    if isinstance(node, ast.Import):
                        mods.update(a.name.split(".")[0] for a in node.names)
                    elif isinstance(node, ast.ImportFrom) and node.module:
                        mods.add(node.module.split(".")[0])
    return mods


def test_oracle_and_cuda_path_are_independent():
    assert "bit_moe_routed_b200" not in _imports(os.path.join(ROOT, "oracle"))
    assert "oracle" not in _imports(os.path.join(ROOT, "bit_moe_routed_b200"))
    assert "synth" not in _imports(os.path.join(ROOT, "bit_moe_routed_b200"))
    for p in ("oracle", "synth"):
        assert p not in open(os.path.join(ROOT, "bit_moe_routed_b200", "__init__.py")).read() \
            .split('"""')[2]


def test_gemv_switch_host(L):
    """moe_set_gemv_max_tokens takes 0 (tile kernels only) or a positive bound, and
    rejects a negative one with a message; the workspace of a single token holds the
    GEMV path's fp32 hidden state (k + 1 rows of f)."""
    assert L.moe_set_gemv_max_tokens(-1) == bm.MOE_ERR_INVALID_ARG
    assert b"t=-1" in L.moe_last_error()
    try:
        assert L.moe_set_gemv_max_tokens(0) == bm.MOE_OK
    finally:
        assert L.moe_set_gemv_max_tokens(bm.GEMV_MAX_TOKENS) == bm.MOE_OK
    one = bm.workspace_size(1, 6, 256, 4096, 2048)
    two = bm.workspace_size(2, 6, 256, 4096, 2048)
    assert one >= 7 * 2048 * 4
    assert two > 0


def test_binding_descriptors_marshal_on_the_host():
    """The binding's weight descriptors build their C structs from tensors (no GPU)."""
    import torch
    import bit_moe_routed_b200 as bm
    E, d, f = 3, 512, 256
    mk = lambda *s: torch.zeros(s, dtype=torch.uint8)  # noqa: E731
    w = bm.LayerWeights(mk(E + 1, f, d // 2), mk(E + 1, f, d // 32), mk(E + 1, f, d // 2),
                        mk(E + 1, f, d // 32), mk(E + 1, d, f // 2), mk(E + 1, d, f // 32))
    st = w.struct()
    assert (w.E, w.d, w.f) == (E, d, f) and (st.E, st.d, st.f) == (E, d, f)
    q = bm.Q2Experts(mk(E, f, d // 4), mk(E, f, d // 128), mk(E, f, d // 4), mk(E, f, d // 128),
                     mk(E, d, f // 4), mk(E, d, f // 128))
    assert q.struct().gate_codes == q.gate_codes.data_ptr()
    h = bm.HostExperts(*(getattr(w, n)[:E] for n in bm._NAMES6))
    assert h.struct().down_scales == w.down_scales.data_ptr()
