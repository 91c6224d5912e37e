"""CPU checks of the C ABI library: it loads without a GPU, exports every
function that include/moe_capi.h declares, and rejects bad arguments on the
host (before any device work) with the documented codes."""
import ctypes
import os
import re

import pytest

from __graft_entry__ import ROOT, build

HEADER = os.path.join(ROOT, "include", "moe_capi.h")


@pytest.fixture(scope="module")
def capi():
    build()
    from mixture_experts_layer_40_b200 import capi as c
    return c


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_abi():
    names = declared_functions()
    for required in ["moe_quantize_1x128", "moe_route", "moe_forward", "moe_update_bias",
                     "moe_workspace_size", "moe_get_status"]:
        assert required in names


def test_library_exports_every_declared_symbol(capi):
    lib = ctypes.CDLL(capi.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(declared_functions()) == set(capi.SIGNATURES)


def test_workspace_layout(capi):
    sh = capi.shape_of(4096, 7168, 256, 8, 2048)
    L = capi.moe_workspace_layout(sh)
    assert L.routed_cap % 128 == 0 and L.routed_cap >= 4096 * 8 + 256 * 127
    assert L.rows_total == L.routed_cap + 4096
    offs = [getattr(L, f) for f in capi._LAYOUT_FIELDS]
    assert all(o % 256 == 0 for o in offs)
    assert offs == sorted(offs) and L.total == capi.moe_workspace_size(sh)
    assert L.y_rows + L.rows_total * 7168 * 2 <= L.total


@pytest.mark.parametrize("shape", [(-1, 256, 16, 4, 128), (64, 200, 16, 4, 128), (64, 256, 16, 4, 100),
                                   (64, 256, 15, 4, 128), (64, 256, 16, 17, 128), (64, 256, 16, 0, 128),
                                   (64, 128, 16, 4, 128), (64, 256, 2048, 4, 128)])
def test_bad_shapes_rejected(capi, shape):
    sh = capi.shape_of(*shape)
    assert capi.moe_workspace_size(sh) == 0
    w = capi.moe_weights(1, 1, 1, 1, 1)
    rc = capi.LIB.moe_forward(sh, ctypes.byref(w), 16, 16, 16, None, None, None, 256, 1 << 30, None)
    assert rc == -1  # MOE_ERR_SHAPE


@pytest.mark.parametrize("groups,top", [(3, 1), (8, 3), (64, 4), (4, 8), (8, 0), (32, 2)])
def test_bad_group_shapes_rejected(capi, groups, top):
    # node-limited routing needs N % G == 0, 1 <= M <= G <= 32, K % M == 0 and
    # K / M <= N / G (here N = 64, K = 8; G = 32 leaves 2 experts per group
    # for K / M = 4)
    assert capi.moe_workspace_size(capi.shape_of(64, 256, 64, 8, 128, groups, top)) == 0


@pytest.mark.parametrize("groups,top", [(0, 0), (8, 4), (8, 8), (1, 1), (32, 8), (4, 1)])
def test_group_shapes_accepted(capi, groups, top):
    assert capi.moe_workspace_size(capi.shape_of(64, 256, 64, 8, 128, groups, top)) > 0


def test_balance_stats_rejects_bad_arguments(capi):
    import torch
    sh = capi.shape_of(64, 256, 64, 8, 128)
    need = capi.moe_workspace_size(sh)
    buf = torch.empty(need + 256, dtype=torch.uint8)
    ws = ctypes.c_void_p((buf.data_ptr() + 255) // 256 * 256)   # host memory: never touched
    ids = torch.zeros((64, 8), dtype=torch.int32)
    f = torch.empty((1, 64))
    loss = torch.empty((1,))
    lib = capi.LIB
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    # MOE_ERR_SHAPE = -1, MOE_ERR_NULL = -2, MOE_ERR_WORKSPACE = -6
    assert lib.moe_balance_stats(sh, 0, 1e-4, ws, need, p(ids), p(f), p(f), p(loss), None) == -1
    assert lib.moe_balance_stats(sh, 64, 1e-4, None, need, p(ids), p(f), p(f), p(loss), None) == -2
    assert lib.moe_balance_stats(sh, 64, 1e-4, ws, 16, p(ids), p(f), p(f), p(loss), None) == -6


def test_empty_batch_shape_accepted(capi):
    # T = 0 is an empty batch (no work; counts cleared), not a bad shape
    assert capi.moe_workspace_size(capi.shape_of(0, 7168, 256, 8, 2048)) > 0


def test_null_and_alignment_rejected(capi):
    sh = capi.shape_of(64, 256, 16, 4, 128)
    w = capi.moe_weights(16, 16, 16, 16, 16)
    assert capi.LIB.moe_forward(sh, ctypes.byref(w), None, 16, 16, None, None, None, 256, 1 << 30, None) == -2
    assert capi.LIB.moe_forward(sh, ctypes.byref(w), 16, 16, 16, None, None, None, 128, 1 << 30, None) == -7
    assert capi.LIB.moe_forward(sh, ctypes.byref(w), 16, 16, 16, None, None, None, 256, 1024, None) == -6
    assert capi.LIB.moe_quantize_1x128(16, 4, 100, 16, 16, None) == -1
    assert capi.LIB.moe_quantize_1x128(None, 0, 128, None, None, None) == 0
    assert capi.LIB.moe_quantize_1x128(None, 2, 128, None, None, None) == -2
    assert capi.LIB.moe_quantize_1x128(8, 4, 128, 16, 16, None) == -7
    assert capi.LIB.moe_quantize_128x128(16, 100, 128, 16, 16, None) == -1
    assert capi.LIB.moe_update_bias(None, 16, 16, 4, 2, 0.001, None) == -2
    assert capi.LIB.moe_expert_up(256, 128, 0, 16, 16, 128, 16, 16, 16, 16, 16, 16, None, None) == -1


def test_split_gate_rejects_bad_arguments(capi):
    lib = capi.LIB
    # MOE_ERR_NULL = -2, MOE_ERR_SHAPE = -1, MOE_ERR_ALIGN = -7
    assert lib.moe_split_gate(None, 16, 256, 16, None) == -2
    assert lib.moe_split_gate(16, 16, 256, None, None) == -2
    assert lib.moe_split_gate(16, 0, 256, 16, None) == -1
    assert lib.moe_split_gate(8, 16, 256, 16, None) == -7
    # a misaligned pre-split buffer in the weights is refused before any work
    sh = capi.shape_of(64, 256, 16, 4, 128)
    w = capi.moe_weights(16, 16, 16, 16, 16, 8)
    assert lib.moe_forward(sh, ctypes.byref(w), 16, 16, 16, None, None, None, 256, 1 << 30, None) == -7


def test_split_gate_buffer_size_checked_in_the_binding(capi):
    import torch
    gate_w = torch.zeros(16, 256)
    small = torch.zeros(3 * 16 * 256 - 1, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="gate_split"):
        capi.moe_split_gate(gate_w, small)
    sh = capi.shape_of(64, 256, 16, 4, 128)
    with pytest.raises(ValueError, match="gate_split"):
        capi.moe_ep_dispatch(sh, 1, None, None, None, None, None, None, gate_split=small)
    with pytest.raises(ValueError, match="gate_split"):
        capi.moe_ep_dispatch_peer(sh, 1, 0, 64, None, None, None, None, None, None,
                                  gate_split=small)


def _prototypes():
    """name -> (return type, [parameter declarations]) of every function the
    header declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    out = {}
    for ret, name, params in re.findall(r"\b(int|size_t|int64_t|void)\s+(moe_[a-z0-9_]+)\s*"
                                        r"\(([^)]*)\)\s*;", text):
        ps = [p.strip() for p in params.split(",") if p.strip() and p.strip() != "void"]
        out[name] = (ret, ps)
    return out


def test_binding_signatures_match_the_header(capi):
    """Every prototype of include/moe_capi.h against the ctypes signature the
    binding sets: the same number of parameters, and each of the same kind
    (pointer, 32- or 64-bit integer, size, float, or the shape struct passed
    by value), so no argument can land in another's place."""
    protos = _prototypes()
    assert set(protos) == set(declared_functions())
    assert set(protos) == set(capi.SIGNATURES)
    scalar = {"int32_t": ctypes.c_int32, "int": ctypes.c_int, "int64_t": ctypes.c_int64,
              "size_t": ctypes.c_size_t, "float": ctypes.c_float, "moe_shape": capi.moe_shape}
    rets = {"int": ctypes.c_int, "size_t": ctypes.c_size_t, "int64_t": ctypes.c_int64}
    for name, (ret, params) in protos.items():
        res, args = capi.SIGNATURES[name]
        assert res is rets[ret], name
        assert len(args) == len(params), f"{name}: {len(args)} argtypes, {len(params)} in the header"
        for decl, arg in zip(params, args):
            if "*" in decl:
                # device or host pointers: void* in the binding, or a typed
                # pointer to a struct or pointer array the binding builds
                assert arg is ctypes.c_void_p or issubclass(arg, ctypes._Pointer), (name, decl)
                if "moe_weights" in decl or "moe_ws_layout" in decl:
                    assert issubclass(arg, ctypes._Pointer), (name, decl)
            else:
                ctype = decl.replace("const ", "").split()[0]
                assert arg is scalar[ctype], (name, decl, arg)


def test_product_fails_loudly_without_the_library(tmp_path):
    """With libmoe_b200.so absent, importing the binding, the layer or the
    expert-parallel driver raises ImportError naming the missing library:
    there is no CPU fallback to run instead."""
    import shutil
    import subprocess
    import sys
    pkg = os.path.join(ROOT, "mixture_experts_layer_40_b200")
    shutil.copytree(pkg, tmp_path / "mixture_experts_layer_40_b200",
                    ignore=shutil.ignore_patterns("*.so", "csrc", "__pycache__"))
    for mod in ("capi", "layer", "ep"):
        r = subprocess.run([sys.executable, "-c", f"import mixture_experts_layer_40_b200.{mod}"],
                           cwd=tmp_path, capture_output=True, text=True, timeout=300)
        assert r.returncode != 0, mod
        assert "ImportError" in r.stderr and "no CPU fallback" in r.stderr, (mod, r.stderr[-500:])


def _imports(path):
    """Top-level module names imported anywhere in a Python file, with the
    function each import sits in (None at module level)."""
    import ast
    tree = ast.parse(open(path).read())
    found = []

    def walk(node, fn):
        for child in ast.iter_child_nodes(node):
            name = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else fn
            if isinstance(child, ast.Import):
                found.extend((a.name.split(".")[0], fn) for a in child.names)
            elif isinstance(child, ast.ImportFrom) and child.module and child.level == 0:
                found.append((child.module.split(".")[0], fn))
            walk(child, name)
    walk(tree, None)
    return found


def test_oracle_and_product_are_independent():
    """The product package never imports the oracle and the oracle never
    imports the product; the CUDA sources do not name it. bench.py reaches
    the oracle only from its CPU-baseline helpers (oracle_setup,
    oracle_sample_step), which the reference arm and the cpu_baseline leg
    call; the smoke check imports it inside smoke() only."""
    import glob
    pkg = os.path.join(ROOT, "mixture_experts_layer_40_b200")
    for f in glob.glob(os.path.join(pkg, "*.py")):
        assert all(m != "oracle" for m, _ in _imports(f)), f
    for f in glob.glob(os.path.join(ROOT, "oracle", "*.py")):
        assert all(m != "mixture_experts_layer_40_b200" for m, _ in _imports(f)), f
    for f in glob.glob(os.path.join(pkg, "csrc", "*")) + glob.glob(os.path.join(ROOT, "include", "*")):
        assert "oracle" not in open(f).read().lower(), f
    users = {fn for m, fn in _imports(os.path.join(ROOT, "bench.py")) if m == "oracle"}
    assert users == {"oracle_setup", "oracle_sample_step"}, users
    users = {fn for m, fn in _imports(os.path.join(ROOT, "__graft_entry__.py")) if m == "oracle"}
    assert users == {"smoke"}, users
