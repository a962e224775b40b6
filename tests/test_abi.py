"""The C-ABI library: it loads, exports every symbol include/moe_decode.h declares,
and rejects bad arguments on the host (no GPU work is launched here)."""
import ctypes
import os

import pytest

import moe_decode_persistent_b200 as mdp


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(mdp.LIB):
        mdp.build()
    return mdp.lib()


def test_exports_every_declared_symbol(L):
    names = mdp.declared_symbols()
    assert len(names) >= 8
    for name in names:
        assert hasattr(L, name), name


def test_bounds_checked_build_exports_the_same_symbols():
    if not os.path.exists(mdp.CHECKED_LIB):
        mdp.build()
    C = mdp.lib(checked=True)
    for name in mdp.declared_symbols():
        assert hasattr(C, name), name
    assert C is not mdp.lib()


def test_strerror_is_distinct_per_code(L):
    codes = [0, -1, -2, -3, -4, -5, -6, -7, -8, -9]
    msgs = [mdp.strerror(c) for c in codes]
    assert len(set(msgs)) == len(codes)
    assert mdp.strerror(-99) == "unknown error"


def _cfg(**kw):
    base = dict(hidden=256, n_experts=64, top_k_max=4, inter=128, shared_inter=128, max_batch=1,
                n_layers=1, eps=1e-6)
    base.update(kw)
    return mdp.Config(**base)


def _weights():
    w = mdp.LayerWeights()
    for name, _ in mdp.LayerWeights._fields_:
        if name != "router_bias":
            setattr(w, name, 0x1000)
    return w


@pytest.mark.parametrize("kw,code", [
    (dict(max_batch=0), mdp.MOE_ERR_INVALID_ARG),
    (dict(max_batch=65), mdp.MOE_ERR_INVALID_ARG),
    (dict(top_k_max=0), mdp.MOE_ERR_INVALID_ARG),
    (dict(top_k_max=33), mdp.MOE_ERR_INVALID_ARG),
    (dict(n_layers=0), mdp.MOE_ERR_INVALID_ARG),
    (dict(hidden=100), mdp.MOE_ERR_UNSUPPORTED_SHAPE),
    (dict(hidden=384), mdp.MOE_ERR_UNSUPPORTED_SHAPE),
    (dict(inter=48), mdp.MOE_ERR_UNSUPPORTED_SHAPE),
    (dict(n_experts=40), mdp.MOE_ERR_UNSUPPORTED_SHAPE),
    (dict(n_experts=2048, top_k_max=4), mdp.MOE_ERR_UNSUPPORTED_SHAPE),
    (dict(max_batch=64, top_k_max=32), mdp.MOE_ERR_UNSUPPORTED_SHAPE),
])
def test_create_rejects_bad_config_before_touching_the_gpu(L, kw, code):
    h = ctypes.c_void_p()
    cfg = _cfg(**kw)
    w = _weights()
    assert L.moe_decode_create(ctypes.byref(cfg), ctypes.byref(w), 0, ctypes.byref(h)) == code
    assert not h.value


def test_create_rejects_null_pointers(L):
    h = ctypes.c_void_p()
    cfg = _cfg()
    assert L.moe_decode_create(None, None, 0, ctypes.byref(h)) == mdp.MOE_ERR_INVALID_ARG
    w = _weights()
    w.w_down = None
    assert L.moe_decode_create(ctypes.byref(cfg), ctypes.byref(w), 0, ctypes.byref(h)) == mdp.MOE_ERR_INVALID_ARG


def test_null_handle_calls_are_rejected(L):
    v = ctypes.c_int(0)
    assert L.moe_decode_step(None, 0x1000, 0x2000, 1, 1, None, None) == mdp.MOE_ERR_INVALID_ARG
    assert L.moe_decode_step_host(None, 0x1000, 0x2000, 1, 1, None, None) == mdp.MOE_ERR_INVALID_ARG
    assert L.moe_decode_get_status(None, ctypes.byref(v)) == mdp.MOE_ERR_INVALID_ARG
    assert L.moe_decode_set_debug(None, 0, 100) == mdp.MOE_ERR_INVALID_ARG
    assert L.moe_decode_launches_per_step(None) == mdp.MOE_ERR_INVALID_ARG
    assert L.moe_decode_set_tc_min_batch(None, 1) == mdp.MOE_ERR_INVALID_ARG
    assert L.moe_decode_step_path(None, 1) == mdp.MOE_ERR_INVALID_ARG
    L.moe_decode_destroy(None)


def test_product_binding_does_not_import_the_oracle():
    import sys
    import subprocess

    code = ("import sys, moe_decode_persistent_b200; "
            "assert 'oracle' not in sys.modules, 'binding imported the oracle'")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    subprocess.run([sys.executable, "-c", code], check=True, cwd=root)
    src = open(os.path.join(root, "moe_decode_persistent_b200", "__init__.py")).read()
    assert "import oracle" not in src and "from oracle" not in src


def test_cuda_sources_and_oracle_share_no_headers():
    """The CUDA path includes only its own headers and the public ABI header; the oracle
    includes only its own header: neither side compiles any of the other's code."""
    import glob
    import re

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    local = re.compile(r'#include\s+"([^"]+)"')
    csrc = glob.glob(os.path.join(root, "moe_decode_persistent_b200", "csrc", "*"))
    for f in csrc:
        for inc in local.findall(open(f).read()):
            assert inc in ("kernel_params.h", "moe_decode.h", "ptx.cuh"), (f, inc)
    for f in glob.glob(os.path.join(root, "oracle", "*.[ch]")):
        for inc in local.findall(open(f).read()):
            assert inc == "moe_oracle.h", (f, inc)


def test_row_buffer_checks_of_the_binding():
    """Tensors passed as x/y must hold bf16 values or their bit patterns, be contiguous,
    sit on the expected device and hold batch x hidden elements; violations fail with
    MOE_ERR_INVALID_ARG before the library is called. Raw pointers pass through."""
    import torch

    check = mdp._check_rows
    bf = torch.zeros((4, 64), dtype=torch.bfloat16)
    for ok in (bf, bf.view(torch.int16), bf.view(torch.uint16), bf[:2], None, 0x1000):
        check(ok, "x", 2, 64, "cpu", "step")
    check(bf, "x", 0, 64, "cpu", "step")  # an empty batch is the library's to reject
    bad = [torch.zeros((4, 64), dtype=torch.float32), torch.zeros((4, 64), dtype=torch.float16),
           torch.zeros((64, 4), dtype=torch.bfloat16).t(), torch.zeros((1, 64), dtype=torch.bfloat16)]
    for t in bad:
        with pytest.raises(mdp.MoeDecodeError) as err:
            check(t, "x", 2, 64, "cpu", "step")
        assert err.value.code == mdp.MOE_ERR_INVALID_ARG
    with pytest.raises(mdp.MoeDecodeError) as err:
        check(bf, "x", 2, 64, "cuda", "step")  # a host tensor where device memory is expected
    assert err.value.code == mdp.MOE_ERR_INVALID_ARG
