"""Layers with FP8 expert weights (E4M3 codes, one power-of-two scale per 128 x 128
block) on the tensor-core kernel, against the FP8 oracle: the bf16 layer evaluated on the
dequantised weights (value(code) x scale, exactly bf16), so the tolerances are the bf16
path's. The codes stream as one byte each, one 128-column K block per stage, and the
CTA's routing warps turn them, times their block's scale, into the bf16 A operand of
the MMA in tensor memory."""
import numpy as np
import pytest

import synth

from harness import check_all, gpu_layer_outputs, make_handle, routing_oracle, run_gpu

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

W = synth.Workload
CASES = [
    W("fp8_b1_k8", B=1, H=512, E=256, k=8, I=256, Is=256, seed=51, experts="fp8"),
    W("fp8_ragged_b5_e384", B=5, H=1024, E=384, k=6, I=256, Is=512, seed=52, experts="fp8"),
    # H = 128: the down tile pair has one tile; one scale block a row, so the scale groups
    # of consecutive experts share 16-byte groups
    W("fp8_half_pair_b9_h128", B=9, H=128, E=384, k=5, I=256, Is=128, seed=53, experts="fp8"),
    W("fp8_zipf_b64_k16", B=64, H=512, E=128, k=16, I=128, Is=256, seed=54, router="zipf", experts="fp8"),
    W("fp8_2layer_b4", B=4, H=512, E=256, k=8, I=128, Is=128, seed=55, layers=2, rows="correlated", nseq=1,
      rows_per_seq=4, experts="fp8"),
    # coverage codes: each block's codes share one exponent field (all 16 across the
    # blocks, subnormal blocks included), scaled so every code carries full weight
    W("fp8_cover_b4", B=4, H=512, E=128, k=8, I=256, Is=128, seed=56, experts="fp8_cover"),
    # H = I = 128: one scale block a row, so a row's scale sits at any of the 4 places of
    # its 16-byte group
    W("fp8_cover_b3_h128_i128", B=3, H=128, E=256, k=4, I=128, Is=128, seed=57, experts="fp8_cover"),
]


@pytest.fixture(autouse=True)
def _cuda_only():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    import gc

    gc.collect()
    torch.cuda.empty_cache()


def _run_and_check(wl):
    import moe_decode_persistent_b200 as mdp

    layers = [wl.device_layer_fp8(l) for l in range(wl.layers)]
    h = make_handle(wl, layers, fp8=True)
    assert h.step_path(wl.B) == mdp.PATH_TENSOR_CORE
    assert h.launches_per_step() == wl.layers  # an FP8 stack runs one launch per layer
    x = wl.x_host()
    out = run_gpu(h, wl, x, n_layers=wl.layers)
    assert out["status"] == 0, f"device status {out['status']}"
    rows = list(range(wl.B))
    mid = gpu_layer_outputs(wl, layers, x, fp8=True) if wl.layers > 1 else []
    check_all(wl, out, x, rows, routing_oracle(wl, x, rows, wl.layers, mid), tag=wl.name, fp8=True)
    return h, out


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_fp8_workloads_match_oracle(wl):
    h, _ = _run_and_check(wl)
    h.close()


@pytest.mark.parametrize("cfg", sorted(synth.FP8_WORKLOADS))
def test_fp8_full_size_every_row(cfg):
    h, _ = _run_and_check(synth.FP8_WORKLOADS[cfg])
    h.close()


def test_fp8_deterministic_and_jitter_invariant():
    import moe_decode_persistent_b200 as mdp

    wl = CASES[3]
    layers = [wl.device_layer_fp8(0)]
    h = make_handle(wl, layers, fp8=True)
    x = wl.x_host()
    a = run_gpu(h, wl, x)
    h.set_debug(mdp.DEBUG_JITTER)
    b = run_gpu(h, wl, x)
    h.set_debug(0)
    assert a["status"] == 0 and b["status"] == 0
    assert np.array_equal(a["y"], b["y"])
    h.close()


def test_fp8_needs_a_shape_the_tensor_core_kernel_tiles():
    """FP8 experts run on the tensor-core kernel only: 96 experts (not a multiple of 128)
    are refused at create time, before anything is allocated."""
    import moe_decode_persistent_b200 as mdp

    fake = dict(gamma=0x1000, w_router=0x1000, w_gate_q=0x1000, w_gate_scale=0x1000, w_up_q=0x1000,
                w_up_scale=0x1000, w_down_q=0x1000, w_down_scale=0x1000, ws_gate=0x1000, ws_up=0x1000,
                ws_down=0x1000)
    with pytest.raises(mdp.MoeDecodeError) as e:
        mdp.MoeDecode(512, 96, 4, 256, 256, 4, [fake], fp8=True)
    assert e.value.code == mdp.MOE_ERR_UNSUPPORTED_SHAPE


def _dequantised_bf16(layer):
    """bf16 expert weights value(code) x block scale (exact), by torch's float8 decode."""
    out = {}
    for name in ("gate", "up", "down"):
        q, sc = layer[f"w_{name}_q"], layer[f"w_{name}_scale"]
        w = q.view(torch.float8_e4m3fn).float()
        w = w * sc.repeat_interleave(128, dim=1).repeat_interleave(128, dim=2)
        wb = w.to(torch.bfloat16)
        assert torch.equal(wb.float(), w)  # the weights are exactly bf16 values
        out[f"w_{name}"] = wb
    return out


@pytest.mark.parametrize("idx", [0, 5])
def test_fp8_step_is_the_bf16_step_on_the_dequantised_weights_bit_for_bit(idx):
    """An FP8 layer runs the bf16 layer on value(code) x scale: the same kernel path on
    the dequantised bf16 weights gives the same output bits (the MMAs see identical
    operands in the same order), for ordinary and for coverage codes."""
    import moe_decode_persistent_b200 as mdp

    wl = CASES[idx]
    lq = wl.device_layer_fp8(0)
    lb = {k: v for k, v in lq.items() if not k.startswith("w_") or k.startswith(("w_router", "ws_"))}
    lb.update(_dequantised_bf16(lq))
    hq = make_handle(wl, [lq], fp8=True)
    hb = make_handle(wl, [lb], tc_min_batch=1)
    assert hq.step_path(wl.B) == hb.step_path(wl.B) == mdp.PATH_TENSOR_CORE
    x = wl.x_host()
    a, b = run_gpu(hq, wl, x), run_gpu(hb, wl, x)
    assert a["status"] == 0 and b["status"] == 0
    assert np.array_equal(a["y"], b["y"])
    hq.close()
    hb.close()


def test_fp8_scales_outside_the_exact_range_are_refused():
    """Scales must be powers of two in [2^-117, 2^7] and 4-byte aligned: anything else
    is refused at create time (MOE_ERR_INVALID_ARG) instead of giving inexact weights."""
    import moe_decode_persistent_b200 as mdp

    wl = CASES[0]
    base = wl.device_layer_fp8(0)
    for bad in (3.0, 2.0 ** 8, 2.0 ** -118, float("inf"), 0.0):
        lay = dict(base)
        sc = base["w_up_scale"].clone()
        sc.view(-1)[5] = bad
        lay["w_up_scale"] = sc
        with pytest.raises(mdp.MoeDecodeError) as e:
            make_handle(wl, [lay], fp8=True)
        assert e.value.code == mdp.MOE_ERR_INVALID_ARG, bad
    lay = dict(base)
    lay["w_down_scale"] = base["w_down_scale"].data_ptr() + 2  # a float pointer 2 bytes off
    with pytest.raises(mdp.MoeDecodeError) as e:
        make_handle(wl, [lay], fp8=True)
    assert e.value.code == mdp.MOE_ERR_INVALID_ARG
    for edge in (2.0 ** -117, 2.0 ** 7, -(2.0 ** -3)):  # the range's ends and a negative scale pass
        lay = dict(base)
        sc = base["w_gate_scale"].clone()
        sc.view(-1)[0] = edge
        lay["w_gate_scale"] = sc
        make_handle(wl, [lay], fp8=True).close()


def test_fp8_cover_codes_on_the_device_match_the_host_generator():
    wl = CASES[5]
    lay = wl.device_layer_fp8(0)
    for e in (0, 77):
        host = wl.expert_fp8_host(0, e)
        for name in ("gate", "up", "down"):
            assert np.array_equal(lay[f"w_{name}_q"][e].cpu().numpy(), host[name][0])
            assert np.array_equal(lay[f"w_{name}_scale"][e].cpu().numpy(), host[name][1])
