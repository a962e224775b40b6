"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small workloads run the oracle on every row; they span several tiles, K splits
and ragged tails (batch not a multiple of the row group, odd k, k = E, k = 1,
a skewed router, correlated rows, two layers). Both kernels of the batch-shape
switch are checked: the CUDA-core kernel on every workload, the tensor-core kernel
on the workloads whose dimensions are multiples of 128 (half tile pairs, batches
that are not a multiple of 16, hot experts chosen by every row, k = 32, the
largest slot count). The five measured workloads run at full size with the oracle
on sampled rows (rows are independent) plus properties checked on every row.
"""
import dataclasses

import numpy as np
import pytest

import oracle
import synth

from harness import bf, check_all, gpu_layer_outputs, make_handle, routing_oracle, run_gpu

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

W = synth.Workload
SMALL = [
    synth.WORKLOADS[0],
    W("ragged_b5_k6", B=5, H=1024, E=96, k=6, I=256, Is=512, seed=21),
    W("b13_k3", B=13, H=512, E=64, k=3, I=128, Is=256, seed=22),
    W("b64_k16", B=64, H=256, E=64, k=16, I=128, Is=128, seed=23),
    W("k_equals_E", B=2, H=256, E=32, k=32, I=64, Is=64, seed=24),
    W("zipf_b16", B=16, H=512, E=128, k=8, I=256, Is=256, seed=25, router="zipf"),
    W("corr_2layer", B=8, H=512, E=64, k=4, I=128, Is=256, seed=26, layers=2, rows="correlated",
      nseq=2, rows_per_seq=4),
    W("b1_k1", B=1, H=256, E=32, k=1, I=32, Is=32, seed=27),
    W("b7_h2048", B=7, H=2048, E=64, k=5, I=512, Is=768 - 256, seed=28),
]


# tensor-core shapes: every dimension a multiple of 128
TC_SMALL = [
    W("tc_b1_k8", B=1, H=512, E=256, k=8, I=256, Is=256, seed=31),
    W("tc_ragged_b5_e384", B=5, H=1024, E=384, k=6, I=256, Is=512, seed=32),
    W("tc_b64_k16", B=64, H=512, E=128, k=16, I=128, Is=256, seed=33),
    W("tc_zipf_b17", B=17, H=768, E=256, k=8, I=256, Is=512, seed=34, router="zipf"),
    W("tc_half_pairs_b9_h128", B=9, H=128, E=384, k=5, I=128, Is=128, seed=38),
    W("tc_corr_2layer_b32", B=32, H=512, E=256, k=8, I=128, Is=128, seed=35, layers=2, rows="correlated",
      nseq=4, rows_per_seq=8),
    W("tc_k32_b3_h256", B=3, H=256, E=128, k=32, I=128, Is=128, seed=36),
    W("tc_b2_h2048", B=2, H=2048, E=128, k=2, I=512, Is=768, seed=37),
    W("tc_b4_k16_e512", B=4, H=512, E=512, k=16, I=128, Is=128, seed=39),
    # stacks of three layers in one launch: the middle layer both waits for its input
    # rows and counts its output rows; one row (the one-row routing path) and four
    W("tc_3layer_b4", B=4, H=512, E=256, k=8, I=128, Is=128, seed=44, layers=3, rows="correlated",
      nseq=1, rows_per_seq=4),
    W("tc_3layer_b1", B=1, H=512, E=256, k=8, I=256, Is=256, seed=45, layers=3),
]


TC_BY_NAME = {w.name: w for w in TC_SMALL}


def _layers(wl):
    return [wl.device_layer(l) for l in range(wl.layers)]


def _free():
    import gc

    gc.collect()
    torch.cuda.empty_cache()


@pytest.fixture(autouse=True)
def _cuda_only():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    _free()


def run_and_check(wl, rows=None, handle=None, layers=None, tc_min_batch=None):
    layers = layers if layers is not None else _layers(wl)
    h = handle or make_handle(wl, layers, tc_min_batch=tc_min_batch)
    x = wl.x_host()
    out = run_gpu(h, wl, x, n_layers=wl.layers)
    assert out["status"] == 0, f"device status {out['status']}"
    rows = list(range(wl.B)) if rows is None else rows
    mid = gpu_layer_outputs(wl, layers, x, tc_min_batch=_switch_of(h, wl)) if wl.layers > 1 else []
    route = routing_oracle(wl, x, rows, wl.layers, mid)
    err, _ = check_all(wl, out, x, rows, route, tag=wl.name)
    if handle is None:
        h.close()
    return out, err


def _launches(h, wl):
    """Launches one step makes: the tensor-core path runs a stack of layers in one launch,
    the CUDA-core path launches once per layer."""
    import moe_decode_persistent_b200 as mdp

    return 1 if h.step_path(wl.B) == mdp.PATH_TENSOR_CORE else wl.layers


def test_tc_layer_stack_runs_in_one_launch_and_recovers_from_a_timeout():
    """A three-layer stack on the tensor-core path is one launch per step. A step whose
    first normalised row is withheld times out in every CTA (status MOE_ERR_TIMEOUT);
    the counters of every layer are reset by the launch's last CTA, so the next step on
    the same handle is correct."""
    import moe_decode_persistent_b200 as mdp

    wl = TC_BY_NAME["tc_3layer_b4"]
    layers = _layers(wl)
    h = make_handle(wl, layers, tc_min_batch=1)
    assert h.step_path(wl.B) == mdp.PATH_TENSOR_CORE and h.launches_per_step() == 1
    x = wl.x_host()
    h.set_debug(mdp.DEBUG_WITHHOLD_NREADY, wait_ms=300)
    bad = run_gpu(h, wl, x, n_layers=wl.layers)
    assert bad["status"] == mdp.MOE_ERR_TIMEOUT
    h.set_debug(0)
    for _ in range(2):
        run_and_check(wl, handle=h, layers=layers)
    h.close()


def _switch_of(h, wl):
    """tc_min_batch that reproduces the path h takes for wl's batch."""
    import moe_decode_persistent_b200 as mdp

    return 1 if h.step_path(wl.B) == mdp.PATH_TENSOR_CORE else 0


@pytest.mark.parametrize("wl", SMALL, ids=[w.name for w in SMALL])
def test_small_workloads_match_oracle(wl):
    run_and_check(wl)


@pytest.mark.parametrize("path", ["tensor_core", "cuda_core"])
@pytest.mark.parametrize("wl", TC_SMALL, ids=[w.name for w in TC_SMALL])
def test_tc_shaped_workloads_match_oracle_on_both_paths(wl, path):
    import moe_decode_persistent_b200 as mdp

    tc = path == "tensor_core"
    layers = _layers(wl)
    h = make_handle(wl, layers, tc_min_batch=1 if tc else 0)
    assert h.step_path(wl.B) == (mdp.PATH_TENSOR_CORE if tc else mdp.PATH_CUDA_CORE)
    run_and_check(wl, handle=h, layers=layers)
    h.close()


def test_cuda_core_only_shapes_never_take_the_tensor_core_path():
    import moe_decode_persistent_b200 as mdp

    wl = SMALL[3]  # E = 64: not a multiple of 128
    layers = _layers(wl)
    h = make_handle(wl, layers, tc_min_batch=1)
    assert h.step_path(wl.B) == mdp.PATH_CUDA_CORE
    h.close()


@pytest.mark.parametrize("name", ["tc_zipf_b17", "tc_b4_k16_e512", "tc_3layer_b4"])
def test_tc_deterministic_and_jitter_invariant(name):
    """Bitwise the same output under random per-CTA delays: every reduction runs in a
    fixed order whichever CTA finishes last, within a layer and across the layers of a
    stack run in one launch."""
    import moe_decode_persistent_b200 as mdp

    wl = TC_BY_NAME[name]
    layers = _layers(wl)
    h = make_handle(wl, layers, tc_min_batch=1)
    x = wl.x_host()
    a = run_gpu(h, wl, x)
    b = run_gpu(h, wl, x)
    h.set_debug(mdp.DEBUG_JITTER)
    c = run_gpu(h, wl, x)
    h.set_debug(0)
    for o in (a, b, c):
        assert o["status"] == 0
    assert np.array_equal(a["y"], b["y"]) and np.array_equal(a["y"], c["y"])
    assert np.array_equal(a["layers"][0]["logits"], c["layers"][0]["logits"])
    h.close()


def test_tc_timeout_is_reported_and_handle_recovers():
    import moe_decode_persistent_b200 as mdp

    wl = TC_BY_NAME["tc_ragged_b5_e384"]
    layers = _layers(wl)
    h = make_handle(wl, layers, tc_min_batch=1)
    x = wl.x_host()
    h.set_debug(mdp.DEBUG_WITHHOLD_NREADY, wait_ms=300)
    bad = run_gpu(h, wl, x)
    assert bad["status"] == mdp.MOE_ERR_TIMEOUT
    h.set_debug(0)
    good = run_and_check(wl, handle=h, layers=layers)[0]
    assert good["status"] == 0
    h.close()


def test_tc_one_row_steps_never_take_an_earlier_steps_choices():
    """One-row steps read the row's choices from words tagged with the launch's epoch.
    A run of one-row steps on distinct inputs, interleaved with a multi-row step and an
    aborted step, must route every step from its own logits (a stale tag would hand a
    step the previous step's experts)."""
    import moe_decode_persistent_b200 as mdp

    wl = TC_BY_NAME["tc_ragged_b5_e384"]
    layers = _layers(wl)
    h = make_handle(wl, layers, tc_min_batch=1)
    pool = wl.x_pool_host(7)
    plan = [(0, 1), (1, 1), (2, 4), (3, 1), ("abort", 1), (4, 1), (5, 1), (6, 1)]
    prev = None
    changed = 0
    for v, B in plan:
        if v == "abort":
            h.set_debug(mdp.DEBUG_WITHHOLD_NREADY, wait_ms=300)
            bad = run_gpu(h, wl, pool[0][:B])
            h.set_debug(0)
            assert bad["status"] == mdp.MOE_ERR_TIMEOUT
            continue
        x = pool[v][:B].copy()
        assert h.step_path(B) == mdp.PATH_TENSOR_CORE
        out = run_gpu(h, wl, x)
        assert out["status"] == 0, f"input {v}: device status {out['status']}"
        rows = list(range(B))
        check_all(wl, out, x, rows, routing_oracle(wl, x, rows, 1, []), tag=f"input {v}")
        if B == 1:
            chosen = set(out["layers"][0]["idx"][0].tolist())
            changed += prev is not None and chosen != prev
            prev = chosen
    # consecutive one-row steps chose different experts, so a stale read would have shown
    assert changed >= 3
    h.close()


def test_rejected_steps_launch_nothing_and_leave_the_handle_usable():
    """Calls outside the step's contract -- an empty batch, more rows than configured,
    top_k of 0 or above the configured maximum, y aliasing x, an output buffer off
    16-byte alignment -- return MOE_ERR_INVALID_ARG before anything is launched: the
    buffers keep their contents, the device status stays clear and the next step is
    correct."""
    import moe_decode_persistent_b200 as mdp

    wl = TC_BY_NAME["tc_ragged_b5_e384"]
    layers = _layers(wl)
    h = make_handle(wl, layers, tc_min_batch=1)
    x = torch.from_numpy(wl.x_host().view(np.int16)).view(torch.bfloat16).cuda()
    x_before = x.clone()
    y = torch.full_like(x, 7.0)
    y_off = torch.full((x.numel() + 8,), 7.0, dtype=torch.bfloat16, device="cuda")[1:1 + x.numel()].view(x.shape)
    assert y_off.data_ptr() % 16 != 0
    cases = [(x, y, 0, wl.k), (x, y, wl.B + 1, wl.k), (x, y, wl.B, 0), (x, y, wl.B, wl.k + 1),
             (x, x, wl.B, wl.k), (x, y_off, wl.B, wl.k)]
    for xi, yi, B, k in cases:
        with pytest.raises(mdp.MoeDecodeError) as err:
            h.step(xi, yi, B, k)
        assert err.value.code == mdp.MOE_ERR_INVALID_ARG, (B, k)
    torch.cuda.synchronize()
    assert h.status() == 0
    assert torch.equal(x, x_before)
    assert bool((y == 7.0).all()) and bool((y_off == 7.0).all())
    run_and_check(wl, handle=h, layers=layers)
    h.close()


@pytest.mark.parametrize("path", ["tensor_core", "cuda_core"])
def test_nonfinite_input_is_reported_and_handle_recovers(path):
    import moe_decode_persistent_b200 as mdp

    wl = TC_BY_NAME["tc_ragged_b5_e384"]
    layers = _layers(wl)
    h = make_handle(wl, layers, tc_min_batch=1 if path == "tensor_core" else 0)
    x = wl.x_host().copy()
    x[2, 17] = 0x7FC0  # a bf16 NaN: row 2's normalised row and logits become NaN
    bad = run_gpu(h, wl, x)
    assert bad["status"] == mdp.MOE_ERR_NONFINITE
    good = run_and_check(wl, handle=h, layers=layers)[0]
    assert good["status"] == 0
    h.close()


def test_tc_smaller_batch_and_k_than_configured():
    wl = TC_BY_NAME["tc_b64_k16"]
    layers = _layers(wl)
    h = make_handle(wl, layers, tc_min_batch=1)
    for B, k in ((1, 16), (3, 4), (16, 8), (33, 16), (63, 1)):
        sub = dataclasses.replace(wl, B=B, k=k)
        run_and_check(sub, handle=h, layers=layers)
    h.close()


def test_device_generator_matches_host():
    wl = W("gen", B=1, H=512, E=32, k=2, I=128, Is=256, seed=99)
    lay = wl.device_layer(0)
    rng = np.random.default_rng(0)
    for name, kind, numel, sigma, mean in wl.device_specs(0):
        t = lay[name].reshape(-1)
        for start in rng.integers(0, max(1, numel - 300), 3):
            got = t[int(start):int(start) + 300].view(torch.int16).cpu().numpy().view(np.uint16)
            want = synth.fill_host(wl.seed, synth.tensor_id(0, kind), int(start), len(got), sigma, mean)
            assert np.array_equal(got, want), name


def test_bitwise_deterministic_and_jitter_invariant():
    import moe_decode_persistent_b200 as mdp

    wl = SMALL[1]
    layers = _layers(wl)
    h = make_handle(wl, layers)
    x = wl.x_host()
    a = run_gpu(h, wl, x)
    b = run_gpu(h, wl, x)
    h.set_debug(mdp.DEBUG_JITTER)
    c = run_gpu(h, wl, x)
    h.set_debug(0)
    for o in (a, b, c):
        assert o["status"] == 0
    assert np.array_equal(a["y"], b["y"]) and np.array_equal(a["y"], c["y"])
    assert np.array_equal(a["layers"][0]["logits"], c["layers"][0]["logits"])
    h.close()


def test_timeout_is_reported_and_handle_recovers():
    import moe_decode_persistent_b200 as mdp

    wl = SMALL[2]
    layers = _layers(wl)
    h = make_handle(wl, layers)
    x = wl.x_host()
    h.set_debug(mdp.DEBUG_WITHHOLD_NREADY, wait_ms=300)
    bad = run_gpu(h, wl, x)
    assert bad["status"] == mdp.MOE_ERR_TIMEOUT
    h.set_debug(0)
    good = run_and_check(wl, handle=h, layers=layers)[0]
    assert good["status"] == 0
    h.close()


def test_host_entry_point_matches_device_entry_point():
    wl = SMALL[1]
    layers = _layers(wl)
    h = make_handle(wl, layers)
    x = wl.x_host()
    dev = run_gpu(h, wl, x)
    xh = torch.from_numpy(x.view(np.int16)).pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    h.step_host(xh, yh, wl.B, wl.k, stream=torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert h.status() == 0
    assert np.array_equal(yh.numpy().view(np.uint16), dev["y"])
    h.close()


def test_smaller_batch_and_k_than_configured():
    wl = SMALL[1]
    layers = _layers(wl)
    h = make_handle(wl, layers)
    sub = dataclasses.replace(wl, B=3, k=4)
    out, _ = run_and_check(sub, handle=h, layers=layers)
    assert h.launches_per_step() == 1
    h.close()


FULL = [(1, None), (2, None), (3, None), (4, None), (1, 0), (2, 0), (3, 0), (4, 0)]


@pytest.mark.parametrize("cfg,tc_min_batch", FULL,
                         ids=[f"config{c}-" + {None: "switch", 0: "cuda_core", 1: "tensor_core"}[t] for c, t in FULL])
def test_full_size_workload(cfg, tc_min_batch):
    """A measured workload at full size, every row: indices = the oracle's top-k of the
    GPU's own logits, softmax weights, logits against the oracle router (each layer on
    the input it received), and the output of every row against the oracle chain on
    the GPU's selections."""
    wl = synth.WORKLOADS[cfg]
    layers = _layers(wl)
    h = make_handle(wl, layers, tc_min_batch=tc_min_batch)
    x = wl.x_host()
    out = run_gpu(h, wl, x, n_layers=wl.layers)
    assert out["status"] == 0
    assert h.launches_per_step() == _launches(h, wl)
    for l in range(wl.layers):
        np.testing.assert_allclose(out["layers"][l]["w"].sum(axis=1), 1.0, atol=1e-5)
    rows = list(range(wl.B))
    mid = gpu_layer_outputs(wl, layers, x, tc_min_batch=_switch_of(h, wl)) if wl.layers > 1 else []
    route = routing_oracle(wl, x, rows, wl.layers, mid)
    check_all(wl, out, x, rows, route, tag=wl.name)
    h.close()
