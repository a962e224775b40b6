"""The bounds-checked build (libmoe_decode_checked.so, compiled with MOE_BOUNDS_CHECK).

Every global or shared-memory index that the routing schedule produces is range-checked
there before it is used; a failed check reports MOE_ERR_BOUNDS through the device status
and abandons the step without touching the memory. The build stands in for a memory
checker: the parity workloads below must run clean on it (status 0, outputs within the
oracle tolerances) on both kernels and on a layer stack run in one launch, and a schedule
entry pointed one slot row past the schedule (still inside the workspace, so nothing
outside it is read either way) must be reported and leave the handle usable.
"""
import numpy as np
import pytest

import synth

from harness import check_all, gpu_layer_outputs, make_handle, routing_oracle, run_gpu

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

W = synth.Workload
CASES = [
    (W("chk_ragged_b5_k6", B=5, H=1024, E=96, k=6, I=256, Is=512, seed=21), 0),
    (W("chk_corr_2layer", B=8, H=512, E=64, k=4, I=128, Is=256, seed=26, layers=2, rows="correlated",
       nseq=2, rows_per_seq=4), 0),
    (W("chk_tc_b1_k8", B=1, H=512, E=256, k=8, I=256, Is=256, seed=31), 1),
    (W("chk_tc_ragged_b5_e384", B=5, H=1024, E=384, k=6, I=256, Is=512, seed=32), 1),
    (W("chk_tc_b64_k16", B=64, H=512, E=128, k=16, I=128, Is=256, seed=33), 1),
    (W("chk_tc_3layer_b4", B=4, H=512, E=256, k=8, I=128, Is=128, seed=44, layers=3, rows="correlated",
       nseq=1, rows_per_seq=4), 1),
]


@pytest.fixture(autouse=True)
def _cuda_only():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("wl,tc", CASES, ids=[f"{w.name}-{'tc' if t else 'cc'}" for w, t in CASES])
def test_checked_build_runs_the_parity_workloads_clean(wl, tc):
    layers = [wl.device_layer(l) for l in range(wl.layers)]
    h = make_handle(wl, layers, tc_min_batch=tc, checked=True)
    x = wl.x_host()
    out = run_gpu(h, wl, x, n_layers=wl.layers)
    assert out["status"] == 0, f"device status {out['status']}"
    rows = list(range(wl.B))
    mid = gpu_layer_outputs(wl, layers, x, tc_min_batch=tc) if wl.layers > 1 else []
    check_all(wl, out, x, rows, routing_oracle(wl, x, rows, wl.layers, mid), tag=f"checked {wl.name}")
    h.close()


@pytest.mark.parametrize("B", [1, 5])
def test_checked_build_reports_a_slot_row_past_the_schedule(B):
    """Row 0's first choice is pointed at the first slot row past the schedule (the
    one-row schedule at B = 1, the general one at B = 5): the combine's check reports
    MOE_ERR_BOUNDS; the next step on the same handle is clean and correct."""
    import moe_decode_persistent_b200 as mdp

    wl = W("chk_bad_slot", B=B, H=512, E=256, k=8, I=128, Is=128, seed=46)
    layers = [wl.device_layer(0)]
    h = make_handle(wl, layers, tc_min_batch=1, checked=True)
    x = wl.x_host()
    h.set_debug(mdp.DEBUG_BAD_SLOT)
    bad = run_gpu(h, wl, x)
    assert bad["status"] == mdp.MOE_ERR_BOUNDS
    h.set_debug(0)
    out = run_gpu(h, wl, x)
    assert out["status"] == 0
    rows = list(range(B))
    check_all(wl, out, x, rows, routing_oracle(wl, x, rows, 1, []), tag="after the reported step")
    h.close()
