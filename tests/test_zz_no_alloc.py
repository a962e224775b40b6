"""The no-allocation entry point (moe_decode_step_noalloc).

It is for callers that cannot allocate device memory -- code inside a framework or
plugin that owns all device memory, allocator callbacks, processes with a memory
budget fixed up front: the step runs on the library's own built-in scratch array
instead of a handle's workspace. Its output must match the regular entry point's on
the same inputs, on two calls in a row (the second call reuses the scratch the
first one left behind), and the fp64 oracle on every row. This file is collected
last on purpose, and it also passes when run alone.
"""
import numpy as np
import pytest

import synth

from harness import bf, check_all, make_handle, routing_oracle, run_gpu

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

W = synth.Workload
CASES = [
    W("noalloc_b3", B=3, H=1024, E=96, k=6, I=256, Is=512, seed=41),
    # the largest batch and top-k the scratch is sized for (its worst-case unit and tile counts)
    W("noalloc_b4_k16", B=4, H=1024, E=96, k=16, I=256, Is=512, seed=42),
    # two layers: the shared layer-to-layer buffer, the next layer's prefetch, counters reused
    W("noalloc_2layer_b4", B=4, H=512, E=64, k=4, I=128, Is=256, seed=43, layers=2, rows="correlated",
      nseq=1, rows_per_seq=4),
    synth.WORKLOADS[1],
]


def _noalloc(wl, layers, x_bits, B=None):
    import moe_decode_persistent_b200 as mdp

    B = B or wl.B
    x = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).cuda()
    y = torch.full_like(x, float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mdp.step_noalloc(wl.H, wl.E, wl.I, wl.Is, layers, x, y, B, wl.k, eps=wl.eps,
                     stream=torch.cuda.current_stream(), device_status=status)
    torch.cuda.synchronize()
    return y.view(torch.int16).cpu().numpy().view(np.uint16), int(status.item())


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_noalloc_matches_regular_entry_point_twice_and_the_oracle(wl):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    layers = [wl.device_layer(l) for l in range(wl.layers)]
    h = make_handle(wl, layers, tc_min_batch=0)            # the kernel the no-allocation step runs
    xs = [wl.x_host(), wl.x_pool_host(2)[1]]
    for x_bits in xs:                                      # two calls in a row
        ref = run_gpu(h, wl, x_bits, n_layers=wl.layers)
        assert ref["status"] == 0
        got, status = _noalloc(wl, layers, x_bits)
        assert status == 0
        # same tolerance as the parity tests' tight bound (one bf16 step + 1e-3)
        d = np.abs(bf(got) - bf(ref["y"]))
        assert np.all(np.isfinite(bf(got)))
        ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(bf(ref["y"])), 2.0 ** -126))) - 7)
        assert np.all(d <= ulp + 1e-3)
        # and every row against the oracle, on the routing the regular step chose (the two
        # entry points run the same kernel: their selections are the same)
        rows = list(range(wl.B))
        mid = []
        if wl.layers > 1:
            h1 = make_handle(wl, layers[:1], tc_min_batch=0)
            mid = [run_gpu(h1, wl, x_bits)["y"]]
            h1.close()
        route = routing_oracle(wl, x_bits, rows, wl.layers, mid)
        ref_as_noalloc = dict(ref, y=got)
        check_all(wl, ref_as_noalloc, x_bits, rows, route, tag=f"noalloc {wl.name}")
    h.close()


def test_noalloc_rejects_sizes_beyond_its_limits_and_a_missing_status():
    import moe_decode_persistent_b200 as mdp

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wl = synth.WORKLOADS[2]                                # batch 8 > 4
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(mdp.MoeDecodeError) as e:
        mdp.step_noalloc(wl.H, wl.E, wl.I, wl.Is, [dict(gamma=0x1000)], 0x1000, 0x2000, wl.B, wl.k,
                         device_status=status)
    assert e.value.code == mdp.MOE_ERR_UNSUPPORTED_SHAPE
    small = CASES[0]
    with pytest.raises(mdp.MoeDecodeError) as e:             # a third layer
        mdp.step_noalloc(small.H, small.E, small.I, small.Is, [dict(gamma=0x1000)] * 3, 0x1000, 0x2000,
                         small.B, small.k, device_status=status)
    assert e.value.code == mdp.MOE_ERR_UNSUPPORTED_SHAPE
    layers = [small.device_layer(0)]
    x = torch.zeros((small.B, small.H), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros_like(x)
    with pytest.raises(mdp.MoeDecodeError) as e:             # no status word
        mdp.step_noalloc(small.H, small.E, small.I, small.Is, layers, x, y, small.B, small.k)
    assert e.value.code == mdp.MOE_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert int(status.item()) == 0
