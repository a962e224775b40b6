"""The no-allocation entry point (moe_decode_step_noalloc).

It is for callers that cannot allocate device memory: the step runs on the
library's own built-in scratch array instead of a handle's workspace. Its output
must match the regular entry point's on the same inputs, on two calls in a row
(the second call reuses the scratch the first one left behind). This file is
collected last on purpose, and it also passes when run alone.
"""
import numpy as np
import pytest

import synth

from harness import bf, make_handle, run_gpu

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wl", [
    synth.Workload("noalloc_b3", B=3, H=1024, E=96, k=6, I=256, Is=512, seed=41),
    synth.WORKLOADS[1],
], ids=["small_b3", "b1_h7168_e896_k16"])
def test_noalloc_matches_regular_entry_point_twice(wl):
    import moe_decode_persistent_b200 as mdp

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    layers = [wl.device_layer(l) for l in range(wl.layers)]
    h = make_handle(wl, layers)
    xs = [wl.x_host(), wl.x_pool_host(2)[1]]
    for x_bits in xs:                                    # two calls in a row
        ref = run_gpu(h, wl, x_bits)["y"]
        x = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).cuda()
        y = torch.full_like(x, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        mdp.step_noalloc(wl.H, wl.E, wl.I, wl.Is, layers, x, y, wl.B, wl.k, eps=wl.eps,
                         stream=torch.cuda.current_stream(), device_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        got = y.view(torch.int16).cpu().numpy().view(np.uint16)
        # same tolerance as the parity tests' tight bound (one bf16 step + 1e-3)
        d = np.abs(bf(got) - bf(ref))
        assert np.all(np.isfinite(bf(got)))
        ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(bf(ref)), 2.0 ** -126))) - 7)
        assert np.all(d <= ulp + 1e-3)
    h.close()


def test_noalloc_rejects_sizes_beyond_its_limits():
    import moe_decode_persistent_b200 as mdp

    wl = synth.WORKLOADS[2]                               # batch 8 > 4
    with pytest.raises(mdp.MoeDecodeError) as e:
        mdp.step_noalloc(wl.H, wl.E, wl.I, wl.Is, [dict(gamma=0x1000)], 0x1000, 0x2000, wl.B, wl.k)
    assert e.value.code == mdp.MOE_ERR_UNSUPPORTED_SHAPE
