"""Expert parallelism on one GPU: the ranks of an expert-parallel layer run one after
another (each with only its own experts' weights), and their fp32 partial outputs are
summed as the all-reduce would. Each rank's partial is compared with the oracle's part
for that expert range and the sum, rounded by the library's conversion kernel, with the
oracle's layer -- both on the GPU's own selections (a near tie makes another set valid).
Ranks whose range holds none of a row's experts still write that row (x + s on rank 0,
zero elsewhere)."""
import numpy as np
import pytest

import oracle
import synth

from harness import check_y, oracle_rows_selected

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

W = synth.Workload
CASES = [
    (W("ep_b4_e256", B=4, H=512, E=256, k=8, I=256, Is=256, seed=61), 2),
    (W("ep_b4_e256_w3", B=4, H=512, E=256, k=8, I=256, Is=256, seed=61), 3),
    (W("ep_b1_e256", B=1, H=512, E=256, k=8, I=128, Is=128, seed=62), 2),   # the one-row schedule
    (W("ep_b2_k2_e384", B=2, H=256, E=384, k=2, I=128, Is=128, seed=63), 4),  # ranks with no expert
    (W("ep_b16_zipf", B=16, H=512, E=128, k=8, I=128, Is=128, seed=64, router="zipf"), 2),
]


@pytest.fixture(autouse=True)
def _cuda_only():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    import gc

    gc.collect()
    torch.cuda.empty_cache()


def _oracle_part(wl, x, e0, e1, with_rs, sel):
    dims = dict(H=wl.H, E=wl.E, k=wl.k, I=wl.I, Is=wl.Is, eps=wl.eps)
    sg, su, sd = wl.shared_host(0)
    Wt = dict(gamma=wl.gamma_host(0), w_router=wl.w_router_host(0), router_bias=wl.bias_host(0),
              experts={e: wl.expert_host(0, e) for e in np.unique(sel) if e0 <= e < e1},
              ws_gate=sg, ws_up=su, ws_down=sd)
    return oracle.layer_partial(dims, Wt, x, e0, e1, with_rs, selection=sel)


@pytest.mark.parametrize("wl,world", CASES, ids=[f"{w.name}_x{n}" for w, n in CASES])
def test_rank_partials_and_their_sum_match_the_oracle(wl, world):
    import moe_decode_persistent_b200 as mdp
    from moe_decode_persistent_b200 import expert_parallel as ep

    layer = wl.device_layer(0)
    x = wl.x_host()
    B, H, k = wl.B, wl.H, wl.k
    xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    total = torch.zeros((B, H), dtype=torch.float32, device="cuda")
    sels, parts = [], []
    for r in range(world):
        e0, e1 = ep.expert_range(wl.E, world, r)
        h = mdp.MoeDecode(H, wl.E, k, wl.I, wl.Is, B, [ep.local_experts(layer, e0, e1)], eps=wl.eps,
                          expert_range=(e0, e1))
        assert h.step_path(B) == mdp.PATH_TENSOR_CORE
        part = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
        dbg = [dict(logits=torch.zeros((B, wl.E), device="cuda"),
                    topk_idx=torch.full((B, k), -1, dtype=torch.int32, device="cuda"),
                    topk_w=torch.zeros((B, k), device="cuda"),
                    n_unique=torch.zeros(1, dtype=torch.int32, device="cuda"))]
        h.step_partial(xt, part, B, k, residual_shared=ep.adds_residual_shared(r),
                       stream=torch.cuda.current_stream(), debug=dbg)
        torch.cuda.synchronize()
        assert h.status() == 0
        sel = dbg[0]["topk_idx"].cpu().numpy()
        local = np.unique(sel[(sel >= e0) & (sel < e1)])
        assert int(dbg[0]["n_unique"].item()) == len(local), "unique experts scheduled on this rank"
        sels.append(sel)
        parts.append((e0, e1, part.cpu().numpy()))
        total += part
        h.close()
    for s in sels[1:]:
        assert np.array_equal(s, sels[0]), "every rank routes every row the same way"
    sel = sels[0]
    for r, (e0, e1, got) in enumerate(parts):
        assert np.all(np.isfinite(got)), f"rank {r}: a row was not written"
        want = _oracle_part(wl, x, e0, e1, ep.adds_residual_shared(r), sel)
        bar = 2e-3 + 2e-2 * float(np.max(np.abs(want)))
        assert np.max(np.abs(got - want)) <= bar, f"rank {r} [{e0}, {e1}): max |d| {np.max(np.abs(got - want)):.3e}"
    y = torch.empty((B, H), dtype=torch.bfloat16, device="cuda")
    mdp.partial_to_bf16(total, y, 0, torch.cuda.current_stream())
    torch.cuda.synchronize()
    yb = y.view(torch.int16).cpu().numpy().view(np.uint16)
    orc = oracle_rows_selected(wl, x, list(range(B)), [dict(idx=sel)])
    check_y(yb, orc, tag=f"{wl.name} over {world} ranks")


def test_partial_to_bf16_rounds_to_nearest_even():
    import moe_decode_persistent_b200 as mdp

    rng = np.random.default_rng(5)
    v = np.concatenate([rng.standard_normal(4093).astype(np.float32) * 100,
                        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -0.0, 3.0e38], dtype=np.float32)])
    src = torch.from_numpy(v).cuda()
    out = torch.empty(v.size, dtype=torch.bfloat16, device="cuda")
    mdp.partial_to_bf16(src, out, 0)
    torch.cuda.synchronize()
    want = torch.from_numpy(v).to(torch.bfloat16)
    assert torch.equal(out.cpu().view(torch.int16), want.view(torch.int16))


def test_expert_range_handles_reject_bad_ranges_and_multi_layer_partials():
    import moe_decode_persistent_b200 as mdp

    wl = CASES[0][0]
    layer = wl.device_layer(0)
    for e0, e1 in ((0, 0), (5, 3), (0, wl.E + 1), (-1, 4)):
        with pytest.raises(mdp.MoeDecodeError) as e:
            mdp.MoeDecode(wl.H, wl.E, wl.k, wl.I, wl.Is, wl.B, [layer], expert_range=(e0, e1))
        assert e.value.code == mdp.MOE_ERR_INVALID_ARG
    # an expert range needs the tensor-core kernel: every dimension a multiple of 128
    with pytest.raises(mdp.MoeDecodeError) as e:
        mdp.MoeDecode(wl.H, 96, wl.k, wl.I, wl.Is, wl.B, [layer], expert_range=(0, 48))
    assert e.value.code == mdp.MOE_ERR_UNSUPPORTED_SHAPE
    two = mdp.MoeDecode(wl.H, wl.E, wl.k, wl.I, wl.Is, wl.B, [layer, layer])
    x = torch.zeros((wl.B, wl.H), dtype=torch.bfloat16, device="cuda")
    part = torch.zeros((wl.B, wl.H), dtype=torch.float32, device="cuda")
    with pytest.raises(mdp.MoeDecodeError) as e:
        two.step_partial(x, part, wl.B, wl.k)
    assert e.value.code == mdp.MOE_ERR_INVALID_ARG
    two.close()
    fw = synth.Workload("ep_fp8", B=2, H=512, E=128, k=4, I=128, Is=128, seed=65, experts="fp8")
    fl = fw.device_layer_fp8(0)
    hf = mdp.MoeDecode(fw.H, fw.E, fw.k, fw.I, fw.Is, fw.B, [fl], fp8=True)
    x2 = torch.zeros((fw.B, fw.H), dtype=torch.bfloat16, device="cuda")
    p2 = torch.zeros((fw.B, fw.H), dtype=torch.float32, device="cuda")
    with pytest.raises(mdp.MoeDecodeError) as e:  # FP8 handles have no partial step
        hf.step_partial(x2, p2, fw.B, fw.k)
    assert e.value.code == mdp.MOE_ERR_INVALID_ARG
    hf.close()


def test_whole_layer_partial_is_the_step_before_rounding():
    """A whole-layer handle's partial step (every expert, residual and shared expert) is
    the layer's fp32 output: rounded, it is the ordinary step's output bit for bit."""
    import moe_decode_persistent_b200 as mdp

    wl = CASES[0][0]
    layer = wl.device_layer(0)
    h = mdp.MoeDecode(wl.H, wl.E, wl.k, wl.I, wl.Is, wl.B, [layer])
    h.set_tc_min_batch(1)
    x = torch.from_numpy(wl.x_host().view(np.int16)).view(torch.bfloat16).cuda()
    y = torch.empty_like(x)
    h.step(x, y, wl.B, wl.k)
    part = torch.empty((wl.B, wl.H), dtype=torch.float32, device="cuda")
    h.step_partial(x, part, wl.B, wl.k)
    torch.cuda.synchronize()
    assert h.status() == 0
    assert torch.equal(part.to(torch.bfloat16).view(torch.int16), y.view(torch.int16))
    h.close()

