"""Expert parallelism on the CPU: the partition of the experts over the ranks and the one
all-reduce per step, with gloo ranks (world sizes 2 and 3) standing in for GPUs and the
oracle's expert-range part standing in for each rank's kernel output. The sum over the
ranks must be the whole layer's unrounded output: every expert counted exactly once, the
residual and shared expert exactly once (rank 0)."""
import datetime
import os
import socket

import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")

from moe_decode_persistent_b200 import expert_parallel as ep  # noqa: E402

LAYER = synth.Workload("ep_tiny", B=5, H=64, E=24, k=6, I=32, Is=48, seed=11)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("E,world", [(896, 1), (896, 2), (896, 3), (896, 8), (24, 5), (7, 7)])
def test_expert_ranges_partition_the_experts_contiguously(E, world):
    ranges = [ep.expert_range(E, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == E
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0
    sizes = [e1 - e0 for e0, e1 in ranges]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    assert [ep.adds_residual_shared(r) for r in range(world)].count(True) == 1


def test_expert_range_rejects_impossible_splits():
    for args in ((4, 5, 0), (8, 2, 2), (8, 0, 0), (8, 2, -1)):
        with pytest.raises(ValueError):
            ep.expert_range(*args)


def test_local_experts_are_views_of_the_rank_range():
    E, I, H = 6, 4, 8
    layer = dict(w_gate=torch.arange(E * I * H).reshape(E, I, H), w_up=torch.zeros(E, I, H),
                 w_down=torch.ones(E, H, I), gamma="g")
    loc = ep.local_experts(layer, 2, 5)
    assert loc["gamma"] == "g" and loc["w_gate"].shape == (3, I, H)
    assert loc["w_gate"].data_ptr() == layer["w_gate"][2].data_ptr() and loc["w_gate"].is_contiguous()
    assert torch.equal(loc["w_gate"][0], layer["w_gate"][2])


def _rank_partial(rank, world):
    dims = dict(H=LAYER.H, E=LAYER.E, k=LAYER.k, I=LAYER.I, Is=LAYER.Is, eps=LAYER.eps)
    e0, e1 = ep.expert_range(LAYER.E, world, rank)
    sg, su, sd = LAYER.shared_host(0)
    W = dict(gamma=LAYER.gamma_host(0), w_router=LAYER.w_router_host(0), router_bias=LAYER.bias_host(0),
             experts={e: LAYER.expert_host(0, e) for e in range(e0, e1)}, ws_gate=sg, ws_up=su, ws_down=sd)
    return oracle.layer_partial(dims, W, LAYER.x_host(), e0, e1, ep.adds_residual_shared(rank))


def _worker(rank, world, port, out_dir):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    part = torch.from_numpy(_rank_partial(rank, world))
    ep.reduce_partials(part)
    np.save(os.path.join(out_dir, f"rank{rank}.npy"), part.numpy())
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_all_reduce_of_the_rank_parts_is_the_layer(tmp_path, world):
    import torch.multiprocessing as mp

    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    dims = dict(H=LAYER.H, E=LAYER.E, k=LAYER.k, I=LAYER.I, Is=LAYER.Is, eps=LAYER.eps)
    sg, su, sd = LAYER.shared_host(0)
    W = dict(gamma=LAYER.gamma_host(0), w_router=LAYER.w_router_host(0), router_bias=LAYER.bias_host(0),
             experts={e: LAYER.expert_host(0, e) for e in range(LAYER.E)}, ws_gate=sg, ws_up=su, ws_down=sd)
    full = oracle.layer(dims, W, LAYER.x_host())["y_pre"]
    for r in range(world):
        got = np.load(tmp_path / f"rank{r}.npy")
        np.testing.assert_allclose(got, full, rtol=1e-12, atol=1e-12)
