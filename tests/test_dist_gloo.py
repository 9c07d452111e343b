"""World-size-2 gloo tests (CPU) of the multi-process host logic: corpus
calibration split over ranks equals calibration of the whole corpus, the
row sharding covers every row exactly once, and the job time is the max over
ranks. The per-rank reduction is the CPU oracle's amax (no GPU here)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world_size, port, results):
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    from w8a8_smoothquant_int8_02_b200 import dist as sqdist, synth, workloads
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world_size,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        case = workloads.TINY
        d = synth.generate(case)
        x_cal = d["x_cal"]  # [16, 64] fp32, channels 3 and 41 are outliers
        # uneven split: 16 tokens over 2 ranks, plus an empty-shard case
        sl = sqdist.shard_rows(x_cal.shape[0], world_size, rank)
        shard = torch.from_numpy(np.ascontiguousarray(x_cal[sl]))
        amax = sqdist.calibrate_activation_amax(
            shard, lambda t: torch.from_numpy(oracle.amax(t.numpy(), True)))
        empty = torch.from_numpy(np.ascontiguousarray(x_cal[:0] if rank == 1 else x_cal))
        amax_e = sqdist.calibrate_activation_amax(
            empty, lambda t: torch.from_numpy(oracle.amax(t.numpy(), True)))
        t = sqdist.max_over_ranks(1.5 + rank)
        results[rank] = (amax.numpy().tobytes(), amax_e.numpy().tobytes(), t, (sl.start, sl.stop))
    finally:
        dist.destroy_process_group()


def test_distributed_calibration_equals_whole_corpus():
    import oracle
    from w8a8_smoothquant_int8_02_b200 import synth, workloads
    world_size = 2
    # the result store runs in a spawned process too: this test process may
    # already have threads (OpenMP in the oracle, torch), and fork would copy
    # them half-way
    manager = mp.get_context("spawn").Manager()
    results = manager.dict()
    port = _free_port()
    mp.spawn(_worker, args=(world_size, port, results), nprocs=world_size, join=True)
    whole = oracle.amax(synth.generate(workloads.TINY)["x_cal"], True)
    spans = []
    for r in range(world_size):
        amax_b, amax_e, t, span = results[r]
        np.testing.assert_array_equal(np.frombuffer(amax_b, np.float32), whole)
        np.testing.assert_array_equal(np.frombuffer(amax_e, np.float32), whole)
        assert t == 2.5
        spans.append(span)
    assert spans[0][0] == 0 and spans[-1][1] == 16 and spans[0][1] == spans[1][0]


@pytest.mark.parametrize("n,w", [(0, 3), (1, 2), (7, 3), (4096, 8), (5, 8)])
def test_shard_rows_partition(n, w):
    from w8a8_smoothquant_int8_02_b200 import dist as sqdist
    covered = []
    sizes = []
    for r in range(w):
        sl = sqdist.shard_rows(n, w, r)
        covered.extend(range(sl.start, sl.stop))
        sizes.append(sl.stop - sl.start)
    assert covered == list(range(n))
    assert max(sizes) - min(sizes) <= 1
