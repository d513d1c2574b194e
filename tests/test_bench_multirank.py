"""Host logic of the multi-GPU bench path on CPU: two gloo ranks.

Each rank runs its own replica of the workload (weak scaling, no collective on
the data path); the only collectives are the barrier and the max of the
per-rank timings, and the reported value is all ranks' FLOPs over the slowest
rank's time.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    ms = 10.0 + 5.0 * rank  # rank 1 is the slowest
    mx = bench.reduce_max(ms, dist)
    dist.barrier()
    q.put((rank, mx, bench.aggregate(1e12, mx, world)))
    dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, agg in res:
        assert mx == 15.0
        assert agg == pytest.approx(2e12 / 15e-3 / 1e12)


def test_single_process_reduce_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.5, None) == 3.5
    assert bench.aggregate(5e12, 1000.0, 1) == pytest.approx(5.0)


def test_flop_and_byte_counts_match_the_oracle():
    sys.path.insert(0, ROOT)
    import bench
    import isa_synth
    from oracle import isa_oracle as O
    for w in isa_synth.all_workloads().values():
        f = bench.flops_per_call(w)
        g = O.executed_flops(w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s, w.alpha_f)
        for key in ("coarse", "route", "exact", "taylor", "total"):
            assert f[key] == pytest.approx(g[key], rel=1e-12), (w.name, key)
    w = isa_synth.WORKLOADS["bf16_n32768_b128"]
    hb = bench.hbm_bytes_per_call(w)
    assert hb["pool"] == 3 * 40 * 32768 * 128 * 2
    assert hb["gather"] == 2 * 2 * 40 * 32 * 128 * 128 * 2


def test_roofline_peak_follows_the_timed_region():
    sys.path.insert(0, ROOT)
    import bench
    peaks = {"bf16_tflops": 1659.6, "bf16_tflops_sustained": 1382.4, "hbm_gbs": 6552.6}
    # a 0.1 s timed region sits below the power cap's reaction time: the burst GEMM figure
    assert bench.roofline_peak(peaks, 0.1) == (1659.6, "burst")
    # a seconds-long one runs under the power cap: the sustained figure
    assert bench.roofline_peak(peaks, 1.06) == (1382.4, "sustained")
    assert bench.roofline_peak({"bf16_tflops": 1590.0}, 5.0) == (1590.0, "burst")


def test_weak_scaling_units_differ_per_rank():
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    import isa_synth
    w = isa_synth.Workload("u", 1, 2, 64, 256, 256, 64, 0.5, 0.5, 0.1, 1.0, 0.5, "f32")
    q0 = bench.workload_inputs(w, batch=0)[0]
    q1 = bench.workload_inputs(w, batch=1)[0]
    assert q0.shape == q1.shape == (1, 2, 512, 64)
    assert not np.array_equal(q0, q1)
    # batch element r is the draw of slice (r, h) of the generator
    np.testing.assert_array_equal(q1[0, 1], isa_synth.make_slice(w, 0, 1, 1, 0)[0])


def test_ragged_workload_counts_by_hand():
    sys.path.insert(0, ROOT)
    import bench
    import isa_synth
    from oracle import isa_oracle_ragged as R
    w = isa_synth.RAGGED["bf16_n32800_b128_ragged"]
    assert bench.is_ragged(w) and not bench.is_ragged(isa_synth.WORKLOADS["bf16_n32768_b128"])
    # ceil(16300 / 128) = 128 source and ceil(16500 / 128) = 129 context blocks; k = ceil(0.25 * 129) = 33,
    # n_flat = floor(0.6 * 257) = 154, n_new = 161; every block counts b rows and b keys
    n_q, k, n_flat, n_new = 257, 33, 154, 161
    assert len(R.block_bounds(w.L_src, w.L_ctx, w.b)) == n_q
    f = bench.flops_per_call(w)
    assert f["exact"] == 4.0 * (n_q - n_flat) * 128 * n_new * 128 * 128 * 40
    assert f["taylor"] == 4.0 * n_flat * 128 * n_new * 128 * 40
    assert f["coarse"] == 2.0 * 128 * n_q * 128 * 40 and f["route"] == 2.0 * n_q * n_new * 128 * 40
    hb = bench.hbm_bytes_per_call(w)
    assert hb["pool"] == 3 * 40 * 32800 * 128 * 2 and hb["gather"] == 2 * 2 * 40 * k * 128 * 128 * 2
