"""Head-parallel sharding of the pass over ranks, on CPU with gloo (no GPU).

The (batch, head) slices are independent through every stage, so a pass split
by slice over ranks, each rank computing its contiguous range, followed by an
all-gather of O, must reproduce the one-rank pass exactly. The per-rank compute
here is the CPU oracle on tiny shapes (on a GPU it is the CUDA library); what is
tested is the host logic around it: the slice assignment and the gather.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_attention_isa_b200 import sharding  # noqa: E402

# B=2, H=3: 6 slices, so 4 ranks split them unevenly (2, 2, 1, 1)
SHAPE = dict(B=2, H=3, L_src=256, L_ctx=256, D=64, b=64, alpha_s=0.5, alpha_f=0.5)


@pytest.mark.parametrize("n,world", [(40, 8), (40, 3), (6, 4), (3, 5), (1, 1), (0, 2), (65535, 7)])
def test_slice_ranges_cover_every_slice_once(n, world):
    seen = []
    prev_stop = 0
    for r in range(world):
        a, z = sharding.slice_range(r, world, n)
        assert a == prev_stop and z >= a
        prev_stop = z
        seen += list(range(a, z))
    assert seen == list(range(n))
    counts = sharding.slice_counts(n, world)
    assert sum(counts) == n and max(counts) - min(counts) <= 1


def test_slice_range_rejects_bad_rank():
    with pytest.raises(ValueError):
        sharding.slice_range(2, 2, 10)
    with pytest.raises(ValueError):
        sharding.slice_counts(10, 0)


def _inputs():
    import isa_synth
    w = isa_synth.Workload("shard", SHAPE["B"], SHAPE["H"], SHAPE["D"], SHAPE["L_src"], SHAPE["L_ctx"], SHAPE["b"],
                           SHAPE["alpha_s"], SHAPE["alpha_f"], 0.1, 1.0, 0.5, "f32")
    return isa_synth.make_inputs(w, 3)


def _oracle_compute(q, k, v, out, L_src, L_ctx, b, alpha_s, alpha_f, alpha_ns):
    """Per-rank compute: the CPU oracle on a [1, S, N, D] batch (test stand-in for the CUDA call)."""
    import torch
    from oracle import isa_oracle as O
    r = O.isa_forward_ref(q.numpy(), k.numpy(), v.numpy(), L_src, L_ctx, b, alpha_s, alpha_f, alpha_ns=alpha_ns)
    out.copy_(torch.from_numpy(r["out"]))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, res):
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    from block_sparse_attention_isa_b200 import sharding as S
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    q, k, v = (torch.from_numpy(x.astype(np.float64)) for x in _inputs())
    full = S.forward_sharded(q, k, v, SHAPE["L_src"], SHAPE["L_ctx"], SHAPE["b"], SHAPE["alpha_s"],
                             SHAPE["alpha_f"], compute=_oracle_compute)
    part, rng = S.forward_sharded(q, k, v, SHAPE["L_src"], SHAPE["L_ctx"], SHAPE["b"], SHAPE["alpha_s"],
                                  SHAPE["alpha_f"], gather=False, compute=_oracle_compute)
    res.put((rank, full.numpy(), part.numpy(), rng))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_sharded_pass_equals_one_rank_pass(world):
    from oracle import isa_oracle as O
    q, k, v = _inputs()
    ref = O.isa_forward_ref(q.astype(np.float64), k.astype(np.float64), v.astype(np.float64), SHAPE["L_src"],
                            SHAPE["L_ctx"], SHAPE["b"], SHAPE["alpha_s"], SHAPE["alpha_f"])["out"]
    ctx = mp.get_context("spawn")
    res = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank, args=(r, world, port, res)) for r in range(world)]
    for p in ps:
        p.start()
    got = sorted((res.get(timeout=300) for _ in ps), key=lambda t: t[0])
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    n = SHAPE["B"] * SHAPE["H"]
    flat_ref = ref.reshape(n, *ref.shape[2:])
    covered = []
    for rank, full, part, (a, z) in got:
        # the gathered output is the one-rank output, bit for bit, on every rank
        np.testing.assert_array_equal(full, ref)
        # each rank's own part is its slice range of it
        np.testing.assert_array_equal(part, flat_ref[a:z])
        covered += list(range(a, z))
    assert covered == list(range(n))
