"""Host-side multi-process logic on CPU with gloo, world size 2: bench.py's
replica timing (max over ranks, throughput summed over ranks), and the
intra-expert split's exchange (each rank's part of the layer, one all-reduce
of the partial sums, one bf16 round; in fp64 from the oracle's parts, and
through the binding's moe.decode_split with fp32 parts) against the whole
layer's oracle."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    ws, r, local = bench.dist_env()
    assert (ws, r, local) == (world, rank, rank)
    mx = bench.max_over_ranks(10.0 + 5.0 * rank, ws)
    sm = bench.sum_over_ranks(1.0 + rank, ws)
    out[rank] = (mx, sm)
    dist.barrier()
    dist.destroy_process_group()


def test_max_and_sum_over_two_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == (15.0, 3.0)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.sum_over_ranks(3.5, 1) == 3.5


def _split_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    sys.path[:0] = [here, os.path.dirname(here)]
    import numpy as np
    import oracle
    from cases import Layer
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    L = Layer(256, 128, 16, 4, 3, seed=9, device="cpu", shared=True)
    part = torch.from_numpy(L.oracle_part(rank, world)["y64"].copy())
    dist.all_reduce(part, op=dist.ReduceOp.SUM)
    y = np.array([[oracle.bf16_round(v) for v in row] for row in part.numpy()], dtype=np.uint16)
    whole = L.oracle()["y64"]
    ref = np.array([[oracle.bf16_round(v) for v in row] for row in whole], dtype=np.uint16)
    # the binding's own exchange step (moe.decode_split) with the part's
    # kernel replaced by its oracle and the bf16 round done by torch (the
    # ranks here have no GPU)
    from mxfp4_weight_streaming_fp8_b200 import moe

    class OraclePart:
        def decode(self, x, y=None):
            y.copy_(torch.from_numpy(L.oracle_part(rank, world)["y64"]).float())
            return y

    def round_bf16(y32, y=None, stream=None):
        return y.copy_(y32.to(torch.bfloat16))

    moe.round_bf16 = round_bf16
    yb = moe.decode_split(OraclePart(), L.x, y32=torch.empty(L.M, L.H), y=torch.empty(L.M, L.H, dtype=torch.bfloat16))
    ulps = np.abs(yb.view(torch.int16).numpy().astype(np.int32) - ref.view(np.int16).astype(np.int32))
    out[rank] = (bool(np.array_equal(y, ref)), float(np.max(np.abs(part.numpy() - whole))),
                 float(np.abs(whole).max()), int(ulps.max()))
    dist.barrier()
    dist.destroy_process_group()


def test_split_parts_all_reduced_over_two_ranks_match_the_layer():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    for r in range(2):
        same, err, scale, ulps = out[r]
        assert same
        assert err <= 1e-12 * scale
        assert ulps <= 1  # fp32 parts added in fp32, then rounded
