"""Data-parallel layer (token-sharded H, one all-reduce, row-sharded sweep): host logic on CPU.

The shard plan, the H all-reduce and the row gather of post_weight_quantization_18_b200.sharded
run here on gloo ranks with the oracle standing in for the per-rank arithmetic, and must give
what one process gives on the whole layer: H to rounding (the sum is regrouped by rank), and,
from the same H, bit-identical packed words and fp16 parameters (rows are independent given U).
"""
import datetime
import os
import queue
import socket
import time

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs(n, d, N, seed):
    import layer_inputs as li
    X = li.activations(N, d, chan_sigma=1.0, outlier_frac=0.01, outlier_mult=20.0,
                       dtype=torch.float32, seed=seed).numpy().astype(np.float64)
    W = li.weight(n, d, 0.02, torch.float32, seed=seed + 1).numpy().astype(np.float64)
    return W, X


def test_split_range_partitions():
    from post_weight_quantization_18_b200.sharded import split_range
    for total in (0, 1, 15, 16, 17, 100, 1000, 4097):
        for world in (1, 2, 3, 7, 8):
            for align in (1, 16):
                parts = [split_range(total, world, r, align) for r in range(world)]
                assert parts[0][0] == 0 and parts[-1][1] == total
                for (a0, b0), (a1, b1) in zip(parts, parts[1:]):
                    assert b0 == a1
                units = [-(-(b - a) // align) for a, b in parts]
                assert max(units) - min(units) <= 1
                for a, b in parts:
                    assert a <= b and (a % align == 0 or a == total)
                    assert (b - a) % align == 0 or b == total


def test_plan_rejects_rankless_rows():
    from post_weight_quantization_18_b200.sharded import plan
    with pytest.raises(ValueError):
        plan(1000, 32, 3, 0)           # 32 rows in 16-row shares cannot feed 3 ranks
    p = plan(1000, 33, 3, 2)
    assert p.rows == (32, 33) and p.max_rows == 16


def _worker(rank, world, port, q, case):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    from oracle import hessian as oh, layer as ol, pack as opk
    from post_weight_quantization_18_b200 import sharded as sh
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        n, d, N, bits, g, act = case
        W, X = _inputs(n, d, N, seed=77)
        p = sh.plan(N, n, world, rank)
        t0, t1 = p.tokens
        r0, r1 = p.rows
        # Per-rank partial H: upper triangle only, the lower triangle left at zero.
        H = torch.from_numpy(np.triu(oh.hessian(X[t0:t1])) if t1 > t0 else np.zeros((d, d)))
        sh.allreduce_hessian(H)
        Hu = H.numpy()
        Hs = np.triu(Hu) + np.triu(Hu, 1).T
        # Row-sharded sweep from the reduced H (the column-by-column route: per-row arithmetic).
        res = ol.gptq_layer(W[r0:r1], Hs, bits=bits, group_size=g, act_order=act, route="chol")
        words, s16, z16 = opk.pack(res["codes"], res["S"], res["Z"], bits)
        got = [sh.gather_rows(torch.from_numpy(np.ascontiguousarray(a).view(dt)), p)
               for a, dt in ((words, np.int32), (s16, np.float16), (z16, np.float16))]
        q.put((rank, Hu, Hs, [t.numpy() for t in got]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [
    (2, (48, 256, 1000, 4, 128, False)),   # ragged token split (1000 = 62.5 units of 16)
    (3, (40, 128, 24, 3, 64, True)),       # rank 2 without tokens, act-order, 3-bit, 16/16/8 rows
])
def test_sharded_layer_matches_one_process(world, case):
    from oracle import hessian as oh, layer as ol, pack as opk
    n, d, N, bits, g, act = case
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, case)) for r in range(world)]
    for p in procs:
        p.start()
    res = []
    deadline = time.monotonic() + 300
    while len(res) < world:
        try:
            res.append(q.get(timeout=1))
        except queue.Empty:
            failed = [p.exitcode for p in procs if p.exitcode not in (None, 0)]
            assert not failed and time.monotonic() < deadline, f"worker exit codes {failed}"
    res.sort(key=lambda r: r[0])
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    W, X = _inputs(n, d, N, seed=77)
    H_full = oh.hessian(X)
    iu = np.triu_indices(d)
    for rank, Hu, Hs, got in res:
        # Every rank holds the same reduced H (bit for bit), equal to the whole H to rounding,
        # with a zero lower triangle.
        np.testing.assert_array_equal(Hu, res[0][1])
        assert np.all(np.tril(Hu, -1) == 0)
        rel = np.abs(Hu[iu] - H_full[iu]).max() / np.abs(H_full).max()
        assert rel <= 1e-13, rel
    # From that H, the gathered packed layer equals one process on all rows.
    ref = ol.gptq_layer(W, res[0][2], bits=bits, group_size=g, act_order=act, route="chol")
    words, s16, z16 = opk.pack(ref["codes"], ref["S"], ref["Z"], bits)
    for rank, _, _, got in res:
        np.testing.assert_array_equal(got[0].view(np.uint32), words)
        np.testing.assert_array_equal(got[1].view(np.uint16), s16)
        np.testing.assert_array_equal(got[2].view(np.uint16), z16)


def _gpu_worker(port, q, case):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    import post_weight_quantization_18_b200 as G
    from post_weight_quantization_18_b200 import sharded as sh
    from gpu_util import make_inputs
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        n, d, N, bits, g, act = case
        W, X = make_inputs(n, d, N, seed=123)
        Wd, Xd = W.cuda(), X.cuda()
        p = sh.plan(N, n, 1, 0)
        out, (qw, s16, z16) = sh.quantize_layer_sharded(Wd, Xd, p, bits=bits, group_size=g,
                                                        act_order=act, gather=True)
        ref = G.quantize_layer(Wd, X=Xd, bits=bits, group_size=g, act_order=act)
        rq, rs, rz = ref.pack()
        torch.cuda.synchronize()
        same = [torch.equal(out.codes, ref.codes), torch.equal(out.perm, ref.perm),
                torch.equal(out.g_idx, ref.g_idx), torch.equal(qw, rq),
                torch.equal(s16.view(torch.int16), rs.view(torch.int16)),
                torch.equal(z16.view(torch.int16), rz.view(torch.int16))]
        q.put(same)
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_sharded_layer_on_one_gpu_matches_quantize_layer():
    """The sharded driver as a one-rank NCCL group on the GPU: the collectives and the gather
    around the library calls leave the single-process result unchanged, bit for bit."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    proc = ctx.Process(target=_gpu_worker, args=(_free_port(), q, (384, 1024, 3000, 4, 128, True)))
    proc.start()
    try:
        same = q.get(timeout=240)
    finally:
        proc.join(60)
        if proc.is_alive():
            proc.kill()
    assert proc.exitcode == 0
    assert same == [True] * 6, same
