"""The N > 1 host logic on CPU ranks (gloo).

* bench.py's timing: the job time is the slowest rank's, and with one
  independent call per rank the job's ms per call is that time divided by the
  calls all ranks made.
* Head sharding: the library's partition (svg_head_shard) covers every head
  exactly once, and the binding's all-gather (gather_heads) assembles the
  ranks' blocks into the single-rank result of the whole call; gather_output
  does the same for outputs in the [B, L, H, d] layout, whose head blocks are
  not contiguous.
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
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.argv = ["bench.py"]
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_step_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        bench.barrier(world)
        out[rank] = (bench.max_over_ranks(local_step_ms, world), bench.job_ms_per_call(local_step_ms, world))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_and_weak_scaling():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(world):
        slowest, per_call = res[r]
        assert slowest == pytest.approx(15.0)
        assert per_call == pytest.approx(7.5)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    sys.argv = ["bench.py"]
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.job_ms_per_call(3.25, 1) == 3.25


# ---------------------------------------------------------------- head sharding

def test_head_shards_cover_every_head_exactly_once():
    """The library's head partition: contiguous blocks in rank order that
    cover 0 .. n-1 exactly once, sizes differing by at most one."""
    sys.path.insert(0, ROOT)
    from sparse_attention_video_profile_b200 import svg
    for n in (0, 1, 2, 7, 24, 48, 100):
        for world in (1, 2, 3, 4, 8, 16):
            seen = []
            sizes = []
            for r in range(world):
                first, count = svg.svg_head_shard(n, r, world)
                assert first == len(seen)
                seen.extend(range(first, first + count))
                sizes.append(count)
            assert seen == list(range(n))
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(svg.SvgError):
        svg.svg_head_shard(4, 2, 2)


def _shard_worker(rank, world, port, out):
    """One rank of a head-sharded call on CPU: the rank computes its block of
    heads with the fp64 oracle (a host stand-in for the GPU call, used only as
    the checker's reference), writes it into full-size tensors and fills the
    other ranks' blocks with the binding's all-gather (gloo)."""
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from sparse_attention_video_profile_b200 import svg, synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl = synth.WORKLOADS["small"]
        q, k, v = synth.make_qkv(wl, seed=7, device="cpu")
        rows = synth.sample_rows(wl.L, wl.S, 7)
        qn, kn, vn = (t.double().numpy() for t in (q, k, v))
        n = wl.B * wl.H
        first, count = svg.svg_head_shard(n, rank, world)
        o = torch.zeros(wl.B, wl.H, wl.L, wl.d, dtype=torch.float64)
        mse = torch.zeros(wl.B, wl.H, 2, dtype=torch.float64)
        label = torch.full((wl.B, wl.H), -1, dtype=torch.int8)
        blk = slice(first, first + count)
        bq, bk, bv = (x.reshape(n, wl.L, wl.d)[blk][None] for x in (qn, kn, vn))
        m, lab = oracle.profile_heads(bq, bk, bv, wl.N, wl.F, wl.a1, wl.a2, rows)
        ob = oracle.sparse_attention(bq, bk, bv, lab, wl.N, wl.F, wl.a1, wl.a2)
        o.view(n, wl.L, wl.d)[blk] = torch.from_numpy(ob[0])
        mse.view(n, 2)[blk] = torch.from_numpy(m[0])
        label.view(n)[blk] = torch.from_numpy(lab[0].astype(np.int8))
        for t in (o, mse, label):
            svg.gather_heads(t, n, rank, world)
        out[rank] = (o.numpy(), mse.numpy(), label.numpy(), (first, count))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_head_sharded_call_assembles_the_single_rank_result(world):
    import numpy as np
    sys.path.insert(0, ROOT)
    import oracle
    from sparse_attention_video_profile_b200 import synth
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_shard_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(300)
            assert p.exitcode == 0
        res = dict(out)
    wl = synth.WORKLOADS["small"]
    q, k, v = synth.make_qkv(wl, seed=7, device="cpu")
    qn, kn, vn = (t.double().numpy() for t in (q, k, v))
    rows = synth.sample_rows(wl.L, wl.S, 7)
    ref_mse, ref_label = oracle.profile_heads(qn, kn, vn, wl.N, wl.F, wl.a1, wl.a2, rows)
    ref_o = oracle.sparse_attention(qn, kn, vn, ref_label, wl.N, wl.F, wl.a1, wl.a2)
    blocks = sorted(res[r][3] for r in range(world))
    assert [f for f, _ in blocks] == list(np.cumsum([0] + [c for _, c in blocks])[:-1])
    assert sum(c for _, c in blocks) == wl.B * wl.H
    for r in range(world):
        o, mse, label, _ = res[r]
        np.testing.assert_array_equal(label, ref_label)
        np.testing.assert_array_equal(mse, ref_mse)
        np.testing.assert_array_equal(o, ref_o)


def _layout_gather_worker(rank, world, port, out):
    """Each rank writes only its own block of heads of a [B, L, H, d] output
    (value = a code of (b, h, x, c)) and gathers the rest."""
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from sparse_attention_video_profile_b200 import svg
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        B, H, L, d = 2, 3, 5, 4
        code = torch.arange(B * H * L * d, dtype=torch.float32).view(B, H, L, d).transpose(1, 2).contiguous()
        o = torch.full_like(code, -1.0)
        first, count = svg.svg_head_shard(B * H, rank, world)
        for g in range(first, first + count):
            o[g // H, :, g % H] = code[g // H, :, g % H]
        svg.gather_output(o, B * H, rank, world, "blhd")
        out[rank] = bool(torch.equal(o, code))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gather_output_blhd(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_layout_gather_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(300)
            assert p.exitcode == 0
        res = dict(out)
    assert all(res[r] for r in range(world))
