"""Multi-rank host logic on CPU: world size 2 over gloo.

A multi-GPU job runs one process per GPU with no data-path collective (every
(batch, head) pair is independent); these tests run the same helpers bench.py
uses (block_causal_linear_b200.ranks) in two gloo processes:

- head sharding: each rank streams its slice of one problem's heads through
  the oracle (three blocks, commit on each) and the gathered outputs and
  states equal the unsharded run bit for bit;
- weak scaling: the ranks' problems have the same shape and different inputs;
- the collectives of the timing path: MIN over ranks for the step count, MAX
  for the times, and the job throughput from the slowest rank.
"""
import os
import socket
import sys

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


def _worker(rank, world, port, errfile):
    try:
        sys.path.insert(0, ROOT)
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        from datetime import timedelta

        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
        import oracle as orc
        from block_causal_linear_b200 import ranks, synth

        # ---- head sharding of one problem (configuration 1 shape, 6 heads)
        w = synth.WORKLOADS[1].shrink(H=6)
        calls = list(synth.stream(w, "cpu"))
        h0, h1 = ranks.head_slice(w.H, world, rank)
        st = orc.State(w.B, h1 - h0, w.d)
        outs = []
        for (_, _, q, k, v) in calls:
            outs.append(orc.block_forward(q[:, :, h0:h1].contiguous(), k[:, :, h0:h1].contiguous(),
                                          v[:, :, h0:h1].contiguous(), st, commit=True, eps=w.eps))
        mine = {"h": (h0, h1), "out": np.concatenate(outs, 1), "S": st.S.copy(), "Z": st.Z.copy()}
        got = [None] * world
        dist.all_gather_object(got, mine)
        if rank == 0:
            got.sort(key=lambda x: x["h"][0])
            assert got[0]["h"][0] == 0 and got[-1]["h"][1] == w.H
            assert all(a["h"][1] == b["h"][0] for a, b in zip(got, got[1:]))
            full = orc.State(w.B, w.H, w.d)
            ref = np.concatenate([orc.block_forward(q, k, v, full, commit=True, eps=w.eps)
                                  for (_, _, q, k, v) in calls], 1)
            assert np.array_equal(np.concatenate([x["out"] for x in got], 2), ref)
            assert np.array_equal(np.concatenate([x["S"] for x in got], 1), full.S)
            assert np.array_equal(np.concatenate([x["Z"] for x in got], 1), full.Z)

        # ---- weak scaling: same shape, own inputs
        wr = ranks.rank_workload(synth.WORKLOADS[2], rank)
        q = synth.random_qkv(1, 16, 4, 32, seed=wr.seed)[0]
        shapes = [None] * world
        dist.all_gather_object(shapes, ((wr.B, wr.n_total, wr.H, wr.d), wr.seed, q))
        if rank == 0:
            assert len({s[0] for s in shapes}) == 1
            assert len({s[1] for s in shapes}) == world
            assert not torch.equal(shapes[0][2], shapes[1][2])

        # ---- timing collectives
        assert ranks.agree_steps(20 + 7 * rank, dist) == 20
        tmax = ranks.max_over_ranks([1.0 + rank, 10.0 - rank, 0.5], dist)
        assert tmax == [float(world), 10.0, 0.5]
        v = ranks.job_throughput(1000, world, 4, tmax[0])
        assert v == pytest.approx(1000 * world * 4 / (world / 1e3))
        dist.barrier()
        dist.destroy_process_group()
    except BaseException as e:  # report to the parent, which fails the test
        import traceback

        with open(errfile, "a") as f:
            f.write(f"rank {rank}: {e!r}\n{traceback.format_exc()}\n")
        raise


def test_two_ranks_gloo(orc, tmp_path):
    errfile = str(tmp_path / "errors.txt")
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, errfile)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
        p.join()
    err = open(errfile).read() if os.path.exists(errfile) else ""
    assert not alive, "a rank did not finish"
    assert all(p.exitcode == 0 for p in procs), err
    assert not err, err


def test_head_slice_partitions():
    sys.path.insert(0, ROOT)
    from block_causal_linear_b200 import ranks

    for H in (1, 2, 4, 6, 8, 12, 64, 66):
        for world in (1, 2, 3, 4, 8):
            sl = [ranks.head_slice(H, world, r) for r in range(world)]
            assert sl[0][0] == 0 and sl[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(sl, sl[1:]))
            sizes = [b - a for a, b in sl]
            if H % 4 == 0:
                assert all(s % 4 == 0 for s in sizes)
                assert max(sizes) - min(sizes) <= 4
            else:
                assert max(sizes) - min(sizes) <= 1
    assert ranks.head_slice(64, 8, 3) == (24, 32)
    with pytest.raises(ValueError):
        ranks.head_slice(64, 2, 2)


def _split_worker(rank, world, port, errfile):
    """Token split of one block over `world` gloo ranks with oracle steps:
    reduce the slice, all-gather the partial sums in rank order, add them to
    the state in that order, apply the slice's queries."""
    try:
        sys.path.insert(0, ROOT)
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        from datetime import timedelta

        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
        import oracle as orc
        from block_causal_linear_b200 import ranks, synth

        B, N, H, d = 1, 23, 3, 32
        q, k, v = synth.random_qkv(B, N, H, d, seed=17)
        prior = synth.random_qkv(B, 9, H, d, seed=18)
        st = orc.State(B, H, d)
        orc.block_forward(*prior, st, commit=True)
        t0, t1 = ranks.token_slice(N, world, rank)

        def reduce_fn(kk, vv):
            KV, z = orc.block_kv(kk, vv)
            return torch.from_numpy(np.concatenate([KV.reshape(B, H, d * d), z], -1))

        def gather_fn(partial):
            parts = [torch.empty_like(partial) for _ in range(world)]
            dist.all_gather(parts, partial)
            return torch.stack(parts)

        def apply_fn(qq, gathered):
            S, Z = st.S.copy(), st.Z.copy()
            for r in range(world):                       # rank order
                S += gathered[r, :, :, : d * d].numpy().reshape(B, H, d, d)
                Z += gathered[r, :, :, d * d:].numpy()
            st.S, st.Z = S, Z                            # commit
            return orc.apply(qq, S, Z)

        out = ranks.token_split_block(q[:, t0:t1].contiguous(), k[:, t0:t1].contiguous(),
                                      v[:, t0:t1].contiguous(), reduce_fn, gather_fn, apply_fn)
        got = [None] * world
        dist.all_gather_object(got, (t0, out, st.S, st.Z))
        if rank == 0:
            ref_st = orc.State(B, H, d)
            orc.block_forward(*prior, ref_st, commit=True)
            ref = orc.block_forward(q, k, v, ref_st, commit=True)
            got.sort(key=lambda x: x[0])
            assert np.abs(np.concatenate([x[1] for x in got], 1) - ref).max() <= 1e-12 * np.abs(ref).max()
            assert all(np.array_equal(x[2], got[0][2]) and np.array_equal(x[3], got[0][3]) for x in got)
            assert np.abs(got[0][2] - ref_st.S).max() <= 1e-12 * np.abs(ref_st.S).max()
        dist.barrier()
        dist.destroy_process_group()
    except BaseException as e:
        import traceback

        with open(errfile, "a") as f:
            f.write(f"rank {rank}: {e!r}\n{traceback.format_exc()}\n")
        raise


def test_token_split_two_ranks_gloo(orc, tmp_path):
    errfile = str(tmp_path / "errors.txt")
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, errfile)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
        p.join()
    err = open(errfile).read() if os.path.exists(errfile) else ""
    assert not alive, "a rank did not finish"
    assert all(p.exitcode == 0 for p in procs), err


def test_token_slice_partitions():
    sys.path.insert(0, ROOT)
    from block_causal_linear_b200 import ranks

    for N in (0, 1, 7, 100, 8190):
        for world in (1, 2, 3, 8):
            for align in (1, 15, 390):
                sl = [ranks.token_slice(N, world, r, align) for r in range(world)]
                assert sl[0][0] == 0 and sl[-1][1] == N
                assert all(a[1] == b[0] for a, b in zip(sl, sl[1:]))
                assert all(a[0] % align == 0 for a in sl if a[0] < N)


def _split_stream_worker(rank, world, port, errfile):
    """The host logic of `bench.py --shard tokens`: a RoPE stream of 2 blocks x
    2 passes whose blocks are split by frames over 4 ranks, 2 per process
    (ranks.split_call, ranks.split_frame_offsets), with oracle steps and a
    gloo all-gather; every call's outputs, concatenated in rank order, equal
    the oracle's unsplit stream, and all 4 ranks commit the same state."""
    try:
        sys.path.insert(0, ROOT)
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        from datetime import timedelta

        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
        import oracle as orc
        from block_causal_linear_b200 import ranks, synth

        B, H, d, Hg, Wg, F = 1, 2, 32, 3, 5, 4           # 4 frames of 3 x 5 per block
        N, align, R_local = F * Hg * Wg, Hg * Wg, 2
        R = world * R_local
        local = [rank * R_local + j for j in range(R_local)]
        calls = [(blk, p, *synth.random_qkv(B, N, H, d, seed=40 + 2 * blk + p)) for blk in range(2) for p in range(2)]
        states = [orc.State(B, H, d) for _ in local]
        t_next = 0
        mine = []
        for i, (blk, p, q, k, v) in enumerate(calls):
            commit = p == 1
            offs = ranks.split_frame_offsets(t_next, N, R, align)
            sl = [offs[r] for r in local]

            def reduce_fn(j, kk, vv):
                KV, z = orc.block_kv(kk, vv, rope=orc.make_rope(Hg, Wg, t_offset=sl[j][2]))
                return torch.from_numpy(np.concatenate([KV.reshape(B, H, d * d), z], -1))

            def gather_fn(parts):
                stacked = torch.stack(parts)
                every = [torch.empty_like(stacked) for _ in range(world)]
                dist.all_gather(every, stacked)
                return torch.cat(every)                  # global rank order

            def apply_fn(j, qq, gathered):
                st = states[j]
                S, Z = st.S.copy(), st.Z.copy()
                for r in range(R):
                    S += gathered[r, :, :, : d * d].numpy().reshape(B, H, d, d)
                    Z += gathered[r, :, :, d * d:].numpy()
                if commit:
                    st.S, st.Z = S, Z
                return orc.apply(qq, S, Z, rope=orc.make_rope(Hg, Wg, t_offset=sl[j][2]))

            outs = ranks.split_call([q[:, t0:t1].contiguous() for t0, t1, _ in sl],
                                    [(k[:, t0:t1].contiguous(), v[:, t0:t1].contiguous()) for t0, t1, _ in sl],
                                    reduce_fn, gather_fn, apply_fn)
            mine += [(i, local[j], outs[j]) for j in range(R_local)]
            if commit:
                t_next += F
        got = [None] * world
        dist.all_gather_object(got, (mine, [(s.S, s.Z) for s in states]))
        if rank == 0:
            ref_st = orc.State(B, H, d)
            every = [x for g in got for x in g[0]]
            sts = [s for g in got for s in g[1]]
            for i, (blk, p, q, k, v) in enumerate(calls):
                ref = orc.block_forward(q, k, v, ref_st, commit=p == 1, rope=orc.make_rope(Hg, Wg, t_offset=F * blk))
                parts = sorted((r, o) for c, r, o in every if c == i)
                g = np.concatenate([o for _, o in parts], 1)
                assert np.abs(g - ref).max() <= 1e-12 * np.abs(ref).max()
            assert all(np.array_equal(s[0], sts[0][0]) and np.array_equal(s[1], sts[0][1]) for s in sts)
            assert np.abs(sts[0][0] - ref_st.S).max() <= 1e-12 * np.abs(ref_st.S).max()
            assert np.abs(sts[0][1] - ref_st.Z).max() <= 1e-12 * np.abs(ref_st.Z).max()
        dist.barrier()
        dist.destroy_process_group()
    except BaseException as e:
        import traceback

        with open(errfile, "a") as f:
            f.write(f"rank {rank}: {e!r}\n{traceback.format_exc()}\n")
        raise


def test_token_split_stream_four_ranks_on_two_gloo_processes(orc, tmp_path):
    errfile = str(tmp_path / "errors.txt")
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_split_stream_worker, args=(r, world, port, errfile)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
        p.join()
    err = open(errfile).read() if os.path.exists(errfile) else ""
    assert not alive, "a rank did not finish"
    assert all(p.exitcode == 0 for p in procs), err


def test_split_frame_offsets():
    sys.path.insert(0, ROOT)
    from block_causal_linear_b200 import ranks

    offs = ranks.split_frame_offsets(7, 3 * 15, 3, 15)
    assert offs == [(0, 15, 7), (15, 30, 8), (30, 45, 9)]
    offs = ranks.split_frame_offsets(0, 100, 4, 1)
    assert [o[:2] for o in offs] == [(0, 25), (25, 50), (50, 75), (75, 100)] and all(o[2] == o[0] for o in offs)
