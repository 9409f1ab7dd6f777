"""The per-rank bucket step (ShardedBucket) with real processes on CPU.

Each rank: its own gradients into the full bucket -> reduce-scatter (gloo,
sum) into its slice -> step of the slice alone -> all-gather of the bf16
slices.  The slice bucket is stepped by the oracle here (there is no GPU),
so this checks the collective plumbing and the per-rank layout around the
step: every rank must end with the whole-bucket oracle step's bf16 bucket,
and rank r with slice r of its master weights, codes and scales.  The
clipped step (step_clipped: slice norms, all-reduce of their squares) must
give the whole bucket's norm and its clipped step.

Gradients are small multiples of 2^-8 (at most 64 in size), so their sum
over up to four ranks is exact in bf16 whatever order the reduction takes.
"""
import datetime
import os
import socket
import time

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

CASES = {
    # W[512,256] in 16-row blocks, bias and norm as one block each
    "tiny": ([512, 512, 256], [256, 1, 1], [16, 512, 256], [0, 0, 0]),
    # 2-D blocks cut by slice boundaries, a short last block, a 1-D tensor
    "tiles": ([96, 40, 100, 5], [64, 32, 32, 16], [8, 4, 16, 5], [16, 16, 0, 0]),
    # one tensor that leaves most slices empty
    "empty": ([1000, 48], [1, 16], [1000, 48], [0, 0]),
}
STEPS = 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _hp(t):
    return dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, step=t)


def _master(rows, cols):
    rng = np.random.default_rng(7)
    return [rng.normal(0.0, 0.02, size=(r, c)).astype(np.float32) for r, c in zip(rows, cols)]


def _grad(rows, cols, rank, t):
    """Rank `rank`'s gradients at step t (float32, exact in bf16)."""
    rng = np.random.default_rng(1000 * t + rank)
    return [(rng.integers(-64, 65, size=(r, c)) * 2.0 ** -8).astype(np.float32) for r, c in zip(rows, cols)]


def _bf16_bits(x):
    bits = np.ascontiguousarray(x, np.float32).view(np.uint32)
    assert not np.any(bits & 0xFFFF), "value not exact in bf16"
    return (bits >> 16).astype(np.uint16)


class OracleSlice:
    """The slice bucket of one rank, held and stepped by the oracle."""

    def __init__(self, rk):
        import oracle
        self.rk = rk
        self.b = oracle.Bucket(rk["rows"], rk["cols"], rk["k"], rk["offsets"], rk["s"], 1,
                               block_cols=rk["block_cols"])
        self.stream = None

    def array(self, which):
        a = {0: self.b.p, 1: self.b.pb, 2: self.b.g, 3: self.b.mq, 4: self.b.vq}[which]
        t = torch.from_numpy(a)
        return t.view(torch.int16).view(torch.bfloat16) if a.dtype == np.uint16 else t

    def views(self, which):
        flat = self.array(which)
        return [flat[int(o):int(o) + int(r * c)].view(int(r), int(c))
                for r, c, o in zip(self.rk["rows"], self.rk["cols"], self.rk["offsets"])]

    def step(self, hp, grad_scale):
        self.b.step(hp, hp["step"], grad_scale)

    def grad_norm(self, grad_scale, out):
        import oracle
        out[0] = oracle.grad_norm(self.b.g, grad_scale)


def _worker(rank, world, port, case, outdir, max_norm=None):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import ragged_bucket_layout_b200 as rb
        from ragged_bucket_layout_b200.sharded import ShardedBucket

        rows, cols, k, bc = CASES[case]
        plan = rb.dbuf_plan(rows, cols, k, world, 16, block_cols=bc)
        info = rb.dbuf_plan_info(plan)
        local = OracleSlice(oracle.rank_bucket(rows, cols, k, info["offsets"], info["slice"], world, rank, bc))
        sb = ShardedBucket(plan, local=local)
        assert (sb.rank, sb.world) == (rank, world)
        full = _master(rows, cols)
        for i, a, b, v in sb.local_views(rb.DBUF_MASTER_F32):
            v.copy_(torch.from_numpy(full[i][a:b]))
        norms = []
        for t in range(1, STEPS + 1):
            for g, x in zip(sb.grad_views(), _grad(rows, cols, rank, t)):
                g.copy_(torch.from_numpy(x))
            if max_norm is None:
                work = sb.step(_hp(t), async_op=(t == STEPS))
            else:
                norm, work = sb.step_clipped(_hp(t), max_norm, async_op=(t == STEPS))
                norms.append(norm)
            if work is not None:
                work.wait()
        np.savez(os.path.join(outdir, f"rank{rank}.npz"), param=sb.param.view(torch.int16).numpy(), norms=norms,
                 p=local.b.p, mq=local.b.mq, vq=local.b.vq, sm=local.b.scale_m, sv=local.b.scale_v,
                 first_block=sb.rank_plan.first_block, n=sb.rank_plan.n)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case,world,max_norm", [("tiny", 2, None), ("tiny", 4, None), ("tiles", 2, None),
                                                  ("tiles", 4, None), ("empty", 4, None), ("tiny", 4, 1.0),
                                                  ("tiles", 2, 1e3)])
def test_sharded_step_equals_the_whole_bucket(case, world, max_norm, tmp_path):
    """max_norm set: the clipped step (global norm over all ranks' slices);
    1.0 clips every step, 1e3 none."""
    import oracle

    mp.start_processes(_worker, args=(world, _free_port(), case, str(tmp_path), max_norm), nprocs=world,
                       join=True, start_method="spawn")
    rows, cols, k, bc = CASES[case]
    st, off, s = oracle.plan(rows, cols, k, world, 16)
    assert st == 0
    W = oracle.Bucket(rows, cols, k, off, s, world, block_cols=bc)
    for i, x in enumerate(_master(rows, cols)):
        W.p[W.tensor_slice(i)] = x.ravel()
    want_norms = []
    for t in range(1, STEPS + 1):
        per_rank = [_grad(rows, cols, r, t) for r in range(world)]
        for i in range(len(rows)):
            W.g[W.tensor_slice(i)] = _bf16_bits(sum(g[i] for g in per_rank).ravel())
        gs = 1.0 / world
        if max_norm is not None:
            norm = oracle.grad_norm(W.g, gs)
            want_norms.append(norm)
            gs = oracle.clipped_scale(norm, gs, max_norm)
            assert (gs < np.float32(1.0 / world)) == (max_norm == 1.0)
        W.step(_hp(t), t, gs)
    parts = 0
    for r in range(world):
        got = np.load(tmp_path / f"rank{r}.npz")
        sl = slice(r * s, (r + 1) * s)
        assert np.array_equal(got["param"].view(np.uint16), W.pb), f"rank {r}: gathered bf16 bucket"
        assert np.array_equal(got["p"].view(np.uint32), W.p[sl].view(np.uint32)), f"rank {r}: master"
        assert np.array_equal(got["mq"], W.mq[sl]) and np.array_equal(got["vq"], W.vq[sl]), f"rank {r}: codes"
        fb, nb = int(got["first_block"]), got["sm"].size
        assert np.array_equal(got["sm"], W.scale_m[fb:fb + nb]) and np.array_equal(got["sv"], W.scale_v[fb:fb + nb])
        parts += int(got["n"])
        if max_norm is not None:
            np.testing.assert_allclose(got["norms"], want_norms, rtol=1e-13)
    assert parts >= len(rows)
    if case == "empty":
        assert any(int(np.load(tmp_path / f"rank{r}.npz")["n"]) == 0 for r in range(world))


# ------------------------------------------------------------ distributed Muon

MUON_CASES = {
    # rows, cols of 2-D matrices (a tall one, a wide one); each is one block
    "mats": ([64, 48, 96, 32, 40], [32, 64, 16, 32, 24]),
    # two matrices for four ranks: two ranks hold none
    "few": ([128, 16], [64, 16]),
}
MUON_HP = dict(lr=0.02, momentum=0.95, weight_decay=0.01, eps=1e-7, ns_steps=5, nesterov=1)


def _muon_matrix_step(p, pb, g_bits, mom, R, C, hp, gs):
    """One Muon step of one matrix from the oracle's pieces, in place on the
    fp32 master p, its bf16 copy pb and the momentum (flat views)."""
    import oracle
    U = oracle.muon_momentum(mom, g_bits, hp["momentum"], gs, nesterov=True)
    X = oracle.newton_schulz(U.reshape(R, C).astype(np.float64), hp["ns_steps"], hp["eps"])
    lrs = np.float32(hp["lr"] * oracle.muon_update_scale(R, C))
    decay = np.float32(1.0 - hp["lr"] * hp["weight_decay"])
    p[:] = p * decay - lrs * X.astype(np.float32).ravel()
    pb[:] = oracle.bf16_round(p)


class OracleMuon:
    """Muon state of the matrices in one rank's slice bucket, stepped with
    the oracle's pieces."""

    def __init__(self, local):
        self.local = local
        rk = local.rk
        self.mats = [(int(o), int(r), int(c)) for r, c, o in zip(rk["rows"], rk["cols"], rk["offsets"])]
        self.mom = [np.zeros(r * c, np.float32) for _, r, c in self.mats]

    def step(self, hp, grad_scale):
        b = self.local.b
        for (o, R, C), mom in zip(self.mats, self.mom):
            sl = slice(o, o + R * C)
            _muon_matrix_step(b.p[sl], b.pb[sl], b.g[sl], mom, R, C, hp, grad_scale)


def _muon_worker(rank, world, port, case, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import ragged_bucket_layout_b200 as rb
        from ragged_bucket_layout_b200.sharded import ShardedMuon

        rows, cols = MUON_CASES[case]
        plan = rb.dbuf_plan(rows, cols, rows, world, 16)            # k = rows: one block per matrix
        info = rb.dbuf_plan_info(plan)
        local = OracleSlice(oracle.rank_bucket(rows, cols, rows, info["offsets"], info["slice"], world, rank))
        sm = ShardedMuon(plan, local=local, muon=OracleMuon(local))
        full = _master(rows, cols)
        for i, a, b, v in sm.local_views(rb.DBUF_MASTER_F32):
            assert (a, b) == (0, rows[i])                          # whole matrices only
            v.copy_(torch.from_numpy(full[i]))
        for t in range(1, STEPS + 1):
            for g, x in zip(sm.grad_views(), _grad(rows, cols, rank, t)):
                g.copy_(torch.from_numpy(x))
            sm.step(MUON_HP)
        np.savez(os.path.join(outdir, f"rank{rank}.npz"), param=sm.param.view(torch.int16).numpy(), p=local.b.p,
                 mats=np.array(sm.matrices, np.int64), mom=np.concatenate([np.zeros(0, np.float32)] + sm.muon.mom))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case,world", [("mats", 2), ("mats", 4), ("few", 4)])
def test_sharded_muon_steps_every_matrix_once_on_its_rank(case, world, tmp_path):
    import oracle

    mp.start_processes(_muon_worker, args=(world, _free_port(), case, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    rows, cols = MUON_CASES[case]
    st, off, s = oracle.plan(rows, cols, rows, world, 16)
    assert st == 0
    W = oracle.Bucket(rows, cols, rows, off, s, world)
    moms = [np.zeros(r * c, np.float32) for r, c in zip(rows, cols)]
    for i, x in enumerate(_master(rows, cols)):
        W.p[W.tensor_slice(i)] = x.ravel()
    for t in range(1, STEPS + 1):
        per_rank = [_grad(rows, cols, r, t) for r in range(world)]
        for i in range(len(rows)):
            sl = W.tensor_slice(i)
            W.g[sl] = _bf16_bits(sum(g[i] for g in per_rank).ravel())
            _muon_matrix_step(W.p[sl], W.pb[sl], W.g[sl], moms[i], rows[i], cols[i], MUON_HP, 1.0 / world)
    owners = []
    for r in range(world):
        got = np.load(tmp_path / f"rank{r}.npz")
        assert np.array_equal(got["param"].view(np.uint16), W.pb), f"rank {r}: gathered bf16 bucket"
        assert np.array_equal(got["p"].view(np.uint32), W.p[r * s:(r + 1) * s].view(np.uint32)), f"rank {r}"
        mats = got["mats"].tolist()
        want_mom = np.concatenate([np.zeros(0, np.float32)] + [moms[i] for i in mats])
        assert np.array_equal(got["mom"], want_mom), f"rank {r}: momentum"
        owners += mats
    assert sorted(owners) == list(range(len(rows)))               # every matrix on exactly one rank
    assert len(set(owners)) == len(rows) and world > 1


def test_sharded_muon_refuses_a_split_matrix():
    """With blocks of fewer rows than the matrix, a slice boundary can cut a
    matrix; Muon needs it whole on one rank, so the plan is refused."""
    import oracle
    import ragged_bucket_layout_b200 as rb
    from ragged_bucket_layout_b200.sharded import ShardedMuon

    rows, cols = [64, 64], [32, 32]
    plan = rb.dbuf_plan(rows, cols, [8, 8], 4, 16)
    info = rb.dbuf_plan_info(plan)
    assert any(a > 0 for q in range(4) for _, a, _ in rb.dbuf_plan_rank(plan, q).parts)
    for q in range(4):
        local = OracleSlice(oracle.rank_bucket(rows, cols, [8, 8], info["offsets"], info["slice"], 4, q))
        parts = rb.dbuf_plan_rank(plan, q).parts
        if all(a == 0 and b == rows[i] for i, a, b in parts):
            continue
        with pytest.raises(ValueError, match="k = rows"):
            ShardedMuon(plan, rank=q, world=4, local=local, muon=object(), check_plan=False)


def test_sharded_bucket_checks_its_arguments():
    """A plan for another number of ranks, or a plan that is not from
    dbuf_plan (no tensor shapes), is refused before any collective."""
    import oracle
    import ragged_bucket_layout_b200 as rb
    from ragged_bucket_layout_b200.sharded import ShardedBucket

    rows, cols, k, bc = CASES["tiny"]
    plan = rb.dbuf_plan(rows, cols, k, 4, 16)
    info = rb.dbuf_plan_info(plan)
    local = OracleSlice(oracle.rank_bucket(rows, cols, k, info["offsets"], info["slice"], 4, 0))
    with pytest.raises(ValueError, match="4 slices for 2 ranks"):
        ShardedBucket(plan, rank=0, world=2, local=local, check_plan=False)
    bare = rb.Plan(plan.handle, plan.n, plan.m)            # same layout, no shapes
    try:
        with pytest.raises(ValueError, match="dbuf_plan"):
            ShardedBucket(bare, rank=0, world=4, local=local, check_plan=False)
    finally:
        bare.handle = None                                 # owned by `plan`
    sb = ShardedBucket(plan, rank=0, world=4, local=local, check_plan=False)
    assert [tuple(v.shape) for v in sb.grad_views()] == list(zip(rows, cols))
    assert sb.grad.numel() == sb.param.numel() == info["bucket"]


def _multi_worker(rank, world, port, outdir):
    """Two buckets stepped back to back, each all-gather left in flight while
    the next bucket's reduce-scatter and step run (the overlap pattern)."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import ragged_bucket_layout_b200 as rb
        from ragged_bucket_layout_b200.sharded import ShardedBucket

        sbs, locals_ = [], []
        for case in ("tiny", "tiles"):
            rows, cols, k, bc = CASES[case]
            plan = rb.dbuf_plan(rows, cols, k, world, 16, block_cols=bc)
            info = rb.dbuf_plan_info(plan)
            local = OracleSlice(oracle.rank_bucket(rows, cols, k, info["offsets"], info["slice"], world, rank, bc))
            sb = ShardedBucket(plan, local=local)
            full = _master(rows, cols)
            for i, a, b, v in sb.local_views(rb.DBUF_MASTER_F32):
                v.copy_(torch.from_numpy(full[i][a:b]))
            sbs.append(sb)
            locals_.append(local)
        for t in range(1, STEPS + 1):
            works = []
            for sb, case in zip(sbs, ("tiny", "tiles")):
                rows, cols, _, _ = CASES[case]
                for g, x in zip(sb.grad_views(), _grad(rows, cols, rank, t)):
                    g.copy_(torch.from_numpy(x))
                works.append(sb.step(_hp(t), async_op=True))
            for w in works:
                w.wait()
        for j, (sb, local) in enumerate(zip(sbs, locals_)):
            np.savez(os.path.join(outdir, f"rank{rank}_b{j}.npz"), param=sb.param.view(torch.int16).numpy(),
                     p=local.b.p)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_buckets_with_all_gathers_in_flight(tmp_path):
    import oracle

    world = 2
    mp.start_processes(_multi_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for j, case in enumerate(("tiny", "tiles")):
        rows, cols, k, bc = CASES[case]
        st, off, s = oracle.plan(rows, cols, k, world, 16)
        W = oracle.Bucket(rows, cols, k, off, s, world, block_cols=bc)
        for i, x in enumerate(_master(rows, cols)):
            W.p[W.tensor_slice(i)] = x.ravel()
        for t in range(1, STEPS + 1):
            per_rank = [_grad(rows, cols, r, t) for r in range(world)]
            for i in range(len(rows)):
                W.g[W.tensor_slice(i)] = _bf16_bits(sum(g[i] for g in per_rank).ravel())
            W.step(_hp(t), t, 1.0 / world)
        for r in range(world):
            got = np.load(tmp_path / f"rank{r}_b{j}.npz")
            assert np.array_equal(got["param"].view(np.uint16), W.pb), f"bucket {case}, rank {r}"
            assert np.array_equal(got["p"].view(np.uint32), W.p[r * s:(r + 1) * s].view(np.uint32))


def _disagree_worker(rank, world, port, outdir):
    """Rank 1 lists the same tensors in another order: every rank must get
    an error at construction, before any reduce-scatter."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import ragged_bucket_layout_b200 as rb
        from ragged_bucket_layout_b200.sharded import ShardedBucket

        rows, cols, k, bc = CASES["tiles"]
        if rank == 1:
            rows, cols, k, bc = rows[::-1], cols[::-1], k[::-1], bc[::-1]
        plan = rb.dbuf_plan(rows, cols, k, world, 16, block_cols=bc)
        info = rb.dbuf_plan_info(plan)
        local = OracleSlice(oracle.rank_bucket(rows, cols, k, info["offsets"], info["slice"], world, rank, bc))
        try:
            ShardedBucket(plan, local=local)
            msg = "no error"
        except RuntimeError as e:
            msg = str(e)
        with open(os.path.join(outdir, f"rank{rank}.txt"), "w") as f:
            f.write(msg)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_ranks_that_disagree_on_the_plan_all_fail_at_construction(tmp_path):
    world = 2
    mp.start_processes(_disagree_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        msg = (tmp_path / f"rank{r}.txt").read_text()
        assert "disagree on the bucket plan" in msg and "[1]" in msg, msg


def _leaver_worker(rank, world, port, outdir):
    """Rank 1 leaves between steps (after one step, with nothing in flight);
    rank 0's next step must end with an error, not wait for ever."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=10))
    import oracle
    import ragged_bucket_layout_b200 as rb
    from ragged_bucket_layout_b200.sharded import ShardedBucket

    rows, cols, k, bc = CASES["tiny"]
    plan = rb.dbuf_plan(rows, cols, k, world, 16, block_cols=bc)
    info = rb.dbuf_plan_info(plan)
    local = OracleSlice(oracle.rank_bucket(rows, cols, k, info["offsets"], info["slice"], world, rank, bc))
    sb = ShardedBucket(plan, local=local)
    sb.step(_hp(1))
    if rank == 1:
        return                                   # leaves: its sockets close when the process exits
    t0 = time.monotonic()
    try:
        sb.step(_hp(2))
        msg = "no error"
    except RuntimeError as e:
        msg = f"error after {time.monotonic() - t0:.1f} s: {type(e).__name__}"
    with open(os.path.join(outdir, "rank0.txt"), "w") as f:
        f.write(msg)


def test_a_rank_that_leaves_makes_the_next_step_fail(tmp_path):
    mp.start_processes(_leaver_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    msg = (tmp_path / "rank0.txt").read_text()
    assert msg.startswith("error after"), msg
    assert float(msg.split()[2]) < 30.0, msg
