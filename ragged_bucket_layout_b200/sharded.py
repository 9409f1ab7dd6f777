"""One rank's side of a data-parallel bucket step over the RaggedShard layout.

veScale-FSDP (paper Sec. 3 and Sec. 5; page sections "1. RaggedShard" and
"3. DBuffer"): the gradient bucket is reduce-scattered so that rank r gets
slice r = [r s, (r+1) s); rank r runs the 8-bit Adam step over the whole
blocks of that slice alone (no block straddles a slice, so the step itself
exchanges nothing); the bf16 parameters are all-gathered back into the full
bucket, where every tensor is a view at its planned offset.

Per rank this holds:
  * the full bf16 gradient and parameter buckets, m*s elements each: the
    buffers the two collectives work on, tensors as zero-copy views;
  * a bucket of one slice (dbuf_plan_rank) with this rank's fp32 master
    weights, 8-bit codes and scales: 1/m of the optimizer state.
The collectives are torch.distributed's (NCCL between GPUs), issued on the
slice bucket's stream; the step is the library's fused kernel.  With
async_op the all-gather is left in flight, so the next bucket's
reduce-scatter and step can be queued behind it.

ShardedMuon is the same flow for a bucket of 2-D matrices planned with one
block per matrix: each matrix then lies whole in one slice, and its rank
runs the library's Muon step on it.
"""
import contextlib
import ctypes
import hashlib
import math

from . import (DBUF_GRAD_BF16, DBUF_PARAM_BF16, DBuffer, Muon, dbuf_plan_info, dbuf_plan_rank)


class ShardedBucket:
    """Rank `rank` of `world` for the bucket of `plan` (planned with
    m = world).  `local` replaces the slice bucket (a DBuffer of
    dbuf_plan_rank(plan, rank) on `device` by default) with any object that
    has array(which), views(which) and step(hp, grad_scale), plus
    grad_norm(grad_scale, out) for step_clipped, e.g. a host-side model of
    it.  With NCCL, make the rank's GPU the current device first (the plan
    check and the collectives run there)."""

    def __init__(self, plan, rank=None, world=None, group=None, device="cuda", local=None, check_plan=True):
        """check_plan: compare a digest of the plan across the group first
        (one all_gather_object), and raise on every rank if they differ."""
        import torch
        import torch.distributed as dist

        self.group = group
        self.rank = dist.get_rank(group) if rank is None else int(rank)
        self.world = dist.get_world_size(group) if world is None else int(world)
        if plan.m != self.world:
            raise ValueError(f"the plan has {plan.m} slices for {self.world} ranks")
        if getattr(plan, "shapes", None) is None:
            raise ValueError("ShardedBucket needs a plan made by dbuf_plan")
        info = dbuf_plan_info(plan)
        if check_plan and self.world > 1:
            self._check_same_plan(plan, info)
        self.plan = plan
        self.rank_plan = dbuf_plan_rank(plan, self.rank)
        self.slice, self.offsets = info["slice"], info["offsets"]
        self.local = DBuffer(self.rank_plan, device=device) if local is None else local
        dev = self.local.array(DBUF_GRAD_BF16).device
        with self._on_stream():
            self.grad = torch.zeros(info["bucket"], dtype=torch.bfloat16, device=dev)
            self.param = torch.zeros(info["bucket"], dtype=torch.bfloat16, device=dev)

    def _check_same_plan(self, plan, info):
        """Every rank plans its bucket on its own; if the ranks' tensor lists
        differ (another order, another shape), the collectives would mix
        unrelated data.  Compare digests of the plans and fail loudly."""
        import torch.distributed as dist
        desc = repr((plan.shapes, getattr(plan, "k", None), getattr(plan, "block_cols", None),
                     info["slice"], info["offsets"], plan.m))
        mine = hashlib.sha256(desc.encode()).hexdigest()
        digests = [None] * self.world
        dist.all_gather_object(digests, mine, group=self.group)
        bad = [r for r, d in enumerate(digests) if d != digests[0]]
        if bad:
            raise RuntimeError(f"ranks disagree on the bucket plan (ranks {bad} differ from rank 0); "
                               "every rank must pass the same tensors in the same order")

    def _on_stream(self):
        import torch
        s = getattr(self.local, "stream", None)
        return torch.cuda.stream(s) if s is not None else contextlib.nullcontext()

    def _full_views(self, flat):
        return [flat[o:o + r * c].view(r, c) for o, (r, c) in zip(self.offsets, self.plan.shapes)]

    def grad_views(self):
        """Each tensor's gradient in the full bucket (where backward writes)."""
        return self._full_views(self.grad)

    def param_views(self):
        """Each tensor's bf16 parameters in the full bucket (the forward's
        weights; filled by the all-gather)."""
        return self._full_views(self.param)

    def local_views(self, which):
        """This rank's rows of each tensor in the slice bucket:
        [(tensor id, row_begin, row_end, view)] for the tensors it holds."""
        return [(i, a, b, v) for (i, a, b), v in zip(self.rank_plan.parts, self.local.views(which))]

    def all_gather_params(self, async_op=False):
        """Gather every rank's bf16 slice into the full parameter bucket."""
        import torch.distributed as dist
        with self._on_stream():
            return dist.all_gather_into_tensor(self.param, self.local.array(DBUF_PARAM_BF16), group=self.group,
                                               async_op=async_op)

    def _reduce_scatter(self):
        import torch.distributed as dist
        dist.reduce_scatter_tensor(self.local.array(DBUF_GRAD_BF16), self.grad, group=self.group)

    def step_clipped(self, hp, max_norm, grad_scale=None, async_op=False):
        """step() with global-norm clipping over the whole bucket, as the
        single-bucket dbuf_adam8_step_clipped does it:
        grad_scale * min(1, max_norm / (norm + 1e-6)), formed in double and
        rounded to float once.  Each rank takes its slice's norm with the
        library's grad-norm kernel, and an all-reduce sums the squares.
        The coefficient is formed on the host, so this waits for the
        reduce-scatter and the norm.  Returns (norm, all-gather handle or
        None)."""
        import torch
        import torch.distributed as dist
        gs = ctypes.c_float(1.0 / self.world if grad_scale is None else float(grad_scale)).value
        mx = ctypes.c_float(float(max_norm)).value
        if not mx > 0:
            raise ValueError("max_norm must be > 0")
        dev = self.grad.device
        with self._on_stream():
            self._reduce_scatter()
            part = torch.zeros(1, dtype=torch.float64, device=dev)
            self.local.grad_norm(gs, part)
            sq = torch.tensor([part.item() ** 2], dtype=torch.float64, device=dev)
            dist.all_reduce(sq, group=self.group)
            norm = math.sqrt(sq.item())
            coef = mx / (norm + 1e-6)
            self._local_step(hp, gs if coef >= 1.0 else gs * coef)   # rounded to float by the binding
        return norm, self.all_gather_params(async_op=async_op)

    def step(self, hp, grad_scale=None, async_op=False):
        """Reduce-scatter (sum) the gradient bucket into this rank's slice,
        step the slice with grad_scale (default 1/world: the mean), then
        all-gather the bf16 slices.  Returns the all-gather's work handle
        when async_op is set."""
        gs = 1.0 / self.world if grad_scale is None else float(grad_scale)
        with self._on_stream():
            self._reduce_scatter()
            self._local_step(hp, gs)
        return self.all_gather_params(async_op=async_op)

    def _local_step(self, hp, grad_scale):
        self.local.step(hp, grad_scale)


class ShardedMuon(ShardedBucket):
    """Distributed Muon over a bucket in which every tensor is one block
    (planned with k = rows).  The planner then keeps each matrix whole inside
    one slice, so the bucket's reduce-scatter delivers each matrix's summed
    gradient to a single rank: the redistribution of a full 2-D matrix to a
    root rank that the pages' distributed Muon does (8-bit Adam and
    distributed Muon case study, paper Sec. 6.3).  That rank runs the
    library's Muon step on it (momentum, Newton-Schulz on tensor cores,
    update), and the all-gather brings the bf16 matrices back to every
    rank.  The momentum of a matrix lives only on its rank.  `muon`
    replaces the library's Muon state (as `local` replaces the slice
    bucket) with any object that has step(hp, grad_scale).  hp takes the
    keys of MUON_DEFAULTS."""

    def __init__(self, plan, rank=None, world=None, group=None, device="cuda", local=None, muon=None,
                 check_plan=True):
        super().__init__(plan, rank, world, group, device, local, check_plan)
        for i, a, b in self.rank_plan.parts:
            if a != 0 or b != plan.shapes[i][0]:
                raise ValueError(f"tensor {i} is split between ranks: plan a Muon bucket with k = rows")
        self.matrices = [i for i, _, _ in self.rank_plan.parts]   # the tensors this rank steps
        if muon is not None:
            self.muon = muon
        else:
            # dbuf_muon_create needs at least one tensor; a rank without any
            # has only padding, which stays zero.
            self.muon = Muon(self.local, range(self.rank_plan.n)) if self.rank_plan.n else None

    def _local_step(self, hp, grad_scale):
        if self.muon is not None:
            self.muon.step(hp, grad_scale)
