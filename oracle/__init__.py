"""CPU oracle of the ragged-bucket 8-bit Adam step (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the product
library.  The planner and the 8-bit Adam step live in ``oracle.cpp`` (plain
C++, fp32 in one fixed operation order); this module marshals numpy arrays
for them and holds, in plain numpy, the row-wise (FSDP2-style) baseline
layout, the rank buckets (one device's slice as a bucket of its own) and
the Muon pieces (fp32 momentum, float64 Newton-Schulz).

Every function cites the part of the veScale-FSDP description it follows; the
parity status of each is stated in ``oracle.cpp``'s header.
"""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

OK, EINVAL, EINFEASIBLE = 0, 1, 2
CXXFLAGS = ["-O2", "-std=c++17", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
            "-fno-fast-math", "-fno-unsafe-math-optimizations"]


def build(force=False):
    """Compile oracle.cpp into liboracle.so (g++, no FMA contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["g++", *CXXFLAGS, "-o", _LIB, _SRC])
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    P = ctypes.c_void_p
    i32, i64, f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    lib.orc_plan.restype = ctypes.c_int
    lib.orc_plan.argtypes = [P, P, P, i32, i32, i64, i64, i32, P, P]
    lib.orc_place_fixed.restype = ctypes.c_int
    lib.orc_place_fixed.argtypes = [P, P, P, i32, i32, i64, i64, i32, P]
    lib.orc_exists_placement.restype = ctypes.c_int
    lib.orc_exists_placement.argtypes = [P, P, i32, i64, i32, i64]
    lib.orc_bruteforce_min_bucket.restype = i64
    lib.orc_bruteforce_min_bucket.argtypes = [P, P, P, i32, i32, i64]
    lib.orc_check_layout.restype = ctypes.c_int
    lib.orc_check_layout.argtypes = [P, P, P, i32, i32, i64, P, i64]
    lib.orc_adam8_step.restype = None
    lib.orc_adam8_step.argtypes = [i64, P, P, P, P, P, P, P, P, P, P,
                                   f32, f32, f32, f32, f32, i64, f32, i32]
    lib.orc_adam8_step_tiles.restype = None
    lib.orc_adam8_step_tiles.argtypes = [i64, P, P, P, P, P, P, P, P, P, P, P, P,
                                         f32, f32, f32, f32, f32, i64, f32, i32]
    lib.orc_step_scalars.restype = None
    lib.orc_step_scalars.argtypes = [f32, f32, f32, f32, f32, i64, P]
    lib.orc_pack.restype = None
    lib.orc_pack.argtypes = [i64, P, P, f32]
    lib.orc_accumulate.restype = None
    lib.orc_accumulate.argtypes = [i64, P, P, f32]
    lib.orc_grad_norm.restype = ctypes.c_double
    lib.orc_grad_norm.argtypes = [i64, P, f32]
    lib.orc_clip_coef.restype = ctypes.c_double
    lib.orc_clip_coef.argtypes = [ctypes.c_double, f32]
    lib.orc_clipped_scale.restype = ctypes.c_float
    lib.orc_clipped_scale.argtypes = [ctypes.c_double, f32, f32]
    lib.orc_bf16_round.restype = None
    lib.orc_bf16_round.argtypes = [i64, P, P]
    _lib = lib
    return lib


def _i64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.int64))


def _ptr(a):
    return a.ctypes.data if a.size else None


# ---------------------------------------------------------------- layout ---

def plan(rows, cols, k, m, align=16, max_bucket=0, literal=False):
    """Structure-aware bucket layout (paper Sec. 4 as the pages give it: sort by
    block size descending, then place with block alignment at every slice
    boundary and padding only between tensors).

    Returns (status, offsets[n] in input order, slice size s).
    """
    rows, cols, k = _i64(rows), _i64(cols), _i64(k)
    n = rows.size
    off = np.zeros(max(n, 1), dtype=np.int64)
    s = np.zeros(1, dtype=np.int64)
    st = _load().orc_plan(_ptr(rows), _ptr(cols), _ptr(k), n, int(m), int(align), int(max_bucket),
                          1 if literal else 0, off.ctypes.data, s.ctypes.data)
    return st, off[:n].copy(), int(s[0])


def place_fixed(rows, cols, k, m, align, s, literal=False):
    """Greedy placement in planner order at one fixed slice size s.
    Returns (placed?, offsets in input order)."""
    rows, cols, k = _i64(rows), _i64(cols), _i64(k)
    off = np.zeros(max(rows.size, 1), dtype=np.int64)
    ok = _load().orc_place_fixed(_ptr(rows), _ptr(cols), _ptr(k), rows.size, int(m), int(align),
                                 int(s), 1 if literal else 0, off.ctypes.data)
    return bool(ok), off[:rows.size].copy()


def planner_order(rows, cols, k):
    """Input indices in planner order: block size descending, then element
    count descending, then input position (plain numpy, for the tests)."""
    rows, cols, k = _i64(rows), _i64(cols), _i64(k)
    n, b = rows * cols, k * cols
    return np.array(sorted(range(rows.size), key=lambda i: (-b[i], -n[i], i)), dtype=np.int64)


def exists_placement(n_elems, b_elems, s, m, align):
    """Exhaustive search: any placement of the tensors in this order at slice size s?"""
    n, b = _i64(n_elems), _i64(b_elems)
    return bool(_load().orc_exists_placement(_ptr(n), _ptr(b), n.size, int(s), int(m), int(align)))


def bruteforce_min_bucket(rows, cols, k, m, align):
    """True minimum bucket size over every order and placement (tiny inputs)."""
    rows, cols, k = _i64(rows), _i64(cols), _i64(k)
    return int(_load().orc_bruteforce_min_bucket(_ptr(rows), _ptr(cols), _ptr(k), rows.size,
                                                 int(m), int(align)))


def check_layout(rows, cols, k, m, align, offsets, s):
    """Bit mask of broken layout rules (0 = valid); see oracle.cpp."""
    rows, cols, k, off = _i64(rows), _i64(cols), _i64(k), _i64(offsets)
    return int(_load().orc_check_layout(_ptr(rows), _ptr(cols), _ptr(k), rows.size, int(m),
                                        int(align), _ptr(off), int(s)))


def blocks(rows, cols, k, offsets):
    """Quantisation blocks of a planned bucket, numbered in bucket order
    (tensors by ascending offset, blocks in row order inside a tensor).

    RaggedShard's unit (paper Sec. 3): k whole rows, the last block of a tensor
    may be shorter.  Returns (start, length) int64 arrays.
    """
    rows, cols, k, off = _i64(rows), _i64(cols), _i64(k), _i64(offsets)
    starts, lens = [], []
    for i in np.argsort(off, kind="stable"):
        n, b = int(rows[i] * cols[i]), int(k[i] * cols[i])
        nb = -(-n // b)
        st = int(off[i]) + b * np.arange(nb, dtype=np.int64)
        ln = np.full(nb, b, dtype=np.int64)
        ln[-1] = n - b * (nb - 1)
        starts.append(st)
        lens.append(ln)
    if not starts:
        return np.zeros(0, np.int64), np.zeros(0, np.int64)
    return np.concatenate(starts), np.concatenate(lens)


def tiles(rows, cols, k, block_cols, offsets):
    """Quantisation blocks of a planned bucket when a tensor's blocks are
    k rows x block_cols columns (the 2-D 32x32 blocks the 8-bit Adam case
    study allows per parameter; block_cols = 0, or >= cols, means whole
    rows).  Numbered in bucket order: tensors by ascending offset, row blocks
    top to bottom, column tiles left to right inside a row block; the last
    row block and the last column tile may be smaller.  Returns int64 arrays
    (base, trows, width, stride): tile j covers elements
    base + r * stride + c for r < trows, c < width."""
    rows, cols, k, off = _i64(rows), _i64(cols), _i64(k), _i64(offsets)
    bc = _i64(block_cols) if block_cols is not None else np.zeros_like(rows)
    base, trows, width, stride = [], [], [], []
    for i in np.argsort(off, kind="stable"):
        R, C, K = int(rows[i]), int(cols[i]), int(k[i])
        W = C if int(bc[i]) <= 0 or int(bc[i]) >= C else int(bc[i])
        for r0 in range(0, R, K):
            nr = min(K, R - r0)
            for c0 in range(0, C, W):
                base.append(int(off[i]) + r0 * C + c0)
                trows.append(nr)
                width.append(min(W, C - c0))
                stride.append(C)
    mk = lambda a: np.asarray(a, dtype=np.int64)
    return mk(base), mk(trows), mk(width), mk(stride)


def shards(rows, cols, offsets, s, m):
    """RaggedShard placement (paper Sec. 3; devices hold different numbers of
    whole blocks): for each tensor and rank, the rows [begin, end) of the
    tensor that lie in slice r = [r s, (r+1) s) of the bucket."""
    out = []
    for R, C, o in zip(_i64(rows), _i64(cols), _i64(offsets)):
        per = []
        for r in range(m):
            lo, hi = max(int(o), r * s), min(int(o) + int(R * C), (r + 1) * s)
            if hi <= lo:
                first = min(int(R), max(0, -(-(r * s - int(o)) // int(C))))
                per.append((first, first))
            else:
                per.append(((lo - int(o)) // int(C), (hi - int(o)) // int(C)))
        out.append(per)
    return out


def rank_bucket(rows, cols, k, offsets, s, m, r, block_cols=None):
    """The part of a bucket that rank r holds (paper Sec. 3; each device
    quantises the whole blocks of its own slice [r s, (r+1) s)), described
    as a bucket of its own with one slice of s elements.

    Each tensor's elements [o, o + rows*cols) are intersected with the slice;
    a non-empty intersection is whole rows (interior slice boundaries are
    block edges) and becomes a tensor of those rows, same cols, k and
    block_cols, at its offset minus r s.  Returns a dict with the parts
    (parent id, row_begin, row_end) in parent order, their rows, cols, k,
    block_cols and offsets, and first_block, the number of the parent's
    quantisation blocks (numbered in bucket order) that come before the
    slice.
    """
    rows, cols, k, off = _i64(rows), _i64(cols), _i64(k), _i64(offsets)
    bc = _i64(block_cols) if block_cols is not None else np.zeros_like(rows)
    lo, hi = int(r) * int(s), (int(r) + 1) * int(s)
    out = dict(parts=[], rows=[], cols=[], k=[], block_cols=[], offsets=[])
    first_block = 0
    for i in range(rows.size):
        R, C, K, o = int(rows[i]), int(cols[i]), int(k[i]), int(off[i])
        tiles_per_row_block = 1 if bc[i] <= 0 or bc[i] >= C else -(-C // int(bc[i]))
        a, b = max(o, lo), min(o + R * C, hi)
        # Row blocks of the tensor that start before the slice.
        first_row_in = R if o + R * C <= lo else max(0, lo - o) // C
        first_block += tiles_per_row_block * (-(-first_row_in // K))
        if b <= a:
            continue
        assert (a - o) % C == 0 and (b - o) % C == 0, "a slice boundary cuts a row"
        assert ((a - o) // C) % K == 0, "a slice boundary cuts a block"
        out["parts"].append((i, (a - o) // C, (b - o) // C))
        out["rows"].append((b - a) // C)
        out["cols"].append(C)
        out["k"].append(K)
        out["block_cols"].append(int(bc[i]))
        out["offsets"].append(a - lo)
    for key in ("rows", "cols", "k", "block_cols", "offsets"):
        out[key] = np.asarray(out[key], dtype=np.int64)
    out["first_block"] = first_block
    out["s"] = int(s)
    return out


def padding_mask(rows, cols, offsets, bucket):
    """Boolean mask of bucket elements that belong to no tensor."""
    mask = np.ones(bucket, dtype=bool)
    for r, c, o in zip(_i64(rows), _i64(cols), _i64(offsets)):
        mask[int(o):int(o) + int(r * c)] = False
    return mask


# ---------------------------------------------------------------- update ---

def step_scalars(lr, beta1, beta2, eps, wd, t):
    """(b1, 1-b1, b2, 1-b2, sqrt(1-b2^t), eps*sqrt(1-b2^t), lr*sqrt(1-b2^t)/(1-b1^t),
    1-lr*wd) as float32."""
    out = np.zeros(8, dtype=np.float32)
    _load().orc_step_scalars(lr, beta1, beta2, eps, wd, int(t), out.ctypes.data)
    return out


def adam8_step(start, length, sidx, p, g_bits, mq, vq, scale_m, scale_v, pb_bits, hp, t,
               grad_scale, threads=1):
    """Block-wise 8-bit Adam (the 8-bit Adam case study, paper Sec. 6.3: each
    device quantises its own blocks) over the listed blocks, in place.

    p float32, g_bits uint16 (bf16), mq int8, vq uint8, pb_bits uint16 are
    indexed by bucket element; scale_m/scale_v float32 by sidx[j].
    """
    start, length, sidx = _i64(start), _i64(length), _i64(sidx)
    assert p.dtype == np.float32 and g_bits.dtype == np.uint16 and pb_bits.dtype == np.uint16
    assert mq.dtype == np.int8 and vq.dtype == np.uint8
    assert scale_m.dtype == np.float32 and scale_v.dtype == np.float32
    for a in (p, g_bits, mq, vq, scale_m, scale_v, pb_bits):
        assert a.flags.c_contiguous
    if start.size:
        hi = int(np.max(start + length))
        assert hi <= min(p.size, g_bits.size, mq.size, vq.size, pb_bits.size)
        assert int(np.max(sidx)) < min(scale_m.size, scale_v.size)
    _load().orc_adam8_step(start.size, _ptr(start), _ptr(length), _ptr(sidx), _ptr(p), _ptr(g_bits),
                           _ptr(mq), _ptr(vq), _ptr(scale_m), _ptr(scale_v), _ptr(pb_bits),
                           hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"], int(t),
                           float(grad_scale), int(threads))


def pack(src_bits, dst_bits, scale):
    """Copy-in of the row-wise FSDP baseline: dst = bf16(float(src) * scale)."""
    assert src_bits.dtype == np.uint16 and dst_bits.dtype == np.uint16
    assert dst_bits.size >= src_bits.size and dst_bits.flags.c_contiguous
    src = np.ascontiguousarray(src_bits)
    _load().orc_pack(src.size, _ptr(src), _ptr(dst_bits), float(scale))


def accumulate(src_bits, dst_bits, scale):
    """DBuffer group add (gradient accumulation; paper Sec. 5 lists add among
    the fused group operations): dst = bf16(float(dst) + float(src) * scale)."""
    assert src_bits.dtype == np.uint16 and dst_bits.dtype == np.uint16
    assert dst_bits.size >= src_bits.size and dst_bits.flags.c_contiguous
    src = np.ascontiguousarray(src_bits)
    _load().orc_accumulate(src.size, _ptr(src), _ptr(dst_bits), float(scale))


def grad_norm(g_bits, scale):
    """L2 norm of float(g) * scale over an array (squares summed in double)."""
    g = np.ascontiguousarray(g_bits, dtype=np.uint16)
    return float(_load().orc_grad_norm(g.size, _ptr(g), float(scale)))


def clip_coef(norm, max_norm):
    """Clipping coefficient min(1, max_norm / (norm + 1e-6)) in double."""
    return float(_load().orc_clip_coef(float(norm), float(max_norm)))


def clipped_scale(norm, grad_scale, max_norm):
    """grad_scale after global-norm clipping, rounded to float once."""
    return float(_load().orc_clipped_scale(float(norm), float(grad_scale), float(max_norm)))


def rowwise_layout(rows, cols, m):
    """Row-wise even sharding, the FSDP2 / Megatron-FSDP baseline of the
    veScale-FSDP pages (comparison of sharding formats, "row-wise" entry):
    tensor t is cut along dim 0 into m shards of q_t = ceil(rows_t / m) rows
    (the last shards shorter or empty) and each shard is padded to q_t rows in
    the communication buffer.  Rank r's chunk concatenates its padded shards
    of every tensor in order; an AllGather output holds the m chunks in rank
    order.  Returns (q, offsets of each tensor's shard within a chunk, chunk
    size in elements)."""
    rows = np.asarray(rows, dtype=np.int64)
    cols = np.asarray(cols, dtype=np.int64)
    q = (rows + m - 1) // m
    sizes = q * cols
    off = np.concatenate([[0], np.cumsum(sizes)[:-1]]).astype(np.int64)
    return q, off, int(sizes.sum())


def _rowwise_rows(rows_t, q_t, r):
    r0 = r * q_t
    return r0, max(r0, min(rows_t, r0 + q_t))


def rowwise_copy_out(gathered_bits, rows, cols, m):
    """Interleaved copy-out after the AllGather of the row-wise baseline (the
    pages' per-parameter copy-out with interleaved addresses): tensor t's rows
    [r q_t, min(rows_t, (r+1) q_t)) are the first rows of its shard in chunk r.
    Returns one bf16-bits array of rows_t * cols_t elements per tensor."""
    q, off, C = rowwise_layout(rows, cols, m)
    outs = []
    for t in range(len(q)):
        n_t = int(rows[t]) * int(cols[t])
        out = np.zeros(n_t, dtype=np.uint16)
        for r in range(m):
            r0, r1 = _rowwise_rows(int(rows[t]), int(q[t]), r)
            k = (r1 - r0) * int(cols[t])
            src = r * C + int(off[t])
            out[r0 * int(cols[t]):r0 * int(cols[t]) + k] = gathered_bits[src:src + k]
        outs.append(out)
    return outs


def rowwise_copy_in(grads_bits, rows, cols, m, scale):
    """Interleaved copy-in before the ReduceScatter of the row-wise baseline
    (the pages' per-parameter copy-in): each tensor's rows go to the shard of
    the rank that owns them as bf16(float(g) * scale); padding rows are zero.
    Returns the m * chunk bf16-bits buffer."""
    q, off, C = rowwise_layout(rows, cols, m)
    buf = np.zeros(m * C, dtype=np.uint16)
    for t in range(len(q)):
        g = np.ascontiguousarray(grads_bits[t], dtype=np.uint16).reshape(-1)
        for r in range(m):
            r0, r1 = _rowwise_rows(int(rows[t]), int(q[t]), r)
            k = (r1 - r0) * int(cols[t])
            if k == 0:
                continue
            dst = r * C + int(off[t])
            seg = np.zeros(k, dtype=np.uint16)
            pack(g[r0 * int(cols[t]):r0 * int(cols[t]) + k], seg, scale)
            buf[dst:dst + k] = seg
    return buf


def bf16_round(x):
    """float32 -> bf16 bits, round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.size, dtype=np.uint16)
    _load().orc_bf16_round(x.size, _ptr(x), _ptr(out))
    return out


def adam8_step_tiles(base, trows, width, stride, sidx, p, g_bits, mq, vq, scale_m, scale_v, pb_bits, hp, t,
                     grad_scale, threads=1):
    """Block-wise 8-bit Adam over 2-D tiles (see tiles()), in place: each
    tile is quantised as one block, as adam8_step does for a contiguous one."""
    base, trows, width, stride, sidx = _i64(base), _i64(trows), _i64(width), _i64(stride), _i64(sidx)
    assert p.dtype == np.float32 and g_bits.dtype == np.uint16 and pb_bits.dtype == np.uint16
    assert mq.dtype == np.int8 and vq.dtype == np.uint8
    assert scale_m.dtype == np.float32 and scale_v.dtype == np.float32
    for a in (p, g_bits, mq, vq, scale_m, scale_v, pb_bits):
        assert a.flags.c_contiguous
    if base.size:
        hi = int(np.max(base + (trows - 1) * stride + width))
        assert hi <= min(p.size, g_bits.size, mq.size, vq.size, pb_bits.size)
        assert int(np.max(sidx)) < min(scale_m.size, scale_v.size)
    _load().orc_adam8_step_tiles(base.size, _ptr(base), _ptr(trows), _ptr(width), _ptr(stride), _ptr(sidx),
                                 _ptr(p), _ptr(g_bits), _ptr(mq), _ptr(vq), _ptr(scale_m), _ptr(scale_v),
                                 _ptr(pb_bits), hp["lr"], hp["beta1"], hp["beta2"], hp["eps"],
                                 hp["weight_decay"], int(t), float(grad_scale), int(threads))


# ------------------------------------------------------------------ Muon ---
#
# Distributed Muon on RaggedShard (the pages' case study "8-bit Adam and
# distributed Muon", paper Sec. 6.3): each 2-D parameter is gathered whole on
# one rank, its Newton-Schulz preconditioner runs there, and the result goes
# back to the original placement.  The pages give neither the iteration nor
# its coefficients; the reading here is Muon as published by its authors
# (K. Jordan et al., 2024): heavy-ball momentum with the Nesterov form, the
# quintic Newton-Schulz iteration X <- aX + (b A + c A^2) X with A = X X^T and
# (a, b, c) = (3.4445, -4.7750, 2.0315), started from the momentum divided by
# its Frobenius norm, on the wide orientation of the matrix, and an update
# scaled by sqrt(max(1, rows/cols)) with decoupled weight decay.

NS_COEFFS = (3.4445, -4.7750, 2.0315)


def muon_momentum(mom, g_bits, beta, grad_scale, nesterov=True):
    """Muon's momentum in fp32, every operation rounded on its own, in place
    on mom (float32):  t = g * grad_scale;  mom = beta * mom + t;  returns the
    direction U = t + beta * mom (Nesterov) or mom."""
    assert mom.dtype == np.float32
    g = (np.asarray(g_bits, dtype=np.uint32) << 16).view(np.float32)
    b = np.float32(beta)
    t = g * np.float32(grad_scale)
    mom[:] = b * mom + t
    return t + b * mom if nesterov else mom.copy()


def newton_schulz(U, steps=5, eps=1e-7):
    """Orthogonalisation of Muon in float64: X = U / (||U||_F + eps), then
    `steps` quintic iterations on the orientation with rows <= cols."""
    X = np.asarray(U, dtype=np.float64)
    X = X / (np.linalg.norm(X) + eps)
    tall = X.shape[0] > X.shape[1]
    if tall:
        X = X.T
    a, b, c = NS_COEFFS
    for _ in range(steps):
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = a * X + B @ X
    return X.T if tall else X


def muon_update_scale(rows, cols):
    """sqrt(max(1, rows / cols)), the step's shape factor."""
    return float(np.sqrt(max(1.0, rows / cols)))


class Bucket:
    """Whole-bucket state on the host, stepped by the oracle.

    Arrays follow the DBuffer picture (paper Sec. 5): one flat buffer per
    kind, tensors are slices at their planned offsets.  Padding holds zeros;
    the bf16 copy of padding is set to zero on every step.
    """

    def __init__(self, rows, cols, k, offsets, s, m, block_cols=None):
        self.rows, self.cols, self.k = _i64(rows), _i64(cols), _i64(k)
        self.offsets = _i64(offsets)
        self.s, self.m = int(s), int(m)
        self.size = self.s * self.m
        bc = np.zeros_like(self.rows) if block_cols is None else _i64(block_cols)
        self.tiled = bool(np.any((bc > 0) & (bc < self.cols)))
        if self.tiled:
            self.tiles = tiles(self.rows, self.cols, self.k, bc, self.offsets)
            nb = self.tiles[0].size
        else:
            self.start, self.length = blocks(self.rows, self.cols, self.k, self.offsets)
            nb = self.start.size
        self.sidx = np.arange(nb, dtype=np.int64)
        self.pad = padding_mask(self.rows, self.cols, self.offsets, self.size)
        S, B = self.size, nb
        self.p = np.zeros(S, np.float32)
        self.g = np.zeros(S, np.uint16)
        self.mq = np.zeros(S, np.int8)
        self.vq = np.zeros(S, np.uint8)
        self.pb = np.zeros(S, np.uint16)
        self.scale_m = np.zeros(B, np.float32)
        self.scale_v = np.zeros(B, np.float32)

    def tensor_slice(self, i):
        o = int(self.offsets[i])
        return slice(o, o + int(self.rows[i] * self.cols[i]))

    def step(self, hp, t, grad_scale, threads=1):
        if self.tiled:
            adam8_step_tiles(*self.tiles, self.sidx, self.p, self.g, self.mq, self.vq,
                             self.scale_m, self.scale_v, self.pb, hp, t, grad_scale, threads)
        else:
            adam8_step(self.start, self.length, self.sidx, self.p, self.g, self.mq, self.vq,
                       self.scale_m, self.scale_v, self.pb, hp, t, grad_scale, threads)
        self.pb[self.pad] = 0
