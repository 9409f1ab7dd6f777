"""Python binding of libdbuf, the B200 ragged-bucket 8-bit Adam library.

Argument marshalling only: every step of the path (planning, the bucket step,
the copy-in, the padding zeroing) runs in the C++/CUDA library, whose C-ABI is
declared in ``include/dbuf.h``; this module gives the same entry points the
same names.  ``DBuffer`` adds PyTorch views of a bucket whose device memory
PyTorch allocated (PyTorch is used for memory and streams only).

There is no fallback: importing this package without a built ``libdbuf.so``
raises ImportError.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdbuf.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is not built; run `python -c 'import __graft_entry__ as g; g.build()'` "
        "or `python ragged_bucket_layout_b200/build.py`")
_lib = ctypes.CDLL(LIB_PATH)

DBUF_OK, DBUF_EINVAL, DBUF_EINFEASIBLE, DBUF_ENOMEM, DBUF_ECUDA, DBUF_EDEVICE = range(6)
DBUF_MASTER_F32, DBUF_PARAM_BF16, DBUF_GRAD_BF16, DBUF_M_I8, DBUF_V_U8 = range(5)
_STATUS_NAMES = {0: "DBUF_OK", 1: "DBUF_EINVAL", 2: "DBUF_EINFEASIBLE", 3: "DBUF_ENOMEM",
                 4: "DBUF_ECUDA", 5: "DBUF_EDEVICE"}


class DbufError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{_STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class dbuf_tensor_desc(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("k", ctypes.c_int64),
                ("block_cols", ctypes.c_int64)]


class dbuf_adam_hparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float), ("step", ctypes.c_int64)]


class dbuf_view(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("offset_elems", ctypes.c_int64)]


class dbuf_work_item(ctypes.Structure):
    _fields_ = [("first_elem", ctypes.c_int64), ("first_block", ctypes.c_int64), ("n_elems", ctypes.c_int64),
                ("block_elems", ctypes.c_int32), ("kind", ctypes.c_int32), ("n_blocks", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


_P, _PP = ctypes.c_void_p, ctypes.POINTER(ctypes.c_void_p)
_i32, _i64, _f32, _sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_pi64 = ctypes.POINTER(ctypes.c_int64)
_SIGS = {
    "dbuf_plan": (ctypes.c_int, [ctypes.POINTER(dbuf_tensor_desc), _i32, _i32, _i64, _i64, _PP]),
    "dbuf_plan_info": (ctypes.c_int, [_P, _pi64, _pi64, _pi64, _pi64, _pi64]),
    "dbuf_plan_free": (None, [_P]),
    "dbuf_plan_shards": (ctypes.c_int, [_P, _P]),
    "dbuf_plan_rank": (ctypes.c_int, [_P, _i32, _PP, _pi64]),
    "dbuf_plan_dims": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)]),
    "dbuf_required_bytes": (_sz, [_P]),
    "dbuf_create": (ctypes.c_int, [_P, _P, _sz, _P, _PP]),
    "dbuf_pack_grads": (ctypes.c_int, [_P, _PP, _f32, _P]),
    "dbuf_accumulate_grads": (ctypes.c_int, [_P, _PP, _f32, _P]),
    "dbuf_grad_norm": (ctypes.c_int, [_P, _f32, _P, _P]),
    "dbuf_grad_norm_noalloc": (ctypes.c_int, [_P, _i64, _f32, _P, _P]),
    "dbuf_adam8_step_clipped": (ctypes.c_int, [_P, ctypes.POINTER(dbuf_adam_hparams), _f32, _f32, _P, _P]),
    "dbuf_adam8_step": (ctypes.c_int, [_P, ctypes.POINTER(dbuf_adam_hparams), _f32, _P]),
    "dbuf_adam8_step_host": (ctypes.c_int, [_P, ctypes.POINTER(dbuf_adam_hparams), _f32, _P, _P, _P]),
    "dbuf_unpack_views": (ctypes.c_int, [_P, ctypes.c_int, ctypes.POINTER(dbuf_view)]),
    "dbuf_bucket": (ctypes.c_int, [_P, ctypes.c_int, _PP, _pi64]),
    "dbuf_scales": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.POINTER(ctypes.c_float)), _pi64]),
    "dbuf_get_device_status": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int32), _P]),
    "dbuf_clear_device_status": (ctypes.c_int, [_P, _P]),
    "dbuf_work_table": (ctypes.c_int, [_P, ctypes.POINTER(dbuf_work_item), _i64, _pi64]),
    "dbuf_destroy": (None, [_P]),
    "dbuf_last_error": (ctypes.c_char_p, []),
    "dbuf_muon_create": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int32), _i32, _P, _PP]),
    "dbuf_muon_step": (ctypes.c_int, [_P, _P, _f32, _P]),
    "dbuf_muon_orthogonalize": (ctypes.c_int, [_P, _P, _i64, _i64, _i32, _f32, _P, _P]),
    "dbuf_muon_momentum": (ctypes.c_int, [_P, _i32, ctypes.POINTER(ctypes.POINTER(ctypes.c_float)), _pi64]),
    "dbuf_muon_destroy": (None, [_P]),
    "dbuf_rowwise_layout": (ctypes.c_int, [ctypes.POINTER(dbuf_tensor_desc), _i32, _i32, _pi64, _pi64, _pi64]),
    "dbuf_rowwise_create": (ctypes.c_int, [ctypes.POINTER(dbuf_tensor_desc), _i32, _i32, _P, _PP]),
    "dbuf_rowwise_info": (ctypes.c_int, [_P, _pi64, _pi64, _pi64]),
    "dbuf_rowwise_copy_out": (ctypes.c_int, [_P, _P, _PP, _P]),
    "dbuf_rowwise_copy_in": (ctypes.c_int, [_P, _PP, _f32, _P, _P]),
    "dbuf_rowwise_status": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int32), _P]),
    "dbuf_rowwise_destroy": (None, [_P]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


def dbuf_last_error():
    return _lib.dbuf_last_error().decode()


def _check(st):
    if st != DBUF_OK:
        raise DbufError(st, dbuf_last_error())


def _stream(s):
    if s is None:
        return None
    if hasattr(s, "cuda_stream"):
        return ctypes.c_void_p(s.cuda_stream)
    return ctypes.c_void_p(int(s))


# ------------------------------------------------------------------ plans

class Plan:
    """Owner of a dbuf_plan_t (freed with dbuf_plan_free)."""

    def __init__(self, handle, n, m=None):
        self.handle = handle
        self.n = n
        self.m = m
        self._free = _lib.dbuf_plan_free   # held here: module globals may be gone at interpreter exit

    def __del__(self):
        if getattr(self, "handle", None):
            self._free(self.handle)
            self.handle = None


def dbuf_plan(rows, cols, k, m, align_elems=16, max_bucket_elems=0, block_cols=None):
    """Plan a bucket.  block_cols[i] > 0 (and < cols[i]) cuts tensor i's k-row
    blocks into tiles of that many columns, each with its own scales."""
    n = len(rows)
    bc = [0] * n if block_cols is None else [int(x) for x in block_cols]
    descs = (dbuf_tensor_desc * max(n, 1))(*[dbuf_tensor_desc(int(r), int(c), int(q), b)
                                             for r, c, q, b in zip(rows, cols, k, bc)])
    out = ctypes.c_void_p()
    _check(_lib.dbuf_plan(descs, n, int(m), int(align_elems), int(max_bucket_elems), ctypes.byref(out)))
    plan = Plan(out.value, n, int(m))
    plan.shapes = [(int(r), int(c)) for r, c in zip(rows, cols)]
    plan.k = [int(q) for q in k]
    plan.block_cols = bc
    plan.align = int(align_elems)
    return plan


def dbuf_plan_info(plan):
    n = dbuf_plan_dims(plan)[0]
    s, b, p, nb = (ctypes.c_int64() for _ in range(4))
    offs = (ctypes.c_int64 * max(n, 1))()
    _check(_lib.dbuf_plan_info(plan.handle, ctypes.byref(s), ctypes.byref(b), ctypes.byref(p),
                               ctypes.byref(nb), offs))
    return dict(slice=s.value, bucket=b.value, padding=p.value, n_blocks=nb.value,
                offsets=[offs[i] for i in range(n)])


def dbuf_plan_shards(plan, m=None):
    """RaggedShard placement: [[(row_begin, row_end) for each rank] for each
    tensor].  m defaults to the plan's own slice count."""
    n, pm = dbuf_plan_dims(plan)
    if m is not None and int(m) != pm:
        raise ValueError(f"m must be the plan's slice count ({pm})")
    m = pm
    arr = (ctypes.c_int64 * max(2 * n * m, 1))()
    _check(_lib.dbuf_plan_shards(plan.handle, arr))
    return [[(arr[2 * (i * m + r)], arr[2 * (i * m + r) + 1]) for r in range(m)] for i in range(n)]


def dbuf_plan_rank(plan, rank):
    """The bucket rank `rank` holds, as a plan of its own (m = 1, bucket =
    one slice).  The result also carries `rank`, `first_block` (the parent's
    index of its block 0) and `parts`: for each of its tensors, in order,
    (parent tensor id, row_begin, row_end)."""
    if plan.m is None:
        raise ValueError("dbuf_plan_rank needs a plan made by dbuf_plan (m unknown)")
    out, fb = ctypes.c_void_p(), ctypes.c_int64()
    _check(_lib.dbuf_plan_rank(plan.handle, int(rank), ctypes.byref(out), ctypes.byref(fb)))
    if getattr(plan, "shapes", None) is not None:
        # This rank's row ranges only: O(n), not the n*m table of dbuf_plan_shards.
        info = dbuf_plan_info(plan)
        lo, hi = int(rank) * info["slice"], (int(rank) + 1) * info["slice"]
        parts = []
        for i, (o, (R, C)) in enumerate(zip(info["offsets"], plan.shapes)):
            a, b = min(R * C, max(0, lo - o)), min(R * C, max(0, hi - o))
            if b > a:
                parts.append((i, a // C, b // C))
    else:
        parts = [(i, a, b) for i, per in enumerate(dbuf_plan_shards(plan, plan.m)) for a, b in [per[rank]] if b > a]
    sub = Plan(out.value, len(parts), 1)
    if dbuf_plan_dims(sub) != (len(parts), 1):
        raise DbufError(DBUF_EINVAL, f"rank {rank}: the library's rank plan has {dbuf_plan_dims(sub)[0]} tensors, "
                                     f"the binding found {len(parts)}")
    sub.rank, sub.first_block, sub.parts = int(rank), fb.value, parts
    if getattr(plan, "shapes", None) is not None:
        sub.shapes = [(b - a, plan.shapes[i][1]) for i, a, b in parts]
    return sub


def dbuf_plan_dims(plan):
    """(number of tensors, number of slices) as the library holds them."""
    n, m = ctypes.c_int32(), ctypes.c_int32()
    _check(_lib.dbuf_plan_dims(plan.handle, ctypes.byref(n), ctypes.byref(m)))
    return n.value, m.value


def dbuf_plan_free(plan):
    if plan.handle:
        _lib.dbuf_plan_free(plan.handle)
        plan.handle = None


def dbuf_required_bytes(plan):
    return int(_lib.dbuf_required_bytes(plan.handle))


# ---------------------------------------------------------------- buckets

def dbuf_create(plan, device_base=None, base_bytes=0, stream=None):
    out = ctypes.c_void_p()
    _check(_lib.dbuf_create(plan.handle, device_base, int(base_bytes), _stream(stream), ctypes.byref(out)))
    return out.value


def dbuf_destroy(db):
    _lib.dbuf_destroy(db)


def _hp(hp):
    return dbuf_adam_hparams(hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"], int(hp["step"]))


def dbuf_pack_grads(db, grad_ptrs, scale, stream=None):
    arr = (ctypes.c_void_p * max(len(grad_ptrs), 1))(*[int(p) for p in grad_ptrs])
    _check(_lib.dbuf_pack_grads(db, arr, float(scale), _stream(stream)))


def dbuf_accumulate_grads(db, grad_ptrs, scale, stream=None):
    arr = (ctypes.c_void_p * max(len(grad_ptrs), 1))(*[int(p) for p in grad_ptrs])
    _check(_lib.dbuf_accumulate_grads(db, arr, float(scale), _stream(stream)))


def dbuf_grad_norm(db, grad_scale, norm_dev_ptr, stream=None):
    _check(_lib.dbuf_grad_norm(db, float(grad_scale), norm_dev_ptr, _stream(stream)))


def dbuf_grad_norm_noalloc(grad_ptr, n_elems, grad_scale, norm_dev_ptr, stream=None):
    """Allocation-free gradient norm over a plain bf16 device array."""
    _check(_lib.dbuf_grad_norm_noalloc(grad_ptr, int(n_elems), float(grad_scale), norm_dev_ptr, _stream(stream)))


def dbuf_adam8_step_clipped(db, hp, grad_scale, max_norm, norm_dev_ptr=None, stream=None):
    h = _hp(hp)
    _check(_lib.dbuf_adam8_step_clipped(db, ctypes.byref(h), float(grad_scale), float(max_norm), norm_dev_ptr,
                                        _stream(stream)))


def dbuf_adam8_step(db, hp, grad_scale, stream=None):
    h = _hp(hp)
    _check(_lib.dbuf_adam8_step(db, ctypes.byref(h), float(grad_scale), _stream(stream)))


def dbuf_adam8_step_host(db, hp, grad_scale, grads_host_ptr, params_host_ptr, stream=None):
    h = _hp(hp)
    _check(_lib.dbuf_adam8_step_host(db, ctypes.byref(h), float(grad_scale), grads_host_ptr,
                                     params_host_ptr, _stream(stream)))


def dbuf_unpack_views(db, which, n):
    out = (dbuf_view * max(n, 1))()
    _check(_lib.dbuf_unpack_views(db, int(which), out))
    return [(out[i].ptr or 0, out[i].rows, out[i].cols, out[i].offset_elems) for i in range(n)]


def dbuf_bucket(db, which):
    p, n = ctypes.c_void_p(), ctypes.c_int64()
    _check(_lib.dbuf_bucket(db, int(which), ctypes.byref(p), ctypes.byref(n)))
    return p.value or 0, n.value


def dbuf_scales(db):
    p, n = ctypes.POINTER(ctypes.c_float)(), ctypes.c_int64()
    _check(_lib.dbuf_scales(db, ctypes.byref(p), ctypes.byref(n)))
    return ctypes.cast(p, ctypes.c_void_p).value or 0, n.value


def dbuf_get_device_status(db, stream=None):
    code = ctypes.c_int32()
    _check(_lib.dbuf_get_device_status(db, ctypes.byref(code), _stream(stream)))
    return code.value


def dbuf_work_table(plan):
    """Work table of the step kernel as a list of dicts (host introspection)."""
    n = ctypes.c_int64()
    _check(_lib.dbuf_work_table(plan.handle, None, 0, ctypes.byref(n)))
    arr = (dbuf_work_item * max(n.value, 1))()
    _check(_lib.dbuf_work_table(plan.handle, arr, n.value, ctypes.byref(n)))
    return [dict(first_elem=a.first_elem, first_block=a.first_block, n_elems=a.n_elems,
                 block_elems=a.block_elems, kind=a.kind, n_blocks=a.n_blocks, tile_cols=a.reserved)
            for a in arr[:n.value]]


def dbuf_clear_device_status(db, stream=None):
    _check(_lib.dbuf_clear_device_status(db, _stream(stream)))


# ------------------------------------------------------ distributed Muon

class dbuf_muon_hparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("momentum", ctypes.c_float), ("weight_decay", ctypes.c_float),
                ("eps", ctypes.c_float), ("ns_steps", ctypes.c_int32), ("nesterov", ctypes.c_int32)]


MUON_DEFAULTS = dict(lr=0.02, momentum=0.95, weight_decay=0.0, eps=1e-7, ns_steps=5, nesterov=1)


class Muon:
    """Muon state for some 2-D tensors of a DBuffer (owner of a dbuf_muon_t);
    all work goes through the C-ABI on the DBuffer's stream."""

    def __init__(self, dbuffer, ids):
        self.D = dbuffer
        ids = [int(i) for i in ids]
        arr = (ctypes.c_int32 * max(len(ids), 1))(*ids)
        h = ctypes.c_void_p()
        _check(_lib.dbuf_muon_create(dbuffer.handle, arr, len(ids), _stream(dbuffer.stream), ctypes.byref(h)))
        self.handle, self.ids = h, ids
        self._destroy = _lib.dbuf_muon_destroy   # held here: module globals may be gone at interpreter exit

    def close(self):
        if getattr(self, "handle", None):
            self._destroy(self.handle)
            self.handle = None

    def __del__(self):
        self.close()

    def step(self, hp, grad_scale):
        h = dbuf_muon_hparams(**{**MUON_DEFAULTS, **hp})
        _check(_lib.dbuf_muon_step(self.handle, ctypes.byref(h), float(grad_scale), _stream(self.D.stream)))

    def orthogonalize(self, u, steps=5, eps=1e-7, out=None):
        """bf16 Newton-Schulz of a 2-D fp32 CUDA tensor."""
        import torch
        rows, cols = u.shape
        out = torch.empty((rows, cols), dtype=torch.bfloat16, device=u.device) if out is None else out
        _check(_lib.dbuf_muon_orthogonalize(self.handle, u.data_ptr(), rows, cols, int(steps), float(eps),
                                            out.data_ptr(), _stream(self.D.stream)))
        return out

    def momentum(self, j):
        """fp32 momentum of listed tensor j as a 1-D view (borrowed device memory)."""
        import torch
        p, n = ctypes.POINTER(ctypes.c_float)(), ctypes.c_int64()
        _check(_lib.dbuf_muon_momentum(self.handle, int(j), ctypes.byref(p), ctypes.byref(n)))
        addr = ctypes.cast(p, ctypes.c_void_p).value
        return _wrap_device_f32(addr, n.value, self.D.base)


def _wrap_device_f32(addr, n, like):
    """A float32 tensor over n elements of device memory at addr (no copy)."""
    import torch

    class _Arr:
        pass
    a = _Arr()
    a.__cuda_array_interface__ = {"shape": (n,), "typestr": "<f4", "data": (addr, False), "version": 3}
    return torch.as_tensor(a, device=like.device)


# --------------------------------------------- row-wise baseline layout

def dbuf_rowwise_layout(rows, cols, m):
    """Row-wise (FSDP2-style) layout on the host: (chunk_elems, shard_rows, offsets)."""
    n = len(rows)
    descs = (dbuf_tensor_desc * max(n, 1))(*[dbuf_tensor_desc(int(r), int(c), 1, 0) for r, c in zip(rows, cols)])
    chunk = ctypes.c_int64()
    q = (ctypes.c_int64 * max(n, 1))()
    off = (ctypes.c_int64 * max(n, 1))()
    _check(_lib.dbuf_rowwise_layout(descs, n, int(m), ctypes.byref(chunk), q, off))
    return chunk.value, list(q[:n]), list(off[:n])


class Rowwise:
    """Row-wise (FSDP2-style) sharded layout of a tensor list and its
    interleaved copy-in / copy-out (the copies the bucket layout avoids).
    Owner of a dbuf_rowwise_t; all work goes through the C-ABI."""

    def __init__(self, rows, cols, m, stream=None):
        n = len(rows)
        descs = (dbuf_tensor_desc * max(n, 1))(*[dbuf_tensor_desc(int(r), int(c), 1, 0) for r, c in zip(rows, cols)])
        h = ctypes.c_void_p()
        _check(_lib.dbuf_rowwise_create(descs, n, int(m), _stream(stream), ctypes.byref(h)))
        self.handle, self.n, self.m = h, n, int(m)
        self._destroy = _lib.dbuf_rowwise_destroy   # held here: module globals may be gone at interpreter exit
        chunk = ctypes.c_int64()
        q = (ctypes.c_int64 * max(n, 1))()
        off = (ctypes.c_int64 * max(n, 1))()
        _check(_lib.dbuf_rowwise_info(self.handle, ctypes.byref(chunk), q, off))
        self.chunk, self.shard_rows, self.offsets = chunk.value, list(q[:n]), list(off[:n])

    def close(self):
        if getattr(self, "handle", None):
            self._destroy(self.handle)
            self.handle = None

    def __del__(self):
        self.close()

    @staticmethod
    def _ptrs(ts):
        return (ctypes.c_void_p * max(len(ts), 1))(*[int(t.data_ptr()) if hasattr(t, "data_ptr") else int(t)
                                                     for t in ts])

    def copy_out(self, gathered, params, stream=None):
        """params[i] <- tensor i's rows from the m chunks of `gathered`."""
        _check(_lib.dbuf_rowwise_copy_out(self.handle, int(gathered.data_ptr()), self._ptrs(params),
                                          _stream(stream)))

    def copy_in(self, grads, scale, rs_input, stream=None):
        """rs_input <- bf16(float(g) * scale) of every tensor at its ranks' shards; padding rows 0."""
        _check(_lib.dbuf_rowwise_copy_in(self.handle, self._ptrs(grads), float(scale), int(rs_input.data_ptr()),
                                         _stream(stream)))

    def status(self, stream=None):
        code = ctypes.c_int32()
        _check(_lib.dbuf_rowwise_status(self.handle, ctypes.byref(code), _stream(stream)))
        return code.value


# ----------------------------------------------------- PyTorch-owned buckets

_DTYPES = None


def _dtypes():
    global _DTYPES
    if _DTYPES is None:
        import torch
        _DTYPES = {DBUF_MASTER_F32: (torch.float32, 4), DBUF_PARAM_BF16: (torch.bfloat16, 2),
                   DBUF_GRAD_BF16: (torch.bfloat16, 2), DBUF_M_I8: (torch.int8, 1), DBUF_V_U8: (torch.uint8, 1)}
    return _DTYPES


class DBuffer:
    """A bucket whose single device allocation is a PyTorch uint8 tensor.

    Views are slices of that tensor (zero-copy); all work goes through the
    C-ABI calls above on the given (or current) CUDA stream.
    """

    def __init__(self, plan, device="cuda", stream=None, alloc=None):
        """alloc: optional allocation hook, called once as alloc(nbytes).  It
        returns a contiguous 1-D uint8 tensor of at least nbytes on the
        device, 256-byte aligned (e.g. a slice of the caller's memory pool),
        and the bucket lives there.  A hook that returns None or raises
        MemoryError gives DbufError(DBUF_ENOMEM), before any device work;
        so does running out of memory on the default path."""
        import torch
        self.plan = plan
        self.info = dbuf_plan_info(plan)
        nbytes = max(dbuf_required_bytes(plan), 256)
        if alloc is None:
            try:
                base = torch.empty(nbytes, dtype=torch.uint8, device=device)
            except torch.OutOfMemoryError as e:
                raise DbufError(DBUF_ENOMEM, f"allocating {nbytes} bytes: {e}") from e
        else:
            try:
                base = alloc(nbytes)
            except MemoryError as e:
                raise DbufError(DBUF_ENOMEM, f"allocation hook failed for {nbytes} bytes: {e}") from e
            if base is None:
                raise DbufError(DBUF_ENOMEM, f"allocation hook returned no memory for {nbytes} bytes")
            if not isinstance(base, torch.Tensor) or base.dtype != torch.uint8 or base.dim() != 1 \
                    or not base.is_contiguous():
                raise DbufError(DBUF_EINVAL, "allocation hook must return a contiguous 1-D uint8 tensor")
        self.base = base
        self.stream = stream if stream is not None else torch.cuda.current_stream(self.base.device)
        self._destroy = _lib.dbuf_destroy   # held here: module globals may be gone at interpreter exit
        self.handle = dbuf_create(plan, self.base.data_ptr(), self.base.numel(), self.stream)

    def close(self):
        if getattr(self, "handle", None):
            self._destroy(self.handle)
            self.handle = None

    def __del__(self):
        self.close()

    def _view(self, ptr, elems, which):
        dt, es = _dtypes()[which]
        off = ptr - self.base.data_ptr()
        return self.base[off:off + elems * es].view(dt)

    def array(self, which):
        ptr, elems = dbuf_bucket(self.handle, which)
        return self._view(ptr, elems, which)

    def views(self, which):
        out = []
        for ptr, rows, cols, _ in dbuf_unpack_views(self.handle, which, dbuf_plan_dims(self.plan)[0]):
            out.append(self._view(ptr, rows * cols, which).view(rows, cols))
        return out

    def scales(self):
        import torch
        ptr, nb = dbuf_scales(self.handle)
        off = ptr - self.base.data_ptr()
        return self.base[off:off + nb * 8].view(torch.float32).view(nb, 2)

    def step(self, hp, grad_scale):
        dbuf_adam8_step(self.handle, hp, grad_scale, self.stream)

    def step_host(self, hp, grad_scale, grads_host_ptr, params_host_ptr):
        dbuf_adam8_step_host(self.handle, hp, grad_scale, grads_host_ptr, params_host_ptr, self.stream)

    def pack(self, grads, scale):
        dbuf_pack_grads(self.handle, [g.data_ptr() for g in grads], scale, self.stream)

    def accumulate(self, grads, scale):
        dbuf_accumulate_grads(self.handle, [g.data_ptr() for g in grads], scale, self.stream)

    def grad_norm(self, grad_scale, out):
        """Writes the norm into `out` (a float64 CUDA tensor with one element)."""
        dbuf_grad_norm(self.handle, grad_scale, out.data_ptr(), self.stream)

    def step_clipped(self, hp, grad_scale, max_norm, out=None):
        dbuf_adam8_step_clipped(self.handle, hp, grad_scale, max_norm, out.data_ptr() if out is not None else None,
                                self.stream)

    def device_status(self):
        return dbuf_get_device_status(self.handle, self.stream)
