"""Python binding of libsplitzip: lossless exponent-split coding of BF16 / FP8 E5M2
KV-cache tensors on a B200 GPU (SplitZip project page, Abstract and FAQ).

Argument marshalling only: the functions below have the names of the C ABI in
include/splitzip.h and pass torch tensors' device pointers and the current CUDA
stream to it.  Every step of the codec runs in the library's CUDA kernels.
Importing this package loads libsplitzip.so and raises ImportError if it has not
been built (python fp8_kv_cache_exp_b200/build.py); there is no other path.
"""
import ctypes
import os

import torch

__all__ = [
    "SZ_BF16", "SZ_FP8_E5M2", "SZ_OK", "SplitZipError", "lib", "lib_path",
    "sz_status_string", "sz_workspace_bytes", "sz_workspace_bytes_batched", "sz_stream_bytes",
    "sz_max_compressed_size", "sz_workspace_init", "sz_plan", "sz_plan_batched",
    "sz_compressed_size", "sz_compressed_sizes", "sz_encode", "sz_encode_batched",
    "sz_encode_reuse", "sz_encode_reuse_batched", "sz_plan_paged_batched", "sz_encode_paged_batched",
    "sz_decode_paged_batched", "sz_encode_reuse_paged_batched", "sz_paged_t", "paged", "sz_enable_peer_access",
    "sz_decode",
    "sz_decode_batched", "sz_last_device_status", "sz_encode_noalloc", "dtype_of", "elem_bytes", "numel_of",
    "new_workspace", "new_plans", "Batch",
]

SZ_BF16 = 0
SZ_FP8_E5M2 = 1

SZ_OK = 0
SZ_ERR_INVALID_ARG = 1
SZ_ERR_UNSUPPORTED_DTYPE = 2
SZ_ERR_BUFFER_TOO_SMALL = 3
SZ_ERR_CORRUPT_STREAM = 4
SZ_ERR_CUDA = 5
SZ_ERR_TIMEOUT = 6
SZ_ERR_PLAN_MISMATCH = 7
SZ_ERR_INTERNAL = 8

SZ_HEADER_BYTES = 64
SZ_BLOCK_ELEMS = 4096
SZ_MAX_BATCH = 256
SZ_NOALLOC_MAX_ELEMS = 1 << 27
SZ_FLAG_RAW_BLOCKS = 1

lib_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsplitzip.so")


class sz_paged_t(ctypes.Structure):
    """C layout of sz_paged_t (include/splitzip.h): a tensor held in pages of a pool."""
    _fields_ = [("pool", ctypes.c_void_p), ("pages", ctypes.c_void_p), ("pool_pages", ctypes.c_uint64),
                ("page_bytes", ctypes.c_uint64), ("page_elems", ctypes.c_uint32)]


def _load():
    if not os.path.exists(lib_path):
        raise ImportError("libsplitzip.so is not built (%s); run: python fp8_kv_cache_exp_b200/build.py"
                          % lib_path)
    L = ctypes.CDLL(lib_path)
    vp, u64, sz, i32 = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_size_t, ctypes.c_int
    pvp, pu64, psz = ctypes.POINTER(vp), ctypes.POINTER(u64), ctypes.POINTER(sz)
    ppg = ctypes.POINTER(sz_paged_t)
    sigs = {
        "sz_status_string": (ctypes.c_char_p, [i32]),
        "sz_workspace_bytes": (sz, [i32, u64]),
        "sz_workspace_bytes_batched": (sz, [i32, i32, pu64]),
        "sz_stream_bytes": (sz, [i32, u64, u64]),
        "sz_max_compressed_size": (sz, [i32, u64]),
        "sz_workspace_init": (i32, [vp, sz, vp]),
        "sz_plan": (i32, [i32, vp, u64, vp, sz, vp, vp]),
        "sz_plan_batched": (i32, [i32, i32, pvp, pu64, vp, sz, vp, vp]),
        "sz_compressed_size": (i32, [vp, pu64, vp]),
        "sz_compressed_sizes": (i32, [i32, vp, pu64, vp]),
        "sz_plan_set_flags": (i32, [i32, vp, ctypes.c_uint, vp]),
        "sz_encode": (i32, [i32, vp, vp, u64, vp, sz, vp, sz, vp]),
        "sz_encode_batched": (i32, [i32, i32, vp, pvp, pu64, pvp, psz, vp, sz, vp]),
        "sz_encode_reuse": (i32, [i32, vp, vp, u64, vp, sz, vp, vp, sz, vp]),
        "sz_encode_reuse_batched": (i32, [i32, i32, vp, pvp, pu64, pvp, psz, vp, vp, sz, vp]),
        "sz_plan_paged_batched": (i32, [i32, i32, ppg, pu64, vp, sz, vp, vp]),
        "sz_encode_paged_batched": (i32, [i32, i32, vp, ppg, pu64, pvp, psz, vp, sz, vp]),
        "sz_decode_paged_batched": (i32, [i32, i32, pvp, psz, ppg, pu64, vp, sz, vp]),
        "sz_encode_reuse_paged_batched": (i32, [i32, i32, vp, ppg, pu64, pvp, psz, vp, vp, sz, vp]),
        "sz_decode": (i32, [i32, vp, sz, vp, u64, vp, sz, vp]),
        "sz_decode_batched": (i32, [i32, i32, pvp, psz, pvp, pu64, vp, sz, vp]),
        "sz_last_device_status": (i32, [vp, vp]),
        "sz_enable_peer_access": (i32, [i32, i32]),
        "sz_encode_noalloc": (i32, [i32, vp, vp, u64, vp, sz, vp, vp]),
    }
    for name, (res, args) in sigs.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


lib = _load()


class SplitZipError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = int(status)
        super().__init__("%s%s (status %d)" % (where + ": " if where else "",
                                              sz_status_string(status), self.status))


def sz_status_string(status: int) -> str:
    return lib.sz_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != SZ_OK:
        raise SplitZipError(status, where)


def dtype_of(x: torch.Tensor) -> int:
    """Codec dtype of a tensor: bfloat16 -> SZ_BF16, float8_e5m2 -> SZ_FP8_E5M2."""
    if x.dtype == torch.bfloat16:
        return SZ_BF16
    if x.dtype == torch.float8_e5m2:
        return SZ_FP8_E5M2
    raise TypeError("unsupported tensor dtype %s (bfloat16 or float8_e5m2)" % x.dtype)


def elem_bytes(dtype: int) -> int:
    return 2 if dtype == SZ_BF16 else 1


def numel_of(x: torch.Tensor, dtype: int) -> int:
    """Elements of the codec dtype held by a tensor (any torch dtype view)."""
    return x.numel() * x.element_size() // elem_bytes(dtype)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(x: torch.Tensor) -> int:
    """Device address of a tensor's first element; the library reads and writes
    its bytes as one contiguous run, so strided views are refused."""
    if not x.is_contiguous():
        raise ValueError("tensor must be contiguous (the codec addresses its bytes as one run)")
    return x.data_ptr()


def _p(x: torch.Tensor):
    return ctypes.c_void_p(_ptr(x))


def _arr(ctype, values):
    values = list(values)
    return (ctype * len(values))(*values)


# ------------------------------------------------------------------- sizes

def sz_workspace_bytes(dtype: int, n: int) -> int:
    return int(lib.sz_workspace_bytes(dtype, n))


def sz_workspace_bytes_batched(dtype: int, ns) -> int:
    ns = list(ns)
    return int(lib.sz_workspace_bytes_batched(dtype, len(ns), _arr(ctypes.c_uint64, ns)))


def sz_stream_bytes(dtype: int, n: int, E: int) -> int:
    return int(lib.sz_stream_bytes(dtype, n, E))


def sz_max_compressed_size(dtype: int, n: int) -> int:
    return int(lib.sz_max_compressed_size(dtype, n))


def new_workspace(dtype: int, ns, device="cuda", stream=None) -> torch.Tensor:
    """A zero-initialised workspace for a batch with element counts ns."""
    ws = torch.empty(sz_workspace_bytes_batched(dtype, ns), dtype=torch.uint8, device=device)
    sz_workspace_init(ws, stream)
    return ws


def new_plans(T: int, device="cuda") -> torch.Tensor:
    return torch.zeros((T, SZ_HEADER_BYTES), dtype=torch.uint8, device=device)


# ------------------------------------------------------------- the calls

def sz_workspace_init(ws: torch.Tensor, stream=None):
    _check(lib.sz_workspace_init(_p(ws), ws.nbytes, _stream(stream)), "sz_workspace_init")


def sz_plan(dtype: int, x: torch.Tensor, ws: torch.Tensor, plan: torch.Tensor, stream=None):
    _check(lib.sz_plan(dtype, _p(x), numel_of(x, dtype), _p(ws), ws.nbytes, _p(plan),
                       _stream(stream)), "sz_plan")


def sz_plan_batched(dtype: int, xs, ws: torch.Tensor, plans: torch.Tensor, stream=None):
    xs = list(xs)
    T = len(xs)
    _check(lib.sz_plan_batched(dtype, T, _arr(ctypes.c_void_p, [_ptr(x) for x in xs]),
                               _arr(ctypes.c_uint64, [numel_of(x, dtype) for x in xs]),
                               _p(ws), ws.nbytes, _p(plans), _stream(stream)), "sz_plan_batched")


def sz_compressed_size(plan: torch.Tensor, stream=None) -> int:
    out = ctypes.c_uint64(0)
    _check(lib.sz_compressed_size(_p(plan), ctypes.byref(out), _stream(stream)), "sz_compressed_size")
    return int(out.value)


def sz_compressed_sizes(plans: torch.Tensor, stream=None):
    T = plans.shape[0]
    out = (ctypes.c_uint64 * T)()
    _check(lib.sz_compressed_sizes(T, _p(plans), out, _stream(stream)), "sz_compressed_sizes")
    return [int(v) for v in out]


def sz_plan_set_flags(plans: torch.Tensor, flags: int, stream=None):
    """Set the header flags (0 or SZ_FLAG_RAW_BLOCKS) of every plan in `plans`."""
    _check(lib.sz_plan_set_flags(plans.shape[0] if plans.dim() == 2 else 1, _p(plans), int(flags),
                                 _stream(stream)), "sz_plan_set_flags")


def sz_encode(dtype: int, plan: torch.Tensor, x: torch.Tensor, out: torch.Tensor, ws: torch.Tensor,
              stream=None):
    _check(lib.sz_encode(dtype, _p(plan), _p(x), numel_of(x, dtype), _p(out), out.nbytes, _p(ws),
                         ws.nbytes, _stream(stream)), "sz_encode")


def sz_encode_batched(dtype: int, plans: torch.Tensor, xs, outs, ws: torch.Tensor, stream=None):
    xs, outs = list(xs), list(outs)
    T = len(xs)
    _check(lib.sz_encode_batched(
        dtype, T, _p(plans), _arr(ctypes.c_void_p, [_ptr(x) for x in xs]),
        _arr(ctypes.c_uint64, [numel_of(x, dtype) for x in xs]),
        _arr(ctypes.c_void_p, [_ptr(o) for o in outs]),
        _arr(ctypes.c_size_t, [o.nbytes for o in outs]), _p(ws), ws.nbytes, _stream(stream)),
        "sz_encode_batched")


def _opt(t):
    return None if t is None else _p(t)


def sz_encode_reuse(dtype: int, codebook: torch.Tensor, x: torch.Tensor, out: torch.Tensor, ws: torch.Tensor,
                    total: torch.Tensor = None, stream=None):
    """Encode with the codebook of an earlier plan (codebook reuse); `total`, if
    given, is a device int64 tensor that receives the stream's length."""
    _check(lib.sz_encode_reuse(dtype, _p(codebook), _p(x), numel_of(x, dtype), _p(out), out.nbytes, _opt(total),
                               _p(ws), ws.nbytes, _stream(stream)), "sz_encode_reuse")


def sz_encode_reuse_batched(dtype: int, codebooks: torch.Tensor, xs, outs, ws: torch.Tensor,
                            totals: torch.Tensor = None, stream=None):
    """Codebook reuse for a batch: tensor t uses the codebook of plan t of `codebooks`;
    `totals`, if given, is a device int64 tensor of T stream lengths."""
    xs, outs = list(xs), list(outs)
    T = len(xs)
    _check(lib.sz_encode_reuse_batched(
        dtype, T, _p(codebooks), _arr(ctypes.c_void_p, [_ptr(x) for x in xs]),
        _arr(ctypes.c_uint64, [numel_of(x, dtype) for x in xs]),
        _arr(ctypes.c_void_p, [_ptr(o) for o in outs]),
        _arr(ctypes.c_size_t, [o.nbytes for o in outs]), _opt(totals), _p(ws), ws.nbytes, _stream(stream)),
        "sz_encode_reuse_batched")


def paged(dtype: int, pool: torch.Tensor, pages: torch.Tensor, page_elems: int, page_bytes: int = None,
          pool_pages: int = None) -> sz_paged_t:
    """Descriptor of a tensor held in pages of `pool` (a contiguous device tensor):
    `pages` (device int32) lists its page ids in element order, each page holds
    `page_elems` of its elements, and pages are `page_bytes` apart (default
    page_elems x element bytes).  The pool, the page table and the descriptor's
    numbers must stay as they are while a call that uses it runs."""
    if pages.dtype != torch.int32:
        raise TypeError("page ids are int32")
    pb = page_elems * elem_bytes(dtype) if page_bytes is None else int(page_bytes)
    npages = pool.nbytes // pb if pool_pages is None else int(pool_pages)
    d = sz_paged_t(_ptr(pool), _ptr(pages), npages, pb, int(page_elems))
    d._refs = (pool, pages)  # the descriptor keeps the pool and the page table alive
    return d


def _paged_arr(descs):
    descs = list(descs)
    return (sz_paged_t * len(descs))(*descs)


def sz_plan_paged_batched(dtype: int, srcs, ns, ws: torch.Tensor, plans: torch.Tensor, stream=None):
    """Plans of T paged tensors (descriptors from paged(); ns: element counts)."""
    srcs, ns = list(srcs), [int(v) for v in ns]
    _check(lib.sz_plan_paged_batched(dtype, len(srcs), _paged_arr(srcs), _arr(ctypes.c_uint64, ns), _p(ws),
                                     ws.nbytes, _p(plans), _stream(stream)), "sz_plan_paged_batched")


def sz_encode_paged_batched(dtype: int, plans: torch.Tensor, srcs, ns, outs, ws: torch.Tensor, stream=None):
    srcs, ns, outs = list(srcs), [int(v) for v in ns], list(outs)
    _check(lib.sz_encode_paged_batched(dtype, len(srcs), _p(plans), _paged_arr(srcs), _arr(ctypes.c_uint64, ns),
                                       _arr(ctypes.c_void_p, [_ptr(o) for o in outs]),
                                       _arr(ctypes.c_size_t, [o.nbytes for o in outs]), _p(ws), ws.nbytes,
                                       _stream(stream)), "sz_encode_paged_batched")


def sz_encode_reuse_paged_batched(dtype: int, codebooks: torch.Tensor, srcs, ns, outs, ws: torch.Tensor,
                                  totals: torch.Tensor = None, stream=None):
    srcs, ns, outs = list(srcs), [int(v) for v in ns], list(outs)
    _check(lib.sz_encode_reuse_paged_batched(
        dtype, len(srcs), _p(codebooks), _paged_arr(srcs), _arr(ctypes.c_uint64, ns),
        _arr(ctypes.c_void_p, [_ptr(o) for o in outs]), _arr(ctypes.c_size_t, [o.nbytes for o in outs]),
        _opt(totals), _p(ws), ws.nbytes, _stream(stream)), "sz_encode_reuse_paged_batched")


def sz_decode_paged_batched(dtype: int, comps, dsts, ns, ws: torch.Tensor, comp_bytes=None, stream=None):
    comps, dsts, ns = list(comps), list(dsts), [int(v) for v in ns]
    cbs = [c.nbytes for c in comps] if comp_bytes is None else [int(b) for b in comp_bytes]
    _check(lib.sz_decode_paged_batched(dtype, len(comps), _arr(ctypes.c_void_p, [_ptr(c) for c in comps]),
                                       _arr(ctypes.c_size_t, cbs), _paged_arr(dsts), _arr(ctypes.c_uint64, ns),
                                       _p(ws), ws.nbytes, _stream(stream)), "sz_decode_paged_batched")


def sz_decode(dtype: int, comp: torch.Tensor, out: torch.Tensor, ws: torch.Tensor, comp_bytes=None,
              stream=None):
    cb = comp.nbytes if comp_bytes is None else int(comp_bytes)
    _check(lib.sz_decode(dtype, _p(comp), cb, _p(out), numel_of(out, dtype), _p(ws), ws.nbytes,
                         _stream(stream)), "sz_decode")


def sz_decode_batched(dtype: int, comps, outs, ws: torch.Tensor, comp_bytes=None, stream=None):
    comps, outs = list(comps), list(outs)
    T = len(comps)
    cbs = [c.nbytes for c in comps] if comp_bytes is None else [int(b) for b in comp_bytes]
    _check(lib.sz_decode_batched(
        dtype, T, _arr(ctypes.c_void_p, [_ptr(c) for c in comps]), _arr(ctypes.c_size_t, cbs),
        _arr(ctypes.c_void_p, [_ptr(o) for o in outs]),
        _arr(ctypes.c_uint64, [numel_of(o, dtype) for o in outs]), _p(ws), ws.nbytes,
        _stream(stream)), "sz_decode_batched")


class Batch:
    """A fixed batch marshalled once for repeated batched calls.

    The pointer and size arrays of sz_plan_batched / sz_encode_batched /
    sz_decode_batched are built here; plan(), encode() and decode() pass them
    straight to those C entry points.  For KV-cache buffers that stay in place
    across steps this takes the per-call marshalling off the host.  The
    tensors must stay alive and must not move while the Batch is in use.

    xs: the raw tensors (encode input, decode output when decs is None);
    outs: one stream buffer per tensor (encode output, decode input);
    decs: decode outputs (default: xs); comp_bytes: bytes of each stream
    that decode may read (default: the stream buffers' sizes).
    """

    def __init__(self, dtype: int, xs, outs, ws: torch.Tensor, plans: torch.Tensor, decs=None,
                 comp_bytes=None, src_pages=None, dst_pages=None, n=None, raw_blocks=False):
        """src_pages / dst_pages: paged() descriptors of the inputs / decode outputs
        (then xs / decs are not read, and n gives the element counts).
        raw_blocks: plan() marks the plans so that blocks that would expand are
        stored raw (SZ_FLAG_RAW_BLOCKS)."""
        outs = list(outs)
        self._flags = SZ_FLAG_RAW_BLOCKS if raw_blocks else 0
        self._src_pages = None if src_pages is None else _paged_arr(src_pages)
        self._dst_pages = None if dst_pages is None else _paged_arr(dst_pages)
        if src_pages is not None or dst_pages is not None:
            if n is None:
                raise ValueError("paged batches need the element counts n")
            ns = [int(v) for v in n]
            self.dtype, self.T = int(dtype), len(outs)
            self._keep = (xs, outs, decs, ws, plans, src_pages, dst_pages)
            self._n = self._dn = _arr(ctypes.c_uint64, ns)
            self._in = None if xs is None else _arr(ctypes.c_void_p, [_ptr(x) for x in xs])
            self._dec = None if decs is None else _arr(ctypes.c_void_p, [_ptr(d) for d in decs])
            self._out = _arr(ctypes.c_void_p, [_ptr(o) for o in outs])
            self._cap = _arr(ctypes.c_size_t, [o.nbytes for o in outs])
            cbs = [o.nbytes for o in outs] if comp_bytes is None else [int(b) for b in comp_bytes]
            self._cb = _arr(ctypes.c_size_t, cbs)
            self._ws, self._wsb, self._plans = _p(ws), ws.nbytes, _p(plans)
            return
        xs = list(xs)
        decs = xs if decs is None else list(decs)
        if not (len(xs) == len(outs) == len(decs)) or not 1 <= len(xs) <= SZ_MAX_BATCH:
            raise ValueError("xs, outs and decs must have the same length, 1..%d" % SZ_MAX_BATCH)
        if plans.shape[0] < len(xs):
            raise ValueError("one 64-byte plan per tensor")
        self.dtype, self.T = int(dtype), len(xs)
        self._keep = (xs, outs, decs, ws, plans)
        self._in = _arr(ctypes.c_void_p, [_ptr(x) for x in xs])
        self._n = _arr(ctypes.c_uint64, [numel_of(x, dtype) for x in xs])
        self._out = _arr(ctypes.c_void_p, [_ptr(o) for o in outs])
        self._cap = _arr(ctypes.c_size_t, [o.nbytes for o in outs])
        cbs = [o.nbytes for o in outs] if comp_bytes is None else [int(b) for b in comp_bytes]
        self._cb = _arr(ctypes.c_size_t, cbs)
        self._dec = _arr(ctypes.c_void_p, [_ptr(d) for d in decs])
        self._dn = _arr(ctypes.c_uint64, [numel_of(d, dtype) for d in decs])
        self._ws, self._wsb, self._plans = _p(ws), ws.nbytes, _p(plans)

    def plan(self, stream=None):
        if self._src_pages is not None:
            _check(lib.sz_plan_paged_batched(self.dtype, self.T, self._src_pages, self._n, self._ws, self._wsb,
                                             self._plans, _stream(stream)), "sz_plan_paged_batched")
        else:
            _check(lib.sz_plan_batched(self.dtype, self.T, self._in, self._n, self._ws, self._wsb,
                                       self._plans, _stream(stream)), "sz_plan_batched")
        if self._flags:
            _check(lib.sz_plan_set_flags(self.T, self._plans, self._flags, _stream(stream)), "sz_plan_set_flags")

    def encode(self, stream=None):
        if self._src_pages is not None:
            _check(lib.sz_encode_paged_batched(self.dtype, self.T, self._plans, self._src_pages, self._n,
                                               self._out, self._cap, self._ws, self._wsb, _stream(stream)),
                   "sz_encode_paged_batched")
            return
        _check(lib.sz_encode_batched(self.dtype, self.T, self._plans, self._in, self._n, self._out,
                                     self._cap, self._ws, self._wsb, _stream(stream)), "sz_encode_batched")

    def encode_reuse(self, codebooks: torch.Tensor = None, totals: torch.Tensor = None, stream=None):
        """Encode with reused codebooks: plan t of `codebooks` (default: this batch's
        plans, as left by an earlier plan()) for tensor t, no histogram pass."""
        cbs = self._plans if codebooks is None else _p(codebooks)
        if codebooks is not None:
            self._keep_cb = codebooks
        if self._src_pages is not None:
            _check(lib.sz_encode_reuse_paged_batched(self.dtype, self.T, cbs, self._src_pages, self._n, self._out,
                                                     self._cap, _opt(totals), self._ws, self._wsb,
                                                     _stream(stream)), "sz_encode_reuse_paged_batched")
            return
        _check(lib.sz_encode_reuse_batched(self.dtype, self.T, cbs, self._in, self._n, self._out, self._cap,
                                           _opt(totals), self._ws, self._wsb, _stream(stream)),
               "sz_encode_reuse_batched")

    def decode(self, stream=None):
        if self._dst_pages is not None:
            _check(lib.sz_decode_paged_batched(self.dtype, self.T, self._out, self._cb, self._dst_pages, self._dn,
                                               self._ws, self._wsb, _stream(stream)), "sz_decode_paged_batched")
            return
        _check(lib.sz_decode_batched(self.dtype, self.T, self._out, self._cb, self._dec, self._dn,
                                     self._ws, self._wsb, _stream(stream)), "sz_decode_batched")


def sz_enable_peer_access(device: int, peer: int):
    """Let this library's kernels on `device` read `peer`'s memory (see the C header)."""
    _check(lib.sz_enable_peer_access(int(device), int(peer)), "sz_enable_peer_access")


def sz_last_device_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronise; return (and clear) the workspace's device error word."""
    return int(lib.sz_last_device_status(_p(ws), _stream(stream)))


def sz_encode_noalloc(dtype: int, plan: torch.Tensor, x: torch.Tensor, out: torch.Tensor,
                      status: torch.Tensor = None, stream=None):
    """Encode with the library's own scratch (no workspace argument); `status`, if given,
    is a device int32 tensor that receives the call's device error word."""
    _check(lib.sz_encode_noalloc(dtype, _p(plan), _p(x), numel_of(x, dtype), _p(out), out.nbytes,
                                 _p(status) if status is not None else None, _stream(stream)),
           "sz_encode_noalloc")
