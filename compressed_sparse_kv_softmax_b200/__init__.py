"""Python binding of libcskv.so (hybrid compressed sparse KV attention for B200).

Argument marshalling only: torch tensors become device pointers and byte
strides, the current torch CUDA stream becomes the launch stream, and every
non-zero status raises `CskvError`.  All computation runs in the library's
CUDA kernels; there is no CPU fallback.  Importing the package without a
built libcskv.so raises ImportError.

With CSKV_CHECK=1 in the environment the package loads the checked build
libcskv_check.so instead (same entry points; its kernels test every index
they read from device memory and record DEV_BOUNDS in the device status word
when one is out of range).  CSKV_SPLITS=<n> makes the attention use n splits
per query row (tuning only; read once by the library).

Cache planes follow the C descriptor (include/cskv.h): for B sequences of
`cap` slots, `data` is [B, cap, ...] with one slot per row; E4M3_BF16 caches
add `scale` [B, cap, >= d_nope/64] fp32 and `rope` [B, cap, d_rope] bf16.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
CHECKED = os.environ.get("CSKV_CHECK", "0") not in ("", "0")
LIB_PATH = os.path.join(_HERE, "libcskv_check.so" if CHECKED else "libcskv.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python compressed_sparse_kv_softmax_b200/build.py"
        f"{' --check' if CHECKED else ''}`")

_lib = ctypes.CDLL(LIB_PATH)

OK, ERR_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_WORKSPACE, ERR_SCRATCH_LIMIT, ERR_DEVICE = (
    0, -1, -2, -3, -4, -5, -6)
# device-side events (bits of cskv_check_device_errors)
DEV_INDEXER_WAIT, DEV_TOPK_BARRIER, DEV_ATTN_WAIT, DEV_ROW_FAILED, DEV_BOUNDS = 1, 2, 4, 8, 16
FMT_F32, FMT_E4M3_BF16, FMT_E4M3_VEC, FMT_MXFP4 = 0, 1, 2, 3
_FMT = {"f32": FMT_F32, "e4m3": FMT_E4M3_BF16, "e4m3vec": FMT_E4M3_VEC, "mxfp4": FMT_MXFP4}


class CskvCache(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("d_nope", ctypes.c_int32), ("d_rope", ctypes.c_int32),
                ("ring", ctypes.c_int32), ("cap", ctypes.c_int64),
                ("data", ctypes.c_void_p), ("data_stride", ctypes.c_int64),
                ("scale", ctypes.c_void_p), ("scale_stride", ctypes.c_int64),
                ("rope", ctypes.c_void_p), ("rope_stride", ctypes.c_int64),
                ("block_table", ctypes.c_void_p), ("block_size", ctypes.c_int64),
                ("num_blocks", ctypes.c_int64)]


_P = ctypes.c_void_p
_PC = ctypes.POINTER(CskvCache)
_I, _I64, _F, _SZ = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t

_lib.csa_compress.argtypes = [_I, _P, _P, _I64, _PC, _PC, _PC, _P, _P, _I, _I, _PC, _PC, _PC, _P]
_lib.hca_compress.argtypes = [_I, _P, _P, _I64, _PC, _PC, _P, _P, _I, _I, _PC, _PC, _P]
_lib.csa_compress_channel_gate.argtypes = [_I, _P, _P, _I64, _PC, _PC, _PC, _P, _P, _P, _P, _I,
                                           _I, _PC, _PC, _PC, _P]
_lib.hca_compress_channel_gate.argtypes = [_I, _P, _P, _I64, _PC, _PC, _P, _P, _I, _I, _PC, _PC,
                                           _P]
_lib.indexer_score.argtypes = _lib.indexer_select.argtypes = [_I, _I, _P, _P, _P, _P, _I, _I, _PC,
                                                             _I, _I, _I64, _P, _P, _P, _SZ, _P]
_lib.indexer_topk.argtypes = [_I, _I, _P, _P, _P, _P, _I, _I, _PC, _I, _I, _I64, _P, _P, _P,
                              _SZ, _P]
_lib.hybrid_attn_decode.argtypes = [_I, _P, _P, _I, _F, _PC, _PC, _I, _P, _I, _I64, _PC, _PC,
                                    _I, _P, _P, _P, _SZ, _P]
_lib.hybrid_attn_prefill.argtypes = [_I, _I, _P, _P, _I, _F, _PC, _PC, _I, _P, _I, _I64, _PC,
                                     _PC, _I, _P, _P, _P, _SZ, _P]
_lib.cskv_indexer_workspace_size.argtypes = [_I, _I, _I64, _I]
_lib.cskv_indexer_workspace_size.restype = _SZ
_lib.cskv_attn_workspace_size.argtypes = [_I, _I, _I, _I, _I64, _I]
_lib.cskv_attn_workspace_size.restype = _SZ
_lib.indexer_topk_noalloc.argtypes = [_I, _I, _P, _P, _P, _P, _I, _I, _PC, _I, _I, _I64, _P,
                                      _P, _P]
_lib.indexer_topk_noalloc.restype = _I
_lib.cskv_noalloc_scratch_bytes.restype = _SZ
_lib.cskv_ring_store.argtypes = [_I, _P, _I, ctypes.POINTER(_PC), ctypes.POINTER(_PC), _P]
_lib.cskv_ring_store.restype = _I
_lib.cskv_check_device_errors.argtypes = [_P, ctypes.POINTER(ctypes.c_uint32)]
_lib.cskv_check_device_errors.restype = _I
_lib.cskv_debug_topk_barrier_spins.argtypes = [ctypes.c_uint32]
_lib.cskv_debug_topk_barrier_spins.restype = ctypes.c_uint32
_lib.cskv_debug_indexer_stall.argtypes = [ctypes.c_uint32]
_lib.cskv_debug_indexer_stall.restype = ctypes.c_uint32
_lib.cskv_error_string.argtypes = [_I]
_lib.cskv_error_string.restype = ctypes.c_char_p
_lib.cskv_version.restype = _I
_lib.cskv_build_checked.restype = _I
for _name in ("csa_compress", "hca_compress", "csa_compress_channel_gate",
              "hca_compress_channel_gate", "indexer_topk", "indexer_score", "indexer_select",
              "hybrid_attn_decode", "hybrid_attn_prefill"):
    getattr(_lib, _name).restype = _I


class CskvError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.cskv_error_string(status).decode()} (status {status})")


def _check(status: int, where: str):
    if status != OK:
        raise CskvError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _slot_bytes(t):
    # bytes between consecutive slots of a [B, cap, ...] plane
    return t.stride(1) * t.element_size()


def cache_struct(c):
    """C descriptor for a cache given as a dict of planes
    {"fmt": "f32"|"e4m3"|"e4m3vec"|"mxfp4", "d_nope", "d_rope", "ring", "cap", "data",
    "scale", "rope"} and, for a paged cache, "block_table", "block_size", "num_blocks"
    (or None).  A CskvCache is returned as it is: callers that pass the same
    cache every step can build its descriptor once."""
    if c is None or isinstance(c, CskvCache):
        return c
    s = CskvCache()
    s.fmt = _FMT[c["fmt"]]
    s.d_nope, s.d_rope = int(c["d_nope"]), int(c["d_rope"])
    s.ring, s.cap = int(bool(c["ring"])), int(c["cap"])
    s.data, s.data_stride = c["data"].data_ptr(), _slot_bytes(c["data"])
    sc, rp = c.get("scale"), c.get("rope")
    if sc is not None:
        s.scale, s.scale_stride = sc.data_ptr(), _slot_bytes(sc)
    if rp is not None:
        s.rope, s.rope_stride = rp.data_ptr(), _slot_bytes(rp)
    bt = c.get("block_table")
    if bt is not None:
        # paged: the planes hold num_blocks x block_size rows shared by all
        # sequences; block_table [B][cap / block_size] int32
        s.block_table, s.block_size = bt.data_ptr(), int(c["block_size"])
        s.num_blocks = int(c["num_blocks"])
    return s


def _ref(s):
    return None if s is None else ctypes.byref(s)


def _ikref(c):
    return ctypes.byref(cache_struct(c))


def _stream(stream):
    if stream is not None:
        return ctypes.c_void_p(stream)
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ring_store_args(B, pos, src, ring, stream=None):
    ss = [cache_struct(c) for c in src]
    rs = [cache_struct(c) for c in ring]
    n = len(ss)
    sp = (_PC * n)(*[ctypes.pointer(c) for c in ss])
    rp = (_PC * n)(*[ctypes.pointer(c) for c in rs])
    return (B, _ptr(pos), n, sp, rp, _stream(stream))


def ring_store(B, pos, src, ring, stream=None):
    """Copies each sequence's new token (slot 0 of every cache in `src`) into
    slot pos[b] % cap of the matching raw ring in `ring` (lists of caches)."""
    _check(_lib.cskv_ring_store(*_ring_store_args(B, pos, src, ring, stream)), "cskv_ring_store")


def indexer_workspace_size(B, Tq, max_entries, k) -> int:
    return int(_lib.cskv_indexer_workspace_size(B, Tq, max_entries, k))


def attn_workspace_size(B, Tq, Hq, Dv, max_entries, window) -> int:
    return int(_lib.cskv_attn_workspace_size(B, Tq, Hq, Dv, max_entries, window))


def workspace(nbytes: int, device="cuda"):
    """A zero-filled uint8 device buffer with at least nbytes past its first
    256-byte boundary (zero-filled so that the first indexer call already
    finds a clean score histogram)."""
    import torch
    return torch.zeros(max(int(nbytes), 1) + 256, dtype=torch.uint8, device=device)


def _ws(ws):
    # returns (aligned pointer, usable bytes)
    p = ws.data_ptr()
    ap = (p + 255) & ~255
    return ctypes.c_void_p(ap), ws.numel() - (ap - p)


# ---- argument marshalling of each call (device pointers, descriptors, sizes)

def _csa_compress_args(B, t_begin, t_end, max_new, raw_k, raw_v, raw_ik, gate_w, gate_b, pool,
                       stride, out_k, out_v, out_ik, stream=None):
    cs = [cache_struct(c) for c in (raw_k, raw_v, raw_ik, out_k, out_v, out_ik)]
    return (B, _ptr(t_begin), _ptr(t_end), int(max_new), _ref(cs[0]), _ref(cs[1]), _ref(cs[2]),
            _ptr(gate_w), _ptr(gate_b), pool, stride, _ref(cs[3]), _ref(cs[4]), _ref(cs[5]),
            _stream(stream))


def _hca_compress_args(B, t_begin, t_end, max_new, raw_k, raw_v, gate_w, gate_b, pool, stride,
                       out_k, out_v, stream=None):
    cs = [cache_struct(c) for c in (raw_k, raw_v, out_k, out_v)]
    return (B, _ptr(t_begin), _ptr(t_end), int(max_new), _ref(cs[0]), _ref(cs[1]),
            _ptr(gate_w), _ptr(gate_b), pool, stride, _ref(cs[2]), _ref(cs[3]), _stream(stream))


def _csa_compress_channel_gate_args(B, t_begin, t_end, max_new, raw_k, raw_v, raw_ik, gate_w,
                                    gate_b, gate_w_ik, gate_b_ik, pool, stride, out_k, out_v,
                                    out_ik, stream=None):
    cs = [cache_struct(c) for c in (raw_k, raw_v, raw_ik, out_k, out_v, out_ik)]
    return (B, _ptr(t_begin), _ptr(t_end), int(max_new), _ref(cs[0]), _ref(cs[1]), _ref(cs[2]),
            _ptr(gate_w), _ptr(gate_b), _ptr(gate_w_ik), _ptr(gate_b_ik), pool, stride,
            _ref(cs[3]), _ref(cs[4]), _ref(cs[5]), _stream(stream))


def _indexer_args(B, Tq, q_pos, q_ik, q_ik_scale, head_w, H_I, d_I, ik, stride, k, max_entries,
                  out_idx, out_score, ws, stream=None):
    wp, wn = _ws(ws)
    return (B, Tq, _ptr(q_pos), _ptr(q_ik), _ptr(q_ik_scale), _ptr(head_w), H_I, d_I,
            _ikref(ik), stride, k, int(max_entries), _ptr(out_idx), _ptr(out_score), wp, wn,
            _stream(stream))


def _attn_decode_args(B, ctx_len, q, Hq, sm_scale, comp_k, comp_v, comp_stride, sel, k,
                      max_entries, win_k, win_v, window, out, lse, ws, stream=None):
    cs = [cache_struct(c) for c in (comp_k, comp_v, win_k, win_v)]
    wp, wn = _ws(ws)
    return (B, _ptr(ctx_len), _ptr(q), Hq, sm_scale, _ref(cs[0]), _ref(cs[1]), comp_stride,
            _ptr(sel), k, int(max_entries), _ref(cs[2]), _ref(cs[3]), window, _ptr(out),
            _ptr(lse), wp, wn, _stream(stream))


def _attn_prefill_args(B, Tq, q_pos, q, Hq, sm_scale, comp_k, comp_v, comp_stride, sel, k,
                       max_entries, win_k, win_v, window, out, lse, ws, stream=None):
    cs = [cache_struct(c) for c in (comp_k, comp_v, win_k, win_v)]
    wp, wn = _ws(ws)
    return (B, Tq, _ptr(q_pos), _ptr(q), Hq, sm_scale, _ref(cs[0]), _ref(cs[1]), comp_stride,
            _ptr(sel), k, int(max_entries), _ref(cs[2]), _ref(cs[3]), window, _ptr(out),
            _ptr(lse), wp, wn, _stream(stream))


_MARSHAL = {
    "csa_compress": _csa_compress_args,
    "hca_compress": _hca_compress_args,
    "csa_compress_channel_gate": _csa_compress_channel_gate_args,
    "hca_compress_channel_gate": _hca_compress_args,
    "indexer_topk": _indexer_args,
    "indexer_score": _indexer_args,
    "indexer_select": _indexer_args,
    "hybrid_attn_decode": _attn_decode_args,
    "hybrid_attn_prefill": _attn_prefill_args,
    "cskv_ring_store": _ring_store_args,
}


class PreparedCall:
    """One library call with its arguments marshalled once.  A decode step
    repeats the same calls on the same buffers every token: where the
    tensors' addresses, the cache descriptors and the stream stay fixed, a
    prepared call skips the marshalling (and calling it is all the host does
    per launch).  prepare("hybrid_attn_decode", *args) takes the arguments of
    the function of that name."""
    __slots__ = ("_fn", "_args", "_name")

    def __init__(self, name, args):
        self._fn, self._args, self._name = getattr(_lib, name), args, name

    def __call__(self):
        rc = self._fn(*self._args)
        if rc != OK:
            raise CskvError(rc, self._name)


def prepare(name, *args, **kw) -> PreparedCall:
    return PreparedCall(name, _MARSHAL[name](*args, **kw))


def csa_compress(*args, **kw):
    _check(_lib.csa_compress(*_csa_compress_args(*args, **kw)), "csa_compress")


def hca_compress(*args, **kw):
    _check(_lib.hca_compress(*_hca_compress_args(*args, **kw)), "hca_compress")


def csa_compress_channel_gate(*args, **kw):
    """csa_compress with one gate per channel: gate_b [pool][D], the indexer
    keys' own gate_w_ik [d_I] and gate_b_ik [pool][d_I]."""
    _check(_lib.csa_compress_channel_gate(*_csa_compress_channel_gate_args(*args, **kw)),
           "csa_compress_channel_gate")


def hca_compress_channel_gate(*args, **kw):
    """hca_compress with one gate per channel: gate_b [pool][D]."""
    _check(_lib.hca_compress_channel_gate(*_hca_compress_args(*args, **kw)),
           "hca_compress_channel_gate")


def indexer_topk(B, Tq, q_pos, q_ik, q_ik_scale, head_w, H_I, d_I, ik, stride, k, max_entries,
                 out_idx, out_score, ws, stream=None):
    _check(_lib.indexer_topk(*_indexer_args(B, Tq, q_pos, q_ik, q_ik_scale, head_w, H_I, d_I,
                                            ik, stride, k, max_entries, out_idx, out_score, ws,
                                            stream)), "indexer_topk")


def indexer_score(B, Tq, q_pos, q_ik, q_ik_scale, head_w, H_I, d_I, ik, stride, k, max_entries,
                  out_idx, out_score, ws, stream=None):
    """First half of indexer_topk: scores and histogram into the workspace."""
    _check(_lib.indexer_score(*_indexer_args(B, Tq, q_pos, q_ik, q_ik_scale, head_w, H_I, d_I,
                                             ik, stride, k, max_entries, out_idx, out_score, ws,
                                             stream)), "indexer_score")


def indexer_select(B, Tq, q_pos, q_ik, q_ik_scale, head_w, H_I, d_I, ik, stride, k, max_entries,
                   out_idx, out_score, ws, stream=None):
    """Second half of indexer_topk: the top-k from the workspace's scores."""
    _check(_lib.indexer_select(*_indexer_args(B, Tq, q_pos, q_ik, q_ik_scale, head_w, H_I, d_I,
                                              ik, stride, k, max_entries, out_idx, out_score, ws,
                                              stream)), "indexer_select")


def indexer_topk_noalloc(B, Tq, q_pos, q_ik, q_ik_scale, head_w, H_I, d_I, ik, stride, k,
                         max_entries, out_idx, out_score, stream=None):
    """indexer_topk without a workspace, for callers that cannot allocate one:
    the library's fixed device scratch array is used instead (see cskv.h).
    Calls that overlap on the GPU share that array and must be serialised."""
    _check(_lib.indexer_topk_noalloc(B, Tq, _ptr(q_pos), _ptr(q_ik), _ptr(q_ik_scale),
                                     _ptr(head_w), H_I, d_I, _ikref(ik), stride, k,
                                     int(max_entries), _ptr(out_idx), _ptr(out_score),
                                     _stream(stream)), "indexer_topk_noalloc")


def noalloc_scratch_bytes() -> int:
    return int(_lib.cskv_noalloc_scratch_bytes())


def hybrid_attn_decode(*args, **kw):
    _check(_lib.hybrid_attn_decode(*_attn_decode_args(*args, **kw)), "hybrid_attn_decode")


def hybrid_attn_prefill(*args, **kw):
    _check(_lib.hybrid_attn_prefill(*_attn_prefill_args(*args, **kw)), "hybrid_attn_prefill")


def check_device_errors(stream=None) -> int:
    """Waits for the stream, then reads and clears the device's sticky event
    bits (DEV_*); returns them (0: nothing recorded).  Raises on a CUDA error."""
    ev = ctypes.c_uint32(0)
    st = _lib.cskv_check_device_errors(_stream(stream), ctypes.byref(ev))
    if st not in (OK, ERR_DEVICE):
        raise CskvError(st, "cskv_check_device_errors")
    return int(ev.value)


def debug_topk_barrier_spins(spins: int) -> int:
    """Polls of the multi-CTA selection's row meeting point before a CTA
    gives up (tests of the failure path); returns the previous setting."""
    return int(_lib.cskv_debug_topk_barrier_spins(int(spins)))


def debug_indexer_stall(polls: int) -> int:
    """Test hook of the failure path (see cskv_debug_indexer_stall): with
    polls > 0 the first scoring CTA misses a tile and its waits run out after
    `polls` polls; 0 switches it off.  Returns the previous setting."""
    return int(_lib.cskv_debug_indexer_stall(int(polls)))


def error_string(status: int) -> str:
    return _lib.cskv_error_string(status).decode()


def version() -> int:
    return int(_lib.cskv_version())


def build_checked() -> bool:
    """True for the checked build (libcskv_check.so, CSKV_CHECK=1)."""
    return bool(_lib.cskv_build_checked())


lib = _lib
