"""ctypes binding of the BasisKV sm_100a library (``include/basiskv.h``).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of ``libbasiskv.so``.  torch supplies device memory (``data_ptr``) and
the current stream.  There is no fallback: if the shared library is missing or
no sm_100 device is present, the calls raise.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbasiskv.so")

BASISKV_OK = 0
BASISKV_ERR_INVALID_ARG = -1
BASISKV_ERR_OOM = -2
BASISKV_ERR_CUDA = -3
BASISKV_ERR_UNSUPPORTED = -4
BASISKV_ERR_CAPACITY = -5
BASISKV_ERR_STATE = -6

BASISKV_STATUS_BAD_SLOT = 1
BASISKV_STATUS_TIMEOUT = 2
BASISKV_STATUS_BAD_PAGE = 4
BASISKV_STATUS_PART_OVERFLOW = 8
BASISKV_STATUS_BAD_LENGTH = 16
BASISKV_STATUS_DEBUG_BOUNDS = 32  # debug build only

BASISKV_DTYPE_BF16 = 0
BASISKV_DTYPE_F32 = 1

BASISKV_KEYS_NATIVE = 0
BASISKV_KEYS_INT8 = 1

# every entry point declared in include/basiskv.h
EXPORTED = (
    "basiskv_create", "basiskv_destroy", "basiskv_append_page", "basiskv_append_tokens",
    "basiskv_reset_seq", "basiskv_load_page_table", "basiskv_decode_attn",
    "basiskv_decode_attn_host", "basiskv_route", "basiskv_get_status", "basiskv_profile_begin",
    "basiskv_profile_end", "basiskv_last_launch", "basiskv_last_error", "basiskv_version",
    "basiskv_decode_attn_noalloc", "basiskv_decode_attn_latent", "basiskv_encode_rows",
    "basiskv_quantize_keys", "basiskv_encode_tokens", "basiskv_append_page_copy",
    "basiskv_noalloc_status",
)


class basiskv_params(ctypes.Structure):
    _fields_ = [
        ("max_batch", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
        ("gqa_group", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("page_size", ctypes.c_int32), ("rank_r", ctypes.c_int32),
        ("rank_s", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32),
        ("max_topk", ctypes.c_int32), ("num_slots", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("k_format", ctypes.c_int32),
        ("z_pool", ctypes.c_void_p), ("r_pool", ctypes.c_void_p), ("k_pool", ctypes.c_void_p),
        ("w_zk", ctypes.c_void_p), ("b_r", ctypes.c_void_p), ("b_v", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p),
    ]


class BasisKVError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"basiskv error {code}: {msg}")
        self.code = code


_lib = None


def load(path: str = LIB_PATH):
    """Load libbasiskv.so and declare its signatures.  Raises if missing."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m compressed_kv_cache_routing_b200.build`")
    lib = ctypes.CDLL(path)
    H = ctypes.c_void_p
    i32, vp, f32 = ctypes.c_int, ctypes.c_void_p, ctypes.c_float
    sigs = {
        "basiskv_create": [ctypes.POINTER(basiskv_params), ctypes.POINTER(ctypes.c_void_p)],
        "basiskv_destroy": [H],
        "basiskv_append_page": [H, i32, i32, i32, vp],
        "basiskv_append_page_copy": [H, i32, i32, i32, vp, vp, vp, vp, vp],
        "basiskv_append_tokens": [H, i32, i32, vp],
        "basiskv_reset_seq": [H, i32, vp],
        "basiskv_load_page_table": [H, i32, vp, i32, vp, vp],
        "basiskv_decode_attn": [H, i32, vp, i32, f32, vp, vp, vp],
        "basiskv_decode_attn_host": [H, i32, vp, i32, f32, vp, vp, vp],
        "basiskv_decode_attn_latent": [H, i32, vp, i32, f32, vp, vp, vp],
        "basiskv_encode_rows": [H, i32, i32, i32, vp, vp, vp],
        "basiskv_quantize_keys": [H, vp, ctypes.c_int64, ctypes.c_int64, vp],
        "basiskv_encode_tokens": [H, i32, vp, vp, vp, vp, vp],
        "basiskv_route": [H, i32, vp, i32, vp, vp, vp],
        "basiskv_get_status": [H, ctypes.POINTER(ctypes.c_uint32), i32],
        "basiskv_profile_begin": [H, i32],
        "basiskv_profile_end": [H, vp, ctypes.POINTER(ctypes.c_int)],
        "basiskv_last_launch": [H, ctypes.POINTER(ctypes.c_int * 6)],
        "basiskv_version": [],
        "basiskv_decode_attn_noalloc": [ctypes.POINTER(basiskv_params), i32, vp, vp, vp, i32, f32, vp,
                                        vp, vp],
        "basiskv_noalloc_status": [ctypes.POINTER(ctypes.c_uint32)],
    }
    for name, args in sigs.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.basiskv_last_error.argtypes = []
    lib.basiskv_last_error.restype = ctypes.c_char_p
    if path == LIB_PATH:
        _lib = lib
    return lib


def _check(rc: int) -> None:
    if rc != BASISKV_OK:
        raise BasisKVError(rc, load().basiskv_last_error().decode())


def _stream(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t) -> int | None:
    if t is None:
        return None
    return int(t.data_ptr()) if t.numel() else None


# ---- thin wrappers with the C names --------------------------------------
def basiskv_create(params: basiskv_params) -> int:
    h = ctypes.c_void_p()
    _check(load().basiskv_create(ctypes.byref(params), ctypes.byref(h)))
    return h.value


def basiskv_destroy(h: int) -> None:
    _check(load().basiskv_destroy(h))


def basiskv_append_page(h, seq, slot, n_tokens, stream=None):
    _check(load().basiskv_append_page(h, seq, slot, n_tokens, _stream(stream)))


def basiskv_append_page_copy(h, seq, slot, z, r, k, k_scale=None, stream=None):
    """Copy one page's rows (z [Hkv][n][r], r [Hkv][n][s] or None, k
    [Hkv][n][d], k_scale [Hkv][n] with int8 keys) into pool slot ``slot``
    and append it to sequence ``seq`` with n valid tokens."""
    _check(load().basiskv_append_page_copy(h, seq, slot, int(z.shape[1]), _ptr(z), _ptr(r), _ptr(k), _ptr(k_scale),
                                           _stream(stream)))


def basiskv_append_tokens(h, seq, n_tokens, stream=None):
    _check(load().basiskv_append_tokens(h, seq, n_tokens, _stream(stream)))


def basiskv_reset_seq(h, seq, stream=None):
    _check(load().basiskv_reset_seq(h, seq, _stream(stream)))


def basiskv_load_page_table(h, page_table: np.ndarray, seq_lens: np.ndarray, stream=None):
    pt = np.ascontiguousarray(page_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    _check(load().basiskv_load_page_table(h, int(sl.shape[0]), pt.ctypes.data, int(pt.shape[1]),
                                          sl.ctypes.data, _stream(stream)))


def basiskv_decode_attn(h, q, topk, softmax_scale, out, sel_out=None, stream=None, batch=None):
    b = int(q.shape[0]) if batch is None else batch
    _check(load().basiskv_decode_attn(h, b, _ptr(q), topk, float(softmax_scale), _ptr(out),
                                      _ptr(sel_out), _stream(stream)))


def basiskv_decode_attn_latent(h, q, topk, softmax_scale, zbar_out, sel_out=None, stream=None, batch=None):
    """zbar_out [batch][Hq][r] fp32: the softmax-weighted latent, before B_v."""
    b = int(q.shape[0]) if batch is None else batch
    _check(load().basiskv_decode_attn_latent(h, b, _ptr(q), topk, float(softmax_scale), _ptr(zbar_out),
                                             _ptr(sel_out), _stream(stream)))


def basiskv_encode_rows(h, slot, row0, k, v, stream=None):
    """Encode k, v [Hkv][n][d] (pool dtype, device) into rows [row0, row0+n)
    of pool slot ``slot``: K as given, Z and R by least squares."""
    _check(load().basiskv_encode_rows(h, slot, row0, int(k.shape[1]), _ptr(k), _ptr(v), _stream(stream)))


def basiskv_encode_tokens(h, slots, rows, k, v, stream=None):
    """Encode k, v [n][Hkv][d] (pool dtype, device) into row rows[i] of pool
    slot slots[i] (device int32 tensors [n]) for every token i, one launch."""
    _check(load().basiskv_encode_tokens(h, int(k.shape[0]), _ptr(slots), _ptr(rows), _ptr(k), _ptr(v),
                                        _stream(stream)))


def basiskv_quantize_keys(h, k, row0=0, stream=None):
    """Quantise keys k [n][d] (pool dtype, device; any leading shape whose
    rows follow the pool's flat row order) into the handle's int8 key pool
    and scales, rows [row0, row0 + n)."""
    n = int(k.numel() // k.shape[-1]) if k.numel() else 0
    _check(load().basiskv_quantize_keys(h, _ptr(k), int(row0), n, _stream(stream)))


def basiskv_decode_attn_host(h, q_host, topk, softmax_scale, out_host, sel_host=None, stream=None):
    """q_host, out_host, sel_host: host torch tensors (pinned for async copies)."""
    _check(load().basiskv_decode_attn_host(h, int(q_host.shape[0]), _ptr(q_host), topk,
                                           float(softmax_scale), _ptr(out_host), _ptr(sel_host),
                                           _stream(stream)))


def basiskv_route(h, q, topk, scores_out=None, sel_out=None, stream=None):
    _check(load().basiskv_route(h, int(q.shape[0]), _ptr(q), topk, _ptr(scores_out), _ptr(sel_out),
                                _stream(stream)))


def basiskv_get_status(h, clear=False) -> int:
    st = ctypes.c_uint32()
    _check(load().basiskv_get_status(h, ctypes.byref(st), int(bool(clear))))
    return st.value


def basiskv_profile_begin(h, max_calls):
    _check(load().basiskv_profile_begin(h, max_calls))


def basiskv_profile_end(h, max_calls):
    """Per recorded call: dict of arrays (ms) for the prep, routing,
    selection and attention grids and the whole call."""
    ms = np.zeros((max(max_calls, 1), 5), np.float32)
    n = ctypes.c_int()
    _check(load().basiskv_profile_end(h, ms.ctypes.data, ctypes.byref(n)))
    ms = ms[:n.value]
    return {"prep": ms[:, 0], "route": ms[:, 1], "select": ms[:, 2], "attn": ms[:, 3], "total": ms[:, 4]}


def basiskv_last_launch(h):
    info = (ctypes.c_int * 6)()
    _check(load().basiskv_last_launch(h, ctypes.byref(info)))
    keys = ("route_pages_per_cta", "route_ctas", "attn_splits", "attn_ctas", "route_tensor_core",
            "attn_tensor_core")
    d = dict(zip(keys, list(info)))
    d["attn_shared_ring"] = int(d["attn_tensor_core"] == 2)  # 1: a ring per warp, 2: one per CTA
    d["attn_tensor_core"] = int(d["attn_tensor_core"] > 0)
    return d


def basiskv_decode_attn_noalloc(params, page_table, seq_lens, q, topk, softmax_scale, out,
                                sel_out=None, stream=None):
    """Decode step without a handle or any device allocation (see basiskv.h):
    for callers that may not allocate device memory.  ``page_table`` and
    ``seq_lens`` are device int32 tensors; the library's fixed scratch array
    is shared by all calls, so calls must not overlap on the GPU."""
    import torch
    batch = int(seq_lens.shape[0])
    if seq_lens.dtype != torch.int32 or seq_lens.dim() != 1 or not seq_lens.is_contiguous():
        raise ValueError("seq_lens must be a contiguous int32 vector [batch]")
    if (page_table.dtype != torch.int32 or not page_table.is_contiguous()
            or tuple(page_table.shape) != (batch, params.max_pages_per_seq)):
        raise ValueError(f"page_table must be contiguous int32 [{batch}][{params.max_pages_per_seq}]"
                         " (the row length is params.max_pages_per_seq)")
    _check(load().basiskv_decode_attn_noalloc(ctypes.byref(params), batch,
                                              _ptr(page_table), _ptr(seq_lens), _ptr(q), topk,
                                              float(softmax_scale), _ptr(out), _ptr(sel_out),
                                              _stream(stream)))


def basiskv_noalloc_status() -> int:
    """Status bits of the last allocation-free call on the current device
    (synchronises the device)."""
    st = ctypes.c_uint32()
    _check(load().basiskv_noalloc_status(ctypes.byref(st)))
    return st.value


def basiskv_version() -> int:
    return load().basiskv_version()


# ---- convenience object over a workload's device tensors -------------------
class BasisKV:
    """Owns one library handle bound to a set of device pools and bases.

    ``pools`` must stay alive (and unmodified during calls) for the handle's
    lifetime; the object keeps references to them.
    """

    def __init__(self, *, z_pool, r_pool, k_pool, w_zk, b_r, b_v, gqa_group, max_batch,
                 max_pages_per_seq, max_topk, k_scale=None):
        """An int8 ``k_pool`` holds key codes and needs ``k_scale``
        [slots][Hkv][P] fp32 (BASISKV_KEYS_INT8)."""
        import torch
        if not torch.cuda.is_available():
            raise RuntimeError("no CUDA device: the BasisKV library has no CPU path")
        bf16 = z_pool.dtype == torch.bfloat16
        int8_keys = k_pool.dtype == torch.int8
        if int8_keys != (k_scale is not None):
            raise ValueError("int8 keys and k_scale go together")
        self._keep = (z_pool, r_pool, k_pool, w_zk, b_r, b_v, k_scale)
        p = basiskv_params()
        p.max_batch = max_batch
        p.num_kv_heads = int(z_pool.shape[1])
        p.gqa_group = gqa_group
        p.head_dim = int(k_pool.shape[3])
        p.page_size = int(z_pool.shape[2])
        p.rank_r = int(z_pool.shape[3])
        p.rank_s = int(r_pool.shape[3])
        p.max_pages_per_seq = max_pages_per_seq
        p.max_topk = max_topk
        p.num_slots = int(z_pool.shape[0])
        p.dtype = BASISKV_DTYPE_BF16 if bf16 else BASISKV_DTYPE_F32
        p.k_format = BASISKV_KEYS_INT8 if int8_keys else BASISKV_KEYS_NATIVE
        p.k_scale = _ptr(k_scale)
        p.z_pool = _ptr(z_pool)
        p.r_pool = _ptr(r_pool)
        p.k_pool = _ptr(k_pool)
        p.w_zk = _ptr(w_zk)
        p.b_r = _ptr(b_r)
        p.b_v = _ptr(b_v)
        self.params = p
        self.handle = basiskv_create(p)

    @classmethod
    def for_workload(cls, w, max_topk=None):
        s = w.spec
        obj = cls(z_pool=w.z_pool, r_pool=w.r_pool, k_pool=w.k_pool, w_zk=w.w_zk, b_r=w.b_r,
                  b_v=w.b_v, gqa_group=s.gqa_group, max_batch=s.batch,
                  max_pages_per_seq=max(1, w.page_table.shape[1]),
                  max_topk=max_topk if max_topk is not None else max(s.topk, 1))
        basiskv_load_page_table(obj.handle, np.where(w.page_table >= 0, w.page_table, 0), w.seq_lens)
        return obj

    def close(self):
        if getattr(self, "handle", None):
            basiskv_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
