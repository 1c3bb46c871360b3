"""BasisKV float64 CPU oracle -- TEST INFRASTRUCTURE ONLY.

Thin ctypes wrapper over ``basiskv_oracle.c`` (plain C, float64 loops).  Only
the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
use it; the CUDA library never imports, links or calls anything here, and the
two share no code.

What it computes follows "BasisKV: Value Latents for Communication and Key
Routing", English abstract: routing keys predicted from the Value latents plus
a Key-specific residual (Khat = Z.W_zk + R.B_r), page selection by those keys,
then exact QK softmax attention over the selected pages only, with values held
as latents and expanded by B_v.  The C source's header lists the readings
taken where the abstract is silent.

Inputs are host numpy arrays holding the *stored* values: bf16 pools and
queries as their raw 16-bit patterns (``np.uint16``/``np.int16``), fp32 as
``np.float32``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "basiskv_oracle.c")
_LIB = os.path.join(_HERE, "libbasiskv_oracle.so")

BF16 = 0
F32 = 1
KEYS_NATIVE = 0
KEYS_INT8 = 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP, -O2, IEEE arithmetic)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Problem(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
        ("gqa_group", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("page_size", ctypes.c_int32), ("rank_r", ctypes.c_int32),
        ("rank_s", ctypes.c_int32), ("topk", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("num_slots", ctypes.c_int32),
        ("ld_pt", ctypes.c_int32), ("latent", ctypes.c_int32),
        ("k_format", ctypes.c_int32),
        ("softmax_scale", ctypes.c_double),
        ("q", ctypes.c_void_p), ("z_pool", ctypes.c_void_p),
        ("r_pool", ctypes.c_void_p), ("k_pool", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p),
        ("w_zk", ctypes.c_void_p), ("b_r", ctypes.c_void_p), ("b_v", ctypes.c_void_p),
        ("page_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
        ("unit_mask", ctypes.c_void_p),
    ]


_lib = None


def lib(path: str | None = None):
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if path is not None:
        l = ctypes.CDLL(path)
    elif _lib is not None:
        return _lib
    else:
        l = ctypes.CDLL(build())
    P = ctypes.POINTER(_Problem)
    vp = ctypes.c_void_p
    l.oracle_route.argtypes = [P, vp, vp, vp]
    l.oracle_attend.argtypes = [P, vp, vp]
    l.oracle_decode.argtypes = [P, ctypes.c_int, vp, vp, vp, vp]
    for f in (l.oracle_route, l.oracle_attend, l.oracle_decode):
        f.restype = ctypes.c_int
    l.oracle_max_threads.restype = ctypes.c_int
    l.oracle_set_threads.argtypes = [ctypes.c_int]
    if path is None:
        _lib = l
    return l


@dataclass
class Problem:
    """One decode step's stored inputs, host side.

    Layouts: q [B][Hkv*G][d]; z_pool [slots][Hkv][P][r]; r_pool [slots][Hkv][P][s];
    k_pool [slots][Hkv][P][d]; w_zk [Hkv][r][d], b_r [Hkv][s][d], b_v [Hkv][r][d]
    (fp32); page_table [B][ld_pt] int32; seq_lens [B] int32.
    With ``k_scale`` [slots][Hkv][P] float32 given, k_pool holds int8 key
    codes and the key of a row is its scale times its codes.
    """
    q: np.ndarray
    z_pool: np.ndarray
    r_pool: np.ndarray
    k_pool: np.ndarray
    w_zk: np.ndarray
    b_r: np.ndarray
    b_v: np.ndarray
    page_table: np.ndarray
    seq_lens: np.ndarray
    gqa_group: int
    topk: int
    softmax_scale: float
    dtype: int  # BF16 (raw 16-bit patterns) or F32
    latent: bool = False  # outputs zbar [B][Hq][r] (before B_v) instead of [B][Hq][d]
    k_scale: np.ndarray | None = None  # per-token key scales: k_pool holds int8 codes

    def __post_init__(self):
        conv = (lambda a: np.ascontiguousarray(a).view(np.uint16)) if self.dtype == BF16 else \
            (lambda a: np.ascontiguousarray(a, dtype=np.float32))
        self.q = conv(self.q)
        self.z_pool = conv(self.z_pool)
        self.r_pool = conv(self.r_pool)
        if self.k_scale is None:
            self.k_pool = conv(self.k_pool)
        else:
            if np.asarray(self.k_pool).dtype != np.int8:
                raise ValueError("with k_scale, k_pool must hold int8 codes")
            self.k_pool = np.ascontiguousarray(self.k_pool)
            self.k_scale = np.ascontiguousarray(self.k_scale, dtype=np.float32)
            if self.k_scale.shape != self.k_pool.shape[:3]:
                raise ValueError("k_scale must be [slots][Hkv][P]")
        self.w_zk = np.ascontiguousarray(self.w_zk, dtype=np.float32)
        self.b_r = np.ascontiguousarray(self.b_r, dtype=np.float32)
        self.b_v = np.ascontiguousarray(self.b_v, dtype=np.float32)
        self.page_table = np.ascontiguousarray(self.page_table, dtype=np.int32)
        self.seq_lens = np.ascontiguousarray(self.seq_lens, dtype=np.int32)
        if self.page_table.ndim != 2:
            raise ValueError("page_table must be [B][ld_pt]")

    @property
    def batch(self):
        return int(self.seq_lens.shape[0])

    @property
    def num_kv_heads(self):
        return int(self.z_pool.shape[1])

    @property
    def head_dim(self):
        return int(self.k_pool.shape[3])

    @property
    def page_size(self):
        return int(self.z_pool.shape[2])

    @property
    def rank_r(self):
        return int(self.z_pool.shape[3])

    @property
    def rank_s(self):
        return int(self.r_pool.shape[3]) if self.r_pool.ndim == 4 else 0

    def _struct(self, unit_mask=None) -> _Problem:
        p = _Problem()
        p.batch = self.batch
        p.num_kv_heads = self.num_kv_heads
        p.gqa_group = self.gqa_group
        p.head_dim = self.head_dim
        p.page_size = self.page_size
        p.rank_r = self.rank_r
        p.rank_s = self.rank_s
        p.topk = self.topk
        p.dtype = self.dtype
        p.num_slots = int(self.z_pool.shape[0])
        p.ld_pt = int(self.page_table.shape[1])
        p.latent = int(bool(self.latent))
        p.k_format = KEYS_NATIVE if self.k_scale is None else KEYS_INT8
        p.softmax_scale = float(self.softmax_scale)
        p.q = self.q.ctypes.data
        p.z_pool = self.z_pool.ctypes.data
        p.r_pool = self.r_pool.ctypes.data if self.r_pool.size else None
        p.k_pool = self.k_pool.ctypes.data
        p.k_scale = self.k_scale.ctypes.data if self.k_scale is not None else None
        p.w_zk = self.w_zk.ctypes.data
        p.b_r = self.b_r.ctypes.data if self.b_r.size else None
        p.b_v = self.b_v.ctypes.data
        p.page_table = self.page_table.ctypes.data
        p.seq_lens = self.seq_lens.ctypes.data
        p.unit_mask = unit_mask.ctypes.data if unit_mask is not None else None
        return p


def _mask(prob: Problem, units):
    if units is None:
        return None
    m = np.zeros(prob.batch * prob.num_kv_heads, dtype=np.uint8)
    m[np.asarray(units, dtype=np.int64)] = 1
    return m


def route(prob: Problem, units=None, library=None):
    """Page scores [B][Hkv][ld_pt] (-inf past n_b), selection [B][Hkv][topk]
    (ascending, -1 padded) and the ranked gap S_(k) - S_(k+1) [B][Hkv]."""
    U = prob.batch * prob.num_kv_heads
    scores = np.full((prob.batch, prob.num_kv_heads, prob.page_table.shape[1]), -np.inf)
    sel = np.full((prob.batch, prob.num_kv_heads, prob.topk), -1, dtype=np.int32)
    gap = np.full((prob.batch, prob.num_kv_heads), np.nan)
    mask = _mask(prob, units)  # must outlive the call: the struct holds its address
    st = prob._struct(mask)
    l = library if library is not None else lib()
    rc = l.oracle_route(ctypes.byref(st), scores.ctypes.data, sel.ctypes.data, gap.ctypes.data)
    if rc:
        raise ValueError(f"oracle_route failed: {rc}")
    assert U == sel.shape[0] * sel.shape[1]
    return scores, sel, gap


def attend(prob: Problem, sel: np.ndarray, units=None, library=None):
    """Exact attention over the pages in ``sel``; out [B][Hkv*G][d] float64
    ([B][Hkv*G][r], the latent before B_v, when ``prob.latent``)."""
    sel = np.ascontiguousarray(sel, dtype=np.int32)
    out = np.zeros((prob.batch, prob.num_kv_heads * prob.gqa_group, prob.rank_r if prob.latent else prob.head_dim))
    mask = _mask(prob, units)  # must outlive the call: the struct holds its address
    st = prob._struct(mask)
    l = library if library is not None else lib()
    rc = l.oracle_attend(ctypes.byref(st), sel.ctypes.data, out.ctypes.data)
    if rc:
        raise ValueError(f"oracle_attend failed: {rc}")
    return out


def decode(prob: Problem, units=None, want_scores=False, library=None):
    """The whole decode step.  Returns (out [B][Hq][d] f64 ([B][Hq][r] when
    ``prob.latent``), sel, scores, gap)."""
    scores = np.full((prob.batch, prob.num_kv_heads, prob.page_table.shape[1]), -np.inf)
    sel = np.full((prob.batch, prob.num_kv_heads, prob.topk), -1, dtype=np.int32)
    gap = np.full((prob.batch, prob.num_kv_heads), np.nan)
    out = np.zeros((prob.batch, prob.num_kv_heads * prob.gqa_group, prob.rank_r if prob.latent else prob.head_dim))
    mask = _mask(prob, units)  # must outlive the call: the struct holds its address
    st = prob._struct(mask)
    l = library if library is not None else lib()
    rc = l.oracle_decode(ctypes.byref(st), int(bool(want_scores)), scores.ctypes.data,
                         sel.ctypes.data, gap.ctypes.data, out.ctypes.data)
    if rc:
        raise ValueError(f"oracle_decode failed: {rc}")
    return out, sel, scores, gap


def _round_to_storage(x: np.ndarray, dtype: int) -> np.ndarray:
    """float64 -> the stored value as float64: fp32, or bf16 by rounding the
    fp32 value to nearest, ties to even (on its bit pattern)."""
    f = np.asarray(x, dtype=np.float32)
    if dtype == F32:
        return f.astype(np.float64)
    bits = f.view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) >> 16 << 16
    return bits.astype(np.uint32).view(np.float32).astype(np.float64)


def encode(k: np.ndarray, v: np.ndarray, w_zk: np.ndarray, b_r: np.ndarray, b_v: np.ndarray, dtype: int):
    """The stored rows for incoming keys and values ("BasisKV: Value Latents
    for Communication and Key Routing", English abstract: values are kept as
    rank-r latents, and a Key-specific residual holds what the Value latent
    cannot predict).  Least-squares reading, per KV head:
        Z = V . pinv(B_v)                          (the latent nearest to V)
        R = (K - Z_stored . W_zk) . pinv(B_r)      (the residual of the stored latent)
    k, v: [Hkv][n][d]; returns (Z [Hkv][n][r], R [Hkv][n][s]) as the stored
    values (rounded to ``dtype``), in float64."""
    v = np.asarray(v, dtype=np.float64)
    Z = np.stack([_round_to_storage(v[h] @ np.linalg.pinv(b_v[h].astype(np.float64)), dtype)
                  for h in range(v.shape[0])])
    return Z, encode_residual(k, Z, w_zk, b_r, dtype)


def encode_residual(k: np.ndarray, z: np.ndarray, w_zk: np.ndarray, b_r: np.ndarray, dtype: int):
    """The residual rows R = (K - Z . W_zk) . pinv(B_r), rounded to ``dtype``,
    for the stored latents ``z`` [Hkv][n][r]; [Hkv][n][s] float64."""
    k = np.asarray(k, dtype=np.float64)
    s = b_r.shape[1] if b_r.size else 0
    R = np.zeros(k.shape[:2] + (s,))
    for h in range(k.shape[0]):
        if s:
            res = k[h] - np.asarray(z[h], dtype=np.float64) @ w_zk[h].astype(np.float64)
            R[h] = _round_to_storage(res @ np.linalg.pinv(b_r[h].astype(np.float64)), dtype)
    return R


def quantize_keys(k: np.ndarray):
    """int8 codes and per-row scales of keys k [..., d] (the stored values,
    as float32 or float64 that float32 holds exactly).

    Lossy key compression in the manner of "PackKV: Reducing KV Cache Memory
    Footprint through LLM-Aware Lossy Compression" (abstract: keys are stored
    compressed, and decompression is folded into the attention product),
    read as symmetric int8 with one scale per token:
        scale = max_c |k_c| / 127        (IEEE float32 division)
        code  = rint(k_c / scale)        (float32 division, ties to even)
    so the largest entry maps to +-127 and a row of zeros has scale 0 and
    codes 0.  Every step is done in float32, the precision the decision is
    taken in.  Returns (codes int8 [..., d], scales float32 [...])."""
    k = np.asarray(k)
    kf = k.astype(np.float32)
    if not np.array_equal(kf.astype(np.float64), np.asarray(k, dtype=np.float64)):
        raise ValueError("keys must be exactly representable in float32")
    amax = np.abs(kf).max(axis=-1)
    scale = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    q = np.rint((kf / safe[..., None]).astype(np.float32))
    q = np.where(scale[..., None] > 0, q, 0)
    return np.clip(q, -127, 127).astype(np.int8), scale


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(lib().oracle_max_threads())
