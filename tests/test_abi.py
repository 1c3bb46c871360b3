"""The C-ABI library loads and exports every entry point include/basiskv.h
declares; host-side argument validation (no GPU needed)."""
import ctypes
import os
import re

import pytest

from compressed_kv_cache_routing_b200 import basiskv as bk
from compressed_kv_cache_routing_b200 import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "basiskv.h")


def declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"BASISKV_API\s+[\w\s\*]*?\b(basiskv_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return bk.load()


def test_every_declared_symbol_is_exported(lib):
    names = declared()
    assert len(names) >= 10
    assert sorted(bk.EXPORTED) == names
    for n in names:
        assert hasattr(lib, n), n


def test_version(lib):
    hdr = open(HEADER).read()
    assert bk.basiskv_version() == int(re.search(r"#define BASISKV_VERSION (\d+)", hdr).group(1))


def _params(**kw):
    p = bk.basiskv_params()
    base = dict(max_batch=2, num_kv_heads=2, gqa_group=4, head_dim=128, page_size=64, rank_r=32,
                rank_s=16, max_pages_per_seq=8, max_topk=4, num_slots=16, dtype=0, k_format=0,
                z_pool=0x1000, r_pool=0x2000, k_pool=0x3000, w_zk=0x4000, b_r=0x5000, b_v=0x6000)
    base.update(kw)
    for k, v in base.items():
        setattr(p, k, v)
    return p


@pytest.mark.parametrize("bad", [
    dict(max_batch=0), dict(num_kv_heads=0), dict(gqa_group=0), dict(gqa_group=9),
    dict(head_dim=0), dict(page_size=0), dict(rank_r=0), dict(rank_r=129), dict(rank_s=-1),
    dict(max_pages_per_seq=0), dict(max_topk=0), dict(num_slots=0), dict(dtype=7),
    dict(k_format=2), dict(k_format=1), dict(k_format=1, k_scale=0x7008), dict(z_pool=None), dict(k_pool=None), dict(r_pool=None),
    dict(b_v=None), dict(w_zk=0x1001), dict(k_pool=0x3008),
])
def test_create_rejects_bad_params(lib, bad):
    h = ctypes.c_void_p()
    rc = lib.basiskv_create(ctypes.byref(_params(**bad)), ctypes.byref(h))
    assert rc == bk.BASISKV_ERR_INVALID_ARG
    assert h.value is None
    assert lib.basiskv_last_error()


def test_null_handle_calls_fail(lib):
    assert lib.basiskv_destroy(None) == 0
    assert lib.basiskv_decode_attn(None, 1, None, 1, 1.0, None, None, None) == bk.BASISKV_ERR_INVALID_ARG
    assert lib.basiskv_append_page(None, 0, 0, 1, None) == bk.BASISKV_ERR_INVALID_ARG
    st = ctypes.c_uint32()
    assert lib.basiskv_get_status(None, ctypes.byref(st), 0) == bk.BASISKV_ERR_INVALID_ARG
