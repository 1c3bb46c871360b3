"""The seeded input generator: shapes, determinism, junk placement, and the
planted score margin at the k boundary (checked with the oracle)."""
import numpy as np
import pytest
import torch

from compressed_kv_cache_routing_b200 import workloads as W
from oracle import oracle
from helpers import to_problem

SMALL = {
    "tiny": W.SPECS["tiny"],
    "llama3_8b_decode": W.shrink("llama3_8b_decode", batch=2, len_lo=4096, len_hi=4096, topk=16),
    "long_context": W.shrink("long_context", batch=2, len_lo=3000, len_hi=5000, topk=16),
    "high_concurrency": W.shrink("high_concurrency", batch=3, len_lo=700, len_hi=1500),
    "dense_limit": W.shrink("dense_limit", batch=2, len_lo=1000, len_hi=1000, topk=16),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_shapes_and_determinism(name):
    spec = SMALL[name]
    a = W.generate(spec)
    b = W.generate(spec)
    for f in ("q", "z_pool", "r_pool", "k_pool", "w_zk", "b_r", "b_v"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f
    assert np.array_equal(a.page_table, b.page_table)
    s = spec
    assert a.q.shape == (s.batch, s.num_q_heads, s.head_dim)
    assert a.z_pool.shape == (a.num_slots, s.num_kv_heads, s.page_size, s.rank_r)
    assert a.r_pool.shape == (a.num_slots, s.num_kv_heads, s.page_size, s.rank_s)
    assert a.k_pool.shape == (a.num_slots, s.num_kv_heads, s.page_size, s.head_dim)
    assert ((a.seq_lens >= s.len_lo) & (a.seq_lens <= s.len_hi)).all()
    st = torch.bfloat16 if s.dtype == "bf16" else torch.float32
    assert a.q.dtype == st and a.k_pool.dtype == st
    # every referenced slot distinct and in range; tails and spare slots hold junk
    n = a.num_pages
    used = np.concatenate([a.page_table[b, :n[b]] for b in range(s.batch)])
    assert len(set(used.tolist())) == len(used) and used.min() >= 0 and used.max() < a.num_slots
    for b in range(s.batch):
        tail = int(a.seq_lens[b]) - (int(n[b]) - 1) * s.page_size
        if tail < s.page_size:
            sl = a.page_table[b, n[b] - 1]
            assert (a.k_pool[sl, :, tail:] == W.JUNK).all()
            assert (a.k_pool[sl, :, tail - 1] != W.JUNK).any()
    spare = np.setdiff1d(np.arange(a.num_slots), used)
    assert spare.size >= 1 and (a.z_pool[torch.as_tensor(spare)] == W.JUNK).all()
    if s.dense:
        assert torch.equal(a.b_v[0], torch.eye(s.rank_r))


@pytest.mark.parametrize("name", ["tiny", "llama3_8b_decode", "long_context", "high_concurrency"])
def test_planted_margin(name):
    """The k planted pages are exactly the selection and the float64 gap at
    the k boundary is at least 1e-2 on every (sequence, KV head)."""
    w = W.generate(SMALL[name])
    prob = to_problem(w)
    _, sel, gap = oracle.route(prob)
    n = w.num_pages
    checked = 0
    for b in range(w.spec.batch):
        for kvh in range(w.spec.num_kv_heads):
            if min(w.spec.topk, n[b]) < n[b]:
                assert gap[b, kvh] >= 1e-2
                got = sel[b, kvh][sel[b, kvh] >= 0]
                assert np.array_equal(got, w.planted[(b, kvh)])
                checked += 1
    assert checked > 0


def test_algorithmic_bytes_llama_formula():
    """2 L (r+s) + 2 k P (d+r) bytes per (sequence, KV head) for bf16."""
    w = W.generate(SMALL["llama3_8b_decode"])
    s = w.spec
    per_unit = 2 * 4096 * (32 + 16) + 2 * 16 * 64 * (128 + 32)
    assert w.algorithmic_bytes()["total"] == per_unit * s.batch * s.num_kv_heads


@pytest.mark.parametrize("name", ["tiny", "llama3_8b_decode", "long_context", "high_concurrency"])
def test_near_margin_plant(name):
    """The near-margin plant puts the planted pages just above the k-th
    boundary: they are exactly the oracle's selection and every routed unit's
    float64 gap lies in [1e-2, 1] (delta ~ U(0.05, 0.5), doubled only where
    rounding left a page short)."""
    from margin import OracleScorer
    w = W.generate(SMALL[name], scorer=OracleScorer())
    prob = to_problem(w)
    _, sel, gap = oracle.route(prob)
    n = w.num_pages
    gaps = []
    for b in range(w.spec.batch):
        for kvh in range(w.spec.num_kv_heads):
            if min(w.spec.topk, n[b]) < n[b]:
                got = sel[b, kvh][sel[b, kvh] >= 0]
                assert np.array_equal(got, w.planted[(b, kvh)])
                gaps.append(gap[b, kvh])
    assert gaps and min(gaps) >= W.MARGIN and max(gaps) <= 1.0
    # the strong plant's margin is far wider on the same draws
    _, _, gap_strong = oracle.route(to_problem(W.generate(SMALL[name])))
    assert np.nanmin(gap_strong[np.isfinite(gap_strong)]) > 5 * max(gaps)


def test_near_margin_plant_only_moves_planted_rows():
    """Both plants draw the same lengths, tables, bases, queries and latents;
    the residuals and keys differ only in the planted rows."""
    from margin import OracleScorer
    spec = SMALL["llama3_8b_decode"]
    a = W.generate(spec)
    b = W.generate(spec, scorer=OracleScorer())
    for f in ("q", "z_pool", "w_zk", "b_r", "b_v"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f
    assert np.array_equal(a.page_table, b.page_table)
    diff_r = (a.r_pool != b.r_pool).any(-1)
    diff_k = (a.k_pool != b.k_pool).any(-1)
    planted_rows = torch.zeros_like(diff_r)
    P = spec.page_size
    for (bb, kvh), pages in b.planted.items():
        for j in pages.tolist():
            slot = int(b.page_table[bb, j])
            planted_rows[slot, kvh] |= diff_r[slot, kvh]
    assert not (diff_r & ~planted_rows).any()
    assert int(diff_r.sum()) == sum(len(p) for p in b.planted.values())
    assert not (diff_k & ~diff_r).any()
