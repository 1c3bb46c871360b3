"""Parity of the CUDA path (through the C ABI) with the float64 oracle.

Selections must match bit for bit; outputs within a row-normalised max
relative error of 2e-3 (max over (b, h) of |y - y*|_inf / |y*|_inf), the
bound for bf16 storage with fp32 accumulation.  Page scores from the routing
kernel are compared too (relative 1e-3).
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

from compressed_kv_cache_routing_b200 import basiskv as bk
from compressed_kv_cache_routing_b200 import workloads as W
from oracle import oracle
from helpers import to_problem

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3
SCORE_TOL = 1e-3


def setup_module():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from compressed_kv_cache_routing_b200 import build
    build.build()


def gpu_decode(w, topk=None, scale=None, kv=None, max_topk=None):
    s = w.spec
    topk = s.topk if topk is None else topk
    scale = s.softmax_scale if scale is None else scale
    own = kv is None
    if own:
        kv = bk.BasisKV.for_workload(w, max_topk=max(topk, max_topk or 0))
    B = len(w.seq_lens)
    out = torch.full((B, s.num_q_heads, s.head_dim), float("nan"), device="cuda")
    sel = torch.full((B, s.num_kv_heads, topk), -7, device="cuda", dtype=torch.int32)
    bk.basiskv_decode_attn(kv.handle, w.q[:B], topk, scale, out, sel)
    torch.cuda.synchronize()
    assert bk.basiskv_get_status(kv.handle, clear=True) == 0
    res = out.cpu().numpy(), sel.cpu().numpy()
    if own:
        kv.close()
    return res


def gpu_decode_latent(w):
    """basiskv_decode_attn_latent: zbar [B][Hq][r] and the selection."""
    s = w.spec
    kv = bk.BasisKV.for_workload(w)
    B = len(w.seq_lens)
    zbar = torch.full((B, s.num_q_heads, s.rank_r), float("nan"), device="cuda")
    sel = torch.full((B, s.num_kv_heads, s.topk), -7, device="cuda", dtype=torch.int32)
    bk.basiskv_decode_attn_latent(kv.handle, w.q[:B], s.topk, s.softmax_scale, zbar, sel)
    torch.cuda.synchronize()
    assert bk.basiskv_get_status(kv.handle, clear=True) == 0
    res = zbar.cpu().numpy(), sel.cpu().numpy()
    kv.close()
    return res


def gpu_scores(w, topk=None):
    s = w.spec
    topk = s.topk if topk is None else topk
    kv = bk.BasisKV.for_workload(w, max_topk=topk)
    B = len(w.seq_lens)
    sc = torch.zeros((B, s.num_kv_heads, w.page_table.shape[1]), device="cuda")
    sel = torch.zeros((B, s.num_kv_heads, topk), device="cuda", dtype=torch.int32)
    bk.basiskv_route(kv.handle, w.q[:B], topk, sc, sel)
    torch.cuda.synchronize()
    assert bk.basiskv_get_status(kv.handle) == 0
    kv.close()
    return sc.cpu().numpy(), sel.cpu().numpy()


def out_error(out, ref, mask=None):
    """Max over rows of |y - y*|_inf / |y*|_inf; rows with y* == 0 must be 0."""
    worst = 0.0
    for idx in np.ndindex(ref.shape[:2]):
        if mask is not None and not mask[idx]:
            continue
        y, ys = out[idx].astype(np.float64), ref[idx]
        den = np.abs(ys).max()
        if den == 0:
            assert np.abs(y).max() == 0, idx
            continue
        worst = max(worst, np.abs(y - ys).max() / den)
    return worst


def unit_rows(w, units):
    m = np.zeros((len(w.seq_lens), w.spec.num_q_heads), bool)
    for u in units:
        b, kvh = divmod(u, w.spec.num_kv_heads)
        m[b, kvh * w.spec.gqa_group:(kvh + 1) * w.spec.gqa_group] = True
    return m


SMALL = {
    "tiny": W.SPECS["tiny"],
    "llama3_8b_decode": W.shrink("llama3_8b_decode", batch=3, len_lo=2500, len_hi=5000, topk=16),
    # units of 64 stages and more take the shared-ring attention kernel (here
    # beside unrouted units of sequences with fewer pages than k)
    "llama_shared_ring": W.shrink("llama3_8b_decode", batch=3, len_lo=2500, len_hi=5000, topk=40),
    "long_context": W.shrink("long_context", batch=2, len_lo=6000, len_hi=9000, topk=32),
    "high_concurrency": W.shrink("high_concurrency", batch=6, len_lo=700, len_hi=1500, topk=8),
    "dense_limit": W.shrink("dense_limit", batch=2, len_lo=900, len_hi=1100, topk=32),
    # shapes outside the compiled tensor-core set run the generic kernels
    "generic_bf16": W.WorkloadSpec("generic_bf16", 2, 3, 3, 96, 24, 20, 12, 4, 300, 500, "bf16",
                                   1 / math.sqrt(96), 0.5, False, 7),
    "gqa8": W.shrink("llama3_8b_decode", batch=2, len_lo=3000, len_hi=4000, topk=12, gqa_group=8,
                     num_kv_heads=4),
    "gqa2": W.shrink("llama3_8b_decode", batch=2, len_lo=3000, len_hi=4000, topk=12, gqa_group=2),
    "gqa1": W.shrink("llama3_8b_decode", batch=2, len_lo=2000, len_hi=3000, topk=10, gqa_group=1),
    # head_dim 64 on the tensor-core kernels (two channels per lane in the fold)
    "head_dim64": W.shrink("llama3_8b_decode", batch=3, len_lo=1500, len_hi=3000, topk=12, head_dim=64,
                           rank_r=16, rank_s=8, page_size=32),
    "fp32_llama_shape": W.shrink("llama3_8b_decode", batch=2, len_lo=1000, len_hi=2000, topk=8,
                                 dtype="f32"),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_parity(name):
    w = W.generate(SMALL[name], device="cuda")
    prob = to_problem(w)
    ref_out, ref_sel, ref_sc, gap = oracle.decode(prob, want_scores=True)
    out, sel = gpu_decode(w)
    assert np.array_equal(sel, ref_sel), name
    err = out_error(out, ref_out)
    print(f"{name}: max row rel err {err:.3e}")
    assert err <= OUT_TOL
    # routing scores of every unit (routing forced even where k >= n_b)
    sc, sel_r = gpu_scores(w)
    _, _, full_sc, _ = oracle.decode(to_problem(w, topk=1), want_scores=True)
    n = w.num_pages
    for b in range(len(n)):
        a, r = sc[b, :, :n[b]], full_sc[b, :, :n[b]]
        assert np.all(np.abs(a - r) <= SCORE_TOL * np.maximum(1.0, np.abs(r))), name
        assert np.all(np.isneginf(sc[b, :, n[b]:]))


def test_claimed_routing_chunks_score_every_page():
    """Units of 512 pages and more: the routing grid hands out a quarter of
    the pages in chunks claimed at run time.  Every page's score must be
    written on every call, whichever warp claims it: the score buffer is
    poisoned before each call, and two calls with different queries on one
    handle must each match the oracle's scores page for page."""
    spec = W.shrink("llama3_8b_decode", batch=3, len_lo=560 * 64, len_hi=700 * 64, topk=16)
    w = W.generate(spec, device="cuda")
    assert w.num_pages.max() >= 512
    kv = bk.BasisKV.for_workload(w, max_topk=16)
    B, n = len(w.seq_lens), w.num_pages
    for call in range(2):
        if call == 1:
            w.q = (w.q * 0.5).contiguous()  # exact in bf16: every score halves, the order stays
        sc = torch.full((B, w.spec.num_kv_heads, w.page_table.shape[1]), float("nan"), device="cuda")
        sel = torch.full((B, w.spec.num_kv_heads, 16), -7, device="cuda", dtype=torch.int32)
        bk.basiskv_route(kv.handle, w.q, 16, sc, sel)
        torch.cuda.synchronize()
        assert bk.basiskv_get_status(kv.handle) == 0
        got = sc.cpu().numpy()
        _, ref_sel, ref_sc, _ = oracle.decode(to_problem(w, topk=16), want_scores=True)
        for b in range(B):
            a, r = got[b, :, :n[b]], ref_sc[b, :, :n[b]]
            assert np.isfinite(a).all(), (call, b)
            assert np.all(np.abs(a - r) <= SCORE_TOL * np.maximum(1.0, np.abs(r))), (call, b)
        assert np.array_equal(sel.cpu().numpy(), ref_sel), call
        out, dsel = gpu_decode(w, kv=kv)
        assert np.array_equal(dsel, ref_sel), call
    kv.close()


FULL = ["tiny", "llama3_8b_decode", "long_context", "high_concurrency", "dense_limit"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled(name):
    """Full workload sizes in the benchmark's launch configuration; the oracle
    checks a sample of units one by one, and every routed unit must pick its
    planted pages (the unique top-k once the margin holds)."""
    w = W.generate(name, device="cuda")
    out, sel = gpu_decode(w)
    s = w.spec
    U = s.batch * s.num_kv_heads
    rng = np.random.default_rng(123)
    units = sorted(set([0, U - 1] + rng.choice(U, size=min(U, 4), replace=False).tolist()))
    prob = to_problem(w)
    ref_out, ref_sel, _, gap = oracle.decode(prob, units=units)
    for u in units:
        b, kvh = divmod(u, s.num_kv_heads)
        assert np.array_equal(sel[b, kvh], ref_sel[b, kvh]), (name, u)
        if min(s.topk, w.num_pages[b]) < w.num_pages[b]:
            assert gap[b, kvh] >= 1e-2
    err = out_error(out, ref_out, unit_rows(w, units))
    print(f"{name}: sampled units {units}: max row rel err {err:.3e}")
    assert err <= OUT_TOL
    for (b, kvh), pages in w.planted.items():
        got = sel[b, kvh][sel[b, kvh] >= 0]
        assert np.array_equal(got, pages), (name, b, kvh)
    assert np.isfinite(out).all()


def _with_lengths(spec, lens, **kw):
    w = W.generate(spec, device="cuda")
    w.seq_lens = np.asarray(lens, np.int32)
    for k, v in kw.items():
        setattr(w, k, v)
    return w


def test_edge_lengths_and_mixed_routing():
    """Empty sequence, one token, exactly one page, one page plus one token,
    and sequences with fewer pages than k next to routed ones."""
    spec = W.shrink("llama3_8b_decode", batch=7, len_lo=4000, len_hi=4000, topk=8)
    w = _with_lengths(spec, [0, 1, 64, 65, 4000, 8 * 64, 8 * 64 + 1])
    prob = to_problem(w)
    ref_out, ref_sel, _, _ = oracle.decode(prob)
    out, sel = gpu_decode(w)
    assert np.array_equal(sel, ref_sel)
    assert (sel[0] == -1).all() and (out[0] == 0).all()
    assert out_error(out, ref_out) <= OUT_TOL


def test_shared_ring_with_many_short_units():
    """Two long sequences take the shared-ring attention kernel (units of 80
    stages); the other 46 sequences have from 0 to 7 pages, so most units
    are unrouted and a few stages long, and a CTA's chunk holds dozens of
    segments."""
    batch = 48
    rng = np.random.default_rng(11)
    lens = rng.integers(0, 7 * 64, size=batch)
    lens[:6] = [0, 1, 64, 65, 5000, 6000]
    spec = W.shrink("llama3_8b_decode", batch=batch, len_lo=6000, len_hi=6000, topk=40)
    w = _with_lengths(spec, lens)
    kv = bk.BasisKV.for_workload(w)
    ref_out, ref_sel, _, _ = oracle.decode(to_problem(w))
    out, sel = gpu_decode(w, kv=kv)
    assert bk.basiskv_last_launch(kv.handle)["attn_shared_ring"] == 1
    kv.close()
    assert np.array_equal(sel, ref_sel)
    assert (sel[0] == -1).all() and (out[0] == 0).all()
    assert out_error(out, ref_out) <= OUT_TOL


def test_topk_one_and_max():
    spec = W.shrink("high_concurrency", batch=3, len_lo=900, len_hi=1400, topk=1)
    w = W.generate(spec, device="cuda")
    for k in (1, 2, 45):
        ref_out, ref_sel, _, _ = oracle.decode(to_problem(w, topk=k))
        out, sel = gpu_decode(w, topk=k)
        assert np.array_equal(sel, ref_sel), k
        assert out_error(out, ref_out) <= OUT_TOL


def test_units_with_many_pages():
    """More than 2048 pages per unit, with exact ties in one sequence."""
    spec = W.shrink("llama3_8b_decode", batch=2, len_lo=2100 * 16, len_hi=2100 * 16 + 15, topk=40, page_size=16)
    w = W.generate(spec, device="cuda")
    pt = w.page_table.copy()
    pt[1, :] = pt[1, np.arange(pt.shape[1]) % 5]     # five distinct pages, repeated: ties everywhere
    w.page_table = pt
    prob = to_problem(w)
    ref_out, ref_sel, _, _ = oracle.decode(prob)
    assert w.num_pages.min() > 2048
    out, sel = gpu_decode(w)
    assert np.array_equal(sel, ref_sel)
    assert out_error(out, ref_out) <= OUT_TOL


def test_batch_past_the_parameter_plan():
    """More than 512 sequences: the work plan is written by the prep grid
    instead of travelling in the kernel parameters."""
    spec = W.shrink("llama3_8b_decode", batch=600, len_lo=1, len_hi=400, topk=3)
    w = W.generate(spec, device="cuda")
    prob = to_problem(w)
    ref_out, ref_sel, _, _ = oracle.decode(prob)
    out, sel = gpu_decode(w)
    assert np.array_equal(sel, ref_sel)
    assert out_error(out, ref_out) <= OUT_TOL


@pytest.mark.parametrize("name", ["llama3_8b_decode", "high_concurrency", "dense_limit", "head_dim64", "tiny",
                                  "generic_bf16"])
def test_latent_output(name):
    """The weighted latent before B_v, on the tensor-core and CUDA-core
    kernels, against the oracle's latent mode."""
    w = W.generate(SMALL[name], device="cuda")
    prob = dataclasses.replace(to_problem(w), latent=True)
    ref_z, ref_sel, _, _ = oracle.decode(prob)
    zbar, sel = gpu_decode_latent(w)
    assert np.array_equal(sel, ref_sel), name
    assert out_error(zbar, ref_z) <= OUT_TOL


def test_latent_output_edge_lengths_and_large_batch():
    """Zero-length sequences get zbar = 0 (r wide) on both the parameter-plan
    path and the prep-grid path (more than 512 sequences)."""
    for spec, lens in [(W.shrink("llama3_8b_decode", batch=5, len_lo=4000, len_hi=4000, topk=8),
                        [0, 1, 65, 4000, 8 * 64]),
                       (W.shrink("llama3_8b_decode", batch=600, len_lo=1, len_hi=400, topk=3), None)]:
        w = _with_lengths(spec, lens) if lens is not None else W.generate(spec, device="cuda")
        if lens is None:
            w.seq_lens[::7] = 0
            w.page_table[::7] = 0
        prob = dataclasses.replace(to_problem(w), latent=True)
        ref_z, ref_sel, _, _ = oracle.decode(prob)
        zbar, sel = gpu_decode_latent(w)
        assert np.array_equal(sel, ref_sel)
        assert out_error(zbar, ref_z) <= OUT_TOL
        empty = np.asarray(w.seq_lens) == 0
        assert (zbar[empty] == 0).all() and (sel[empty] == -1).all()


def test_shared_prefix_pages():
    """Sequences whose page tables point at the same slots for a common prefix
    (pages shared between sequences, as a prompt cache would): each sequence
    routes and attends over its own table; the shared slots are read where
    they are referenced."""
    spec = W.shrink("llama3_8b_decode", batch=4, len_lo=3000, len_hi=4000, topk=12)
    w = W.generate(spec, device="cuda")
    pt = w.page_table.copy()
    prefix = 20
    for b in range(1, 4):
        pt[b, :prefix] = pt[0, :prefix]
    w.page_table = pt
    prob = to_problem(w)
    ref_out, ref_sel, _, _ = oracle.decode(prob)
    out, sel = gpu_decode(w)
    assert np.array_equal(sel, ref_sel)
    assert out_error(out, ref_out) <= OUT_TOL


def test_exact_ties_go_to_lower_page():
    """Logical pages sharing a physical slot score exactly the same."""
    spec = W.shrink("llama3_8b_decode", batch=2, len_lo=64 * 40, len_hi=64 * 40, topk=6)
    w = W.generate(spec, device="cuda")
    pt = w.page_table.copy()
    pt[0, :] = pt[0, 0]                              # every page identical
    pt[1, :] = pt[1, np.arange(pt.shape[1]) % 3]     # three distinct pages, repeated
    w.page_table = pt
    prob = to_problem(w)
    ref_out, ref_sel, sc, gap = oracle.decode(prob, want_scores=True)
    assert (ref_sel[0] == np.arange(6)).all()
    out, sel = gpu_decode(w)
    assert np.array_equal(sel, ref_sel)
    assert out_error(out, ref_out) <= OUT_TOL


def test_deterministic_and_host_entry_point():
    w = W.generate(SMALL["llama3_8b_decode"], device="cuda")
    s = w.spec
    kv = bk.BasisKV.for_workload(w)
    o1, s1 = gpu_decode(w, kv=kv)
    o2, s2 = gpu_decode(w, kv=kv)
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)
    for pinned in (True, False):  # kernels write pinned results in place; pageable ones are copied back
        qh = w.q.cpu()
        oh = torch.full((s.batch, s.num_q_heads, s.head_dim), float("nan"), dtype=torch.float32)
        sh = torch.full((s.batch, s.num_kv_heads, s.topk), -7, dtype=torch.int32)
        if pinned:
            qh, oh, sh = qh.pin_memory(), oh.pin_memory(), sh.pin_memory()
        bk.basiskv_decode_attn_host(kv.handle, qh, s.topk, s.softmax_scale, oh, sh)
        assert np.array_equal(oh.numpy(), o1) and np.array_equal(sh.numpy(), s1)
    kv.close()


def test_two_handles_on_two_streams():
    """Handles keep their own scratch and claim counters: two handles
    decoding on two streams at the same time, several calls each with no
    synchronisation in between, both stay equal to the oracle."""
    ws = [W.generate(W.shrink("llama3_8b_decode", batch=4, len_lo=40000, len_hi=42000, topk=24), device="cuda"),
          W.generate(SMALL["high_concurrency"], device="cuda")]
    kvs = [bk.BasisKV.for_workload(w) for w in ws]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs, sels = [], []
    for w in ws:
        s = w.spec
        outs.append(torch.full((s.batch, s.num_q_heads, s.head_dim), float("nan"), device="cuda"))
        sels.append(torch.full((s.batch, s.num_kv_heads, s.topk), -7, device="cuda", dtype=torch.int32))
    torch.cuda.synchronize()
    for _ in range(5):
        for w, kv, st, o, sl in zip(ws, kvs, streams, outs, sels):
            bk.basiskv_decode_attn(kv.handle, w.q, w.spec.topk, w.spec.softmax_scale, o, sl,
                                   stream=st.cuda_stream)
    torch.cuda.synchronize()
    for w, kv, o, sl in zip(ws, kvs, outs, sels):
        assert bk.basiskv_get_status(kv.handle) == 0
        ref_out, ref_sel, _, _ = oracle.decode(to_problem(w))
        assert np.array_equal(sl.cpu().numpy(), ref_sel)
        assert out_error(o.cpu().numpy(), ref_out) <= OUT_TOL
        kv.close()


def test_incremental_page_table_matches_bulk_load():
    w = W.generate(SMALL["high_concurrency"], device="cuda")
    s = w.spec
    ref_out, ref_sel = gpu_decode(w)
    kv = bk.BasisKV(z_pool=w.z_pool, r_pool=w.r_pool, k_pool=w.k_pool, w_zk=w.w_zk, b_r=w.b_r,
                    b_v=w.b_v, gqa_group=s.gqa_group, max_batch=s.batch,
                    max_pages_per_seq=w.page_table.shape[1], max_topk=s.topk)
    P = s.page_size
    for b, L in enumerate(w.seq_lens.tolist()):
        n = -(-L // P)
        for j in range(n):
            if j == n - 1 and L - j * P < P:
                first = max(1, (L - j * P) // 2)  # partial page: append, then grow it
                bk.basiskv_append_page(kv.handle, b, int(w.page_table[b, j]), first)
                if L - j * P > first:
                    bk.basiskv_append_tokens(kv.handle, b, L - j * P - first)
            else:
                bk.basiskv_append_page(kv.handle, b, int(w.page_table[b, j]), P)
    out, sel = gpu_decode(w, kv=kv)
    assert np.array_equal(out, ref_out) and np.array_equal(sel, ref_sel)
    partial = [b for b, L in enumerate(w.seq_lens.tolist()) if L % P]
    assert partial, "the workload should have a sequence ending in a partial page"
    with pytest.raises(bk.BasisKVError) as e:
        bk.basiskv_append_page(kv.handle, partial[0], 0, 1)
    assert e.value.code == bk.BASISKV_ERR_STATE
    bk.basiskv_reset_seq(kv.handle, 0)
    out2, sel2 = gpu_decode(w, kv=kv)
    assert (sel2[0] == -1).all() and (out2[0] == 0).all()
    assert np.array_equal(out2[1:], ref_out[1:]) and np.array_equal(sel2[1:], ref_sel[1:])
    kv.close()


def test_invalid_calls_rejected():
    w = W.generate(SMALL["tiny"], device="cuda")
    kv = bk.BasisKV.for_workload(w)
    out = torch.empty((1, 4, 64), device="cuda")
    for topk in (0, -1, w.spec.topk + 1):
        with pytest.raises(bk.BasisKVError) as e:
            bk.basiskv_decode_attn(kv.handle, w.q, topk, 0.1, out)
        assert e.value.code == bk.BASISKV_ERR_INVALID_ARG
    with pytest.raises(bk.BasisKVError):
        bk.basiskv_load_page_table(kv.handle, np.full((1, 64), 10 ** 6), np.array([1024]))
    kv.close()


def _rebuilt_by_copy(w, k_pool, k_scale=None):
    """A handle over empty pools filled page by page with
    basiskv_append_page_copy from w's pools (same slots)."""
    s = w.spec
    z2, r2, k2 = torch.zeros_like(w.z_pool), torch.zeros_like(w.r_pool), torch.zeros_like(k_pool)
    sc2 = torch.zeros_like(k_scale) if k_scale is not None else None
    kv = bk.BasisKV(z_pool=z2, r_pool=r2, k_pool=k2, w_zk=w.w_zk, b_r=w.b_r, b_v=w.b_v, gqa_group=s.gqa_group,
                    max_batch=s.batch, max_pages_per_seq=w.page_table.shape[1], max_topk=s.topk, k_scale=sc2)
    P = s.page_size
    for b, L in enumerate(w.seq_lens.tolist()):
        for j in range(-(-L // P)):
            slot, n = int(w.page_table[b, j]), min(P, L - j * P)
            bk.basiskv_append_page_copy(kv.handle, b, slot, w.z_pool[slot, :, :n].contiguous(),
                                        w.r_pool[slot, :, :n].contiguous(), k_pool[slot, :, :n].contiguous(),
                                        k_scale[slot, :, :n].contiguous() if k_scale is not None else None)
    return kv


@pytest.mark.parametrize("int8", [False, True])
def test_append_page_copy_matches_prefilled_pools(int8):
    """Pages copied into empty pools by basiskv_append_page_copy decode to
    the same bits as the same pages written in place."""
    w = W.generate(SMALL["llama3_8b_decode"], device="cuda")
    s = w.spec
    if int8:
        k_pool = torch.empty(tuple(w.k_pool.shape), dtype=torch.int8, device="cuda")
        k_scale = torch.empty(tuple(w.k_pool.shape[:3]), device="cuda")
        ref = bk.BasisKV(z_pool=w.z_pool, r_pool=w.r_pool, k_pool=k_pool, w_zk=w.w_zk, b_r=w.b_r, b_v=w.b_v,
                         gqa_group=s.gqa_group, max_batch=s.batch, max_pages_per_seq=w.page_table.shape[1],
                         max_topk=s.topk, k_scale=k_scale)
        bk.basiskv_quantize_keys(ref.handle, w.k_pool)
        bk.basiskv_load_page_table(ref.handle, np.where(w.page_table >= 0, w.page_table, 0), w.seq_lens)
    else:
        k_pool, k_scale = w.k_pool, None
        ref = bk.BasisKV.for_workload(w)
    kv = _rebuilt_by_copy(w, k_pool, k_scale)
    outs = []
    for h in (ref, kv):
        out = torch.empty((s.batch, s.num_q_heads, s.head_dim), device="cuda")
        sel = torch.empty((s.batch, s.num_kv_heads, s.topk), device="cuda", dtype=torch.int32)
        bk.basiskv_decode_attn(h.handle, w.q, s.topk, s.softmax_scale, out, sel)
        torch.cuda.synchronize()
        assert bk.basiskv_get_status(h.handle) == 0
        outs.append((out.cpu(), sel.cpu()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    kv.close()
    ref.close()


def test_append_page_copy_refused_copies_nothing():
    w = W.generate(SMALL["llama3_8b_decode"], device="cuda")
    s = w.spec
    z2, r2, k2 = torch.zeros_like(w.z_pool), torch.zeros_like(w.r_pool), torch.zeros_like(w.k_pool)
    kv = bk.BasisKV(z_pool=z2, r_pool=r2, k_pool=k2, w_zk=w.w_zk, b_r=w.b_r, b_v=w.b_v, gqa_group=s.gqa_group,
                    max_batch=s.batch, max_pages_per_seq=4, max_topk=s.topk)
    zs, rs, ks = w.z_pool[0, :, :5].contiguous(), w.r_pool[0, :, :5].contiguous(), w.k_pool[0, :, :5].contiguous()
    bk.basiskv_append_page_copy(kv.handle, 0, 1, zs, rs, ks)          # a partial page: the sequence ends here
    with pytest.raises(bk.BasisKVError):
        bk.basiskv_append_page_copy(kv.handle, 0, 2, zs, rs, ks)      # appending after a partial page
    torch.cuda.synchronize()
    assert torch.count_nonzero(z2[2]) == 0 and torch.count_nonzero(k2[2]) == 0
    assert torch.equal(z2[1, :, :5], zs) and torch.count_nonzero(z2[1, :, 5:]) == 0
    kv.close()


# ---- near the selection margin ---------------------------------------------
# The planted pages sit just above the best unplanted page (gap >= 1e-2 in
# float64 on the stored bits, typically 0.05), the regime where a routing
# score error could move a page across the k-th boundary.
NEAR = ["tiny", "llama3_8b_decode", "llama_shared_ring", "long_context", "high_concurrency", "generic_bf16",
        "gqa8", "gqa2", "gqa1", "head_dim64", "fp32_llama_shape"]


def _near(spec):
    from margin import OracleScorer
    return W.generate(spec, device="cuda", scorer=OracleScorer())


def _check_margin(w, gap):
    n = w.num_pages
    gaps = [gap[b, h] for (b, h) in w.planted]
    assert gaps and min(gaps) >= W.MARGIN and max(gaps) <= 1.0, (min(gaps), max(gaps))
    return min(gaps)


@pytest.mark.parametrize("name", NEAR)
def test_small_parity_near_margin(name):
    w = _near(SMALL[name])
    prob = to_problem(w)
    ref_out, ref_sel, _, gap = oracle.decode(prob)
    g = _check_margin(w, gap)
    out, sel = gpu_decode(w)
    assert np.array_equal(sel, ref_sel), name
    err = out_error(out, ref_out)
    print(f"{name}: smallest gap {g:.4f}, max row rel err {err:.3e}")
    assert err <= OUT_TOL


@pytest.mark.parametrize("name", ["llama3_8b_decode", "long_context", "high_concurrency"])
def test_full_size_near_margin(name):
    """Full workload sizes, in the benchmark's launch configuration, with the
    planted pages just above the boundary: the selection of EVERY unit equals
    the oracle's (which equals the planted set), every routed unit's gap lies
    in [1e-2, 1], and sampled units' outputs match the oracle."""
    w = _near(W.SPECS[name])
    out, sel = gpu_decode(w)
    s = w.spec
    prob = to_problem(w)
    _, ref_sel_all, gap_all = oracle.route(prob)
    g = _check_margin(w, gap_all)
    assert np.array_equal(sel, ref_sel_all), name
    for (b, kvh), pages in w.planted.items():
        assert np.array_equal(sel[b, kvh][sel[b, kvh] >= 0], pages), (name, b, kvh)
    U = s.batch * s.num_kv_heads
    rng = np.random.default_rng(321)
    units = sorted(set([0, U - 1] + rng.choice(U, size=min(U, 4), replace=False).tolist()))
    ref_out, ref_sel, _, _ = oracle.decode(prob, units=units)
    err = out_error(out, ref_out, unit_rows(w, units))
    print(f"{name}: smallest gap {g:.4f} over {len(w.planted)} units; sampled units {units}: "
          f"max row rel err {err:.3e}")
    assert err <= OUT_TOL
