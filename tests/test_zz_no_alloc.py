"""The allocation-free decode entry point, for callers that may not allocate
device memory (they cannot create a handle, whose set-up allocates).

It must give the same selection and, within the parity tolerance, the same
output as the handle-based entry point and as the float64 oracle, on two
calls in a row (the second call reuses the library's fixed scratch array left
by the first).  Faults in the device-side page table and lengths, which the
host never sees, must be reported by its status reader.  This file is
collected last so that a failure here comes after every other test.
"""
import numpy as np
import pytest
import torch

from compressed_kv_cache_routing_b200 import basiskv as bk
from compressed_kv_cache_routing_b200 import workloads as W

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3


def _row_err(out, ref):
    worst = 0.0
    for idx in np.ndindex(ref.shape[:2]):
        den = np.abs(ref[idx]).max()
        if den == 0:
            assert np.abs(out[idx]).max() == 0
            continue
        worst = max(worst, np.abs(out[idx].astype(np.float64) - ref[idx]).max() / den)
    return worst


@pytest.mark.parametrize("spec", [
    W.shrink("llama3_8b_decode", batch=3, len_lo=2500, len_hi=5000, topk=16),
    W.SPECS["tiny"],
], ids=["llama3_shape_bf16", "tiny_fp32"])
def test_noalloc_matches_handle_entry_point(spec):
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    from compressed_kv_cache_routing_b200 import build
    build.build()
    w = W.generate(spec, device="cuda")
    s = w.spec
    B = s.batch
    kv = bk.BasisKV.for_workload(w)
    ref_out = torch.empty((B, s.num_q_heads, s.head_dim), device="cuda")
    ref_sel = torch.empty((B, s.num_kv_heads, s.topk), device="cuda", dtype=torch.int32)
    bk.basiskv_decode_attn(kv.handle, w.q, s.topk, s.softmax_scale, ref_out, ref_sel)
    torch.cuda.synchronize()
    params = kv.params  # same pools, bases and shapes; no handle is used below

    table = torch.as_tensor(np.where(w.page_table >= 0, w.page_table, 0), dtype=torch.int32,
                            device="cuda").contiguous()
    lens = torch.as_tensor(w.seq_lens, dtype=torch.int32, device="cuda")
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        sel = torch.full_like(ref_sel, -7)
        bk.basiskv_decode_attn_noalloc(params, table, lens, w.q, s.topk, s.softmax_scale, out, sel)
        torch.cuda.synchronize()
        assert torch.equal(sel, ref_sel), f"selection differs on call {call}"
        err = _row_err(out.cpu().numpy(), ref_out.cpu().numpy().astype(np.float64))
        assert err <= OUT_TOL, f"call {call}: max row relative error {err:.3e}"
    kv.close()


def test_noalloc_rejects_oversize_request():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    w = W.generate(W.SPECS["tiny"], device="cuda")
    kv = bk.BasisKV.for_workload(w)
    p = bk.basiskv_params.from_buffer_copy(kv.params)
    p.max_batch = 4096
    p.max_pages_per_seq = 4096  # 4096 sequences x 4096 pages of scores: far above the scratch
    B = 4096
    table = torch.zeros((B, 4096), dtype=torch.int32, device="cuda")
    lens = torch.zeros(B, dtype=torch.int32, device="cuda")
    q = torch.zeros((B, 4, 64), device="cuda")
    out = torch.zeros((B, 4, 64), device="cuda")
    with pytest.raises(bk.BasisKVError) as e:
        bk.basiskv_decode_attn_noalloc(p, table, lens, q, 8, 0.125, out)
    assert e.value.code == bk.BASISKV_ERR_CAPACITY
    assert "scratch" in str(e.value)
    kv.close()


def _noalloc(params, w, table=None, lens=None, topk=None):
    s = w.spec
    topk = s.topk if topk is None else topk
    B = len(w.seq_lens)
    if table is None:
        table = torch.as_tensor(np.where(w.page_table >= 0, w.page_table, 0), dtype=torch.int32,
                                device="cuda").contiguous()
    if lens is None:
        lens = torch.as_tensor(w.seq_lens, dtype=torch.int32, device="cuda")
    out = torch.full((B, s.num_q_heads, s.head_dim), float("nan"), device="cuda")
    sel = torch.full((B, s.num_kv_heads, topk), -7, device="cuda", dtype=torch.int32)
    bk.basiskv_decode_attn_noalloc(params, table, lens, w.q, topk, s.softmax_scale, out, sel)
    torch.cuda.synchronize()
    return out.cpu().numpy(), sel.cpu().numpy(), bk.basiskv_noalloc_status()


def _params(w, k_pool=None, k_scale=None, max_topk=None):
    s = w.spec
    kv = bk.BasisKV(z_pool=w.z_pool, r_pool=w.r_pool, k_pool=w.k_pool if k_pool is None else k_pool,
                    w_zk=w.w_zk, b_r=w.b_r, b_v=w.b_v, gqa_group=s.gqa_group, max_batch=s.batch,
                    max_pages_per_seq=w.page_table.shape[1], max_topk=max_topk or s.topk, k_scale=k_scale)
    p = bk.basiskv_params.from_buffer_copy(kv.params)
    return kv, p


def test_noalloc_matches_oracle_with_int8_keys_and_ragged_lengths():
    """Directly against the oracle: bf16 keys and int8 keys (the device
    quantiser's codes, equal to the oracle's), on a batch holding an empty
    sequence, a one-token sequence, sequences with no more pages than top-k
    (every page used, identity selection) and routed ones."""
    from oracle import oracle
    from helpers import to_problem
    from test_gpu_int8_keys import oracle_int8
    spec = W.shrink("llama3_8b_decode", batch=6, len_lo=3000, len_hi=3000, topk=8)
    w = W.generate(spec, device="cuda")
    w.seq_lens = np.array([0, 1, 8 * 64, 5 * 64 + 3, 3000, 2900], np.int32)
    for int8 in (False, True):
        if int8:
            codes = torch.empty(tuple(w.k_pool.shape), dtype=torch.int8, device="cuda")
            scales = torch.empty(tuple(w.k_pool.shape[:3]), device="cuda")
            kv, p = _params(w, codes, scales)
            bk.basiskv_quantize_keys(kv.handle, w.k_pool)
            torch.cuda.synchronize()
            prob = oracle_int8(w)
            assert np.array_equal(codes.cpu().numpy(), prob.k_pool)
        else:
            kv, p = _params(w)
            prob = to_problem(w)
        ref_out, ref_sel, _, _ = oracle.decode(prob)
        for call in range(2):
            out, sel, status = _noalloc(p, w)
            assert status == 0, (int8, call, status)
            assert np.array_equal(sel, ref_sel), (int8, call)
            assert (sel[0] == -1).all() and (out[0] == 0).all()
            assert (sel[2] == np.arange(8)).all() and (sel[3, :, 6:] == -1).all()
            assert _row_err(out, ref_out) <= OUT_TOL, (int8, call)
        kv.close()


def test_noalloc_reports_bad_slot_and_overlong_length():
    """A page-table entry outside the pool and a length longer than a table
    row are seen only on the device: the call stays inside its buffers,
    reports them through basiskv_noalloc_status, and the next good call
    clears the bits and is correct again."""
    spec = W.shrink("llama3_8b_decode", batch=3, len_lo=2000, len_hi=2000, topk=8)
    w = W.generate(spec, device="cuda")
    kv, p = _params(w)
    ref_out, ref_sel, status = _noalloc(p, w)
    assert status == 0
    table = torch.as_tensor(np.where(w.page_table >= 0, w.page_table, 0), dtype=torch.int32, device="cuda")
    bad = table.clone()
    bad[1, 3] = w.num_slots + 5
    out, sel, status = _noalloc(p, w, table=bad)
    assert status & bk.BASISKV_STATUS_BAD_SLOT
    assert np.array_equal(out[0], ref_out[0]) and np.array_equal(sel[2], ref_sel[2])
    lens = torch.as_tensor(w.seq_lens, dtype=torch.int32, device="cuda").clone()
    lens[2] = (w.page_table.shape[1] + 7) * spec.page_size  # more pages than a row holds
    out, sel, status = _noalloc(p, w, lens=lens)
    assert status & bk.BASISKV_STATUS_BAD_LENGTH
    assert np.isfinite(out).all() and ((sel >= -1) & (sel < w.page_table.shape[1])).all()
    assert np.array_equal(out[:2], ref_out[:2]) and np.array_equal(sel[:2], ref_sel[:2])
    out, sel, status = _noalloc(p, w)
    assert status == 0 and np.array_equal(out, ref_out) and np.array_equal(sel, ref_sel)
    kv.close()


def test_noalloc_scratch_formula():
    """The byte count in the rejection message equals the header's formula
    batch * Hkv * (8 + 4 * max_pages + 4 * topk + 4 * min(16, topk) * G * (r + 2)),
    each piece rounded up to 256 bytes."""
    import re
    w = W.generate(W.SPECS["tiny"], device="cuda")
    kv, p = _params(w)
    a256 = lambda x: (x + 255) // 256 * 256
    for B, pages, topk in ((8192, 300, 8), (2000, 1000, 40)):
        p.max_batch, p.max_pages_per_seq, p.max_topk = B, pages, topk
        table = torch.zeros((B, pages), dtype=torch.int32, device="cuda")
        lens = torch.zeros(B, dtype=torch.int32, device="cuda")
        q = torch.zeros((B, 4, 64), device="cuda")
        out = torch.zeros((B, 4, 64), device="cuda")
        with pytest.raises(bk.BasisKVError) as e:
            bk.basiskv_decode_attn_noalloc(p, table, lens, q, topk, 0.125, out)
        assert e.value.code == bk.BASISKV_ERR_CAPACITY
        need = int(re.search(r"needs (\d+) bytes", str(e.value)).group(1))
        U, G, r, sp = B * 1, 4, 16, min(16, topk)
        formula = a256(4) + a256(8 * U) + a256(4 * U * pages) + a256(4 * U * topk) + \
            a256(4 * U * sp * G * 2) + a256(4 * U * sp * G * r)
        assert need == formula, (need, formula)
    kv.close()
