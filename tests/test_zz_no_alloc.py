"""The allocation-free decode entry point, for callers that may not allocate
device memory (they cannot create a handle, whose set-up allocates).

It must give the same selection and, within the parity tolerance, the same
output as the handle-based entry point, on two calls in a row (the second
call reuses the library's fixed scratch array left by the first).  This file
is collected last so that a failure here comes after every other test.
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
