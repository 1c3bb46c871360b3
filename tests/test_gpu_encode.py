"""basiskv_encode_rows against the oracle's least-squares encode, and the
whole pipeline: pages encoded on the device from raw keys and values, then
decoded, against the oracle run on the same pools."""
import dataclasses

import numpy as np
import pytest
import torch

from compressed_kv_cache_routing_b200 import basiskv as bk
from compressed_kv_cache_routing_b200 import workloads as W
from oracle import oracle
from helpers import to_problem, widen

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3


def _host(t, bf16):
    t = t.detach().cpu().contiguous()
    return t.view(torch.int16).numpy().view(np.uint16) if bf16 else t.numpy()


@pytest.mark.parametrize("name,dtype", [("llama3_8b_decode", "bf16"), ("llama3_8b_decode", "f32"),
                                        ("high_concurrency", "bf16")])
def test_encode_rows_matches_oracle(name, dtype):
    spec = W.shrink(name, batch=2, len_lo=600, len_hi=900, topk=4, dtype=dtype)
    w = W.generate(spec, device="cuda")
    s = w.spec
    bf16 = dtype == "bf16"
    kv = bk.BasisKV.for_workload(w)
    g = torch.Generator(device="cuda").manual_seed(11)
    tdt = torch.bfloat16 if bf16 else torch.float32
    slot = w.z_pool.shape[0] - 1
    for row0, n in [(0, s.page_size), (3, 5)]:
        k = torch.randn((s.num_kv_heads, n, s.head_dim), generator=g, device="cuda").to(tdt)
        v = torch.randn((s.num_kv_heads, n, s.head_dim), generator=g, device="cuda").to(tdt)
        bk.basiskv_encode_rows(kv.handle, slot, row0, k, v)
        torch.cuda.synchronize()
        Zr, Rr = oracle.encode(widen(_host(k, bf16), oracle.BF16 if bf16 else oracle.F32),
                               widen(_host(v, bf16), oracle.BF16 if bf16 else oracle.F32),
                               w.w_zk.cpu().numpy(), w.b_r.cpu().numpy(), w.b_v.cpu().numpy(),
                               oracle.BF16 if bf16 else oracle.F32)
        dt = oracle.BF16 if bf16 else oracle.F32
        Kg = widen(_host(w.k_pool[slot, :, row0:row0 + n], bf16), dt)
        Zg = widen(_host(w.z_pool[slot, :, row0:row0 + n], bf16), dt)
        Rg = widen(_host(w.r_pool[slot, :, row0:row0 + n], bf16), dt)
        assert np.array_equal(Kg, widen(_host(k, bf16), dt))  # keys stored as given
        # fp32 arithmetic against float64: one bf16 step, or fp32 dot-product
        # error; the residual is checked against the latent the device stored
        Rr = oracle.encode_residual(widen(_host(k, bf16), dt), Zg, w.w_zk.cpu().numpy(), w.b_r.cpu().numpy(), dt)
        step, floor = (2.0 ** -7, 2.0 ** -9) if bf16 else (1e-5, 1e-4)
        for got, ref in ((Zg, Zr), (Rg, Rr)):
            assert np.all(np.abs(got - ref) <= step * np.abs(ref) + floor * np.abs(ref).max()), (row0, n)
    assert bk.basiskv_get_status(kv.handle) == 0
    kv.close()


def test_encode_then_decode():
    """Every page of every sequence encoded on the device from raw K and V,
    then decoded (all pages selected, so no routing near-ties): the outputs
    match the oracle on the pools the device wrote, and V is reproduced
    through the latents as far as its projection on B_v allows."""
    spec = W.shrink("llama3_8b_decode", batch=2, len_lo=700, len_hi=1000, topk=64)
    w = W.generate(spec, device="cuda")
    s = w.spec
    kv = bk.BasisKV.for_workload(w)
    g = torch.Generator(device="cuda").manual_seed(5)
    for b in range(s.batch):
        L = int(w.seq_lens[b])
        for j in range(-(-L // s.page_size)):
            n = min(s.page_size, L - j * s.page_size)
            k = torch.randn((s.num_kv_heads, n, s.head_dim), generator=g, device="cuda").to(torch.bfloat16)
            v = torch.randn((s.num_kv_heads, n, s.head_dim), generator=g, device="cuda").to(torch.bfloat16)
            bk.basiskv_encode_rows(kv.handle, int(w.page_table[b, j]), 0, k, v)
    out = torch.empty((s.batch, s.num_q_heads, s.head_dim), device="cuda")
    sel = torch.empty((s.batch, s.num_kv_heads, s.topk), device="cuda", dtype=torch.int32)
    bk.basiskv_decode_attn(kv.handle, w.q, s.topk, s.softmax_scale, out, sel)
    torch.cuda.synchronize()
    assert bk.basiskv_get_status(kv.handle) == 0
    ref_out, ref_sel, _, _ = oracle.decode(to_problem(w))   # the pools as the device left them
    assert np.array_equal(sel.cpu().numpy(), ref_sel)
    o, r = out.cpu().numpy().astype(np.float64), ref_out
    for bb in range(s.batch):
        for h in range(s.num_q_heads):
            assert np.abs(o[bb, h] - r[bb, h]).max() <= OUT_TOL * np.abs(r[bb, h]).max()
    kv.close()


def test_encode_rejects_bad_rows():
    w = W.generate(W.SPECS["tiny"], device="cuda")
    kv = bk.BasisKV.for_workload(w)
    s = w.spec
    k = torch.zeros((s.num_kv_heads, 2, s.head_dim), device="cuda")
    with pytest.raises(bk.BasisKVError):
        bk.basiskv_encode_rows(kv.handle, 0, s.page_size - 1, k, k)   # rows past the page
    with pytest.raises(bk.BasisKVError):
        bk.basiskv_encode_rows(kv.handle, w.z_pool.shape[0], 0, k, k)  # slot past the pools
    kv.close()


def _pool_rows(w, slot, rows):
    """(K, Z, R) rows of one slot, every KV head, as host tensors."""
    return tuple(t[slot, :, rows].detach().cpu().clone() for t in (w.k_pool, w.z_pool, w.r_pool))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_encode_tokens_matches_encode_rows(dtype):
    """One launch for a list of tokens at scattered (slot, row) positions
    writes exactly the bits that basiskv_encode_rows writes for the same
    token, and those agree with the oracle's encode."""
    spec = W.shrink("llama3_8b_decode", batch=2, len_lo=600, len_hi=900, topk=4, dtype=dtype)
    w = W.generate(spec, device="cuda")
    s = w.spec
    bf16 = dtype == "bf16"
    dt = oracle.BF16 if bf16 else oracle.F32
    tdt = torch.bfloat16 if bf16 else torch.float32
    kv = bk.BasisKV.for_workload(w)
    g = torch.Generator(device="cuda").manual_seed(21)
    n = 13
    nslots = w.z_pool.shape[0]
    slots = torch.tensor([(nslots - 1 - (i % 5)) for i in range(n)], dtype=torch.int32, device="cuda")
    rows = torch.tensor([(7 * i + 3) % s.page_size for i in range(n)], dtype=torch.int32, device="cuda")
    k = torch.randn((n, s.num_kv_heads, s.head_dim), generator=g, device="cuda").to(tdt)
    v = torch.randn((n, s.num_kv_heads, s.head_dim), generator=g, device="cuda").to(tdt)
    bk.basiskv_encode_tokens(kv.handle, slots, rows, k, v)
    torch.cuda.synchronize()
    got = [_pool_rows(w, int(slots[i]), int(rows[i])) for i in range(n)]
    # the same tokens through encode_rows, one call per token (last writer wins
    # for repeated positions, so compare against the last token per position)
    last = {}
    for i in range(n):
        last[(int(slots[i]), int(rows[i]))] = i
    for (sl, rw), i in last.items():
        bk.basiskv_encode_rows(kv.handle, sl, rw, k[i:i + 1].transpose(0, 1).contiguous(),
                               v[i:i + 1].transpose(0, 1).contiguous())
        torch.cuda.synchronize()
        ref = _pool_rows(w, sl, rw)
        for a_, b_ in zip(got[i], ref):
            assert torch.equal(a_, b_), (sl, rw)
        kh = widen(_host(k[i], bf16), dt)[:, None, :]
        vh = widen(_host(v[i], bf16), dt)[:, None, :]
        Zr, _ = oracle.encode(kh, vh, w.w_zk.cpu().numpy(), w.b_r.cpu().numpy(), w.b_v.cpu().numpy(), dt)
        Zg = widen(_host(ref[1], bf16), dt)[:, None, :]
        step, floor = (2.0 ** -7, 2.0 ** -9) if bf16 else (1e-5, 1e-4)
        assert np.all(np.abs(Zg - Zr) <= step * np.abs(Zr) + floor * np.abs(Zr).max())
    assert bk.basiskv_get_status(kv.handle) == 0
    kv.close()


def test_encode_tokens_flags_positions_outside_the_pool():
    w = W.generate(W.SPECS["tiny"], device="cuda")
    s = w.spec
    kv = bk.BasisKV.for_workload(w)
    before = [t.clone() for t in (w.k_pool, w.z_pool, w.r_pool)]
    nslots = w.z_pool.shape[0]
    slots = torch.tensor([nslots, -1, 0], dtype=torch.int32, device="cuda")
    rows = torch.tensor([0, 0, s.page_size], dtype=torch.int32, device="cuda")
    k = torch.ones((3, s.num_kv_heads, s.head_dim), device="cuda")
    bk.basiskv_encode_tokens(kv.handle, slots, rows, k, k)
    torch.cuda.synchronize()
    assert bk.basiskv_get_status(kv.handle, clear=True) & bk.BASISKV_STATUS_BAD_SLOT
    for a_, b_ in zip(before, (w.k_pool, w.z_pool, w.r_pool)):
        assert torch.equal(a_, b_)
    kv.close()


def test_encode_after_a_smaller_handle_is_created():
    """Shared-memory limits belong to the kernels, not to a handle: creating
    a handle with smaller shapes must not break a larger one's launches."""
    big = W.generate(W.shrink("dense_limit", batch=1, len_lo=200, len_hi=200, topk=4), device="cuda")
    small = W.generate(W.shrink("llama3_8b_decode", batch=1, len_lo=200, len_hi=200, topk=2), device="cuda")
    kb = bk.BasisKV.for_workload(big)
    ks = bk.BasisKV.for_workload(small)
    s = big.spec
    k = torch.randn((s.num_kv_heads, 3, s.head_dim), device="cuda").to(torch.bfloat16)
    bk.basiskv_encode_rows(kb.handle, 0, 0, k, k)
    slots = torch.zeros(2, dtype=torch.int32, device="cuda")
    rows = torch.tensor([4, 5], dtype=torch.int32, device="cuda")
    bk.basiskv_encode_tokens(kb.handle, slots, rows, k[:, :2].transpose(0, 1).contiguous(),
                             k[:, :2].transpose(0, 1).contiguous())
    torch.cuda.synchronize()
    assert bk.basiskv_get_status(kb.handle) == 0
    ks.close()
    kb.close()
