"""Keys stored as int8 codes with one fp32 scale per token, through the C ABI.

The device quantiser must reproduce the oracle's codes and scales bit for
bit (same float32 decisions); decoding with the int8 pool must then match the
oracle run on those codes: selection bit for bit, output within the same
2e-3 row-normalised bound as the native-key path.
"""
import dataclasses

import numpy as np
import pytest
import torch

from compressed_kv_cache_routing_b200 import basiskv as bk
from compressed_kv_cache_routing_b200 import workloads as W
from oracle import oracle
from helpers import to_problem, widen
from test_gpu_parity import SMALL, OUT_TOL, out_error, unit_rows

pytestmark = pytest.mark.gpu


def setup_module():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from compressed_kv_cache_routing_b200 import build
    build.build()


def int8_handle(w, max_topk=None):
    """A handle over w's pools with the keys quantised on the device."""
    s = w.spec
    codes = torch.full(tuple(w.k_pool.shape), 99, dtype=torch.int8, device="cuda")
    scales = torch.full(tuple(w.k_pool.shape[:3]), float("nan"), device="cuda")
    kv = bk.BasisKV(z_pool=w.z_pool, r_pool=w.r_pool, k_pool=codes, w_zk=w.w_zk, b_r=w.b_r, b_v=w.b_v,
                    gqa_group=s.gqa_group, max_batch=s.batch, max_pages_per_seq=max(1, w.page_table.shape[1]),
                    max_topk=max(s.topk, max_topk or 0), k_scale=scales)
    bk.basiskv_quantize_keys(kv.handle, w.k_pool)
    bk.basiskv_load_page_table(kv.handle, np.where(w.page_table >= 0, w.page_table, 0), w.seq_lens)
    torch.cuda.synchronize()
    return kv, codes, scales


def oracle_int8(w):
    """The oracle's problem for w with the oracle's own quantisation of its keys."""
    prob = to_problem(w)
    keys = widen(prob.k_pool, prob.dtype).astype(np.float32)
    codes, scales = oracle.quantize_keys(keys)
    return dataclasses.replace(prob, k_pool=codes, k_scale=scales)


def decode_int8(kv, w, topk=None, latent=False):
    s = w.spec
    topk = s.topk if topk is None else topk
    B = len(w.seq_lens)
    width = s.rank_r if latent else s.head_dim
    out = torch.full((B, s.num_q_heads, width), float("nan"), device="cuda")
    sel = torch.full((B, s.num_kv_heads, topk), -7, device="cuda", dtype=torch.int32)
    fn = bk.basiskv_decode_attn_latent if latent else bk.basiskv_decode_attn
    fn(kv.handle, w.q[:B], topk, s.softmax_scale, out, sel)
    torch.cuda.synchronize()
    assert bk.basiskv_get_status(kv.handle, clear=True) == 0
    return out.cpu().numpy(), sel.cpu().numpy()


INT8 = ["tiny", "llama3_8b_decode", "llama_shared_ring", "long_context", "high_concurrency", "dense_limit",
        "generic_bf16", "gqa8", "gqa1", "head_dim64", "fp32_llama_shape"]


@pytest.mark.parametrize("name", INT8)
def test_quantize_and_decode_parity(name):
    w = W.generate(SMALL[name], device="cuda")
    kv, codes, scales = int8_handle(w)
    prob = oracle_int8(w)
    assert np.array_equal(codes.cpu().numpy(), prob.k_pool), name
    assert np.array_equal(scales.cpu().numpy(), prob.k_scale), name
    ref_out, ref_sel, _, _ = oracle.decode(prob)
    out, sel = decode_int8(kv, w)
    assert np.array_equal(sel, ref_sel), name
    err = out_error(out, ref_out)
    print(f"{name} int8 keys: max row rel err {err:.3e}")
    assert err <= OUT_TOL
    kv.close()


@pytest.mark.parametrize("name", ["llama3_8b_decode", "head_dim64"])
def test_latent_output_with_int8_keys(name):
    w = W.generate(SMALL[name], device="cuda")
    kv, _, _ = int8_handle(w)
    prob = dataclasses.replace(oracle_int8(w), latent=True)
    ref, ref_sel, _, _ = oracle.decode(prob)
    zb, sel = decode_int8(kv, w, latent=True)
    assert np.array_equal(sel, ref_sel)
    assert out_error(zb, ref) <= OUT_TOL
    kv.close()


def test_int8_keys_edge_lengths_and_all_pages():
    """Empty, one-token and partial-page sequences, and k >= n_b (no
    routing), with int8 keys."""
    spec = W.shrink("llama3_8b_decode", batch=7, len_lo=4000, len_hi=4000, topk=8)
    w = W.generate(spec, device="cuda")
    w.seq_lens = np.asarray([0, 1, 64, 65, 4000, 8 * 64, 8 * 64 + 1], np.int32)
    kv, _, _ = int8_handle(w, max_topk=64)
    prob = oracle_int8(w)
    for topk in (8, 64):
        ref_out, ref_sel, _, _ = oracle.decode(dataclasses.replace(prob, topk=topk))
        out, sel = decode_int8(kv, w, topk=topk)
        assert np.array_equal(sel, ref_sel), topk
        assert out_error(out, ref_out) <= OUT_TOL, topk
    kv.close()


def test_zero_key_rows_have_zero_scale():
    spec = W.shrink("llama3_8b_decode", batch=1, len_lo=200, len_hi=200, topk=2)
    w = W.generate(spec, device="cuda")
    w.k_pool[0, :, :5] = 0
    kv, codes, scales = int8_handle(w)
    assert (scales[0, :, :5] == 0).all() and (codes[0, :, :5] == 0).all()
    kv.close()


def test_full_size_int8_sampled():
    """The Llama-3-8B decode shape at full size with int8 keys: codes and
    scales bit-exact on the sampled sequences' pages, sampled units against
    the oracle, and the planted pages selected."""
    w = W.generate("llama3_8b_decode", device="cuda")
    kv, codes, scales = int8_handle(w)
    out, sel = decode_int8(kv, w)
    s = w.spec
    U = s.batch * s.num_kv_heads
    units = sorted(set([0, U - 1] + np.random.default_rng(7).choice(U, size=4, replace=False).tolist()))
    # the oracle quantises the slots of the sampled sequences itself (the
    # other rows are never read for those units)
    prob = to_problem(w)
    oc = np.zeros(prob.k_pool.shape, np.int8)
    osc = np.zeros(prob.k_pool.shape[:3], np.float32)
    for b in sorted({u // s.num_kv_heads for u in units}):
        slots = w.page_table[b, :w.num_pages[b]]
        oc[slots], osc[slots] = oracle.quantize_keys(widen(prob.k_pool[slots], prob.dtype).astype(np.float32))
        assert np.array_equal(codes[torch.from_numpy(slots).cuda()].cpu().numpy(), oc[slots])
        assert np.array_equal(scales[torch.from_numpy(slots).cuda()].cpu().numpy(), osc[slots])
    prob = dataclasses.replace(prob, k_pool=oc, k_scale=osc)
    ref_out, ref_sel, _, _ = oracle.decode(prob, units=units)
    for u in units:
        b, kvh = divmod(u, s.num_kv_heads)
        assert np.array_equal(sel[b, kvh], ref_sel[b, kvh]), u
    err = out_error(out, ref_out, unit_rows(w, units))
    print(f"full-size int8 keys: sampled units {units}: max row rel err {err:.3e}")
    assert err <= OUT_TOL
    for (b, kvh), pages in w.planted.items():
        assert np.array_equal(sel[b, kvh][sel[b, kvh] >= 0], pages)
    kv.close()


def test_encode_rows_with_int8_keys():
    """encode_rows on an int8-key handle stores the quantised keys (codes and
    scale as the oracle's quantiser gives them) next to Z and R."""
    spec = W.shrink("llama3_8b_decode", batch=2, len_lo=600, len_hi=900, topk=4)
    w = W.generate(spec, device="cuda")
    s = w.spec
    kv, codes, scales = int8_handle(w)
    g = torch.Generator(device="cuda").manual_seed(5)
    slot = w.z_pool.shape[0] - 1
    k = torch.randn((s.num_kv_heads, 7, s.head_dim), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((s.num_kv_heads, 7, s.head_dim), generator=g, device="cuda").to(torch.bfloat16)
    bk.basiskv_encode_rows(kv.handle, slot, 2, k, v)
    torch.cuda.synchronize()
    kh = widen(k.cpu().view(torch.int16).numpy().view(np.uint16), oracle.BF16).astype(np.float32)
    c_ref, s_ref = oracle.quantize_keys(kh)
    assert np.array_equal(codes[slot, :, 2:9].cpu().numpy(), c_ref)
    assert np.array_equal(scales[slot, :, 2:9].cpu().numpy(), s_ref)
    assert bk.basiskv_get_status(kv.handle) == 0
    kv.close()


def test_quantize_keys_rejected_without_int8_pool():
    w = W.generate(SMALL["llama3_8b_decode"], device="cuda")
    kv = bk.BasisKV.for_workload(w)
    with pytest.raises(bk.BasisKVError):
        bk.basiskv_quantize_keys(kv.handle, w.k_pool)
    kv.close()


@pytest.mark.parametrize("name", ["llama3_8b_decode", "long_context", "high_concurrency", "gqa8", "head_dim64"])
def test_decode_parity_near_margin(name):
    """int8 keys on inputs whose planted pages sit just above the k-th
    boundary (routing reads no keys, so the selection margin is the same)."""
    from margin import OracleScorer
    w = W.generate(SMALL[name], device="cuda", scorer=OracleScorer())
    kv, codes, scales = int8_handle(w)
    prob = oracle_int8(w)
    ref_out, ref_sel, _, gap = oracle.decode(prob)
    assert min(gap[b, h] for (b, h) in w.planted) >= W.MARGIN
    out, sel = decode_int8(kv, w)
    assert np.array_equal(sel, ref_sel), name
    assert out_error(out, ref_out) <= OUT_TOL
    kv.close()
