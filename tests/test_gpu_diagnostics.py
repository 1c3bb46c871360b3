"""The routing diagnostic (sketch routing against exact-key routing, and the
attention error of the sketch's pages) against the same quantities from the
oracle: its routing on the real problem and on a copy whose latents are the
keys themselves (W_zk = I, no residual)."""
import dataclasses

import numpy as np
import pytest

from compressed_kv_cache_routing_b200 import diagnostics as D
from compressed_kv_cache_routing_b200 import workloads as W
from oracle import oracle
from helpers import to_problem

pytestmark = pytest.mark.gpu


def _oracle_report(w):
    prob = to_problem(w)
    s = w.spec
    _, sel_s, _ = oracle.route(prob)
    slots, hkv, P, d = prob.k_pool.shape
    exact = dataclasses.replace(prob, z_pool=prob.k_pool, r_pool=np.zeros((slots, hkv, P, 0), prob.k_pool.dtype),
                                w_zk=np.broadcast_to(np.eye(d, dtype=np.float32), (hkv, d, d)).copy(),
                                b_r=np.zeros((hkv, 0, d), np.float32))
    _, sel_e, _ = oracle.route(exact)
    n = -(-np.asarray(w.seq_lens) // P)
    recall = np.ones((len(n), hkv))
    for b in range(len(n)):
        kb = min(s.topk, int(n[b]))
        if 0 < kb < n[b]:
            for h in range(hkv):
                recall[b, h] = len(set(sel_s[b, h, :kb]) & set(sel_e[b, h, :kb])) / kb
    out_s, _, _, _ = oracle.decode(prob)
    out_d, _, _, _ = oracle.decode(dataclasses.replace(prob, topk=max(1, int(n.max()))))
    den = np.abs(out_d).max(axis=2)
    err = np.where(den > 0, np.abs(out_s - out_d).max(axis=2) / np.where(den > 0, den, 1.0), 0.0)
    return recall, err


@pytest.mark.parametrize("spec,exact_recall", [
    (W.SPECS["tiny"], True),
    (W.shrink("llama3_8b_decode", batch=2, len_lo=2000, len_hi=3000, topk=12), False),
])
def test_routing_recall_matches_oracle(spec, exact_recall):
    w = W.generate(spec, device="cuda")
    r = D.routing_recall_for(w)
    recall, err = _oracle_report(w)
    if exact_recall:   # fp32 pools: the device's scores order pages as the oracle does
        assert np.array_equal(r["recall"], recall)
    else:              # bf16: near-equal exact-key scores may order differently
        assert abs(r["mean_recall"] - recall.mean()) <= 0.02
    assert np.all((r["recall"] >= 0) & (r["recall"] <= 1))
    assert np.abs(r["attn_err"] - err).max() <= 5e-3


def test_key_quantization_error_against_the_oracle():
    """The int8-key deviation reported on the device equals the oracle's:
    its decode on its own quantisation of the keys against its decode on
    the full-precision keys (both within the parity bound of each other)."""
    from test_gpu_int8_keys import oracle_int8
    w = W.generate(W.shrink("llama3_8b_decode", batch=3, len_lo=2500, len_hi=5000, topk=16), device="cuda")
    r = D.key_quantization_error(w)
    assert r["same_selection"]
    out, sel, _, _ = oracle.decode(to_problem(w))
    out8, sel8, _, _ = oracle.decode(oracle_int8(w))
    assert np.array_equal(sel, sel8)
    den = np.abs(out).max(axis=2)
    ref = np.abs(out8 - out).max(axis=2) / den
    assert r["err"].shape == ref.shape
    # the device error differs from the oracle's by at most the two paths'
    # own parity errors (2e-3 each, relative to the same rows)
    assert np.all(np.abs(r["err"] - ref) <= 4e-3 + 1e-6), np.abs(r["err"] - ref).max()
    print(f"int8 keys: device mean/max deviation {r['mean_err']:.3e}/{r['max_err']:.3e}, "
          f"oracle {ref.mean():.3e}/{ref.max():.3e}")
