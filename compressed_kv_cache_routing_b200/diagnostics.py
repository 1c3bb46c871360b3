"""Routing diagnostics, run on the device through the library's own calls.

BasisKV routes with a sketch of the keys: the page score comes from
q.Khat with Khat = Z.W_zk + R.B_r ("BasisKV: Value Latents for
Communication and Key Routing", English abstract: the Value latents predict
part of the Key information needed for routing and a residual adds the
rest).  This module measures how much that approximation costs:

* recall: per (sequence, KV head), the fraction of the pages that routing on
  the exact keys (score from q.K, same page max over heads and tokens) would
  select which the sketch also selects;
* attention error: per (sequence, query head), the largest deviation of the
  output over the sketch's pages from the output over every page, relative
  to the latter's largest entry.

Exact-key routing is the same routing step on a second handle that sees the
key pool as its latents, with W_zk = I and no residual, so that q.Khat = q.K.

A second diagnostic measures what storing the keys as int8 codes with a
per-token scale costs ("PackKV: Reducing KV Cache Memory Footprint through
LLM-Aware Lossy Compression", abstract: lossy key compression at a small
accuracy cost): the same decode step with the keys quantised on the device,
against the step with the full-precision keys.  Routing reads no keys, so
the selections must be identical; the output deviation is reported per
(sequence, query head), relative to the row's largest entry.

    python -m compressed_kv_cache_routing_b200.diagnostics [--int8] [workload ...]
"""
from __future__ import annotations

import numpy as np
import torch

from . import basiskv as bk


def _exact_key_handle(k_pool, gqa_group, max_batch, max_pages, max_topk):
    slots, hkv, P, d = k_pool.shape
    eye = torch.eye(d, device=k_pool.device).expand(hkv, d, d).contiguous()
    empty_r = torch.empty((slots, hkv, P, 0), dtype=k_pool.dtype, device=k_pool.device)
    return bk.BasisKV(z_pool=k_pool, r_pool=empty_r, k_pool=k_pool, w_zk=eye,
                      b_r=torch.empty((hkv, 0, d), device=k_pool.device), b_v=eye, gqa_group=gqa_group,
                      max_batch=max_batch, max_pages_per_seq=max_pages, max_topk=max_topk)


def routing_recall(*, q, z_pool, r_pool, k_pool, w_zk, b_r, b_v, page_table, seq_lens, gqa_group, topk,
                   softmax_scale):
    """Recall of sketch routing against exact-key routing, and the attention
    error of the sketch's selection against attention over every page.

    Tensors as for ``BasisKV`` (device); ``page_table`` [B][max_pages] and
    ``seq_lens`` [B] are host int32 arrays; ``k_pool`` holds the keys in the
    pool dtype (not int8 codes).  Returns a dict with ``recall``
    [B][Hkv] (1 where every page is selected anyway), ``attn_err`` [B][Hq],
    and their means."""
    if k_pool.dtype == torch.int8:
        raise ValueError("routing_recall needs the full-precision keys: exact-key routing reads them as latents")
    page_table = np.ascontiguousarray(np.where(page_table >= 0, page_table, 0), dtype=np.int32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, max_pages = page_table.shape
    hkv = int(z_pool.shape[1])
    P = int(z_pool.shape[2])
    n = -(-seq_lens // P)
    all_pages = max(1, int(n.max()) if B else 1)
    dev = q.device
    sketch = bk.BasisKV(z_pool=z_pool, r_pool=r_pool, k_pool=k_pool, w_zk=w_zk, b_r=b_r, b_v=b_v,
                        gqa_group=gqa_group, max_batch=B, max_pages_per_seq=max(1, max_pages),
                        max_topk=max(topk, all_pages))
    exact = _exact_key_handle(k_pool, gqa_group, B, max(1, max_pages), topk)
    try:
        for h in (sketch, exact):
            bk.basiskv_load_page_table(h.handle, page_table, seq_lens)
        sel = {}
        for name, h in (("sketch", sketch), ("exact", exact)):
            sc = torch.empty((B, hkv, max(1, max_pages)), device=dev)
            s = torch.empty((B, hkv, topk), device=dev, dtype=torch.int32)
            bk.basiskv_route(h.handle, q, topk, sc, s)
            sel[name] = s
        d = int(k_pool.shape[3])
        out_s = torch.empty((B, hkv * gqa_group, d), device=dev)
        out_d = torch.empty_like(out_s)
        bk.basiskv_decode_attn(sketch.handle, q, topk, softmax_scale, out_s)
        bk.basiskv_decode_attn(sketch.handle, q, all_pages, softmax_scale, out_d)
        torch.cuda.synchronize(dev)
        for h in (sketch, exact):
            if bk.basiskv_get_status(h.handle, clear=True):
                raise RuntimeError("device status set during the diagnostic")
        ss, se = sel["sketch"].cpu().numpy(), sel["exact"].cpu().numpy()
        o_s, o_d = out_s.cpu().numpy().astype(np.float64), out_d.cpu().numpy().astype(np.float64)
    finally:
        sketch.close()
        exact.close()
    recall = np.ones((B, hkv))
    for b in range(B):
        kb = min(topk, int(n[b]))
        if kb == 0 or kb == n[b]:
            continue
        for h in range(hkv):
            recall[b, h] = len(set(ss[b, h, :kb].tolist()) & set(se[b, h, :kb].tolist())) / kb
    den = np.abs(o_d).max(axis=2)
    err = np.where(den > 0, np.abs(o_s - o_d).max(axis=2) / np.where(den > 0, den, 1.0), 0.0)
    return {"recall": recall, "attn_err": err, "mean_recall": float(recall.mean()),
            "mean_attn_err": float(err.mean()), "max_attn_err": float(err.max())}


def routing_recall_for(w, topk=None):
    """routing_recall on a synthetic workload (workloads.generate on the device)."""
    s = w.spec
    return routing_recall(q=w.q, z_pool=w.z_pool, r_pool=w.r_pool, k_pool=w.k_pool, w_zk=w.w_zk, b_r=w.b_r,
                          b_v=w.b_v, page_table=w.page_table, seq_lens=w.seq_lens, gqa_group=s.gqa_group,
                          topk=s.topk if topk is None else topk, softmax_scale=s.softmax_scale)


def key_quantization_error(w, topk=None):
    """Output deviation caused by int8 keys on workload ``w`` (device
    tensors): decode with w's keys and with the same keys quantised by
    basiskv_quantize_keys.  Returns ``err`` [B][Hq] (max |y8 - y| / max |y|
    per row), its mean and max, and whether the selections agree."""
    s = w.spec
    topk = s.topk if topk is None else topk
    dev = w.q.device
    B = len(w.seq_lens)
    pt = np.ascontiguousarray(np.where(w.page_table >= 0, w.page_table, 0), dtype=np.int32)
    codes = torch.empty(tuple(w.k_pool.shape), dtype=torch.int8, device=dev)
    scales = torch.empty(tuple(w.k_pool.shape[:3]), dtype=torch.float32, device=dev)
    common = dict(z_pool=w.z_pool, r_pool=w.r_pool, w_zk=w.w_zk, b_r=w.b_r, b_v=w.b_v, gqa_group=s.gqa_group,
                  max_batch=B, max_pages_per_seq=max(1, pt.shape[1]), max_topk=topk)
    native = bk.BasisKV(k_pool=w.k_pool, **common)
    int8 = bk.BasisKV(k_pool=codes, k_scale=scales, **common)
    try:
        bk.basiskv_quantize_keys(int8.handle, w.k_pool)
        res = []
        for h in (native, int8):
            bk.basiskv_load_page_table(h.handle, pt, w.seq_lens)
            out = torch.empty((B, s.num_q_heads, s.head_dim), device=dev)
            sel = torch.empty((B, s.num_kv_heads, topk), device=dev, dtype=torch.int32)
            bk.basiskv_decode_attn(h.handle, w.q[:B], topk, s.softmax_scale, out, sel)
            res.append((out, sel))
        torch.cuda.synchronize(dev)
        for h in (native, int8):
            if bk.basiskv_get_status(h.handle, clear=True):
                raise RuntimeError("device status set during the diagnostic")
        (o, sl), (o8, sl8) = [(x.cpu().numpy().astype(np.float64), y.cpu().numpy()) for x, y in res]
    finally:
        native.close()
        int8.close()
    den = np.abs(o).max(axis=2)
    err = np.where(den > 0, np.abs(o8 - o).max(axis=2) / np.where(den > 0, den, 1.0), 0.0)
    return {"err": err, "mean_err": float(err.mean()), "max_err": float(err.max()),
            "same_selection": bool(np.array_equal(sl, sl8))}


def main(argv=None):
    import sys
    from . import workloads as W
    args = list(argv if argv is not None else sys.argv[1:])
    int8 = "--int8" in args
    names = [a for a in args if a != "--int8"] or ["llama3_8b_decode"]
    for name in names:
        w = W.generate(name, device="cuda")
        if int8:
            r = key_quantization_error(w)
            print(f"{name:18s} int8 keys: same selection {r['same_selection']}  output deviation: "
                  f"mean {r['mean_err']:.3e} max {r['max_err']:.3e}")
        else:
            r = routing_recall_for(w)
            print(f"{name:18s} mean recall {r['mean_recall']:.4f}  attention error vs every page: "
                  f"mean {r['mean_attn_err']:.3e} max {r['max_attn_err']:.3e}")


if __name__ == "__main__":
    main()
