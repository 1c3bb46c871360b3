"""Writes tiny_oracle.json: the oracle's result on the seeded "tiny" workload
(batch 1, 1 KV head, GQA 4, d 64, 1024 tokens, page 16, r 16, s 8, top-8,
fp32, seed 0), and the same with the keys quantised to int8 by the oracle's
quantiser and in latent-output mode.  Calls only the generator and oracle/.
Run from the repo root:
    python tests/golden/make_golden.py
"""
import dataclasses
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path[:0] = [ROOT, os.path.join(ROOT, "tests")]

from compressed_kv_cache_routing_b200 import workloads as W  # noqa: E402
from oracle import oracle  # noqa: E402
from helpers import to_problem  # noqa: E402


def input_digest(prob):
    h = hashlib.sha256()
    for a in (prob.q, prob.z_pool, prob.r_pool, prob.k_pool, prob.w_zk, prob.b_r, prob.b_v,
              prob.page_table, prob.seq_lens):
        h.update(a.tobytes())
    return h.hexdigest()


def int8_problem(prob):
    codes, scales = oracle.quantize_keys(prob.k_pool)
    return dataclasses.replace(prob, k_pool=codes, k_scale=scales)


def main():
    w = W.generate("tiny")
    prob = to_problem(w)
    out, sel, scores, gap = oracle.decode(prob, want_scores=True)
    n = int(w.num_pages[0])
    doc = {
        "what": "oracle result on the seeded tiny workload; regression fixture",
        "written_by": "tests/golden/make_golden.py (generator + oracle only)",
        "input_sha256": input_digest(prob),
        "sel": sel[0, 0].tolist(),
        "gap": float(gap[0, 0]),
        "page_scores": [float(x) for x in scores[0, 0, :n]],
        "out": [[float(x) for x in row] for row in out[0]],
    }
    p8 = int8_problem(prob)
    out8, sel8, _, _ = oracle.decode(p8)
    doc["int8_keys"] = {
        "codes_sha256": hashlib.sha256(p8.k_pool.tobytes()).hexdigest(),
        "scales_sha256": hashlib.sha256(p8.k_scale.tobytes()).hexdigest(),
        "sel": sel8[0, 0].tolist(),
        "out": [[float(x) for x in row] for row in out8[0]],
    }
    zb, _, _, _ = oracle.decode(dataclasses.replace(prob, latent=True))
    doc["latent"] = {"out": [[float(x) for x in row] for row in zb[0]]}
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json"), "w") as f:
        json.dump(doc, f, indent=1)


if __name__ == "__main__":
    main()
