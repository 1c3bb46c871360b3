"""Regression: the oracle still gives the stored result on the seeded tiny
workload (tests/golden/tiny_oracle.json, written by make_golden.py)."""
import json
import os

import numpy as np
import pytest

from compressed_kv_cache_routing_b200 import workloads as W
from oracle import oracle
from helpers import to_problem

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_oracle.json")


def test_tiny_golden():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "make_golden", os.path.join(os.path.dirname(GOLDEN), "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    with open(GOLDEN) as f:
        doc = json.load(f)
    w = W.generate("tiny")
    prob = to_problem(w)
    if mg.input_digest(prob) != doc["input_sha256"]:
        pytest.fail("the tiny workload's inputs changed; regenerate the fixture only "
                    "if the generator change is intended")
    out, sel, scores, gap = oracle.decode(prob, want_scores=True)
    assert sel[0, 0].tolist() == doc["sel"]
    assert gap[0, 0] == doc["gap"]
    n = len(doc["page_scores"])
    assert np.array_equal(scores[0, 0, :n], np.array(doc["page_scores"]))
    assert np.array_equal(out[0], np.array(doc["out"]))


def test_tiny_golden_int8_keys_and_latent():
    """The same fixture's int8-key result (the oracle's own quantisation of
    the keys, then decode) and latent-mode result."""
    import dataclasses
    import hashlib
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "make_golden", os.path.join(os.path.dirname(GOLDEN), "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    with open(GOLDEN) as f:
        doc = json.load(f)
    prob = to_problem(W.generate("tiny"))
    p8 = mg.int8_problem(prob)
    g8 = doc["int8_keys"]
    assert hashlib.sha256(p8.k_pool.tobytes()).hexdigest() == g8["codes_sha256"]
    assert hashlib.sha256(p8.k_scale.tobytes()).hexdigest() == g8["scales_sha256"]
    out8, sel8, _, _ = oracle.decode(p8)
    assert sel8[0, 0].tolist() == g8["sel"]
    assert np.array_equal(out8[0], np.array(g8["out"]))
    zb, _, _, _ = oracle.decode(dataclasses.replace(prob, latent=True))
    assert np.array_equal(zb[0], np.array(doc["latent"]["out"]))


def test_unit_sampling_matches_full_run():
    """Oracle on a subset of units equals the full run on those units."""
    spec = W.shrink("high_concurrency", batch=6, len_lo=700, len_hi=1500, topk=8)
    w = W.generate(spec)
    prob = to_problem(w)
    full = oracle.decode(prob)
    units = [1, 7, 30, 47]
    part = oracle.decode(prob, units=units)
    for u in units:
        b, kvh = divmod(u, spec.num_kv_heads)
        G = spec.gqa_group
        assert np.array_equal(part[1][b, kvh], full[1][b, kvh])
        assert np.array_equal(part[0][b, kvh * G:(kvh + 1) * G], full[0][b, kvh * G:(kvh + 1) * G])
    assert (part[1][0, 0] == -1).all()  # unit 0 not computed
