"""Each plausible mistake planted in a copy of the oracle must fail at least
one pin.  The copies are compiled on the CPU into a temporary directory; the
real oracle source is never modified."""
import os
import subprocess

import pytest

from oracle import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "basiskv_oracle.c")

# (name, text in the oracle, replacement)
MUTANTS = [
    ("drop_residual_term",
     "acc += widen(p->r_pool, rrow + a, p->dtype) * (double)Br[(size_t)a * d + c];", ""),
    ("drop_latent_term",
     "acc += widen(p->z_pool, zrow + a, p->dtype) * (double)W[(size_t)a * d + c];", ""),
    ("transpose_w_zk", "(double)W[(size_t)a * d + c]", "(double)W[(size_t)c * r + a]"),
    ("transpose_b_v", "(double)Bv[(size_t)a * d + c]", "(double)Bv[(size_t)c * r + a]"),
    ("sum_over_heads_not_max", "if (u > best) best = u;", "best = (best == -INFINITY ? 0.0 : best) + u;"),
    ("ties_to_higher_index", "return (x->page > y->page) - (x->page < y->page);",
     "return (x->page < y->page) - (x->page > y->page);"),
    ("ascending_scores", "if (x->score > y->score) return -1;", "if (x->score > y->score) return 1;"),
    ("route_ignores_length", "if (t >= L) break;", ""),
    ("attend_ignores_length", "if (j * P + a >= L) break;", ""),
    ("no_normalisation", "for (int a = 0; a < r; ++a) zbar[a] /= den;", ""),
    ("softmax_sign", "exp(score[t] - mx)", "exp(mx - score[t])"),
    ("no_softmax_scale", "score[m] = p->softmax_scale * dot;", "score[m] = dot;"),
    ("head_grouping_strided", "(size_t)kvh * G + h) * d + c, p->dtype);",
     "(size_t)h * p->num_kv_heads + kvh) * d + c, p->dtype);"),
    ("attend_head_grouping_strided", "const size_t qoff = ((size_t)b * p->num_kv_heads * G + (size_t)kvh * G + h) * d;",
     "const size_t qoff = ((size_t)b * p->num_kv_heads * G + (size_t)h * p->num_kv_heads + kvh) * d;"),
    ("route_ignores_page_table", "const size_t zrow = pool_row(p, slot, kvh, i, r);",
     "const size_t zrow = pool_row(p, j, kvh, i, r);"),
    ("attend_ignores_page_table", "const size_t krow = pool_row(p, slot, kvh, a, 1);",
     "const size_t krow = pool_row(p, j, kvh, a, 1);"),
    ("selection_unsorted", "qsort(chosen, (size_t)kb, sizeof(int), int_cmp);", ""),
    ("bf16_low_half", "uint32_t bits = (uint32_t)((const uint16_t *)base)[idx] << 16;",
     "uint32_t bits = (uint32_t)((const uint16_t *)base)[idx];"),
    ("gap_wrong_neighbour", "order[kb - 1].score - order[kb].score", "order[0].score - order[kb].score"),
    ("latent_before_normalisation",
     "        for (int a = 0; a < r; ++a) zbar[a] /= den;\n        if (p->latent) {",
     "        if (p->latent) {\n            for (int a = 0; a < r; ++a) o[a] = zbar[a];\n            continue;\n        }\n"
     "        for (int a = 0; a < r; ++a) zbar[a] /= den;\n        if (p->latent) {"),
    ("head_rows_shifted", "double *o = out + (size_t)h * width;",
     "double *o = out + (size_t)(h > 0 ? h - 1 : 0) * width;"),
    ("int8_scale_ignored", "(double)((const int8_t *)p->k_pool)[idx] * (double)p->k_scale[row];",
     "(double)((const int8_t *)p->k_pool)[idx];"),
    ("int8_scale_per_page", "(double)p->k_scale[row];", "(double)p->k_scale[row / p->page_size];"),
    ("int8_codes_unsigned", "(double)((const int8_t *)p->k_pool)[idx]", "(double)((const uint8_t *)p->k_pool)[idx]"),
    ("kv_head_stride_in_pool", "return (((size_t)slot * p->num_kv_heads + kvh) * p->page_size + i) * (size_t)width;",
     "return (((size_t)slot * p->num_kv_heads) * p->page_size + i) * (size_t)width;"),
]


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, source, name, old, new):
    assert source.count(old) >= 1, f"mutation anchor for {name} not found"
    src = tmp_path / f"{name}.c"
    src.write_text(source.replace(old, new))
    so = tmp_path / f"{name}.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(so),
                           str(src), "-lm"])
    lib = oracle.lib(str(so))
    failed = []
    for pin in oracle_pins.PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"


# Mistakes planted in a copy of the numpy key quantizer; each must fail one
# of the quantizer pins.
PY_MUTANTS = [
    ("round_half_away", "q = np.rint((kf / safe[..., None]).astype(np.float32))",
     "q = np.trunc((kf / safe[..., None]).astype(np.float32) + np.copysign(0.5, kf))"),
    ("scale_over_128", "scale = (amax / np.float32(127.0)).astype(np.float32)",
     "scale = (amax / np.float32(128.0)).astype(np.float32)"),
    ("truncate_codes", "q = np.rint((kf / safe[..., None]).astype(np.float32))",
     "q = np.trunc((kf / safe[..., None]).astype(np.float32))"),
    ("max_not_abs", "amax = np.abs(kf).max(axis=-1)", "amax = kf.max(axis=-1)"),
    ("reciprocal_multiply", "q = np.rint((kf / safe[..., None]).astype(np.float32))",
     "q = np.rint((kf * (np.float32(1.0) / safe[..., None])).astype(np.float32))"),
]


@pytest.mark.parametrize("name,old,new", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_quantizer_mutant_is_caught(name, old, new):
    import inspect
    import textwrap
    import numpy as np
    src = textwrap.dedent(inspect.getsource(oracle.quantize_keys))
    assert src.count(old) == 1, f"mutation anchor for {name} not found"
    ns = {"np": np}
    exec(compile(src.replace(old, new), f"<{name}>", "exec"), ns)
    failed = []
    for pin in oracle_pins.QPINS:
        try:
            pin(ns["quantize_keys"])
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every quantizer pin"
