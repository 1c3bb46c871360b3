"""Pins for the float64 oracle: checks against closed forms, hand-worked cases,
brute force and invariants that follow from the definition of BasisKV decode
attention ("BasisKV: Value Latents for Communication and Key Routing",
English abstract), never against the oracle's own formulas.

Every ``pin_*`` takes an oracle library handle and raises AssertionError on a
mismatch, so the same pins run against the real oracle
(test_oracle_pins.py) and against deliberately broken copies of it
(test_oracle_mutants.py), which must each fail at least one pin.
"""
import dataclasses
import math

import numpy as np
import torch

from oracle import oracle
from helpers import widen, logical

JUNK = 100.0


def bf16_bits(x):
    """fp32 values -> stored bf16 bit patterns (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def make_problem(rng, B=2, Hkv=2, G=3, d=8, P=4, r=4, s=2, lens=(9, 6), topk=2,
                 dtype=oracle.F32, scale=None, spare=3, bv_identity=False):
    """Random problem with a shuffled page table, junk past each sequence end
    and in unreferenced slots."""
    lens = np.asarray(lens, dtype=np.int32)
    n = -(-lens // P)
    ld = max(int(n.max()) if len(n) else 1, 1)
    slots = int(n.sum()) + spare
    perm = rng.permutation(slots)
    table = np.zeros((B, ld), dtype=np.int32)
    off = 0
    for b in range(B):
        table[b, :n[b]] = perm[off:off + n[b]]
        off += n[b]
    Zp = rng.standard_normal((slots, Hkv, P, r)).astype(np.float32)
    Rp = rng.standard_normal((slots, Hkv, P, s)).astype(np.float32)
    Kp = rng.standard_normal((slots, Hkv, P, d)).astype(np.float32)
    used = set()
    for b in range(B):
        for j in range(n[b]):
            used.add(int(table[b, j]))
            valid = min(P, int(lens[b]) - j * P)
            for pool in (Zp, Rp, Kp):
                pool[table[b, j], :, valid:] = JUNK
    for sl in range(slots):
        if sl not in used:
            Zp[sl] = JUNK
            Rp[sl] = JUNK
            Kp[sl] = JUNK
    q = rng.standard_normal((B, Hkv * G, d)).astype(np.float32)
    W = (rng.standard_normal((Hkv, r, d)) / math.sqrt(r)).astype(np.float32)
    Br = (rng.standard_normal((Hkv, s, d)) / math.sqrt(r)).astype(np.float32)
    if bv_identity:
        assert r == d
        Bv = np.broadcast_to(np.eye(d, dtype=np.float32), (Hkv, d, d)).copy()
    else:
        Bv = (rng.standard_normal((Hkv, r, d)) / math.sqrt(r)).astype(np.float32)
    conv = bf16_bits if dtype == oracle.BF16 else (lambda a: a)
    return oracle.Problem(q=conv(q), z_pool=conv(Zp), r_pool=conv(Rp), k_pool=conv(Kp),
                          w_zk=W, b_r=Br, b_v=Bv, page_table=table, seq_lens=lens,
                          gqa_group=G, topk=topk,
                          softmax_scale=1.0 / math.sqrt(d) if scale is None else scale,
                          dtype=dtype)


def all_pages(prob):
    """Selection listing every valid page of every unit."""
    n = -(-prob.seq_lens // prob.page_size)
    sel = np.full((prob.batch, prob.num_kv_heads, prob.topk), -1, dtype=np.int32)
    for b in range(prob.batch):
        m = min(int(n[b]), prob.topk)
        sel[b, :, :m] = np.arange(m)
    return sel


def dense_attention(prob):
    """Textbook softmax attention over every valid token with values V = Z.B_v:
    out_h = softmax(scale * K q_h) V."""
    G, d = prob.gqa_group, prob.head_dim
    out = np.zeros((prob.batch, prob.num_kv_heads * G, d))
    q = widen(prob.q, prob.dtype)
    for b in range(prob.batch):
        if prob.seq_lens[b] == 0:
            continue
        K, Z, _ = logical(prob, b)
        for kvh in range(prob.num_kv_heads):
            V = Z[kvh] @ prob.b_v[kvh].astype(np.float64)
            for h in range(G):
                logits = prob.softmax_scale * (K[kvh] @ q[b, kvh * G + h])
                w = np.exp(logits - logits.max())
                out[b, kvh * G + h] = (w / w.sum()) @ V
    return out


def rel_err(a, b):
    den = max(np.abs(b).max(), 1e-300)
    return np.abs(a - b).max() / den


# --------------------------------------------------------------------------
def pin_dense_limit(lib):
    """Every page selected => the method is exact softmax attention over
    (K, V = Z.B_v).  Checked with B_v = I, r = d (the dense limiting case) and
    with a general rank-r B_v, ragged lengths, an empty sequence and G = 3."""
    rng = np.random.default_rng(11)
    for kw in (dict(d=8, r=8, s=0, bv_identity=True), dict(d=8, r=4, s=2),
               dict(d=6, r=3, s=1, G=1, Hkv=3)):
        prob = make_problem(rng, B=3, lens=(13, 0, 7), P=4, topk=8, **kw)
        out, sel, _, _ = oracle.decode(prob, library=lib)
        ref = dense_attention(prob)
        assert rel_err(out, ref) < 1e-12, ("dense limit", rel_err(out, ref))
        assert (sel == all_pages(prob)).all()


def _hand_problem():
    """G = 2, d = 2, P = 2, r = 2, s = 1, L = 5 (three pages, the last with one
    valid token), k = 2, softmax scale 1, fp32.
      W_zk = [[1, 2], [0, 1]]   (rows: latent, columns: channel)
      B_r  = [[0, -1]]
      q_0 = [1, 0], q_1 = [0, 1]
      token:   Z         R     Khat = Z.W_zk + R.B_r    q_0.Khat  q_1.Khat
        t0   [1, 0]     [0]    [1, 2]                       1        2
        t1   [0, 1]     [1]    [0, 1] + [0,-1] = [0, 0]     0        0
        t2   [-1, 0]    [2]    [-1,-2] + [0,-2] = [-1,-4]  -1       -4
        t3   [2, -1]    [0]    [2, 3]                       2        3
        t4   [0, 2]     [0]    [0, 2]                       0        2
        t5   junk (past L)
    page scores (max over both heads and the page's valid tokens):
      S_0 = 2, S_1 = 3, S_2 = 2.  Top-2: page 1, then the tie S_0 = S_2 goes to
      the lower page 0 => selection [0, 1], ranked gap S_(2) - S_(3) = 0.
    Keys K are set equal to Khat, B_v = I."""
    Z = np.array([[1, 0], [0, 1], [-1, 0], [2, -1], [0, 2], [JUNK, JUNK]], np.float32)
    R = np.array([[0], [1], [2], [0], [0], [JUNK]], np.float32)
    K = np.array([[1, 2], [0, 0], [-1, -4], [2, 3], [0, 2], [JUNK, JUNK]], np.float32)
    # physical slots in reverse order of the logical pages
    table = np.array([[2, 1, 0]], np.int32)
    def pool(x):
        p = np.zeros((3, 1, 2, x.shape[1]), np.float32)
        for j in range(3):
            p[table[0, j], 0] = x[2 * j:2 * j + 2]
        return p
    return oracle.Problem(
        q=np.array([[[1, 0], [0, 1]]], np.float32), z_pool=pool(Z), r_pool=pool(R), k_pool=pool(K),
        w_zk=np.array([[[1, 2], [0, 1]]], np.float32), b_r=np.array([[[0, -1]]], np.float32),
        b_v=np.eye(2, dtype=np.float32)[None], page_table=table, seq_lens=np.array([5], np.int32),
        gqa_group=2, topk=2, softmax_scale=1.0, dtype=oracle.F32), Z


def pin_hand_routing(lib):
    """The hand-worked routing example above: scores, tie-break and gap."""
    prob, _ = _hand_problem()
    scores, sel, gap = oracle.route(prob, library=lib)
    assert np.array_equal(scores[0, 0], [2.0, 3.0, 2.0]), scores
    assert sel[0, 0].tolist() == [0, 1], sel
    assert gap[0, 0] == 0.0, gap


def pin_hand_attention(lib):
    """Attention of the hand example over the selected tokens t0..t3:
    head 0 logits (1, 0, -1, 2), head 1 logits (2, 0, -4, 3); out_h is the
    softmax-weighted mean of Z_t0..Z_t3 (B_v = I)."""
    prob, Z = _hand_problem()
    out, sel, _, _ = oracle.decode(prob, library=lib)
    assert sel[0, 0].tolist() == [0, 1]
    Zs = Z[:4].astype(np.float64)
    for h, logits in enumerate(([1, 0, -1, 2], [2, 0, -4, 3])):
        e = np.array([math.exp(x) for x in logits])
        expect = (e[0] * Zs[0] + e[1] * Zs[1] + e[2] * Zs[2] + e[3] * Zs[3]) / e.sum()
        assert rel_err(out[0, h], expect) < 1e-14, (h, out[0, h], expect)


def pin_one_token(lib):
    """L = 1: a softmax over one term is 1, so out_h = Z_0.B_v for any q.
    L = 0: the output is zero and nothing is selected."""
    rng = np.random.default_rng(3)
    prob = make_problem(rng, B=2, Hkv=2, G=2, d=8, P=4, r=4, s=2, lens=(1, 0), topk=3)
    out, sel, _, _ = oracle.decode(prob, library=lib)
    Zp = widen(prob.z_pool, prob.dtype)
    for kvh in range(2):
        z0 = Zp[prob.page_table[0, 0], kvh, 0]
        for h in range(2):
            assert rel_err(out[0, kvh * 2 + h], z0 @ prob.b_v[kvh].astype(np.float64)) < 1e-13
    assert (out[1] == 0).all()
    assert sel[0, :, 0].tolist() == [0, 0] and (sel[0, :, 1:] == -1).all() and (sel[1] == -1).all()


def pin_two_tokens_sigmoid(lib):
    """L = 2 in one page: out = sigma(D) Z_0 + (1 - sigma(D)) Z_1 (then B_v),
    D = scale * q.(K_0 - K_1)."""
    rng = np.random.default_rng(5)
    prob = make_problem(rng, B=1, Hkv=1, G=3, d=8, P=4, r=4, s=2, lens=(2,), topk=1, scale=0.7)
    out, _, _, _ = oracle.decode(prob, library=lib)
    slot = prob.page_table[0, 0]
    K = widen(prob.k_pool, prob.dtype)[slot, 0]
    Z = widen(prob.z_pool, prob.dtype)[slot, 0]
    q = widen(prob.q, prob.dtype)[0]
    for h in range(3):
        D = 0.7 * (q[h] @ (K[0] - K[1]))
        sg = 1.0 / (1.0 + math.exp(-D))
        expect = (sg * Z[0] + (1 - sg) * Z[1]) @ prob.b_v[0].astype(np.float64)
        assert rel_err(out[0, h], expect) < 1e-13


def _latent(prob):
    return dataclasses.replace(prob, latent=True)


def pin_latent_two_tokens(lib):
    """Latent output mode (the rank-r weighted latent BasisKV keeps until the
    output projection): L = 2 in one page gives
    zbar = sigma(D) Z_0 + (1 - sigma(D)) Z_1, D = scale * q.(K_0 - K_1), with
    no B_v applied."""
    rng = np.random.default_rng(5)
    prob = _latent(make_problem(rng, B=1, Hkv=1, G=3, d=8, P=4, r=4, s=2, lens=(2,), topk=1, scale=0.7))
    out, _, _, _ = oracle.decode(prob, library=lib)
    assert out.shape == (1, 3, 4)
    slot = prob.page_table[0, 0]
    K = widen(prob.k_pool, prob.dtype)[slot, 0]
    Z = widen(prob.z_pool, prob.dtype)[slot, 0]
    q = widen(prob.q, prob.dtype)[0]
    for h in range(3):
        D = 0.7 * (q[h] @ (K[0] - K[1]))
        sg = 1.0 / (1.0 + math.exp(-D))
        assert rel_err(out[0, h], sg * Z[0] + (1 - sg) * Z[1]) < 1e-13


def pin_latent_one_token(lib):
    """Latent mode, L = 1: zbar = Z_0 whatever q is; L = 0: zero rows, r wide."""
    rng = np.random.default_rng(3)
    prob = _latent(make_problem(rng, B=2, Hkv=2, G=2, d=8, P=4, r=4, s=2, lens=(1, 0), topk=3))
    out, _, _, _ = oracle.decode(prob, library=lib)
    assert out.shape == (2, 4, 4)
    Zp = widen(prob.z_pool, prob.dtype)
    for kvh in range(2):
        for h in range(2):
            assert rel_err(out[0, kvh * 2 + h], Zp[prob.page_table[0, 0], kvh, 0]) < 1e-15
    assert (out[1] == 0).all()


def pin_latent_times_bv_is_value(lib):
    """The value output is the latent output times B_v, head by head, and both
    modes select the same pages (bf16 storage, ragged lengths, GQA 3)."""
    rng = np.random.default_rng(17)
    prob = make_problem(rng, B=3, Hkv=2, G=3, d=8, P=4, r=4, s=2, lens=(13, 3, 9), topk=2,
                        dtype=oracle.BF16)
    out, sel, _, _ = oracle.decode(prob, library=lib)
    zb, sel_l, _, _ = oracle.decode(_latent(prob), library=lib)
    assert np.array_equal(sel, sel_l)
    for b in range(3):
        for kvh in range(2):
            for h in range(3):
                row = kvh * 3 + h
                assert rel_err(zb[b, row] @ prob.b_v[kvh].astype(np.float64), out[b, row]) < 1e-12


def _bases(rng, hkv=2, d=16, r=6, s=4):
    W = rng.standard_normal((hkv, r, d)).astype(np.float32)
    Br = rng.standard_normal((hkv, s, d)).astype(np.float32)
    Bv = rng.standard_normal((hkv, r, d)).astype(np.float32)
    return W, Br, Bv


def pin_encode_recovers_latents(lib):
    """Encode: values in the row space of B_v and keys in the span of the
    prediction plus the residual basis come back as their exact latents
    (up to fp32 storage)."""
    rng = np.random.default_rng(23)
    W, Br, Bv = _bases(rng)
    Z0 = rng.standard_normal((2, 5, 6)).astype(np.float32).astype(np.float64)
    R0 = rng.standard_normal((2, 5, 4)).astype(np.float32).astype(np.float64)
    V = np.einsum("hna,had->hnd", Z0, Bv.astype(np.float64))
    K = np.einsum("hna,had->hnd", Z0, W.astype(np.float64)) + np.einsum("hnb,hbd->hnd", R0, Br.astype(np.float64))
    Z, R = oracle.encode(K, V, W, Br, Bv, oracle.F32)
    assert rel_err(Z, Z0) < 1e-6 and rel_err(R, R0) < 1e-5


def pin_encode_least_squares(lib):
    """Encode of arbitrary keys and values: what is left is orthogonal to
    the basis rows (the normal equations of the least-squares fit), for both
    the latent and the residual; bf16 storage leaves the latent on its grid."""
    rng = np.random.default_rng(29)
    W, Br, Bv = _bases(rng)
    V = rng.standard_normal((2, 7, 16))
    K = rng.standard_normal((2, 7, 16))
    Z, R = oracle.encode(K, V, W, Br, Bv, oracle.F32)
    for h in range(2):
        bv, w, br = (m[h].astype(np.float64) for m in (Bv, W, Br))
        lv = (V[h] - Z[h] @ bv) @ bv.T
        assert np.abs(lv).max() < 1e-4 * np.abs(V[h]).max() * np.abs(bv).max()
        lk = (K[h] - Z[h] @ w - R[h] @ br) @ br.T
        assert np.abs(lk).max() < 1e-4 * np.abs(K[h]).max() * np.abs(br).max()
    Zb, _ = oracle.encode(K, V, W, Br, Bv, oracle.BF16)
    assert np.array_equal(widen(bf16_bits(Zb), oracle.BF16), Zb)
    assert rel_err(Zb, Z) < 2 ** -8
    # the bf16 rounding itself against torch's conversion (nearest, ties even)
    x = np.concatenate([rng.standard_normal(4096) * 10.0 ** rng.integers(-3, 4, 4096),
                        [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0]])
    assert np.array_equal(oracle._round_to_storage(x, oracle.BF16), widen(bf16_bits(x), oracle.BF16))


def pin_folded_scores(lib):
    """Page scores against the folded form  u = Z.(W_zk q) + R.(B_r q)
    (associativity), evaluated with numpy matmuls on the gathered sequence,
    for bf16 and fp32 storage."""
    rng = np.random.default_rng(7)
    for dt in (oracle.F32, oracle.BF16):
        prob = make_problem(rng, B=2, Hkv=2, G=3, d=16, P=4, r=8, s=4, lens=(15, 9), topk=2, dtype=dt)
        scores, _, _ = oracle.route(prob, library=lib)
        q = widen(prob.q, prob.dtype)
        for b in range(prob.batch):
            L = prob.seq_lens[b]
            _, Z, R = logical(prob, b)
            for kvh in range(prob.num_kv_heads):
                qs = q[b, kvh * 3:(kvh + 1) * 3]                       # [G][d]
                qt = prob.w_zk[kvh].astype(np.float64) @ qs.T           # [r][G]
                qh = prob.b_r[kvh].astype(np.float64) @ qs.T            # [s][G]
                u = Z[kvh] @ qt + R[kvh] @ qh                           # [L][G]
                n = -(-L // prob.page_size)
                pad = np.full((n * prob.page_size, 3), -np.inf)
                pad[:L] = u
                ref = pad.reshape(n, -1).max(axis=1)
                assert rel_err(scores[b, kvh, :n], ref) < 1e-12
                assert np.isneginf(scores[b, kvh, n:]).all()


def pin_selection_order(lib):
    """Brute-force check of the selection on tiny problems with many exact
    ties (several logical pages mapped onto one physical slot): exactly
    min(k, n) pages, listed ascending, and every selected page outranks every
    unselected one (higher score, or equal score and lower index)."""
    rng = np.random.default_rng(13)
    for trial in range(30):
        n = int(rng.integers(1, 9))
        P = 2
        L = int(rng.integers((n - 1) * P + 1, n * P + 1))
        k = int(rng.integers(1, 7))
        prob = make_problem(rng, B=1, Hkv=1, G=2, d=4, P=P, r=2, s=1, lens=(L,), topk=k, spare=1)
        # fold pages onto at most 3 distinct slots => exact ties
        prob.page_table[0, :n] = prob.page_table[0, rng.integers(0, min(n, 3), size=n)]
        prob.seq_lens[0] = n * P  # every page full so folded pages score equal
        scores, sel, gap = oracle.route(prob, library=lib)
        S = scores[0, 0, :n]
        chosen = [j for j in sel[0, 0].tolist() if j >= 0]
        assert len(chosen) == min(k, n)
        assert chosen == sorted(chosen) and len(set(chosen)) == len(chosen)
        assert (sel[0, 0, len(chosen):] == -1).all()
        rest = [j for j in range(n) if j not in chosen]
        for i in chosen:
            for j in rest:
                assert S[i] > S[j] or (S[i] == S[j] and i < j), (S, chosen)
        if rest:
            assert gap[0, 0] == min(S[i] for i in chosen) - max(S[j] for j in rest)
        else:
            assert math.isinf(gap[0, 0])


def pin_all_ties_lower_index(lib):
    """Every page on the same slot => all scores equal => the k lowest pages."""
    rng = np.random.default_rng(17)
    prob = make_problem(rng, B=1, Hkv=2, G=2, d=4, P=2, r=2, s=1, lens=(12,), topk=4)
    prob.page_table[0, :] = prob.page_table[0, 0]
    _, sel, gap = oracle.route(prob, library=lib)
    assert (sel[0] == np.arange(4)).all() and (gap == 0).all()


def pin_topk_exceeds_pages(lib):
    """k > n_b: every page selected, the rest padded with -1, gap +inf."""
    rng = np.random.default_rng(19)
    prob = make_problem(rng, B=2, Hkv=1, G=2, d=4, P=4, r=2, s=2, lens=(7, 16), topk=5)
    _, sel, gap = oracle.route(prob, library=lib)
    assert sel[0, 0].tolist() == [0, 1, -1, -1, -1]
    assert sel[1, 0].tolist() == [0, 1, 2, 3, -1]
    assert np.isinf(gap).all()


def pin_slot_permutation(lib):
    """Moving pages to other physical slots (and the table with them) changes
    nothing: page identity is logical."""
    rng = np.random.default_rng(23)
    prob = make_problem(rng, B=2, Hkv=2, G=2, d=8, P=4, r=4, s=2, lens=(14, 11), topk=2)
    out, sel, sc, gap = oracle.decode(prob, want_scores=True, library=lib)
    perm = rng.permutation(prob.z_pool.shape[0])
    inv = np.argsort(perm)
    moved = oracle.Problem(q=prob.q, z_pool=prob.z_pool[inv], r_pool=prob.r_pool[inv],
                           k_pool=prob.k_pool[inv], w_zk=prob.w_zk, b_r=prob.b_r, b_v=prob.b_v,
                           page_table=perm[prob.page_table].astype(np.int32), seq_lens=prob.seq_lens,
                           gqa_group=2, topk=2, softmax_scale=prob.softmax_scale, dtype=prob.dtype)
    out2, sel2, sc2, gap2 = oracle.decode(moved, want_scores=True, library=lib)
    assert np.array_equal(out, out2) and np.array_equal(sel, sel2) and np.array_equal(sc, sc2)


def pin_linear_in_bv(lib):
    """For a fixed selection, out is linear in B_v."""
    rng = np.random.default_rng(29)
    prob = make_problem(rng, B=1, Hkv=2, G=2, d=8, P=4, r=4, s=2, lens=(13,), topk=2)
    sel = oracle.route(prob, library=lib)[1]
    B1 = prob.b_v.copy()
    B2 = (rng.standard_normal(B1.shape)).astype(np.float32)
    outs = []
    for Bv in (B1, B2, B1 + B2):
        prob.b_v = np.ascontiguousarray(Bv)
        outs.append(oracle.attend(prob, sel, library=lib))
    # B1 + B2 is rounded to fp32; compare against the exactly-summed expansion
    assert rel_err(outs[0] + outs[1], outs[2]) < 1e-6


def pin_group_is_per_head(lib):
    """With the selection fixed, query head h of a GQA group gets the same
    output as a single-head problem holding only q_h (heads in a group share
    the KV head and nothing else); q_h lives at q[b][kvh*G + h]."""
    rng = np.random.default_rng(31)
    G = 3
    prob = make_problem(rng, B=2, Hkv=2, G=G, d=8, P=4, r=4, s=2, lens=(10, 15), topk=2)
    sel = oracle.route(prob, library=lib)[1]
    out = oracle.attend(prob, sel, library=lib)
    for h in range(G):
        single = oracle.Problem(q=prob.q.reshape(2, 2, G, 8)[:, :, h].copy(), z_pool=prob.z_pool,
                                r_pool=prob.r_pool, k_pool=prob.k_pool, w_zk=prob.w_zk, b_r=prob.b_r,
                                b_v=prob.b_v, page_table=prob.page_table, seq_lens=prob.seq_lens,
                                gqa_group=1, topk=2, softmax_scale=prob.softmax_scale, dtype=prob.dtype)
        o1 = oracle.attend(single, sel, library=lib)
        assert np.array_equal(o1, out.reshape(2, 2, G, 8)[:, :, h])


def pin_softmax_shift(lib):
    """Adding one vector v to every key of a unit adds the constant
    scale*q_h.v to all of head h's logits, which softmax ignores.  Values are
    small dyadic numbers so the shifted keys are exact in fp32."""
    rng = np.random.default_rng(37)
    prob = make_problem(rng, B=1, Hkv=1, G=2, d=8, P=4, r=4, s=2, lens=(16,), topk=4)
    prob.k_pool = np.round(prob.k_pool * 8) / 8
    prob.q = np.round(prob.q * 8) / 8
    sel = all_pages(prob)
    out = oracle.attend(prob, sel, library=lib)
    v = np.round(rng.standard_normal(8) * 8) / 8
    shifted = prob.k_pool.copy()
    shifted[prob.page_table[0, :4]] += v.astype(np.float32)
    prob.k_pool = np.ascontiguousarray(shifted, dtype=np.float32)
    out2 = oracle.attend(prob, sel, library=lib)
    assert rel_err(out2, out) < 1e-13


def pin_zero_residual(lib):
    """s = 0 equals any s with an all-zero residual."""
    rng = np.random.default_rng(41)
    prob = make_problem(rng, B=2, Hkv=2, G=2, d=8, P=4, r=4, s=3, lens=(15, 6), topk=2)
    prob.r_pool[:] = 0.0
    sc1 = oracle.route(prob, library=lib)[0]
    no_r = oracle.Problem(q=prob.q, z_pool=prob.z_pool, r_pool=np.zeros(prob.z_pool.shape[:3] + (0,), np.float32),
                          k_pool=prob.k_pool, w_zk=prob.w_zk, b_r=np.zeros((2, 0, 8), np.float32),
                          b_v=prob.b_v, page_table=prob.page_table, seq_lens=prob.seq_lens,
                          gqa_group=2, topk=2, softmax_scale=prob.softmax_scale, dtype=prob.dtype)
    sc0 = oracle.route(no_r, library=lib)[0]
    assert np.array_equal(sc0, sc1)


def pin_bf16_widening(lib):
    """bf16 storage holds exactly the values of the rounded fp32 tensors."""
    rng = np.random.default_rng(43)
    pb = make_problem(rng, B=1, Hkv=2, G=2, d=8, P=4, r=4, s=2, lens=(11,), topk=2, dtype=oracle.BF16)
    pf = oracle.Problem(q=widen(pb.q, pb.dtype).astype(np.float32),
                        z_pool=widen(pb.z_pool, pb.dtype).astype(np.float32),
                        r_pool=widen(pb.r_pool, pb.dtype).astype(np.float32),
                        k_pool=widen(pb.k_pool, pb.dtype).astype(np.float32),
                        w_zk=pb.w_zk, b_r=pb.b_r, b_v=pb.b_v, page_table=pb.page_table,
                        seq_lens=pb.seq_lens, gqa_group=2, topk=2, softmax_scale=pb.softmax_scale,
                        dtype=oracle.F32)
    # widening itself: a bf16 pattern is the top half of the fp32 pattern
    assert widen(np.array([0x3FC0], np.uint16), oracle.BF16)[0] == 1.5
    ob = oracle.decode(pb, want_scores=True, library=lib)
    of = oracle.decode(pf, want_scores=True, library=lib)
    for a, b in zip(ob, of):
        assert np.array_equal(a, b)


def pin_scale_invariance_of_routing(lib):
    """Page scores are linear in q (doubling q doubles every score exactly),
    so the selection does not move."""
    rng = np.random.default_rng(47)
    prob = make_problem(rng, B=1, Hkv=2, G=2, d=8, P=4, r=4, s=2, lens=(19,), topk=2)
    sc, sel, _ = oracle.route(prob, library=lib)
    prob.q = np.ascontiguousarray(prob.q * 2, dtype=np.float32)
    sc2, sel2, _ = oracle.route(prob, library=lib)
    assert np.array_equal(sc2, 2 * sc) and np.array_equal(sel, sel2)


def pin_masked_tail(lib):
    """Values stored past L_b never matter (junk 100 vs junk -7)."""
    rng = np.random.default_rng(53)
    prob = make_problem(rng, B=2, Hkv=1, G=2, d=8, P=4, r=4, s=2, lens=(9, 6), topk=1)
    a = oracle.decode(prob, want_scores=True, library=lib)
    for pool in (prob.z_pool, prob.r_pool, prob.k_pool):
        pool[pool == JUNK] = -7.0
    b = oracle.decode(prob, want_scores=True, library=lib)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


# ---- keys stored as int8 codes with one scale per token ---------------------
def _int8_keys(prob, codes, scales):
    return dataclasses.replace(prob, k_pool=codes, k_scale=scales)


def _grid_keys(rng, shape):
    """Keys that int8 with a per-row scale holds exactly: integer codes in
    [-127, 127] with one entry of each row at +-127, times a power of two."""
    codes = rng.integers(-127, 128, size=shape).astype(np.int8)
    flat = codes.reshape(-1, shape[-1])
    flat[np.arange(flat.shape[0]), rng.integers(0, shape[-1], size=flat.shape[0])] = \
        rng.choice(np.array([-127, 127], dtype=np.int8), size=flat.shape[0])
    scales = np.ldexp(1.0, rng.integers(-12, 3, size=shape[:-1])).astype(np.float32)
    return codes, scales, (codes.astype(np.float64) * scales[..., None]).astype(np.float32)


def pin_int8_keys_exact_grid(lib):
    """Keys on an int8 grid: the quantizer returns that grid (codes and
    scales), and decoding with the codes gives the very same selection, page
    scores and output as decoding with the float keys (the product code x
    scale is the key itself)."""
    rng = np.random.default_rng(31)
    prob = make_problem(rng, B=3, Hkv=2, G=2, d=8, P=4, r=4, s=2, lens=(14, 5, 0), topk=2)
    codes, scales, keys = _grid_keys(rng, prob.k_pool.shape)
    c2, s2 = oracle.quantize_keys(keys)
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales)
    ref = oracle.decode(dataclasses.replace(prob, k_pool=keys), library=lib, want_scores=True)
    got = oracle.decode(_int8_keys(prob, codes, scales), library=lib, want_scores=True)
    assert np.array_equal(ref[0], got[0]) and np.array_equal(ref[1], got[1])
    assert np.array_equal(ref[2], got[2])


def pin_int8_two_tokens(lib):
    """L = 2 in one page with int8 keys: out = sigma(D) Z_0 + (1 - sigma(D)) Z_1
    (then B_v) with D = scale * q.(s_0 c_0 - s_1 c_1), written out by hand."""
    rng = np.random.default_rng(37)
    prob = make_problem(rng, B=1, Hkv=1, G=2, d=8, P=4, r=4, s=2, lens=(2,), topk=1, scale=0.3)
    codes = rng.integers(-127, 128, size=prob.k_pool.shape).astype(np.int8)
    scales = rng.uniform(0.001, 0.05, size=prob.k_pool.shape[:3]).astype(np.float32)
    out, _, _, _ = oracle.decode(_int8_keys(prob, codes, scales), library=lib)
    slot = prob.page_table[0, 0]
    c0, c1 = codes[slot, 0, 0].astype(np.float64), codes[slot, 0, 1].astype(np.float64)
    s0, s1 = float(scales[slot, 0, 0]), float(scales[slot, 0, 1])
    Z = widen(prob.z_pool, prob.dtype)[slot, 0]
    q = widen(prob.q, prob.dtype)[0]
    for h in range(2):
        D = 0.3 * (s0 * (q[h] @ c0) - s1 * (q[h] @ c1))
        sg = 1.0 / (1.0 + math.exp(-D))
        expect = (sg * Z[0] + (1 - sg) * Z[1]) @ prob.b_v[0].astype(np.float64)
        assert rel_err(out[0, h], expect) < 1e-13


def pin_int8_keys_dense_limit(lib):
    """Every page selected, int8 keys: exact softmax attention over the
    dequantised keys K_t = s_t c_t (brute force, every valid token)."""
    rng = np.random.default_rng(41)
    prob = make_problem(rng, B=2, Hkv=2, G=3, d=8, P=4, r=8, s=0, lens=(11, 6), topk=4, bv_identity=True)
    codes = rng.integers(-127, 128, size=prob.k_pool.shape).astype(np.int8)
    scales = rng.uniform(0.001, 0.05, size=prob.k_pool.shape[:3]).astype(np.float32)
    out, _, _, _ = oracle.decode(_int8_keys(prob, codes, scales), library=lib)
    deq = codes.astype(np.float64) * scales[..., None].astype(np.float64)  # [slots][Hkv][P][d]
    Z = widen(prob.z_pool, prob.dtype)
    q = widen(prob.q, prob.dtype)
    for b in range(2):
        L = int(prob.seq_lens[b])
        toks = [(int(prob.page_table[b, t // 4]), t % 4) for t in range(L)]
        for kvh in range(2):
            K = np.stack([deq[sl, kvh, i] for sl, i in toks])
            V = np.stack([Z[sl, kvh, i] for sl, i in toks])  # B_v = I
            for h in range(3):
                logits = prob.softmax_scale * (K @ q[b, kvh * 3 + h])
                w = np.exp(logits - logits.max())
                assert rel_err(out[b, kvh * 3 + h], (w / w.sum()) @ V) < 1e-12


def pin_int8_routing_reads_no_keys(lib):
    """Routing uses only Z and R: int8 keys of any content leave the page
    scores and the selection of the float-key problem unchanged."""
    rng = np.random.default_rng(43)
    prob = make_problem(rng, B=2, Hkv=2, G=2, d=8, P=4, r=4, s=2, lens=(15, 9), topk=2)
    codes = rng.integers(-127, 128, size=prob.k_pool.shape).astype(np.int8)
    scales = rng.uniform(0.0, 3.0, size=prob.k_pool.shape[:3]).astype(np.float32)
    a = oracle.route(prob, library=lib)
    b = oracle.route(_int8_keys(prob, codes, scales), library=lib)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


# ---- the key quantizer (host side of the oracle, numpy) ---------------------
def qpin_hand_rows(quantize):
    """Hand rows with exact scales (max 15.875 = 127 / 8, so scale = 1/8):
    entries 2.5 and 3.5 scales away tie and go to the even code, the largest
    entry maps to +-127, a row of zeros has scale 0 and codes 0, and a lone
    negative maximum maps to -127."""
    rows = np.array([[15.875, 0.3125, 0.4375, -0.3125, -0.4375, 0.0, 1.0, -15.875],
                     [0.0] * 8,
                     [0.0, -3.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0],
                     [111.125, 5.6875, -5.6875, 10.9375, 0.0, 0.0, 0.0, 0.0]], dtype=np.float32)
    c, s = quantize(rows)
    assert c.dtype == np.int8 and s.dtype == np.float32
    assert c[0].tolist() == [127, 2, 4, -2, -4, 0, 8, -127], c[0]
    assert s[0] == np.float32(0.125)
    # scale 111.125 / 127 = 0.875 exactly; 5.6875 and 10.9375 are 6.5 and 12.5
    # scales, exact ties that a quotient formed through the float32 reciprocal
    # of the scale misses
    assert s[3] == np.float32(0.875) and c[3].tolist() == [127, 6, -6, 12, 0, 0, 0, 0], c[3]
    assert s[1] == 0 and (c[1] == 0).all()
    assert c[2].tolist() == [0, -127, 0, 0, 0, 0, 0, 0] and s[2] == np.float32(np.float32(3.0) / np.float32(127.0))


def qpin_error_bound(quantize):
    """Random rows (bf16-like magnitudes with outlier channels): every code is
    within half a step of k / scale (float32 rounding aside), the largest
    |code| of every row is 127, and the scale is max|k| / 127 in float32."""
    rng = np.random.default_rng(47)
    k = (rng.standard_normal((64, 128)) * np.exp(rng.normal(0, 0.5, 128))).astype(np.float32)
    c, s = quantize(k)
    assert np.array_equal(s, (np.abs(k).max(axis=1) / np.float32(127.0)).astype(np.float32))
    dev = np.abs(c.astype(np.float64) - k.astype(np.float64) / s[:, None].astype(np.float64))
    assert dev.max() <= 0.5 + 1e-5, dev.max()
    assert (np.abs(c.astype(np.int32)).max(axis=1) == 127).all()


def qpin_shape_and_grid(quantize):
    """Leading dimensions are kept and exact grids come back unchanged."""
    rng = np.random.default_rng(53)
    codes, scales, keys = _grid_keys(rng, (3, 2, 4, 16))
    c, s = quantize(keys)
    assert c.shape == codes.shape and s.shape == scales.shape
    assert np.array_equal(c, codes) and np.array_equal(s, scales)


QPINS = [v for k, v in sorted(globals().items()) if k.startswith("qpin_")]
