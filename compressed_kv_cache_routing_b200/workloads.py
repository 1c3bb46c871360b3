"""Seeded synthetic decode workloads for BasisKV routed attention.

This module only *draws inputs*: it computes no page score, selection,
softmax or output.  Both the CUDA path (tests, bench) and the float64 oracle
(tests) consume what it produces, and the stored tensors it returns are the
ground truth for both sides.

Recipe (all five named workloads follow it; shapes in ``SPECS``):

* lengths  L_b: numpy ``default_rng(seed)``, integers uniform on the closed
  interval [len_lo, len_hi] (constant when the two are equal);
* pages: n_b = ceil(L_b / P) pages per sequence; the pool has
  ``sum(n_b) + max(1, sum(n_b) // 32)`` slots, and logical pages are placed on
  a random permutation of the slots (numpy rng), so the page table really
  indirects and some slots are never referenced;
* bulk tensors from ``torch.Generator(device).manual_seed(seed)`` in this
  order: W_zk [Hkv][r][d], B_r [Hkv][s][d], B_v [Hkv][r][d] ~ N(0, 1/r)
  (B_v = I for the dense workload), q [B][Hq][d] ~ N(0,1)*q_std, Z pool
  [slots][Hkv][P][r] ~ N(0,1), R pool [slots][Hkv][P][s] ~ N(0,1), per-channel
  outlier scales c [Hkv][d] = exp(sigma * N(0,1)) (LogNormal(0, sigma); ones
  when sigma = 0), then noise eps [slots][Hkv][P][d] ~ N(0,1) drawn slot chunk
  by slot chunk;
* q, Z and R are rounded to the storage dtype (round-to-nearest-even);
* planted alignment (only when s > 0 and k < n_b): per (b, kvh), k pages are
  drawn without replacement, and in each one token t* uniformly among the
  page's valid tokens, with delta ~ U(0.05, 0.5); its residual row moves
  along a unit vector g,  R_t* += alpha * g,  and is re-rounded.  Two ways to
  pick g and alpha:
    - strong (no scorer given): g is the unit vector along
      B_r . (sum of the group's stored queries) and
      alpha = (beta0 + delta) * G / |B_r . sum_h q_h|, with
      beta0 = 20 * sqrt((1 + s/r) * mean_h |q_h|^2), twenty times the
      standard deviation of one token's routing score under this
      distribution: the planted pages lead by a wide margin;
    - near margin (``scorer`` given): the planted page is put just above
      the best unplanted one, at tau + delta, tau being the largest page
      score of the unit's unplanted pages.  The scores come from the caller's
      ``scorer`` (this module computes none): ``page_scores(w)`` gives every
      page's score in float64 from the stored values, and
      ``token_scores(w, b, kvh, slot, tok, r_rows)`` the G per-head scores of
      given tokens with their residual rows replaced by ``r_rows``.  A
      token's scores are affine in its residual row, so their response to
      each unit residual direction gives the gradient of each head's score;
      g is the normalised sum of the heads' gradients and alpha the least
      step that lifts the token's best head score to tau + delta.  After
      rounding, the page scores are recomputed from the stored bits; every
      planted page that is not at least 1e-2 above tau gets its delta
      doubled and is planted again from its original row, until all are;
* keys K = (Zs . W_zk + Rs . B_r + 0.05 * eps) * c from the *stored* Zs, Rs,
  rounded to the storage dtype (dense workload: K ~ N(0,1) independent of Z);
  with the near-margin plant, K is first built from the unplanted residuals
  and the planted rows' keys are rebuilt from their final residuals and the
  same eps;
* every token slot past L_b in a sequence's last page, and every unreferenced
  slot, holds JUNK (=100.0) in Z, R and K, so a missing mask changes results.

Readings of the workload descriptions are listed in the design notes; in
particular the planted alignment is realised on the cache side (through the
key residual) so that q keeps exactly its stated distribution and V = Z.B_v
is untouched.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace, field

import numpy as np
import torch

JUNK = 100.0


@dataclass(frozen=True)
class WorkloadSpec:
    name: str
    batch: int
    num_kv_heads: int
    gqa_group: int
    head_dim: int
    page_size: int
    rank_r: int
    rank_s: int
    topk: int
    len_lo: int
    len_hi: int
    dtype: str          # "bf16" or "f32"
    q_std: float
    outlier_sigma: float
    dense: bool
    seed: int
    noise_std: float = 0.05

    @property
    def num_q_heads(self) -> int:
        return self.num_kv_heads * self.gqa_group

    @property
    def max_pages(self) -> int:
        return -(-self.len_hi // self.page_size)

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    def with_(self, **kw) -> "WorkloadSpec":
        return replace(self, **kw)


SPECS = {
    # batch 1, 1 KV head, GQA 4, d 64, 1024 tokens, page 16, r 16, s 8, top-8, fp32, seed 0
    "tiny": WorkloadSpec("tiny", 1, 1, 4, 64, 16, 16, 8, 8, 1024, 1024, "f32",
                         1.0 / 8.0, 0.0, False, 0),
    # Llama-3-8B-shaped decode: 16 x 32q/8kv heads, d 128, 32768 tokens, page 64, r 32, s 16, top-64
    "llama3_8b_decode": WorkloadSpec("llama3_8b_decode", 16, 8, 4, 128, 64, 32, 16, 64,
                                     32768, 32768, "bf16", 1.0 / math.sqrt(128), 0.5, False, 1),
    # long context: 4 sequences, ragged 98304..131072 tokens, top-128
    "long_context": WorkloadSpec("long_context", 4, 8, 4, 128, 64, 32, 16, 128,
                                 98304, 131072, "bf16", 1.0 / math.sqrt(128), 0.5, False, 2),
    # high concurrency: 128 sequences, ragged 4096..8192, page 32, r 24, s 8, top-32
    "high_concurrency": WorkloadSpec("high_concurrency", 128, 8, 4, 128, 32, 24, 8, 32,
                                     4096, 8192, "bf16", 1.0 / math.sqrt(128), 0.5, False, 3),
    # dense limit: r = d = 128, B_v = I, s = 0, top-k = every page
    "dense_limit": WorkloadSpec("dense_limit", 8, 8, 4, 128, 64, 128, 0, 256,
                                16384, 16384, "bf16", 1.0 / math.sqrt(128), 0.0, True, 4),
}


@dataclass
class Workload:
    spec: WorkloadSpec
    seq_lens: np.ndarray          # [B] int32
    page_table: np.ndarray        # [B][max_pages] int32, -1 past n_b
    num_slots: int
    q: torch.Tensor               # [B][Hq][d] storage dtype
    z_pool: torch.Tensor          # [slots][Hkv][P][r]
    r_pool: torch.Tensor          # [slots][Hkv][P][s]
    k_pool: torch.Tensor          # [slots][Hkv][P][d]
    w_zk: torch.Tensor            # [Hkv][r][d] fp32
    b_r: torch.Tensor             # [Hkv][s][d] fp32
    b_v: torch.Tensor             # [Hkv][r][d] fp32
    planted: dict = field(default_factory=dict)   # (b, kvh) -> sorted planted pages

    @property
    def context_tokens(self) -> int:
        return int(self.seq_lens.sum())

    @property
    def num_pages(self) -> np.ndarray:
        return -(-self.seq_lens.astype(np.int64) // self.spec.page_size)

    def algorithmic_bytes(self, int8_keys: bool = False) -> dict:
        """Bytes the routed path must move per call: the routing read of every
        valid token's Z and R rows (units with k < n_b), and the selected pages'
        K and Z (whole pages).  Dense units (k >= n_b) read K and Z of every page.
        With int8 keys a key row is d one-byte codes plus a 4-byte scale."""
        s = self.spec
        es = 2 if s.dtype == "bf16" else 4
        kbytes = s.head_dim + 4 if int8_keys else s.head_dim * es
        route = attn = 0
        for L, n in zip(self.seq_lens.tolist(), self.num_pages.tolist()):
            kb = min(s.topk, n)
            if kb < n:
                route += s.num_kv_heads * L * (s.rank_r + s.rank_s) * es
            attn += s.num_kv_heads * kb * s.page_size * (kbytes + s.rank_r * es)
        return {"route": route, "attn": attn, "total": route + attn}


def _storage(dtype: str):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def generate(spec: WorkloadSpec | str, device: str | torch.device = "cpu",
             slot_chunk: int = 2048, scorer=None) -> Workload:
    """Draw one workload following the recipe in the module docstring.  With
    ``scorer`` the planted pages sit just above the k-th boundary (the near
    margin plant); without it they lead by a wide margin."""
    if isinstance(spec, str):
        spec = SPECS[spec]
    s = spec
    if s.len_lo < 0 or s.len_hi < s.len_lo:
        raise ValueError("bad length range")
    if s.dense and s.rank_r != s.head_dim:
        raise ValueError("the dense workload needs r == d (B_v = I)")
    dev = torch.device(device)
    st = _storage(s.dtype)
    rng = np.random.default_rng(s.seed)

    if s.len_lo == s.len_hi:
        lens = np.full(s.batch, s.len_lo, dtype=np.int32)
    else:
        lens = rng.integers(s.len_lo, s.len_hi, endpoint=True, size=s.batch).astype(np.int32)
    npages = -(-lens.astype(np.int64) // s.page_size)
    total = int(npages.sum())
    num_slots = total + max(1, total // 32)
    perm = rng.permutation(num_slots).astype(np.int32)
    table = np.full((s.batch, max(s.max_pages, 1)), -1, dtype=np.int32)
    off = 0
    for b in range(s.batch):
        n = int(npages[b])
        table[b, :n] = perm[off:off + n]
        off += n

    g = torch.Generator(device=dev).manual_seed(s.seed)
    Hkv, G, d, P, r, rs = s.num_kv_heads, s.gqa_group, s.head_dim, s.page_size, s.rank_r, s.rank_s

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=torch.float32)

    w_zk = randn(Hkv, r, d) / math.sqrt(r)
    b_r = randn(Hkv, rs, d) / math.sqrt(r)
    if s.dense:
        b_v_draw = randn(Hkv, r, d)  # keep the draw order identical across workloads
        del b_v_draw
        b_v = torch.eye(r, device=dev).expand(Hkv, r, d).contiguous()
    else:
        b_v = randn(Hkv, r, d) / math.sqrt(r)
    q = (randn(s.batch, s.num_q_heads, d) * s.q_std).to(st)
    z = randn(num_slots, Hkv, P, r).to(st)
    rr = randn(num_slots, Hkv, P, rs).to(st)
    c = torch.exp(s.outlier_sigma * randn(Hkv, d)) if s.outlier_sigma > 0 else torch.ones(Hkv, d, device=dev)

    planted = {}
    rows = None  # the planted rows, one per planted page
    if not s.dense and rs > 0:
        qd = q.double().view(s.batch, Hkv, G, d)
        v = torch.einsum("ksd,bkd->bks", b_r.double(), qd.sum(2))          # [B][Hkv][s]
        vnorm = v.norm(dim=-1).clamp_min(1e-30)
        ghat = v / vnorm[..., None]
        sigma = torch.sqrt((1.0 + rs / r) * (qd * qd).sum(-1).mean(-1))      # [B][Hkv]
        beta0 = 20.0 * sigma
        rows = {k: [] for k in ("slot", "kvh", "tok", "b", "page", "delta", "alpha")}
        vnorm_h = vnorm.cpu().numpy()
        beta0_h = beta0.cpu().numpy()
        for b in range(s.batch):
            n = int(npages[b])
            kb = min(s.topk, n)
            if kb >= n:
                continue
            for kvh in range(Hkv):
                pages = np.sort(rng.choice(n, size=kb, replace=False))
                planted[(b, kvh)] = pages
                for j in pages.tolist():
                    valid = min(P, int(lens[b]) - j * P)
                    t = int(rng.integers(0, valid))
                    delta = float(rng.uniform(0.05, 0.5))
                    rows["slot"].append(int(table[b, j]))
                    rows["kvh"].append(kvh)
                    rows["tok"].append(t)
                    rows["b"].append(b)
                    rows["page"].append(j)
                    rows["delta"].append(delta)
                    rows["alpha"].append((beta0_h[b, kvh] + delta) * G / vnorm_h[b, kvh])
        rows = {k: np.asarray(v_) for k, v_ in rows.items()}
        if not rows["slot"].size:
            rows = None
        elif scorer is None:
            si = torch.as_tensor(rows["slot"], device=dev, dtype=torch.long)
            ki = torch.as_tensor(rows["kvh"], device=dev, dtype=torch.long)
            ti = torch.as_tensor(rows["tok"], device=dev, dtype=torch.long)
            bi = torch.as_tensor(rows["b"], device=dev, dtype=torch.long)
            al = torch.as_tensor(rows["alpha"], device=dev, dtype=torch.float64)
            add = al[:, None] * ghat[bi, ki]                                  # [n][s] f64
            rr[si, ki, ti] = (rr[si, ki, ti].double() + add).to(st)

    margin = rows is not None and scorer is not None
    eps_rows = None
    if margin:
        eps_rows = torch.empty((len(rows["slot"]), d), device=dev)
        slots_t = torch.as_tensor(rows["slot"], device=dev, dtype=torch.long)
        kvh_t = torch.as_tensor(rows["kvh"], device=dev, dtype=torch.long)
        tok_t = torch.as_tensor(rows["tok"], device=dev, dtype=torch.long)
    k = torch.empty(num_slots, Hkv, P, d, device=dev, dtype=st)
    for s0 in range(0, num_slots, slot_chunk):
        s1 = min(num_slots, s0 + slot_chunk)
        eps = randn(s1 - s0, Hkv, P, d)
        if margin:  # keep the noise of the rows the plant will rebuild
            m = (slots_t >= s0) & (slots_t < s1)
            if bool(m.any()):
                eps_rows[m] = eps[slots_t[m] - s0, kvh_t[m], tok_t[m]]
        if s.dense:
            k[s0:s1] = eps.to(st)
            continue
        kf = torch.einsum("nkpr,krd->nkpd", z[s0:s1].float(), w_zk)
        if rs > 0:
            kf += torch.einsum("nkps,ksd->nkpd", rr[s0:s1].float(), b_r)
        kf += s.noise_std * eps
        kf *= c[None, :, None, :]
        k[s0:s1] = kf.to(st)

    # junk past the end of each sequence and in unreferenced slots
    for b in range(s.batch):
        n = int(npages[b])
        tail = int(lens[b]) - (n - 1) * P if n > 0 else P
        if n > 0 and tail < P:
            slot = int(table[b, n - 1])
            z[slot, :, tail:] = JUNK
            rr[slot, :, tail:] = JUNK
            k[slot, :, tail:] = JUNK
    unused = np.setdiff1d(np.arange(num_slots), table[table >= 0])
    if unused.size:
        ui = torch.as_tensor(unused, device=dev, dtype=torch.long)
        z[ui] = JUNK
        rr[ui] = JUNK
        k[ui] = JUNK

    w = Workload(spec=s, seq_lens=lens, page_table=table, num_slots=num_slots, q=q,
                 z_pool=z, r_pool=rr, k_pool=k, w_zk=w_zk.contiguous(),
                 b_r=b_r.contiguous(), b_v=b_v.contiguous(), planted=planted)
    if margin:
        _plant_near_margin(w, rows, eps_rows, c, scorer)
    return w


MARGIN = 1e-2        # the smallest gap allowed at the k boundary
_MAX_PLANT_ROUNDS = 40


def _plant_near_margin(w: Workload, rows: dict, eps_rows: torch.Tensor, c: torch.Tensor, scorer) -> None:
    """Lift each planted page to tau + delta (module docstring, near-margin
    plant).  The scores are the scorer's; this function only draws, rounds
    and solves for the step length along the chosen direction."""
    s = w.spec
    dev = w.r_pool.device
    st = w.r_pool.dtype
    n = len(rows["slot"])
    si = torch.as_tensor(rows["slot"], device=dev, dtype=torch.long)
    ki = torch.as_tensor(rows["kvh"], device=dev, dtype=torch.long)
    ti = torch.as_tensor(rows["tok"], device=dev, dtype=torch.long)
    r0 = w.r_pool[si, ki, ti].double().cpu().numpy()                      # [n][s] stored, unplanted
    bi, kv, pg = rows["b"], rows["kvh"], rows["page"]
    scores = np.asarray(scorer.page_scores(w), dtype=np.float64)
    tau = np.empty(n)
    for (b, kvh), pages in w.planted.items():
        nb = int(w.num_pages[b])
        keep = np.ones(nb, bool)
        keep[pages] = False
        sel = (bi == b) & (kv == kvh)
        tau[sel] = scores[b, kvh, :nb][keep].max()
    args = (bi, kv, rows["slot"], rows["tok"])
    u0 = np.asarray(scorer.token_scores(w, *args, r0), dtype=np.float64)   # [n][G]
    grad = np.empty(u0.shape + (s.rank_s,))
    for i in range(s.rank_s):
        e = r0.copy()
        e[:, i] += 1.0
        grad[..., i] = np.asarray(scorer.token_scores(w, *args, e), dtype=np.float64) - u0
    gsum = grad.sum(axis=1)
    gdir = gsum / np.maximum(np.linalg.norm(gsum, axis=1, keepdims=True), 1e-300)
    slope = np.einsum("ngs,ns->ng", grad, gdir)                          # [n][G]
    delta = rows["delta"].astype(np.float64).copy()
    todo = np.arange(n)
    for _ in range(_MAX_PLANT_ROUNDS):
        target = tau[todo] + delta[todo]
        up = slope[todo] > 0
        need = np.where(up, (target[:, None] - u0[todo]) / np.where(up, slope[todo], 1.0), np.inf)
        alpha = np.where(u0[todo].max(axis=1) >= target, 0.0, np.maximum(need.min(axis=1), 0.0))
        if not np.isfinite(alpha).all():
            raise RuntimeError("a planted token's score cannot be raised along its residual")
        idx = torch.as_tensor(todo, device=dev, dtype=torch.long)
        r_new = torch.as_tensor(r0[todo] + alpha[:, None] * gdir[todo], device=dev).float().to(st)
        w.r_pool[si[idx], ki[idx], ti[idx]] = r_new
        # the planted rows' keys, from their final residual and the same noise
        zf = w.z_pool[si[idx], ki[idx], ti[idx]].float()
        kf = torch.empty((len(todo), s.head_dim), device=dev)
        for h in range(s.num_kv_heads):
            m = ki[idx] == h
            if bool(m.any()):
                kf[m] = zf[m] @ w.w_zk[h] + r_new[m].float() @ w.b_r[h]
        kf += s.noise_std * eps_rows[idx]
        kf *= c[ki[idx]]
        w.k_pool[si[idx], ki[idx], ti[idx]] = kf.to(st)
        scores = np.asarray(scorer.page_scores(w), dtype=np.float64)
        short = scores[bi, kv, pg] - tau < MARGIN
        if not short.any():
            return
        todo = np.nonzero(short)[0]
        delta[todo] *= 2.0
    raise RuntimeError("the near-margin plant did not reach the margin")


def shrink(spec: WorkloadSpec | str, batch: int | None = None, len_lo: int | None = None,
           len_hi: int | None = None, seed: int | None = None, **kw) -> WorkloadSpec:
    """A smaller variant of a named workload (same shapes per token), for
    parity tests the oracle finishes in seconds."""
    if isinstance(spec, str):
        spec = SPECS[spec]
    upd = dict(kw)
    if batch is not None:
        upd["batch"] = batch
    if len_lo is not None:
        upd["len_lo"] = len_lo
    if len_hi is not None:
        upd["len_hi"] = len_hi
    if seed is not None:
        upd["seed"] = seed
    return spec.with_(**upd)
