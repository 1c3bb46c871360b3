"""The scorer the near-margin plant of the workload generator asks for.

Page scores come from the float64 oracle (routing only, from the stored
bits), so the margin the generator enforces is the margin the oracle sees.
Token scores, which only guide how far a planted row is moved, are plain
numpy float64: q_h . (Z_t W_zk + R_t B_r) with R_t replaced by the given
rows.  Whatever they guide, the generator checks the result against the
oracle's page scores before it accepts a plant.
"""
import dataclasses

import numpy as np
import torch

from oracle import oracle
from helpers import widen


class OracleScorer:
    def __init__(self):
        self._prob = None
        self._key = None

    def _problem(self, w):
        """Host copy of the stored inputs routing reads; the residual pool is
        copied again on every call because the plant rewrites it."""
        bf16 = w.spec.dtype == "bf16"

        def host(t):
            t = t.detach().cpu().contiguous()
            return t.view(torch.int16).numpy() if bf16 else t.numpy()

        if self._key != id(w):
            s = w.spec
            # routing never reads the keys: a one-slot key pool carries the shape
            self._prob = oracle.Problem(
                q=host(w.q), z_pool=host(w.z_pool), r_pool=host(w.r_pool), k_pool=host(w.k_pool[:1]),
                w_zk=w.w_zk.cpu().numpy(), b_r=w.b_r.cpu().numpy(), b_v=w.b_v.cpu().numpy(),
                page_table=np.where(w.page_table >= 0, w.page_table, 0).astype(np.int32),
                seq_lens=w.seq_lens, gqa_group=s.gqa_group, topk=s.topk,
                softmax_scale=s.softmax_scale, dtype=oracle.BF16 if bf16 else oracle.F32)
            self._key = id(w)
        else:
            self._prob = dataclasses.replace(self._prob, r_pool=host(w.r_pool))
        return self._prob

    def page_scores(self, w):
        prob = self._problem(w)
        routed = [b * w.spec.num_kv_heads + h for (b, h) in w.planted]
        scores, _, _ = oracle.route(prob, units=routed)
        return scores

    def token_scores(self, w, b, kvh, slot, tok, r_rows):
        s = w.spec
        dt = oracle.BF16 if s.dtype == "bf16" else oracle.F32
        bf16 = s.dtype == "bf16"

        def host(t):
            t = t.detach().cpu().contiguous()
            return t.view(torch.int16).numpy() if bf16 else t.numpy()

        si = torch.as_tensor(np.asarray(slot), dtype=torch.long, device=w.z_pool.device)
        ki = torch.as_tensor(np.asarray(kvh), dtype=torch.long, device=w.z_pool.device)
        ti = torch.as_tensor(np.asarray(tok), dtype=torch.long, device=w.z_pool.device)
        z = widen(host(w.z_pool[si, ki, ti]), dt)                     # [n][r]
        q = widen(host(w.q), dt).reshape(s.batch, s.num_kv_heads, s.gqa_group, s.head_dim)
        wz = w.w_zk.double().cpu().numpy()
        br = w.b_r.double().cpu().numpy()
        r_rows = np.asarray(r_rows, dtype=np.float64)
        kvh = np.asarray(kvh)
        b = np.asarray(b)
        out = np.empty((len(b), s.gqa_group))
        for h in np.unique(kvh):
            m = kvh == h
            khat = z[m] @ wz[h] + r_rows[m] @ br[h]                  # [n_h][d]
            out[m] = np.einsum("ngd,nd->ng", q[b[m], h], khat)
        return out
