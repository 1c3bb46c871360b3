"""Test helpers: hand a workload's stored tensors to the oracle."""
import numpy as np
import torch

from oracle import oracle


def to_problem(w, topk=None, softmax_scale=None):
    """Oracle problem holding exactly the stored values of workload ``w``."""
    s = w.spec
    bf16 = s.dtype == "bf16"

    def host(t):
        t = t.detach().cpu().contiguous()
        return t.view(torch.int16).numpy() if bf16 else t.numpy()

    return oracle.Problem(
        q=host(w.q), z_pool=host(w.z_pool), r_pool=host(w.r_pool), k_pool=host(w.k_pool),
        w_zk=w.w_zk.cpu().numpy(), b_r=w.b_r.cpu().numpy(), b_v=w.b_v.cpu().numpy(),
        page_table=np.where(w.page_table >= 0, w.page_table, 0).astype(np.int32),
        seq_lens=w.seq_lens, gqa_group=s.gqa_group,
        topk=s.topk if topk is None else topk,
        softmax_scale=s.softmax_scale if softmax_scale is None else softmax_scale,
        dtype=oracle.BF16 if bf16 else oracle.F32)


def widen(a, dtype):
    """Stored values to float64 (bf16 bit patterns or fp32)."""
    if dtype == oracle.BF16:
        bits = np.ascontiguousarray(a).view(np.uint16).astype(np.uint32) << 16
        return bits.view(np.float32).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


def logical(prob, b):
    """Token-major views of sequence b's K, Z, R ([Hkv][L][.]) gathered
    through the page table, for brute-force checks."""
    L = int(prob.seq_lens[b])
    P = prob.page_size
    n = -(-L // P)
    slots = prob.page_table[b, :n]
    K = widen(prob.k_pool, prob.dtype)[slots]          # [n][Hkv][P][d]
    Z = widen(prob.z_pool, prob.dtype)[slots]
    R = widen(prob.r_pool, prob.dtype)[slots] if prob.rank_s else np.zeros(Z.shape[:3] + (0,))
    def flat(x):
        x = np.transpose(x, (1, 0, 2, 3)).reshape(x.shape[1], n * P, x.shape[3])
        return x[:, :L]
    return flat(K), flat(Z), flat(R)
