"""Attention-score fidelity of the compressed cache: how closely the compressed path's logits follow the exact
ones ("turboquant-pytorch", V3: Attention Score Accuracy -- cosine similarity, top-1 match, top-5 match of the
scores at 8K context).  Reading of the page's metrics (it gives numbers, not formulas): per (sequence, query
head), the cosine similarity of the two logit vectors over the sequence's tokens; top-1 match = the exact
argmax token is the compressed argmax; top-k match = the exact argmax token is among the compressed k best.
All three are averaged over (sequence, query head).  Evaluation code on torch tensors, not part of the hot
path: the compressed logits come from tq_attend_scores."""
from __future__ import annotations

import torch


def exact_scores(q: torch.Tensor, k: torch.Tensor, scale: float | None = None) -> torch.Tensor:
    """Logits of the uncompressed cache: q [B, H_q, d] fp16, k [B, H_kv, T, d] fp16 -> [B, H_q, T] f32
    (fp32 products of the fp16 inputs)."""
    b, hq, d = q.shape
    hkv = k.shape[1]
    g = hq // hkv
    scale = d ** -0.5 if scale is None else scale
    qq = q.float().view(b, hkv, g, d)
    return (torch.einsum("bhgd,bhtd->bhgt", qq, k.float()) * scale).reshape(b, hq, -1)


def score_fidelity(approx: torch.Tensor, exact: torch.Tensor, seq_lens=None, k: int = 5) -> dict:
    """Mean cosine similarity, top-1 match and top-k match of approx vs exact logits [B, H_q, T]."""
    b, hq, t = exact.shape
    lens = [t] * b if seq_lens is None else [int(x) for x in seq_lens]
    cos, top1, topk, n = 0.0, 0.0, 0.0, 0
    for bi in range(b):
        ln = lens[bi]
        if ln == 0:
            continue
        a = approx[bi, :, :ln].double()
        e = exact[bi, :, :ln].double()
        cos += torch.nn.functional.cosine_similarity(a, e, dim=-1).sum().item()
        ea = e.argmax(dim=-1)
        top1 += (a.argmax(dim=-1) == ea).sum().item()
        kk = min(k, ln)
        topk += (a.topk(kk, dim=-1).indices == ea[:, None]).any(dim=-1).sum().item()
        n += hq
    if n == 0:
        return {"cosine": float("nan"), "top1": float("nan"), f"top{k}": float("nan"), "pairs": 0}
    return {"cosine": cos / n, "top1": top1 / n, f"top{k}": topk / n, "pairs": n}
