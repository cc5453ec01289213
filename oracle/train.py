"""fp64 autograd oracle of one training-time MSA routing layer.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module; the library under
``routed_sparse_attention_b200`` never does.

Plain PyTorch CPU operations in float64; torch.autograd supplies the
gradients, which the tests pin against central finite differences.  The
forward is the inference path itself, restated with torch ops so that it is
differentiable; the tests pin it to the C oracle (``oracle.decode``,
``oracle.route``), written independently.

Method ("EverMind-AI/MSA: Memory Sparse Attention for 100M-Token Contexts",
sections "How MSA compresses and routes documents" and "MSA against a
conventional RAG stack": routing and generation form one differentiable loop
trained end to end; "EverMind Releases Memory-Sparse Attention Code for
Long-Context AI Models", section "Implementation Details": continued
pre-training uses an auxiliary routing loss).  The pages give no formula for
either; the readings taken here:

* The layer's forward is the inference forward: route, take the top_k
  documents (a selection, no gradient), attend over [their pooled K/V ++ the
  local K/V] with the global RoPE offset top_k.  Gradients reach the query,
  the pooled K/V rows of the selected documents and the local K/V.
* The router score is differentiable (cosine per head with norms clamped at
  1e-12 and values clamped to [-1, 1], mean over heads, max over query tokens
  and the document's chunks: the gradient follows the maximising token and
  chunk) and is trained by the auxiliary loss alone: per query, the
  cross-entropy of a softmax over all documents' scores / tau against the
  query's set of relevant documents,
      loss_b = logsumexp_d(S_d / tau) - logsumexp_{d in P_b}(S_d / tau).

Parity status: the forward and the scores are pinned to the C oracle; the
gradients are pinned by finite differences; the two readings above are parity
unpinned against the upstream project.
"""
from __future__ import annotations

import math

import torch

F64 = torch.float64


def rope_rotate(x: torch.Tensor, pos: torch.Tensor, theta: float) -> torch.Tensor:
    """Rotate-half RoPE of x [..., d] at positions pos (broadcast over x[..., 0])."""
    d = x.shape[-1]
    h = d // 2
    inv = theta ** (-2.0 * torch.arange(h, dtype=F64) / d)
    ang = pos.to(F64)[..., None] * inv
    c, s = torch.cos(ang), torch.sin(ang)
    x0, x1 = x[..., :h], x[..., h:]
    return torch.cat([x0 * c - x1 * s, x1 * c + x0 * s], dim=-1)


def doc_scores(qr: torch.Tensor, kr_pool: torch.Tensor, doc_chunk_off, n_kv_heads: int) -> torch.Tensor:
    """Router score of every document, [B][D], differentiable in qr and kr_pool."""
    B, T, Hq, dr = qr.shape
    G = Hq // n_kv_heads
    kk = kr_pool[:, torch.arange(Hq) // G]                        # [C][Hq][dr]
    qn = torch.linalg.vector_norm(qr, dim=-1).clamp_min(1e-12)     # [B][T][Hq]
    kn = torch.linalg.vector_norm(kk, dim=-1).clamp_min(1e-12)     # [C][Hq]
    dots = torch.einsum("bthi,chi->btch", qr, kk)
    cos = (dots / (qn[:, :, None, :] * kn[None, None])).clamp(-1.0, 1.0)
    per_chunk = cos.mean(dim=-1).max(dim=1).values                 # [B][C]: max over query tokens
    off = [int(o) for o in doc_chunk_off]
    return torch.stack([per_chunk[:, off[s]:off[s + 1]].max(dim=1).values for s in range(len(off) - 1)], dim=1)


def select(scores: torch.Tensor, top_k: int) -> torch.Tensor:
    """Top-k documents per query by (score desc, index asc)."""
    out = []
    for row in scores.detach():
        order = sorted(range(row.numel()), key=lambda s: (-float(row[s]), s))
        out.append(order[:top_k])
    return torch.tensor(out, dtype=torch.int64)


def route_loss(scores: torch.Tensor, positives, tau: float) -> torch.Tensor:
    """Auxiliary routing loss per query, [B]."""
    z = scores / tau
    return torch.stack([torch.logsumexp(z[b], 0) - torch.logsumexp(z[b, list(positives[b])], 0)
                        for b in range(z.shape[0])])


def attention(q, sel, doc_chunk_off, k_pool, v_pool, local_k, local_v, top_k: int, theta: float,
              n_kv_heads: int):
    """(out [B][T][H_q][d], lse [B][T][H_q]) of the sparse attention.

    q: [B][T][H_q][d] (unrotated); sel: [B][top_k]; k_pool, v_pool: [C][H_kv][d]
    (keys as stored, with their document-local rotation); local_k, local_v:
    lists of B tensors [H_kv][L_b + T][d] (keys unrotated).  Key j of the
    local context sits at global position top_k + j and the query token t at
    top_k + L_b + t; token t sees the memory and local keys j <= L_b + t."""
    B, T, Hq, d = q.shape
    G = Hq // n_kv_heads
    off = [int(o) for o in doc_chunk_off]
    outs, lses = [], []
    for b in range(B):
        rows = torch.cat([torch.arange(off[s], off[s + 1]) for s in sel[b].tolist()])
        nmem = rows.numel()
        Ltot = local_k[b].shape[1]
        Lb = Ltot - T
        kpos = top_k + torch.arange(Ltot)
        qpos = top_k + Lb + torch.arange(T)
        vis = torch.arange(nmem + Ltot)[None, :] < (nmem + Lb + torch.arange(T) + 1)[:, None]   # [T][nk]
        ob, lb = [], []
        for h in range(Hq):
            g = h // G
            K = torch.cat([k_pool[rows, g], rope_rotate(local_k[b][g], kpos, theta)])
            V = torch.cat([v_pool[rows, g], local_v[b][g]])
            qrot = rope_rotate(q[b, :, h], qpos, theta)                           # [T][d]
            logits = (qrot @ K.T) / math.sqrt(d)
            logits = logits.masked_fill(~vis, float("-inf"))
            lse = torch.logsumexp(logits, dim=1)                                  # [T]
            ob.append(torch.exp(logits - lse[:, None]) @ V)
            lb.append(lse)
        outs.append(torch.stack(ob, dim=1))                                       # [T][Hq][d]
        lses.append(torch.stack(lb, dim=1))
    return torch.stack(outs), torch.stack(lses)
