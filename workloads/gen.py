"""Seeded synthetic inputs for the Memory Sparse Attention hot path.

This module is the only thing the CPU oracle and the CUDA path share: it draws
the inputs (memory banks, router queries, decode queries, local K/V) and holds
none of the method's arithmetic.  Every tensor is drawn from its own seeded
generator keyed by (seed, tensor tag, slice), so a tensor never depends on the
order in which others were drawn.

Recipe (all values N(0,1) unless stated):
  * document lengths: fixed, or clip(round(median * exp(sigma * z)), lo, hi)
    with z ~ N(0,1) (numpy PCG64);
  * per-token banks: K, V, Kr of shape [tokens][H_kv][dim];
  * pooled banks (memories too large to hold per token): each pooled chunk
    element is drawn as N(0, 1/n_c), n_c the tokens in that chunk -- the law of
    the mean of n_c standard normals;
  * needles: needle j is matched to one (query b_j, token t_j); every token
    (per-token banks) or pooled chunk (pooled banks) of the needle document
    carries, for kv-head g, the mean of Qr[b_j, t_j, h] over the query heads h
    of group g plus 0.1 * N(0,1) noise (scaled by 1/sqrt(n_c) once pooled);
  * local contexts: L_b fixed or uniform in [lo, hi]; each query's local K/V
    hold L_b context tokens followed by its T query tokens' own K/V, laid out
    head-major [H_kv][L_b + T][dim] and concatenated over queries.
"""
from __future__ import annotations

import hashlib

import numpy as np
import torch

from .configs import Workload

_SLICE = 1 << 24          # elements per seeded slice
_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _seed(*parts) -> int:
    h = hashlib.blake2b(repr(parts).encode(), digest_size=8).digest()
    return int.from_bytes(h, "little") & 0x7FFF_FFFF_FFFF_FFFF


def storage_dtype(w: Workload) -> torch.dtype:
    return _DT[w.dtype]


def _randn(n: int, seed: int, tag: str, device, out_dtype, row: int = 1,
           row_scale: torch.Tensor | None = None) -> torch.Tensor:
    """n standard normals (fp32 draw, then rounded to out_dtype).

    row_scale, when given, multiplies element e by row_scale[e // row]; slices
    are whole rows so that the scale lookup stays a plain repeat.
    """
    out = torch.empty(n, dtype=out_dtype, device=device)
    rows_per_slice = max(1, _SLICE // row)
    step = rows_per_slice * row
    for i, s in enumerate(range(0, n, step)):
        m = min(step, n - s)
        g = torch.Generator(device=device)
        g.manual_seed(_seed(seed, tag, i))
        x = torch.randn(m, generator=g, device=device, dtype=torch.float32)
        if row_scale is not None:
            r0 = s // row
            sc = row_scale[r0:r0 + m // row].to(device=device, dtype=torch.float32)
            x = (x.view(-1, row) * sc.view(-1, 1)).view(-1)
        out[s:s + m] = x.to(out_dtype)
    return out


def doc_lengths(w: Workload) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(_seed(w.mem_seed, "doc_len")))
    if w.lognormal_sigma == 0.0:
        return np.full(w.n_docs, w.doc_len, dtype=np.int64)
    z = rng.standard_normal(w.n_docs)
    L = np.rint(w.doc_len * np.exp(w.lognormal_sigma * z))
    return np.clip(L, w.len_clip[0], w.len_clip[1]).astype(np.int64)


def offsets(lengths: np.ndarray) -> np.ndarray:
    off = np.zeros(len(lengths) + 1, dtype=np.int64)
    np.cumsum(lengths, out=off[1:])
    return off


def local_lengths(w: Workload) -> np.ndarray:
    lo, hi = w.local_len
    if lo == hi:
        return np.full(w.B, lo, dtype=np.int64)
    rng = np.random.Generator(np.random.PCG64(_seed(w.seed, "local_len")))
    return rng.integers(lo, hi + 1, size=w.B).astype(np.int64)


def needle_targets(w: Workload):
    """(needle docs, [(b_j, t_j)]) -- distinct docs, each matched to one query token."""
    if w.n_needles == 0:
        return np.zeros(0, dtype=np.int64), []
    rng = np.random.Generator(np.random.PCG64(_seed(w.mem_seed, w.seed, "needles")))
    docs = rng.choice(w.n_docs, size=w.n_needles, replace=False).astype(np.int64)
    if w.B == 1:
        targets = [(0, (j * w.T) // w.n_needles) for j in range(w.n_needles)]
    else:
        assert w.n_needles <= w.B * w.T
        targets = [(j % w.B, (j // w.B) % w.T) for j in range(w.n_needles)]
    return docs, targets


def _pool_rows(doc_len: np.ndarray, chunk: int):
    """Synthesis helper: tokens per pooled chunk and the doc of each chunk."""
    n_ch = (doc_len + chunk - 1) // chunk
    doc_of = np.repeat(np.arange(len(doc_len)), n_ch)
    first = offsets(n_ch)[:-1]
    idx_in_doc = np.arange(int(n_ch.sum())) - first[doc_of]
    n_tok = np.minimum(chunk, doc_len[doc_of] - idx_in_doc * chunk)
    return n_ch, doc_of, n_tok


def make_queries(w: Workload, device="cpu") -> dict:
    dt = storage_dtype(w)
    Hq, Hkv, d, dr, T, B = (w.n_q_heads, w.n_kv_heads, w.head_dim, w.router_dim,
                            w.T, w.B)
    qr = _randn(B * T * Hq * dr, w.seed, "qr", "cpu", dt).view(B, T, Hq, dr)
    q = _randn(B * T * Hq * d, w.seed, "q", "cpu", dt).view(B, T, Hq, d)
    L = local_lengths(w)
    tot = L + T
    loff = offsets(tot)
    n_loc = int(loff[-1]) * Hkv * d
    big = n_loc > (1 << 26)
    gdev = device if big else "cpu"
    lk = _randn(n_loc, w.seed, "local_k", gdev, dt).to(device)
    lv = _randn(n_loc, w.seed, "local_v", gdev, dt).to(device)
    return dict(qr=qr.to(device), q=q.to(device), local_len=L, local_off=loff,
                local_k=lk, local_v=lv)


def make_memory(w: Workload, qr: torch.Tensor, device="cpu",
                host_interleaved: bool = False) -> dict:
    """Memory bank of workload w.  qr (any device) supplies the needle signal.

    Per-token workloads return k_tok/v_tok/kr_tok [N_tok][H_kv][dim]; pooled
    workloads return k_pool/v_pool/kr_pool [C][H_kv][dim].  With
    host_interleaved, pooled K/V are returned instead as one pinned host tensor
    host_kv holding, per document, its K chunks followed by its V chunks.
    """
    dt = storage_dtype(w)
    Hkv, d, dr, G = w.n_kv_heads, w.head_dim, w.router_dim, w.group
    L = doc_lengths(w)
    tok_off = offsets(L)
    n_tok = int(tok_off[-1])
    ndocs, targets = needle_targets(w)
    qr32 = qr.detach().to("cpu", torch.float32)
    sig = None
    if len(ndocs):
        # signal[j][g] = mean over heads of group g of Qr[b_j, t_j, :]
        sig = torch.stack([qr32[b, t].view(Hkv, G, dr).mean(dim=1) for (b, t) in targets])
    out = dict(doc_len=L, doc_tok_off=tok_off, needle_docs=ndocs,
               needle_targets=targets)
    big_dev = device
    if w.per_token:
        out["k_tok"] = _randn(n_tok * Hkv * d, w.mem_seed, "k_tok", big_dev, dt).view(n_tok, Hkv, d)
        out["v_tok"] = _randn(n_tok * Hkv * d, w.mem_seed, "v_tok", big_dev, dt).view(n_tok, Hkv, d)
        kr = _randn(n_tok * Hkv * dr, w.mem_seed, "kr_tok", big_dev, dt).view(n_tok, Hkv, dr)
        for j, doc in enumerate(ndocs):
            a, b = int(tok_off[doc]), int(tok_off[doc + 1])
            noise = _randn((b - a) * Hkv * dr, w.mem_seed, ("needle", j), "cpu",
                           torch.float32).view(b - a, Hkv, dr)
            kr[a:b] = (sig[j].unsqueeze(0) + 0.1 * noise).to(dt).to(big_dev)
        out["kr_tok"] = kr
        return out

    n_ch, doc_of, ntok = _pool_rows(L, w.chunk)
    C = int(n_ch.sum())
    scale = torch.from_numpy(1.0 / np.sqrt(ntok.astype(np.float64))).float()
    kr = _randn(C * Hkv * dr, w.mem_seed, "kr_pool", big_dev, dt, Hkv * dr, scale).view(C, Hkv, dr)
    ch_off = offsets(n_ch)
    for j, doc in enumerate(ndocs):
        a, b = int(ch_off[doc]), int(ch_off[doc + 1])
        noise = _randn((b - a) * Hkv * dr, w.mem_seed, ("needle", j), "cpu",
                       torch.float32).view(b - a, Hkv, dr)
        s = scale[a:b].view(-1, 1, 1)
        kr[a:b] = (sig[j].unsqueeze(0) + 0.1 * noise * s).to(dt).to(big_dev)
    out["kr_pool"] = kr
    k = _randn(C * Hkv * d, w.mem_seed, "k_pool", big_dev, dt, Hkv * d, scale)
    v = _randn(C * Hkv * d, w.mem_seed, "v_pool", big_dev, dt, Hkv * d, scale)
    if not host_interleaved:
        out["k_pool"] = k.view(C, Hkv, d)
        out["v_pool"] = v.view(C, Hkv, d)
        return out
    # per document: [K chunks of doc][V chunks of doc]
    first = torch.from_numpy(ch_off[:-1][doc_of])
    nch = torch.from_numpy(n_ch[doc_of])
    c = torch.arange(C, dtype=torch.int64)
    dst_k = (c + first).to(big_dev)
    dst_v = (c + first + nch).to(big_dev)
    host = torch.empty(2 * C, Hkv, d, dtype=dt, pin_memory=(str(device) != "cpu"))
    step = max(1, _SLICE // (Hkv * d))
    staging = torch.empty(2 * C, Hkv, d, dtype=dt, device=big_dev) if str(big_dev) != "cpu" else host
    staging.index_copy_(0, dst_k, k.view(C, Hkv, d))
    staging.index_copy_(0, dst_v, v.view(C, Hkv, d))
    del k, v
    if staging is not host:
        for s in range(0, 2 * C, step):
            host[s:s + step].copy_(staging[s:s + step])
        del staging
    out["host_kv"] = host
    return out


def generate(w: Workload, device="cpu", host_interleaved: bool = False) -> dict:
    qs = make_queries(w, device)
    mem = make_memory(w, qs["qr"], device, host_interleaved=host_interleaved)
    qs.update(mem)
    return qs
