"""Buffer owners around the C ABI: a pooled memory bank, a router and a decoder.

They allocate the device / pinned buffers each stage needs once and then call
libmsa; they hold no arithmetic of their own.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (Index, Layout, chunk_offsets, decode_workspace_size, encode_memory, kr_inv_norms, rope_local,
               fetch_selected, fetch_staging_size, rope_table, route, route_scores,
               route_workspace_size, sparse_decode)


def _i64(x) -> torch.Tensor:
    if isinstance(x, np.ndarray):
        x = torch.from_numpy(x)
    return x.to(torch.int64).contiguous()


class Bank:
    """A pooled memory bank: Kr (and K/V) in device memory, or K/V in pinned
    host memory (the host tier).  Built either by encoding per-token K/V/Kr
    (stage 1 on the GPU) or from already pooled tensors."""

    def __init__(self, layout: Layout, doc_tok_off, *, k_tok=None, v_tok=None, kr_tok=None,
                 kr_pool=None, k_pool=None, v_pool=None, host_kv=None, device="cuda",
                 stream=None, inv_norms=True):
        """inv_norms: keep the router keys' inverse norms with the bank (one pass
        over Kr now, read by every tensor-core routing scan)."""
        self.layout = layout
        tok = _i64(doc_tok_off)
        self.doc_tok_off_host = tok
        self.doc_chunk_off_host, self.max_doc_chunks, self.max_doc_len = chunk_offsets(
            tok, layout.c.chunk_size)
        self.n_docs = tok.numel() - 1
        self.n_chunks = int(self.doc_chunk_off_host[-1])
        self.doc_chunk_off = self.doc_chunk_off_host.to(device)
        H, d, dr = layout.c.n_kv_heads, layout.c.head_dim, layout.c.router_dim
        dt = layout.torch_dtype
        if kr_tok is not None:
            self.doc_tok_off = tok.to(device)
            self.rope = rope_table(layout, int(self.max_doc_len), device, stream)
            C = self.n_chunks
            self.k = torch.empty(C, H, d, dtype=dt, device=device)
            self.v = torch.empty(C, H, d, dtype=dt, device=device)
            self.kr = torch.empty(C, H, dr, dtype=dt, device=device)
            encode_memory(layout, self.doc_tok_off, self.doc_chunk_off, C, int(self.max_doc_len),
                          k_tok, v_tok, kr_tok, self.rope, self.k, self.v, self.kr, stream)
            self.host_kv = None
        else:
            self.kr, self.k, self.v, self.host_kv = kr_pool, k_pool, v_pool, host_kv
        self.index = Index(self.doc_chunk_off, self.kr, self.k, self.v, self.host_kv,
                           self.doc_chunk_off_host if self.host_kv is not None else None,
                           self.max_doc_chunks)
        self.kr_inv_norm = None
        if inv_norms:
            self.kr_inv_norm = kr_inv_norms(layout, self.index, device, stream)
            self.index = Index(self.doc_chunk_off, self.kr, self.k, self.v, self.host_kv,
                               self.doc_chunk_off_host if self.host_kv is not None else None,
                               self.max_doc_chunks, self.kr_inv_norm)

    @property
    def host_tier(self) -> bool:
        return self.host_kv is not None


class Router:
    """Routing (stage 2) for `batch` queries of T tokens against one bank."""

    def __init__(self, bank: Bank, batch: int, T: int, top_k: int, device="cuda"):
        self.bank, self.B, self.T, self.k = bank, batch, T, top_k
        n = route_workspace_size(bank.layout, bank.n_docs, batch, T, top_k)
        self.ws = torch.empty(n, dtype=torch.uint8, device=device)
        self.idx = torch.empty(batch, top_k, dtype=torch.int32, device=device)
        self.score = torch.empty(batch, top_k, dtype=torch.float64, device=device)
        self.idx_host = (torch.empty(batch, top_k, dtype=torch.int32, pin_memory=True)
                         if bank.host_tier else None)

    def __call__(self, qr, stream=None):
        route(self.bank.layout, self.bank.index, qr, self.k, self.idx, self.score, self.idx_host,
              self.ws, stream)
        return self.idx, self.score

    def fast_scores(self, qr, stream=None) -> torch.Tensor:
        out = torch.empty(self.B, self.bank.n_docs, dtype=torch.float32, device=self.ws.device)
        route_scores(self.bank.layout, self.bank.index, qr, out, self.ws, stream)
        return out


class Decoder:
    """Sparse decode (stage 3) for fixed local lengths; for a host-tier bank
    it also owns the staging buffer of the fetched documents."""

    def __init__(self, bank: Bank, batch: int, T: int, top_k: int, local_off, device="cuda",
                 stream=None):
        L = bank.layout
        self.bank, self.B, self.T, self.k = bank, batch, T, top_k
        self.local_off = _i64(local_off)
        ltot = (self.local_off[1:] - self.local_off[:-1]).max().item()
        self.rope = rope_table(L, int(top_k + ltot), device, stream)
        self.ws = torch.zeros(decode_workspace_size(L, batch, T, self.local_off), dtype=torch.uint8,
                              device=device)
        self.out = torch.empty(batch, T, L.c.n_q_heads, L.c.head_dim, dtype=L.torch_dtype,
                               device=device)
        self.staging = None
        if bank.host_tier:
            self.staging = torch.empty(fetch_staging_size(L, bank.index, batch, top_k),
                                       dtype=torch.uint8, device=device)

    def fetch(self, sel_host, sel_ready, fetch_stream, fetch_done=None, timeout_ms=10000):
        fetch_selected(self.bank.layout, self.bank.index, self.B, self.k, sel_host, sel_ready,
                       timeout_ms, self.staging, fetch_stream, fetch_done)

    def rotate_local(self, src, dst, new_tokens=None, stream=None):
        """Writes RoPE(src, top_k + j) into the key cache dst: every local token,
        or only the last `new_tokens` of each query (the tokens a step appends)."""
        first = None
        if new_tokens is not None:
            first = (self.local_off[1:] - self.local_off[:-1]) - int(new_tokens)
        rope_local(self.bank.layout, self.local_off, self.k, src, dst, self.rope, first, stream)
        return dst

    def __call__(self, q, local_k, local_v, sel_idx, wait_event=None, stream=None):
        """local_k: the rotated key cache (see rotate_local)."""
        sparse_decode(self.bank.layout, self.bank.index, q, local_k, local_v, self.local_off,
                      sel_idx, self.k, self.rope, self.out, self.ws, self.staging, wait_event,
                      stream)
        return self.out
