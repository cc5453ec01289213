"""Buffer owners around the C ABI: a pooled memory bank, a router and a decoder.

They allocate the device / pinned buffers each stage needs once and then call
libmsa; they hold no arithmetic of their own.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (Index, Layout, StreamEncoder, advance_local_len, append_local, append_local_devlen,
               attention_backward_workspace_size, chunk_offsets, sparse_decode_devlen,
               decode_workspace_size, encode_memory, fetch_selected, fetch_selected_device, fetch_staging_size,
               index_file_info, index_load,
               index_save, interleave_expand, kr_inv_norms, rope_local, rope_table, route, route_loss_backward,
               route_loss_forward, route_loss_workspace_size, route_scores, route_workspace_size,
               sparse_attention_backward, sparse_attention_forward, sparse_decode)


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

    @classmethod
    def from_stream(cls, layout: Layout, batches, *, max_batch_tokens: int, max_batch_docs: int,
                    max_doc_len: int, capacity_chunks: int, host_tier=True, device="cuda", inv_norms=True):
        """Streaming offline encode: `batches` yields (doc_tok_off [n+1] from 0,
        k_tok, v_tok, kr_tok) per batch of whole documents, in host memory
        (pinned, for the copies to overlap) or on the device.  Kr lands on the
        device; K/V in pinned host memory (host_tier) or on the device."""
        H, d, dr = layout.c.n_kv_heads, layout.c.head_dim, layout.c.router_dim
        dt = layout.torch_dtype
        kr = torch.empty(capacity_chunks, H, dr, dtype=dt, device=device)
        k = v = host_kv = None
        if host_tier:
            host_kv = torch.empty(2 * capacity_chunks, H, d, dtype=dt, pin_memory=True)
        else:
            k = torch.empty(capacity_chunks, H, d, dtype=dt, device=device)
            v = torch.empty(capacity_chunks, H, d, dtype=dt, device=device)
        enc = StreamEncoder(layout, max_batch_tokens, max_batch_docs, max_doc_len, capacity_chunks, kr,
                            k_out=k, v_out=v, host_kv_out=host_kv)
        try:
            for tok, kt, vt, krt in batches:
                enc.push(tok, kt, vt, krt)
            n_docs, C, _, coff = enc.finish()
        finally:
            enc.close()
        return cls._from_parts(layout, None, coff, kr[:C], None if k is None else k[:C],
                               None if v is None else v[:C], None if host_kv is None else host_kv[:2 * C],
                               device, inv_norms)

    @classmethod
    def _from_parts(cls, layout, doc_tok_off, doc_chunk_off_host, kr, k, v, host_kv, device, inv_norms):
        """A bank around already pooled tensors (per-token offsets may be None)."""
        bank = cls.__new__(cls)
        bank.layout = layout
        bank.doc_tok_off_host = doc_tok_off
        coff = _i64(doc_chunk_off_host)
        bank.doc_chunk_off_host = coff
        bank.n_docs = coff.numel() - 1
        bank.n_chunks = int(coff[-1])
        bank.max_doc_chunks = int((coff[1:] - coff[:-1]).max())
        bank.max_doc_len = None
        bank.doc_chunk_off = coff.to(device)
        bank.kr, bank.k, bank.v, bank.host_kv = kr, k, v, host_kv
        bank.index = Index(bank.doc_chunk_off, kr, k, v, host_kv, coff if host_kv is not None else None,
                           bank.max_doc_chunks)
        bank.kr_inv_norm = None
        if inv_norms:
            bank.kr_inv_norm = kr_inv_norms(layout, bank.index, device)
            bank.index = Index(bank.doc_chunk_off, kr, k, v, host_kv, coff if host_kv is not None else None,
                               bank.max_doc_chunks, bank.kr_inv_norm)
        return bank

    def save(self, path: str, stream=None):
        """Writes the pooled bank to one index file (msa_index_save)."""
        index_save(path, self.layout, Index(self.doc_chunk_off, self.kr, self.k, self.v, self.host_kv,
                                            self.doc_chunk_off_host, self.max_doc_chunks), stream)

    @classmethod
    def load(cls, path: str, device="cuda", verify=True, inv_norms=True, stream=None):
        """A bank from an index file: Kr (and a device bank's K/V) on the
        device; a host-tier bank's K/V in pinned host memory."""
        layout, n_docs, C, _, host = index_file_info(path)
        H, d, dr = layout.c.n_kv_heads, layout.c.head_dim, layout.c.router_dim
        dt = layout.torch_dtype
        coff = torch.empty(n_docs + 1, dtype=torch.int64)
        kr = torch.empty(C, H, dr, dtype=dt, device=device)
        k = v = host_kv = None
        if host:
            host_kv = torch.empty(2 * C, H, d, dtype=dt, pin_memory=True)
        else:
            k = torch.empty(C, H, d, dtype=dt, device=device)
            v = torch.empty(C, H, d, dtype=dt, device=device)
        index_load(path, coff, kr, k=k, v=v, host_kv=host_kv, verify=verify, stream=stream)
        return cls._from_parts(layout, None, coff, kr, k, v, host_kv, device, inv_norms)


class Router:
    """Routing (stage 2) for `batch` queries of T tokens against one bank."""

    def __init__(self, bank: Bank, batch: int, T: int, top_k: int, device="cuda"):
        self.bank, self.B, self.T, self.k = bank, batch, T, top_k
        n = route_workspace_size(bank.layout, bank.n_docs, bank.n_chunks, batch, T, top_k)
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
    """Sparse decode (stage 3) over a local key/value cache of fixed capacity
    per query (row offsets `local_off`); `local_len` (host, per query) is the
    live length, the full capacity when None.  For a host-tier bank it also
    owns the staging buffer of the fetched documents."""

    def __init__(self, bank: Bank, batch: int, T: int, top_k: int, local_off, device="cuda",
                 stream=None, local_len=None, max_top_k=None):
        """max_top_k: the largest number of documents a later set_top_k may ask
        for (rotary table and host-tier staging are sized for it)."""
        L = bank.layout
        self.bank, self.B, self.T, self.k, self.device = bank, batch, T, top_k, device
        self.max_k = max(top_k, max_top_k or top_k)
        self.local_off = _i64(local_off)
        self.cap = self.local_off[1:] - self.local_off[:-1]
        self.local_len = None if local_len is None else _i64(local_len)
        self.rope = rope_table(L, int(self.max_k + self.cap.max().item()), device, stream)
        self.ws = torch.zeros(0, dtype=torch.uint8, device=device)
        self._fit_ws()
        self.out = torch.empty(batch, T, L.c.n_q_heads, L.c.head_dim, dtype=L.torch_dtype,
                               device=device)
        self.staging = None
        if bank.host_tier:
            self.staging = torch.empty(fetch_staging_size(L, bank.index, batch, self.max_k),
                                       dtype=torch.uint8, device=device)

    def set_top_k(self, k: int):
        """Documents per query of the following calls (global RoPE offset k)."""
        if not 1 <= k <= self.max_k:
            raise ValueError(f"top_k {k} outside [1, {self.max_k}]")
        self.k = int(k)

    def _fit_ws(self):
        need = decode_workspace_size(self.bank.layout, self.B, self.T, self.local_off, self.local_len)
        if need == 0:
            raise ValueError("decode plan rejected: check local lengths against T and the capacities")
        if need > self.ws.numel():             # zero-filled, as the decode's counters require
            self.ws = torch.zeros(need, dtype=torch.uint8, device=self.device)

    def lengths(self) -> torch.Tensor:
        """Live local tokens per query (host int64)."""
        return self.cap.clone() if self.local_len is None else self.local_len.clone()

    def set_lengths(self, local_len):
        """New live lengths (host, per query), e.g. after appending tokens."""
        self.local_len = _i64(local_len)
        self._fit_ws()

    def fetch(self, sel_host, sel_ready, fetch_stream, fetch_done=None, timeout_ms=10000):
        fetch_selected(self.bank.layout, self.bank.index, self.B, self.k, sel_host, sel_ready,
                       timeout_ms, self.staging, fetch_stream, fetch_done)

    def fetch_device(self, sel_idx, stream=None):
        """Host-tier fetch by one kernel on `stream`, reading the device
        selection sel_idx (after the routing, in stream order)."""
        fetch_selected_device(self.bank.layout, self.bank.index, self.B, self.k, sel_idx, self.staging, stream)

    def append(self, k_new, v_new, k_rot, v, k_raw=None, stream=None):
        """Appends one token per query (k_new, v_new [B][H_kv][d], key
        unrotated) at the live lengths and advances them by one: one launch
        writes the value, the raw key (when k_raw is given) and the key rotated
        at top_k + len_b."""
        lens = self.lengths()
        append_local(self.bank.layout, self.local_off, lens, k_new, v_new, self.k, self.rope, k_rot, v, k_raw,
                     stream)
        self.set_lengths(lens + 1)

    def rotate_local(self, src, dst, new_tokens=None, stream=None):
        """Writes RoPE(src, top_k + j) into the key cache dst: every live local
        token, or only the last `new_tokens` of each query (the tokens a step
        appends)."""
        first = None
        if new_tokens is not None:
            first = self.lengths() - int(new_tokens)
        rope_local(self.bank.layout, self.local_off, self.k, src, dst, self.rope, first, stream,
                   local_len_host=self.local_len)
        return dst

    def __call__(self, q, local_k, local_v, sel_idx, wait_event=None, stream=None):
        """local_k: the rotated key cache (see rotate_local)."""
        sparse_decode(self.bank.layout, self.bank.index, q, local_k, local_v, self.local_off,
                      sel_idx, self.k, self.rope, self.out, self.ws, self.staging, wait_event,
                      stream, local_len_host=self.local_len)
        return self.out


class RoutedDecodeLoop:
    """Several routing layers per generated token, each with its own memory
    bank, router and local key/value cache ("EverMind-AI/MSA: Memory Sparse
    Attention for 100M-Token Contexts", section "How MSA compresses and routes
    documents": routing runs in the upper layers, and the local context grows
    by the generated tokens).

    Every layer keeps, per query, a cache of `capacity[b]` tokens laid out
    [H_kv][capacity][head_dim] (raw keys for the record, rotated keys for the
    decode, values).  `prefill` loads the prompt's K/V; each `step` appends one
    token per query to every layer's cache (its key rotated at top_k + j),
    routes the token's router query -- or, with route_once, reuses the first
    step's selection for the whole answer -- fetches host-tier documents, and
    decodes the token.  The queries of a step are [B][1][H_q][d]."""

    def __init__(self, banks, batch: int, top_k: int, prompt_len, capacity, route_once=False,
                 device="cuda", graph=False):
        """graph=True (with route_once): after the first token, every token's
        work on all layers is one CUDA graph replay (see `token`)."""
        if graph and not route_once:
            raise ValueError("graph replay needs route_once: routing and fetching stay on the host path")
        self.banks, self.B, self.k, self.route_once, self.device = list(banks), batch, top_k, route_once, device
        self.graph = graph
        prompt_len = _i64(prompt_len)
        cap = _i64(capacity)
        if torch.any(cap < prompt_len + 1):
            raise ValueError("capacity must leave room for at least one generated token")
        self.local_off = torch.zeros(batch + 1, dtype=torch.int64)
        self.local_off[1:] = torch.cumsum(cap, 0)
        self.routers, self.decoders, self.caches, self.sel = [], [], [], []
        for bank in self.banks:
            L = bank.layout
            H, d = L.c.n_kv_heads, L.c.head_dim
            rows = int(self.local_off[-1]) * H * d
            self.routers.append(Router(bank, batch, 1, top_k, device))
            self.decoders.append(Decoder(bank, batch, 1, top_k, self.local_off, device,
                                         local_len=prompt_len.clone()))
            self.caches.append(dict(k_raw=torch.zeros(rows, dtype=L.torch_dtype, device=device),
                                    k_rot=torch.zeros(rows, dtype=L.torch_dtype, device=device),
                                    v=torch.zeros(rows, dtype=L.torch_dtype, device=device)))
            self.sel.append(None)
        self.routed_steps = 0
        if graph:
            # live lengths in device memory, shared by the layers; decode
            # workspaces planned for the capacities; static token inputs
            self.len_dev = prompt_len.to(device)
            self.inputs = []
            for bank, dec in zip(self.banks, self.decoders):
                L = bank.layout
                dec.ws = torch.zeros(decode_workspace_size(L, batch, 1, self.local_off, None), dtype=torch.uint8,
                                     device=device)
                self.inputs.append(dict(
                    q=torch.zeros(batch, 1, L.c.n_q_heads, L.c.head_dim, dtype=L.torch_dtype, device=device),
                    k_new=torch.zeros(batch, L.c.n_kv_heads, L.c.head_dim, dtype=L.torch_dtype, device=device),
                    v_new=torch.zeros(batch, L.c.n_kv_heads, L.c.head_dim, dtype=L.torch_dtype, device=device)))
            self._graph = None
            self.tokens = 0

    def _rows(self, layer, b, j0, j1):
        """Views of query b's rows [j0, j1) of every head in a cache tensor."""
        L = self.banks[layer].layout
        H, d = L.c.n_kv_heads, L.c.head_dim
        cap = int(self.local_off[b + 1] - self.local_off[b])
        base = int(self.local_off[b]) * H * d
        c = self.caches[layer]
        return [t[base:base + H * cap * d].view(H, cap, d)[:, j0:j1] for t in (c["k_raw"], c["v"])]

    def prefill(self, layer: int, k_prompt, v_prompt):
        """Prompt K/V of one layer: per query b a [H_kv][prompt_len_b][head_dim]
        tensor (lists of B tensors); keys unrotated."""
        dec = self.decoders[layer]
        lens = dec.lengths()
        for b in range(self.B):
            kr, vv = self._rows(layer, b, 0, int(lens[b]))
            kr.copy_(k_prompt[b])
            vv.copy_(v_prompt[b])
        c = self.caches[layer]
        dec.rotate_local(c["k_raw"], c["k_rot"])

    def step(self, layer: int, qr, q, k_new, v_new, stream=None):
        """One generated token on one layer: append k_new, v_new ([B][H_kv][d],
        unrotated key) to the cache, route qr ([B][1][H_q][d_r]) or reuse the
        first selection, decode q ([B][1][H_q][d]).  Returns (output
        [B][1][H_q][d], selected documents [B][top_k])."""
        if self.graph:
            raise RuntimeError("a graph-mode loop advances with token()")
        dec, router, c = self.decoders[layer], self.routers[layer], self.caches[layer]
        dec.append(k_new, v_new, c["k_rot"], c["v"], c["k_raw"], stream)
        if self.sel[layer] is None or not self.route_once:
            idx, _ = router(qr, stream=stream)
            self.sel[layer] = idx
            if self.banks[layer].host_tier:
                st = stream or torch.cuda.current_stream()
                ready, done = torch.cuda.Event(), torch.cuda.Event()
                ready.record(st)
                dec.fetch(router.idx_host, ready, st, done)
                st.wait_event(done)
            self.routed_steps += 1
        out = dec(q, c["k_rot"], c["v"], self.sel[layer], stream=stream)
        return out, self.sel[layer]

    def _token_work(self):
        """One token on every layer, lengths on the device: the appends at the
        current length, one advance, then the decodes (the layers' caches are
        independent, so this order is the per-layer one)."""
        for li, (bank, dec, c) in enumerate(zip(self.banks, self.decoders, self.caches)):
            x = self.inputs[li]
            append_local_devlen(bank.layout, self.local_off, self.len_dev, x["k_new"], x["v_new"], self.k, dec.rope,
                                c["k_rot"], c["v"], c["k_raw"])
        advance_local_len(self.len_dev, 1)
        for li, (bank, dec, c) in enumerate(zip(self.banks, self.decoders, self.caches)):
            sparse_decode_devlen(bank.layout, bank.index, self.inputs[li]["q"], c["k_rot"], c["v"], self.local_off,
                                 self.len_dev, self.sel[li], self.k, dec.rope, dec.out, dec.ws, dec.staging)

    def token(self, qr=None):
        """Graph mode: one generated token on every layer from the static
        buffers in `inputs[layer]` (q [B][1][H_q][d], k_new and v_new
        [B][H_kv][d], key unrotated), which the caller fills first.  The first
        call routes each layer once with qr[layer] ([B][1][H_q][d_r]),
        fetches host-tier documents and runs the token directly; the second
        records the token's launches into a CUDA graph; every later call is one
        graph replay.  Returns the layers' outputs [B][1][H_q][d] (buffers
        that the next token overwrites)."""
        if not self.graph:
            raise RuntimeError("token() is the graph mode; use step() otherwise")
        if self.tokens == 0:
            if qr is None:
                raise ValueError("the first token routes: pass the router queries, one per layer")
            st = torch.cuda.current_stream()
            for li, (bank, router, dec) in enumerate(zip(self.banks, self.routers, self.decoders)):
                idx, _ = router(qr[li])
                self.sel[li] = idx
                if bank.host_tier:
                    ready, done = torch.cuda.Event(), torch.cuda.Event()
                    ready.record(st)
                    dec.fetch(router.idx_host, ready, st, done)
                    st.wait_event(done)
                self.routed_steps += 1
            self._token_work()
        elif self._graph is None:
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            self._graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self._graph, stream=side):
                self._token_work()
            torch.cuda.current_stream().wait_stream(side)
            self._graph.replay()
        else:
            self._graph.replay()
        self.tokens += 1
        return [dec.out for dec in self.decoders]

    def lengths(self) -> torch.Tensor:
        """Live local tokens per query (host int64)."""
        if self.graph:
            return self.len_dev.cpu()
        return self.decoders[0].lengths()


class MemoryInterleave:
    """Multi-hop retrieval on one memory bank: rounds of retrieval -> context
    expansion -> generation ("EverMind-AI/MSA: Memory Sparse Attention for
    100M-Token Contexts", section "How MSA compresses and routes documents";
    "EverMind Releases Memory-Sparse Attention Code for Long-Context AI
    Models", section "Core Contributions").

    Each round (`expand`) routes the round's router query for the
    |S| + per_round best documents and appends the first per_round of them
    that are not in the query's selected set S (msa_interleave_expand), so
    every query's set grows by the same count; the local keys are then rotated
    again at the new global offset k = |S|.  `generate` appends one token per
    query and decodes it over [memory of S, joining order ++ local context].
    Everything stays on the device except, for a host-tier bank, the set's
    copy in pinned memory that drives the fetch of the new documents."""

    def __init__(self, bank: Bank, batch: int, per_round: int, max_docs: int, prompt_len, capacity,
                 device="cuda"):
        if not 1 <= per_round <= max_docs <= 64:
            raise ValueError("need 1 <= per_round <= max_docs <= 64")
        self.bank, self.B, self.p, self.max_docs, self.device = bank, batch, per_round, max_docs, device
        prompt_len = _i64(prompt_len)
        cap = _i64(capacity)
        if torch.any(cap < prompt_len + 1):
            raise ValueError("capacity must leave room for at least one generated token")
        self.local_off = torch.zeros(batch + 1, dtype=torch.int64)
        self.local_off[1:] = torch.cumsum(cap, 0)
        self.routers = {}
        self.decoder = Decoder(bank, batch, 1, per_round, self.local_off, device, local_len=prompt_len.clone(),
                               max_top_k=max_docs)
        L = bank.layout
        rows = int(self.local_off[-1]) * L.c.n_kv_heads * L.c.head_dim
        self.k_raw = torch.zeros(rows, dtype=L.torch_dtype, device=device)
        self.k_rot = torch.zeros(rows, dtype=L.torch_dtype, device=device)
        self.v = torch.zeros(rows, dtype=L.torch_dtype, device=device)
        # two set buffers (the round reads one and writes the other)
        self._sets = [torch.empty(batch * max_docs, dtype=torch.int32, device=device) for _ in range(2)]
        self._set_host = (torch.empty(batch * max_docs, dtype=torch.int32, pin_memory=True)
                          if bank.host_tier else None)
        self.prompt_len = prompt_len.clone()
        self.n = 0
        self.sel = None

    def reset(self):
        """Start a new question on the same prompt: empty set, prompt length."""
        self.n, self.sel = 0, None
        self.decoder.set_top_k(self.p)
        self.decoder.set_lengths(self.prompt_len)

    def _rows(self, b, j0, j1):
        L = self.bank.layout
        H, d = L.c.n_kv_heads, L.c.head_dim
        cap = int(self.local_off[b + 1] - self.local_off[b])
        base = int(self.local_off[b]) * H * d
        return [t[base:base + H * cap * d].view(H, cap, d)[:, j0:j1] for t in (self.k_raw, self.v)]

    def prefill(self, k_prompt, v_prompt):
        """Prompt K/V per query b: [H_kv][prompt_len_b][head_dim], keys unrotated."""
        lens = self.decoder.lengths()
        for b in range(self.B):
            kr, vv = self._rows(b, 0, int(lens[b]))
            kr.copy_(k_prompt[b])
            vv.copy_(v_prompt[b])

    def expand(self, qr, stream=None):
        """One retrieval + context-expansion round for the router query qr
        ([B][T][H_q][d_r]).  Returns the selected set [B][|S|] (device int32)."""
        m = self.n + self.p
        if m > self.max_docs:
            raise ValueError(f"the selected set would exceed max_docs = {self.max_docs}")
        if m not in self.routers:
            self.routers[m] = Router(self.bank, self.B, qr.shape[1], m, self.device)
        ranked, _ = self.routers[m](qr, stream=stream)
        old = None if self.n == 0 else self.sel
        new = self._sets[(self.n // self.p) % 2][: self.B * m].view(self.B, m)
        host = None if self._set_host is None else self._set_host[: self.B * m].view(self.B, m)
        interleave_expand(self.bank.n_docs, ranked, old, new, host, stream)
        self.n, self.sel = m, new
        self.decoder.set_top_k(m)
        if self.bank.host_tier:
            st = stream or torch.cuda.current_stream()
            ready, done = torch.cuda.Event(), torch.cuda.Event()
            ready.record(st)
            self.decoder.fetch(host, ready, st, done)
            st.wait_event(done)
        self.decoder.rotate_local(self.k_raw, self.k_rot, stream=stream)   # new global offset
        return new

    def generate(self, q, k_new, v_new, stream=None):
        """One token per query over the current set: append k_new, v_new
        ([B][H_kv][d], key unrotated), decode q ([B][1][H_q][d])."""
        if self.sel is None:
            raise RuntimeError("expand (a retrieval round) must come before generate")
        self.decoder.append(k_new, v_new, self.k_rot, self.v, self.k_raw, stream)
        return self.decoder(q, self.k_rot, self.v, self.sel, stream=stream)


class TrainLayer:
    """One training-time routing layer on a device-tier bank: forward = route
    (top_k, no gradient), sparse attention (with its log-sum-exp) and the
    auxiliary routing loss; backward = their gradients.  Local K/V use the
    capacity layout of the decode ([H_kv][capacity][d] per query) with keys
    unrotated; the layer keeps the rotated copy the attention reads."""

    def __init__(self, bank: Bank, batch: int, T: int, top_k: int, local_off, local_len=None, tau=0.1,
                 device="cuda"):
        if bank.host_tier:
            raise ValueError("training runs on a device-tier bank")
        L = bank.layout
        self.bank, self.B, self.T, self.k, self.tau, self.device = bank, batch, T, top_k, tau, device
        self.local_off = _i64(local_off)
        self.cap = self.local_off[1:] - self.local_off[:-1]
        self.local_len = None if local_len is None else _i64(local_len)
        self.router = Router(bank, batch, T, top_k, device)
        self.rope = rope_table(L, int(top_k + self.cap.max().item()), device)
        self.ws_fwd = torch.zeros(decode_workspace_size(L, batch, T, self.local_off, self.local_len),
                                  dtype=torch.uint8, device=device)
        self.ws_bwd = torch.empty(attention_backward_workspace_size(L, batch, T), dtype=torch.uint8, device=device)
        self.ws_loss = torch.empty(route_loss_workspace_size(L, bank.index, batch, T), dtype=torch.uint8,
                                   device=device)
        H, d = L.c.n_kv_heads, L.c.head_dim
        self.out = torch.empty(batch, T, L.c.n_q_heads, d, dtype=L.torch_dtype, device=device)
        self.lse = torch.empty(batch, T, L.c.n_q_heads, dtype=torch.float32, device=device)
        self.loss = torch.empty(batch, dtype=torch.float32, device=device)
        self.k_rot = torch.empty(int(self.local_off[-1]) * H * d, dtype=L.torch_dtype, device=device)

    def forward(self, q, qr, local_k, local_v, pos_off, pos_doc, stream=None):
        """Returns (out [B][T][H_q][d], loss [B], selected [B][top_k])."""
        L, I = self.bank.layout, self.bank.index
        sel, _ = self.router(qr, stream)
        rope_local(L, self.local_off, self.k, local_k, self.k_rot, self.rope, None, stream,
                   local_len_host=self.local_len)
        sparse_attention_forward(L, I, q, self.k_rot, local_v, self.local_off, sel, self.k, self.rope, self.out,
                                 self.lse, self.ws_fwd, stream, self.local_len)
        route_loss_forward(L, I, qr, pos_off, pos_doc, self.tau, self.loss, self.ws_loss, stream=stream)
        self._saved = (q, qr, local_v, pos_off, pos_doc)
        return self.out, self.loss, sel

    def grad_buffers(self):
        """Zeroed fp32 gradient tensors for backward(): q, local_k (unrotated
        keys) and local_v in their own layouts, the bank's mem_k / mem_v
        [C][H_kv][d] and kr [C][H_kv][d_r], and qr."""
        L = self.bank.layout
        q, qr = self._saved[0], self._saved[1]
        H, d, dr = L.c.n_kv_heads, L.c.head_dim, L.c.router_dim
        C = self.bank.n_chunks
        dev = self.device
        return dict(q=torch.empty(q.shape, dtype=torch.float32, device=dev),
                    local_k=torch.zeros(self.k_rot.numel(), dtype=torch.float32, device=dev),
                    local_v=torch.zeros(self.k_rot.numel(), dtype=torch.float32, device=dev),
                    mem_k=torch.zeros(C, H, d, dtype=torch.float32, device=dev),
                    mem_v=torch.zeros(C, H, d, dtype=torch.float32, device=dev),
                    qr=torch.empty(qr.shape, dtype=torch.float32, device=dev),
                    kr=torch.zeros(C, H, dr, dtype=torch.float32, device=dev))

    def attention_backward(self, dout, g, stream=None):
        """The sparse attention's part of backward() into the buffers g."""
        L, I = self.bank.layout, self.bank.index
        q, local_v = self._saved[0], self._saved[2]
        sparse_attention_backward(L, I, q, self.k_rot, local_v, self.local_off, self.router.idx, self.k, self.rope,
                                  self.out, self.lse, dout, g["q"], g["mem_k"], g["mem_v"], g["local_k"],
                                  g["local_v"], self.ws_bwd, stream, self.local_len)

    def loss_backward(self, dloss, g, stream=None):
        """The routing loss's part of backward() into the buffers g."""
        L, I = self.bank.layout, self.bank.index
        qr, pos_off, pos_doc = self._saved[1], self._saved[3], self._saved[4]
        route_loss_backward(L, I, qr, pos_off, pos_doc, self.tau, dloss, g["qr"], g["kr"], self.ws_loss, stream)

    def backward(self, dout, dloss, stream=None):
        """Gradients of sum(out * dout) + sum(loss * dloss), as fp32 tensors
        (see grad_buffers for their layouts)."""
        g = self.grad_buffers()
        self.attention_backward(dout, g, stream)
        self.loss_backward(dloss, g, stream)
        return g
