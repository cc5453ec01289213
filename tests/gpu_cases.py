"""Shared set-up for the GPU parity tests: one workload's seeded inputs on the
GPU, the library objects around them, and host copies for the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from routed_sparse_attention_b200 import Layout
from routed_sparse_attention_b200.runtime import Bank, Decoder, Router
from workloads import gen

BF16_TOL = 2e-2     # absolute, bf16 attention outputs
F32_TOL = 1e-5      # absolute, fp32 attention outputs
ROUTE_EPS = 1.0 / 4096.0   # certified bound on |fast score - exact score|


def out_tol(w):
    return F32_TOL if w.dtype == "f32" else BF16_TOL


class Case:
    """Inputs of workload w on the GPU plus the library objects that use them."""

    def __init__(self, w, device="cuda", mutate=None, pooled=None, inv_norms=True, decode=True):
        """mutate(x) may edit the generated tensors before the bank is built;
        pooled=(k, v, kr) replaces the bank with these pooled tensors;
        inv_norms=False leaves the router-key norms to the scan itself."""
        self.w = w
        self.x = gen.generate(w, device=device, host_interleaved=w.kv_on_host)
        self.layout = Layout.of(w)
        x = self.x
        if mutate is not None:
            mutate(x)
        if pooled is not None:
            x["k_pool"], x["v_pool"], x["kr_pool"] = (t.to(device) for t in pooled)
            w = self.w = w.replace(per_token=False)
        if w.per_token:
            self.bank = Bank(self.layout, x["doc_tok_off"], k_tok=x["k_tok"], v_tok=x["v_tok"],
                             kr_tok=x["kr_tok"], device=device, inv_norms=inv_norms)
        else:
            self.bank = Bank(self.layout, x["doc_tok_off"], kr_pool=x["kr_pool"],
                             k_pool=x.get("k_pool"), v_pool=x.get("v_pool"),
                             host_kv=x.get("host_kv"), device=device, inv_norms=inv_norms)
        self.router = Router(self.bank, w.B, w.T, w.top_k, device)
        self.decoder = None
        if decode:
            self.decoder = Decoder(self.bank, w.B, w.T, w.top_k, x["local_off"], device)
            # the key cache decode reads: every local key rotated at top_k + j
            x["local_k_rot"] = self.decoder.rotate_local(x["local_k"], torch.empty_like(x["local_k"]))
        torch.cuda.synchronize()

    @property
    def chunk_off(self) -> np.ndarray:
        return oracle.chunk_offsets(self.x["doc_tok_off"], self.w.chunk)

    def route(self):
        idx, sc = self.router(self.x["qr"])
        torch.cuda.synchronize()
        return idx.cpu().numpy(), sc.cpu().numpy()

    def decode(self, sel_dev):
        x = self.x
        if self.bank.host_tier:
            sel_host = sel_dev.cpu().to(torch.int32).pin_memory()
            s = torch.cuda.current_stream()
            ev = torch.cuda.Event()
            ev.record(s)
            done = torch.cuda.Event()
            done.record(s)                              # creates the event handle
            self.decoder.fetch(sel_host, ev, s, done)
            out = self.decoder(x["q"], x["local_k_rot"], x["local_v"], sel_dev, wait_event=done)
        else:
            out = self.decoder(x["q"], x["local_k_rot"], x["local_v"], sel_dev)
        torch.cuda.synchronize()
        return out.float().cpu().numpy()

    # ---- oracle side (host copies of the same generated inputs)
    def oracle_route(self, kr=None, queries=None):
        qr = self.x["qr"].cpu()
        if queries is not None:
            qr = qr[queries]
        kr = self.x["kr_pool"].cpu() if kr is None else kr
        return oracle.route(qr, self.chunk_off, kr, self.w.top_k, self.w.n_kv_heads, want_scores=True)

    def oracle_decode(self, sel, k_pool=None, v_pool=None, queries=None):
        """Oracle decode for the given queries (all by default)."""
        w, x = self.w, self.x
        B = w.B
        queries = list(range(B)) if queries is None else list(queries)
        loff = x["local_off"]
        d, H = w.head_dim, w.n_kv_heads
        lk_all, lv_all = x["local_k"], x["local_v"]
        q = x["q"].cpu()[queries]
        lks, lvs, lo = [], [], [0]
        for b in queries:
            a, e = int(loff[b]) * H * d, int(loff[b + 1]) * H * d
            lks.append(lk_all[a:e].cpu())
            lvs.append(lv_all[a:e].cpu())
            lo.append(lo[-1] + int(loff[b + 1] - loff[b]))
        lk, lv = torch.cat(lks), torch.cat(lvs)
        if self.bank.host_tier:
            return oracle.decode(q, sel, self.chunk_off, x["host_kv"], None, np.array(lo), lk, lv,
                                 w.top_k, w.rope_theta, H, kv_layout=oracle.KV_DOC_INTERLEAVED)
        kp = x["k_pool"].cpu() if k_pool is None else k_pool
        vp = x["v_pool"].cpu() if v_pool is None else v_pool
        return oracle.decode(q, sel, self.chunk_off, kp, vp, np.array(lo), lk, lv, w.top_k,
                             w.rope_theta, H)
