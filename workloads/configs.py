"""Named synthetic workloads for the Memory Sparse Attention hot path.

Each workload fixes the shapes, dtypes and value distributions of one memory
bank plus the queries that decode against it.  The shapes follow the pages'
description of the method (Qwen3-4B-like attention heads, memories from 1M to
100M tokens; "EverMind-AI/MSA: Memory Sparse Attention for 100M-Token
Contexts", sections "What the evaluation numbers do and do not show" and "The
hardware floor and the missing licence file").  Nothing in this module computes
any part of the method: it only names sizes.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str                 # storage / arithmetic type of the bank: "f32" or "bf16"
    n_docs: int
    doc_len: int               # fixed length in tokens, or median when lognormal
    lognormal_sigma: float     # 0.0 = fixed lengths
    len_clip: tuple            # (lo, hi) clip of lognormal lengths
    chunk: int                 # pooling chunk size (tokens)
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    router_dim: int
    T: int                     # query tokens per call
    B: int                     # independent queries per call
    local_len: tuple           # (lo, hi) local context tokens per query (uniform); lo == hi: fixed
    top_k: int
    n_needles: int
    per_token: bool            # True: per-token K/V/Kr are generated and encoded;
                               # False: pooled chunks are generated directly
    kv_on_host: bool           # pooled K/V kept in pinned host memory
    rope_theta: float = 1.0e6
    seed: int = 0              # seeds the queries and local contexts
    mem_seed: int = 0          # seeds the memory bank (shared banks share it)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


# tiny fp32 memory: 64 docs x 512 tokens, 4 heads of 64 dims, T=4, one needle
TINY_F32 = Workload(
    name="tiny-fp32-64x512", dtype="f32", n_docs=64, doc_len=512,
    lognormal_sigma=0.0, len_clip=(512, 512), chunk=64, n_q_heads=4,
    n_kv_heads=4, head_dim=64, router_dim=64, T=4, B=1, local_len=(128, 128),
    top_k=4, n_needles=1, per_token=True, kv_on_host=False, seed=1000, mem_seed=1000)

# 1M-token memory (4096 docs x 256 tokens), Qwen3-4B-like heads, T=64 query tokens
MEM_1M = Workload(
    name="1m-bf16-4096x256-T64", dtype="bf16", n_docs=4096, doc_len=256,
    lognormal_sigma=0.0, len_clip=(256, 256), chunk=64, n_q_heads=32,
    n_kv_heads=8, head_dim=128, router_dim=128, T=64, B=1,
    local_len=(2048, 2048), top_k=16, n_needles=16, per_token=True,
    kv_on_host=False, seed=1001, mem_seed=1001)

# 16M-token memory: 65,536 docs with lognormal lengths (median 256, clip 32..4096)
MEM_16M = Workload(
    name="16m-bf16-lognormal-65536docs", dtype="bf16", n_docs=65536,
    doc_len=256, lognormal_sigma=0.3, len_clip=(32, 4096), chunk=64,
    n_q_heads=32, n_kv_heads=8, head_dim=128, router_dim=128, T=1, B=1,
    local_len=(4096, 4096), top_k=16, n_needles=0, per_token=False,
    kv_on_host=False, seed=1002, mem_seed=1002)

# 100M-token memory: 390,625 docs x 256 tokens; pooled K/V in pinned host memory
MEM_100M = Workload(
    name="100m-bf16-390625x256-hosttier", dtype="bf16", n_docs=390625,
    doc_len=256, lognormal_sigma=0.0, len_clip=(256, 256), chunk=64,
    n_q_heads=32, n_kv_heads=8, head_dim=128, router_dim=128, T=1, B=1,
    local_len=(4096, 4096), top_k=16, n_needles=0, per_token=False,
    kv_on_host=True, seed=1003, mem_seed=1003)

# 32 independent T=1 queries on the 16M-token lognormal memory, own local ctx 1024..8192
MEM_16M_B32 = Workload(
    name="16m-bf16-lognormal-batch32", dtype="bf16", n_docs=65536,
    doc_len=256, lognormal_sigma=0.3, len_clip=(32, 4096), chunk=64,
    n_q_heads=32, n_kv_heads=8, head_dim=128, router_dim=128, T=1, B=32,
    local_len=(1024, 8192), top_k=32, n_needles=32, per_token=False,
    kv_on_host=False, seed=1004, mem_seed=1002)

ALL = [TINY_F32, MEM_1M, MEM_16M, MEM_100M, MEM_16M_B32]
BY_NAME = {w.name: w for w in ALL}
