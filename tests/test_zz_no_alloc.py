"""msa_route_noalloc: routing for callers that may not allocate device memory.

Some users embed this library where they cannot call cudaMalloc -- for example
inside a host application that owns all device memory, or in a serving loop
that cannot afford cudaMalloc's device-wide synchronisation -- so they cannot
hand msa_route a workspace.  msa_route_noalloc serves them from a 16 MiB
scratch array built into the library.  These tests call it through the C ABI
twice in a row (different queries each time, so the second call runs on the
first call's leftover scratch) and check each result against msa_route with a
caller workspace: identical document indices and identical fp64 scores, the
bar every routing test here uses.  One query row takes the CUDA-core scan; a
batch of 8 takes the tensor-core scan, on a bank cut so that its plan lands
256 bytes under the scratch's size.  A size beyond the built-in scratch is
refused before anything runs.

This file is named so that pytest collects it last.
"""
import pytest
import torch

import routed_sparse_attention_b200 as msa
from routed_sparse_attention_b200 import Layout
from routed_sparse_attention_b200.runtime import Bank, Router
from workloads import MEM_16M, gen

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

MAX_BYTES = 16 << 20


def _same_as_route(lay, bank, router, queries, k):
    for qr in queries:
        idx_ref, sc_ref = router(qr)
        idx_ref, sc_ref = idx_ref.clone(), sc_ref.clone()
        B = qr.shape[0]
        idx = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
        sc = torch.zeros(B, k, dtype=torch.float64, device="cuda")
        msa.route_noalloc(lay, bank.index, qr, k, idx, sc)
        torch.cuda.synchronize()
        assert torch.equal(idx, idx_ref)
        assert torch.equal(sc, sc_ref)
    assert msa.device_status() == 0


def test_route_noalloc_matches_route_on_two_calls_in_a_row():
    w = MEM_16M
    x = gen.generate(w, device="cuda")
    lay = Layout.of(w)
    bank = Bank(lay, x["doc_tok_off"], kr_pool=x["kr_pool"], k_pool=x["k_pool"], v_pool=x["v_pool"])
    need = msa.route_workspace_size(lay, bank.n_docs, bank.n_chunks, 1, 1, w.top_k)
    assert 0 < need <= MAX_BYTES
    router = Router(bank, 1, 1, w.top_k)
    queries = [x["qr"], gen.make_queries(w.replace(seed=w.seed + 7), "cuda")["qr"]]
    _same_as_route(lay, bank, router, queries, w.top_k)

    # a batch whose workspace exceeds the built-in scratch is refused up front
    big = torch.zeros(64, 1, w.n_q_heads, w.router_dim, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(64, w.top_k, dtype=torch.int32, device="cuda")
    with pytest.raises(msa.MSAError) as e:
        msa.route_noalloc(lay, bank.index, big, w.top_k, out)
    assert e.value.status == 4


def test_route_noalloc_tensor_core_scan_just_under_the_limit():
    """8 single-token queries (tensor-core scan) over the first documents of
    the 16M-token bank, as many as keep the plan within the scratch."""
    w = MEM_16M.replace(B=8, local_len=(8, 8))
    x = gen.generate(w, device="cuda")
    lay = Layout.of(w)
    coff = gen.offsets((gen.doc_lengths(w) + w.chunk - 1) // w.chunk)
    tok = x["doc_tok_off"]

    def need(d):
        return msa.route_workspace_size(lay, d, int(coff[d]), w.B, 1, w.top_k)

    lo, hi = 1, w.n_docs                      # largest document count that fits
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if need(mid) <= MAX_BYTES:
            lo = mid
        else:
            hi = mid
    D = lo
    assert MAX_BYTES - 4096 < need(D) <= MAX_BYTES
    C = int(coff[D])
    bank = Bank(lay, tok[:D + 1], kr_pool=x["kr_pool"][:C], k_pool=x["k_pool"][:C], v_pool=x["v_pool"][:C])
    assert bank.n_chunks == C
    router = Router(bank, w.B, 1, w.top_k)
    queries = [x["qr"], gen.make_queries(w.replace(seed=w.seed + 11), "cuda")["qr"]]
    _same_as_route(lay, bank, router, queries, w.top_k)

    # one more document no longer fits and is refused
    bank2 = Bank(lay, tok[:D + 2], kr_pool=x["kr_pool"][:int(coff[D + 1])], inv_norms=False)
    out = torch.empty(w.B, w.top_k, dtype=torch.int32, device="cuda")
    with pytest.raises(msa.MSAError) as e:
        msa.route_noalloc(lay, bank2.index, x["qr"], w.top_k, out)
    assert e.value.status == 4
