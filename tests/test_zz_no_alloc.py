"""msa_route_noalloc: routing for callers that may not allocate device memory.

Some users embed this library where they cannot call cudaMalloc -- for example
inside a host application that owns all device memory, or in a serving loop
that cannot afford cudaMalloc's device-wide synchronisation -- so they cannot
hand msa_route a workspace.  msa_route_noalloc serves them from a 16 MiB
scratch array built into the library.  This test calls it through the C ABI
twice in a row (different queries each time, so the second call runs on the
first call's leftover scratch) and checks each result against msa_route with a
caller workspace: identical document indices and identical fp64 scores, the
bar every routing test here uses.  It also checks that a size beyond the
built-in scratch is refused before anything runs.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import routed_sparse_attention_b200 as msa
from routed_sparse_attention_b200 import Layout
from routed_sparse_attention_b200.runtime import Bank, Router
from workloads import MEM_16M, gen

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)


def test_route_noalloc_matches_route_on_two_calls_in_a_row():
    w = MEM_16M
    x = gen.generate(w, device="cuda")
    lay = Layout.of(w)
    bank = Bank(lay, x["doc_tok_off"], kr_pool=x["kr_pool"], k_pool=x["k_pool"], v_pool=x["v_pool"])
    need = msa.route_workspace_size(lay, bank.n_docs, 1, 1, w.top_k)
    assert 0 < need <= 16 << 20
    router = Router(bank, 1, 1, w.top_k)
    queries = [x["qr"], gen.make_queries(w.replace(seed=w.seed + 7), "cuda")["qr"]]
    for qr in queries:
        idx_ref, sc_ref = router(qr)
        idx_ref, sc_ref = idx_ref.clone(), sc_ref.clone()
        idx = torch.full((1, w.top_k), -1, dtype=torch.int32, device="cuda")
        sc = torch.zeros(1, w.top_k, dtype=torch.float64, device="cuda")
        msa.route_noalloc(lay, bank.index, qr, w.top_k, idx, sc)
        torch.cuda.synchronize()
        assert torch.equal(idx, idx_ref)
        assert torch.equal(sc, sc_ref)
    assert msa.device_status() == 0

    # a batch whose workspace exceeds the built-in scratch is refused up front
    big = torch.zeros(64, 1, w.n_q_heads, w.router_dim, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(64, w.top_k, dtype=torch.int32, device="cuda")
    with pytest.raises(msa.MSAError) as e:
        msa.route_noalloc(lay, bank.index, big, w.top_k, out)
    assert e.value.status == 4
