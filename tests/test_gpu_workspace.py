"""msa_route writes nothing past a workspace of exactly msa_route_workspace_size
bytes.

The workspace is the head of a larger buffer whose tail (a guard region) holds
a known byte pattern; after routing, the guard must be unchanged and the result
must equal routing with a generous workspace.  Cases: one query row (CUDA-core
scan), a batch of 8 single-token queries and one 64-token query (tensor-core
scan, whose tile table grows with the bank's chunk count), on the 16M-token
lognormal memory (306,369 pooled chunks).
"""
import pytest
import torch

import routed_sparse_attention_b200 as msa
from routed_sparse_attention_b200 import Layout
from routed_sparse_attention_b200.runtime import Bank
from workloads import MEM_16M, gen

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

GUARD = 1 << 20
PATTERN = 0xA5


@pytest.fixture(scope="module")
def bank16m():
    w = MEM_16M
    x = gen.generate(w, device="cuda")
    lay = Layout.of(w)
    bank = Bank(lay, x["doc_tok_off"], kr_pool=x["kr_pool"], k_pool=x["k_pool"], v_pool=x["v_pool"])
    torch.cuda.synchronize()
    return w, lay, bank


@pytest.mark.parametrize("B,T", [(1, 1), (8, 1), (1, 64)])
def test_route_stays_inside_an_exact_workspace(bank16m, B, T):
    w, lay, bank = bank16m
    q = gen.make_queries(w.replace(B=B, T=T, local_len=(8, 8), seed=w.seed + 100 * B + T), "cuda")["qr"]
    k = 16
    need = msa.route_workspace_size(lay, bank.n_docs, bank.n_chunks, B, T, k)
    assert need > 0 and need % 256 == 0
    buf = torch.full((need + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
    ws = buf[:need]
    idx = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    sc = torch.zeros(B, k, dtype=torch.float64, device="cuda")
    msa.route(lay, bank.index, q, k, idx, sc, ws=ws)

    roomy = torch.empty(need + (64 << 20), dtype=torch.uint8, device="cuda")
    idx2 = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    sc2 = torch.zeros(B, k, dtype=torch.float64, device="cuda")
    msa.route(lay, bank.index, q, k, idx2, sc2, ws=roomy)
    torch.cuda.synchronize()
    assert bool((buf[need:] == PATTERN).all()), "routing wrote past its workspace"
    assert torch.equal(idx, idx2) and torch.equal(sc, sc2)
    assert msa.device_status() == 0
