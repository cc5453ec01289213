"""GPU parity of Memory Interleave: rounds of retrieval -> context expansion
-> generation (runtime.MemoryInterleave over msa_route, msa_interleave_expand,
msa_rope_local and msa_sparse_decode).

Every round's selected set must equal the oracle's expansion of the previous
set bit for bit, and every generated token must match the oracle's decode over
[the set's documents in joining order ++ the live local context] with the
global RoPE offset k = |S|, within the bf16 tolerance.  The expansion kernel
is also checked alone against the oracle on given document scores, at the set
size limits and with ties, and on a set that holds a document twice."""
import numpy as np
import pytest
import torch

import oracle
import routed_sparse_attention_b200 as msa
from gpu_cases import BF16_TOL
from routed_sparse_attention_b200 import Layout
from routed_sparse_attention_b200.runtime import Bank, MemoryInterleave
from workloads import Workload, gen

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

BASE = Workload(name="interleave", dtype="bf16", n_docs=300, doc_len=200, lognormal_sigma=0.5,
                len_clip=(1, 1000), chunk=64, n_q_heads=32, n_kv_heads=8, head_dim=128, router_dim=128,
                T=1, B=3, local_len=(1, 1), top_k=8, n_needles=0, per_token=False, kv_on_host=False,
                seed=700, mem_seed=800)


def _bank(host: bool, B: int):
    w = BASE.replace(name="interleave-host" if host else "interleave", kv_on_host=host, B=B)
    qr0 = torch.zeros(w.B, w.T, w.n_q_heads, w.router_dim)
    x = gen.make_memory(w, qr0, "cuda", host_interleaved=host)
    bank = Bank(Layout.of(w), x["doc_tok_off"], kr_pool=x["kr_pool"], k_pool=x.get("k_pool"),
                v_pool=x.get("v_pool"), host_kv=x.get("host_kv"))
    return w, x, bank


def _randn(g, *shape):
    return torch.randn(*shape, generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("host,B,query_mode", [(False, 3, "drift"), (True, 2, "drift"), (False, 2, "constant")],
                         ids=["device-B3-drift", "hosttier-B2-drift", "device-B2-constant"])
def test_interleave_rounds_expand_and_decode(host, B, query_mode):
    w, x, bank = _bank(host, B)
    H, d, Hq, dr = w.n_kv_heads, w.head_dim, w.n_q_heads, w.router_dim
    p, rounds, gen_per_round = 4, 3, 2
    prompt = [17, 29, 5][:B]
    mi = MemoryInterleave(bank, B, p, p * rounds, torch.tensor(prompt),
                          torch.tensor(prompt) + rounds * gen_per_round)
    g = torch.Generator().manual_seed(4321 + B)
    kp = [_randn(g, H, prompt[b], d) for b in range(B)]
    vp = [_randn(g, H, prompt[b], d) for b in range(B)]
    mi.prefill([t.cuda() for t in kp], [t.cuda() for t in vp])
    coff = oracle.chunk_offsets(x["doc_tok_off"], w.chunk)
    kr_host = x["kr_pool"].cpu()
    qr0 = torch.randn(B, 1, Hq, dr, generator=g)
    ref_sel = np.zeros((B, 0), np.int32)
    overlap = 0
    for r in range(rounds):
        # "drift": each hop's router query stays close to the last one, so the
        # ranking keeps documents that are already selected and the expansion
        # has to skip them
        qr = qr0 if query_mode == "constant" else qr0 + 0.35 * torch.randn(B, 1, Hq, dr, generator=g)
        qr = qr.to(torch.bfloat16)
        sel = mi.expand(qr.cuda())
        torch.cuda.synchronize()
        ranked, _ = oracle.route(qr, coff, kr_host, ref_sel.shape[1] + p, H)
        overlap += sum(len(set(ranked[b].tolist()) & set(ref_sel[b].tolist())) for b in range(B))
        ref_sel = oracle.interleave_expand(qr, coff, kr_host, ref_sel, p, H)
        assert np.array_equal(sel.cpu().numpy(), ref_sel), r
        k = ref_sel.shape[1]
        for t in range(gen_per_round):
            q = _randn(g, B, 1, Hq, d)
            kn, vn = _randn(g, B, H, d), _randn(g, B, H, d)
            out = mi.generate(q.cuda(), kn.cuda(), vn.cuda())
            torch.cuda.synchronize()
            for b in range(B):
                kp[b] = torch.cat([kp[b], kn[b].unsqueeze(1)], dim=1)
                vp[b] = torch.cat([vp[b], vn[b].unsqueeze(1)], dim=1)
            lens = [kp[b].shape[1] for b in range(B)]
            loff = np.concatenate([[0], np.cumsum(lens)])
            lk = torch.cat([kp[b].reshape(-1) for b in range(B)])
            lv = torch.cat([vp[b].reshape(-1) for b in range(B)])
            if host:
                ref = oracle.decode(q, ref_sel, coff, x["host_kv"], None, loff, lk, lv, k, w.rope_theta, H,
                                    kv_layout=oracle.KV_DOC_INTERLEAVED)
            else:
                ref = oracle.decode(q, ref_sel, coff, x["k_pool"].cpu(), x["v_pool"].cpu(), loff, lk, lv, k,
                                    w.rope_theta, H)
            err = float(np.max(np.abs(out.float().cpu().numpy() - ref)))
            print(f"[interleave round {r} token {t} |S|={k}] max |out - oracle| = {err:.3e}")
            assert err <= BF16_TOL, (r, t, err)
    assert overlap > 0, "no round re-ranked an already selected document: the exclusion went untested"
    if query_mode == "constant":                      # R rounds of one query = its top R*p
        want, _ = oracle.route(qr0.to(torch.bfloat16), coff, kr_host, rounds * p, H)
        assert np.array_equal(ref_sel, want)
    assert msa.device_status() == 0


def _ranking(ds, m):
    """Top-m documents by (score desc, index asc): what msa_route returns."""
    D = ds.shape[1]
    return np.stack([np.lexsort((np.arange(D), -row))[:m] for row in ds]).astype(np.int32)


@pytest.mark.parametrize("n,p", [(0, 5), (8, 4), (60, 4), (1, 63), (31, 2), (32, 32)])
def test_expand_kernel_matches_oracle_on_given_scores(n, p):
    rng = np.random.default_rng(n * 100 + p)
    B, D = 37, 200
    ds = np.round(rng.standard_normal((B, D)), 1)               # coarse: many ties
    # old sets: half from each query's ranking (which the expansion must then
    # skip), half from outside it, in random order
    top = _ranking(ds, n + p)
    old = np.zeros((B, n), np.int32)
    for b in range(B):
        inside = top[b][: (n + 1) // 2]
        outside = rng.choice(np.setdiff1d(np.arange(D), top[b]), n - len(inside), replace=False)
        old[b] = rng.permutation(np.concatenate([inside, outside]))
    want = oracle.interleave_expand_scores(ds, old, p)
    ranked = torch.from_numpy(_ranking(ds, n + p)).cuda()
    got = torch.full((B, n + p), -7, dtype=torch.int32, device="cuda")
    host = torch.empty(B, n + p, dtype=torch.int32, pin_memory=True)
    msa.interleave_expand(D, ranked, torch.from_numpy(old).cuda() if n else None, got, host)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), want)
    assert np.array_equal(host.numpy(), want)
    assert msa.device_status() == 0


def test_expand_kernel_flags_a_set_with_a_document_twice():
    B, D, n, p = 2, 50, 3, 2
    ds = np.linspace(1.0, 0.0, D)[None].repeat(B, 0)
    ranked = torch.from_numpy(_ranking(ds, n + p)).cuda()      # documents 0..4
    old = torch.tensor([[0, 0, 1], [7, 8, 9]], dtype=torch.int32, device="cuda")
    got = torch.empty(B, n + p, dtype=torch.int32, device="cuda")
    msa.interleave_expand(D, ranked, old, got)
    torch.cuda.synchronize()
    assert msa.device_status() & 0x10                          # MSA_DEV_BAD_SET
    assert got[1].tolist() == [7, 8, 9, 0, 1]                   # the valid query is served
    assert got[0].tolist()[:3] == [0, 0, 1]
    assert msa.device_status() == 0                             # the status word was cleared
