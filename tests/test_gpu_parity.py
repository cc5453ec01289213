"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle on
the same seeded inputs.  Routing indices must be identical and the certified
exact scores bit-identical doubles; attention outputs within 2e-2 (bf16) or
1e-5 (fp32) absolute; pooled vectors within one rounding of their dtype."""
import numpy as np
import pytest
import torch

import oracle
import routed_sparse_attention_b200 as msa
from gpu_cases import ROUTE_EPS, Case, out_tol
from workloads import MEM_16M, MEM_16M_B32, MEM_1M, MEM_100M, TINY_F32, Workload, gen

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)


def assert_status_clean():
    assert msa.device_status() == 0


def round_like(a: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    return torch.from_numpy(a).to(dtype)


def check_pooled(gpu: torch.Tensor, ref: np.ndarray, dtype: torch.dtype):
    g = gpu.float().cpu().numpy().astype(np.float64)
    if dtype == torch.float32:
        assert np.max(np.abs(g - ref)) <= 1e-5
    else:   # one bf16 rounding (2^-8 relative) plus fp32 accumulation
        assert np.all(np.abs(g - ref) <= (2.0 ** -8 + 1e-5) * np.abs(ref) + 1e-6)


def check_out(w, out, ref):
    """Decode output within the dtype's absolute tolerance; the error is
    printed (visible with pytest -s)."""
    err = float(np.max(np.abs(out - ref)))
    print(f"[{w.name}] max |out - oracle| = {err:.3e} (tolerance {out_tol(w):.0e})")
    assert err <= out_tol(w)


def check_route(case: Case, queries=None):
    idx, sc = case.route()
    oi, osc, ods = case.oracle_route(queries=queries)
    if queries is not None:
        idx, sc = idx[queries], sc[queries]
    assert np.array_equal(idx, oi), f"indices differ:\n{idx}\n{oi}"
    assert np.array_equal(sc, osc), "exact scores differ"
    return idx, ods


# ------------------------------------------------------------------ tiny fp32

def test_tiny_fp32_encode_route_decode():
    w = TINY_F32
    case = Case(w)
    x = case.x
    kp, vp, krp = oracle.encode(x["doc_tok_off"], x["k_tok"].cpu(), x["v_tok"].cpu(),
                                x["kr_tok"].cpu(), w.chunk, w.rope_theta)
    check_pooled(case.bank.k, kp, torch.float32)
    check_pooled(case.bank.v, vp, torch.float32)
    check_pooled(case.bank.kr, krp, torch.float32)
    assert np.array_equal(case.bank.doc_chunk_off_host.numpy(), case.chunk_off)
    # whole GPU chain selects the planted needle
    idx_chain, _ = case.route()
    assert int(x["needle_docs"][0]) in idx_chain[0].tolist()
    # route + decode on the oracle-encoded bank (same bytes on both sides)
    pooled = tuple(round_like(a, torch.float32) for a in (kp, vp, krp))
    c2 = Case(w, pooled=pooled)
    idx, _ = check_route(c2)
    out = c2.decode(c2.router.idx)
    ref = c2.oracle_decode(idx)
    check_out(w, out, ref)
    assert_status_clean()


# ------------------------------------------------------------------ mid-size, ragged

MID = Workload(
    name="mid-lognormal-5000docs-B3-T2", dtype="bf16", n_docs=5000, doc_len=256,
    lognormal_sigma=0.6, len_clip=(1, 4096), chunk=64, n_q_heads=32, n_kv_heads=8,
    head_dim=128, router_dim=128, T=2, B=3, local_len=(1, 700), top_k=16, n_needles=3,
    per_token=False, kv_on_host=False, seed=77, mem_seed=78)


@pytest.mark.parametrize("w", [
    MID,
    MID.replace(name="mid-T1-B1", T=1, B=1, n_needles=1, local_len=(300, 300)),
    MID.replace(name="mid-T3-B2-k64", T=3, B=2, top_k=64, n_needles=2, local_len=(0, 40)),
    MID.replace(name="mid-hosttier", kv_on_host=True, B=2, T=1, n_needles=2),
    MID.replace(name="mid-f32-H4", dtype="f32", n_q_heads=8, n_kv_heads=4, head_dim=64,
                router_dim=64, n_docs=700, len_clip=(1, 300)),
    # 16 < G*T <= 32 query rows per kv head: two m16 row blocks per CTA
    MID.replace(name="mid-T6-B2", T=6, B=2, n_needles=2, local_len=(100, 900)),
    # head_dim 64 and more than 32 rows per kv head: four row blocks per CTA
    MID.replace(name="mid-d64-T20", n_q_heads=8, n_kv_heads=4, head_dim=64, T=20, B=1,
                n_needles=1, local_len=(50, 500)),
    # 160 query rows: two tensor-core scan passes of 128 rows
    MID.replace(name="mid-T40-B4-2pass", T=40, B=4, n_needles=4, local_len=(10, 300)),
    # the smallest tensor-core scan (5 rows), top_k = 1, documents of 1-64 tokens
    MID.replace(name="mid-B5-k1-short", B=5, T=1, top_k=1, n_needles=5, len_clip=(1, 64),
                local_len=(1, 200)),
    # no context: the query token's own key only (L_b = 0, Ltot = T = 1)
    MID.replace(name="mid-L0-T1-B3", B=3, T=1, n_needles=3, local_len=(0, 0)),
    # host tier with a batch of 8 through the tensor-core scan and decode
    MID.replace(name="mid-hosttier-B8", kv_on_host=True, B=8, T=1, n_needles=8, local_len=(64, 400)),
    # tcgen05 decode with 8 query heads per kv head: 96 rows in one 128-row group
    MID.replace(name="mid-G8-T12-B2-tc", n_q_heads=64, T=12, B=2, n_needles=2, local_len=(40, 500)),
    # tcgen05 decode over three row groups (128 + 128 + 24 rows), no local prefix
    MID.replace(name="mid-T70-B1-3rg", T=70, B=1, n_needles=1, local_len=(0, 0)),
    # tcgen05 decode on the host tier: the memory split gathers from the staging buffer
    MID.replace(name="mid-hosttier-T20-B2-tc", kv_on_host=True, B=2, T=20, n_needles=2, local_len=(30, 400)),
], ids=lambda w: w.name)
def test_mid_route_decode(w):
    case = Case(w)
    idx, ods = check_route(case)
    for j, (b, _) in enumerate(case.x["needle_targets"]):
        assert int(case.x["needle_docs"][j]) in idx[b].tolist()
    out = case.decode(case.router.idx)
    ref = case.oracle_decode(idx)
    check_out(w, out, ref)
    fast = case.router.fast_scores(case.x["qr"]).cpu().numpy()
    assert np.max(np.abs(fast - ods)) <= ROUTE_EPS / 10
    assert_status_clean()


# Single-query decode edges: the memory split's ring of gathered tiles, a
# local context long enough for many tile rounds per split, an almost empty
# context, four query tokens, two queries on the host tier, head_dim 64.
@pytest.mark.parametrize("w", [
    # 64 documents of 2048 tokens: 2048 memory keys through the memory split's two stages
    MID.replace(name="dec-k64-longdocs", B=1, T=1, top_k=64, n_needles=1, lognormal_sigma=0.0,
                doc_len=2048, len_clip=(2048, 2048), n_docs=400, local_len=(50, 50)),
    # 20,000 local tokens: many tiles per local split
    MID.replace(name="dec-local20k", B=1, T=1, n_needles=1, local_len=(20000, 20000)),
    # a one-token context: the query token's own key only
    MID.replace(name="dec-L1", B=1, T=1, n_needles=1, local_len=(1, 1)),
    # T = 4: 16 query rows, causal among the query tokens
    MID.replace(name="dec-T4", B=1, T=4, n_needles=1, local_len=(777, 777)),
    # two queries, host tier
    MID.replace(name="dec-B2-hosttier", B=2, T=1, kv_on_host=True, n_needles=2, local_len=(900, 3000)),
    # head_dim 64, four kv heads, two query tokens
    MID.replace(name="dec-d64-H4", n_q_heads=16, n_kv_heads=4, head_dim=64, router_dim=128, B=1, T=2,
                n_needles=1, local_len=(1500, 1500)),
], ids=lambda w: w.name)
def test_single_query_decode_edges(w):
    case = Case(w)
    idx, _ = check_route(case)
    out = case.decode(case.router.idx)
    check_out(w, out, case.oracle_decode(idx))
    # the same call again: the split counters were left at zero
    out2 = case.decode(case.router.idx)
    assert np.array_equal(out, out2)
    assert_status_clean()


def test_hosttier_device_fetch_equals_the_copy_fetch():
    """msa_fetch_selected_device (one kernel reading the mapped host tier)
    fills every staging slot with the same bytes as the per-document copies;
    the decode from it matches the oracle; a selected document out of range
    raises MSA_DEV_BAD_DOC and leaves its slot alone."""
    w = MID.replace(name="mid-hosttier-devfetch", kv_on_host=True, B=3, T=1, n_needles=3, local_len=(64, 400))
    case = Case(w)
    idx, _ = check_route(case)
    dec = case.decoder
    sel_host = case.router.idx.cpu().to(torch.int32).pin_memory()
    s = torch.cuda.current_stream()
    ev, done = torch.cuda.Event(), torch.cuda.Event()
    ev.record(s)
    done.record(s)
    dec.fetch(sel_host, ev, s, done)
    torch.cuda.synchronize()
    copied = dec.staging.clone()
    dec.staging.fill_(0x5A)
    dec.fetch_device(case.router.idx)
    torch.cuda.synchronize()
    row = w.n_kv_heads * w.head_dim * 2
    slot = 2 * case.bank.max_doc_chunks * row
    coff = case.chunk_off
    for i, doc in enumerate(idx.reshape(-1).tolist()):
        n = 2 * int(coff[doc + 1] - coff[doc]) * row
        assert torch.equal(dec.staging[i * slot:i * slot + n], copied[i * slot:i * slot + n]), i
    out = case.x
    got = dec(out["q"], out["local_k_rot"], out["local_v"], case.router.idx)
    torch.cuda.synchronize()
    check_out(w, got.float().cpu().numpy(), case.oracle_decode(idx))
    assert_status_clean()
    bad = case.router.idx.clone()
    bad[1, 2] = w.n_docs + 5
    before = dec.staging.clone()
    dec.fetch_device(bad)
    torch.cuda.synchronize()
    assert msa.device_status() & msa.DEV_BAD_DOC
    i = 1 * w.top_k + 2
    assert torch.equal(dec.staging[i * slot:(i + 1) * slot], before[i * slot:(i + 1) * slot])
    assert_status_clean()


@pytest.mark.parametrize("w", [
    MID.replace(name="raw-B3-T2", B=3, T=2, n_needles=3, local_len=(10, 500)),
    MID.replace(name="raw-hosttier-B2", B=2, T=1, kv_on_host=True, n_needles=2, local_len=(64, 700)),
], ids=lambda w: w.name)
def test_raw_key_decode_in_one_call(w):
    """msa_sparse_decode_raw takes the unrotated local keys (and fetches the
    host tier itself): the same output, bit for bit, as rotating into a key
    cache and decoding, and the oracle's within the tolerance."""
    case = Case(w)
    idx, _ = check_route(case)
    x, dec = case.x, case.decoder
    ref_out = case.decode(case.router.idx)
    n = msa.sparse_decode_raw_workspace_size(case.layout, case.bank.index, w.B, w.T, w.top_k, x["local_off"])
    assert n > 0
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(dec.out)
    for _ in range(2):                          # a second call on the same workspace
        msa.sparse_decode_raw(case.layout, case.bank.index, x["q"], x["local_k"], x["local_v"], x["local_off"],
                              case.router.idx, w.top_k, dec.rope, out, ws)
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()
        assert np.array_equal(got, ref_out)
        check_out(w, got, case.oracle_decode(idx))
    assert_status_clean()


def test_k_equals_all_documents_and_single_token_docs():
    w = MID.replace(name="k-eq-D", n_docs=24, doc_len=3, lognormal_sigma=1.0, len_clip=(1, 70),
                    top_k=24, B=2, T=1, n_needles=0, local_len=(1, 9))
    assert (gen.doc_lengths(w) == 1).any()
    case = Case(w)
    idx, ods = check_route(case)
    assert all(sorted(r.tolist()) == list(range(24)) for r in idx)
    out = case.decode(case.router.idx)
    check_out(w, out, case.oracle_decode(idx))


def test_exact_ties_and_zero_router_keys():
    w = MID.replace(name="ties", n_docs=300, lognormal_sigma=0.0, doc_len=128, B=1, T=1,
                    n_needles=1, top_k=8)
    holder = {}

    def mutate(x):
        a = int(x["needle_docs"][0])
        b = (a + 37) % w.n_docs
        lo = min(a, b)
        holder["pair"] = (lo, max(a, b))
        kr = x["kr_pool"]
        kr[2 * b:2 * b + 2] = kr[2 * a:2 * a + 2]          # duplicate document -> exact tie
        kr[2 * ((a + 5) % w.n_docs):2 * ((a + 5) % w.n_docs) + 2] = 0   # zero router keys
    case = Case(w, mutate=mutate)
    idx, _ = check_route(case)
    lo, hi = holder["pair"]
    assert idx[0][:2].tolist() == [lo, hi]
    assert case.router.score[0, 0].item() == case.router.score[0, 1].item()


# ------------------------------------------------------------------ 1M-token, T = 64

def test_1m_gpu_encoded_bank_all_docs_route_decode():
    """The 1M configuration as stated: per-token Gaussian K/V/Kr encoded on
    the GPU.  Every pooled vector of all 4096 documents against the oracle's
    encode; then routing (tensor-core scan, T = 64) and decode on the
    GPU-encoded bank against the oracle on the same bytes."""
    w = MEM_1M
    case = Case(w)
    x = case.x
    kp, vp, krp = oracle.encode(x["doc_tok_off"], x["k_tok"].cpu(), x["v_tok"].cpu(),
                                x["kr_tok"].cpu(), w.chunk, w.rope_theta)
    check_pooled(case.bank.k, kp, torch.bfloat16)
    check_pooled(case.bank.v, vp, torch.bfloat16)
    check_pooled(case.bank.kr, krp, torch.bfloat16)
    del kp, vp, krp
    bk, bv, bkr = case.bank.k.cpu(), case.bank.v.cpu(), case.bank.kr.cpu()
    idx, sc = case.route()
    oi, osc, ods = case.oracle_route(kr=bkr)
    assert np.array_equal(idx, oi) and np.array_equal(sc, osc)
    assert set(x["needle_docs"].tolist()) == set(idx[0].tolist())
    out = case.decode(case.router.idx)
    check_out(w, out, case.oracle_decode(idx, k_pool=bk, v_pool=bv))
    fast = case.router.fast_scores(x["qr"]).cpu().numpy()
    assert np.max(np.abs(fast - ods)) <= ROUTE_EPS / 10
    assert_status_clean()


def test_1m_route_decode_T64():
    w = MEM_1M.replace(per_token=False)
    case = Case(w)
    idx, ods = check_route(case)
    assert set(case.x["needle_docs"].tolist()) == set(idx[0].tolist())
    out = case.decode(case.router.idx)
    ref = case.oracle_decode(idx)
    check_out(w, out, ref)
    assert_status_clean()


# ------------------------------------------------------------------ full-size memories

def test_16m_route_decode():
    case = Case(MEM_16M)
    idx, ods = check_route(case)
    out = case.decode(case.router.idx)
    check_out(MEM_16M, out, case.oracle_decode(idx))
    fast = case.router.fast_scores(case.x["qr"]).cpu().numpy()
    assert np.max(np.abs(fast - ods)) <= ROUTE_EPS / 10
    assert_status_clean()


def test_100m_hosttier_route_fetch_decode():
    case = Case(MEM_100M)
    assert case.bank.host_tier
    idx, _ = check_route(case)
    out = case.decode(case.router.idx)
    check_out(MEM_100M, out, case.oracle_decode(idx))
    assert_status_clean()


def test_16m_batch32_all_queries():
    """All 32 queries of the batch: indices and certified scores, decode and
    fast-score error against the oracle, and every query finds its needle."""
    w = MEM_16M_B32
    case = Case(w)
    idx, ods = check_route(case)
    for j, (b, _) in enumerate(case.x["needle_targets"]):
        assert int(case.x["needle_docs"][j]) in idx[b].tolist()
    out = case.decode(case.router.idx)
    check_out(w, out, case.oracle_decode(idx))
    fast = case.router.fast_scores(case.x["qr"]).cpu().numpy()
    assert np.max(np.abs(fast - ods)) <= ROUTE_EPS / 10
    assert_status_clean()


# ------------------------------------------------------------------ global RoPE of local keys

@pytest.mark.parametrize("w", [TINY_F32, MID.replace(name="mid-rope-B2-T3", B=2, T=3, n_needles=2)],
                         ids=lambda w: w.name)
def test_rope_local_matches_oracle_rotation(w):
    """Every local key of the cache equals the oracle's RoPE at top_k + j, one
    rounding to the dtype; rotating only the T new tokens leaves the older
    rows alone and writes the same bytes as the full rotation."""
    case = Case(w)
    x, d, H = case.x, w.head_dim, w.n_kv_heads
    raw = x["local_k"].float().cpu().numpy().astype(np.float64).reshape(-1, d)
    got = x["local_k_rot"].float().cpu().numpy().astype(np.float64).reshape(-1, d)
    loff = x["local_off"]
    for b in range(w.B):
        lt = int(loff[b + 1] - loff[b])
        for g in range(H):
            for j in range(lt):
                row = int(loff[b]) * H + g * lt + j
                ref = oracle.rope(raw[row], w.top_k + j, w.rope_theta)
                mag = np.abs(raw[row][: d // 2]) + np.abs(raw[row][d // 2:])
                mag = np.concatenate([mag, mag])
                rel = 0.0 if w.dtype == "f32" else 2.0 ** -8
                assert np.all(np.abs(got[row] - ref) <= rel * np.abs(ref) + 2e-6 * mag + 1e-30), (b, g, j)
    part = x["local_k"].clone()
    case.decoder.rotate_local(x["local_k"], part, new_tokens=w.T)
    torch.cuda.synchronize()
    for b in range(w.B):
        lt = int(loff[b + 1] - loff[b])
        a0 = int(loff[b]) * H * d
        p = part[a0:a0 + H * lt * d].view(H, lt, d)
        assert torch.equal(p[:, : lt - w.T], x["local_k"][a0:a0 + H * lt * d].view(H, lt, d)[:, : lt - w.T])
        assert torch.equal(p[:, lt - w.T:], x["local_k_rot"][a0:a0 + H * lt * d].view(H, lt, d)[:, lt - w.T:])
    assert_status_clean()


# ------------------------------------------------------------------ router-key norm table

def test_kr_inv_norms_match_fp64_and_both_scan_modes_agree():
    """The bank's inverse-norm table is 1/max(|Kr|, 1e-12) to fp32 accuracy with
    zero padding; routing with it and without it (norms inside the scan)
    returns the same certified indices and scores."""
    w = MID.replace(name="mid-T6-B2-norms", T=6, B=2, n_needles=2, local_len=(100, 900))
    with_tab = Case(w)
    kr = with_tab.bank.kr.float().cpu().numpy().astype(np.float64)     # [C][H][dr]
    C, H = kr.shape[0], kr.shape[1]
    ref = 1.0 / np.maximum(np.sqrt((kr * kr).sum(-1)), 1e-12)          # [C][H]
    tab = with_tab.bank.kr_inv_norm.cpu().numpy().reshape(H, -1)
    P = tab.shape[1]
    assert P % 128 == 0 and P >= C
    assert np.all(np.abs(tab[:, :C] - ref.T) <= 2e-6 * ref.T)
    assert np.all(tab[:, C:] == 0.0)
    idx_a, sc_a = check_route(with_tab)
    without = Case(w, inv_norms=False)
    assert without.bank.kr_inv_norm is None
    idx_b, sc_b = check_route(without)
    assert np.array_equal(idx_a, idx_b) and np.array_equal(sc_a, sc_b)
    assert_status_clean()


# ------------------------------------------------------------------ the largest batches

def test_decode_batch_limit_256_queries():
    """256 queries (the decode's limit): routing in two 128-row tensor-core
    passes, decode of every query against the oracle."""
    w = MID.replace(name="mid-B256", n_docs=400, len_clip=(1, 600), B=256, T=1, top_k=8,
                    n_needles=16, local_len=(1, 48))
    case = Case(w)
    idx, _ = check_route(case)
    out = case.decode(case.router.idx)
    check_out(w, out, case.oracle_decode(idx))
    assert_status_clean()


def test_route_batch_limit_512_queries():
    """512 queries (the routing limit): four tensor-core passes; indices and
    certified scores against the oracle on every query."""
    w = MID.replace(name="mid-B512-route", n_docs=300, len_clip=(1, 400), B=512, T=1, top_k=4,
                    n_needles=8, local_len=(1, 4))
    case = Case(w, decode=False)
    check_route(case)
    assert_status_clean()
