"""Pins of the fp64 CPU oracle against things other than itself.

Each check ties one part of the oracle to a closed form, an invariant, a
brute-force formulation written differently, a library routine on a special
case, or a hand-worked example (tests/golden/hand_examples.json).  The method
is stated in words on the pages:
  [A] "EverMind-AI/MSA: Memory Sparse Attention for 100M-Token Contexts",
      section "How MSA compresses and routes documents";
  [B] "EverMind Releases Memory-Sparse Attention Code for Long-Context AI
      Models", section "Architectural Design and Inference".
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import TINY_F32, gen

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")))
pytestmark = pytest.mark.usefixtures("oracle_lib")


def f32(a):
    return torch.tensor(np.asarray(a, dtype=np.float64), dtype=torch.float32)


def rope_complex(x, pos, theta):
    """Rotary embedding in its complex form: pair i is the complex number
    x[i] + 1j*x[i+d/2], multiplied by exp(1j * pos * theta^(-2i/d))."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    z = x[..., :h] + 1j * x[..., h:]
    freq = theta ** (-np.arange(h) * 2.0 / d)
    pos = np.asarray(pos, dtype=np.float64)[..., None]
    z = z * np.exp(1j * pos * freq)
    return np.concatenate([z.real, z.imag], axis=-1)


# ----------------------------------------------------------------- RoPE

def test_rope_identity_at_position_zero():
    x = np.random.default_rng(0).standard_normal(128)
    assert np.array_equal(oracle.rope(x, 0.0, 1e6), x)


@pytest.mark.parametrize("d", [2, 8, 64, 128])
@pytest.mark.parametrize("theta", [1e4, 1e6])
def test_rope_matches_complex_rotation(d, theta):
    rng = np.random.default_rng(d)
    for pos in [1, 3, 64, 255, 4099, 8300]:
        x = rng.standard_normal(d)
        y = oracle.rope(x, pos, theta)
        # the angle pos*freq carries ~ulp(pos) of rounding on either side
        assert np.allclose(y, rope_complex(x, pos, theta), rtol=0, atol=1e-14 * pos)


def test_rope_frequency_exponent_closed_form():
    # d = 4, theta = 1e6: pair 1 turns at 1e6^(-1/2) = 1e-3 rad per position,
    # so position 1000 turns e_1 by exactly one radian.
    y = oracle.rope(np.array([0.0, 1.0, 0.0, 0.0]), 1000, 1e6)
    assert y == pytest.approx([0.0, math.cos(1.0), 0.0, math.sin(1.0)], abs=1e-13)
    # pair 0 always turns at one radian per position
    y = oracle.rope(np.array([1.0, 0.0, 0.0, 0.0]), 2, 1e6)
    assert y == pytest.approx([math.cos(2.0), 0.0, math.sin(2.0), 0.0], abs=1e-15)


def test_rope_preserves_pair_norms_and_is_relative():
    rng = np.random.default_rng(7)
    d = 64
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    for m, n in [(5, 2), (300, 17), (4100, 4099)]:
        qm, kn = oracle.rope(q, m, 1e6), oracle.rope(k, n, 1e6)
        h = d // 2
        assert np.allclose(qm[:h] ** 2 + qm[h:] ** 2, q[:h] ** 2 + q[h:] ** 2, atol=1e-12)
        assert np.dot(qm, kn) == pytest.approx(np.dot(oracle.rope(q, m - n, 1e6), k), abs=1e-10)
        assert np.allclose(oracle.rope(oracle.rope(q, m, 1e6), n, 1e6),
                           oracle.rope(q, m + n, 1e6), atol=1e-10)


# ----------------------------------------------------------------- pooling CSR

def test_chunk_offsets_ceil_division():
    L = np.array([1, 64, 65, 128, 129, 4096, 32])
    off = np.concatenate([[0], np.cumsum(L)])
    got = oracle.chunk_offsets(off, 64)
    assert got.tolist() == [0, 1, 2, 4, 6, 9, 73, 74]
    with pytest.raises(ValueError):
        oracle.chunk_offsets(np.array([0, 5, 5, 9]), 64)   # empty document


# ----------------------------------------------------------------- encode

def _enc(doc_len, k, v, kr, chunk, theta=1e6):
    off = np.concatenate([[0], np.cumsum(doc_len)]).astype(np.int64)
    return oracle.encode(off, f32(k), f32(v), f32(kr), chunk, theta)


def test_encode_hand_example():
    g = GOLD["encode"]
    n = len(g["k_tok"])
    shp = lambda a: np.asarray(a, dtype=np.float64).reshape(n, 1, -1)
    kp, vp, krp = _enc(g["doc_len"], shp(g["k_tok"]), shp(g["v_tok"]), shp(g["kr_tok"]),
                       g["chunk"], g["theta"])
    off = np.concatenate([[0], np.cumsum(g["doc_len"])])
    assert oracle.chunk_offsets(off, g["chunk"]).tolist() == g["expect_chunk_off"]
    assert np.allclose(kp[:, 0], g["expect_k_pool"], rtol=0, atol=1e-15)
    assert np.array_equal(vp[:, 0], np.asarray(g["expect_v_pool"], dtype=np.float64))
    assert np.array_equal(krp[:, 0], np.asarray(g["expect_kr_pool"], dtype=np.float64))


def test_encode_constant_chunk_pools_to_the_constant():
    rng = np.random.default_rng(1)
    H, d = 2, 8
    c = rng.standard_normal((1, H, d)).astype(np.float32)
    toks = np.repeat(c, 100, axis=0)                       # one doc of 100 tokens
    _, vp, krp = _enc([100], toks, toks, toks, 64)
    want = np.broadcast_to(c.astype(np.float64), (2, H, d))
    assert np.array_equal(vp, want) and np.array_equal(krp, want)


def test_encode_matches_brute_force_complex_form():
    rng = np.random.default_rng(2)
    H, d, dr, chunk, theta = 3, 16, 12, 8, 1e4
    L = np.array([1, 7, 8, 9, 23, 64])
    n = int(L.sum())
    k = rng.standard_normal((n, H, d)).astype(np.float32)
    v = rng.standard_normal((n, H, d)).astype(np.float32)
    kr = rng.standard_normal((n, H, dr)).astype(np.float32)
    kp, vp, krp = _enc(L, k, v, kr, chunk, theta)
    rows_k, rows_v, rows_r = [], [], []
    t0 = 0
    for Ld in L:
        pos = np.arange(Ld)
        krot = rope_complex(np.transpose(k[t0:t0 + Ld].astype(np.float64), (1, 0, 2)), pos, theta)
        krot = np.transpose(krot, (1, 0, 2))
        for s in range(0, Ld, chunk):
            e = min(s + chunk, Ld)
            rows_k.append(krot[s:e].mean(axis=0))
            rows_v.append(v[t0 + s:t0 + e].astype(np.float64).mean(axis=0))
            rows_r.append(kr[t0 + s:t0 + e].astype(np.float64).mean(axis=0))
        t0 += Ld
    assert np.allclose(kp, np.stack(rows_k), atol=1e-12)
    assert np.allclose(vp, np.stack(rows_v), atol=1e-12)
    assert np.allclose(krp, np.stack(rows_r), atol=1e-12)


def test_encode_positions_restart_per_document():
    # swapping two documents swaps their pooled chunks exactly
    rng = np.random.default_rng(3)
    H, d = 2, 8
    a = rng.standard_normal((70, H, d)).astype(np.float32)
    b = rng.standard_normal((30, H, d)).astype(np.float32)
    kp1, _, _ = _enc([70, 30], np.concatenate([a, b]), np.concatenate([a, b]),
                     np.concatenate([a, b]), 64)
    kp2, _, _ = _enc([30, 70], np.concatenate([b, a]), np.concatenate([b, a]),
                     np.concatenate([b, a]), 64)
    assert np.array_equal(kp1[:2], kp2[1:]) and np.array_equal(kp1[2], kp2[0])


def test_encode_chunk_locality():
    rng = np.random.default_rng(4)
    H, d = 1, 4
    x = rng.standard_normal((200, H, d)).astype(np.float32)
    kp1, vp1, _ = _enc([200], x, x, x, 64)
    y = x.copy()
    y[130] += 1.0                                          # token of chunk 2
    kp2, vp2, _ = _enc([200], y, y, y, 64)
    changed = np.where(np.any(kp1 != kp2, axis=(1, 2)))[0].tolist()
    assert changed == [2]
    assert np.where(np.any(vp1 != vp2, axis=(1, 2)))[0].tolist() == [2]


# ----------------------------------------------------------------- route

def _route(qr, kr_pool, chunk_off, top_k, Hkv, scores=True):
    return oracle.route(np.asarray(qr, dtype=np.float64), np.asarray(chunk_off), f32(kr_pool),
                        top_k, Hkv, want_scores=scores)


def test_route_hand_example():
    g = GOLD["route"]
    qr = np.asarray(g["qr"], dtype=np.float64)[None]           # B=1, T=2, H=1, dr=2
    kr = np.asarray(g["kr_pool"], dtype=np.float64)[:, None]
    idx, sc, _ = _route(qr, kr, g["chunk_off"], g["top_k"], g["n_kv_heads"])
    assert idx[0].tolist() == g["expect_idx"]
    assert sc[0] == pytest.approx(g["expect_score"], abs=3e-16)   # one ulp of rounding


def _law_of_cosines_scores(qr, kr, chunk_off, Hkv):
    """Document scores with each cosine computed from the law of cosines,
    cos = (|q|^2 + |k|^2 - |q - k|^2) / (2 |q| |k|)."""
    B, T, Hq, dr = qr.shape
    G = Hq // Hkv
    kk = kr[:, np.arange(Hq) // G]                               # [C][Hq][dr]
    out = np.empty((B, len(chunk_off) - 1))
    for b in range(B):
        q = qr[b][:, None]                                       # [T][1][Hq][dr]
        nq = (q ** 2).sum(-1)
        nk = (kk[None] ** 2).sum(-1)
        diff = ((q - kk[None]) ** 2).sum(-1)
        cs = (nq + nk - diff) / (2 * np.sqrt(nq) * np.sqrt(nk))  # [T][C][Hq]
        per = cs.mean(-1).max(0)                                 # [C]
        for s in range(len(chunk_off) - 1):
            out[b, s] = per[chunk_off[s]:chunk_off[s + 1]].max()
    return out


@pytest.mark.parametrize("Hq,Hkv,T", [(1, 1, 1), (4, 4, 4), (8, 2, 3), (32, 8, 2)])
def test_route_scores_match_law_of_cosines(Hq, Hkv, T):
    rng = np.random.default_rng(Hq * 10 + T)
    dr, D = 16, 40
    L = rng.integers(1, 5, size=D)
    off = np.concatenate([[0], np.cumsum(L)])
    C = int(off[-1])
    qr = rng.standard_normal((2, T, Hq, dr))
    kr = rng.standard_normal((C, Hkv, dr)).astype(np.float32).astype(np.float64)
    idx, sc, ds = _route(qr, kr, off, 5, Hkv)
    ref = _law_of_cosines_scores(qr, kr, off, Hkv)
    assert np.allclose(ds, ref, atol=1e-12)
    assert np.all(ds >= -1.0) and np.all(ds <= 1.0)
    for b in range(2):                                          # Top-k = full sort
        order = sorted(range(D), key=lambda s: (-ds[b, s], s))[:5]
        assert idx[b].tolist() == order


def test_route_special_case_is_cosine_nearest_neighbours():
    from sklearn.neighbors import NearestNeighbors
    rng = np.random.default_rng(11)
    D, dr = 300, 24
    kr = rng.standard_normal((D, 1, dr)).astype(np.float32).astype(np.float64)
    q = rng.standard_normal((1, 1, 1, dr))
    idx, _, _ = _route(q, kr, np.arange(D + 1), 10, 1)
    nn = NearestNeighbors(n_neighbors=10, metric="cosine", algorithm="brute").fit(kr[:, 0])
    _, want = nn.kneighbors(q[0, 0])
    assert idx[0].tolist() == want[0].tolist()


def test_route_head_mapping_and_mean():
    # H_q = 4, H_kv = 2: heads 0,1 read kv head 0; heads 2,3 read kv head 1.
    e = np.eye(4)
    qr = np.stack([e[0], e[0], e[1], e[1]])[None, None]          # [1][1][4][4]
    good = np.stack([e[0], e[1]])                                # matches h // 2
    swapped = np.stack([e[1], e[0]])
    half = np.stack([e[0], e[2]])                                # heads 0,1 -> 1; heads 2,3 -> 0
    kr = np.stack([good, swapped, half])
    _, _, ds = _route(qr, kr, [0, 1, 2, 3], 1, 2)
    assert ds[0].tolist() == [1.0, 0.0, 0.5]


def test_route_max_over_chunks_and_tokens_and_clamp():
    qr = np.array([[[[1.0, 0.0]], [[0.0, 1.0]]]])                # T = 2
    a = [math.cos(1.2), math.sin(1.2)]
    kr = np.array([[[1.0, 0.0]], [a], [[-1.0, 0.0]], [[0.0, 0.0]]])
    _, _, ds = _route(qr, kr, [0, 3, 4], 1, 1)
    assert ds[0, 0] == 1.0
    assert ds[0, 1] == 0.0                                       # zero key scores 0, not NaN
    # x vs alpha*x and vs -x
    x = np.random.default_rng(5).standard_normal(64)
    kr2 = np.stack([3.5 * x, -x])[:, None].astype(np.float32).astype(np.float64)
    _, _, ds2 = _route(kr2[:1, 0][None, None], kr2, [0, 1, 2], 1, 1)
    assert ds2[0, 0] == pytest.approx(1.0, abs=1e-15) and ds2[0, 0] <= 1.0
    assert ds2[0, 1] == pytest.approx(-1.0, abs=1e-15) and ds2[0, 1] >= -1.0


def test_route_ties_lower_index_first_and_permutation_invariance():
    rng = np.random.default_rng(6)
    D, dr = 50, 8
    kr = rng.standard_normal((D, 1, dr))
    kr[17] = kr[3]
    kr[40] = kr[3]                                               # exact triple tie
    q = kr[3:4, 0][None, None] * 1.0
    idx, sc, _ = _route(q, kr.astype(np.float32).astype(np.float64), np.arange(D + 1), 3, 1)
    assert idx[0].tolist() == [3, 17, 40]
    perm = rng.permutation(D)
    kr2 = rng.standard_normal((D, 2, dr)).astype(np.float32).astype(np.float64)
    q2 = rng.standard_normal((1, 2, 4, dr))
    i1, s1, _ = _route(q2, kr2, np.arange(D + 1), 6, 2)
    i2, s2, _ = _route(q2, kr2[perm], np.arange(D + 1), 6, 2)
    assert sorted(perm[i2[0]].tolist()) == sorted(i1[0].tolist())
    assert np.array_equal(np.sort(s1), np.sort(s2))


def test_route_tiny_workload_selects_needle_and_k_equals_D():
    w = TINY_F32
    x = gen.generate(w)
    kp, vp, krp = oracle.encode(x["doc_tok_off"], x["k_tok"], x["v_tok"], x["kr_tok"],
                                w.chunk, w.rope_theta)
    coff = oracle.chunk_offsets(x["doc_tok_off"], w.chunk)
    idx, sc, ds = oracle.route(x["qr"], coff, torch.from_numpy(krp).float(), w.top_k,
                               w.n_kv_heads, want_scores=True)
    assert int(x["needle_docs"][0]) in idx[0].tolist()
    others = np.delete(ds[0], x["needle_docs"])
    assert ds[0, x["needle_docs"][0]] - others.max() >= 0.3
    idx_all, _ = oracle.route(x["qr"], coff, torch.from_numpy(krp).float(), w.n_docs, w.n_kv_heads)
    assert sorted(idx_all[0].tolist()) == list(range(w.n_docs))


# ----------------------------------------------------------------- decode

def _dec_golden(g):
    d = g["d"]
    T, Lb = g["T"], g["L_b"]
    q = np.asarray(g["q"], dtype=np.float64).reshape(1, T, 1, d)
    lk = f32(g["local_k"]).reshape(-1)
    lv = f32(g["local_v"]).reshape(-1)
    return oracle.decode(q, np.asarray([g["sel"]], dtype=np.int32), np.asarray(g["chunk_off"]),
                         f32(g["k_pool"]).reshape(-1, 1, d), f32(g["v_pool"]).reshape(-1, 1, d),
                         np.array([0, Lb + T]), lk, lv, g["top_k"], g["theta"], 1)


def test_decode_hand_example_global_offset():
    g = GOLD["decode_aligned"]
    out = _dec_golden(g)
    assert out.reshape(-1) == pytest.approx(g["expect_out"], abs=2e-6)


def test_decode_hand_example_causal():
    g = GOLD["decode_causal"]
    out = _dec_golden(g)
    assert np.allclose(out.reshape(2, 2), np.asarray(g["expect_out"]), atol=1e-13)


def _sdpa_reference(q, sel, coff, kp, vp, loff, lk, lv, top_k, theta, Hkv):
    """Dense attention via torch's scaled_dot_product_attention in fp64 with an
    explicit mask; keys are rotated with the complex-form RoPE above."""
    B, T, Hq, d = q.shape
    G = Hq // Hkv
    outs = []
    for b in range(B):
        Ltot = int(loff[b + 1] - loff[b])
        Lb = Ltot - T
        rows = np.concatenate([np.arange(coff[s], coff[s + 1]) for s in sel[b]])
        mk, mv = kp[rows], vp[rows]                                   # [nm][Hkv][d]
        base = int(loff[b]) * Hkv * d
        LK = lk[base:base + Hkv * Ltot * d].reshape(Hkv, Ltot, d)
        LV = lv[base:base + Hkv * Ltot * d].reshape(Hkv, Ltot, d)
        LKr = rope_complex(LK, top_k + np.arange(Ltot)[None, :], theta)
        K = np.concatenate([np.transpose(mk, (1, 0, 2)), LKr], axis=1)   # [Hkv][N][d]
        V = np.concatenate([np.transpose(mv, (1, 0, 2)), LV], axis=1)
        qq = rope_complex(np.transpose(q[b], (1, 0, 2)), (top_k + Lb + np.arange(T))[None, :], theta)
        nm = len(rows)
        mask = np.ones((T, nm + Ltot), dtype=bool)
        for t in range(T):
            mask[t, nm + Lb + t + 1:] = False
        Kt = torch.from_numpy(K).repeat_interleave(G, dim=0)
        Vt = torch.from_numpy(V).repeat_interleave(G, dim=0)
        o = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qq), Kt, Vt, attn_mask=torch.from_numpy(mask))
        outs.append(np.transpose(o.numpy(), (1, 0, 2)))
    return np.stack(outs)


@pytest.mark.parametrize("Hq,Hkv,T", [(4, 4, 4), (8, 2, 1), (8, 2, 3)])
def test_decode_k_equals_D_matches_dense_sdpa(Hq, Hkv, T):
    rng = np.random.default_rng(Hq + T)
    d, D, B, theta = 16, 7, 2, 1e4
    L = rng.integers(1, 4, size=D)
    coff = np.concatenate([[0], np.cumsum(L)])
    C = int(coff[-1])
    kp = rng.standard_normal((C, Hkv, d)).astype(np.float32)
    vp = rng.standard_normal((C, Hkv, d)).astype(np.float32)
    Lb = rng.integers(3, 12, size=B)
    loff = np.concatenate([[0], np.cumsum(Lb + T)])
    n = int(loff[-1]) * Hkv * d
    lk = rng.standard_normal(n).astype(np.float32)
    lv = rng.standard_normal(n).astype(np.float32)
    q = rng.standard_normal((B, T, Hq, d)).astype(np.float32).astype(np.float64)
    sel = np.stack([rng.permutation(D) for _ in range(B)]).astype(np.int32)   # k = D
    out = oracle.decode(q, sel, coff, torch.from_numpy(kp), torch.from_numpy(vp), loff,
                        torch.from_numpy(lk), torch.from_numpy(lv), D, theta, Hkv)
    ref = _sdpa_reference(q, sel, coff, kp.astype(np.float64), vp.astype(np.float64), loff,
                          lk.astype(np.float64), lv.astype(np.float64), D, theta, Hkv)
    assert np.allclose(out, ref, atol=1e-12)


def test_decode_zero_query_is_mean_and_rank_order_invariance():
    w = TINY_F32
    x = gen.generate(w)
    kp, vp, krp = oracle.encode(x["doc_tok_off"], x["k_tok"], x["v_tok"], x["kr_tok"],
                                w.chunk, w.rope_theta)
    coff = oracle.chunk_offsets(x["doc_tok_off"], w.chunk)
    kpt, vpt = torch.from_numpy(kp).float(), torch.from_numpy(vp).float()
    sel = np.array([[5, 9, 1, 30]], dtype=np.int32)
    q0 = np.zeros((1, w.T, w.n_q_heads, w.head_dim))
    out = oracle.decode(q0, sel, coff, kpt, vpt, x["local_off"], x["local_k"], x["local_v"],
                        w.top_k, w.rope_theta, w.n_kv_heads)
    Lb = int(x["local_len"][0])
    lv = x["local_v"].double().numpy().reshape(w.n_kv_heads, Lb + w.T, w.head_dim)
    mem = np.concatenate([vpt.double().numpy()[coff[s]:coff[s + 1]] for s in sel[0]])
    for t in range(w.T):
        for h in range(w.n_q_heads):
            vals = np.concatenate([mem[:, h], lv[h, :Lb + t + 1]])
            assert np.allclose(out[0, t, h], vals.mean(0), atol=1e-13)
    q = x["q"].double().numpy()
    o1 = oracle.decode(q, sel, coff, kpt, vpt, x["local_off"], x["local_k"], x["local_v"],
                       w.top_k, w.rope_theta, w.n_kv_heads)
    o2 = oracle.decode(q, sel[:, ::-1].copy(), coff, kpt, vpt, x["local_off"], x["local_k"],
                       x["local_v"], w.top_k, w.rope_theta, w.n_kv_heads)
    assert np.allclose(o1, o2, atol=1e-13)


def test_decode_doc_interleaved_layout_equals_chunk_major():
    rng = np.random.default_rng(9)
    Hkv, d, D = 2, 8, 6
    L = np.array([1, 3, 2, 1, 4, 2])
    coff = np.concatenate([[0], np.cumsum(L)])
    C = int(coff[-1])
    kp = rng.standard_normal((C, Hkv, d)).astype(np.float32)
    vp = rng.standard_normal((C, Hkv, d)).astype(np.float32)
    inter = np.concatenate([np.concatenate([kp[coff[s]:coff[s + 1]], vp[coff[s]:coff[s + 1]]])
                            for s in range(D)])
    q = rng.standard_normal((1, 2, 4, d))
    loff = np.array([0, 7])
    lk = rng.standard_normal(7 * Hkv * d).astype(np.float32)
    lv = rng.standard_normal(7 * Hkv * d).astype(np.float32)
    sel = np.array([[4, 1, 5]], dtype=np.int32)
    a = oracle.decode(q, sel, coff, torch.from_numpy(kp), torch.from_numpy(vp), loff,
                      torch.from_numpy(lk), torch.from_numpy(lv), 3, 1e6, Hkv)
    b = oracle.decode(q, sel, coff, torch.from_numpy(inter), None, loff, torch.from_numpy(lk),
                      torch.from_numpy(lv), 3, 1e6, Hkv, kv_layout=oracle.KV_DOC_INTERLEAVED)
    assert np.array_equal(a, b)


def _bf16_values(g, *shape, scale=1.0):
    """Random bf16 values plus a few edge patterns: +-0, the largest finite
    bf16, the smallest normal and a subnormal, each with both signs."""
    x = (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16).view(-1)
    edge = torch.tensor([0.0, -0.0, 3.3895e38, -3.3895e38, 1.1755e-38, -1.1755e-38, 9.2e-41, -9.2e-41],
                        dtype=torch.float32).to(torch.bfloat16)
    x[:len(edge)] = edge
    return x.view(*shape)


def test_bf16_storage_reads_as_its_exact_fp32_widening():
    """Four of the five workloads store bf16.  The oracle decodes a stored
    bf16 element itself (its top 16 bits of an fp32); torch's bf16 -> fp32
    conversion is exact, so encode, route and decode on bf16 storage must give
    bit-identical doubles to the same values stored as fp32.  A wrong shift,
    byte order or view of the bf16 words changes the values and fails this."""
    g = torch.Generator().manual_seed(2024)
    H, d, dr = 2, 8, 8
    # encode: ragged documents with a partial last chunk
    doc_len = np.array([70, 3, 128, 65])
    tok = np.concatenate([[0], np.cumsum(doc_len)])
    n = int(tok[-1])
    k, v, kr = (_bf16_values(g, n, H, dd, scale=2.0) for dd in (d, d, dr))
    a = oracle.encode(tok, k, v, kr, 64, 1e6)
    b = oracle.encode(tok, k.float(), v.float(), kr.float(), 64, 1e6)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    assert not np.array_equal(a[1], oracle.encode(tok, k, (v.float() * 2).to(torch.bfloat16), kr, 64, 1e6)[1])

    # route: bf16 router keys, including zero and extreme vectors
    D, Hq, T = 9, 4, 3
    coff = np.array([0, 1, 3, 4, 6, 7, 8, 10, 11, 12])
    krp = _bf16_values(g, int(coff[-1]), H, dr)
    qr = torch.randn(2, T, Hq, dr, generator=g).to(torch.bfloat16)
    ia, sa, da = oracle.route(qr, coff, krp, 4, H, want_scores=True)
    ib, sb, db = oracle.route(qr, coff, krp.float(), 4, H, want_scores=True)
    assert np.array_equal(ia, ib) and np.array_equal(sa, sb) and np.array_equal(da, db)

    # decode: chunk-major pooled K/V and the host tier's per-document layout
    C = int(coff[-1])
    kp, vp = _bf16_values(g, C, H, d, scale=0.5), _bf16_values(g, C, H, d, scale=0.5)
    kp[0, 0, :3] = torch.tensor([1.5, -2.0, 0.75]).to(torch.bfloat16)
    vp.view(-1)[2:4] = 0.0                       # keep the extremes out of the softmax
    kp.view(-1)[2:4] = 0.0
    vp.view(-1)[:2] = torch.tensor([7.0, -3.0]).to(torch.bfloat16)
    loff = np.array([0, 5, 12])
    lk = torch.randn(12 * H * d, generator=g).to(torch.bfloat16)
    lv = torch.randn(12 * H * d, generator=g).to(torch.bfloat16)
    q = torch.randn(2, 2, Hq, d, generator=g).to(torch.bfloat16)
    sel = np.array([[4, 0, 7], [1, 8, 2]], dtype=np.int32)
    oa = oracle.decode(q, sel, coff, kp, vp, loff, lk, lv, 3, 1e6, H)
    ob = oracle.decode(q, sel, coff, kp.float(), vp.float(), loff, lk.float(), lv.float(), 3, 1e6, H)
    assert np.all(np.isfinite(oa)) and np.array_equal(oa, ob)
    inter = torch.cat([torch.cat([kp[coff[s]:coff[s + 1]], vp[coff[s]:coff[s + 1]]]) for s in range(D)])
    oc = oracle.decode(q, sel, coff, inter, None, loff, lk, lv, 3, 1e6, H, kv_layout=oracle.KV_DOC_INTERLEAVED)
    od = oracle.decode(q, sel, coff, inter.float(), None, loff, lk.float(), lv.float(), 3, 1e6, H,
                       kv_layout=oracle.KV_DOC_INTERLEAVED)
    assert np.array_equal(oc, od) and np.array_equal(oc, oa)


def test_oracle_rejects_bad_arguments():
    with pytest.raises(ValueError):
        oracle.rope(np.zeros(3), 1, 1e6)
    qr = np.zeros((1, 1, 4, 8))
    with pytest.raises(ValueError):       # top_k > D
        _route(qr, np.zeros((2, 4, 8)), [0, 1, 2], 3, 4)
    with pytest.raises(ValueError):       # H_q not a multiple of H_kv
        _route(qr, np.zeros((2, 3, 8)), [0, 1, 2], 1, 3)


def test_oracle_tiny_regression_fixture():
    """Oracle output on the tiny workload is unchanged since the fixture was written."""
    import importlib.util
    p = os.path.join(os.path.dirname(__file__), "golden", "make_tiny_regression.py")
    spec = importlib.util.spec_from_file_location("make_tiny_regression", p)
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    want = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "tiny_regression.json")))
    got = m.compute()
    for key, val in got.items():
        if isinstance(val, dict):
            for r, v in val.items():
                assert np.allclose(v, want[key][r], rtol=0, atol=1e-13), key
        elif isinstance(val, list):
            assert np.allclose(val, want[key], rtol=0, atol=1e-13), key
        else:
            assert val == want[key], key


# ----------------------------------------------------------------- Memory Interleave

def _interleave_brute(ds_row, selected, p):
    """The p best documents outside `selected`, by a pure-Python full sort."""
    order = sorted((s for s in range(len(ds_row)) if s not in set(selected)),
                   key=lambda s: (-ds_row[s], s))
    return list(selected) + order[:p]


def _interleave_case(seed, B=2, D=60, Hq=8, Hkv=2, dr=16):
    rng = np.random.default_rng(seed)
    L = rng.integers(1, 4, size=D)
    off = np.concatenate([[0], np.cumsum(L)])
    kr = rng.standard_normal((int(off[-1]), Hkv, dr)).astype(np.float32)
    return rng, off, torch.from_numpy(kr), (B, Hq, dr)


def test_interleave_first_round_is_route_top_p():
    rng, off, kr, (B, Hq, dr) = _interleave_case(21)
    qr = rng.standard_normal((B, 1, Hq, dr))
    got = oracle.interleave_expand(qr, off, kr, np.zeros((B, 0), np.int32), 5, 2)
    want, _ = oracle.route(qr, off, kr, 5, 2)
    assert np.array_equal(got, want)


def test_interleave_constant_query_chain_equals_route_top_rp():
    # with the same query every round, R rounds of p documents select exactly
    # the route's top R*p documents, in rank order
    rng, off, kr, (B, Hq, dr) = _interleave_case(22)
    qr = rng.standard_normal((B, 2, Hq, dr))
    sel = np.zeros((B, 0), np.int32)
    for _ in range(4):
        sel = oracle.interleave_expand(qr, off, kr, sel, 3, 2)
    want, _ = oracle.route(qr, off, kr, 12, 2)
    assert np.array_equal(sel, want)


def test_interleave_matches_brute_force_and_keeps_the_old_set():
    rng, off, kr, (B, Hq, dr) = _interleave_case(23)
    sel = np.zeros((B, 0), np.int32)
    for r in range(5):                                           # a new query every round
        qr = rng.standard_normal((B, 1, Hq, dr))
        _, _, ds = oracle.route(qr, off, kr, 1, 2, want_scores=True)
        new = oracle.interleave_expand(qr, off, kr, sel, 4, 2)
        for b in range(B):
            want = _interleave_brute(ds[b], sel[b].tolist(), 4)
            assert new[b].tolist() == want
            assert len(set(new[b].tolist())) == new.shape[1]     # no document twice
        sel = new
    assert sel.shape == (B, 20)


def test_interleave_ties_lower_index_first_and_rejects_bad_sets():
    D, dr = 12, 4
    kr = np.zeros((D, 1, dr), np.float32)
    kr[:, 0, 0] = 1.0                                            # every document ties
    off = np.arange(D + 1)
    qr = np.zeros((1, 1, 1, dr)); qr[..., 0] = 1.0
    sel = oracle.interleave_expand(qr, off, torch.from_numpy(kr), np.array([[5, 2]], np.int32), 3, 1)
    assert sel[0].tolist() == [5, 2, 0, 1, 3]
    with pytest.raises(ValueError):                              # a document twice in the old set
        oracle.interleave_expand(qr, off, torch.from_numpy(kr), np.array([[5, 5]], np.int32), 3, 1)
    with pytest.raises(ValueError):                              # more documents than the memory holds
        oracle.interleave_expand(qr, off, torch.from_numpy(kr), np.array([[5, 2]], np.int32), 11, 1)
