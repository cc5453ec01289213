"""Pins of the fp64 autograd training oracle (oracle/train.py).

* Its forward (attention output and router scores) equals the C oracle's
  decode and routing, which were written independently (and are pinned in
  test_oracle_pins.py), to rounding.
* Its gradients equal central finite differences of the forward.
* The auxiliary loss has a closed form on two documents.
* The log-sum-exp reproduces the output from the logits by a second route.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import train

pytestmark = pytest.mark.usefixtures("oracle_lib")
F64 = torch.float64


def _bank(seed, D=12, Hkv=2, d=16, dr=8, max_chunks=3):
    g = torch.Generator().manual_seed(seed)
    n = torch.randint(1, max_chunks + 1, (D,), generator=g)
    off = torch.cat([torch.zeros(1, dtype=torch.int64), torch.cumsum(n, 0)])
    C = int(off[-1])
    k = torch.randn(C, Hkv, d, generator=g, dtype=F64)
    v = torch.randn(C, Hkv, d, generator=g, dtype=F64)
    kr = torch.randn(C, Hkv, dr, generator=g, dtype=F64)
    return g, off, k, v, kr


def _local(g, B, Hkv, d, T, prefix):
    ks = [torch.randn(Hkv, prefix[b] + T, d, generator=g, dtype=F64) for b in range(B)]
    vs = [torch.randn(Hkv, prefix[b] + T, d, generator=g, dtype=F64) for b in range(B)]
    return ks, vs


def _flat(ts):
    lens = [t.shape[1] for t in ts]
    return np.concatenate([[0], np.cumsum(lens)]), torch.cat([t.reshape(-1) for t in ts])


@pytest.mark.parametrize("Hq,Hkv,T", [(2, 2, 1), (4, 2, 3), (8, 2, 5)])
def test_attention_forward_equals_c_oracle_decode(Hq, Hkv, T):
    g, off, k, v, kr = _bank(Hq * 10 + T, Hkv=Hkv)
    B, d, top_k, theta = 2, 16, 3, 1e4
    q = torch.randn(B, T, Hq, d, generator=g, dtype=F64)
    sel = torch.tensor([[4, 0, 9], [2, 11, 5]])
    lk, lv = _local(g, B, Hkv, d, T, [3, 7])
    # the C oracle reads f32 / bf16 storage: both sides get the same f32 values
    k, v = k.float().double(), v.float().double()
    lk = [t.float().double() for t in lk]
    lv = [t.float().double() for t in lv]
    out, lse = train.attention(q, sel, off, k, v, lk, lv, top_k, theta, Hkv)
    loff, lkf = _flat(lk)
    _, lvf = _flat(lv)
    ref = oracle.decode(q, sel.numpy().astype(np.int32), off.numpy(), k.float(), v.float(), loff,
                        lkf.float(), lvf.float(), top_k, theta, Hkv)
    assert np.max(np.abs(out.numpy() - ref)) < 1e-12
    assert out.shape == (B, T, Hq, d) and lse.shape == (B, T, Hq)


def test_lse_reproduces_the_output():
    g, off, k, v, kr = _bank(3)
    B, T, Hq, Hkv, d, top_k, theta = 1, 2, 2, 2, 16, 2, 1e4
    q = torch.randn(B, T, Hq, d, generator=g, dtype=F64)
    sel = torch.tensor([[1, 7]])
    lk, lv = _local(g, B, Hkv, d, T, [4])
    out, lse = train.attention(q, sel, off, k, v, lk, lv, top_k, theta, Hkv)
    # sum over keys of exp(logit - lse) * v, keys gathered by hand
    rows = list(range(int(off[1]), int(off[2]))) + list(range(int(off[7]), int(off[8])))
    for t in range(T):
        for h in range(Hq):
            qrot = torch.tensor(oracle.rope(q[0, t, h].numpy(), top_k + 4 + t, theta))
            acc = torch.zeros(d, dtype=F64)
            total = 0.0
            keys = [(k[r, h], v[r, h]) for r in rows]
            keys += [(torch.tensor(oracle.rope(lk[0][h, j].numpy(), top_k + j, theta)), lv[0][h, j])
                     for j in range(4 + t + 1)]
            for kk, vv in keys:
                w = math.exp(float(qrot @ kk) / math.sqrt(d) - float(lse[0, t, h]))
                acc += w * vv
                total += w
            assert abs(total - 1.0) < 1e-12
            assert torch.max(torch.abs(acc - out[0, t, h])) < 1e-12


@pytest.mark.parametrize("Hq,Hkv,T", [(4, 2, 1), (8, 2, 3)])
def test_doc_scores_and_selection_equal_c_oracle_route(Hq, Hkv, T):
    g, off, k, v, kr = _bank(40 + T, D=30, Hkv=Hkv)
    kr32 = kr.float()
    qr = torch.randn(2, T, Hq, 8, generator=g, dtype=F64)
    s = train.doc_scores(qr, kr32.double(), off, Hkv)
    idx, _, ds = oracle.route(qr, off.numpy(), kr32, 6, Hkv, want_scores=True)
    assert np.max(np.abs(s.numpy() - ds)) < 1e-13
    assert np.array_equal(train.select(s, 6).numpy(), idx)


def test_route_loss_closed_form_two_documents():
    s = torch.tensor([[0.3, 0.7]], dtype=F64)
    tau = 0.1
    got = train.route_loss(s, [[0]], tau)
    assert float(got[0]) == pytest.approx(math.log1p(math.exp((0.7 - 0.3) / tau)), rel=1e-14)
    both = train.route_loss(s, [[0, 1]], tau)
    assert float(both[0]) == pytest.approx(0.0, abs=1e-15)


def _central(f, x, idx, h=1e-6):
    """Central difference of the scalar f() in coordinate idx of tensor x."""
    with torch.no_grad():
        old = x[idx].item()
        x[idx] = old + h
        fp = f().item()
        x[idx] = old - h
        fm = f().item()
        x[idx] = old
    return (fp - fm) / (2 * h)


def test_gradients_equal_finite_differences():
    g, off, k, v, kr = _bank(77, D=10, Hkv=2, d=8, dr=8)
    B, T, Hq, Hkv, d, top_k, theta, tau = 2, 3, 4, 2, 8, 3, 1e4, 0.2
    q = torch.randn(B, T, Hq, d, generator=g, dtype=F64)
    qr = torch.randn(B, T, Hq, 8, generator=g, dtype=F64)
    lk, lv = _local(g, B, Hkv, d, T, [2, 5])
    dO = torch.randn(B, T, Hq, d, generator=g, dtype=F64)
    dL = torch.tensor([0.7, -1.3], dtype=F64)
    pos = [[1, 4], [7]]
    leaves = [q, qr, k, v, kr] + lk + lv
    for t in leaves:
        t.requires_grad_(True)
    sel = train.select(train.doc_scores(qr, kr, off, Hkv), top_k)

    def f():
        out, _ = train.attention(q, sel, off, k, v, lk, lv, top_k, theta, Hkv)
        loss = train.route_loss(train.doc_scores(qr, kr, off, Hkv), pos, tau)
        return (out * dO).sum() + (loss * dL).sum()

    f().backward()
    rng = np.random.default_rng(0)
    rows = torch.cat([torch.arange(int(off[s]), int(off[s + 1])) for s in sel.reshape(-1).tolist()])
    checked = 0
    for name, t in (("q", q), ("qr", qr), ("k", k), ("v", v), ("kr", kr), ("lk0", lk[0]), ("lk1", lk[1]),
                    ("lv0", lv[0]), ("lv1", lv[1])):
        for _ in range(6):
            if name in ("k", "v"):                       # rows the attention reads
                idx = (int(rows[rng.integers(len(rows))]), int(rng.integers(Hkv)), int(rng.integers(d)))
            else:
                idx = tuple(int(rng.integers(n)) for n in t.shape)
            fd = _central(f, t.data, idx)
            ad = float(t.grad[idx])
            assert abs(fd - ad) <= 1e-6 * (1 + abs(ad)), (name, idx, fd, ad)
            checked += abs(ad) > 1e-8
    assert checked > 30                                   # most checked coordinates carry gradient
    # documents no query selected and chunks no score maximised receive nothing
    unsel = sorted(set(range(len(off) - 1)) - set(sel.reshape(-1).tolist()))
    for s in unsel:
        assert torch.all(k.grad[int(off[s]):int(off[s + 1])] == 0)
