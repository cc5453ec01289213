"""GPU parity of the training-time routing layer (runtime.TrainLayer over
msa_sparse_attention_forward / _backward and msa_route_loss_forward /
_backward) against the fp64 autograd oracle (oracle/train.py).

Selected documents must equal the oracle's bit for bit; the output, the
log-sum-exp and the loss must match within the arithmetic's tolerance; every
gradient must match the oracle's autograd gradient within a tolerance
relative to that gradient's largest entry, and be exactly zero where the
oracle's is (chunks no query selected, chunks no score maximised, capacity
rows past the live length).

Tolerances.  bf16 banks: the forward is the tensor-core decode (the rotated
query and the softmax weights enter its products as bf16, so logits and lse
carry ~2^-8 relative error) and the output is stored as bf16; the backward
recomputes P = exp(S/sqrt(d) - lse) in fp32 and uses D = sum dO * O with the
bf16 output, so gradients carry a few parts in 1e3 of their scale: 2e-2 of
the largest entry.  fp32 banks: every step in fp32, 2e-4.  The routing loss
is fp32 throughout: loss within 1e-4 relative, gradients within 1e-3 of the
largest entry."""
import numpy as np
import pytest
import torch

from oracle import train
from routed_sparse_attention_b200 import Layout
from routed_sparse_attention_b200 import device_status
from routed_sparse_attention_b200.runtime import Bank, TrainLayer
from workloads import Workload, gen

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

F64 = torch.float64
BASE = Workload(name="train-layer", dtype="bf16", n_docs=120, doc_len=150, lognormal_sigma=0.6, len_clip=(1, 600),
                chunk=64, n_q_heads=32, n_kv_heads=8, head_dim=128, router_dim=128, T=8, B=3,
                local_len=(1, 1), top_k=6, n_needles=0, per_token=False, kv_on_host=False, seed=930, mem_seed=931)


def _rel(got, ref):
    scale = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(got - ref))) / max(scale, 1e-30), scale


# bf16 at head_dim 128 runs the tcgen05 backward (128-key tiles, blocks of 128
# query rows): T = 64 gives 256 rows per kv head, two row blocks, and local
# tiles whose first row block sees none of their keys (prefix 90: keys 128..)
# "extra" overrides the workload: 40 documents of median 600 tokens give the
# tcgen05 backward several 128-key memory tiles; 64 query heads give G = 8
@pytest.mark.parametrize("dtype,T,prefix,d,extra", [
    ("bf16", 8, [50, 130, 7], 128, {}), ("f32", 3, [20, 64, 1], 64, {}),
    ("bf16", 1, [200, 65, 0], 128, {}), ("bf16", 5, [70, 3, 129], 64, {}),
    ("bf16", 64, [90, 0, 190], 128, {}),
    ("bf16", 16, [300, 40, 170], 128, {"top_k": 40, "doc_len": 600, "len_clip": (64, 1200)}),
    ("bf16", 10, [30, 260, 5], 128, {"n_q_heads": 64})],
    ids=["bf16-T8", "f32-T3-d64", "bf16-T1", "bf16-T5-d64", "bf16-T64", "bf16-T16-mem4tiles", "bf16-T10-G8"])
def test_train_layer_forward_backward_match_fp64_autograd(dtype, T, prefix, d, extra):
    w = BASE.replace(dtype=dtype, T=T, **extra)
    if dtype == "f32":
        w = w.replace(head_dim=64, router_dim=64, n_q_heads=8, n_kv_heads=4)
    elif d == 64:                                    # tensor-core backward at head_dim 64, G = 4
        w = w.replace(head_dim=64, n_q_heads=16, n_kv_heads=4)
    B, Hq, Hkv, d, dr, k = w.B, w.n_q_heads, w.n_kv_heads, w.head_dim, w.router_dim, w.top_k
    x = gen.generate(w.replace(per_token=False), device="cuda")
    lay = Layout.of(w)
    bank = Bank(lay, x["doc_tok_off"], kr_pool=x["kr_pool"], k_pool=x["k_pool"], v_pool=x["v_pool"])
    dt = lay.torch_dtype
    g = torch.Generator().manual_seed(5 + T)
    live = [p + T for p in prefix]
    cap = [n + 3 for n in live]                         # spare capacity rows must stay untouched
    loff = np.concatenate([[0], np.cumsum(cap)])
    q = torch.randn(B, T, Hq, d, generator=g).to(dt)
    qr = torch.randn(B, T, Hq, dr, generator=g).to(dt)
    lk = [torch.randn(Hkv, live[b], d, generator=g).to(dt) for b in range(B)]
    lv = [torch.randn(Hkv, live[b], d, generator=g).to(dt) for b in range(B)]
    lk_cache = torch.zeros(int(loff[-1]) * Hkv * d, dtype=dt)
    lv_cache = torch.zeros_like(lk_cache)
    for b in range(B):
        base = int(loff[b]) * Hkv * d
        lk_cache[base:base + Hkv * cap[b] * d].view(Hkv, cap[b], d)[:, :live[b]] = lk[b]
        lv_cache[base:base + Hkv * cap[b] * d].view(Hkv, cap[b], d)[:, :live[b]] = lv[b]
    coff = bank.doc_chunk_off_host
    # relevant documents: each query's best document by the oracle, plus one or two others
    ref_scores = train.doc_scores(qr.double(), bank.kr.cpu().double(), coff, Hkv)
    pos = [[int(train.select(ref_scores[b:b + 1], 1)[0, 0])] + [(7 * b + 3 + j) % w.n_docs for j in range(b % 3)]
           for b in range(B)]
    pos = [sorted(set(p)) for p in pos]
    pos_off = torch.tensor(np.concatenate([[0], np.cumsum([len(p) for p in pos])]), dtype=torch.int32)
    pos_doc = torch.tensor([s for p in pos for s in p], dtype=torch.int32)
    dout = torch.randn(B, T, Hq, d, generator=g).to(dt)
    dloss = torch.tensor([0.8, -1.1, 0.5][:B], dtype=torch.float32)
    tau = 0.1

    layer = TrainLayer(bank, B, T, k, loff, local_len=torch.tensor(live), tau=tau)
    out, loss, sel = layer.forward(q.cuda(), qr.cuda(), lk_cache.cuda(), lv_cache.cuda(), pos_off.cuda(),
                                   pos_doc.cuda())
    grads = layer.backward(dout.cuda(), dloss.cuda())
    torch.cuda.synchronize()
    assert device_status() == 0

    # ---- oracle: fp64 autograd on the same stored values
    kp = bank.k.cpu().double().requires_grad_(True)
    vp = bank.v.cpu().double().requires_grad_(True)
    krp = bank.kr.cpu().double().requires_grad_(True)
    q64 = q.double().requires_grad_(True)
    qr64 = qr.double().requires_grad_(True)
    lk64 = [t.double().requires_grad_(True) for t in lk]
    lv64 = [t.double().requires_grad_(True) for t in lv]
    scores = train.doc_scores(qr64, krp, coff, Hkv)
    ref_sel = train.select(scores, k)
    assert np.array_equal(sel.cpu().numpy(), ref_sel.numpy())
    ref_out, ref_lse = train.attention(q64, ref_sel, coff, kp, vp, lk64, lv64, k, w.rope_theta, Hkv)
    ref_loss = train.route_loss(scores, pos, tau)
    ((ref_out * dout.double()).sum() + (ref_loss * dloss.double()).sum()).backward()

    attn_tol = 2e-2 if dtype == "bf16" else 2e-4
    err_out = float(torch.max(torch.abs(out.float().cpu().double() - ref_out.detach())))
    err_lse = float(torch.max(torch.abs(layer.lse.cpu().double() - ref_lse.detach())))
    print(f"[train {dtype} T={T}] out {err_out:.2e}, lse {err_lse:.2e}")
    assert err_out <= (2e-2 if dtype == "bf16" else 1e-5)
    assert err_lse <= (2e-2 if dtype == "bf16" else 1e-5)
    assert np.allclose(loss.cpu().numpy(), ref_loss.detach().numpy(), rtol=1e-4, atol=1e-5)

    def check(name, got, ref, tol):
        e, scale = _rel(got, ref)
        print(f"[train {dtype} T={T}] d{name}: max error {e:.2e} of max |grad| {scale:.2e}")
        assert scale > 0 and e <= tol, (name, e)

    check("q", grads["q"].cpu().double().numpy(), q64.grad.numpy(), attn_tol)
    rows = torch.cat([torch.arange(int(coff[s]), int(coff[s + 1])) for s in ref_sel.reshape(-1).tolist()]).unique()
    other = torch.ones(bank.n_chunks, dtype=torch.bool)
    other[rows] = False
    for name, got, ref in (("mem_k", grads["mem_k"], kp.grad), ("mem_v", grads["mem_v"], vp.grad)):
        got = got.cpu().double()
        check(name, got[rows].numpy(), ref[rows].numpy(), attn_tol)
        assert torch.all(got[other] == 0), name
    for name, cache_grad, ref_list in (("local_k", grads["local_k"], lk64), ("local_v", grads["local_v"], lv64)):
        gc = cache_grad.cpu().double()
        got = torch.cat([gc[int(loff[b]) * Hkv * d:int(loff[b + 1]) * Hkv * d].view(Hkv, cap[b], d)[:, :live[b]]
                         .reshape(-1) for b in range(B)])
        ref = torch.cat([t.grad.reshape(-1) for t in ref_list])
        check(name, got.numpy(), ref.numpy(), attn_tol)
        spare = torch.cat([gc[int(loff[b]) * Hkv * d:int(loff[b + 1]) * Hkv * d].view(Hkv, cap[b], d)[:, live[b]:]
                           .reshape(-1) for b in range(B)])
        assert torch.all(spare == 0), name
    check("qr", grads["qr"].cpu().double().numpy(), qr64.grad.numpy(), 1e-3)
    gkr = grads["kr"].cpu().double()
    check("kr", gkr.numpy(), krp.grad.numpy(), 1e-3)
    assert torch.equal(gkr != 0, krp.grad != 0)          # the same maximising chunks
