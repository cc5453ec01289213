"""GPU parity of the multi-layer routed decode loop (runtime.RoutedDecodeLoop).

Two routing layers, each with its own memory bank (layer 1 in the host tier),
two queries with prompts of different lengths, three generated tokens.  At
every step and layer the routed documents must equal the oracle's routing of
that step's router query (or of the first step's, with route_once), and the
decoded token must match the oracle's decode over the live local context --
the prompt plus every token appended so far, keys unrotated on the oracle
side -- within the bf16 tolerance."""
import numpy as np
import pytest
import torch

import oracle
from gpu_cases import BF16_TOL
from routed_sparse_attention_b200 import Layout
from routed_sparse_attention_b200.runtime import Bank, RoutedDecodeLoop
from workloads import Workload, gen

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

BASE = Workload(name="loop-layer", dtype="bf16", n_docs=300, doc_len=200, lognormal_sigma=0.5,
                len_clip=(1, 1000), chunk=64, n_q_heads=32, n_kv_heads=8, head_dim=128, router_dim=128,
                T=1, B=2, local_len=(1, 1), top_k=8, n_needles=0, per_token=False, kv_on_host=False,
                seed=500, mem_seed=600)
PROMPT = [20, 35]
STEPS = 3


def layer_bank(i: int, host: bool):
    w = BASE.replace(name=f"loop-layer{i}", mem_seed=600 + i, kv_on_host=host)
    qr0 = torch.zeros(w.B, w.T, w.n_q_heads, w.router_dim)          # no needles: unused
    x = gen.make_memory(w, qr0, "cuda", host_interleaved=host)
    bank = Bank(Layout.of(w), x["doc_tok_off"], kr_pool=x["kr_pool"], k_pool=x.get("k_pool"),
                v_pool=x.get("v_pool"), host_kv=x.get("host_kv"))
    return w, x, bank


def randn(g, *shape):
    return torch.randn(*shape, generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("route_once", [False, True], ids=["route-per-step", "route-once"])
def test_two_layer_loop_appends_routes_and_decodes(route_once):
    layers = [layer_bank(0, False), layer_bank(1, True)]
    w = BASE
    H, d, Hq, dr, k = w.n_kv_heads, w.head_dim, w.n_q_heads, w.router_dim, w.top_k
    B = len(PROMPT)
    loop = RoutedDecodeLoop([bk for _, _, bk in layers], B, k, torch.tensor(PROMPT),
                            torch.tensor(PROMPT) + STEPS, route_once=route_once)
    g = torch.Generator().manual_seed(1234)
    # the oracle's copy of every layer's live local context, keys unrotated
    ctx = []
    for li in range(len(layers)):
        kp = [randn(g, H, PROMPT[b], d) for b in range(B)]
        vp = [randn(g, H, PROMPT[b], d) for b in range(B)]
        loop.prefill(li, [t.cuda() for t in kp], [t.cuda() for t in vp])
        ctx.append((kp, vp))
    first_sel = [None] * len(layers)
    for step in range(STEPS):
        for li, (lw, x, bank) in enumerate(layers):
            qr = randn(g, B, 1, Hq, dr)
            q = randn(g, B, 1, Hq, d)
            kn, vn = randn(g, B, H, d), randn(g, B, H, d)
            out, sel = loop.step(li, qr.cuda(), q.cuda(), kn.cuda(), vn.cuda())
            torch.cuda.synchronize()
            kp, vp = ctx[li]
            for b in range(B):
                kp[b] = torch.cat([kp[b], kn[b].unsqueeze(1)], dim=1)
                vp[b] = torch.cat([vp[b], vn[b].unsqueeze(1)], dim=1)
            coff = oracle.chunk_offsets(x["doc_tok_off"], lw.chunk)
            if route_once and step > 0:
                ref_idx = first_sel[li]
            else:
                ref_idx, _ = oracle.route(qr, coff, x["kr_pool"].cpu(), k, H)
            if first_sel[li] is None:
                first_sel[li] = ref_idx
            got_idx = sel.cpu().numpy()
            assert np.array_equal(got_idx, ref_idx), (step, li)
            lens = [kp[b].shape[1] for b in range(B)]
            assert loop.decoders[li].lengths().tolist() == lens
            loff = np.concatenate([[0], np.cumsum(lens)])
            lk = torch.cat([kp[b].reshape(-1) for b in range(B)])
            lv = torch.cat([vp[b].reshape(-1) for b in range(B)])
            if bank.host_tier:
                ref = oracle.decode(q, ref_idx, coff, x["host_kv"], None, loff, lk, lv, k, lw.rope_theta, H,
                                    kv_layout=oracle.KV_DOC_INTERLEAVED)
            else:
                ref = oracle.decode(q, ref_idx, coff, x["k_pool"].cpu(), x["v_pool"].cpu(), loff, lk, lv, k,
                                    lw.rope_theta, H)
            err = float(np.max(np.abs(out.float().cpu().numpy() - ref)))
            print(f"[loop step {step} layer {li}] max |out - oracle| = {err:.3e}")
            assert err <= BF16_TOL, (step, li, err)
    expected_routes = len(layers) * (1 if route_once else STEPS)
    assert loop.routed_steps == expected_routes


def test_graph_replayed_loop_matches_oracle():
    """Route once, then every token's appends and decodes on both layers as
    one CUDA graph replay, with the live lengths in device memory."""
    layers = [layer_bank(0, False), layer_bank(1, True)]
    w = BASE
    H, d, Hq, dr, k = w.n_kv_heads, w.head_dim, w.n_q_heads, w.router_dim, w.top_k
    B, steps = len(PROMPT), 5
    loop = RoutedDecodeLoop([bk for _, _, bk in layers], B, k, torch.tensor(PROMPT), torch.tensor(PROMPT) + steps,
                            route_once=True, graph=True)
    g = torch.Generator().manual_seed(4321)
    ctx = []
    for li in range(len(layers)):
        kp = [randn(g, H, PROMPT[b], d) for b in range(B)]
        vp = [randn(g, H, PROMPT[b], d) for b in range(B)]
        loop.prefill(li, [t.cuda() for t in kp], [t.cuda() for t in vp])
        ctx.append((kp, vp))
    qr0 = [randn(g, B, 1, Hq, dr) for _ in layers]
    ref_idx = [oracle.route(qr0[li], oracle.chunk_offsets(x["doc_tok_off"], lw.chunk), x["kr_pool"].cpu(), k, H)[0]
               for li, (lw, x, _) in enumerate(layers)]
    for step in range(steps):
        toks = []
        for li in range(len(layers)):
            q, kn, vn = randn(g, B, 1, Hq, d), randn(g, B, H, d), randn(g, B, H, d)
            loop.inputs[li]["q"].copy_(q)
            loop.inputs[li]["k_new"].copy_(kn)
            loop.inputs[li]["v_new"].copy_(vn)
            toks.append((q, kn, vn))
        outs = loop.token([t.cuda() for t in qr0] if step == 0 else None)
        torch.cuda.synchronize()
        assert loop.lengths().tolist() == [p + step + 1 for p in PROMPT]
        for li, (lw, x, bank) in enumerate(layers):
            assert np.array_equal(loop.sel[li].cpu().numpy(), ref_idx[li])
            q, kn, vn = toks[li]
            kp, vp = ctx[li]
            for b in range(B):
                kp[b] = torch.cat([kp[b], kn[b].unsqueeze(1)], dim=1)
                vp[b] = torch.cat([vp[b], vn[b].unsqueeze(1)], dim=1)
            coff = oracle.chunk_offsets(x["doc_tok_off"], lw.chunk)
            loff = np.concatenate([[0], np.cumsum([t.shape[1] for t in kp])])
            lk = torch.cat([t.reshape(-1) for t in kp])
            lv = torch.cat([t.reshape(-1) for t in vp])
            if bank.host_tier:
                ref = oracle.decode(q, ref_idx[li], coff, x["host_kv"], None, loff, lk, lv, k, lw.rope_theta, H,
                                    kv_layout=oracle.KV_DOC_INTERLEAVED)
            else:
                ref = oracle.decode(q, ref_idx[li], coff, x["k_pool"].cpu(), x["v_pool"].cpu(), loff, lk, lv, k,
                                    lw.rope_theta, H)
            err = float(np.max(np.abs(outs[li].float().cpu().numpy() - ref)))
            print(f"[graph loop token {step} layer {li}] max |out - oracle| = {err:.3e}")
            assert err <= BF16_TOL, (step, li, err)
    assert loop.routed_steps == len(layers)
    import routed_sparse_attention_b200 as msa
    assert msa.device_status() == 0


def test_append_local_writes_one_row_per_query_and_head():
    """msa_append_local: the value, the raw key and the key rotated at
    top_k + len_b land in row len_b of every head; the rotated key equals
    msa_rope_local's rotation of the raw row bit for bit; no other row moves."""
    import routed_sparse_attention_b200 as msa
    w = BASE
    lay = Layout.of(w)
    H, d, k = w.n_kv_heads, w.head_dim, 5
    cap, live = [7, 12, 3], [4, 11, 0]
    loff = torch.tensor([0] + list(np.cumsum(cap)), dtype=torch.int64)
    rows = int(loff[-1]) * H * d
    g = torch.Generator().manual_seed(77)
    k_raw = torch.randn(rows, generator=g).to(torch.bfloat16).cuda()
    k_rot = torch.randn(rows, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(rows, generator=g).to(torch.bfloat16).cuda()
    before = [t.clone() for t in (k_raw, k_rot, v)]
    kn = torch.randn(3, H, d, generator=g).to(torch.bfloat16).cuda()
    vn = torch.randn(3, H, d, generator=g).to(torch.bfloat16).cuda()
    rope = msa.rope_table(lay, k + max(cap))
    msa.append_local(lay, loff, torch.tensor(live), kn, vn, k, rope, k_rot, v, k_raw)
    ref_rot = torch.empty_like(k_raw)
    msa.rope_local(lay, loff, k, k_raw, ref_rot, rope, torch.tensor(live), None,
                   local_len_host=torch.tensor(live) + 1)
    torch.cuda.synchronize()
    changed = torch.zeros(rows, dtype=torch.bool, device="cuda")
    for b in range(3):
        for hh in range(H):
            r0 = (int(loff[b]) * H + hh * cap[b] + live[b]) * d
            assert torch.equal(v[r0:r0 + d], vn[b, hh]) and torch.equal(k_raw[r0:r0 + d], kn[b, hh])
            assert torch.equal(k_rot[r0:r0 + d], ref_rot[r0:r0 + d])
            changed[r0:r0 + d] = True
    for t, t0 in zip((k_raw, k_rot, v), before):
        assert torch.equal(t[~changed], t0[~changed])


@pytest.mark.parametrize("B,T", [(2, 1), (3, 4)], ids=["cuda-core-scan", "tensor-core-scan"])
def test_route_captured_in_a_graph_matches_oracle(B, T):
    """Routing captured in a CUDA graph (its kernels after the prep are chained
    by programmatic launch) and replayed on new router queries gives the
    oracle's indices and certified scores bit for bit on every replay."""
    from routed_sparse_attention_b200.runtime import Router
    w, x, bank = layer_bank(0, False)
    k, H = w.top_k, w.n_kv_heads
    coff = oracle.chunk_offsets(x["doc_tok_off"], w.chunk)
    router = Router(bank, B, T, k)
    g = torch.Generator().manual_seed(97 + B)
    qrs = [randn(g, B, T, w.n_q_heads, w.router_dim) for _ in range(3)]
    static_qr = qrs[0].cuda()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        router(static_qr)                              # first call outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        router(static_qr)
    for i in (1, 2, 0, 1):
        static_qr.copy_(qrs[i].cuda())
        graph.replay()
        torch.cuda.synchronize()
        ref_idx, ref_score = oracle.route(qrs[i], coff, x["kr_pool"].cpu(), k, H)
        assert np.array_equal(router.idx.cpu().numpy(), ref_idx), i
        assert np.array_equal(router.score.cpu().numpy(), ref_score), i
    import routed_sparse_attention_b200 as msa
    assert msa.device_status() == 0
