"""GPU parity of the streaming offline encode (msa_encoder_*) and of the
persistent pooled index (msa_index_save / msa_index_load).

Streaming: a bank pushed in ragged batches of whole documents must equal, bit
for bit, the bank msa_encode_memory builds in one launch (the same kernel
arithmetic), and the oracle's fp64 encoding within one bf16 rounding; the host
tier's K/V rows must land in the per-document interleaved layout.  The
pipeline's reuse contract is exercised by double-buffering the inputs.

Index file: save -> load returns the same bytes, its section hashes equal the
format's msa64 computed in Python from the file, the loaded bank routes and
decodes exactly like the original, and a flipped byte is caught."""
import numpy as np
import pytest
import torch

import oracle
import routed_sparse_attention_b200 as msa
from index_spec import msa64_spec, read_sections
from routed_sparse_attention_b200 import Layout, MSAError
from routed_sparse_attention_b200.runtime import Bank, Decoder, Router
from workloads import Workload, gen

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

W = Workload(name="stream-encode", dtype="bf16", n_docs=150, doc_len=150, lognormal_sigma=0.8, len_clip=(1, 700),
             chunk=64, n_q_heads=32, n_kv_heads=8, head_dim=128, router_dim=128, T=1, B=2, local_len=(40, 90),
             top_k=8, n_needles=2, per_token=True, kv_on_host=False, seed=900, mem_seed=901)
GROUPS = [1, 37, 2, 60, 50]           # documents per push


@pytest.fixture(scope="module")
def tokens():
    x = gen.generate(W, device="cpu")
    return x


def _batches(x, groups, kind="pinned"):
    tok = x["doc_tok_off"]
    d0 = 0
    for i, n in enumerate(groups):
        a, b = int(tok[d0]), int(tok[d0 + n])
        rel = torch.from_numpy(np.asarray(tok[d0:d0 + n + 1]) - a)
        ts = [x[key][a:b].contiguous() for key in ("k_tok", "v_tok", "kr_tok")]
        k = kind if kind != "mixed" else ("device", "pinned", "pageable")[i % 3]
        if k == "pinned":
            ts = [t.pin_memory() for t in ts]
        elif k == "device":
            ts = [t.cuda() for t in ts]
        yield (rel, *ts)
        d0 += n


def _limits(x, groups):
    tok = x["doc_tok_off"]
    lens = np.diff(tok)
    ends = np.cumsum([0] + groups)
    max_tok = max(int(tok[ends[i + 1]] - tok[ends[i]]) for i in range(len(groups)))
    return max_tok, max(groups), int(lens.max())


def _expected_host_kv(k, v, coff):
    """Chunk-major K/V to the host tier's rows: per document its K chunks, then its V chunks."""
    out = torch.empty(2 * k.shape[0], *k.shape[1:], dtype=k.dtype)
    for s in range(len(coff) - 1):
        a, b = int(coff[s]), int(coff[s + 1])
        out[2 * a:a + b] = k[a:b]
        out[a + b:2 * b] = v[a:b]
    return out


W32 = W.replace(name="stream-encode-f32", dtype="f32", head_dim=64, router_dim=64, n_q_heads=8, n_kv_heads=4)


@pytest.fixture(scope="module")
def tokens32():
    return gen.generate(W32, device="cpu")


def test_stream_encode_fp32_bank_matches_one_shot_encode(tokens32):
    x, w = tokens32, W32
    lay = Layout.of(w)
    max_tok, max_docs, max_len = _limits(x, GROUPS)
    coff = oracle.chunk_offsets(x["doc_tok_off"], w.chunk)
    bank = Bank.from_stream(lay, _batches(x, GROUPS), max_batch_tokens=max_tok, max_batch_docs=max_docs,
                            max_doc_len=max_len, capacity_chunks=int(coff[-1]), host_tier=True)
    one = Bank(lay, x["doc_tok_off"], k_tok=x["k_tok"].cuda(), v_tok=x["v_tok"].cuda(), kr_tok=x["kr_tok"].cuda())
    torch.cuda.synchronize()
    assert torch.equal(bank.kr.cpu(), one.kr.cpu())
    assert torch.equal(bank.host_kv, _expected_host_kv(one.k.cpu(), one.v.cpu(), coff))
    kp, vp, krp = oracle.encode(x["doc_tok_off"], x["k_tok"], x["v_tok"], x["kr_tok"], w.chunk, w.rope_theta)
    assert np.max(np.abs(bank.kr.cpu().numpy().astype(np.float64) - krp)) <= 1e-5
    assert np.max(np.abs(one.k.cpu().numpy().astype(np.float64) - kp)) <= 1e-5


@pytest.mark.parametrize("host_tier,kind", [(True, "pinned"), (False, "pinned"), (True, "mixed")],
                         ids=["hosttier-pinned", "device-pinned", "hosttier-mixed-inputs"])
def test_stream_encode_matches_one_shot_encode_and_oracle(tokens, host_tier, kind):
    x = tokens
    lay = Layout.of(W)
    max_tok, max_docs, max_len = _limits(x, GROUPS)
    coff_ref = oracle.chunk_offsets(x["doc_tok_off"], W.chunk)
    C = int(coff_ref[-1])
    bank = Bank.from_stream(lay, _batches(x, GROUPS, kind), max_batch_tokens=max_tok, max_batch_docs=max_docs,
                            max_doc_len=max_len, capacity_chunks=C + 3, host_tier=host_tier)
    assert np.array_equal(bank.doc_chunk_off_host.numpy(), coff_ref)
    assert bank.n_chunks == C and bank.max_doc_chunks == int(np.diff(coff_ref).max())
    one = Bank(lay, x["doc_tok_off"], k_tok=x["k_tok"].cuda(), v_tok=x["v_tok"].cuda(), kr_tok=x["kr_tok"].cuda())
    torch.cuda.synchronize()
    assert torch.equal(bank.kr.cpu(), one.kr.cpu())
    if host_tier:
        assert torch.equal(bank.host_kv, _expected_host_kv(one.k.cpu(), one.v.cpu(), coff_ref))
    else:
        assert torch.equal(bank.k.cpu(), one.k.cpu()) and torch.equal(bank.v.cpu(), one.v.cpu())
    # the oracle's fp64 encoding, within one bf16 rounding
    kp, vp, krp = oracle.encode(x["doc_tok_off"], x["k_tok"], x["v_tok"], x["kr_tok"], W.chunk, W.rope_theta)
    for got, ref in ((one.k, kp), (one.v, vp), (bank.kr, krp)):
        g = got.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(g - ref) <= (2.0 ** -8 + 1e-5) * np.abs(ref) + 1e-6)
    # the streamed bank routes like the oracle on its own pooled keys
    router = Router(bank, W.B, W.T, W.top_k)
    idx, _ = router(x["qr"].cuda())
    ref_idx, _ = oracle.route(x["qr"], coff_ref, bank.kr.cpu(), W.top_k, W.n_kv_heads)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert set(x["needle_docs"].tolist()) <= set(ref_idx.reshape(-1).tolist())
    assert msa.device_status() == 0


def test_stream_encode_double_buffered_inputs(tokens):
    """The caller rewrites push i's pinned inputs as soon as push i+1 has returned."""
    x = tokens
    lay = Layout.of(W)
    groups = [5, 20, 3, 40, 12, 30, 40]
    max_tok, max_docs, max_len = _limits(x, groups)
    C = int(oracle.chunk_offsets(x["doc_tok_off"], W.chunk)[-1])
    H, d, dr = W.n_kv_heads, W.head_dim, W.router_dim
    bufs = [[torch.empty(max_tok, H, dim, dtype=torch.bfloat16).pin_memory() for dim in (d, d, dr)]
            for _ in range(2)]
    kr = torch.empty(C, H, dr, dtype=torch.bfloat16, device="cuda")
    host_kv = torch.empty(2 * C, H, d, dtype=torch.bfloat16).pin_memory()
    enc = msa.StreamEncoder(lay, max_tok, max_docs, max_len, C, kr, host_kv_out=host_kv)
    for i, (rel, k, v, r) in enumerate(_batches(x, groups, "pageable")):
        n = int(rel[-1])
        buf = bufs[i % 2]
        for dst, src in zip(buf, (k, v, r)):
            dst[:n].copy_(src)                  # push i-1 returned: push i-2's copy-in is done
        enc.push(rel, *buf)
    nd, nc, _, coff = enc.finish()
    enc.close()
    one = Bank(lay, x["doc_tok_off"], k_tok=x["k_tok"].cuda(), v_tok=x["v_tok"].cuda(), kr_tok=x["kr_tok"].cuda())
    torch.cuda.synchronize()
    assert (nd, nc) == (W.n_docs, C)
    assert torch.equal(kr.cpu(), one.kr.cpu())
    assert torch.equal(host_kv, _expected_host_kv(one.k.cpu(), one.v.cpu(), coff.numpy()))


def test_stream_encode_rejects_overflow_and_stays_usable(tokens):
    x = tokens
    lay = Layout.of(W)
    max_tok, max_docs, max_len = _limits(x, GROUPS)
    coff = oracle.chunk_offsets(x["doc_tok_off"], W.chunk)
    first = int(coff[GROUPS[0] + GROUPS[1]])         # chunks of the first two pushes
    H, d, dr = W.n_kv_heads, W.head_dim, W.router_dim
    kr = torch.empty(first, H, dr, dtype=torch.bfloat16, device="cuda")
    host_kv = torch.empty(2 * first, H, d, dtype=torch.bfloat16).pin_memory()
    enc = msa.StreamEncoder(lay, max_tok, max_docs, max_len, first, kr, host_kv_out=host_kv)
    it = _batches(x, GROUPS)
    enc.push(*next(it))
    b2 = next(it)
    with pytest.raises(MSAError, match="documents"):          # more documents than max_batch_docs
        enc.push(torch.arange(max_docs + 2, dtype=torch.int64), *b2[1:])
    enc.push(*b2)
    with pytest.raises(MSAError, match="capacity"):           # the bank is full
        enc.push(*next(it))
    nd, nc, _, _ = enc.finish()
    enc.close()
    assert (nd, nc) == (GROUPS[0] + GROUPS[1], first)
    with pytest.raises(MSAError, match="tokens"):             # a document longer than max_doc_len
        e2 = msa.StreamEncoder(lay, max_tok, max_docs, 8, first, kr, host_kv_out=host_kv)
        try:
            e2.push(*b2)
        finally:
            e2.close()


# ------------------------------------------------------------------ index file

POOLED = Workload(name="store-pooled", dtype="bf16", n_docs=300, doc_len=200, lognormal_sigma=0.5, len_clip=(1, 1000),
                  chunk=64, n_q_heads=32, n_kv_heads=8, head_dim=128, router_dim=128, T=1, B=2,
                  local_len=(50, 120), top_k=8, n_needles=2, per_token=False, kv_on_host=False, seed=910,
                  mem_seed=911)


def _pooled_bank(w):
    x = gen.generate(w, device="cuda", host_interleaved=w.kv_on_host)
    bank = Bank(Layout.of(w), x["doc_tok_off"], kr_pool=x["kr_pool"], k_pool=x.get("k_pool"),
                v_pool=x.get("v_pool"), host_kv=x.get("host_kv"))
    return x, bank


def _route_decode(w, x, bank):
    router = Router(bank, w.B, w.T, w.top_k)
    dec = Decoder(bank, w.B, w.T, w.top_k, x["local_off"])
    k_rot = dec.rotate_local(x["local_k"], torch.empty_like(x["local_k"]))
    idx, sc = router(x["qr"])
    if bank.host_tier:
        st = torch.cuda.current_stream()
        ready, done = torch.cuda.Event(), torch.cuda.Event()
        ready.record(st)
        dec.fetch(router.idx_host, ready, st, done)
        st.wait_event(done)
    out = dec(x["q"], k_rot, x["local_v"], idx)
    torch.cuda.synchronize()
    return idx.cpu().clone(), sc.cpu().clone(), out.cpu().clone()


@pytest.mark.parametrize("host,dtype", [(False, "bf16"), (True, "bf16"), (False, "f32")],
                         ids=["device-bank", "hosttier-bank", "device-bank-f32"])
def test_index_save_load_round_trip(tmp_path, host, dtype):
    w = POOLED.replace(kv_on_host=host)
    if dtype == "f32":
        w = w.replace(dtype="f32", head_dim=64, router_dim=64, n_q_heads=8, n_kv_heads=4)
    x, bank = _pooled_bank(w)
    path = str(tmp_path / "bank.msaidx")
    bank.save(path)
    lay, nd, nc, mx, kv_host = msa.index_file_info(path)
    assert (nd, nc, mx, kv_host) == (bank.n_docs, bank.n_chunks, bank.max_doc_chunks, host)
    # every section's hash is the format's msa64 of the bytes in the file
    raw = open(path, "rb").read()
    for off, n, h in read_sections(path):
        assert h == msa64_spec(raw[off:off + n])
    assert raw[off + n:] == b"" or set(raw[off + n:]) <= {0}
    loaded = Bank.load(path)
    assert np.array_equal(loaded.doc_chunk_off_host.numpy(), bank.doc_chunk_off_host.numpy())
    assert torch.equal(loaded.kr.cpu(), bank.kr.cpu())
    if host:
        assert torch.equal(loaded.host_kv, bank.host_kv)
    else:
        assert torch.equal(loaded.k.cpu(), bank.k.cpu()) and torch.equal(loaded.v.cpu(), bank.v.cpu())
    a, b = _route_decode(w, x, bank), _route_decode(w, x, loaded)
    for u, v in zip(a, b):
        assert torch.equal(u, v)
    assert msa.device_status() == 0


def test_index_load_catches_a_flipped_byte(tmp_path):
    x, bank = _pooled_bank(POOLED)
    path = tmp_path / "bank.msaidx"
    bank.save(str(path))
    off, n, _ = read_sections(str(path))[1]           # Kr
    raw = bytearray(path.read_bytes())
    raw[off + n // 2] ^= 0x40
    path.write_bytes(bytes(raw))
    with pytest.raises(MSAError, match="checksum"):
        Bank.load(str(path))
    loaded = Bank.load(str(path), verify=False)
    diff = (loaded.kr.cpu().view(torch.int16) != bank.kr.cpu().view(torch.int16)).sum().item()
    assert diff == 1


def test_index_round_trip_several_bounce_pieces(tmp_path):
    """Sections larger than the 64 MiB pinned pieces the copies go through."""
    w = POOLED.replace(name="store-large", n_docs=12500, doc_len=256, lognormal_sigma=0.0, len_clip=(256, 256),
                       n_needles=0)
    x, bank = _pooled_bank(w)
    assert bank.kr.numel() * 2 > 64 << 20
    path = str(tmp_path / "large.msaidx")
    bank.save(path)
    loaded = Bank.load(path)
    assert torch.equal(loaded.kr.cpu(), bank.kr.cpu())
    assert torch.equal(loaded.k.cpu(), bank.k.cpu()) and torch.equal(loaded.v.cpu(), bank.v.cpu())
