"""The C-ABI library loads on a machine without a GPU, exports every entry point
include/msa.h declares, and its host-only logic is correct (no compute calls)."""
import ctypes
import os
import re
import struct

import numpy as np
import pytest
import torch

import oracle
import routed_sparse_attention_b200 as msa
from index_spec import msa64_spec, spec_header
from workloads import MEM_16M, gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    """Every function declared by the headers under include/ (msa.h: the
    path; msa_debug.h: instrumentation and test hooks)."""
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not h.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", h)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(msa_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


def test_debug_hooks_live_apart_from_the_path():
    src = open(os.path.join(ROOT, "include", "msa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    assert "msa_debug_" not in src
    dbg = open(os.path.join(ROOT, "include", "msa_debug.h")).read()
    for n in ("msa_debug_expire_wait", "msa_debug_scan_events", "msa_debug_fail_next_copies"):
        assert n + "(" in dbg


def test_library_exports_every_declared_entry_point():
    L = msa.lib()
    names = declared_entry_points()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), n
    assert sorted(msa.ENTRY_POINTS) == names
    assert msa.version() == 1


def test_library_is_built_for_sm100a():
    log = open(os.path.join(ROOT, "routed_sparse_attention_b200", "build.log")).read()
    assert "arch=compute_100a,code=sm_100a" in log


def test_chunk_offsets_match_oracle_bit_exact():
    L = gen.doc_lengths(MEM_16M)
    tok = gen.offsets(L)
    got, mx, mlen = msa.chunk_offsets(torch.from_numpy(tok), 64)
    want = oracle.chunk_offsets(tok, 64)
    assert np.array_equal(got.numpy(), want)
    assert mx == int(np.max(np.diff(want))) and mlen == int(L.max())


def test_chunk_offsets_reject_empty_documents():
    with pytest.raises(msa.MSAError) as e:
        msa.chunk_offsets(torch.tensor([0, 5, 5, 9]), 64)
    assert e.value.status == 1


def test_status_strings_and_bad_arguments_fail_before_any_launch():
    L = msa.lib()
    assert L.msa_status_string(5) == b"timeout"
    lay = msa.Layout(32, 8, 128, 128, 64, "bf16")
    # NULL layout / index
    rc = L.msa_route(None, None, 1, 1, None, 16, None, None, None, None, 0, None)
    assert rc == 1 and b"layout" in L.msa_last_error()
    # H_q not a multiple of H_kv
    bad = msa.Layout(30, 8, 128, 128, 64, "bf16")
    assert L.msa_rope_table(bad.ref(), 16, None, None) == 1
    # router_dim * element size != 256 is rejected as unsupported
    fake = ctypes.c_void_p(1 << 20)
    idx = msa._Index(10, 10, fake, None, 1, 0, fake, fake, fake, None)
    odd = msa.Layout(32, 8, 128, 64, 64, "bf16")
    rc = L.msa_route(odd.ref(), ctypes.byref(idx), 1, 1, fake, 4, fake, None, None, fake, 1 << 30, None)
    assert rc == 2
    # top_k out of range, workspace too small
    rc = L.msa_route(lay.ref(), ctypes.byref(idx), 1, 1, fake, 11, fake, None, None, fake, 1 << 30, None)
    assert rc == 1
    rc = L.msa_route(lay.ref(), ctypes.byref(idx), 1, 1, fake, 4, fake, None, None, fake, 16, None)
    assert rc == 4
    # decode: local rows shorter than T, and batch beyond the supported maximum
    lo = torch.tensor([0, 3], dtype=torch.int64)
    assert L.msa_decode_workspace_size(lay.ref(), 1, 4, msa._p(lo), None) == 0
    lo = torch.arange(0, 258 * 5, 5, dtype=torch.int64)
    assert L.msa_decode_workspace_size(lay.ref(), 257, 1, msa._p(lo), None) == 0
    lo = torch.tensor([0, 4097], dtype=torch.int64)
    assert L.msa_decode_workspace_size(lay.ref(), 1, 1, msa._p(lo), None) > 0
    # live lengths: at least T, at most the capacity
    ln = torch.tensor([4097], dtype=torch.int64)
    assert L.msa_decode_workspace_size(lay.ref(), 1, 1, msa._p(lo), msa._p(ln)) > 0
    ln = torch.tensor([4098], dtype=torch.int64)
    assert L.msa_decode_workspace_size(lay.ref(), 1, 1, msa._p(lo), msa._p(ln)) == 0
    ln = torch.tensor([3], dtype=torch.int64)
    assert L.msa_decode_workspace_size(lay.ref(), 1, 4, msa._p(lo), msa._p(ln)) == 0
    # routing takes up to 512 queries per call
    rc = L.msa_route(lay.ref(), ctypes.byref(idx), 513, 1, fake, 4, fake, None, None, fake, 1 << 40, None)
    assert rc == 2 and b"512" in L.msa_last_error()


def test_device_fetch_rejects_bad_arguments_before_any_launch():
    L = msa.lib()
    lay = msa.Layout(32, 8, 128, 128, 64, "bf16")
    fake = ctypes.c_void_p(1 << 20)
    host = msa._Index(10, 40, fake, fake, 4, 1, fake, None, None, fake, None)
    dev = msa._Index(10, 40, fake, None, 4, 0, fake, fake, fake, None, None)
    need = L.msa_fetch_staging_size(lay.ref(), ctypes.byref(host), 1, 4)
    assert need == 4 * 2 * 4 * 8 * 128 * 2
    # a device-tier bank has nothing to fetch
    assert L.msa_fetch_selected_device(lay.ref(), ctypes.byref(dev), 1, 4, fake, fake, need, None) == 1
    # missing selection, misaligned staging, bad batch or top_k
    assert L.msa_fetch_selected_device(lay.ref(), ctypes.byref(host), 1, 4, None, fake, need, None) == 1
    assert L.msa_fetch_selected_device(lay.ref(), ctypes.byref(host), 1, 4, fake, ctypes.c_void_p((1 << 20) + 8),
                                       need, None) == 1
    assert L.msa_fetch_selected_device(lay.ref(), ctypes.byref(host), 0, 4, fake, fake, need, None) == 1
    assert L.msa_fetch_selected_device(lay.ref(), ctypes.byref(host), 1, 11, fake, fake, need, None) == 1
    # staging one byte short
    assert L.msa_fetch_selected_device(lay.ref(), ctypes.byref(host), 1, 4, fake, fake, need - 1, None) == 4


def test_raw_key_decode_workspace_and_checks_before_any_launch():
    """msa_sparse_decode_raw's workspace is the decode's, a rotated copy of the
    local keys (whole capacities) and, for the host tier, the staging; a short
    workspace or rejected lengths fail before anything is launched."""
    L = msa.lib()
    lay = msa.Layout(32, 8, 128, 128, 64, "bf16")
    fake = ctypes.c_void_p(1 << 20)
    dev = msa._Index(10, 40, fake, None, 4, 0, fake, fake, fake, None, None)
    host = msa._Index(10, 40, fake, fake, 4, 1, fake, None, None, fake, None)
    lo = torch.tensor([0, 300, 700], dtype=torch.int64)
    ll = torch.tensor([260, 701 - 300 - 1], dtype=torch.int64)
    dec = L.msa_decode_workspace_size(lay.ref(), 2, 1, msa._p(lo), msa._p(ll))
    keys = -(-700 * 8 * 128 * 2 // 256) * 256
    staging = L.msa_fetch_staging_size(lay.ref(), ctypes.byref(host), 2, 4)
    assert dec > 0
    assert L.msa_sparse_decode_raw_workspace_size(lay.ref(), ctypes.byref(dev), 2, 1, 4, msa._p(lo), msa._p(ll)) \
        == dec + keys
    need = L.msa_sparse_decode_raw_workspace_size(lay.ref(), ctypes.byref(host), 2, 1, 4, msa._p(lo), msa._p(ll))
    assert need == dec + keys + -(-staging // 256) * 256
    # live length beyond the capacity: rejected by the plan
    bad = torch.tensor([301, 10], dtype=torch.int64)
    assert L.msa_sparse_decode_raw_workspace_size(lay.ref(), ctypes.byref(dev), 2, 1, 4, msa._p(lo), msa._p(bad)) == 0
    args = (lay.ref(), ctypes.byref(host), 2, 1, fake, fake, fake, msa._p(lo), msa._p(ll), fake, 4, fake, 5000, fake,
            fake)
    assert L.msa_sparse_decode_raw(*args, need - 1, None) == 4
    assert L.msa_sparse_decode_raw(lay.ref(), ctypes.byref(host), 2, 1, fake, None, fake, msa._p(lo), msa._p(ll), fake,
                                   4, fake, 5000, fake, fake, need, None) == 1


def test_route_workspace_size_follows_the_chunk_count():
    """The tensor-core scan (more than 4 query rows on a bf16 bank) keeps one
    entry per 128-chunk tile in the routing workspace, so its size must grow
    with the bank's chunk count; msa_route checks the plan built from the real
    chunk count, so one byte less is refused before any launch."""
    L = msa.lib()
    lay = msa.Layout(32, 8, 128, 128, 64, "bf16")
    D = 65536
    base = msa.route_workspace_size(lay, D, D, 8, 1, 32)
    assert base > 0
    for C in (306_369, 1_562_500, 50_000_000):
        grown = msa.route_workspace_size(lay, D, C, 8, 1, 32)
        tiles = -(-C // 128) - -(-D // 128)
        assert grown - base >= 4 * tiles - 256, (C, grown - base, tiles)
    # a chunk count below the document count is no bank
    assert msa.route_workspace_size(lay, D, D - 1, 8, 1, 32) == 0
    # one byte short of the real plan: refused before anything is launched
    fake = ctypes.c_void_p(1 << 20)
    C = 1_562_500
    idx = msa._Index(D, C, fake, None, 1, 0, fake, fake, fake, None)
    qr = ctypes.c_void_p(1 << 21)
    need = msa.route_workspace_size(lay, D, C, 8, 1, 32)
    rc = L.msa_route(lay.ref(), ctypes.byref(idx), 8, 1, qr, 32, fake, None, None, fake, need - 1, None)
    assert rc == 4 and b"workspace" in L.msa_last_error()
    rc = L.msa_route_scores(lay.ref(), ctypes.byref(idx), 8, 1, qr, fake, fake, need - 1, None)
    assert rc == 4


def test_rope_local_rejects_bad_arguments_before_any_launch():
    L = msa.lib()
    lay = msa.Layout(32, 8, 128, 128, 64, "bf16")
    buf = ctypes.c_void_p(1 << 20)
    lo = torch.tensor([0, 10, 20], dtype=torch.int64)

    def call(B=2, first=None, k=16, src=buf, dst=buf, rope_rows=64, ln=None):
        return L.msa_rope_local(lay.ref(), B, msa._p(lo), msa._p(ln), msa._p(first), k, src, dst, buf, rope_rows,
                                None)

    assert call(B=0) == 2
    assert call(src=None) == 1
    assert call(first=torch.tensor([11, 0], dtype=torch.int64)) == 1 and b"first" in L.msa_last_error()
    assert call(first=torch.tensor([-1, 0], dtype=torch.int64)) == 1
    assert call(rope_rows=25) == 1 and b"rope_rows" in L.msa_last_error()
    assert call(dst=ctypes.c_void_p((1 << 20) + 4096)) == 1 and b"overlap" in L.msa_last_error()
    assert call(src=ctypes.c_void_p((1 << 20) + 8)) == 1 and b"aligned" in L.msa_last_error()
    # nothing left to rotate: accepted without a launch
    assert call(first=torch.tensor([10, 10], dtype=torch.int64)) == 0
    # live lengths within the capacities; first within the live length
    assert call(ln=torch.tensor([11, 3], dtype=torch.int64)) == 1 and b"live length" in L.msa_last_error()
    assert call(ln=torch.tensor([4, 3], dtype=torch.int64), first=torch.tensor([5, 0], dtype=torch.int64)) == 1
    assert call(ln=torch.tensor([4, 3], dtype=torch.int64), first=torch.tensor([4, 3], dtype=torch.int64)) == 0


def test_debug_expire_wait_checks_its_arguments_first():
    L = msa.lib()
    n = ctypes.c_int32(0)
    assert L.msa_debug_expire_wait(-1, ctypes.byref(n), None) == 1
    assert L.msa_debug_expire_wait(20000000, ctypes.byref(n), None) == 1
    assert L.msa_debug_expire_wait(1000, None, None) == 1


def test_device_length_calls_check_their_arguments_first():
    L = msa.lib()
    lay = msa.Layout(32, 8, 128, 128, 64, "bf16")
    buf = ctypes.c_void_p(1 << 20)
    lo = torch.tensor([0, 10, 20], dtype=torch.int64)
    assert L.msa_advance_local_len(0, buf, 1, None) == 1
    assert L.msa_advance_local_len(2, None, 1, None) == 1
    assert L.msa_append_local_devlen(lay.ref(), 2, msa._p(lo), None, buf, buf, 16, buf, 64, None, buf, buf, None) == 1
    # the rotary table must cover top_k + the largest capacity
    assert L.msa_append_local_devlen(lay.ref(), 2, msa._p(lo), buf, buf, buf, 16, buf, 20, None, buf, buf, None) == 1
    assert b"rope_rows" in L.msa_last_error()
    assert L.msa_sparse_decode_devlen(lay.ref(), None, 2, 1, buf, buf, buf, msa._p(lo), None, buf, 16, None, buf, 64,
                                      buf, buf, 1 << 20, None) == 1


def test_append_local_rejects_bad_arguments_before_any_launch():
    L = msa.lib()
    lay = msa.Layout(32, 8, 128, 128, 64, "bf16")
    buf = ctypes.c_void_p(1 << 20)
    lo = torch.tensor([0, 10, 20], dtype=torch.int64)

    def call(B=2, ln=(3, 9), k=16, rope_rows=64, kr=buf, v=buf, raw=None):
        ln = torch.tensor(ln, dtype=torch.int64)
        return L.msa_append_local(lay.ref(), B, msa._p(lo), msa._p(ln), buf, buf, k, buf, rope_rows, raw, kr, v,
                                  None)

    assert call(B=0) == 2
    assert call(kr=None) == 1 and b"missing" in L.msa_last_error()
    assert call(raw=ctypes.c_void_p((1 << 20) + 8)) == 1 and b"aligned" in L.msa_last_error()
    assert call(ln=(3, 10)) == 1 and b"no room" in L.msa_last_error()          # query 1 is full
    assert call(ln=(-1, 0)) == 1
    assert call(rope_rows=25) == 1 and b"rope_rows" in L.msa_last_error()     # 16 + 9 needs 26 rows


def test_interleave_expand_rejects_bad_arguments_before_any_launch():
    L = msa.lib()
    a, o, n_ = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 22), ctypes.c_void_p(1 << 24)

    def call(n_docs=100, B=2, n=4, p=4, ranked=a, old=o, new=n_):
        return L.msa_interleave_expand(n_docs, B, n, p, ranked, old, new, None, None)

    assert call(B=0) == 2 and call(B=513) == 2
    assert call(p=0) == 1 and call(n=-1) == 1
    assert call(n=60, p=5) == 1 and b"exceeds" in L.msa_last_error()          # n + p > 64
    assert call(n_docs=7) == 1 and b"exceeds" in L.msa_last_error()           # n + p > n_docs
    assert call(old=None) == 1 and b"missing" in L.msa_last_error()           # n > 0 needs the old set
    assert call(ranked=None) == 1 and call(new=None) == 1
    # the new set may not overlap the ranking or the old set
    assert call(new=ctypes.c_void_p((1 << 20) + 32)) == 1 and b"overlap" in L.msa_last_error()
    assert call(new=ctypes.c_void_p((1 << 22) + 8)) == 1 and b"overlap" in L.msa_last_error()


def test_kr_inv_norm_count_and_argument_checks():
    L = msa.lib()
    lay = msa.Layout(32, 8, 128, 128, 64, "bf16")
    assert L.msa_kr_inv_norm_count(lay.ref(), 300) == 8 * 384
    assert L.msa_kr_inv_norm_count(lay.ref(), 128) == 8 * 128
    assert L.msa_kr_inv_norm_count(lay.ref(), 0) == 0
    assert L.msa_kr_inv_norm_count(None, 10) == 0
    fake = ctypes.c_void_p(1 << 20)
    idx = msa._Index(10, 10, fake, None, 1, 0, fake, fake, fake, None)
    assert L.msa_kr_inv_norms(lay.ref(), ctypes.byref(idx), None, None) == 1
    assert L.msa_kr_inv_norms(lay.ref(), ctypes.byref(idx), ctypes.c_void_p((1 << 20) + 4), None) == 1
    # a misaligned table in the index is rejected by every call that checks the index
    bad = msa._Index(10, 10, fake, None, 1, 0, fake, fake, fake, None, ctypes.c_void_p((1 << 20) + 4))
    assert L.msa_kr_inv_norms(lay.ref(), ctypes.byref(bad), fake, None) == 1
    assert b"kr_inv_norm" in L.msa_last_error()


def test_fetch_reports_an_injected_copy_failure():
    """A failed host-to-device copy surfaces as MSA_ERR_CUDA (made on the host by
    the library's test hook, so no device is touched)."""
    L = msa.lib()
    lay = msa.Layout(32, 8, 128, 128, 64, "bf16")
    coff = torch.tensor([0, 4, 8], dtype=torch.int64)
    host = torch.zeros(16 * 8 * 128, dtype=torch.bfloat16)
    fake = ctypes.c_void_p(1 << 20)
    idx = msa._Index(2, 8, fake, msa._p(coff), 4, 1, fake, None, None, msa._p(host))
    sel = torch.tensor([[1, 0]], dtype=torch.int32)
    staging_bytes = L.msa_fetch_staging_size(lay.ref(), ctypes.byref(idx), 1, 2)
    assert staging_bytes == 2 * 2 * 4 * 8 * 128 * 2
    L.msa_debug_fail_next_copies(1)
    rc = L.msa_fetch_selected(lay.ref(), ctypes.byref(idx), 1, 2, msa._p(sel), None, 100, fake,
                              staging_bytes, None, None)
    assert rc == 3 and b"fetch copy" in L.msa_last_error()
    # out-of-range selected document is an argument error
    sel2 = torch.tensor([[1, 7]], dtype=torch.int32)
    rc = L.msa_fetch_selected(lay.ref(), ctypes.byref(idx), 1, 2, msa._p(sel2), None, 100, fake,
                              staging_bytes, None, None)
    assert rc == 1
    L.msa_debug_fail_next_copies(0)


# ------------------------------------------------ streaming encoder, index file

def test_encoder_create_and_push_reject_bad_arguments_before_any_allocation():
    L = msa.lib()
    lay = msa.Layout(32, 8, 128, 128, 64, "bf16")
    dev = ctypes.c_void_p(1 << 20)
    h = ctypes.c_void_p()

    def create(max_tok=1024, docs=8, max_len=512, cap=100, kr=dev, k=None, v=None, host=dev, out=True):
        return L.msa_encoder_create(lay.ref(), max_tok, docs, max_len, cap, kr, k, v, host,
                                    ctypes.byref(h) if out else None)

    assert create(out=False) == 1
    assert create(max_tok=0) == 1 and create(docs=0) == 1 and create(max_len=0) == 1 and create(cap=0) == 1
    assert create(kr=None) == 1 and create(kr=ctypes.c_void_p((1 << 20) + 8)) == 1
    assert create(k=dev, v=dev) == 1 and b"not both" in L.msa_last_error()       # host tier and device K/V
    assert create(host=None) == 1 and b"required" in L.msa_last_error()         # device tier without K/V
    assert h.value is None
    tok = torch.tensor([0, 3], dtype=torch.int64)
    assert L.msa_encoder_push(None, 1, msa._p(tok), dev, dev, dev) == 1
    assert L.msa_encoder_finish(None, None, None, None) == 1
    L.msa_encoder_destroy(None)                                                   # a no-op


def test_index_file_info_reads_a_header_written_from_the_spec(tmp_path):
    # the header hash (63 words: the four-lane body and a tail) is the
    # library's msa64; a header hashed by the Python restatement is accepted
    L = msa.lib()
    p = tmp_path / "bank.msaidx"
    p.write_bytes(bytes(spec_header()))
    lay, nd, nc, mx, host = msa.index_file_info(str(p))
    assert (lay.c.n_q_heads, lay.c.n_kv_heads, lay.c.head_dim, lay.c.router_dim, lay.c.chunk_size,
            lay.c.dtype, lay.c.rope_theta) == (32, 8, 128, 128, 64, 1, 1e6)
    assert (nd, nc, mx, host) == (3, 7, 4, True)
    p.write_bytes(bytes(spec_header(host=0, layout=(4, 2, 64, 64, 16, 0), theta=1e4)))
    lay, nd, nc, mx, host = msa.index_file_info(str(p))
    assert (lay.c.head_dim, lay.c.dtype, lay.c.rope_theta, host) == (64, 0, 1e4, False)

    def info_err(data):
        p.write_bytes(bytes(data))
        rc = L.msa_index_file_info(os.fsencode(str(p)), None, None, None, None, None)
        return rc, L.msa_last_error()

    b = spec_header()
    b[0] ^= 1                                                          # magic
    assert info_err(b)[0] == 1 and b"magic" in info_err(b)[1]
    b = spec_header()
    b[60] ^= 1                                                         # n_chunks, header hash now stale
    assert info_err(b)[0] == 1 and b"checksum" in info_err(b)[1]
    b = spec_header()
    struct.pack_into("<Q", b, 72 + 24, 12288)                          # section 1 moved
    struct.pack_into("<Q", b, 504, msa64_spec(bytes(b[:504])))
    assert info_err(b)[0] == 1 and b"placement" in info_err(b)[1]
    b = spec_header()
    struct.pack_into("<I", b, 8, 2)                                    # a later format version
    struct.pack_into("<Q", b, 504, msa64_spec(bytes(b[:504])))
    assert info_err(b)[0] == 2
    assert info_err(spec_header()[:300])[0] == 1                       # truncated
    assert L.msa_index_file_info(os.fsencode(str(tmp_path / "missing")), None, None, None, None, None) == 1


def test_attention_backward_rejects_bad_arguments_before_any_launch():
    """msa_sparse_attention_backward checks the bank tier, shapes, top_k,
    pointers, alignment, offsets, workspace and live lengths on the host; the
    fake device pointers below are never dereferenced."""
    L = msa.lib()
    lay = msa.Layout(32, 8, 128, 128, 64, "bf16")
    fake = ctypes.c_void_p(1 << 20)                  # 16-byte aligned
    odd = ctypes.c_void_p((1 << 20) + 4)
    dev_idx = msa._Index(10, 40, fake, None, 4, 0, fake, fake, fake, None, None)
    host_idx = msa._Index(10, 40, fake, fake, 4, 1, fake, None, None, fake, None)
    lo = torch.tensor([0, 40], dtype=torch.int64)
    need = L.msa_attention_backward_workspace_size(lay.ref(), 1, 2)
    assert need > 0

    def call(index=dev_idx, B=1, T=2, k=4, q=fake, loff=lo, llen=None, ws_bytes=need):
        return L.msa_sparse_attention_backward(
            lay.ref(), ctypes.byref(index), B, T, q, fake, fake, msa._p(loff),
            None if llen is None else msa._p(llen), fake, k, fake, 64, fake, fake, fake, fake, fake, fake,
            fake, fake, fake, ws_bytes, None)

    assert call(index=host_idx) == 2 and b"device-tier" in L.msa_last_error()
    assert call(B=0) == 2
    assert call(T=0) == 1
    assert call(k=0) == 1 and call(k=11) == 1        # top_k in [1, n_docs]
    assert call(q=None) == 1 and b"missing pointer" in L.msa_last_error()
    assert call(q=odd) == 1 and b"aligned" in L.msa_last_error()
    assert call(loff=torch.tensor([1, 40], dtype=torch.int64)) == 1
    assert call(ws_bytes=need - 1) == 4
    assert call(llen=torch.tensor([1], dtype=torch.int64)) == 1 and b"live length" in L.msa_last_error()
    assert call(llen=torch.tensor([41], dtype=torch.int64)) == 1


def test_route_loss_calls_reject_bad_arguments_before_any_launch():
    """The routing loss's forward and backward check shapes, pointers, tau and
    the workspace on the host; the workspace size depends on B, T and the
    bank's documents and chunks as the plan lays it out."""
    L = msa.lib()
    lay = msa.Layout(32, 8, 128, 128, 64, "bf16")
    fake = ctypes.c_void_p(1 << 20)
    idx = msa._Index(10, 40, fake, None, 4, 0, fake, fake, fake, None, None)
    need = L.msa_route_loss_workspace_size(lay.ref(), ctypes.byref(idx), 2, 3)
    # qinv, u, per-chunk best and token, per-document score, token and chunk, lse
    B, T, Hq, Hkv, dr, C, D = 2, 3, 32, 8, 128, 40, 10
    parts = [4 * B * T * Hq, 4 * B * T * Hkv * dr, 4 * B * C, 4 * B * C, 4 * B * D, 4 * B * D, 8 * B * D, 4 * B * 2]
    assert need >= sum(parts)
    assert L.msa_route_loss_workspace_size(lay.ref(), ctypes.byref(idx), 0, 3) == 0
    wide = msa.Layout(32, 32, 128, 128, 64, "bf16")             # H_kv > 16
    assert L.msa_route_loss_workspace_size(wide.ref(), ctypes.byref(idx), 2, 3) == 0

    def fwd(B=2, T=3, qr=fake, tau=0.1, ws_bytes=need):
        return L.msa_route_loss_forward(lay.ref(), ctypes.byref(idx), B, T, qr, fake, fake, tau, fake, None, fake,
                                        ws_bytes, None)

    def bwd(dqr=fake, tau=0.1, ws_bytes=need):
        return L.msa_route_loss_backward(lay.ref(), ctypes.byref(idx), 2, 3, fake, fake, fake, tau, fake, dqr, fake,
                                         fake, ws_bytes, None)

    assert fwd(B=0) == 1 and fwd(T=0) == 1
    assert fwd(qr=None) == 1 and b"missing pointer" in L.msa_last_error()
    assert fwd(tau=0.0) == 1 and fwd(tau=float("nan")) == 1
    assert fwd(ws_bytes=need - 1) == 4
    assert bwd(dqr=None) == 1 and bwd(tau=-1.0) == 1 and bwd(ws_bytes=need - 1) == 4
    assert L.msa_route_loss_forward(wide.ref(), ctypes.byref(idx), 2, 3, fake, fake, fake, 0.1, fake, None, fake,
                                    need, None) == 2


def _ws(counters, s_tot, Hkv, R, D):
    a = lambda x: (x + 255) // 256 * 256
    return a(4 * counters) + a(4 * s_tot * Hkv * R * D) + a(8 * s_tot * Hkv * R)


def test_decode_plan_runs_a_single_query_in_one_wave():
    """The decode's workspace (counters, partial outputs, partial max/sum per
    split) shows the plan's split count.  Without a GPU the library plans for
    148 SMs.

    CUDA-core kernel (head_dim 64), one query, T = 64: R = 256 rows per kv
    head, 32-row CTAs, 8 row groups, 64 units, two CTAs per SM: 296.  2176
    local keys would take 512-key splits (1 memory + 5 local = 6 splits, 384
    CTAs); the split grows until the grid fits one wave: 768 keys, 1 + 3 = 4
    splits, 256 CTAs.  One token (R = 4, 16-row CTAs, 8 units, one CTA per
    SM): 4097 keys in 256-key splits, 1 + 17 = 18 splits, 144 CTAs, already
    one wave.

    Tensor-core kernel (bf16, head_dim 128, R > 64): 128-row CTAs, 2 row
    groups, 16 units, one CTA per SM.  2176 keys in 256-key splits would be
    1 + 9 = 10 splits, 160 CTAs; 320 keys give 1 + 7 = 8 splits, 128 CTAs."""
    L = msa.lib()
    lay = msa.Layout(32, 8, 64, 128, 64, "bf16")
    lo = torch.tensor([0, 2176], dtype=torch.int64)
    got = L.msa_decode_workspace_size(lay.ref(), 1, 64, msa._p(lo), None)
    assert got == _ws(1 * 8 * 8, 4, 8, 256, 64), got
    assert got != _ws(1 * 8 * 8, 6, 8, 256, 64)
    lo = torch.tensor([0, 4097], dtype=torch.int64)
    assert L.msa_decode_workspace_size(lay.ref(), 1, 1, msa._p(lo), None) == _ws(8, 18, 8, 4, 64)
    lay = msa.Layout(32, 8, 128, 128, 64, "bf16")
    lo = torch.tensor([0, 2176], dtype=torch.int64)
    got = L.msa_decode_workspace_size(lay.ref(), 1, 64, msa._p(lo), None)
    assert got == _ws(1 * 8 * 2, 8, 8, 256, 128), got
    assert got != _ws(1 * 8 * 2, 10, 8, 256, 128)
    lo = torch.tensor([0, 4097], dtype=torch.int64)
    assert L.msa_decode_workspace_size(lay.ref(), 1, 1, msa._p(lo), None) == _ws(8, 18, 8, 4, 128)
