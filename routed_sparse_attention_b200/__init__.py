"""Python binding of libmsa, the B200 Memory Sparse Attention C-ABI library.

Argument marshalling only: every step of the path runs in the CUDA kernels of
``csrc/``; torch supplies device memory, pinned host memory and streams.  There
is no CPU fallback -- loading fails loudly when the library cannot be built or
found, and calls raise ``MSAError`` on any non-OK status.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

__all__ = ["lib", "MSAError", "Layout", "Index", "chunk_offsets", "rope_table", "encode_memory", "kr_inv_norms",
           "route_workspace_size", "route", "route_noalloc", "route_scores", "fetch_staging_size", "fetch_selected", "fetch_selected_device",
           "decode_workspace_size", "rope_local", "sparse_decode", "sparse_decode_raw_workspace_size", "sparse_decode_raw", "device_status", "version", "ENTRY_POINTS",
           "interleave_expand", "append_local", "append_local_devlen", "sparse_decode_devlen", "advance_local_len",
           "encode_memory_kv_interleaved", "StreamEncoder", "index_save", "index_file_info",
           "index_load", "sparse_attention_forward", "attention_backward_workspace_size",
           "sparse_attention_backward", "route_loss_workspace_size", "route_loss_forward", "route_loss_backward"]

F32, BF16 = 0, 1
DEV_ROPE_RANGE, DEV_BAD_DOC, DEV_PIPE_TIMEOUT, DEV_BAD_SHAPE, DEV_BAD_SET = 1, 2, 4, 8, 16
STATUS = {0: "MSA_OK", 1: "MSA_ERR_INVALID_ARG", 2: "MSA_ERR_UNSUPPORTED", 3: "MSA_ERR_CUDA",
          4: "MSA_ERR_WORKSPACE_TOO_SMALL", 5: "MSA_ERR_TIMEOUT", 6: "MSA_ERR_INTERNAL"}


class MSAError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class _Layout(ctypes.Structure):
    _fields_ = [("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("router_dim", ctypes.c_int32),
                ("chunk_size", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("rope_theta", ctypes.c_double)]


class _Index(ctypes.Structure):
    _fields_ = [("n_docs", ctypes.c_int64), ("n_chunks", ctypes.c_int64),
                ("doc_chunk_off", ctypes.c_void_p), ("doc_chunk_off_host", ctypes.c_void_p),
                ("max_doc_chunks", ctypes.c_int32), ("kv_on_host", ctypes.c_int32),
                ("kr", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("host_kv", ctypes.c_void_p), ("kr_inv_norm", ctypes.c_void_p)]


P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_SIGS = {
    "msa_version": ([], ctypes.c_int),
    "msa_last_error": ([], ctypes.c_char_p),
    "msa_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "msa_device_status": ([P, P], ctypes.c_int),
    "msa_chunk_offsets": ([I64, P, I32, P, P, P], ctypes.c_int),
    "msa_rope_table": ([P, I32, P, P], ctypes.c_int),
    "msa_encode_memory": ([P, I64, I64, P, P, I64, P, P, P, P, I32, P, P, P, P], ctypes.c_int),
    "msa_encode_memory_kv_interleaved": ([P, I64, I64, P, P, I64, P, P, P, P, I32, P, P, P], ctypes.c_int),
    "msa_encoder_create": ([P, I64, I32, I64, I64, P, P, P, P, P], ctypes.c_int),
    "msa_encoder_push": ([P, I32, P, P, P, P], ctypes.c_int),
    "msa_encoder_finish": ([P, P, P, P], ctypes.c_int),
    "msa_encoder_chunk_offsets": ([P, P], ctypes.c_int),
    "msa_encoder_destroy": ([P], None),
    "msa_index_save": ([ctypes.c_char_p, P, P, P], ctypes.c_int),
    "msa_index_file_info": ([ctypes.c_char_p, P, P, P, P, P], ctypes.c_int),
    "msa_index_load": ([ctypes.c_char_p, I32, P, P, P, P, P, P, P], ctypes.c_int),
    "msa_kr_inv_norm_count": ([P, I64], SZ),
    "msa_kr_inv_norms": ([P, P, P, P], ctypes.c_int),
    "msa_route_workspace_size": ([P, I64, I64, I32, I32, I32], SZ),
    "msa_route": ([P, P, I32, I32, P, I32, P, P, P, P, SZ, P], ctypes.c_int),
    "msa_route_noalloc": ([P, P, I32, I32, P, I32, P, P, P, P], ctypes.c_int),
    "msa_route_scores": ([P, P, I32, I32, P, P, P, SZ, P], ctypes.c_int),
    "msa_interleave_expand": ([I64, I32, I32, I32, P, P, P, P, P], ctypes.c_int),
    "msa_fetch_staging_size": ([P, P, I32, I32], SZ),
    "msa_fetch_selected": ([P, P, I32, I32, P, P, I32, P, SZ, P, P], ctypes.c_int),
    "msa_fetch_selected_device": ([P, P, I32, I32, P, P, SZ, P], ctypes.c_int),
    "msa_decode_workspace_size": ([P, I32, I32, P, P], SZ),
    "msa_append_local": ([P, I32, P, P, P, P, I32, P, I32, P, P, P, P], ctypes.c_int),
    "msa_append_local_devlen": ([P, I32, P, P, P, P, I32, P, I32, P, P, P, P], ctypes.c_int),
    "msa_sparse_decode_devlen": ([P, P, I32, I32, P, P, P, P, P, P, I32, P, P, I32, P, P, SZ, P], ctypes.c_int),
    "msa_advance_local_len": ([I32, P, I64, P], ctypes.c_int),
    "msa_rope_local": ([P, I32, P, P, P, I32, P, P, P, I32, P], ctypes.c_int),
    "msa_sparse_decode": ([P, P, I32, I32, P, P, P, P, P, P, I32, P, P, I32, P, P, SZ, P, P],
                          ctypes.c_int),
    "msa_sparse_decode_raw_workspace_size": ([P, P, I32, I32, I32, P, P], SZ),
    "msa_sparse_decode_raw": ([P, P, I32, I32, P, P, P, P, P, P, I32, P, I32, P, P, SZ, P], ctypes.c_int),
    "msa_sparse_attention_forward": ([P, P, I32, I32, P, P, P, P, P, P, I32, P, I32, P, P, P, SZ, P],
                                     ctypes.c_int),
    "msa_attention_backward_workspace_size": ([P, I32, I32], SZ),
    "msa_sparse_attention_backward": ([P, P, I32, I32, P, P, P, P, P, P, I32, P, I32, P, P, P, P, P, P, P, P,
                                       P, SZ, P], ctypes.c_int),
    "msa_route_loss_workspace_size": ([P, P, I32, I32], SZ),
    "msa_route_loss_forward": ([P, P, I32, I32, P, P, P, ctypes.c_float, P, P, P, SZ, P], ctypes.c_int),
    "msa_route_loss_backward": ([P, P, I32, I32, P, P, P, ctypes.c_float, P, P, P, P, SZ, P], ctypes.c_int),
    "msa_debug_fail_next_copies": ([I32], None),
    "msa_debug_expire_wait": ([I64, P, P], ctypes.c_int),
    "msa_debug_scan_events": ([P, P], None),
}
ENTRY_POINTS = tuple(_SIGS)

_lock = threading.Lock()
_lib = None


def lib():
    """The loaded libmsa.so (built in-tree with nvcc for sm_100a if stale)."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            L = ctypes.CDLL(path)
            for name, (args, res) in _SIGS.items():
                f = getattr(L, name)
                f.argtypes = args
                f.restype = res
            _lib = L
    return _lib


def _check(rc: int):
    if rc != 0:
        raise MSAError(rc, lib().msa_last_error().decode())


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return ctypes.c_void_p(t.data_ptr())


def _stream(s=None):
    s = torch.cuda.current_stream() if s is None else s
    return ctypes.c_void_p(s.cuda_stream)


def _event(e):
    return None if e is None else ctypes.c_void_p(e.cuda_event)


def version() -> int:
    return lib().msa_version()


def scan_events(start=None, stop=None):
    """Record start/stop (torch.cuda.Event, already created) around every later
    router-key scan launch on this thread; no arguments turns it off."""
    lib().msa_debug_scan_events(_event(start), _event(stop))


class Layout:
    def __init__(self, n_q_heads, n_kv_heads, head_dim, router_dim, chunk_size, dtype,
                 rope_theta=1.0e6):
        dt = {torch.float32: F32, torch.bfloat16: BF16, "f32": F32, "bf16": BF16}[dtype]
        self.c = _Layout(n_q_heads, n_kv_heads, head_dim, router_dim, chunk_size, dt, rope_theta)
        self.torch_dtype = torch.bfloat16 if dt == BF16 else torch.float32

    @classmethod
    def of(cls, w):
        """Layout of a workloads.Workload."""
        return cls(w.n_q_heads, w.n_kv_heads, w.head_dim, w.router_dim, w.chunk, w.dtype, w.rope_theta)

    def ref(self):
        return ctypes.byref(self.c)


class Index:
    """A pooled memory bank; keeps references to the tensors it points at."""

    def __init__(self, doc_chunk_off_dev, kr, k=None, v=None, host_kv=None,
                 doc_chunk_off_host=None, max_doc_chunks=0, kr_inv_norm=None):
        self._keep = (doc_chunk_off_dev, kr, k, v, host_kv, doc_chunk_off_host, kr_inv_norm)
        n_docs = doc_chunk_off_dev.numel() - 1
        self.c = _Index(n_docs, kr.shape[0], _p(doc_chunk_off_dev), _p(doc_chunk_off_host),
                        int(max_doc_chunks), 1 if host_kv is not None else 0, _p(kr), _p(k), _p(v),
                        _p(host_kv), _p(kr_inv_norm))
        self.n_docs = n_docs

    def ref(self):
        return ctypes.byref(self.c)


def kr_inv_norms(layout: Layout, index: Index, device="cuda", stream=None) -> torch.Tensor:
    """The bank's inverse router-key norms [H_kv][P] (P = n_chunks rounded up to
    128), for Index(kr_inv_norm=...)."""
    n = lib().msa_kr_inv_norm_count(layout.ref(), index.c.n_chunks)
    if n == 0:
        raise MSAError(1, "kr_inv_norm_count: bad layout or bank")
    out = torch.empty(n, dtype=torch.float32, device=device)
    _check(lib().msa_kr_inv_norms(layout.ref(), index.ref(), _p(out), _stream(stream)))
    return out


def debug_expire_wait(limit_us: int, stream=None) -> int:
    """Runs a bounded wait that must time out; returns the threads that gave up."""
    n = ctypes.c_int32(0)
    _check(lib().msa_debug_expire_wait(int(limit_us), ctypes.byref(n), _stream(stream)))
    return n.value


def device_status(stream=None) -> int:
    bits = ctypes.c_uint32(0)
    _check(lib().msa_device_status(ctypes.byref(bits), _stream(stream)))
    return bits.value


def chunk_offsets(doc_tok_off_host: torch.Tensor, chunk: int):
    """(doc_chunk_off int64 host tensor, max_doc_chunks, max_doc_len)."""
    tok = doc_tok_off_host.to(torch.int64).contiguous()
    out = torch.empty_like(tok)
    mx, ml = ctypes.c_int32(0), ctypes.c_int64(0)
    _check(lib().msa_chunk_offsets(tok.numel() - 1, _p(tok), chunk, _p(out), ctypes.byref(mx),
                                   ctypes.byref(ml)))
    return out, mx.value, ml.value


def rope_table(layout: Layout, n_pos: int, device="cuda", stream=None) -> torch.Tensor:
    t = torch.empty(n_pos, layout.c.head_dim // 2, 2, dtype=torch.float32, device=device)
    _check(lib().msa_rope_table(layout.ref(), n_pos, _p(t), _stream(stream)))
    return t


def encode_memory(layout: Layout, doc_tok_off_dev, doc_chunk_off_dev, n_chunks, max_doc_len,
                  k_tok, v_tok, kr_tok, rope, k_pool, v_pool, kr_pool, stream=None):
    _check(lib().msa_encode_memory(layout.ref(), doc_tok_off_dev.numel() - 1, n_chunks,
                                   _p(doc_tok_off_dev), _p(doc_chunk_off_dev), max_doc_len,
                                   _p(k_tok), _p(v_tok), _p(kr_tok), _p(rope), rope.shape[0],
                                   _p(k_pool), _p(v_pool), _p(kr_pool), _stream(stream)))


def encode_memory_kv_interleaved(layout: Layout, doc_tok_off_dev, doc_chunk_off_dev, n_chunks, max_doc_len,
                                 k_tok, v_tok, kr_tok, rope, kv_pool, kr_pool, stream=None):
    _check(lib().msa_encode_memory_kv_interleaved(layout.ref(), doc_tok_off_dev.numel() - 1, n_chunks,
                                                  _p(doc_tok_off_dev), _p(doc_chunk_off_dev), max_doc_len,
                                                  _p(k_tok), _p(v_tok), _p(kr_tok), _p(rope), rope.shape[0],
                                                  _p(kv_pool), _p(kr_pool), _stream(stream)))


class StreamEncoder:
    """msa_encoder_*: a bank encoded batch by batch into given outputs (Kr on
    the device; K/V on the device, or host_kv in pinned memory)."""

    def __init__(self, layout: Layout, max_batch_tokens, max_batch_docs, max_doc_len, capacity_chunks,
                 kr_out, k_out=None, v_out=None, host_kv_out=None):
        self._keep = (kr_out, k_out, v_out, host_kv_out)
        self.h = ctypes.c_void_p()
        _check(lib().msa_encoder_create(layout.ref(), int(max_batch_tokens), int(max_batch_docs), int(max_doc_len),
                                        int(capacity_chunks), _p(kr_out), _p(k_out), _p(v_out), _p(host_kv_out),
                                        ctypes.byref(self.h)))
        self._inputs = [None, None]      # the last two pushes' inputs stay referenced

    def push(self, doc_tok_off_host, k_tok, v_tok, kr_tok):
        tok = doc_tok_off_host.to(torch.int64).contiguous()
        _check(lib().msa_encoder_push(self.h, tok.numel() - 1, _p(tok), _p(k_tok), _p(v_tok), _p(kr_tok)))
        self._inputs = [self._inputs[1], (k_tok, v_tok, kr_tok)]

    def finish(self):
        """Waits for every batch; returns (n_docs, n_chunks, max_doc_chunks, doc_chunk_off host tensor)."""
        nd, nc, mx = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int32()
        _check(lib().msa_encoder_finish(self.h, ctypes.byref(nd), ctypes.byref(nc), ctypes.byref(mx)))
        off = torch.empty(nd.value + 1, dtype=torch.int64)
        _check(lib().msa_encoder_chunk_offsets(self.h, _p(off)))
        self._inputs = [None, None]
        return nd.value, nc.value, mx.value, off

    def close(self):
        if self.h:
            lib().msa_encoder_destroy(self.h)
            self.h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def index_save(path: str, layout: Layout, index: Index, stream=None):
    _check(lib().msa_index_save(os.fsencode(path), layout.ref(), index.ref(), _stream(stream)))


def index_file_info(path: str):
    """(Layout, n_docs, n_chunks, max_doc_chunks, kv_on_host) from an index file's header."""
    c = _Layout()
    nd, nc, mx, host = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
    _check(lib().msa_index_file_info(os.fsencode(path), ctypes.byref(c), ctypes.byref(nd), ctypes.byref(nc),
                                     ctypes.byref(mx), ctypes.byref(host)))
    lay = Layout(c.n_q_heads, c.n_kv_heads, c.head_dim, c.router_dim, c.chunk_size, "bf16" if c.dtype == BF16
                 else "f32", c.rope_theta)
    return lay, nd.value, nc.value, mx.value, bool(host.value)


def index_load(path: str, doc_chunk_off_host, kr, doc_chunk_off_dev=None, k=None, v=None, host_kv=None,
               verify=True, stream=None):
    _check(lib().msa_index_load(os.fsencode(path), 1 if verify else 0, _p(doc_chunk_off_host),
                                _p(doc_chunk_off_dev), _p(kr), _p(k), _p(v), _p(host_kv), _stream(stream)))


def route_workspace_size(layout: Layout, n_docs, n_chunks, batch, T, top_k) -> int:
    return lib().msa_route_workspace_size(layout.ref(), n_docs, n_chunks, batch, T, top_k)


def route(layout: Layout, index: Index, qr, top_k, out_idx, out_score=None, out_idx_host=None,
          ws=None, stream=None):
    B, T = qr.shape[0], qr.shape[1]
    _check(lib().msa_route(layout.ref(), index.ref(), B, T, _p(qr), top_k, _p(out_idx),
                           _p(out_score), _p(out_idx_host), _p(ws),
                           ws.numel() * ws.element_size() if ws is not None else 0,
                           _stream(stream)))


def route_noalloc(layout: Layout, index: Index, qr, top_k, out_idx, out_score=None,
                  out_idx_host=None, stream=None):
    """msa_route without a caller workspace (the library's built-in scratch)."""
    B, T = qr.shape[0], qr.shape[1]
    _check(lib().msa_route_noalloc(layout.ref(), index.ref(), B, T, _p(qr), top_k, _p(out_idx),
                                   _p(out_score), _p(out_idx_host), _stream(stream)))


def route_scores(layout: Layout, index: Index, qr, out, ws, stream=None):
    B, T = qr.shape[0], qr.shape[1]
    _check(lib().msa_route_scores(layout.ref(), index.ref(), B, T, _p(qr), _p(out), _p(ws),
                                  ws.numel() * ws.element_size(), _stream(stream)))


def interleave_expand(n_docs, ranked, sel_old, sel_new, sel_new_host=None, stream=None):
    """One Memory Interleave expansion round: sel_new [B][n + p] = sel_old
    [B][n] followed by the first p documents of `ranked` [B][n + p] (a routing
    for top_k = n + p) that are not in sel_old.  sel_old may be None for n = 0."""
    B, m = ranked.shape
    n = 0 if sel_old is None else sel_old.shape[1]
    _check(lib().msa_interleave_expand(int(n_docs), B, n, m - n, _p(ranked), _p(sel_old), _p(sel_new),
                                       _p(sel_new_host), _stream(stream)))
    return sel_new


def fetch_staging_size(layout: Layout, index: Index, batch, top_k) -> int:
    return lib().msa_fetch_staging_size(layout.ref(), index.ref(), batch, top_k)


def fetch_selected(layout: Layout, index: Index, batch, top_k, sel_host, sel_ready, timeout_ms,
                   staging, fetch_stream, fetch_done=None):
    _check(lib().msa_fetch_selected(layout.ref(), index.ref(), batch, top_k, _p(sel_host),
                                    _event(sel_ready), timeout_ms, _p(staging),
                                    staging.numel() * staging.element_size(),
                                    _stream(fetch_stream), _event(fetch_done)))


def fetch_selected_device(layout: Layout, index: Index, batch, top_k, sel_idx, staging, stream=None):
    """Host-tier fetch by one kernel reading the device selection (no host wait)."""
    _check(lib().msa_fetch_selected_device(layout.ref(), index.ref(), batch, top_k, _p(sel_idx), _p(staging),
                                           staging.numel() * staging.element_size(), _stream(stream)))


def _opt_i64(t):
    """Host int64 tensor from a tensor, numpy array or sequence (None stays None)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        t = torch.as_tensor(t)
    return t.to(torch.int64).contiguous()


def decode_workspace_size(layout: Layout, batch, T, local_off_host, local_len_host=None) -> int:
    lo, ll = _opt_i64(local_off_host), _opt_i64(local_len_host)
    return lib().msa_decode_workspace_size(layout.ref(), batch, T, _p(lo), _p(ll))


def rope_local(layout: Layout, local_off_host, top_k, src, dst, rope, first_host=None, stream=None,
               local_len_host=None):
    """Global RoPE of local keys: live rows first_host[b] <= j < len_b of query b
    become RoPE(src row, top_k + j); per query [H_kv][capacity][head_dim]."""
    lo, ll, fi = _opt_i64(local_off_host), _opt_i64(local_len_host), _opt_i64(first_host)
    _check(lib().msa_rope_local(layout.ref(), lo.numel() - 1, _p(lo), _p(ll), _p(fi), top_k, _p(src), _p(dst),
                                _p(rope), rope.shape[0], _stream(stream)))
    return dst


def append_local(layout: Layout, local_off_host, local_len_host, k_new, v_new, top_k, rope, k_rot, v,
                 k_raw=None, stream=None):
    """One token per query into the local cache at the live lengths (host
    int64, before the append): value, raw key (optional), rotated key."""
    B = k_new.shape[0]
    if not (k_new.is_contiguous() and v_new.is_contiguous()):
        raise ValueError("append_local: k_new and v_new must be contiguous [B][H_kv][d]")
    lo, ll = _opt_i64(local_off_host), _opt_i64(local_len_host)
    _check(lib().msa_append_local(layout.ref(), B, _p(lo), _p(ll), _p(k_new), _p(v_new), top_k, _p(rope),
                                  rope.shape[0], _p(k_raw), _p(k_rot), _p(v), _stream(stream)))


def append_local_devlen(layout: Layout, local_off_host, local_len_dev, k_new, v_new, top_k, rope, k_rot, v,
                        k_raw=None, stream=None):
    """append_local with the live lengths in device memory (int64 [B])."""
    B = k_new.shape[0]
    if not (k_new.is_contiguous() and v_new.is_contiguous()):
        raise ValueError("append_local: k_new and v_new must be contiguous [B][H_kv][d]")
    lo = _opt_i64(local_off_host)
    _check(lib().msa_append_local_devlen(layout.ref(), B, _p(lo), _p(local_len_dev), _p(k_new), _p(v_new), top_k,
                                         _p(rope), rope.shape[0], _p(k_raw), _p(k_rot), _p(v), _stream(stream)))


def sparse_decode_devlen(layout: Layout, index: Index, q, local_k, local_v, local_off_host, local_len_dev, sel_idx,
                         top_k, rope, out, ws, mem_staging=None, stream=None):
    """sparse_decode with the live lengths in device memory (int64 [B]),
    planned for the capacities: launch parameters stay fixed across tokens."""
    B, T = q.shape[0], q.shape[1]
    lo = _opt_i64(local_off_host)
    _check(lib().msa_sparse_decode_devlen(layout.ref(), index.ref(), B, T, _p(q), _p(local_k), _p(local_v), _p(lo),
                                          _p(local_len_dev), _p(sel_idx), top_k, _p(mem_staging), _p(rope),
                                          rope.shape[0], _p(out), _p(ws), ws.numel() * ws.element_size(),
                                          _stream(stream)))


def advance_local_len(local_len_dev, by=1, stream=None):
    _check(lib().msa_advance_local_len(local_len_dev.numel(), _p(local_len_dev), int(by), _stream(stream)))


def sparse_decode(layout: Layout, index: Index, q, local_k, local_v, local_off_host, sel_idx,
                  top_k, rope, out, ws, mem_staging=None, wait_event=None, stream=None,
                  local_len_host=None):
    B, T = q.shape[0], q.shape[1]
    lo, ll = _opt_i64(local_off_host), _opt_i64(local_len_host)
    _check(lib().msa_sparse_decode(layout.ref(), index.ref(), B, T, _p(q), _p(local_k), _p(local_v),
                                   _p(lo), _p(ll), _p(sel_idx), top_k, _p(mem_staging), _p(rope),
                                   rope.shape[0], _p(out), _p(ws), ws.numel() * ws.element_size(),
                                   _event(wait_event), _stream(stream)))


def sparse_decode_raw_workspace_size(layout: Layout, index: Index, batch, T, top_k, local_off_host,
                                     local_len_host=None) -> int:
    lo, ll = _opt_i64(local_off_host), _opt_i64(local_len_host)
    return lib().msa_sparse_decode_raw_workspace_size(layout.ref(), index.ref(), batch, T, top_k, _p(lo), _p(ll))


def sparse_decode_raw(layout: Layout, index: Index, q, local_k_raw, local_v, local_off_host, sel_idx, top_k, rope,
                      out, ws, stream=None, local_len_host=None):
    """Stage 3 in one call from unrotated local keys (rotation and, for the
    host tier, the fetch inside the call); ws zero-filled before first use."""
    B, T = q.shape[0], q.shape[1]
    lo, ll = _opt_i64(local_off_host), _opt_i64(local_len_host)
    _check(lib().msa_sparse_decode_raw(layout.ref(), index.ref(), B, T, _p(q), _p(local_k_raw), _p(local_v),
                                       _p(lo), _p(ll), _p(sel_idx), top_k, _p(rope), rope.shape[0], _p(out), _p(ws),
                                       ws.numel() * ws.element_size(), _stream(stream)))
    return out


# ------------------------------------------------------------ training layer

def sparse_attention_forward(layout: Layout, index: Index, q, local_k, local_v, local_off_host, sel_idx, top_k,
                             rope, out, lse, ws, stream=None, local_len_host=None):
    B, T = q.shape[0], q.shape[1]
    lo, ll = _opt_i64(local_off_host), _opt_i64(local_len_host)
    _check(lib().msa_sparse_attention_forward(layout.ref(), index.ref(), B, T, _p(q), _p(local_k), _p(local_v),
                                              _p(lo), _p(ll), _p(sel_idx), top_k, _p(rope), rope.shape[0],
                                              _p(out), _p(lse), _p(ws), ws.numel() * ws.element_size(),
                                              _stream(stream)))


def attention_backward_workspace_size(layout: Layout, batch, T) -> int:
    return lib().msa_attention_backward_workspace_size(layout.ref(), batch, T)


def sparse_attention_backward(layout: Layout, index: Index, q, local_k, local_v, local_off_host, sel_idx, top_k,
                              rope, out, lse, dout, d_q, d_mem_k, d_mem_v, d_local_k, d_local_v, ws, stream=None,
                              local_len_host=None):
    B, T = q.shape[0], q.shape[1]
    lo, ll = _opt_i64(local_off_host), _opt_i64(local_len_host)
    _check(lib().msa_sparse_attention_backward(layout.ref(), index.ref(), B, T, _p(q), _p(local_k), _p(local_v),
                                               _p(lo), _p(ll), _p(sel_idx), top_k, _p(rope), rope.shape[0],
                                               _p(out), _p(lse), _p(dout), _p(d_q), _p(d_mem_k), _p(d_mem_v),
                                               _p(d_local_k), _p(d_local_v), _p(ws),
                                               ws.numel() * ws.element_size(), _stream(stream)))


def route_loss_workspace_size(layout: Layout, index: Index, batch, T) -> int:
    return lib().msa_route_loss_workspace_size(layout.ref(), index.ref(), batch, T)


def route_loss_forward(layout: Layout, index: Index, qr, pos_off, pos_doc, tau, loss, ws, doc_score=None,
                       stream=None):
    B, T = qr.shape[0], qr.shape[1]
    _check(lib().msa_route_loss_forward(layout.ref(), index.ref(), B, T, _p(qr), _p(pos_off), _p(pos_doc),
                                        float(tau), _p(loss), _p(doc_score), _p(ws),
                                        ws.numel() * ws.element_size(), _stream(stream)))


def route_loss_backward(layout: Layout, index: Index, qr, pos_off, pos_doc, tau, d_loss, d_qr, d_kr, ws,
                        stream=None):
    B, T = qr.shape[0], qr.shape[1]
    _check(lib().msa_route_loss_backward(layout.ref(), index.ref(), B, T, _p(qr), _p(pos_off), _p(pos_doc),
                                         float(tau), _p(d_loss), _p(d_qr), _p(d_kr), _p(ws),
                                         ws.numel() * ws.element_size(), _stream(stream)))
