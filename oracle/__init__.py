"""Plain fp64 CPU oracle for the Memory Sparse Attention hot path.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the library under
``routed_sparse_attention_b200`` never does and has no CPU fallback.

The arithmetic lives in ``msa_oracle.c`` (plain C, fp64, no fused
multiply-add, OpenMP only across independent documents / heads); this module
compiles it with gcc on first use and marshals numpy / torch CPU arrays.

Parity status of each function (what pins it is in tests/test_oracle_pins.py):
  rope, chunk_offsets, encode, route, decode, interleave_expand -- pinned
  against closed forms, invariants, brute force and library routines.  The choice of RoPE constants
  (theta = 1e6, rotate-half pairing) and the meaning of the global offset
  ("k" = number of retrieved documents) are readings of silent pages: those
  two choices are parity unpinned against the upstream project, and so is
  the reading of a Memory Interleave round (the set grows by the best
  documents not yet selected), which the pages name but do not define.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.c")
_HDR = os.path.join(_HERE, "msa_oracle.h")
_LIB = os.path.join(_HERE, "libmsa_oracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16 = 0, 1
KV_CHUNK_MAJOR, KV_DOC_INTERLEAVED = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, -ffp-contract=off, OpenMP)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            # MSA_ORACLE_LIB lets the mutation test load a deliberately broken copy
            path = os.environ.get("MSA_ORACLE_LIB") or build()
            L = ctypes.CDLL(path)
            P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
            L.orc_set_threads.argtypes = [I]
            L.orc_get_threads.restype = I
            L.orc_rope.argtypes = [P, I, D, D, P]
            L.orc_chunk_offsets.argtypes = [I64, P, I, P]
            L.orc_chunk_offsets.restype = I64
            L.orc_encode.argtypes = [I64, P, I, I, I, I, D, I, P, P, P, P, P, P]
            L.orc_route.argtypes = [I, I, I, I, I, P, I64, P, I, P, I, P, P, P]
            L.orc_interleave_expand.argtypes = [I, I64, P, I, P, I, P]
            L.orc_decode.argtypes = [I, I, I, I, I, D, I, P, I64, P, I, I, P, P, P, P,
                                     P, P, P]
            _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def storage(x):
    """(contiguous numpy array of raw elements, dtype code) for f32 or bf16 data."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().contiguous().cpu()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float32:
                return x.numpy(), F32
            raise TypeError(f"unsupported storage dtype {x.dtype}")
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"unsupported storage dtype {x.dtype}")


def to_f64(x) -> np.ndarray:
    """Exact fp64 copy of f32 / bf16 / f64 data."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().cpu().to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def threads() -> int:
    return int(lib().orc_get_threads())


def rope(x, pos: float, theta: float) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    if lib().orc_rope(_ptr(x), x.shape[-1], float(pos), float(theta), _ptr(y)) != 0:
        raise ValueError("orc_rope: bad argument")
    return y


def chunk_offsets(doc_tok_off, chunk: int) -> np.ndarray:
    off = np.ascontiguousarray(doc_tok_off, dtype=np.int64)
    out = np.empty_like(off)
    if lib().orc_chunk_offsets(len(off) - 1, _ptr(off), int(chunk), _ptr(out)) < 0:
        raise ValueError("orc_chunk_offsets: bad argument")
    return out


def encode(doc_tok_off, k_tok, v_tok, kr_tok, chunk: int, theta: float):
    """Pooled (K, V, Kr) as fp64 arrays [C][H][dim]."""
    off = np.ascontiguousarray(doc_tok_off, dtype=np.int64)
    k, dt = storage(k_tok)
    v, dt2 = storage(v_tok)
    kr, dt3 = storage(kr_tok)
    assert dt == dt2 == dt3
    n_tok, H, d = k_tok.shape
    dr = kr_tok.shape[2]
    C = int(chunk_offsets(off, chunk)[-1])
    kp = np.empty((C, H, d)); vp = np.empty((C, H, d)); krp = np.empty((C, H, dr))
    rc = lib().orc_encode(len(off) - 1, _ptr(off), H, d, dr, int(chunk), float(theta), dt,
                          _ptr(k), _ptr(v), _ptr(kr), _ptr(kp), _ptr(vp), _ptr(krp))
    if rc != 0:
        raise ValueError(f"orc_encode failed ({rc})")
    return kp, vp, krp


def route(qr, doc_chunk_off, kr_pool, top_k: int, n_kv_heads: int, want_scores=False):
    """(idx [B][k] int32, score [B][k] f64[, doc_score [B][D] f64])."""
    q = np.ascontiguousarray(to_f64(qr))
    B, T, Hq, dr = q.shape
    off = np.ascontiguousarray(doc_chunk_off, dtype=np.int64)
    D = len(off) - 1
    kr, dt = storage(kr_pool)
    idx = np.empty((B, top_k), dtype=np.int32)
    sc = np.empty((B, top_k))
    ds = np.empty((B, D)) if want_scores else None
    rc = lib().orc_route(B, T, Hq, int(n_kv_heads), dr, _ptr(q), D, _ptr(off), dt, _ptr(kr),
                         int(top_k), _ptr(idx), _ptr(sc), _ptr(ds) if ds is not None else None)
    if rc != 0:
        raise ValueError(f"orc_route failed ({rc})")
    return (idx, sc, ds) if want_scores else (idx, sc)


def decode(q, sel, doc_chunk_off, k_pool, v_pool, local_off, local_k, local_v,
           top_k: int, theta: float, n_kv_heads: int,
           kv_layout: int = KV_CHUNK_MAJOR) -> np.ndarray:
    """Decode output [B][T][H_q][d] in fp64."""
    qq = np.ascontiguousarray(to_f64(q))
    B, T, Hq, d = qq.shape
    s = np.ascontiguousarray(sel, dtype=np.int32)
    off = np.ascontiguousarray(doc_chunk_off, dtype=np.int64)
    loff = np.ascontiguousarray(local_off, dtype=np.int64)
    kp, dt = storage(k_pool)
    if kv_layout == KV_DOC_INTERLEAVED:
        vp = kp
    else:
        vp, dt2 = storage(v_pool)
        assert dt2 == dt
    lk, dt3 = storage(local_k)
    lv, dt4 = storage(local_v)
    assert dt3 == dt4 == dt
    out = np.empty((B, T, Hq, d))
    rc = lib().orc_decode(B, T, Hq, int(n_kv_heads), d, float(theta), int(top_k), _ptr(s),
                          len(off) - 1, _ptr(off), dt, int(kv_layout), _ptr(kp), _ptr(vp),
                          _ptr(qq), _ptr(loff), _ptr(lk), _ptr(lv), _ptr(out))
    if rc != 0:
        raise ValueError(f"orc_decode failed ({rc})")
    return out


def interleave_expand(qr, doc_chunk_off, kr_pool, selected, per_round: int, n_kv_heads: int):
    """One Memory Interleave round: route qr, then append to each query's
    selected set (`selected` [B][n] int32, n may be 0) the `per_round`
    best-scoring documents not in it.  Returns the new set [B][n + per_round]."""
    off = np.ascontiguousarray(doc_chunk_off, dtype=np.int64)
    _, _, ds = route(qr, off, kr_pool, 1, n_kv_heads, want_scores=True)
    return interleave_expand_scores(ds, selected, per_round)


def interleave_expand_scores(doc_score, selected, per_round: int):
    """The expansion step alone, from given document scores [B][D]."""
    ds = np.ascontiguousarray(doc_score, dtype=np.float64)
    B, D = ds.shape
    old = np.ascontiguousarray(selected, dtype=np.int32).reshape(B, -1)
    n = old.shape[1]
    new = np.empty((B, n + per_round), dtype=np.int32)
    rc = lib().orc_interleave_expand(B, D, _ptr(ds), n, _ptr(old) if n else None,
                                     int(per_round), _ptr(new))
    if rc != 0:
        raise ValueError(f"orc_interleave_expand failed ({rc})")
    return new
