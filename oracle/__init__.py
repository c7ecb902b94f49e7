"""fp64 CPU oracle for Qwen Sparse Attention -- TEST INFRASTRUCTURE ONLY.

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package.  It shares no code with the CUDA library: the
arithmetic lives in ``qsa_oracle.c`` (plain C, fp64, OpenMP over query rows),
compiled here with gcc on first use; this module only marshals arrays.

Every function works on ONE sequence.  Query row ``i`` of a sequence with
``Lq`` queries and ``Lk`` keys sits at position ``t = Lk - Lq + i``.
bf16 inputs are given as torch bf16 tensors or numpy uint16 bit patterns.

The method ("On the Design of Qwen3.8 Next Architecture", reading notes,
section 6, the pooled-key, indexer and budget equations) is written out in
``qsa_oracle.c``; see that file's header for each step's source and for the
readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qsa_oracle.c")
_LIB = os.path.join(_HERE, "libqsa_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library (gcc, -O2, OpenMP, fp64 throughout).

    -ffp-contract=off keeps every multiply and add separately rounded in fp64."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            I = ctypes.c_int
            D = ctypes.c_double
            lib.qsa_oracle_compress.argtypes = [P, I64, I, I, I, D, P]
            lib.qsa_oracle_index_scores.argtypes = [P, P, P, I64, I64, I, I, I, P, I64, P, I64]
            lib.qsa_oracle_select.argtypes = [P, I64, P, I64, I, P]
            lib.qsa_oracle_select_shared.argtypes = [P, I64, P, I64, I, I, I, P]
            lib.qsa_oracle_rope.argtypes = [P, I64, I, P, I, D]
            lib.qsa_oracle_attend.argtypes = [P, P, P, P, I, I64, I64, I, I, I, I, D, P, I64, P, P]
            lib.qsa_oracle_dense.argtypes = [P, P, P, I64, I64, I, I, I, D, P, I64, P, P]
            lib.qsa_oracle_threads.restype = I
            for f in ("qsa_oracle_compress", "qsa_oracle_index_scores", "qsa_oracle_select", "qsa_oracle_select_shared",
                      "qsa_oracle_rope",
                      "qsa_oracle_attend", "qsa_oracle_dense"):
                getattr(lib, f).restype = None
            _lib = lib
    return _lib


def threads() -> int:
    return int(_load().qsa_oracle_threads())


def _bits(x) -> np.ndarray:
    """bf16 tensor or uint16 array -> C-contiguous uint16 bit patterns."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16, x.dtype
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _f64(x) -> np.ndarray:
    if not isinstance(x, np.ndarray):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _f32(x) -> np.ndarray:
    if not isinstance(x, np.ndarray):
        x = x.detach().cpu().float().numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _rows(rows, Lq) -> np.ndarray:
    if rows is None:
        rows = np.arange(Lq, dtype=np.int64)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    assert rows.ndim == 1 and (rows.size == 0 or (rows.min() >= 0 and rows.max() < Lq))
    return rows


def rope(x, pos, rope_dims: int, base: float) -> np.ndarray:
    """Partial RoPE of the last axis of x (fp64 copy): the first rope_dims dims rotate in
    pairs (i, i + rope_dims / 2) by pos * base^(-2i / rope_dims); pos has one entry per
    vector (x reshaped to [n, d])."""
    xv = np.array(x, dtype=np.float64, copy=True)
    d = xv.shape[-1]
    flat = np.ascontiguousarray(xv.reshape(-1, d))
    p = np.ascontiguousarray(np.asarray(pos, dtype=np.int64).reshape(-1))
    assert p.size == flat.shape[0]
    assert rope_dims % 2 == 0 and 0 <= rope_dims <= d
    _load().qsa_oracle_rope(_ptr(flat), flat.shape[0], d, _ptr(p), int(rope_dims), float(base))
    return flat.reshape(xv.shape)


def compress(k_idx, r: int = 4, normalise: bool = True, eps: float = 1e-6, rope_dims: int = 0,
             rope_base: float = 10000.0) -> np.ndarray:
    """kc[b] = RMSNorm(mean of k_idx[b r .. b r + r - 1]) for complete blocks; fp64 [Lk // r, d].
    rope_dims > 0: then the partial RoPE of the pooled key at its block's first position b r."""
    kb = _bits(k_idx)
    Lk, d = kb.shape
    out = np.zeros((Lk // r, d), dtype=np.float64)
    _load().qsa_oracle_compress(_ptr(kb), Lk, r, d, int(normalise), float(eps), _ptr(out))
    if rope_dims > 0:
        out = rope(out, np.arange(out.shape[0], dtype=np.int64) * r, rope_dims, rope_base)
    return out


def index_scores(q_idx, w, kc, Lq: int, Lk: int, r: int = 4, rows=None, ld=None) -> np.ndarray:
    """Indexer scores S[n, b] for query rows ``rows`` (b < b_t; -inf elsewhere); fp64 [nrows, ld]."""
    qb = _bits(q_idx)
    wf = _f32(w)
    kcf = _f64(kc)
    _, H, d = qb.shape
    assert H <= 16 and d <= 256 and kcf.shape[1] == d
    rows = _rows(rows, Lq)
    if ld is None:
        ld = max(1, (Lk - 1) // r + 1)
    out = np.empty((rows.size, ld), dtype=np.float64)
    bt_max = ((Lk - Lq + rows) // r).max() if rows.size else 0
    assert bt_max <= kcf.shape[0] and bt_max <= ld
    _load().qsa_oracle_index_scores(_ptr(qb), _ptr(wf), _ptr(kcf), Lq, Lk, r, H, d,
                                    _ptr(rows), rows.size, _ptr(out), ld)
    return out


def own_blocks(Lq: int, Lk: int, r: int, rows) -> np.ndarray:
    rows = _rows(rows, Lq)
    return ((Lk - Lq + rows) // r).astype(np.int64)


def select(scores, bt, k: int) -> np.ndarray:
    """Own block plus the k-1 best earlier blocks (score desc, index asc); int32 [nrows, k]."""
    s = _f64(scores)
    bt = np.ascontiguousarray(np.asarray(bt, dtype=np.int64))
    assert s.ndim == 2 and bt.shape == (s.shape[0],)
    assert bt.size == 0 or bt.max() <= s.shape[1]
    out = np.empty((s.shape[0], k), dtype=np.int32)
    _load().qsa_oracle_select(_ptr(s), s.shape[1], _ptr(bt), s.shape[0], int(k), _ptr(out))
    return out


def select_shared(scores, lengths, next_n: int, k: int, r: int = 4) -> np.ndarray:
    """One selection per sequence for its next_n queries t = L - next_n .. L - 1, from the
    scores of its last query (row n of scores): the own blocks of all of them forced,
    the rest the best earlier blocks (score desc, index asc); int32 [nrows, k]."""
    s = _f64(scores)
    L = np.ascontiguousarray(np.asarray(lengths, dtype=np.int64))
    assert s.ndim == 2 and L.shape == (s.shape[0],) and next_n >= 1
    assert L.size == 0 or ((L - 1) // r).max() <= s.shape[1]
    out = np.empty((s.shape[0], k), dtype=np.int32)
    _load().qsa_oracle_select_shared(_ptr(s), s.shape[1], _ptr(L), s.shape[0], int(next_n), int(r), int(k),
                                     _ptr(out))
    return out


def attend(q, k, v, sel, Lq: int, Lk: int, r: int = 4, scale: float = 1.0 / 16.0, rows=None):
    """Softmax attention over the selected blocks' tokens (j <= t).  Returns (o, lse) fp64."""
    qb, kb_, vb = _bits(q), _bits(k), _bits(v)
    _, Hq, D = qb.shape
    _, Hkv, D2 = kb_.shape
    assert D == D2 and D <= 1024 and Hq % Hkv == 0
    rows = _rows(rows, Lq)
    sel = np.ascontiguousarray(np.asarray(sel, dtype=np.int32))
    assert sel.shape[0] == rows.size
    o = np.empty((rows.size, Hq, D), dtype=np.float64)
    lse = np.empty((rows.size, Hq), dtype=np.float64)
    _load().qsa_oracle_attend(_ptr(qb), _ptr(kb_), _ptr(vb), _ptr(sel), sel.shape[1], Lq, Lk, r,
                              Hq, Hkv, D, float(scale), _ptr(rows), rows.size, _ptr(o), _ptr(lse))
    return o, lse


def dense(q, k, v, Lq: int, Lk: int, scale: float = 1.0 / 16.0, rows=None):
    """Dense causal GQA attention (query t sees keys 0..t).  Returns (o, lse) fp64."""
    qb, kb_, vb = _bits(q), _bits(k), _bits(v)
    _, Hq, D = qb.shape
    _, Hkv, _ = kb_.shape
    rows = _rows(rows, Lq)
    o = np.empty((rows.size, Hq, D), dtype=np.float64)
    lse = np.empty((rows.size, Hq), dtype=np.float64)
    _load().qsa_oracle_dense(_ptr(qb), _ptr(kb_), _ptr(vb), Lq, Lk, Hq, Hkv, D, float(scale),
                             _ptr(rows), rows.size, _ptr(o), _ptr(lse))
    return o, lse


def qsa_layer(q, k, v, q_idx, k_idx, w, Lq: int, Lk: int, r: int = 4, budget: int = 512,
              scale: float = 1.0 / 16.0, rows=None, normalise: bool = True, eps: float = 1e-6):
    """The whole chain for one sequence: compress -> scores -> select -> attend."""
    rows = _rows(rows, Lq)
    kc = compress(k_idx, r, normalise, eps)
    s = index_scores(q_idx, w, kc, Lq, Lk, r, rows)
    sel = select(s, own_blocks(Lq, Lk, r, rows), budget)
    o, lse = attend(q, k, v, sel, Lq, Lk, r, scale, rows)
    return dict(kc=kc, scores=s, sel=sel, o=o, lse=lse)
