"""Python binding of libqsa.so (the C ABI declared in include/qsa.h).

Argument marshalling only: every step of the QSA path runs in the library's
CUDA kernels.  torch supplies device memory and the current stream.  If the
shared library is missing this module raises at import time -- there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# QSA_DEBUG_BUILD=1 loads the QSA_DEBUG_CHECKS build (short waits, fault injection)
LIB_PATH = os.path.join(_HERE, "libqsa_debug.so" if os.environ.get("QSA_DEBUG_BUILD") == "1" else "libqsa.so")

QSA_OK = 0
QSA_ERR_INVALID_ARG = 1
QSA_ERR_UNSUPPORTED = 2
QSA_ERR_WORKSPACE_TOO_SMALL = 3
QSA_ERR_CUDA = 4
QSA_ERR_TIMEOUT = 5
QSA_ERR_DEVICE_CHECK = 6
QSA_ERR_SCRATCH_LIMIT = 7
STATIC_SCRATCH_BYTES = 16 * 1024 * 1024  # QSA_STATIC_SCRATCH_BYTES
QSA_COMPRESS_NO_NORM = 0x1
QSA_INDEX_ROPE = 0x2
(OP_COMPRESS, OP_INDEX, OP_SELECT, OP_PREFILL, OP_DECODE, OP_DENSE, OP_DECODE_PAGED, OP_INDEX_SELECT,
 OP_INDEX_SELECT_PAGED, OP_DECODE_MTP) = range(10)

EXPORTED = (
    "qsa_config_init", "qsa_compress_keys", "qsa_index_scores", "qsa_select_blocks", "qsa_index_select",
    "qsa_sparse_attn_prefill", "qsa_sparse_attn_decode", "qsa_sparse_attn_decode_paged",
    "qsa_sparse_attn_decode_static_scratch", "qsa_compress_keys_paged", "qsa_index_select_paged",
    "qsa_index_select_mtp", "qsa_sparse_attn_decode_mtp",
    "qsa_dense_attn_prefill",
    "qsa_workspace_size", "qsa_status_string", "qsa_get_device_status", "qsa_version", "qsa_debug_inject",
    "qsa_rope_queries", "qsa_sparse_attn_decode_window", "qsa_merge_attn_states",
)


class Config(ctypes.Structure):
    _fields_ = [
        ("r", ctypes.c_int32),
        ("budget_blocks", ctypes.c_int32),
        ("n_heads_q", ctypes.c_int32),
        ("n_heads_kv", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("n_heads_idx", ctypes.c_int32),
        ("idx_dim", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
        ("rms_eps", ctypes.c_float),
        ("flags", ctypes.c_uint32),
        ("kv_chunk_blocks", ctypes.c_int32),
        ("rope_dims", ctypes.c_int32),
        ("rope_base", ctypes.c_float),
    ]


class QSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s" % (where, _lib.qsa_status_string(status).decode()))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("%s is not built (python -m block_sparse_long_09_b200.build --all)"
                          % os.path.basename(LIB_PATH))
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    CP = ctypes.POINTER(Config)
    sig = {
        "qsa_config_init": (None, [CP]),
        "qsa_compress_keys": (I32, [CP, P, P, P, I32, I64, P, I32, P, P]),
        "qsa_index_scores": (I32, [CP, P, P, P, I64, P, P, P, I32, I64, I32, I64, I64, P, I64, P, SZ, P]),
        "qsa_select_blocks": (I32, [CP, P, I64, P, P, I32, I64, I64, P, P, SZ, P]),
        "qsa_index_select": (I32, [CP, P, P, P, I64, P, P, P, I32, I64, I32, I64, I64, I64, P, P, SZ, P]),
        "qsa_compress_keys_paged": (I32, [CP, P, P, I64, I32, P, I32, P, I32, I64, P, I32, P]),
        "qsa_index_select_paged": (I32, [CP, P, P, P, I64, I32, P, I32, P, I32, I64, P, P, SZ, P]),
        "qsa_index_select_mtp": (I32, [CP, P, P, P, I64, P, P, I32, I32, I64, P, P, SZ, P]),
        "qsa_sparse_attn_decode_mtp": (I32, [CP, P, P, P, P, I32, I64, I32, P, P, P, P, SZ, P]),
        "qsa_sparse_attn_prefill": (I32, [CP, P, P, P, P, P, P, I32, I64, I64, I64, I64, I64, P, P, P, SZ, P]),
        "qsa_sparse_attn_decode": (I32, [CP, P, P, P, P, I32, I64, P, P, P, P, SZ, P]),
        "qsa_sparse_attn_decode_static_scratch": (I32, [CP, P, P, P, P, I32, I64, P, P, P, P]),
        "qsa_sparse_attn_decode_paged": (I32, [CP, P, P, P, I64, I32, P, I32, P, I32, P, P, P, P, SZ, P]),
        "qsa_dense_attn_prefill": (I32, [CP, P, P, P, P, P, I32, I64, I64, I32, I64, P, P, P, SZ, P]),
        "qsa_workspace_size": (SZ, [CP, I32, I32, I64, I64]),
        "qsa_status_string": (ctypes.c_char_p, [I32]),
        "qsa_get_device_status": (I32, [P, ctypes.POINTER(I32), I32]),
        "qsa_version": (I32, []),
        "qsa_debug_inject": (I32, [I32]),
        "qsa_rope_queries": (I32, [CP, P, P, P, I32, I64, P]),
        "qsa_sparse_attn_decode_window": (I32, [CP, P, P, P, P, I32, I64, P, P, P, P, P, P, P, SZ, P]),
        "qsa_merge_attn_states": (I32, [CP, P, P, I32, I64, P, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()


def library() -> ctypes.CDLL:
    return _lib


def default_config(**overrides) -> Config:
    c = Config()
    _lib.qsa_config_init(ctypes.byref(c))
    for k, v in overrides.items():
        setattr(c, k, v)
    return c


def _check(status: int, where: str):
    if status != QSA_OK:
        raise QSAError(status, where)


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "tensors must be contiguous CUDA tensors"
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _cfg(cfg: Optional[Config]) -> Config:
    return cfg if cfg is not None else default_config()


def _check_sel(sel, rows: int, cfg: Config):
    """A selection buffer must be int32 [>= rows, budget_blocks], contiguous: the kernels
    address row i at sel + i * budget_blocks and cannot see the tensor's extent."""
    if sel.dtype != torch.int32 or sel.dim() != 2 or not sel.is_contiguous():
        raise ValueError("sel must be a contiguous int32 [rows, budget_blocks] tensor")
    if sel.shape[1] != cfg.budget_blocks or sel.shape[0] < rows:
        raise ValueError("sel is %s; the call needs [>= %d, %d] (cfg.budget_blocks)"
                         % (tuple(sel.shape), rows, cfg.budget_blocks))


def workspace_size(op: int, batch: int, rows: int = 0, max_len_k: int = 0, cfg: Optional[Config] = None) -> int:
    return int(_lib.qsa_workspace_size(ctypes.byref(_cfg(cfg)), op, batch, rows, max_len_k))


def device_status(clear: bool = True) -> int:
    st = ctypes.c_int32(0)
    _check(_lib.qsa_get_device_status(_stream(), ctypes.byref(st), 1 if clear else 0), "qsa_get_device_status")
    return int(st.value)


def compress_keys(k_idx, cu_seqlens_k, cu_blocks, kc=None, blk_begin=None, max_new_blocks: int = 0,
                  cfg: Optional[Config] = None, n_blocks: Optional[int] = None):
    """kc[b] = RMSNorm(mean of the r indexer keys of block b) for every complete block,
    stored as a compensated bf16 pair: kc has shape [n_blocks, 2, idx_dim] (hi, lo)."""
    cfg = _cfg(cfg)
    batch = cu_seqlens_k.numel() - 1
    if kc is None:
        if n_blocks is None:
            n_blocks = int(cu_blocks[-1].item())
        kc = torch.empty((n_blocks, 2, cfg.idx_dim), dtype=torch.bfloat16, device=k_idx.device)
    _check(_lib.qsa_compress_keys(ctypes.byref(cfg), _p(k_idx), _p(cu_seqlens_k), _p(cu_blocks), batch,
                                  k_idx.shape[0], _p(blk_begin), max_new_blocks, _p(kc), _stream()),
           "qsa_compress_keys")
    return kc


def rope_queries(q_idx, cu_seqlens_q, cu_seqlens_k, cfg: Optional[Config] = None):
    """Partial RoPE of the indexer queries in place (q_idx [total_q, 4, 128] bf16), each row
    at its position t; cfg must carry QSA_INDEX_ROPE (the pooled keys rotate the same way)."""
    cfg = _cfg(cfg)
    _check(_lib.qsa_rope_queries(ctypes.byref(cfg), _p(q_idx), _p(cu_seqlens_q), _p(cu_seqlens_k),
                                 cu_seqlens_q.numel() - 1, q_idx.shape[0], _stream()),
           "qsa_rope_queries")
    return q_idx


def index_scores(q_idx, w, kc, cu_seqlens_q, cu_seqlens_k, cu_blocks, max_len_q: int, ld: int,
                 row_begin: int = 0, row_end: Optional[int] = None, scores=None, cfg: Optional[Config] = None):
    """Indexer scores for packed query rows [row_begin, row_end); row i at scores[i - row_begin]."""
    cfg = _cfg(cfg)
    total_q = q_idx.shape[0]
    if row_end is None:
        row_end = total_q
    if scores is None:
        scores = torch.empty((max(row_end - row_begin, 1), ld), dtype=torch.float32, device=q_idx.device)
    assert scores.shape[1] == ld
    _check(_lib.qsa_index_scores(ctypes.byref(cfg), _p(q_idx), _p(w), _p(kc), kc.shape[0], _p(cu_seqlens_q),
                                 _p(cu_seqlens_k), _p(cu_blocks), cu_seqlens_q.numel() - 1, total_q, max_len_q,
                                 row_begin, row_end, _p(scores), ld, None, 0, _stream()),
           "qsa_index_scores")
    return scores


def index_select(q_idx, w, kc, cu_seqlens_q, cu_seqlens_k, cu_blocks, max_len_q: int, max_len_k: int,
                 row_begin: int = 0, row_end: Optional[int] = None, sel=None, ws=None, cfg: Optional[Config] = None):
    """Indexer + top-k selection for packed rows [row_begin, row_end) without writing the
    rows' full score rows (qsa_index_select); sel[i] for those rows."""
    cfg = _cfg(cfg)
    total_q = q_idx.shape[0]
    if row_end is None:
        row_end = total_q
    if sel is None:
        sel = torch.empty((total_q, cfg.budget_blocks), dtype=torch.int32, device=q_idx.device)
    batch = cu_seqlens_q.numel() - 1
    need = workspace_size(OP_INDEX_SELECT, batch, row_end - row_begin, max_len_k, cfg)
    if ws is None:
        ws = torch.empty((max(need, 16),), dtype=torch.uint8, device=q_idx.device)
    _check_sel(sel, row_end, cfg)
    _check(_lib.qsa_index_select(ctypes.byref(cfg), _p(q_idx), _p(w), _p(kc), kc.shape[0], _p(cu_seqlens_q),
                                 _p(cu_seqlens_k), _p(cu_blocks), batch, total_q, max_len_q, max_len_k, row_begin,
                                 row_end, _p(sel), _p(ws), ws.numel(), _stream()),
           "qsa_index_select")
    return sel


def compress_keys_paged(k_idx_pages, kc_pages, block_table, cu_seqlens_k, max_len_k: int, blk_begin=None,
                        max_new_blocks: int = 0, cfg: Optional[Config] = None):
    """Compressed keys of a paged cache: k_idx_pages [num_pages, page_size, 128] bf16 ->
    kc_pages [num_pages, page_size / r, 2, 128] bf16 (hi, lo), through block_table
    [batch, max_pages]."""
    cfg = _cfg(cfg)
    num_pages, page_size = k_idx_pages.shape[0], k_idx_pages.shape[1]
    _check(_lib.qsa_compress_keys_paged(ctypes.byref(cfg), _p(k_idx_pages), _p(kc_pages), num_pages, page_size,
                                        _p(block_table), block_table.shape[1], _p(cu_seqlens_k),
                                        cu_seqlens_k.numel() - 1, max_len_k, _p(blk_begin), max_new_blocks,
                                        _stream()),
           "qsa_compress_keys_paged")
    return kc_pages


def index_select_paged(q_idx, w, kc_pages, page_size: int, block_table, cu_seqlens_k, max_len_k: int, sel=None,
                       ws=None, cfg: Optional[Config] = None):
    """Decode indexer + top-k over a paged kc cache (one query per sequence)."""
    cfg = _cfg(cfg)
    batch = q_idx.shape[0]
    if sel is None:
        sel = torch.empty((batch, cfg.budget_blocks), dtype=torch.int32, device=q_idx.device)
    if ws is None:
        ws = torch.empty((max(workspace_size(OP_INDEX_SELECT_PAGED, batch, batch, max_len_k, cfg), 16),),
                         dtype=torch.uint8, device=q_idx.device)
    _check_sel(sel, batch, cfg)
    _check(_lib.qsa_index_select_paged(ctypes.byref(cfg), _p(q_idx), _p(w), _p(kc_pages), kc_pages.shape[0],
                                       page_size, _p(block_table), block_table.shape[1], _p(cu_seqlens_k), batch,
                                       max_len_k, _p(sel), _p(ws), ws.numel(), _stream()),
           "qsa_index_select_paged")
    return sel


def index_select_mtp(q_idx, w, kc, cu_seqlens_k, cu_blocks, next_n: int, max_len_k: int, sel=None, ws=None,
                     cfg: Optional[Config] = None):
    """The shared selection of a multi-token decode step: one per sequence, from the
    scores of its last query (q_idx [batch, 4, 128], w [batch, 4]), every query's own
    block kept; sel [batch, k]."""
    cfg = _cfg(cfg)
    batch = cu_seqlens_k.numel() - 1
    if sel is None:
        sel = torch.empty((batch, cfg.budget_blocks), dtype=torch.int32, device=q_idx.device)
    if ws is None:
        ws = torch.empty((max(workspace_size(OP_INDEX_SELECT, batch, batch, max_len_k, cfg), 16),),
                         dtype=torch.uint8, device=q_idx.device)
    _check_sel(sel, batch, cfg)
    _check(_lib.qsa_index_select_mtp(ctypes.byref(cfg), _p(q_idx), _p(w), _p(kc), kc.shape[0], _p(cu_seqlens_k),
                                     _p(cu_blocks), batch, next_n, max_len_k, _p(sel), _p(ws), ws.numel(),
                                     _stream()),
           "qsa_index_select_mtp")
    return sel


def sparse_attn_decode_mtp(q, k_cache, v_cache, cu_seqlens_k, sel, o=None, lse=None, ws=None,
                           want_lse: bool = False, cfg: Optional[Config] = None):
    """Attention of next_n queries per sequence (q [batch, next_n, 24, 256]) over one
    shared selection per sequence, each query cut to its own tokens."""
    cfg = _cfg(cfg)
    batch, next_n = q.shape[0], q.shape[1]
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((batch, next_n, cfg.n_heads_q), dtype=torch.float32, device=q.device)
    need = workspace_size(OP_DECODE_MTP, batch, batch, 0, cfg)
    if ws is None and need > 0:
        ws = torch.empty((need,), dtype=torch.uint8, device=q.device)
    _check_sel(sel, batch, cfg)
    _check(_lib.qsa_sparse_attn_decode_mtp(ctypes.byref(cfg), _p(q), _p(k_cache), _p(v_cache), _p(cu_seqlens_k),
                                           batch, k_cache.shape[0], next_n, _p(sel), _p(o), _p(lse), _p(ws),
                                           ws.numel() if ws is not None else 0, _stream()),
           "qsa_sparse_attn_decode_mtp")
    return (o, lse) if want_lse or lse is not None else o


def select_blocks(scores, cu_seqlens_q, cu_seqlens_k, total_q: int, row_begin: int = 0,
                  row_end: Optional[int] = None, sel=None, cfg: Optional[Config] = None):
    """Own block + best k-1 earlier blocks per row; sel[i] for packed rows i in [row_begin, row_end)."""
    cfg = _cfg(cfg)
    if row_end is None:
        row_end = total_q
    if sel is None:
        sel = torch.empty((total_q, cfg.budget_blocks), dtype=torch.int32, device=scores.device)
    _check_sel(sel, row_end, cfg)
    _check(_lib.qsa_select_blocks(ctypes.byref(cfg), _p(scores), scores.shape[1], _p(cu_seqlens_q),
                                  _p(cu_seqlens_k), cu_seqlens_q.numel() - 1, row_begin, row_end, _p(sel),
                                  None, 0, _stream()),
           "qsa_select_blocks")
    return sel


def sparse_attn_prefill(q, k, v, sel, cu_seqlens_q, cu_seqlens_k, row_begin: int = 0,
                        row_end: Optional[int] = None, o=None, lse=None, want_lse: bool = False,
                        cfg: Optional[Config] = None, ws=None, max_len_k: Optional[int] = None):
    """Sparse attention over the selected blocks.  With a workspace (allocated here
    when ws is None) long contexts run the L2-blocked key-chunk schedule."""
    cfg = _cfg(cfg)
    total_q = q.shape[0]
    if row_end is None:
        row_end = total_q
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((total_q, cfg.n_heads_q), dtype=torch.float32, device=q.device)
    if max_len_k is None:
        max_len_k = int((cu_seqlens_k[1:] - cu_seqlens_k[:-1]).max().item())
    batch = cu_seqlens_q.numel() - 1
    need = workspace_size(OP_PREFILL, batch, row_end - row_begin, max_len_k, cfg)
    if ws is None and need > 0:
        ws = torch.empty((need,), dtype=torch.uint8, device=q.device)
    _check_sel(sel, row_end, cfg)
    _check(_lib.qsa_sparse_attn_prefill(ctypes.byref(cfg), _p(q), _p(k), _p(v), _p(sel), _p(cu_seqlens_q),
                                        _p(cu_seqlens_k), batch, total_q, k.shape[0], max_len_k, row_begin, row_end,
                                        _p(o), _p(lse), _p(ws), ws.numel() if ws is not None else 0, _stream()),
           "qsa_sparse_attn_prefill")
    return (o, lse) if want_lse or lse is not None else o


def sparse_attn_decode(q, k_cache, v_cache, cu_seqlens_k, sel, o=None, lse=None, ws=None, want_lse: bool = False,
                       cfg: Optional[Config] = None):
    cfg = _cfg(cfg)
    batch = q.shape[0]
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((batch, cfg.n_heads_q), dtype=torch.float32, device=q.device)
    need = workspace_size(OP_DECODE, batch, batch, 0, cfg)
    if ws is None and need > 0:
        ws = torch.empty((need,), dtype=torch.uint8, device=q.device)
    _check_sel(sel, batch, cfg)
    _check(_lib.qsa_sparse_attn_decode(ctypes.byref(cfg), _p(q), _p(k_cache), _p(v_cache), _p(cu_seqlens_k),
                                       batch, k_cache.shape[0], _p(sel), _p(o), _p(lse), _p(ws),
                                       ws.numel() if ws is not None else 0, _stream()),
           "qsa_sparse_attn_decode")
    return (o, lse) if want_lse or lse is not None else o


def sparse_attn_decode_paged(q, k_pages, v_pages, block_table, cu_seqlens_k, sel, o=None, lse=None, ws=None,
                             want_lse: bool = False, cfg: Optional[Config] = None):
    """Decode attention over a paged K/V pool [num_pages, page_size, 2, 256] with a
    block table [batch, max_pages]; cu_seqlens_k gives the sequence lengths."""
    cfg = _cfg(cfg)
    batch = q.shape[0]
    num_pages, page_size = k_pages.shape[0], k_pages.shape[1]
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((batch, cfg.n_heads_q), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = torch.empty((workspace_size(OP_DECODE_PAGED, batch, batch, 0, cfg),), dtype=torch.uint8, device=q.device)
    _check_sel(sel, batch, cfg)
    _check(_lib.qsa_sparse_attn_decode_paged(ctypes.byref(cfg), _p(q), _p(k_pages), _p(v_pages), num_pages, page_size,
                                             _p(block_table), block_table.shape[1], _p(cu_seqlens_k), batch, _p(sel),
                                             _p(o), _p(lse), _p(ws), ws.numel(), _stream()),
           "qsa_sparse_attn_decode_paged")
    return (o, lse) if want_lse or lse is not None else o


def sparse_attn_decode_window(q, k_local, v_local, cu_seqlens_k, tok_local, blk_lo, blk_hi, sel, o=None, lse=None,
                              ws=None, cfg: Optional[Config] = None):
    """One context-parallel shard's decode attention: the selected blocks inside
    [blk_lo[s], blk_hi[s]) of each sequence, whose tokens sit in k_local / v_local from
    row tok_local[s] on; cu_seqlens_k holds the global lengths.  Returns the partial
    (o, lse) for qsa_merge_attn_states."""
    cfg = _cfg(cfg)
    batch = q.shape[0]
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((batch, cfg.n_heads_q), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = torch.empty((workspace_size(OP_DECODE_PAGED, batch, batch, 0, cfg),), dtype=torch.uint8,
                         device=q.device)
    _check_sel(sel, batch, cfg)
    _check(_lib.qsa_sparse_attn_decode_window(ctypes.byref(cfg), _p(q), _p(k_local), _p(v_local), _p(cu_seqlens_k),
                                              batch, k_local.shape[0], _p(tok_local), _p(blk_lo), _p(blk_hi),
                                              _p(sel), _p(o), _p(lse), _p(ws), ws.numel(), _stream()),
           "qsa_sparse_attn_decode_window")
    return o, lse


def merge_attn_states(o_parts, lse_parts, o=None, lse=None, cfg: Optional[Config] = None):
    """o, lse of rows from the partial states of several shards: o_parts [P, rows, 24, 256]
    bf16, lse_parts [P, rows, 24] fp32."""
    cfg = _cfg(cfg)
    parts, rows = o_parts.shape[0], o_parts.shape[1]
    if o is None:
        o = torch.empty(o_parts.shape[1:], dtype=o_parts.dtype, device=o_parts.device)
    if lse is None:
        lse = torch.empty(lse_parts.shape[1:], dtype=torch.float32, device=o_parts.device)
    _check(_lib.qsa_merge_attn_states(ctypes.byref(cfg), _p(o_parts), _p(lse_parts), parts, rows, _p(o), _p(lse),
                                      _stream()),
           "qsa_merge_attn_states")
    return o, lse


def sparse_attn_decode_static_scratch(q, k_cache, v_cache, cu_seqlens_k, sel, o, lse=None,
                                      cfg: Optional[Config] = None):
    """Decode attention into the caller's `o` (and `lse`), using the library's fixed
    device scratch: neither this wrapper nor the call allocates device memory.
    Calls that overlap on the GPU share that scratch and race."""
    cfg = _cfg(cfg)
    _check_sel(sel, q.shape[0], cfg)
    _check(_lib.qsa_sparse_attn_decode_static_scratch(ctypes.byref(cfg), _p(q), _p(k_cache), _p(v_cache),
                                                      _p(cu_seqlens_k), q.shape[0], k_cache.shape[0], _p(sel),
                                                      _p(o), _p(lse), _stream()),
           "qsa_sparse_attn_decode_static_scratch")
    return o


def dense_attn_prefill(q, k, v, cu_seqlens_q, cu_seqlens_k, max_len_q: int, o=None, lse=None,
                       want_lse: bool = False, cfg: Optional[Config] = None, max_len_k: Optional[int] = None,
                       ws=None):
    """Dense causal attention; max_len_q == 1 runs split-K flash decoding."""
    cfg = _cfg(cfg)
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((q.shape[0], cfg.n_heads_q), dtype=torch.float32, device=q.device)
    if max_len_k is None:
        max_len_k = int((cu_seqlens_k[1:] - cu_seqlens_k[:-1]).max().item())
    batch = cu_seqlens_q.numel() - 1
    need = workspace_size(OP_DENSE, batch, q.shape[0], max_len_k, cfg) if max_len_q == 1 else 0
    if ws is None and need > 0:
        ws = torch.empty((need,), dtype=torch.uint8, device=q.device)
    _check(_lib.qsa_dense_attn_prefill(ctypes.byref(cfg), _p(q), _p(k), _p(v), _p(cu_seqlens_q), _p(cu_seqlens_k),
                                       batch, q.shape[0], k.shape[0], max_len_q, max_len_k, _p(o), _p(lse),
                                       _p(ws), ws.numel() if ws is not None else 0, _stream()),
           "qsa_dense_attn_prefill")
    return (o, lse) if want_lse or lse is not None else o


class Prefill:
    """One QSA layer's prefill through the C ABI, with query rows processed in
    chunks (the pages measure with 16K-token chunks).  Buffers are allocated
    once and reused across calls of the same shape.  fused=True (default) selects
    with qsa_index_select (no score rows in memory); fused=False materialises each
    chunk's scores (qsa_index_scores) and selects on them (qsa_select_blocks)."""

    def __init__(self, seqlens, chunk_rows: int = 16384, cfg: Optional[Config] = None, device="cuda",
                 fused: bool = True, attn_rows: int = 4096):
        self.cfg = _cfg(cfg)
        r = self.cfg.r
        self.seqlens = [int(x) for x in seqlens]
        self.total = sum(self.seqlens)
        self.max_len = max(self.seqlens)
        self.n_blocks = sum(L // r for L in self.seqlens)
        self.ld = max(4, ((self.max_len - 1) // r + 3) // 4 * 4)  # a multiple of 4
        self.chunk = int(chunk_rows)
        self.attn_rows = int(attn_rows)
        if self.chunk <= 0 or self.attn_rows <= 0:
            raise ValueError("chunk_rows and attn_rows must be positive")
        self.fused = bool(fused)
        self.device = torch.device(device)
        cu = [0]
        for L in self.seqlens:
            cu.append(cu[-1] + L)
        cb = [0]
        for L in self.seqlens:
            cb.append(cb[-1] + L // r)
        self.cu = torch.tensor(cu, dtype=torch.int32, device=self.device)
        self.cu_blocks = torch.tensor(cb, dtype=torch.int32, device=self.device)
        self.kc = torch.empty((max(self.n_blocks, 1), 2, self.cfg.idx_dim), dtype=torch.bfloat16, device=self.device)
        rows = min(self.chunk, self.total)
        if self.fused:
            self.scores = None
            need = workspace_size(OP_INDEX_SELECT, len(self.seqlens), rows, self.max_len, self.cfg)
            self.ws_sel = torch.empty((max(need, 16),), dtype=torch.uint8, device=self.device)
        else:
            self.scores = torch.empty((rows, self.ld), dtype=torch.float32, device=self.device)
            self.ws_sel = None
        self.sel = torch.empty((self.total, self.cfg.budget_blocks), dtype=torch.int32, device=self.device)
        need = workspace_size(OP_PREFILL, len(self.seqlens), rows, self.max_len, self.cfg)
        self.ws = torch.empty((need,), dtype=torch.uint8, device=self.device) if need > 0 else None

    def attend(self, q, k, v, o=None, lse=None):
        """Sparse attention of every row, one launch per attn_rows rows (persistent CTAs over
        each launch's rows; on B200, launches of 2048 to 4096 rows ran the 262144-row prefill
        about 6% faster than one launch over all rows, with less spread), or, with the
        key-chunked schedule (its workspace is sized per chunk_rows), chunk by chunk."""
        if o is None:
            o = torch.empty_like(q)
        step = self.chunk if self.ws is not None else self.attn_rows
        for r0 in range(0, self.total, step):
            r1 = min(self.total, r0 + step)
            sparse_attn_prefill(q, k, v, self.sel, self.cu, self.cu, r0, r1, o=o, lse=lse, cfg=self.cfg, ws=self.ws,
                                max_len_k=self.max_len)
        return o

    def index_select(self, q_idx, w, k_idx):
        compress_keys(k_idx, self.cu, self.cu_blocks, kc=self.kc, cfg=self.cfg)
        for r0 in range(0, self.total, self.chunk):
            r1 = min(self.total, r0 + self.chunk)
            self.select_chunk(q_idx, w, r0, r1)
        return self.sel

    def select_chunk(self, q_idx, w, r0: int, r1: int):
        """Selection of rows [r0, r1) from the compressed keys already in self.kc."""
        kc = self.kc[: self.n_blocks]
        if self.fused:
            index_select(q_idx, w, kc, self.cu, self.cu, self.cu_blocks, self.max_len, self.max_len, r0, r1,
                         sel=self.sel, ws=self.ws_sel, cfg=self.cfg)
        else:
            index_scores(q_idx, w, kc, self.cu, self.cu, self.cu_blocks, self.max_len, self.ld, r0, r1,
                         scores=self.scores, cfg=self.cfg)
            select_blocks(self.scores, self.cu, self.cu, self.total, r0, r1, sel=self.sel, cfg=self.cfg)

    def __call__(self, q, k, v, q_idx, w, k_idx, o=None, lse=None):
        self.index_select(q_idx, w, k_idx)
        return self.attend(q, k, v, o=o, lse=lse)

    def from_host(self, q, k, v, q_idx, w, k_idx, o, lse=None, pipe_rows: int = 8192):
        """The whole prefill from host memory, copies overlapped with the compute.

        q, k, v, q_idx, w, k_idx are host tensors and o (and lse) host outputs, all
        pinned so that the copies run asynchronously.  One copy stream brings in k_idx,
        then q_idx and w per selection chunk, then k, v and q per attention chunk of
        pipe_rows rows; the current stream compresses, selects and attends each chunk as
        soon as its inputs have landed; a second copy stream returns each chunk's output
        while the next one is computed.  The device buffers are allocated on the first
        call and reused.  The current stream waits for the last copy back, so events
        recorded on it around the call time the whole step; it returns o."""
        dev = torch.device(self.device)
        cur = torch.cuda.current_stream(dev)
        if getattr(self, "_copy_streams", None) is None:
            self._copy_streams = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
        h2d, d2h = self._copy_streams
        host = {"q": q, "k": k, "v": v, "q_idx": q_idx, "w": w, "k_idx": k_idx}
        stage = getattr(self, "_stage", None)
        if stage is None or any(stage[n].shape != t.shape or stage[n].dtype != t.dtype for n, t in host.items()):
            stage = {n: torch.empty(t.shape, dtype=t.dtype, device=dev) for n, t in host.items()}
            stage["o"] = torch.empty(o.shape, dtype=o.dtype, device=dev)
            self._stage = stage
        d_lse = None
        if lse is not None:
            if getattr(self, "_stage_lse", None) is None or self._stage_lse.shape != lse.shape:
                self._stage_lse = torch.empty(lse.shape, dtype=lse.dtype, device=dev)
            d_lse = self._stage_lse
        if self.ws is not None:  # the key-chunked schedule's workspace holds self.chunk rows
            pipe_rows = min(int(pipe_rows), self.chunk)
        plan = prefill_copy_plan(self.total, self.chunk, int(pipe_rows), self.cfg.r)
        h2d.wait_stream(cur)  # the previous step's compute is done with the buffers
        d2h.wait_stream(cur)

        def put(name, a, b):
            if b > a:
                stage[name][a:b].copy_(host[name][a:b], non_blocking=True)

        with torch.cuda.stream(h2d):
            put("k_idx", 0, self.total)
            ev_kidx = h2d.record_event()
            ev_sel = []
            for (_, _), (a, b) in plan["select"]:
                put("q_idx", a, b)
                put("w", a, b)
                ev_sel.append(h2d.record_event())
            ev_att = []
            for (_, _), (ka, kb), (qa, qb) in plan["attend"]:
                put("k", ka, kb)
                put("v", ka, kb)
                put("q", qa, qb)
                ev_att.append(h2d.record_event())
        cur.wait_event(ev_kidx)
        compress_keys(stage["k_idx"], self.cu, self.cu_blocks, kc=self.kc, cfg=self.cfg)
        for ((r0, r1), _), e in zip(plan["select"], ev_sel):
            cur.wait_event(e)
            self.select_chunk(stage["q_idx"], stage["w"], r0, r1)
        ev_out = []
        sub = self.chunk if self.ws is not None else self.attn_rows  # launches within a copy chunk
        for ((r0, r1), _, _), e in zip(plan["attend"], ev_att):
            cur.wait_event(e)
            for a in range(r0, r1, sub):
                sparse_attn_prefill(stage["q"], stage["k"], stage["v"], self.sel, self.cu, self.cu, a, min(r1, a + sub),
                                    o=stage["o"], lse=d_lse, cfg=self.cfg, ws=self.ws, max_len_k=self.max_len)
            ev_out.append(cur.record_event())
        with torch.cuda.stream(d2h):
            for ((r0, r1), _, _), e in zip(plan["attend"], ev_out):
                d2h.wait_event(e)
                o[r0:r1].copy_(stage["o"][r0:r1], non_blocking=True)
                if lse is not None:
                    lse[r0:r1].copy_(d_lse[r0:r1], non_blocking=True)
            done = d2h.record_event()
        cur.wait_event(done)
        return o


class MtpStep:
    """One multi-token decode step for a fixed batch: next_n new queries per sequence
    (q [batch, next_n, 24, 256]; q_idx [batch, 4, 128] and w [batch, 4] of the last of
    them) attend one shared selection.  The step recomputes the compressed blocks its
    tokens may have completed (refresh_blocks [batch] int32: the first block to
    recompute per sequence, then refresh_count blocks; blocks not yet complete are
    skipped), makes the shared selection (qsa_index_select_mtp) and attends
    (qsa_sparse_attn_decode_mtp).  The launches can be captured once in a CUDA graph
    and replayed (graph=True): the tensors passed here are the graph's fixed inputs,
    refreshed in place by the caller."""

    def __init__(self, q, q_idx, w, k_cache, v_cache, k_idx, kc, cu_seqlens_k, cu_blocks, max_len_k: int,
                 refresh_blocks=None, refresh_count: Optional[int] = None, cfg: Optional[Config] = None,
                 graph: bool = True):
        self.cfg = _cfg(cfg)
        if q.dim() != 4:
            raise ValueError("q must be [batch, next_n, heads, head_dim]")
        self.q, self.q_idx, self.w = q, q_idx, w
        self.k_cache, self.v_cache, self.k_idx, self.kc = k_cache, v_cache, k_idx, kc
        self.cu_k, self.cu_b = cu_seqlens_k, cu_blocks
        self.batch, self.next_n = q.shape[0], q.shape[1]
        self.max_len_k = int(max_len_k)
        self.refresh = refresh_blocks
        r = self.cfg.r
        self.refresh_count = int(refresh_count) if refresh_count is not None else (self.next_n + r - 1) // r + 1
        dev = q.device
        self.sel = torch.empty((self.batch, self.cfg.budget_blocks), dtype=torch.int32, device=dev)
        self.ws_sel = torch.empty((max(workspace_size(OP_INDEX_SELECT, self.batch, self.batch, max_len_k, self.cfg),
                                       16),), dtype=torch.uint8, device=dev)
        self.ws = torch.empty((max(workspace_size(OP_DECODE_MTP, self.batch, self.batch, 0, self.cfg), 16),),
                              dtype=torch.uint8, device=dev)
        self.o = torch.empty_like(q)
        self.graph = None
        self.run()  # first call outside any capture (one-time kernel attribute setup)
        if graph:
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.run()
            self.graph = g

    def run(self):
        if self.refresh is not None:
            compress_keys(self.k_idx, self.cu_k, self.cu_b, kc=self.kc, blk_begin=self.refresh,
                          max_new_blocks=self.refresh_count, cfg=self.cfg)
        index_select_mtp(self.q_idx, self.w, self.kc, self.cu_k, self.cu_b, self.next_n, self.max_len_k, sel=self.sel,
                         ws=self.ws_sel, cfg=self.cfg)
        sparse_attn_decode_mtp(self.q, self.k_cache, self.v_cache, self.cu_k, self.sel, o=self.o, ws=self.ws,
                               cfg=self.cfg)
        return self.o

    def __call__(self):
        if self.graph is not None:
            self.graph.replay()
            return self.o
        return self.run()


def prefill_copy_plan(total: int, select_rows: int, attend_rows: int, r: int = 4):
    """The row ranges of Prefill.from_host: for each selection chunk (r0, r1) the rows of
    q_idx and w copied before it, and for each attention chunk (r0, r1) the rows of k, v
    and of q copied before it.  Every row is copied once, in order.  The indexer reads
    whole 64-row tiles, so a selection chunk's copy reaches 63 rows past r1; the attention
    loads whole micro-blocks, so its k and v copy reaches r - 1 rows past r1 (those keys
    are masked, but must hold finite values)."""
    if select_rows <= 0 or attend_rows <= 0:
        raise ValueError("chunk sizes must be positive")
    sel, att = [], []
    done = 0
    for r0 in range(0, total, select_rows):
        r1 = min(total, r0 + select_rows)
        hi = min(total, r1 + 63)
        sel.append(((r0, r1), (done, max(done, hi))))
        done = max(done, hi)
    kv_done = q_done = 0
    for r0 in range(0, total, attend_rows):
        r1 = min(total, r0 + attend_rows)
        kv_hi = max(kv_done, min(total, r1 + r - 1))
        att.append(((r0, r1), (kv_done, kv_hi), (q_done, r1)))
        kv_done, q_done = kv_hi, r1
    return {"select": sel, "attend": att}


class DecodeStep:
    """One QSA decode step for a fixed batch, one new query per sequence: refresh
    the compressed block each sequence just completed, select the top k
    (qsa_index_select: the hi-plane scan of every earlier block and the exact
    rescoring of each row's near-threshold window; fused=False: the exact scores,
    then the selector), and run the decode attention (the batch's tiles spread
    evenly over the CTAs) and the merge of the row pieces.  The launches can be
    captured once in a CUDA graph and replayed (graph=True): the tensors passed
    here are the graph's fixed inputs, so a caller refreshes them in place."""

    def __init__(self, q, q_idx, w, k_cache, v_cache, k_idx, kc, cu_seqlens_k, cu_blocks, max_len_k: int,
                 refresh_blocks=None, cfg: Optional[Config] = None, graph: bool = True, fused: bool = True):
        self.cfg = _cfg(cfg)
        r = self.cfg.r
        self.q, self.q_idx, self.w = q, q_idx, w
        self.k_cache, self.v_cache, self.k_idx, self.kc = k_cache, v_cache, k_idx, kc
        self.cu_k, self.cu_b = cu_seqlens_k, cu_blocks
        self.batch = q.shape[0]
        dev = q.device
        self.cu_q = torch.arange(self.batch + 1, dtype=torch.int32, device=dev)
        self.refresh = refresh_blocks  # [batch] int32 block ids to recompute, or None
        self.ld = max(4, ((max_len_k - 1) // r + 3) // 4 * 4)
        self.max_len_k = int(max_len_k)
        self.fused = bool(fused)
        self.scores = None if self.fused else torch.empty((self.batch, self.ld), dtype=torch.float32, device=dev)
        self.ws_sel = torch.empty((max(workspace_size(OP_INDEX_SELECT, self.batch, self.batch, max_len_k, self.cfg),
                                       16),), dtype=torch.uint8, device=dev) if self.fused else None
        self.sel = torch.empty((self.batch, self.cfg.budget_blocks), dtype=torch.int32, device=dev)
        self.o = torch.empty_like(q)
        self.ws = torch.empty((max(workspace_size(OP_DECODE, self.batch, self.batch, max_len_k, self.cfg), 16),),
                              dtype=torch.uint8, device=dev)
        self.graph = None
        self.run()  # first call outside any capture (one-time kernel attribute setup)
        if graph:
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.run()
            self.graph = g

    def run(self):
        if self.refresh is not None:
            compress_keys(self.k_idx, self.cu_k, self.cu_b, kc=self.kc, blk_begin=self.refresh, max_new_blocks=1,
                          cfg=self.cfg)
        if self.fused:
            index_select(self.q_idx, self.w, self.kc, self.cu_q, self.cu_k, self.cu_b, 1, self.max_len_k,
                         sel=self.sel, ws=self.ws_sel, cfg=self.cfg)
        else:
            index_scores(self.q_idx, self.w, self.kc, self.cu_q, self.cu_k, self.cu_b, 1, self.ld,
                         scores=self.scores, cfg=self.cfg)
            select_blocks(self.scores, self.cu_q, self.cu_k, self.batch, sel=self.sel, cfg=self.cfg)
        sparse_attn_decode(self.q, self.k_cache, self.v_cache, self.cu_k, self.sel, o=self.o, ws=self.ws,
                           cfg=self.cfg)
        return self.o

    def __call__(self):
        if self.graph is not None:
            self.graph.replay()
            return self.o
        return self.run()
