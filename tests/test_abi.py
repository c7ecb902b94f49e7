"""Host-side checks of the C ABI: the library loads, exports every entry point
declared in include/qsa.h, and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def qsa():
    from block_sparse_long_09_b200 import build
    build.build()
    from block_sparse_long_09_b200 import qsa as q
    return q


def declared_functions():
    text = open(os.path.join(ROOT, "include", "qsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qsa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("qsa_compress_keys", "qsa_index_scores", "qsa_select_blocks", "qsa_sparse_attn_prefill",
              "qsa_sparse_attn_decode"):
        assert n in names


def test_library_exports_every_declared_symbol(qsa):
    lib = qsa.library()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(qsa.EXPORTED) >= set(declared_functions())


def test_config_defaults_and_version(qsa):
    c = qsa.default_config()
    assert (c.r, c.budget_blocks, c.n_heads_q, c.n_heads_kv, c.head_dim, c.n_heads_idx, c.idx_dim) == \
        (4, 512, 24, 2, 256, 4, 128)
    assert abs(c.softmax_scale - 1 / 16) < 1e-9 and abs(c.rms_eps - 1e-6) < 1e-12
    assert qsa.library().qsa_version() >= 100


def test_paged_decode_args_rejected_on_host(qsa):
    import ctypes
    lib = qsa.library()
    cfg = qsa.default_config()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the call returns before any device work
    P = lambda: fake  # noqa: E731
    # page size not a multiple of r = 4
    st = lib.qsa_sparse_attn_decode_paged(ctypes.byref(cfg), P(), P(), P(), 8, 6, P(), 4, P(), 2, P(), P(), None,
                                          P(), 1 << 20, None)
    assert st == qsa.QSA_ERR_INVALID_ARG
    # no block table
    st = lib.qsa_sparse_attn_decode_paged(ctypes.byref(cfg), P(), P(), P(), 8, 16, None, 4, P(), 2, P(), P(), None,
                                          P(), 1 << 20, None)
    assert st == qsa.QSA_ERR_INVALID_ARG
    # a pool whose rows overflow 32-bit tensor coordinates
    st = lib.qsa_sparse_attn_decode_paged(ctypes.byref(cfg), P(), P(), P(), 1 << 30, 16, P(), 4, P(), 2, P(), P(),
                                          None, P(), 1 << 20, None)
    assert st == qsa.QSA_ERR_UNSUPPORTED
    assert qsa.workspace_size(qsa.OP_DECODE_PAGED, 1000, 1000) >= 1000 * 24 * 257 * 4


def test_status_strings(qsa):
    lib = qsa.library()
    for s in range(8):
        assert lib.qsa_status_string(s).decode().startswith("QSA")


def test_unsupported_config_rejected_on_host(qsa):
    lib = qsa.library()
    for field, value in (("r", 8), ("n_heads_q", 32), ("head_dim", 128), ("budget_blocks", 4096)):
        c = qsa.default_config(**{field: value})
        st = lib.qsa_compress_keys(ctypes.byref(c), None, None, None, 1, 0, None, 0, None, None)
        assert st == qsa.QSA_ERR_UNSUPPORTED, field
    c = qsa.default_config(r=0)
    assert lib.qsa_compress_keys(ctypes.byref(c), None, None, None, 1, 0, None, 0, None, None) == \
        qsa.QSA_ERR_INVALID_ARG


def test_invalid_arguments_rejected_on_host(qsa):
    lib = qsa.library()
    c = qsa.default_config()
    fake = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    # batch <= 0
    assert lib.qsa_compress_keys(ctypes.byref(c), fake, fake, fake, 0, 8, None, 0, fake, None) == \
        qsa.QSA_ERR_INVALID_ARG
    # row range beyond total_q
    assert lib.qsa_index_scores(ctypes.byref(c), fake, fake, fake, 4, fake, fake, fake, 1, 10, 0, 0, 11,
                                fake, 8, None, 0, None) == qsa.QSA_ERR_INVALID_ARG
    # ld <= 0
    assert lib.qsa_select_blocks(ctypes.byref(c), fake, 0, fake, fake, 1, 0, 4, fake, None, 0, None) == \
        qsa.QSA_ERR_INVALID_ARG
    # misaligned q
    assert lib.qsa_sparse_attn_prefill(ctypes.byref(c), ctypes.c_void_p(18), fake, fake, fake, fake, fake, 1, 4,
                                       4, 4, 0, 4, fake, None, None, 0, None) == qsa.QSA_ERR_INVALID_ARG
    # empty row range is a no-op
    assert lib.qsa_sparse_attn_prefill(ctypes.byref(c), fake, fake, fake, fake, fake, fake, 1, 4, 4, 4, 2, 2,
                                       fake, None, None, 0, None) == qsa.QSA_OK


def test_workspace_sizes(qsa):
    assert qsa.workspace_size(qsa.OP_INDEX, 1, 8192, 8192) == 0
    assert qsa.workspace_size(qsa.OP_PREFILL, 1, 8192, 8192) == 0     # single-pass schedule (default)
    assert qsa.workspace_size(qsa.OP_PREFILL, 1, 16384, 262144) == 0
    big = qsa.workspace_size(qsa.OP_PREFILL, 1, 16384, 262144, qsa.default_config(kv_chunk_blocks=8192))
    assert big >= 16384 * 8 * 24 * 257 * 4                             # 8 key chunks of 32768 tokens
    small = qsa.workspace_size(qsa.OP_PREFILL, 1, 1000, 8192, qsa.default_config(kv_chunk_blocks=64))
    assert small >= 1000 * 32 * 24 * 257 * 4
    ws = qsa.workspace_size(qsa.OP_DECODE, 64, 64, 262144)
    assert ws >= 64 * 24 * 257 * 4


def test_fault_injection_is_inert_in_the_release_library(qsa):
    # the release build compiles no injection site: the call is refused before any CUDA call
    assert qsa.LIB_PATH.endswith("libqsa.so")
    assert qsa.library().qsa_debug_inject(1) == qsa.QSA_ERR_UNSUPPORTED
    assert qsa.library().qsa_debug_inject(0) == qsa.QSA_ERR_UNSUPPORTED


def test_binding_refuses_a_selection_that_does_not_match_the_budget(qsa):
    # checked on the host before the library is called (CPU tensors never reach it)
    import torch
    q = torch.zeros((8, 24, 256), dtype=torch.bfloat16)
    kv = torch.zeros((8, 2, 256), dtype=torch.bfloat16)
    cu_ = torch.tensor([0, 8], dtype=torch.int32)
    for bad in (torch.zeros((8, 64), dtype=torch.int32), torch.zeros((4, 512), dtype=torch.int32),
                torch.zeros((8, 512), dtype=torch.int64), torch.zeros((8, 1024), dtype=torch.int32)[:, :512]):
        with pytest.raises(ValueError):
            qsa.sparse_attn_prefill(q, kv, kv, bad, cu_, cu_)
    with pytest.raises(ValueError):
        qsa.sparse_attn_decode(q[:1], kv, kv, cu_, torch.zeros((1, 16), dtype=torch.int32))


def test_rope_config_checked_on_the_host(qsa):
    import ctypes
    lib = qsa.library()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: each call returns before any device work
    c = qsa.default_config()
    assert (c.rope_dims, c.rope_base) == (64, 10000.0)
    # qsa_rope_queries needs QSA_INDEX_ROPE
    assert lib.qsa_rope_queries(ctypes.byref(c), fake, fake, fake, 1, 8, None) == qsa.QSA_ERR_INVALID_ARG
    for dims, base in ((0, 1e4), (12, 1e4), (136, 1e4), (64, 1.0), (64, float("nan"))):
        bad = qsa.default_config(flags=qsa.QSA_INDEX_ROPE, rope_dims=dims, rope_base=base)
        assert lib.qsa_rope_queries(ctypes.byref(bad), fake, fake, fake, 1, 8, None) == qsa.QSA_ERR_INVALID_ARG
        assert lib.qsa_compress_keys(ctypes.byref(bad), fake, fake, fake, 1, 8, None, 0, fake, None) == \
            qsa.QSA_ERR_INVALID_ARG


@pytest.mark.parametrize("total,sel_rows,att_rows", [(1, 1, 1), (9001, 4096, 3000), (70000, 65536, 16384),
                                                     (262144, 65536, 16384), (64, 1000, 7), (5, 2, 3)])
def test_prefill_copy_plan_covers_every_row_once_and_in_time(qsa, total, sel_rows, att_rows):
    """Prefill.from_host's copy plan: each tensor's rows are copied exactly once, in
    order, and every chunk's reads (whole 64-row indexer tiles, whole 4-token blocks of
    keys up to the chunk's last row) are covered by the copies issued before it."""
    r = 4
    plan = qsa.prefill_copy_plan(total, sel_rows, att_rows, r)
    sel, att = plan["select"], plan["attend"]
    # the chunks tile the rows
    assert [c[0] for c in sel] == [(a, min(total, a + sel_rows)) for a in range(0, total, sel_rows)]
    assert [c[0] for c in att] == [(a, min(total, a + att_rows)) for a in range(0, total, att_rows)]
    for ranges in ([c[1] for c in sel], [c[1] for c in att], [c[2] for c in att]):
        pos = 0
        for a, b in ranges:  # contiguous, in order, never backwards
            assert a == pos and b >= a
            pos = b
        assert pos == total   # every row copied, once
    for (r0, r1), (_, hi) in sel:
        assert hi >= min(total, (r1 + 63) // 64 * 64)  # the last indexer tile of the chunk
    for (r0, r1), (_, kv_hi), (_, q_hi) in att:
        assert q_hi >= r1
        assert kv_hi >= min(total, r1 - 1 + r)          # the micro-block holding row r1 - 1, loaded whole
    with pytest.raises(ValueError):
        qsa.prefill_copy_plan(10, 0, 4)


def test_binding_constants_match_the_header(qsa):
    """Every status code, flag and workspace op the binding hard-codes equals the value
    include/qsa.h defines (the binding passes them to the library as plain integers)."""
    text = open(os.path.join(ROOT, "include", "qsa.h")).read()
    defs = {}
    for name, value in re.findall(r"#define\s+(QSA_[A-Z_]+)\s+\(?([0-9x]+)u?", text):
        defs[name] = int(value, 0)
    assert defs["QSA_STATIC_SCRATCH_BYTES"] == 16  # "(16u * 1024u * 1024u)": the first factor
    assert qsa.STATIC_SCRATCH_BYTES == 16 * 1024 * 1024
    for name in ("QSA_OK", "QSA_ERR_INVALID_ARG", "QSA_ERR_UNSUPPORTED", "QSA_ERR_WORKSPACE_TOO_SMALL",
                 "QSA_ERR_CUDA", "QSA_ERR_TIMEOUT", "QSA_ERR_DEVICE_CHECK", "QSA_ERR_SCRATCH_LIMIT",
                 "QSA_COMPRESS_NO_NORM", "QSA_INDEX_ROPE"):
        assert getattr(qsa, name) == defs[name], name
    for name in ("COMPRESS", "INDEX", "SELECT", "PREFILL", "DECODE", "DENSE", "DECODE_PAGED", "INDEX_SELECT",
                 "INDEX_SELECT_PAGED", "DECODE_MTP"):
        assert getattr(qsa, "OP_" + name) == defs["QSA_OP_" + name], name
