"""Prefill.from_host (copies in and out overlapped with the compute, chunk by chunk)
against the device-resident prefill, through the C ABI: the same kernels on the same
rows, so the outputs must be equal bit for bit -- including the first call, whose
device buffers are fresh, and chunk sizes that cut indexer tiles and micro-blocks."""
import pytest
import torch

from block_sparse_long_09_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qsa():
    from block_sparse_long_09_b200 import build
    build.build()
    from block_sparse_long_09_b200 import qsa as q
    assert torch.cuda.is_available()
    q.device_status(clear=True)
    return q


@pytest.mark.parametrize("lengths,k,chunk,pipe", [([9001, 4000], 64, 4096, 3001), ([70000], 512, 16384, 5000),
                                                   ([3, 4097, 130], 16, 1000, 77)])
def test_from_host_equals_resident_prefill(qsa, lengths, k, chunk, pipe):
    cfg = qsa.default_config(budget_blocks=k)
    x = inputs.make_prefill(lengths, seed=91, device="cuda")
    pre = qsa.Prefill(lengths, chunk_rows=chunk, cfg=cfg)
    o_ref = torch.empty_like(x.q)
    lse_ref = torch.empty((x.q.shape[0], 24), dtype=torch.float32, device="cuda")
    pre(x.q, x.k, x.v, x.q_idx, x.w, x.k_idx, o=o_ref, lse=lse_ref)
    sel_ref = pre.sel.clone()
    host = {n: getattr(x, n).cpu().pin_memory() for n in ("q", "k", "v", "q_idx", "w", "k_idx")}
    for rep in range(2):  # the first call stages into fresh buffers, the second reuses them
        o = torch.full(x.q.shape, float("nan"), dtype=x.q.dtype).pin_memory()
        lse = torch.full((x.q.shape[0], 24), float("nan"), dtype=torch.float32).pin_memory()
        pre.sel.fill_(-7)
        pre.from_host(host["q"], host["k"], host["v"], host["q_idx"], host["w"], host["k_idx"], o, lse=lse,
                      pipe_rows=pipe)
        torch.cuda.current_stream().synchronize()
        assert torch.equal(pre.sel, sel_ref)
        assert torch.equal(o, o_ref.cpu())
        assert torch.equal(lse, lse_ref.cpu())
    assert qsa.device_status(clear=True) == 0


def test_attention_launch_chunks_do_not_change_the_output(qsa):
    """Prefill.attend launches the attention per attn_rows rows; every row's arithmetic is
    its own, so one launch over all rows and launches of any size give the same bits."""
    lengths = [20000, 7, 9001]
    cfg = qsa.default_config(budget_blocks=128)
    x = inputs.make_prefill(lengths, seed=92, device="cuda")
    outs = []
    for attn_rows in (sum(lengths), 16384, 1000, 333):
        pre = qsa.Prefill(lengths, chunk_rows=8192, cfg=cfg, attn_rows=attn_rows)
        o = torch.full_like(x.q, float("nan"))
        lse = torch.full((x.q.shape[0], 24), float("nan"), dtype=torch.float32, device="cuda")
        pre(x.q, x.k, x.v, x.q_idx, x.w, x.k_idx, o=o, lse=lse)
        torch.cuda.synchronize()
        outs.append((pre.sel.clone(), o, lse))
    for sel, o, lse in outs[1:]:
        assert torch.equal(sel, outs[0][0])
        assert torch.equal(o, outs[0][1])
        assert torch.equal(lse, outs[0][2])
    assert qsa.device_status(clear=True) == 0
