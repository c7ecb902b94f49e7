"""Run-to-run determinism through the C ABI: the same inputs give the same bits.

The selections are exact (every path ends in an exact top-k with the lower-index tie
rule, whatever order its candidate lists were filled in), the attention's pieces are
merged in a fixed order, so two runs of the prefill, of a decode step (the fused refine
at batch >= 32 and the listed one below) and of a multi-token step must agree bit for
bit, selections and outputs alike.
"""
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


def test_prefill_is_deterministic(qsa):
    lengths = [9001, 3000]
    cfg = qsa.default_config(budget_blocks=64)
    x = inputs.make_prefill(lengths, seed=93, device="cuda")
    runs = []
    for _ in range(2):
        pre = qsa.Prefill(lengths, chunk_rows=4096, cfg=cfg)
        lse = torch.empty((x.q.shape[0], 24), dtype=torch.float32, device="cuda")
        o = pre(x.q, x.k, x.v, x.q_idx, x.w, x.k_idx, lse=lse)
        torch.cuda.synchronize()
        runs.append((pre.sel.clone(), o.clone(), lse.clone()))
    for a, b in zip(*runs):
        assert torch.equal(a, b)
    assert qsa.device_status(clear=True) == 0


@pytest.mark.parametrize("batch", [4, 40])
def test_decode_step_is_deterministic(qsa, batch):
    d = inputs.make_decode(batch, 15000, 30000, seed=94, device="cuda")
    cfg = qsa.default_config()
    kc = qsa.compress_keys(d.k_idx, d.cu_seqlens_k, d.cu_blocks, n_blocks=int(d.cu_blocks[-1]), cfg=cfg)
    last = torch.tensor([L // 4 - 1 for L in d.seqlens], dtype=torch.int32, device="cuda")
    runs = []
    for _ in range(2):
        step = qsa.DecodeStep(d.q, d.q_idx, d.w, d.k_cache, d.v_cache, d.k_idx, kc, d.cu_seqlens_k, d.cu_blocks,
                              max(d.seqlens), refresh_blocks=last, cfg=cfg, graph=False)
        o = step()
        torch.cuda.synchronize()
        runs.append((step.sel.clone(), o.clone()))
    assert torch.equal(runs[0][0], runs[1][0])
    assert torch.equal(runs[0][1], runs[1][1])
    assert qsa.device_status(clear=True) == 0


def test_mtp_step_is_deterministic(qsa):
    d = inputs.make_decode(4, 15000, 30000, seed=95, device="cuda", next_n=4)
    cfg = qsa.default_config()
    kc = qsa.compress_keys(d.k_idx, d.cu_seqlens_k, d.cu_blocks, n_blocks=int(d.cu_blocks[-1]), cfg=cfg)
    runs = []
    for _ in range(2):
        step = qsa.MtpStep(d.q, d.q_idx, d.w, d.k_cache, d.v_cache, d.k_idx, kc, d.cu_seqlens_k, d.cu_blocks,
                           max(d.seqlens), cfg=cfg, graph=False)
        o = step()
        torch.cuda.synchronize()
        runs.append((step.sel.clone(), o.clone()))
    assert torch.equal(runs[0][0], runs[1][0])
    assert torch.equal(runs[0][1], runs[1][1])
    assert qsa.device_status(clear=True) == 0
