"""Decode attention with the library's fixed device scratch
(qsa_sparse_attn_decode_static_scratch) against the workspace entry point
(qsa_sparse_attn_decode) on the same inputs, through the C ABI.

This file is collected last, so that the static-scratch call also runs after
every other test of the session; it needs nothing from them and passes on its
own in a fresh process as well.
"""
import numpy as np
import pytest
import torch

from block_sparse_long_09_b200.inputs import make_decode

K = 512
R = 4


def random_selection(seqlens, k, seed):
    """A valid decode selection per sequence: the own block b_t = (L - 1) // r plus
    up to k - 1 distinct earlier blocks, ascending, padded with -1."""
    g = torch.Generator().manual_seed(seed)
    sel = torch.full((len(seqlens), k), -1, dtype=torch.int32)
    for s, L in enumerate(seqlens):
        bt = (L - 1) // R
        m = min(k - 1, bt)
        earlier = torch.randperm(bt, generator=g)[:m] if m > 0 else torch.empty(0, dtype=torch.int64)
        ids = torch.sort(torch.cat([earlier, torch.tensor([bt])])).values
        sel[s, :ids.numel()] = ids.to(torch.int32)
    return sel


def close(a, b):
    d = (a.double() - b.double()).abs().cpu().numpy()
    assert d.max() <= 2e-2, d.max()
    assert d.mean() <= 1e-3, d.mean()


def case(batch, lo, hi, seed):
    d = make_decode(batch, lo, hi, seed=seed, device="cuda")
    sel = random_selection(d.seqlens, K, seed).cuda()
    return d, sel


@pytest.mark.gpu
def test_static_scratch_decode_matches_workspace_decode_twice_in_a_row():
    from block_sparse_long_09_b200 import qsa
    torch.cuda.set_device(0)
    cfg = qsa.default_config(budget_blocks=K)
    # batch 64 fills most of the scratch (64 sequences x 8 splits on 148 SMs);
    # the second call has fewer, shorter sequences and so overwrites only a part
    cases = [case(64, 2000, 9000, 11), case(5, 300, 3000, 12)]
    refs = []
    for d, sel in cases:
        o, lse = qsa.sparse_attn_decode(d.q, d.k_cache, d.v_cache, d.cu_seqlens_k, sel, want_lse=True, cfg=cfg)
        refs.append((o, lse))
    torch.cuda.synchronize()
    outs = []
    for d, _ in cases:
        outs.append((torch.empty_like(d.q),
                     torch.empty((d.q.shape[0], cfg.n_heads_q), dtype=torch.float32, device="cuda")))
    # two calls in a row on one stream, no synchronisation between them
    for (d, sel), (o, lse) in zip(cases, outs):
        qsa.sparse_attn_decode_static_scratch(d.q, d.k_cache, d.v_cache, d.cu_seqlens_k, sel, o, lse, cfg=cfg)
    torch.cuda.synchronize()
    assert qsa.device_status(clear=True) == 0
    for (o_ref, lse_ref), (o, lse) in zip(refs, outs):
        close(o, o_ref)
        assert np.abs((lse - lse_ref).cpu().numpy()).max() <= 1e-3
    # and the first case once more, after the second one used the scratch
    d, sel = cases[0]
    o, lse = outs[0]
    o.zero_()
    qsa.sparse_attn_decode_static_scratch(d.q, d.k_cache, d.v_cache, d.cu_seqlens_k, sel, o, lse, cfg=cfg)
    torch.cuda.synchronize()
    assert qsa.device_status(clear=True) == 0
    close(o, refs[0][0])
