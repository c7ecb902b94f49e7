"""Context-parallel decode: the K/V cache of a decode batch split by block ranges over
ranks (one process per GPU).

Rank j holds the tokens [j C r, (j + 1) C r) of every sequence (C = block_chunk
micro-blocks of r tokens): their K/V rows, raw indexer keys and compressed keys.  The
rank whose range holds a sequence's last token holds its partial tail too.  One step,
for the new token of every sequence (t = L - 1, own block b_t = floor(t / r)):

  1. indexer scores of the rank's own candidate blocks (complete blocks < b_t in its
     range), written into columns [j C, j C + n) of a [batch, ld] buffer that is zero
     elsewhere (qsa_index_scores on the rank's compressed keys, with per-sequence
     lengths under which exactly its n blocks are candidates: index_lengths);
  2. a sum over the ranks (all-reduce) gives every rank the full score rows: the
     columns are disjoint and x + 0 = x, so the rows are the one-GPU rows;
  3. qsa_select_blocks on the full rows: the one-GPU selection, bit for bit;
  4. qsa_sparse_attn_decode_window: softmax attention over the rank's own selected
     blocks, a partial (o, lse);
  5. an all-gather of the partial states and qsa_merge_attn_states: o = sum_j
     exp(lse_j - lse) o_j with lse = log sum_j exp(lse_j).

The collectives are torch.distributed (NCCL over NVLink on GPUs, gloo in the CPU test).
"""
from __future__ import annotations

import dataclasses
from typing import List, Sequence

import torch


@dataclasses.dataclass
class Shard:
    """What rank j holds of each sequence (lists of length batch)."""
    tok_lo: List[int]      # first token of its range
    tok_hi: List[int]      # one past its last token
    blk_lo: List[int]      # first block of its range (tok_lo / r)
    blk_hi: List[int]      # one past the last block it attends: min(range end, b_t + 1)
    n_cand: List[int]      # its candidate blocks: complete blocks < b_t in its range
    n_kc: List[int]        # its complete blocks (compressed keys held)


def shard_of(lengths: Sequence[int], rank: int, world: int, block_chunk: int, r: int = 4) -> Shard:
    """Rank `rank`'s part of each sequence: tokens [rank C r, (rank + 1) C r) cut to L
    (the last rank of the range also takes everything past world C r)."""
    if block_chunk <= 0 or block_chunk % 4 != 0:
        raise ValueError("block_chunk must be a positive multiple of 4 (16-byte aligned score columns)")
    sh = Shard([], [], [], [], [], [])
    for L in lengths:
        L = int(L)
        lo_t = rank * block_chunk * r
        if lo_t >= L:  # the sequence ends before this rank's range: nothing here
            past = (L + r - 1) // r
            sh.tok_lo.append(L)
            sh.tok_hi.append(L)
            sh.blk_lo.append(past)
            sh.blk_hi.append(past)
            sh.n_cand.append(0)
            sh.n_kc.append(0)
            continue
        hi_t = L if rank == world - 1 else min(L, (rank + 1) * block_chunk * r)
        bt = (L - 1) // r
        b_lo = lo_t // r
        b_end = (hi_t + r - 1) // r  # blocks touched by the range (the partial tail's too)
        sh.tok_lo.append(lo_t)
        sh.tok_hi.append(hi_t)
        sh.blk_lo.append(b_lo)
        sh.blk_hi.append(max(b_lo, min(b_end, bt + 1)))
        sh.n_cand.append(max(0, min(hi_t // r, bt) - b_lo))
        sh.n_kc.append(max(0, hi_t // r - b_lo))
    return sh


def index_lengths(sh: Shard, r: int = 4) -> List[int]:
    """Per-sequence lengths under which the indexer scores exactly a shard's n candidate
    blocks from its compressed keys: own block n (t = L' - 1), and L' / r equal to the
    shard's complete blocks (n, or n + 1 when its last complete block is the own block)."""
    return [max(r * n + 1, r * nkc) for n, nkc in zip(sh.n_cand, sh.n_kc)]


def score_columns(lengths: Sequence[int], r: int = 4) -> int:
    """Columns of the shared score rows: every candidate block b < b_t of every sequence,
    rounded up to a multiple of 4."""
    need = max(max(((int(L) - 1) // r) for L in lengths), 1)
    return (need + 3) // 4 * 4


def _cu(xs, device) -> torch.Tensor:
    out = [0]
    for x in xs:
        out.append(out[-1] + int(x))
    return torch.tensor(out, dtype=torch.int32, device=device)


class ContextParallelDecode:
    """One rank's decode step over its shard of a batch's caches.

    k_local, v_local [sum of its tokens, 2, 256] bf16, k_idx_local [same, 128] bf16: the
    rank's tokens of every sequence, packed in sequence order (as shard_of cuts them).
    """

    def __init__(self, lengths, rank: int, world: int, block_chunk: int, k_local, v_local, k_idx_local, cfg=None,
                 group=None):
        from . import qsa
        self.qsa = qsa
        self.cfg = qsa._cfg(cfg)
        self.rank, self.world, self.group = rank, world, group
        self.lengths = [int(L) for L in lengths]
        self.batch = len(self.lengths)
        self.r = r = self.cfg.r
        dev = k_local.device
        self.sh = sh = shard_of(self.lengths, rank, world, block_chunk, r)
        self.block_chunk = block_chunk
        self.k_local, self.v_local = k_local, v_local
        loc = [hi - lo for lo, hi in zip(sh.tok_lo, sh.tok_hi)]
        self.cu_loc = _cu(loc, dev)
        self.cu_kc = _cu(sh.n_kc, dev)
        # the compressed keys of the rank's complete blocks
        self.kc = qsa.compress_keys(k_idx_local, self.cu_loc, self.cu_kc, n_blocks=max(int(self.cu_kc[-1]), 1),
                                    cfg=self.cfg)
        self.cu_k = _cu(self.lengths, dev)                                  # global lengths
        self.cu_virt = _cu(index_lengths(sh, r), dev)                       # exactly n candidates each
        self.cu_q = torch.arange(self.batch + 1, dtype=torch.int32, device=dev)
        self.ld = score_columns(self.lengths, r)
        self.col0 = rank * block_chunk                                       # this rank's first column
        # rows of ld columns, zero outside this rank's; one spare row so that the view of the
        # rank's columns (the same rows shifted by col0) stays inside the storage
        self._store = torch.zeros(((self.batch + 1) * self.ld,), dtype=torch.float32, device=dev)
        self.mine = self._store[: self.batch * self.ld].view(self.batch, self.ld)
        self.full = torch.empty_like(self.mine)
        self.tok_local = torch.tensor([int(self.cu_loc[s]) for s in range(self.batch)], dtype=torch.int64,
                                      device=dev)
        self.blk_lo = torch.tensor(sh.blk_lo, dtype=torch.int32, device=dev)
        self.blk_hi = torch.tensor(sh.blk_hi, dtype=torch.int32, device=dev)
        self.sel = torch.empty((self.batch, self.cfg.budget_blocks), dtype=torch.int32, device=dev)

    def local_scores(self, q_idx, w):
        """Step 1: this rank's candidate scores in its columns of zero rows."""
        if any(self.sh.n_cand):  # then col0 < ld: the shifted view fits the spare row
            view = self._store[self.col0: self.col0 + self.batch * self.ld].view(self.batch, self.ld)
            self.qsa.index_scores(q_idx, w, self.kc, self.cu_q, self.cu_virt, self.cu_kc, 1, self.ld,
                                  scores=view, cfg=self.cfg)
        return self.mine

    def select(self, full):
        """Step 3: the selection from the full score rows (every rank the same)."""
        return self.qsa.select_blocks(full, self.cu_q, self.cu_k, self.batch, sel=self.sel, cfg=self.cfg)

    def attend(self, q):
        """Step 4: this rank's partial (o, lse) over its own selected blocks."""
        return self.qsa.sparse_attn_decode_window(q, self.k_local, self.v_local, self.cu_k, self.tok_local,
                                                  self.blk_lo, self.blk_hi, self.sel, cfg=self.cfg)

    def __call__(self, q, q_idx, w):
        """One step: (o, lse) of every sequence's new token over the whole cache."""
        import torch.distributed as dist
        self.full.copy_(self.local_scores(q_idx, w))
        if self.world > 1:
            dist.all_reduce(self.full, group=self.group)  # step 2: disjoint columns, zeros elsewhere
        self.select(self.full)
        o, lse = self.attend(q)
        if self.world > 1:  # step 5
            o_all = torch.empty((self.world,) + tuple(o.shape), dtype=o.dtype, device=o.device)
            l_all = torch.empty((self.world,) + tuple(lse.shape), dtype=lse.dtype, device=lse.device)
            dist.all_gather_into_tensor(o_all, o.contiguous(), group=self.group)
            dist.all_gather_into_tensor(l_all, lse.contiguous(), group=self.group)
        else:
            o_all, l_all = o[None], lse[None]
        return self.qsa.merge_attn_states(o_all, l_all, cfg=self.cfg)
