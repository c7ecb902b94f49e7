"""Query-row sharding of one long prefill across ranks (one process per GPU).

A QSA layer's query row t needs its own query, the compressed keys of the blocks
before it and the K/V rows of its selected blocks -- all inside the prefix
[0, t].  So a long sequence splits into contiguous row shards: rank j owns rows
[r0_j, r1_j) with their q, q_idx, w, k, v and k_idx (as a sequence-parallel
previous layer leaves them), and

  1. compresses the micro-blocks of its own rows (r0_j is a multiple of r, so no
     block straddles two ranks),
  2. all-gathers the compressed keys and the K/V rows (NCCL over NVLink on GPUs,
     gloo in the CPU tests),
  3. runs the fused index -> select and the sparse attention for its rows as a
     prefill with L_q = r1_j - r0_j queries against L_k = r1_j keys (the C ABI's
     bottom-right alignment puts query i of the shard at t = r0_j + i).

Rows cost unequal work: the attention gathers 2048 tokens per row (from a prefix,
and so an L2 hit rate, that depends on the row), the indexer grows with the number
of earlier blocks.  row_partition balances a cost a + b * floor(t / r) per row, so
later ranks get fewer rows.

The arithmetic of a row does not depend on which shard holds it, so the sharded
result equals the one-process result bit for bit.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch

ATTN_ROWS = 4096  # query rows per attention launch

# relative cost of a row: a constant part and a part per earlier block, fitted to the
# per-rank times of a 262144-token prefill sharded over 2 ranks on one B200 (0.38 us per
# row and 4.5 ps per (row, block) pair; the second term holds the fused indexer's pairs
# and the attention's falling L2 hit rate, its prefix of K/V growing with the row)
ATTN_ROW_COST = 0.38e-6
INDEX_PAIR_COST = 4.5e-12


def row_partition(n: int, world: int, r: int = 4, attn_cost: float = ATTN_ROW_COST,
                  pair_cost: float = INDEX_PAIR_COST) -> List[Tuple[int, int]]:
    """Contiguous row ranges [r0, r1) of an n-row prefill, one per rank, with equal
    modelled cost; every boundary is a multiple of r (the last range ends at n)."""
    if world < 1 or n < 0:
        raise ValueError("world >= 1 and n >= 0")
    nb = (n + r - 1) // r
    # cost of block-row group g (rows g r .. g r + r - 1, b_t = g for each)
    cum = [0.0]
    for g in range(nb):
        rows = min(r, n - g * r)
        cum.append(cum[-1] + rows * (attn_cost + pair_cost * g))
    total = cum[-1]
    bounds = [0]
    g = 0
    for j in range(1, world):
        target = total * j / world
        while g < nb and cum[g + 1] <= target:
            g += 1
        bounds.append(max(bounds[-1], min(g * r, n)))
    bounds.append(n)
    return [(bounds[j], bounds[j + 1]) for j in range(world)]


def gather_rows(local: torch.Tensor, sizes: Sequence[int], world: int, group=None) -> torch.Tensor:
    """All-gather of unequal row shards (rank j contributes sizes[j] rows of local):
    every rank gets the concatenation.  Shards are padded to the largest one."""
    if world == 1:
        return local
    import torch.distributed as dist
    dtype = local.dtype
    raw = local.contiguous().view(torch.uint8)  # the rows' bytes: every backend moves them
    mx = max(sizes)
    pad = raw.new_zeros((mx,) + tuple(raw.shape[1:]))
    pad[: raw.shape[0]] = raw
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[: sizes[j]] for j, p in enumerate(parts)], dim=0).view(dtype)


class ShardedPrefill:
    """One rank's share of a single-sequence QSA prefill (the library's kernels).

    gather(local, sizes) returns the concatenation of every rank's `local` (an
    NCCL all-gather in a multi-GPU job; see gather_rows).  The rank passes its own
    rows of q [n_local, 24, 256], k, v [n_local, 2, 256], q_idx [n_local, 4, 128],
    k_idx [n_local, 128] and w [n_local, 4]; the result is o for those rows."""

    def __init__(self, n: int, rank: int, world: int, chunk_rows: int = 16384, cfg=None, device="cuda",
                 gather: Optional[Callable] = None, parts: Optional[List[Tuple[int, int]]] = None):
        from . import qsa
        self.qsa = qsa
        self.cfg = qsa.default_config() if cfg is None else cfg
        self.r = self.cfg.r
        self.parts = parts if parts is not None else row_partition(n, world, self.r)
        self.rank, self.world = rank, world
        self.r0, self.r1 = self.parts[rank]
        self.n_local = self.r1 - self.r0
        self.gather = gather if gather is not None else (lambda t, sizes: gather_rows(t, sizes, world))
        self.chunk = int(chunk_rows)
        self.device = torch.device(device)
        dev = self.device
        self.cu_q = torch.tensor([0, self.n_local], dtype=torch.int32, device=dev)
        self.cu_k = torch.tensor([0, self.r1], dtype=torch.int32, device=dev)
        self.cu_b = torch.tensor([0, self.r1 // self.r], dtype=torch.int32, device=dev)
        self.cu_loc = torch.tensor([0, self.n_local], dtype=torch.int32, device=dev)
        self.cu_loc_b = torch.tensor([0, self.n_local // self.r], dtype=torch.int32, device=dev)
        self.sel = torch.empty((max(self.n_local, 1), self.cfg.budget_blocks), dtype=torch.int32, device=dev)
        rows = max(1, min(self.chunk, self.n_local))
        need = qsa.workspace_size(qsa.OP_INDEX_SELECT, 1, rows, max(self.r1, 1), self.cfg)
        self.ws = torch.empty((max(need, 16),), dtype=torch.uint8, device=dev)

    def block_sizes(self) -> List[int]:
        """Compressed blocks each rank contributes (the complete blocks of its rows)."""
        return [(b - a) // self.r for a, b in self.parts]

    def local_blocks(self, k_idx) -> torch.Tensor:
        """Step 1: the compressed keys of this rank's rows [n_local // r, 128] fp16."""
        assert self.r0 % self.r == 0, "shard starts must be multiples of r"
        nb = self.n_local // self.r
        kc = self.qsa.compress_keys(k_idx, self.cu_loc, self.cu_loc_b, n_blocks=max(nb, 1), cfg=self.cfg)
        return kc[:nb].contiguous()

    def attend(self, q, q_idx, w, kc_all, k_all, v_all, o=None):
        """Step 3: index -> select and attention of this rank's rows against the
        gathered prefix (kc_all, k_all, v_all hold at least the rows [0, r1))."""
        qsa = self.qsa
        kc_pre = kc_all[: self.r1 // self.r].contiguous()
        k_pre, v_pre = k_all[: self.r1].contiguous(), v_all[: self.r1].contiguous()
        if o is None:
            o = torch.empty_like(q)
        if self.n_local == 0:
            return o
        for a in range(0, self.n_local, self.chunk):
            b = min(self.n_local, a + self.chunk)
            qsa.index_select(q_idx, w, kc_pre, self.cu_q, self.cu_k, self.cu_b, self.n_local, self.r1, a, b,
                             sel=self.sel, ws=self.ws, cfg=self.cfg)
        for a in range(0, self.n_local, ATTN_ROWS):  # launches of ATTN_ROWS rows, as qsa.Prefill.attend
            qsa.sparse_attn_prefill(q, k_pre, v_pre, self.sel, self.cu_q, self.cu_k, a, min(self.n_local, a + ATTN_ROWS),
                                    o=o, cfg=self.cfg, max_len_k=self.r1)
        return o

    def __call__(self, q, k, v, q_idx, w, k_idx, o=None):
        row_sizes = [b - a for a, b in self.parts]
        kc = self.gather(self.local_blocks(k_idx), self.block_sizes())  # step 2: the all-gathers
        k_all = self.gather(k, row_sizes)
        v_all = self.gather(v, row_sizes)
        return self.attend(q, q_idx, w, kc, k_all, v_all, o=o)
