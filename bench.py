"""QSA benchmark: prefill tokens/s at 262,144 context and decode latency at 131,072.

One step = one pass of the whole QSA hot path on synthetic inputs resident in HBM:
  prefill  batch 1, n = 262,144: compress -> (index -> select) per chunk of query rows (--chunk-rows)
           -> sparse GQA attention                            (value = tokens/s of this part)
  decode   batch 64, every cache 131,072 tokens: refresh of the last compressed block,
           one-row indexer, top-512 select, split-K sparse attention (the "decode" object)
Inputs are drawn by block_sparse_long_09_b200.inputs (seeded, N(0,1) / U(0,1)); every
timed input is far larger than the 126 MB L2, so no flush is needed between steps.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl qsa|reference]
Multi-GPU (torchrun, one rank per GPU): every rank runs its own independent layer
(weak scaling, no collective on the data path); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import tempfile
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

N_PREFILL = 262144
DEC_BATCH = 64
DEC_LEN = 131072
MTP_NEXT_N = 4       # queries per sequence of the multi-token-prediction decode step
CHUNK = 65536          # query rows per fused index -> select launch (1024 row tiles: 7 waves on 148 SMs)
BUDGET = 512
METRIC = "QSA prefill tokens/s at 262K ctx; decode µs/token at 128K; % of roofline"

# DRAM traffic (read + write) of sparse_attn_kernel on the small profiling case
# (`bench.py --profile-case attn`: rows 122880..131071 of a 131072-token prefill,
# 8192 queries x 4 MiB = 34.36 GB gathered), from a one-kernel ncu capture; the
# full launch's traffic is estimated by scaling with the gathered bytes.  Valid
# only for the kernel sources it was taken on (checked by hash), null otherwise.
ATTN_SMALL_TRAFFIC = {"src_sha256_16": "afa9165f2aa7e996", "bytes": 15.96e9, "gather_bytes": 34.36e9}


def attn_src_hash() -> str:
    """Hash of the prefill attention kernel's sources (the traffic figure is valid only for them)."""
    h = hashlib.sha256()
    for f in ("attn.cu", "attn_common.cuh"):
        h.update(open(os.path.join(ROOT, "block_sparse_long_09_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, kind)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


class Clocks:
    """nvidia-smi sampler running during the timed region."""

    def __init__(self, index):
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), "qsa_clocks_rank%d.csv" % index)
        self.index = index

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index),
                 "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def gather_bytes_per_query(n_tokens_selected):
    # K and V, 2 KV heads x 256 dims x 2 bytes each
    return n_tokens_selected * 2 * 256 * 2 * 2


def selected_tokens(n, r=4, k=BUDGET):
    """Sum over queries of |T_t| (tokens actually attended), by the definition."""
    t = np.arange(n, dtype=np.int64)
    bt = t // r
    nblk = np.minimum(k, bt + 1)
    # every selected block is complete except the own block, which holds t - r*bt + 1 tokens
    return int(((nblk - 1) * r + (t - r * bt + 1)).sum())


def index_pairs(n, r=4):
    """Sum over queries of b_t = floor(t / r): the (row, candidate block) pairs the indexer scores."""
    t = np.arange(n, dtype=np.int64)
    return int((t // r).sum())


def decode_bytes(seqlens, kc_bytes_per_block, k=BUDGET, r=4):
    """Bytes one decode step must move: the kc scan, the scores written and read once
    by the selector, and the selected K/V tokens (2 KV heads x 256 x bf16, K and V)."""
    kc = sum((L // r) * kc_bytes_per_block for L in seqlens)
    scores = sum(((L - 1) // r) * 4 * 2 for L in seqlens)
    tok = sum(min(k - 1, (L - 1) // r) * r + ((L - 1) % r + 1) for L in seqlens)
    return kc + scores + gather_bytes_per_query(tok), kc, gather_bytes_per_query(tok)


def ev_ms(pairs):
    return float(np.mean([a.elapsed_time(b) for a, b in pairs])) if pairs else 0.0


def run_qsa(args, rank, world, device):
    from block_sparse_long_09_b200 import inputs, qsa, ranks

    hbm, tflops, tflops_sus, peak_kind = peaks()
    torch.manual_seed(0)
    seeds = ranks.rank_seeds(rank)
    x = inputs.make_prefill([N_PREFILL], seed=seeds["prefill"], device=device)
    cfg = qsa.default_config(budget_blocks=BUDGET)
    chunk = args.chunk_rows
    pre = qsa.Prefill([N_PREFILL], chunk_rows=chunk, cfg=cfg, device=device)
    o = torch.empty_like(x.q)

    d = inputs.make_decode(DEC_BATCH, DEC_LEN, None, seed=seeds["decode"], device=device)
    cu_k = d.cu_seqlens_k
    cu_b = d.cu_blocks
    kc_dec = qsa.compress_keys(d.k_idx, cu_k, cu_b, n_blocks=int(cu_b[-1]), cfg=cfg)
    kc_bpb = kc_dec[0].numel() * kc_dec.element_size()  # bytes of one compressed key
    last_blk = torch.tensor([L // 4 - 1 for L in d.seqlens], dtype=torch.int32, device=device)
    dec = qsa.DecodeStep(d.q, d.q_idx, d.w, d.k_cache, d.v_cache, d.k_idx, kc_dec, cu_k, cu_b, DEC_LEN,
                         refresh_blocks=last_blk, cfg=cfg, graph=True)
    dec_o = dec.o
    stream = torch.cuda.current_stream()
    n_chunks = (N_PREFILL + chunk - 1) // chunk

    ev = {k: [] for k in ("p0", "p1", "a0", "a1", "d0", "d1", "ix")}

    def mk():
        return torch.cuda.Event(enable_timing=True)

    def step(record):
        e = {k: mk() for k in ("p0", "p1", "a0", "a1", "d0", "d1")} if record else None
        if record:
            e["p0"].record(stream)
        # compress, then the fused index -> select per chunk (qsa.Prefill.index_select, with events)
        qsa.compress_keys(x.k_idx, pre.cu, pre.cu_blocks, kc=pre.kc, cfg=cfg)
        for r0 in range(0, N_PREFILL, chunk):
            r1 = min(N_PREFILL, r0 + chunk)
            e0, e1 = (mk(), mk()) if record else (None, None)
            if record:
                e0.record(stream)
            pre.select_chunk(x.q_idx, x.w, r0, r1)
            if record:
                e1.record(stream)
                ev["ix"].append((e0, e1))
        if record:
            e["a0"].record(stream)
        pre.attend(x.q, x.k, x.v, o=o)  # one pass over the keys per query, 4096 rows per launch
        if record:
            e["a1"].record(stream)
            e["p1"].record(stream)
            e["d0"].record(stream)
        dec()  # decode step: one CUDA-graph replay of its five launches
        if record:
            e["d1"].record(stream)
            for k in ("p0", "p1", "a0", "a1", "d0", "d1"):
                ev[k].append(e[k])

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    assert qsa.device_status() == 0, "a kernel flagged a device-side error during warm-up"

    clocks = Clocks(device.index if device.index is not None else 0)
    ranks.barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        step(True)
    t_end.record(stream)
    torch.cuda.synchronize()
    ranks.barrier(world)
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    prefill_ms = ev_ms(list(zip(ev["p0"], ev["p1"])))
    attn_ms = ev_ms(list(zip(ev["a0"], ev["a1"])))
    dec_ms = ev_ms(list(zip(ev["d0"], ev["d1"])))
    index_ms = ev_ms(ev["ix"]) * n_chunks  # per step: all chunks of the fused index -> select
    assert qsa.device_status() == 0, "a kernel flagged a device-side error in the timed region"

    def allmax(v):
        return ranks.max_over_ranks([v], world, device)[0]

    total_ms, prefill_ms, attn_ms, dec_ms, index_ms = ranks.max_over_ranks(
        [total_ms, prefill_ms, attn_ms, dec_ms, index_ms], world, device)

    def timed(fn, reps=5):
        fn()
        torch.cuda.synchronize()
        a, b = mk(), mk()
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return allmax(a.elapsed_time(b) / reps)

    # decode kernels one by one at 131072 (eager launches of the step's calls)
    # the decode selection reads the hi plane of kc (half of each compressed key), then
    # rescores each row's near-threshold window exactly
    dec_select_us = timed(lambda: qsa.index_select(dec.q_idx, dec.w, dec.kc, dec.cu_q, dec.cu_k, dec.cu_b, 1,
                                                   DEC_LEN, sel=dec.sel, ws=dec.ws_sel, cfg=cfg)) * 1e3
    dec_attn_us = timed(lambda: qsa.sparse_attn_decode(d.q, d.k_cache, d.v_cache, cu_k, dec.sel, o=dec_o, ws=dec.ws,
                                                       cfg=cfg)) * 1e3
    step_bytes, kc_scan, dec_gather = decode_bytes(d.seqlens, kc_bpb // 2)

    # multi-token-prediction decode at 131072: next_n = 4 new queries per sequence share one
    # selection (made from the last query's indexer scores) and one gather of its K/V
    g4 = torch.Generator(device=device)
    g4.manual_seed(seeds["decode"] + 7)
    q4 = torch.randn((DEC_BATCH, MTP_NEXT_N, 24, 256), generator=g4, device=device).to(torch.bfloat16)
    sel4 = torch.empty((DEC_BATCH, BUDGET), dtype=torch.int32, device=device)
    o4 = torch.empty_like(q4)
    ws4s = torch.empty((qsa.workspace_size(qsa.OP_INDEX_SELECT, DEC_BATCH, DEC_BATCH, DEC_LEN, cfg),),
                       dtype=torch.uint8, device=device)
    ws4a = torch.empty((max(qsa.workspace_size(qsa.OP_DECODE_MTP, DEC_BATCH, DEC_BATCH, 0, cfg), 16),),
                       dtype=torch.uint8, device=device)

    def mtp_select():
        qsa.index_select_mtp(dec.q_idx, dec.w, dec.kc, dec.cu_k, dec.cu_b, MTP_NEXT_N, DEC_LEN, sel=sel4, ws=ws4s,
                             cfg=cfg)

    def mtp_attend():
        qsa.sparse_attn_decode_mtp(q4, d.k_cache, d.v_cache, cu_k, sel4, o=o4, ws=ws4a, cfg=cfg)

    # the step as a CUDA graph (qsa.MtpStep): refresh of the block the 4 new tokens
    # completed, the shared selection and the attention; its parts launched eagerly
    mtp = qsa.MtpStep(q4, dec.q_idx, dec.w, d.k_cache, d.v_cache, d.k_idx, dec.kc, cu_k, dec.cu_b, DEC_LEN,
                      refresh_blocks=torch.tensor([(L - MTP_NEXT_N) // 4 for L in d.seqlens], dtype=torch.int32,
                                                  device=device), cfg=cfg, graph=True)
    mtp_step_us = timed(mtp, reps=10) * 1e3
    mtp_select_us = timed(mtp_select, reps=10) * 1e3
    mtp_attn_us = timed(mtp_attend, reps=10) * 1e3
    assert qsa.device_status() == 0
    del q4, sel4, o4, ws4s, ws4a, mtp

    # decode at 262144 tokens per sequence: the step, and the attention kernel alone
    del d, dec
    torch.cuda.empty_cache()
    d2 = inputs.make_decode(DEC_BATCH, 262144, None, seed=seeds["decode"] + 1, device=device)
    kc2 = qsa.compress_keys(d2.k_idx, d2.cu_seqlens_k, d2.cu_blocks, n_blocks=int(d2.cu_blocks[-1]), cfg=cfg)
    last2 = torch.tensor([L // 4 - 1 for L in d2.seqlens], dtype=torch.int32, device=device)
    dec2 = qsa.DecodeStep(d2.q, d2.q_idx, d2.w, d2.k_cache, d2.v_cache, d2.k_idx, kc2, d2.cu_seqlens_k,
                          d2.cu_blocks, 262144, refresh_blocks=last2, cfg=cfg, graph=True)
    step262_us = timed(dec2, reps=10) * 1e3
    attn262_us = timed(lambda: qsa.sparse_attn_decode(d2.q, d2.k_cache, d2.v_cache, d2.cu_seqlens_k, dec2.sel,
                                                      o=dec2.o, ws=dec2.ws, cfg=cfg), reps=10) * 1e3
    index262_us = timed(lambda: qsa.index_select(dec2.q_idx, dec2.w, dec2.kc, dec2.cu_q, dec2.cu_k, dec2.cu_b, 1,
                                                 262144, sel=dec2.sel, ws=dec2.ws_sel, cfg=cfg), reps=10) * 1e3
    step262_bytes, kc262, gather262 = decode_bytes(d2.seqlens, kc_bpb // 2)
    assert qsa.device_status() == 0
    del d2, kc2, dec2
    torch.cuda.empty_cache()

    # end to end through the public API: pinned host inputs in, result out, every step
    e2e = None
    if args.e2e_steps > 0:
        host = {k: getattr(x, k).cpu().pin_memory() for k in ("q", "k", "v", "q_idx", "k_idx", "w")}
        o_host = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = o_host.numel() * o_host.element_size()

        def e2e_step():  # copies in and out overlapped with the compute, chunk by chunk
            pre.from_host(host["q"], host["k"], host["v"], host["q_idx"], host["w"], host["k_idx"], o_host,
                          pipe_rows=args.e2e_rows)

        e2e_step()
        torch.cuda.synchronize()
        ranks.barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = allmax(e0.elapsed_time(e1) / args.e2e_steps)
        e2e = {"value": ranks.job_throughput(world, N_PREFILL, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "scope": "prefill 262144 via qsa.Prefill.from_host (pinned host in and out, copies overlapped "
                        "with the compute in chunks of %d rows, attention launches of %d rows)" % (
                            args.e2e_rows, pre.attn_rows)}
        # the same rows as the device-resident path of the timed steps, bit for bit
        assert torch.equal(o_host, o.cpu()), "the copy-overlapped prefill differs from the resident one"
        del host, o_host
        pre._stage = None

    # the build's dense causal attention on the same inputs (the pages' comparison)
    dense = None
    if args.dense:
        dd = inputs.make_decode(DEC_BATCH, DEC_LEN, None, seed=seeds["decode"], device=device)
        cu_dec_q = torch.arange(DEC_BATCH + 1, dtype=torch.int32, device=device)
        dec_o = torch.empty_like(dd.q)
        qsa.dense_attn_prefill(x.q, x.k, x.v, pre.cu, pre.cu, N_PREFILL, o=o, cfg=cfg, max_len_k=N_PREFILL)
        dws = torch.empty((qsa.workspace_size(qsa.OP_DENSE, DEC_BATCH, DEC_BATCH, DEC_LEN, cfg),),
                          dtype=torch.uint8, device=device)
        qsa.dense_attn_prefill(dd.q, dd.k_cache, dd.v_cache, cu_dec_q, dd.cu_seqlens_k, 1, o=dec_o, cfg=cfg,
                               max_len_k=DEC_LEN, ws=dws)
        torch.cuda.synchronize()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        e[0].record(stream)
        qsa.dense_attn_prefill(x.q, x.k, x.v, pre.cu, pre.cu, N_PREFILL, o=o, cfg=cfg, max_len_k=N_PREFILL)
        e[1].record(stream)
        for _ in range(5):
            qsa.dense_attn_prefill(dd.q, dd.k_cache, dd.v_cache, cu_dec_q, dd.cu_seqlens_k, 1, o=dec_o, cfg=cfg,
                                   max_len_k=DEC_LEN, ws=dws)
        e[2].record(stream)
        torch.cuda.synchronize()
        dp_ms = allmax(e[0].elapsed_time(e[1]))
        dd_us = allmax(e[1].elapsed_time(e[2]) / 5 * 1e3)
        dense_flops = 4.0 * 24 * 256 * (N_PREFILL * (N_PREFILL + 1) / 2)
        dense = {"prefill_ms": dp_ms, "prefill_tokens_per_s": N_PREFILL / (dp_ms / 1e3),
                 "prefill_tflops": dense_flops / (dp_ms / 1e3) / 1e12,
                 "qsa_layer_speedup": dp_ms / prefill_ms, "qsa_attention_only_speedup": dp_ms / attn_ms,
                 "decode_step_us": dd_us, "qsa_decode_speedup": dd_us / (dec_ms * 1e3),
                 "pages_context": "7.6x prefill / 4.9x decode at 1M context, kernel level, hardware not stated"}
        del dd

    sel_tok = selected_tokens(N_PREFILL)
    gather = gather_bytes_per_query(1) * sel_tok
    attn_flops = 24 * 256 * 4 * sel_tok
    pairs = index_pairs(N_PREFILL)
    traffic = None
    if attn_src_hash() == ATTN_SMALL_TRAFFIC["src_sha256_16"] and world == 1:
        traffic = ATTN_SMALL_TRAFFIC["bytes"] * gather / ATTN_SMALL_TRAFFIC["gather_bytes"]
    attn_tflops = attn_flops / (attn_ms / 1e3) / 1e12
    # compress; 5 launches of the fused index -> select per chunk; the attention per pre.attn_rows rows
    launches_prefill = 1 + 5 * n_chunks + (N_PREFILL + pre.attn_rows - 1) // pre.attn_rows
    launches_decode = 1 + 4 + 2               # refresh; hi-plane scan, count reset, refine, fallback; attention + merge
    kern = {
        "sparse_attn_prefill": {
            "ms": attn_ms, "bound": "tensor", "flop": attn_flops, "achieved_tflops": attn_tflops,
            "peak_tflops": tflops_sus, "frac": attn_tflops / tflops_sus,
            "gather_bytes": gather, "effective_gather_TBps": gather / (attn_ms / 1e3) / 1e12,
            "dram_traffic_est": traffic,
            "dram_frac": (traffic / (attn_ms / 1e3) / 1e9 / hbm) if traffic else None},
        "index_select": {
            "ms_per_step": index_ms, "bound": "tensor", "method_flop": 1024.0 * pairs,
            "achieved_tflops": 1024.0 * pairs / (index_ms / 1e3) / 1e12, "peak_tflops": tflops_sus,
            "frac": 1024.0 * pairs / (index_ms / 1e3) / 1e12 / tflops_sus,
            "note": "fused: sampled thresholds, candidate lists, exact top-k; no score rows in memory"},
        "decode_131k": {
            "step_us": dec_ms * 1e3, "step_bytes": step_bytes,
            "step_frac": step_bytes / (dec_ms / 1e3) / 1e9 / hbm,
            "index_select_us": dec_select_us, "kc_scan_bytes": kc_scan,
            "index_select_frac": kc_scan / (dec_select_us / 1e6) / 1e9 / hbm,
            "attn_us": dec_attn_us, "attn_bytes": dec_gather,
            "attn_frac": dec_gather / (dec_attn_us / 1e6) / 1e9 / hbm},
        "decode_mtp_131k": {
            "next_n": MTP_NEXT_N, "batch": DEC_BATCH, "step_us": mtp_step_us,
            "us_per_token": mtp_step_us / MTP_NEXT_N,
            "index_select_us": mtp_select_us, "attn_us": mtp_attn_us, "attn_bytes": dec_gather,
            "attn_frac": dec_gather / (mtp_attn_us / 1e6) / 1e9 / hbm,
            "note": "step: qsa.MtpStep graph replay (refresh, shared selection, attention); parts: eager launches; one shared selection and one K/V gather serve the 4 queries of a sequence"},
        "decode_262k": {
            "step_us": step262_us, "step_bytes": step262_bytes,
            "step_frac": step262_bytes / (step262_us / 1e6) / 1e9 / hbm,
            "index_select_us": index262_us, "kc_scan_bytes": kc262,
            "index_select_frac": kc262 / (index262_us / 1e6) / 1e9 / hbm,
            "attn_us": attn262_us, "attn_bytes": gather262,
            "attn_frac": gather262 / (attn262_us / 1e6) / 1e9 / hbm},
    }
    res = {
        "metric": METRIC,
        "value": ranks.job_throughput(world, N_PREFILL, prefill_ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) activations, U(0,1) indexer weights)",
        "config": {"workload": "QSA layer: prefill batch 1 n=262144 (%d-row chunks) + decode batch 64 ctx 131072"
                                % chunk,
                   "budget_blocks": BUDGET, "r": 4, "heads": "24q/2kv/256, indexer 4/128",
                   "prefill_ms": prefill_ms, "attn_prefill_ms": attn_ms, "l2": "inputs > L2, no flush",
                   "parallelism": "independent layer per rank" if world > 1 else "1 GPU"},
        "decode": {"batch": DEC_BATCH, "ctx": DEC_LEN, "step_us": dec_ms * 1e3, "us_per_token": dec_ms * 1e3,
                   "us_per_token_amortized": dec_ms * 1e3 / DEC_BATCH},
        "roofline": {"kernel": "sparse_attn_kernel (prefill)", "bound": "tensor", "achieved": attn_tflops,
                     "peak": tflops_sus, "unit": "TFLOP/s", "frac": attn_tflops / tflops_sus, "traffic": traffic,
                     "peak_kind": peak_kind + " (sustained bf16: the kernel runs inside a long step)",
                     # the bounds' times: the method's flops at the tensor peak, the gathered bytes at
                     # the HBM copy peak (no L2 reuse), and the measured DRAM traffic at that peak
                     "bound_ms": {"tensor": attn_flops / (tflops_sus * 1e12) * 1e3,
                                  "gather_at_hbm": gather / (hbm * 1e9) * 1e3,
                                  "dram_traffic_at_hbm": (traffic / (hbm * 1e9) * 1e3) if traffic else None,
                                  "measured": attn_ms},
                     "note": "gather-bound: 4 MiB of K/V per query against 25 MFLOP; see kernels"},
        "kernels": kern,
        "gpu_launches": args.steps * (launches_prefill + launches_decode),
        "dense": dense,
        "e2e": e2e,
        "clocks": clk,
    }
    return res


def cpu_model() -> str:
    """The host CPU's model string (from /proc/cpuinfo), for the baseline's record."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(seconds: float = 12.0, rows_hint: int = 16):
    """The fp64 oracle, as it stands, on a bounded sample of the prefill workload:
    for each sampled query row the whole chain (scores against every earlier
    compressed block, top-512 selection, attention over the selected tokens),
    after one compression of all keys."""
    import oracle
    from block_sparse_long_09_b200 import inputs

    x = inputs.make_prefill([N_PREFILL], seed=0, device="cuda" if torch.cuda.is_available() else "cpu")

    def bits(t):
        return np.ascontiguousarray(t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16))

    k_idx, k, v = bits(x.k_idx), bits(x.k), bits(x.v)
    rng = np.random.default_rng(0)
    cores = oracle.threads()

    def run(rows):
        rows = np.sort(rows)
        q, q_idx, w = bits(x.q[rows]), bits(x.q_idx[rows]), x.w[rows].cpu().numpy()
        t0 = time.perf_counter()
        kc = oracle.compress(k_idx, 4)
        ld = (N_PREFILL - 1) // 4
        sc = np.empty((len(rows), ld))
        for j, i in enumerate(rows):  # query row j sits at position i: Lq = 1, Lk = i + 1
            sc[j] = oracle.index_scores(q_idx[j:j + 1], w[j:j + 1], kc, 1, int(i) + 1, 4, [0], ld=ld)[0]
        sel = oracle.select(sc, rows // 4, BUDGET)
        for j, i in enumerate(rows):
            oracle.attend(q[j:j + 1], k, v, sel[j:j + 1], 1, int(i) + 1, 4, 1 / 16, [0])
        return time.perf_counter() - t0

    n = rows_hint
    t = run(rng.integers(N_PREFILL // 2, N_PREFILL, n))
    if t < seconds / 3:
        n = max(n, int(n * seconds / max(t, 1e-3)))
        t = run(rng.integers(N_PREFILL // 2, N_PREFILL, n))
    return {"value": n / t, "unit": "tokens/s", "cores": cores, "kind": "oracle", "cpu": cpu_model(),
            "nproc": os.cpu_count(),
            "sample": "%d random query rows from the second half of the 262144-token prefill: compress of all "
                      "keys once, then per row scores, top-512 select and attention, fp64, %.1f s" % (n, t)}


def run_extra_configs(steps: int = 5, warmup: int = 3):
    """The other workloads of the measurement plan, one line each on stderr (the bench's
    own JSON line on stdout is unchanged): prefill of 2 x 65536 tokens with peaked indexer
    keys, decode steps at 262144 tokens and at mixed lengths U{32768 .. 262144}, and the
    1M-token context of the pages' comparison (run_context_1m)."""
    from block_sparse_long_09_b200 import inputs, qsa

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    cfg = qsa.default_config(budget_blocks=BUDGET)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        assert qsa.device_status() == 0
        return e0.elapsed_time(e1) / steps

    # prefill, 2 sequences of 65536 tokens, per-block offsets in k_I (peaked selections)
    lens = [65536, 65536]
    x = inputs.make_prefill(lens, seed=0, peaked=True, device=dev)
    pre = qsa.Prefill(lens, chunk_rows=CHUNK, cfg=cfg, device=dev)
    o = torch.empty_like(x.q)
    ms = timed(lambda: pre(x.q, x.k, x.v, x.q_idx, x.w, x.k_idx, o=o))
    att = timed(lambda: pre.attend(x.q, x.k, x.v, o=o))
    sel_tok = sum(selected_tokens(L) for L in lens)
    print(json.dumps({"workload": "prefill 2 x 65536, peaked k_I (one c_b ~ N(0, 0.5^2) per block)",
                      "prefill_ms": ms, "tokens_per_s": sum(lens) / (ms / 1e3), "attn_ms": att,
                      "attn_gather_TBps": gather_bytes_per_query(1) * sel_tok / (att / 1e3) / 1e12}),
          file=sys.stderr)
    del x, pre, o
    torch.cuda.empty_cache()
    # decode, batch 64, every sequence at 262144 tokens and at mixed lengths
    for name, lo, hi in (("decode batch 64, all L = 262144", 262144, None),
                         ("decode batch 64, L ~ U{32768 .. 262144}", 32768, 262144)):
        d = inputs.make_decode(DEC_BATCH, lo, hi, seed=0, device=dev)
        kc = qsa.compress_keys(d.k_idx, d.cu_seqlens_k, d.cu_blocks, n_blocks=int(d.cu_blocks[-1]), cfg=cfg)
        last = torch.tensor([L // 4 - 1 for L in d.seqlens], dtype=torch.int32, device=dev)
        dec = qsa.DecodeStep(d.q, d.q_idx, d.w, d.k_cache, d.v_cache, d.k_idx, kc, d.cu_seqlens_k, d.cu_blocks,
                             max(d.seqlens), refresh_blocks=last, cfg=cfg, graph=True)
        us = timed(dec) * 1e3
        print(json.dumps({"workload": name, "step_us": us, "us_per_token_amortized": us / DEC_BATCH}),
              file=sys.stderr)
        del d, kc, dec
        torch.cuda.empty_cache()
    run_context_1m(timed, cfg, dev)
    run_sharded_emulation(cfg, dev)


def run_sharded_emulation(cfg, dev, worlds=(2, 4, 8), reps=3):
    """The row-sharded prefill of 262144 tokens (block_sparse_long_09_b200.sharded) with
    its N ranks emulated one after another on this GPU: each rank's fused index -> select
    and attention over its own rows against the gathered prefix, timed alone (no rank
    waits for another).  The slowest rank bounds an N-GPU step; the all-gathers of the
    compressed keys and K/V rows are not run here and are estimated at the measured
    770 GB/s peer bandwidth per direction (each rank receives the others' rows)."""
    from block_sparse_long_09_b200 import inputs, qsa
    from block_sparse_long_09_b200.sharded import ShardedPrefill, row_partition

    n = N_PREFILL
    x = inputs.make_prefill([n], seed=0, device=dev)
    one = qsa.Prefill([n], chunk_rows=CHUNK, cfg=cfg, device=dev)
    o = torch.empty_like(x.q)

    def ev_time(fn):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    one_ms = ev_time(lambda: one(x.q, x.k, x.v, x.q_idx, x.w, x.k_idx, o=o))
    kv_row_bytes = 2 * (2 * 256 * 2) + (2 * 128 * 2) // 4  # a token's K and V rows, a quarter of a compressed key
    for world in worlds:
        parts = row_partition(n, world)
        shards = [ShardedPrefill(n, j, world, chunk_rows=CHUNK, cfg=cfg, parts=parts, device=dev)
                  for j in range(world)]
        kc_all = torch.cat([sh.local_blocks(x.k_idx[a:b].contiguous()) for sh, (a, b) in zip(shards, parts)])
        rank_ms = []
        for sh, (a, b) in zip(shards, parts):
            qa, qia, wa = x.q[a:b].contiguous(), x.q_idx[a:b].contiguous(), x.w[a:b].contiguous()
            oa = torch.empty_like(qa)
            rank_ms.append(ev_time(lambda: sh.attend(qa, qia, wa, kc_all, x.k, x.v, o=oa)))
            del qa, qia, wa, oa
        gather_ms = max((n - (b - a)) * kv_row_bytes for a, b in parts) / 770e9 * 1e3
        assert qsa.device_status() == 0
        print(json.dumps({"workload": "row-sharded prefill of %d tokens, %d ranks emulated on one GPU" % (n, world),
                          "rows_per_rank": [b - a for a, b in parts], "rank_ms": rank_ms,
                          "slowest_rank_ms": max(rank_ms), "balance": min(rank_ms) / max(rank_ms),
                          "one_gpu_ms": one_ms, "gather_ms_estimated": gather_ms,
                          "projected_speedup": one_ms / (max(rank_ms) + gather_ms),
                          "note": "ranks timed one after another; the all-gathers estimated, not run"}),
              file=sys.stderr)
        del shards, kc_all
        torch.cuda.empty_cache()
    del x, one, o
    torch.cuda.empty_cache()


def run_context_1m(timed, cfg, dev):
    """The regime of the pages' kernel-level comparison (1M-token context): the prefill of
    one 1048576-token sequence against this build's dense causal kernel, and decode at
    batch 4 (the pages' decode batch, with next_n = 4) against the dense split-K decode of
    one query per sequence -- a lower bound of any dense step, which reads every cached
    token at least once."""
    from block_sparse_long_09_b200 import inputs, qsa

    n = 1 << 20
    x = inputs.make_prefill([n], seed=0, device=dev)
    pre = qsa.Prefill([n], chunk_rows=CHUNK, cfg=cfg, device=dev)
    o = torch.empty_like(x.q)
    qsa_ms = timed(lambda: pre(x.q, x.k, x.v, x.q_idx, x.w, x.k_idx, o=o))
    att_ms = timed(lambda: pre.attend(x.q, x.k, x.v, o=o))
    qsa.dense_attn_prefill(x.q, x.k, x.v, pre.cu, pre.cu, n, o=o, cfg=cfg, max_len_k=n)  # warm-up
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    qsa.dense_attn_prefill(x.q, x.k, x.v, pre.cu, pre.cu, n, o=o, cfg=cfg, max_len_k=n)
    e1.record()
    torch.cuda.synchronize()
    dense_ms = e0.elapsed_time(e1)
    assert qsa.device_status() == 0
    print(json.dumps({"workload": "prefill 1 x 1048576 (k = 512)", "prefill_ms": qsa_ms,
                      "tokens_per_s": n / (qsa_ms / 1e3), "attn_ms": att_ms, "dense_prefill_ms": dense_ms,
                      "qsa_layer_speedup": dense_ms / qsa_ms, "qsa_attention_only_speedup": dense_ms / att_ms,
                      "pages": "7.6x prefill at 1M context, kernel level, hardware not stated"}), file=sys.stderr)
    del x, pre, o
    torch.cuda.empty_cache()

    batch, next_n = 4, MTP_NEXT_N
    d = inputs.make_decode(batch, n, None, seed=0, device=dev, next_n=next_n)
    kc = qsa.compress_keys(d.k_idx, d.cu_seqlens_k, d.cu_blocks, n_blocks=int(d.cu_blocks[-1]), cfg=cfg)
    q1 = d.q[:, -1].contiguous()  # the last query of each sequence: plain decode
    last = torch.tensor([L // 4 - 1 for L in d.seqlens], dtype=torch.int32, device=dev)
    dec = qsa.DecodeStep(q1, d.q_idx, d.w, d.k_cache, d.v_cache, d.k_idx, kc, d.cu_seqlens_k, d.cu_blocks, n,
                         refresh_blocks=last, cfg=cfg, graph=True)
    dec_us = timed(dec) * 1e3
    mtp = qsa.MtpStep(d.q, d.q_idx, d.w, d.k_cache, d.v_cache, d.k_idx, kc, d.cu_seqlens_k, d.cu_blocks, n,
                      refresh_blocks=torch.tensor([(L - next_n) // 4 for L in d.seqlens], dtype=torch.int32,
                                                  device=dev), cfg=cfg, graph=True)
    mtp_us = timed(mtp) * 1e3
    cu_q = torch.arange(batch + 1, dtype=torch.int32, device=dev)
    dws = torch.empty((qsa.workspace_size(qsa.OP_DENSE, batch, batch, n, cfg),), dtype=torch.uint8, device=dev)
    od = torch.empty_like(q1)
    dense_us = timed(lambda: qsa.dense_attn_prefill(q1, d.k_cache, d.v_cache, cu_q, d.cu_seqlens_k, 1, o=od,
                                                    cfg=cfg, max_len_k=n, ws=dws)) * 1e3
    print(json.dumps({"workload": "decode batch 4 at 1048576 tokens", "step_us": dec_us,
                      "mtp_next_n": next_n, "mtp_step_us": mtp_us, "mtp_us_per_token": mtp_us / next_n,
                      "dense_decode_us": dense_us, "qsa_decode_speedup": dense_us / dec_us,
                      "qsa_mtp_speedup_per_token": dense_us / (mtp_us / next_n),
                      "pages": "4.9x decode at 1M context with next_n = 4, kernel level, hardware not stated"}),
          file=sys.stderr)
    del d, kc, dec, mtp, dws, od
    torch.cuda.empty_cache()


def run_profile_case(case: str, reps: int = 3):
    """Small cases for ncu captures of one kernel (a few GB on the device, K/V larger than L2)."""
    from block_sparse_long_09_b200 import inputs, qsa

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    cfg = qsa.default_config(budget_blocks=BUDGET)
    if case in ("attn", "index", "select", "index_select"):
        n, rows = 131072, 8192
        x = inputs.make_prefill([n], seed=0, device=dev)
        pre = qsa.Prefill([n], chunk_rows=rows, cfg=cfg, device=dev, fused=case in ("attn", "index_select"))
        qsa.compress_keys(x.k_idx, pre.cu, pre.cu_blocks, kc=pre.kc, cfg=cfg)
        r0 = n - rows
        for _ in range(reps):
            pre.select_chunk(x.q_idx, x.w, r0, n)
            if case == "attn":
                qsa.sparse_attn_prefill(x.q, x.k, x.v, pre.sel, pre.cu, pre.cu, r0, n, cfg=cfg, max_len_k=n)
    elif case == "mtp":
        # multi-token decode (next_n = 4) at batch 64 with 65536-token caches
        L = 65536
        d = inputs.make_decode(DEC_BATCH, L, None, seed=2, device=dev, next_n=MTP_NEXT_N)
        kc = qsa.compress_keys(d.k_idx, d.cu_seqlens_k, d.cu_blocks, n_blocks=int(d.cu_blocks[-1]), cfg=cfg)
        for _ in range(reps):
            sel = qsa.index_select_mtp(d.q_idx, d.w, kc, d.cu_seqlens_k, d.cu_blocks, MTP_NEXT_N, L, cfg=cfg)
            qsa.sparse_attn_decode_mtp(d.q, d.k_cache, d.v_cache, d.cu_seqlens_k, sel, cfg=cfg)
    elif case == "decode1m":
        # decode steps at batch 4 with 1048576-token caches (the pages' decode regime): the
        # small-batch selection path (bound and list launches before the refine); 10 GB
        L, B = 1 << 20, 4
        d = inputs.make_decode(B, L, None, seed=1, device=dev)
        cu_q = torch.arange(B + 1, dtype=torch.int32, device=dev)
        kc = qsa.compress_keys(d.k_idx, d.cu_seqlens_k, d.cu_blocks, n_blocks=int(d.cu_blocks[-1]), cfg=cfg)
        ws = torch.empty((qsa.workspace_size(qsa.OP_INDEX_SELECT, B, B, L, cfg),), dtype=torch.uint8, device=dev)
        for _ in range(reps):
            sel = qsa.index_select(d.q_idx, d.w, kc, cu_q, d.cu_seqlens_k, d.cu_blocks, 1, L, ws=ws, cfg=cfg)
            qsa.sparse_attn_decode(d.q, d.k_cache, d.v_cache, d.cu_seqlens_k, sel, cfg=cfg)
    elif case in ("decode", "decode64k", "decode131k"):
        # decode steps of batch 64 (16384-token caches: small; 65536: kc hi planes of 268 MB,
        # above L2, 5.5 GB on the device; 131072: the benchmark's, 11 GB)
        L = {"decode": 16384, "decode64k": 65536, "decode131k": DEC_LEN}[case]
        d = inputs.make_decode(DEC_BATCH, L, None, seed=1, device=dev)
        cu_q = torch.arange(DEC_BATCH + 1, dtype=torch.int32, device=dev)
        kc = qsa.compress_keys(d.k_idx, d.cu_seqlens_k, d.cu_blocks, n_blocks=int(d.cu_blocks[-1]), cfg=cfg)
        ws = torch.empty((qsa.workspace_size(qsa.OP_INDEX_SELECT, DEC_BATCH, DEC_BATCH, L, cfg),), dtype=torch.uint8,
                         device=dev)
        for _ in range(reps):
            sel = qsa.index_select(d.q_idx, d.w, kc, cu_q, d.cu_seqlens_k, d.cu_blocks, 1, L, ws=ws, cfg=cfg)
            qsa.sparse_attn_decode(d.q, d.k_cache, d.v_cache, d.cu_seqlens_k, sel, cfg=cfg)
    torch.cuda.synchronize()
    assert qsa.device_status() == 0
    print("profile case %s done" % case)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="qsa", choices=["qsa", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--e2e-rows", type=int, default=8192, help="query rows per copy chunk of the e2e leg (q, k, v in, o out)")
    ap.add_argument("--chunk-rows", type=int, default=CHUNK,
                    help="query rows per fused index -> select launch of the prefill")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", dest="dense", action="store_false",
                    help="skip the dense causal-attention comparison")
    ap.add_argument("--extra-configs", action="store_true",
                    help="time the other workloads instead (peaked 2 x 65536 prefill, decode at 262144 and mixed "
                         "lengths, the 1M-token comparison, the sharded-prefill emulation) and print them on stderr")
    ap.add_argument("--sharded-emulation", action="store_true",
                    help="time the row-sharded prefill's ranks one after another on this GPU (also part of "
                         "--extra-configs) and print one line per rank count on stderr")
    ap.add_argument("--profile-case", choices=["attn", "index", "select", "index_select", "decode", "decode64k", "decode131k", "decode1m",
                             "mtp"],
                    default=None,
                    help="run one small case for an ncu capture and exit")
    args = ap.parse_args()
    if args.profile_case:
        import block_sparse_long_09_b200.build as bld
        bld.build()
        run_profile_case(args.profile_case)
        return
    if args.extra_configs:
        import block_sparse_long_09_b200.build as bld
        bld.build()
        run_extra_configs(args.steps, args.warmup)
        return
    if args.sharded_emulation:
        import block_sparse_long_09_b200.build as bld
        from block_sparse_long_09_b200 import qsa
        bld.build()
        torch.cuda.set_device(0)
        run_sharded_emulation(qsa.default_config(budget_blocks=BUDGET), torch.device("cuda", 0))
        return

    from block_sparse_long_09_b200 import ranks
    env = ranks.env_ranks()
    world, rank, local = env["world"], env["rank"], env["local"]

    if args.impl == "reference":
        if rank != 0:
            return
        t0 = time.perf_counter()
        steps = []
        for _ in range(args.warmup + args.steps):
            steps.append(cpu_baseline(seconds=4.0, rows_hint=8))
        b = steps[args.warmup:]
        val = float(np.mean([s["value"] for s in b]))
        res = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": args.gpus,
               "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * (time.perf_counter() - t0) / len(steps),
               "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
               "data": "synthetic", "config": {"workload": "QSA prefill batch 1 n=262144, sampled rows (fp64 oracle)"},
               "cpu_baseline": {"value": val, "unit": "tokens/s", "kind": "oracle", "cores": b[0]["cores"],
                                "cpu": b[0]["cpu"], "nproc": b[0]["nproc"], "sample": b[0]["sample"]},
               "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(res))
        return

    import block_sparse_long_09_b200.build as bld
    bld.build()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    ranks.init("nccl", world, device)
    res = run_qsa(args, rank, world, device)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(res))
    ranks.finish(world)


if __name__ == "__main__":
    main()
