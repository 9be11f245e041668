"""Benchmark of the LVSA block-sparse attention path on B200.

A step is one pass of the LVSA hot path over one batch of the Wan-2.1-1.3B-
like 6x-length workload (B=1, 12 heads, D=128, grid 126x30x52 = 196,560
tokens, C=21, T_per=12), with s = step mod T_per: natural-layout Q, K, V in,
natural-layout O out.  The step runs bsa_lvsa_attn_fwd, the one-kernel path
(frame sets computed in the kernel, the reorder fused into its tile loads).
The four-kernel path over the same data (lvsa_mask -> reorder_fwd ->
attn_fwd on the block list -> reorder_inv) is timed too and reported per
kernel.  Inputs (1.8 GB) exceed the 126 MB L2, so no flush is needed.  The
end-to-end figure copies every step's Q, K, V in from pinned host memory
and its O out, overlapped with the neighbouring steps' compute
(pipeline.StreamedSteps).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --kernel-table      # every kernel on every workload, one JSON line each
    python bench.py --draft-pipelines H # the three draft pipelines, twice, on H heads
                                        # of the 40-head draft workload (for profilers)
    python bench.py --hbm-kernels C     # every HBM-bound kernel, twice, on workload C
                                        # (for DRAM-counter captures)

Under torchrun (N > 1) every rank runs its own batch (the path shards over
batch x heads with no data exchange): weak scaling, max time over ranks.
`--impl reference` times the CPU fp64 oracle on a bounded sample instead.
Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import CONFIGS, make_qkv  # noqa: E402

NOMINAL_BF16_TFLOPS = 2250.0  # B200 dense bf16, NVIDIA's figure (context only)

METRIC = "bsattn ms/call + attended TFLOP/s (% BF16 peak), Wan-1.3B-shape 6× length LVSA"

# DRAM bytes per launch of the LVSA step kernel at the full Wan-1.3B 6x
# workload: dram__bytes_read.sum + dram__bytes_write.sum of one ncu capture of
# the same kernel on the first 24 frames (445.7 MB), scaled by the number of
# query pairs (126 / 24).  None whenever the kernel has changed since.
STEP_KERNEL_DRAM_BYTES = 445.7e6 * 126 / 24
STEP_KERNEL_TRAFFIC_SOURCE = ("ncu capture of lvsa_attn_kernel (key masks from the mask warp) "
                              "on the first 24 frames (445.7 MB), scaled by 126/24; not "
                              "measured by this run")


def attended_flops(w) -> float:
    # T*C*P^2 (query, key) pairs per head, 4*D flops each (QK and PV products)
    return float(w.T * w.lvsa_C * w.P * w.P) * w.Hh * w.B * 4 * w.D


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        # the profiling recipe's fallback for this machine's B200s (an earlier
        # measurement: STREAM-style copy, cuBLAS bf16 burst and sustained)
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev: int):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(dev).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            ident = str(dev)
        self.ident = ident

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.ident, f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise maximum of per-rank timings (the whole job is as slow as
    its slowest rank).  Works with any torch.distributed backend; without a
    process group it returns the values unchanged."""
    vals = [float(v) for v in values]
    if dist is None or not dist.is_available() or not dist.is_initialized():
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def weak_scaling_value(flops_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job attended TFLOP/s: every rank ran its own batch in ms_max."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


def cpu_baseline(w, q_h, k_h, v_h, budget_s: float, seed: int = 0):
    """The oracle, as it stands, on a bounded sample of the same workload:
    the LVSA mask of step 0 in full, then masked attention of sampled query
    blocks of one head.  Returns (attended TFLOP/s, threads, description)."""
    import oracle
    nbf = -(-w.P // 128)
    t0 = time.perf_counter()
    A = oracle.lvsa_frame_sets(w.T, w.lvsa_C, w.lvsa_T_per, 0)
    rp, ci = oracle.lvsa_block_csr(A, nbf)
    perm, Np = oracle.frame_layout_perm(w.T, w.H, w.W, 128)
    valid = oracle.slot_valid(perm, Np)
    qs, ks, vs = (oracle.reorder_fwd(x, perm, Np) for x in (q_h, k_h, v_h))
    setup = time.perf_counter() - t0
    rng = np.random.default_rng(seed)
    nb = w.T * nbf
    done, flops, t_att = 0, 0.0, 0.0
    while t_att < budget_s and done < nb:
        qb = int(rng.integers(0, nb))
        t1 = time.perf_counter()
        oracle.masked_attention(qs, ks, vs, valid, 128, rp, ci, False, 1 / math.sqrt(w.D),
                                q_blocks=[qb], heads=[(0, 0)])
        t_att += time.perf_counter() - t1
        nq = int(valid[qb * 128:(qb + 1) * 128].sum())
        keys = sum(int(valid[c * 128:(c + 1) * 128].sum()) for c in ci[rp[qb]:rp[qb + 1]])
        flops += 4.0 * w.D * nq * keys
        done += 1
    threads = torch.get_num_threads()
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        threads = max([i.get("num_threads", 1) for i in info] + [1])
    except Exception:
        pass
    desc = (f"oracle masked attention on {done} random query blocks of head 0 (of "
            f"{nb} x {w.Hh}), LVSA s=0; mask+layout set-up {setup:.1f}s excluded")
    return flops / t_att / 1e12, threads, desc, t_att


def run_reference(args, rank, world):
    """Reference arm: the CPU fp64 oracle, timed on the host cores."""
    if rank != 0:
        return
    w = CONFIGS[args.config]
    q, k, v = make_qkv(w, device="cpu")
    q_h, k_h, v_h = (x[:, :, :1].float().numpy().astype(np.float64) for x in (q, k, v))
    del q, k, v
    vals = []
    desc, thr = "", 1
    # each step samples for at most ref_step_s, less when there are many
    # steps, so the whole run stays near two minutes of host time
    n_all = args.warmup + args.steps
    budget = min(args.ref_step_s, max(0.25, 120.0 / n_all))
    for i in range(n_all):
        if w.lvsa_C:
            val, thr, desc, _ = cpu_baseline(w, q_h, k_h, v_h, budget_s=budget, seed=i)
        else:
            val, thr, desc, _ = cpu_baseline_draft(w, q_h, k_h, v_h, budget, seed=i)
        if i >= args.warmup:
            vals.append(val)
    value = statistics.mean(vals)
    line = {
        "impl": "reference",
        "metric": METRIC if w.lvsa_C else
        f"bsattn ms/call + attended TFLOP/s (% BF16 peak), {w.name}, draft attention",
        "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "global_batch": w.B, "seq_len": w.N,
                   "parallelism": f"dp{world}"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def draft_attended_flops(w, kv_idx_host: np.ndarray, keep: int) -> float:
    """4*D flops per (valid query, valid key) pair of every kept block pair.
    Blocks are the ph x pw tiles of the tile layout, in (t, i, j) order."""
    ph, pw = w.draft_ph, w.draft_pw
    TH, TW = -(-w.H // ph), -(-w.W // pw)
    vi = np.minimum(ph, w.H - np.arange(TH) * ph)
    vj = np.minimum(pw, w.W - np.arange(TW) * pw)
    nv = np.tile(np.outer(vi, vj).ravel(), w.T).astype(np.int64)
    nb = nv.size
    idx = kv_idx_host.reshape(-1, nb, keep)
    pairs = int((nv[None, :, None] * nv[idx]).sum())
    return 4.0 * w.D * pairs


def kernel_table(args):
    """ms per call of every kernel of both paths on every workload, with the
    algorithmic bytes (HBM-bound kernels) or attended flops (attention).  L2
    is flushed (a 256 MB write) before every timed call."""
    import block_sparse_attention_49_b200 as bsa
    from block_sparse_attention_49_b200.pipeline import DraftAttention, LvsaAttention

    pk, pk_kind = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def timed(fn, reps=args.table_reps):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    def emit(cid, kernel, ms, algo_bytes=None, flops=None, note=None, e4m3=False):
        d = {"config": cid, "workload": CONFIGS[cid].name, "kernel": kernel, "ms": round(ms, 4)}
        if algo_bytes is not None:
            gbs = algo_bytes / (ms * 1e-3) / 1e9
            d.update({"algo_bytes": int(algo_bytes), "GB_s": round(gbs, 1),
                      "frac_hbm": round(gbs / pk["hbm_gbs"], 3)})
        if flops is not None:
            tf = flops / (ms * 1e-3) / 1e12
            d.update({"attended_tflop": round(flops / 1e12, 4), "TFLOP_s": round(tf, 1),
                      "frac_bf16_burst": round(tf / pk["bf16_tflops"], 3)})
            if e4m3:
                # 8-bit contraction: measured bf16 peak x the nominal e4m3 / bf16 ratio (2)
                d["frac_e4m3_peak"] = round(tf / (2 * pk["bf16_tflops"]), 3)
        if note:
            d["note"] = note
        print(json.dumps(d), flush=True)

    only = {int(c) for c in args.table_configs.split(",")} if args.table_configs else None
    for cid in sorted(CONFIGS):
        if only is not None and cid not in only:
            continue
        w = CONFIGS[cid]
        q, k, v = make_qkv(w, device="cuda")
        out = torch.empty_like(q)
        tok_bytes = w.B * w.N * w.Hh * w.D * 2
        scale = 1.0 / math.sqrt(w.D)
        if w.lvsa_C:
            blk = w.lvsa_block or 128
            att = LvsaAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, w.lvsa_C, w.lvsa_T_per, block=blk)
            ms = timed(lambda: att.mask(0))
            emit(cid, "lvsa_mask", ms, 4 * (att.col_idx.numel() + att.row_ptr.numel() +
                                            att.frame_sets.numel()),
                 note="launch-latency bound: output is a few MB")
            emit(cid, "reorder_fwd (frame layout, Q K V)", timed(lambda: att.gather(q, k, v)),
                 3 * 2 * tok_bytes)
            flops = attended_flops(w)
            emit(cid, f"attn_fwd (LVSA block list, {blk}-token blocks)",
                 timed(lambda: att.attend(per_head=False)), flops=flops)
            emit(cid, "reorder_inv (frame layout, O)", timed(lambda: att.scatter(out)),
                 2 * tok_bytes)
            fused = att if blk == 128 else LvsaAttention(w.B, w.Hh, w.D, w.T, w.H, w.W,
                                                         w.lvsa_C, w.lvsa_T_per, block=128)
            emit(cid, "lvsa_attn_fwd (fused, natural layout)",
                 timed(lambda: fused.fused(q, k, v, 0, out)), flops=flops)
            bsa.bsa_poll_status(att.plan)
            del att, fused
        if w.dense:
            plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_FRAME, block=w.dense_block)
            nb = plan.nblocks
            rp = torch.arange(0, nb + 1, dtype=torch.int32, device="cuda") * nb
            ci = torch.arange(nb, dtype=torch.int32, device="cuda").repeat(nb)
            shape = (w.B, w.Hh, plan.Npad, w.D)
            qs, ks, vs, os_ = (torch.empty(shape, dtype=torch.bfloat16, device="cuda")
                               for _ in range(4))
            bsa.bsa_reorder_fwd(plan, q, qs, k, ks, v, vs)
            emit(cid, "attn_fwd (dense block list)",
                 timed(lambda: bsa.bsa_attn_fwd(plan, qs, ks, vs, rp, ci, False, scale, os_, None)),
                 flops=4.0 * w.D * w.N * w.N * w.Hh * w.B)
            bsa.bsa_poll_status(plan)
            del qs, ks, vs, os_, plan
        if w.draft_ph:
            att = DraftAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, w.draft_ph, w.draft_pw,
                                 w.draft_sparsity)
            emit(cid, "reorder_fwd (tile layout, Q K V)", timed(lambda: att.gather(q, k, v)),
                 3 * 2 * tok_bytes)
            nb = att.plan.nblocks
            pooled = 2 * w.B * w.Hh * nb * w.D * 8      # fp64 draft logits (the default)
            pooled32 = pooled // 2
            emit(cid, "draft_mask (pool + score/top-k)", timed(att.mask),
                 2 * tok_bytes + 2 * pooled + 4 * att.col_idx.numel(),
                 note=f"k = {att.keep} of {nb} blocks per row")
            kv_host = att.col_idx.cpu().numpy()
            emit(cid, "attn_fwd (draft, per-head block lists)",
                 timed(lambda: att.attend(per_head=True)),
                 flops=draft_attended_flops(w, kv_host, att.keep))
            emit(cid, "reorder_inv (tile layout, O)", timed(lambda: att.scatter(out)),
                 2 * tok_bytes)
            if w.draft_ph * w.draft_pw == 128:
                # the same path with no reorder: pooling and attention on the natural layout
                emit(cid, "draft_mask_natural (pool in place + score/top-k)",
                     timed(lambda: bsa.bsa_draft_mask_natural(att.plan, q, k, att.sparsity,
                                                              att.row_ptr, att.col_idx, None,
                                                              att.workspace)),
                     2 * tok_bytes + 2 * pooled + 4 * att.col_idx.numel())
                emit(cid, "attn_fwd_natural (draft, 5-D tile loads, token-order stores)",
                     timed(lambda: bsa.bsa_attn_fwd_natural(att.plan, q, k, v, att.row_ptr,
                                                            att.col_idx, True, scale, out)),
                     flops=draft_attended_flops(w, kv_host, att.keep))
                emit(cid, "draft pipeline, reorder path (reorder, mask, attention, inverse)",
                     timed(lambda: att(q, k, v, out)),
                     flops=draft_attended_flops(w, kv_host, att.keep))
                emit(cid, "draft pipeline, natural layout (mask, attention)",
                     timed(lambda: att.fused(q, k, v, out)),
                     flops=draft_attended_flops(w, kv_host, att.keep))
                # the optional fp32 draft logits (their own lists)
                att32 = DraftAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, w.draft_ph, w.draft_pw,
                                       w.draft_sparsity, precision=bsa.DRAFT_FP32)
                emit(cid, "draft_mask_natural, fp32 logits",
                     timed(lambda: bsa.bsa_draft_mask_natural(att32.plan, q, k, att32.sparsity,
                                                              att32.row_ptr, att32.col_idx, None,
                                                              att32.workspace)),
                     2 * tok_bytes + 2 * pooled32 + 4 * att32.col_idx.numel())
                emit(cid, "draft pipeline, natural layout, fp32 logits (mask, attention)",
                     timed(lambda: att32.fused(q, k, v, out)),
                     flops=draft_attended_flops(w, att32.col_idx.cpu().numpy(), att32.keep))
                bsa.bsa_poll_status(att32.plan)
                del att32
                if w.D == 128:
                    # 8-bit attention: e4m3 Q, K, V (read twice, written at 1 byte)
                    emit(cid, "quantize_e4m3 (Q K V, per-head scales)",
                         timed(lambda: att.quantize(q, k, v)), 3 * tok_bytes + 3 * tok_bytes // 2)
                    emit(cid, "attn_fwd_natural_e4m3 (8-bit QK and PV)",
                         timed(lambda: bsa.bsa_attn_fwd_natural_e4m3(
                             att.plan, att.q8, att.k8, att.v8, att.fp8_scales, att.row_ptr,
                             att.col_idx, True, scale, out)),
                         flops=draft_attended_flops(w, kv_host, att.keep), e4m3=True)
                    emit(cid, "draft pipeline, 8-bit (mask, quantize, attention)",
                         timed(lambda: att.fused_e4m3(q, k, v, out)),
                         flops=draft_attended_flops(w, kv_host, att.keep))
            bsa.bsa_poll_status(att.plan)
            del att
        del q, k, v, out
        torch.cuda.empty_cache()


def draft_pipelines(heads: int):
    """Runs the draft pipelines (with reorders, on the natural layout, 8-bit,
    and on the natural layout with fp32 draft logits) twice each on `heads`
    heads of the 40-head draft workload: a fixed launch sequence for
    profilers.  Prints one line."""
    import block_sparse_attention_49_b200 as bsa
    from block_sparse_attention_49_b200.pipeline import DraftAttention
    from synth import small_workload

    w = small_workload(CONFIGS[5], Hh=heads)
    q, k, v = make_qkv(w, device="cuda")
    att = DraftAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, w.draft_ph, w.draft_pw, w.draft_sparsity)
    att32 = DraftAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, w.draft_ph, w.draft_pw,
                           w.draft_sparsity, precision=bsa.DRAFT_FP32)
    out = torch.empty_like(q)
    for _ in range(2):
        att(q, k, v, out)
        att.fused(q, k, v, out)
        att.fused_e4m3(q, k, v, out)
        att32.fused(q, k, v, out)
    torch.cuda.synchronize()
    bsa.bsa_poll_status(att.plan)
    bsa.bsa_poll_status(att32.plan)
    print(json.dumps({"draft_pipelines": w.name, "heads": heads}), flush=True)


def hbm_kernels(cid: int):
    """Runs every HBM-bound kernel twice on workload `cid`: the frame- and
    tile-layout reorders (forward and inverse), both draft masks (pooling and
    scoring) and the e4m3 quantization.  A fixed launch sequence for DRAM
    counter captures.  Prints one line with the algorithmic bytes per launch
    of each kernel."""
    import block_sparse_attention_49_b200 as bsa
    from block_sparse_attention_49_b200.pipeline import DraftAttention

    w = CONFIGS[cid]
    q, k, v = make_qkv(w, device="cuda")
    out = torch.empty_like(q)
    tok = w.B * w.N * w.Hh * w.D * 2
    fr = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_FRAME, block=128)
    shape = (w.B, w.Hh, fr.Npad, w.D)
    fq, fk, fv = (torch.empty(shape, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    att = DraftAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, w.draft_ph or 8, w.draft_pw or 16,
                         w.draft_sparsity or 90)
    nb = att.plan.nblocks
    pooled = 2 * w.B * w.Hh * nb * w.D * 8    # fp64 pooled Q and K
    norms = 2 * w.B * w.Hh * nb * 4
    for _ in range(2):
        bsa.bsa_reorder_fwd(fr, q, fq, k, fk, v, fv)
        bsa.bsa_reorder_inv(fr, fq, out)
        att.gather(q, k, v)
        bsa.bsa_reorder_inv(att.plan, att.q_s, out)
        att.mask()
        bsa.bsa_draft_mask_natural(att.plan, q, k, att.sparsity, att.row_ptr, att.col_idx,
                                   None, att.workspace)
        att.quantize(q, k, v)
    torch.cuda.synchronize()
    bsa.bsa_poll_status(fr)
    bsa.bsa_poll_status(att.plan)
    print(json.dumps({
        "hbm_kernels": w.name, "tokens": w.N, "heads": w.Hh, "head_dim": w.D,
        "algo_bytes_per_launch": {
            "reorder_fwd_kernel (Q K V, either layout)": 3 * 2 * tok,
            "reorder_inv_kernel (O, either layout)": 2 * tok,
            "draft_pool_kernel (tile-layout Q K slots read; fp64 values, fp32 copies, norms written)":
                2 * w.B * w.Hh * att.plan.Npad * w.D * 2 + pooled + pooled // 2 + norms,
            "draft_pool_kernel natural (natural Q K read; fp64 values, fp32 copies, norms written)":
                2 * tok + pooled + pooled // 2 + norms,
            "draft_score_reg_kernel (fp32 copies and norms read, lists written)":
                pooled // 2 + norms + 4 * att.col_idx.numel(),
            "e4m3_amax_kernel (Q K V read)": 3 * tok,
            "e4m3_convert_kernel (Q K V read, codes written)": 3 * tok + 3 * tok // 2},
        "slots": {"frame_Npad": fr.Npad, "tile_Npad": att.plan.Npad}}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=3)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    ap.add_argument("--ref-step-s", type=float, default=4.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--frames", type=int, default=0,
                    help="use only the first T frames (small profiling case of the same kernels)")
    ap.add_argument("--kernel-table", action="store_true",
                    help="time every kernel on every workload instead of the step")
    ap.add_argument("--table-reps", type=int, default=10)
    ap.add_argument("--table-configs", default="",
                    help="comma-separated workloads for --kernel-table (default: all)")
    ap.add_argument("--draft-pipelines", type=int, default=0, metavar="HEADS",
                    help="run the three draft pipelines on HEADS heads (profiling)")
    ap.add_argument("--hbm-kernels", type=int, default=0, metavar="CONFIG",
                    help="run every HBM-bound kernel twice on workload CONFIG (profiling)")
    args = ap.parse_args()
    if args.hbm_kernels:
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        hbm_kernels(args.hbm_kernels)
        return
    if args.draft_pipelines:
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        draft_pipelines(args.draft_pipelines)
        return
    if args.kernel_table:
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        kernel_table(args)
        return

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.warmup < 3:
        raise SystemExit("at least 3 warm-up steps")

    import block_sparse_attention_49_b200 as bsa
    bsa.load()  # fails loudly when the library is missing

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    w = CONFIGS[args.config]
    if args.frames:
        from synth import small_workload
        Tc, Hc, Wc = w.field_grid
        w = small_workload(w, T=args.frames, field_grid=(args.frames, Hc, Wc),
                           name=f"{w.name} (first {args.frames} frames)")
    q, k, v = make_qkv(w, device="cuda")
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)
    if w.lvsa_C:
        step_setup = lvsa_step_setup(w, q, k, v, out)
    else:
        step_setup = draft_step_setup(w, q, k, v, out)
    step, flops_step, dominant, extra = step_setup

    # warm-up, then exactly `steps` timed steps between barriers
    for i in range(args.warmup):
        step(i, None)
    extra["poll"]()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = ClockSampler(local)
    clocks.start()
    marks = [ev() for _ in range(args.steps + 1)]
    dom = [(ev(), ev()) for _ in range(args.steps)]
    torch.cuda.synchronize()
    marks[0].record(stream)
    for i in range(args.steps):
        step(args.warmup + i, dom[i])
        marks[i + 1].record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    extra["poll"]()
    ms = marks[0].elapsed_time(marks[-1]) / args.steps
    dom_ms = statistics.mean(a.elapsed_time(b) for a, b in dom)
    ms, dom_ms = max_over_ranks([ms, dom_ms], dist, "cuda")

    # the same path as separate kernels (secondary numbers)
    names, calls_of = extra["breakdown"]
    per = {n: [] for n in names}
    n_sep = max(3, min(args.steps, 10))
    for i in range(args.warmup + n_sep):
        calls = calls_of(i)
        m = [ev() for _ in range(len(calls) + 1)]
        m[0].record(stream)
        for j, c in enumerate(calls):
            c()
            m[j + 1].record(stream)
        if i >= args.warmup:
            torch.cuda.synchronize()
            for j, n in enumerate(names):
                per[n].append(m[j].elapsed_time(m[j + 1]))
    torch.cuda.synchronize()
    extra["poll"]()
    sep_ms = max_over_ranks([statistics.mean(per[n]) for n in names], dist, "cuda")

    # end to end through the public API with host buffers: every step copies
    # its Q, K, V in from pinned host memory and its O back out; the copies
    # of neighbouring steps overlap this step's compute (StreamedSteps)
    from block_sparse_attention_49_b200.pipeline import StreamedSteps
    hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    ho = torch.empty_like(hq).pin_memory()
    streamed = StreamedSteps(q.shape, q.dtype)
    step_fn = extra["host_step"]
    streamed.run(step_fn, (hq, hk, hv), ho, 2)       # warm-up
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = streamed.run(step_fn, (hq, hk, hv), ho, args.e2e_steps)
    torch.cuda.synchronize()
    (e2e_ms,) = max_over_ranks([e0.elapsed_time(e1) / args.e2e_steps], dist, "cuda")
    extra["poll"]()
    del streamed

    pk, pk_kind = peaks()
    burst = pk["bf16_tflops"]
    sustained = pk.get("bf16_tflops_sustained")
    dom_tflops = flops_step / (dom_ms * 1e-3) / 1e12
    tok_bytes = w.B * w.N * w.Hh * w.D * 2
    sep = {}
    for n, t in zip(names, sep_ms):
        d = {"ms": t}
        ab = extra["algo_bytes"].get(n)
        if ab is not None:
            gbs = ab / (t * 1e-3) / 1e9
            d.update({"algo_bytes": ab, "GB_s": gbs, "frac_hbm": gbs / pk["hbm_gbs"]})
        else:
            d["attended_tflops"] = flops_step / (t * 1e-3) / 1e12
        sep[n] = d
    roof = {"bound": "tensor", "achieved": dom_tflops, "peak": burst, "unit": "TFLOP/s",
            "frac": dom_tflops / burst, "traffic": extra["traffic"],
            "peak_kind": f"{pk_kind} bf16 burst (the kernel timed on its own)",
            "kernel": dominant}
    if extra.get("traffic_source"):
        roof["traffic_source"] = extra["traffic_source"]
    # against NVIDIA's nominal dense bf16 figure for B200 (2.25 PFLOP/s), for context
    roof["frac_of_nominal_dense_bf16"] = dom_tflops / NOMINAL_BF16_TFLOPS
    if sustained:
        roof["frac_of_sustained"] = dom_tflops / sustained
        peak_mhz = _peak_sm_mhz(pk)
        if peak_mhz and clk and clk.get("sm_mhz"):
            # the same ratio per clock: sustained peak and kernel each divided
            # by the median SM clock seen while they ran
            roof["frac_of_sustained_per_clock"] = (dom_tflops / clk["sm_mhz"]) / (sustained / peak_mhz)
    line = {
        "metric": extra["metric"],
        "value": weak_scaling_value(flops_step, world, ms),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": dict(extra["config"], workload=w.name, global_batch=w.B * world, seq_len=w.N,
                       heads=w.Hh, head_dim=w.D, parallelism=f"dp{world}",
                       l2=f"inputs ({3 * tok_bytes / 1e9:.2f} GB) "
                          + ("larger than L2; no flush" if 3 * tok_bytes > 126e6
                             else "smaller than L2 (tiny case)")),
        "bsattn_ms_per_call": dom_ms,
        "bsattn_attended_tflops": dom_tflops,
        "bsattn_pct_bf16_peak": 100.0 * dom_tflops / burst,
        "attended_tflop_per_call": flops_step / 1e12,
        "roofline": roof,
        extra["breakdown_key"]: {"ms_per_step": sum(sep_ms), "kernels": sep},
        "gpu_launches": args.steps * extra["launches_per_step"],
        "clocks": clk,
        "e2e": {"value": weak_scaling_value(flops_step, world, e2e_ms), "unit": "TFLOP/s",
                "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": 3 * q.numel() * q.element_size(),
                "d2h_bytes_per_step": out.numel() * out.element_size()},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        q_h, k_h, v_h = (x[:, :, :1].float().cpu().numpy().astype(np.float64) for x in (q, k, v))
        val, thr, desc, _ = extra["cpu_baseline"](w, q_h, k_h, v_h, args.cpu_budget_s)
        line["cpu_baseline"] = {"value": val, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                                "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def _peak_sm_mhz(pk):
    """Median SM clock of the sustained peak measurement, if the peaks file
    records one."""
    for key in ("clocks_under_load", "clocks", "sustained_clocks"):
        c = pk.get(key)
        if isinstance(c, dict):
            for name, val in c.items():
                if "sm" in name and isinstance(val, (int, float)) and val > 100:
                    return float(val)
        elif isinstance(c, (int, float)) and c > 100:
            return float(c)
    return None


def lvsa_step_setup(w, q, k, v, out):
    """The LVSA step: bsa_lvsa_attn_fwd (one kernel, natural layout) with
    s = step mod T_per.  Returns (step, attended flops, kernel name, extras)."""
    import block_sparse_attention_49_b200 as bsa
    from block_sparse_attention_49_b200.pipeline import LvsaAttention
    att = LvsaAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, w.lvsa_C, w.lvsa_T_per, block=128)
    stream = torch.cuda.current_stream()

    def step(i, evs):
        if evs:
            evs[0].record(stream)
        att.fused(q, k, v, i % w.lvsa_T_per, out)
        if evs:
            evs[1].record(stream)

    def calls_of(i):
        s_i = i % w.lvsa_T_per
        return (lambda: att.mask(s_i), lambda: att.gather(q, k, v),
                lambda: att.attend(per_head=False), lambda: att.scatter(out))

    tok_bytes = w.B * w.N * w.Hh * w.D * 2
    scaled = STEP_KERNEL_DRAM_BYTES is not None and w.name == CONFIGS[3].name
    extra = {
        "metric": METRIC,
        "poll": lambda: bsa.bsa_poll_status(att.plan),
        "breakdown": (("lvsa_mask", "reorder_fwd", "attn_fwd_blocklist", "reorder_inv"), calls_of),
        "breakdown_key": "four_kernel_path",
        "algo_bytes": {"lvsa_mask": 4 * (att.col_idx.numel() + att.row_ptr.numel() +
                                         att.frame_sets.numel()),
                       "reorder_fwd": 3 * 2 * tok_bytes, "reorder_inv": 2 * tok_bytes},
        "host_step": lambda dq, dk, dv, dout, i: att.fused(dq, dk, dv, i % w.lvsa_T_per, dout),
        "launches_per_step": 1,
        "traffic": STEP_KERNEL_DRAM_BYTES if scaled else None,
        "traffic_source": STEP_KERNEL_TRAFFIC_SOURCE if scaled else None,
        "config": {"lvsa_C": w.lvsa_C, "lvsa_T_per": w.lvsa_T_per,
                   "steps_s": "s = step mod T_per",
                   "path": "bsa_lvsa_attn_fwd (one kernel, natural layout)",
                   "window_growth": "alternating right/left pointers (plan default)",
                   "lse": "not written (lse = NULL)"},
        "cpu_baseline": lambda w_, qh, kh, vh, budget: cpu_baseline(w_, qh, kh, vh, budget_s=budget),
    }
    return step, attended_flops(w), "lvsa_attn_kernel", extra


def draft_step_setup(w, q, k, v, out):
    """The draft step: bsa_draft_mask_natural (pooling in place, scoring,
    top-k) then bsa_attn_fwd_natural on the natural layout."""
    import block_sparse_attention_49_b200 as bsa
    from block_sparse_attention_49_b200.pipeline import DraftAttention
    att = DraftAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, w.draft_ph, w.draft_pw, w.draft_sparsity)
    if w.draft_ph * w.draft_pw != 128:
        raise SystemExit("the draft step on the natural layout needs pool_h * pool_w = 128")
    stream = torch.cuda.current_stream()
    scale = 1.0 / math.sqrt(w.D)

    def mask():
        bsa.bsa_draft_mask_natural(att.plan, q, k, att.sparsity, att.row_ptr, att.col_idx, None,
                                   att.workspace)

    def attend():
        bsa.bsa_attn_fwd_natural(att.plan, q, k, v, att.row_ptr, att.col_idx, True, scale, out)

    def step(i, evs):
        mask()
        if evs:
            evs[0].record(stream)
        attend()
        if evs:
            evs[1].record(stream)

    mask()
    torch.cuda.synchronize()
    flops = draft_attended_flops(w, att.col_idx.cpu().numpy(), att.keep)
    tok_bytes = w.B * w.N * w.Hh * w.D * 2
    pooled = 2 * w.B * w.Hh * att.plan.nblocks * w.D * 8
    extra = {
        "metric": f"bsattn ms/call + attended TFLOP/s (% BF16 peak), {w.name}, draft attention",
        "poll": lambda: bsa.bsa_poll_status(att.plan),
        "breakdown": (("reorder_fwd", "draft_mask", "attn_fwd_blocklist", "reorder_inv"),
                      lambda i: (lambda: att.gather(q, k, v), att.mask,
                                 lambda: att.attend(per_head=True), lambda: att.scatter(out))),
        "breakdown_key": "reorder_path",
        "algo_bytes": {"reorder_fwd": 3 * 2 * tok_bytes, "reorder_inv": 2 * tok_bytes,
                       "draft_mask": 2 * tok_bytes + 2 * pooled + 4 * att.col_idx.numel()},
        "host_step": lambda dq, dk, dv, dout, i: att.fused(dq, dk, dv, dout),
        "launches_per_step": 3,
        "traffic": None,
        "config": {"draft_pool": f"{w.draft_ph}x{w.draft_pw}", "sparsity_pct": w.draft_sparsity,
                   "keep_per_row": att.keep, "blocks_per_head": att.plan.nblocks,
                   "path": "bsa_draft_mask_natural + bsa_attn_fwd_natural (natural layout)",
                   "lse": "not written (lse = NULL)"},
        "cpu_baseline": cpu_baseline_draft,
    }
    return step, flops, "attn_fwd_kernel (natural layout, draft lists)", extra


def cpu_baseline_draft(w, q_h, k_h, v_h, budget_s: float, seed: int = 0):
    """The oracle on a bounded sample of the draft workload: head 0's draft
    blocks in full, then masked attention of sampled query blocks."""
    import oracle
    t0 = time.perf_counter()
    kv = oracle.draft_blocks(q_h, k_h, w.T, w.H, w.W, w.draft_ph, w.draft_pw, w.draft_sparsity)
    rp, ci = oracle.fixed_k_csr(kv)
    perm, Np = oracle.tile_layout_perm(w.T, w.H, w.W, w.draft_ph, w.draft_pw)
    valid = oracle.slot_valid(perm, Np)
    qs, ks, vs = (oracle.reorder_fwd(x, perm, Np) for x in (q_h, k_h, v_h))
    setup = time.perf_counter() - t0
    blk = w.draft_ph * w.draft_pw
    nb = Np // blk
    rng = np.random.default_rng(seed)
    done, flops, t_att = 0, 0.0, 0.0
    while t_att < budget_s and done < nb:
        qb = int(rng.integers(0, nb))
        t1 = time.perf_counter()
        oracle.masked_attention(qs, ks, vs, valid, blk, rp, ci, True, 1 / math.sqrt(w.D),
                                q_blocks=[qb], heads=[(0, 0)])
        t_att += time.perf_counter() - t1
        nq = int(valid[qb * blk:(qb + 1) * blk].sum())
        keys = sum(int(valid[c * blk:(c + 1) * blk].sum()) for c in ci[rp[qb]:rp[qb + 1]])
        flops += 4.0 * w.D * nq * keys
        done += 1
    threads = torch.get_num_threads()
    desc = (f"oracle masked attention on {done} random query blocks of head 0 (of {nb} x {w.Hh}), "
            f"draft lists of head 0; draft mask and layout set-up {setup:.1f}s excluded")
    return flops / t_att / 1e12, threads, desc, t_att

if __name__ == "__main__":
    main()
