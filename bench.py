#!/usr/bin/env python
"""Benchmark of the block-sparse attention path on B200.

One step = the whole path over one batch: sba_pool_select (pool, score, top-k),
sba_pair_query_blocks (which two query blocks share an attention tile) and
sba_attention_paired over the kept blocks.  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]
                  [--router mean|lse] [--budget B] [--producer] [--compensate first|mean]

The default workload is long_clip (B 2, H 32, D 128, a 31x34x60 latent grid with 15% of
the tokens pruned per sample, ragged lengths, sparsity 0.75): the largest of the five
configurations, the metric being quoted on none of them.

`--router lse` routes with the sub-block log-sum-exp score (sba_pool_select_lse,
16-token sub-blocks) and `--budget` rounds its kept count up to a multiple of B
blocks; the default is the block-mean router with no rounding.  `--producer` treats
the workload's Q and K as the pre-norm projections: each step first applies QK
RMSNorm + 3D RoPE with the block pooling fused (sba_qk_norm_rope_pool), then routes
from those means (sba_pool_select_means) and attends over the normalised Q and K.
`--compensate first` attends with the first-order compensation of the dropped blocks
(sba_attention_compensated, which walks every block), `--compensate mean` with the
mean-key form (sba_attention_mean_compensated); the metric still counts kept-block
FLOPs only.

The line carries a `parity` object: for two heads of the timed workload, the GPU's
routing against the oracle's (rows checked, rows that differ, rows excused as score
ties within 1e-6 relative) and the GPU's output of sampled query blocks against the
oracle fed the GPU's routing (max-abs, mean-abs).

Metric: effective TFLOP/s on the kept blocks, counted as
4 * D * sum_{b,h,I} c_I * sum_{J kept} c_J (c = valid tokens of a block), divided by
the step time.  N > 1 runs one replica per GPU (every (b, h) is independent; there is
no exchange inside the path), so scaling is weak and `value` sums all replicas.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "block-sparse attn effective TFLOP/s (kept blocks) and % of B200 bf16 peak"
SPEC_BF16_TFLOPS = 2250.0
# bytes written between the L2-flushed rounds: four times the 126 MB L2
FLUSH_BYTES = 512 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="long_clip")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-parity", action="store_true")
    ap.add_argument("--router", default="mean", choices=["mean", "lse"])
    ap.add_argument("--budget", type=int, default=1)
    ap.add_argument("--producer", action="store_true")
    ap.add_argument("--compensate", default=None, choices=["first", "mean"])
    ap.add_argument("--prune", type=float, default=None, metavar="RATIO",
                    help="prune each sample to RATIO of its tokens by feature-norm saliency at the start of "
                         "every step (token features of width H*D), then gather Q, K, V")
    ap.add_argument("--attn-kernel", default="auto", choices=["auto", "query_pairs", "cta_pair"],
                    help="D = 128 attention kernel: the default query pairs, or the opt-in CTA pair")
    return ap.parse_args()


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one attention launch,
# from the ncu captures summarised in profiles/attn_kernel_*.md, and the hash
# of the kernel sources it was taken with.  Reported only while the sources match.
ATTN_TRAFFIC = {"480p_dense": (631931392 + 190078976, "46d3116201e64454"),
                "720p": (2971918336 + 803863552, "46d3116201e64454"),
                "long_clip": (2696856064 + 909912576, "46d3116201e64454")}
KERNEL_SOURCES = ("video_dit_block_b200/csrc/attention.cuh", "video_dit_block_b200/csrc/ptx.cuh",
                  "video_dit_block_b200/csrc/common.cuh")


def kernel_source_hash():
    import hashlib
    data = b"".join(open(os.path.join(ROOT, f), "rb").read() for f in KERNEL_SOURCES)
    return hashlib.sha256(data).hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kept_flops(kv_idx, kv_cnt, valid_len, D, block=64):
    """4*D*sum_{b,h,I} c_I * sum_{J in kept(b,h,I)} c_J, exact for partial blocks."""
    B, H, nQ, kmax = kv_idx.shape
    total = 0
    for b in range(B):
        L = int(valid_len[b])
        cI = np.clip(L - block * np.arange(nQ), 0, block).astype(np.int64)          # [nQ]
        idx = kv_idx[b].astype(np.int64)                                               # [H,nQ,kmax]
        live = np.arange(kmax)[None, None, :] < kv_cnt[b][:, :, None]
        cJ = np.where(live, np.clip(L - block * idx, 0, block), 0)
        total += int((cJ.sum(axis=2) * cI[None, :]).sum())
    return 4 * D * total


class ClockSampler:
    """nvidia-smi every 100 ms, started before the warm-up so that it is sampling when
    the timed region begins; each line is stamped on arrival, and only the samples
    that arrive within the timed window (widened by one interval) are summarised."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    INTERVAL_MS = 100

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.window = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.INTERVAL_MS)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def mark(self, t0, t1):
        """The timed region, in time.monotonic() seconds."""
        self.window = (t0, t1)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        pad = self.INTERVAL_MS * 1e-3
        lines = [ln for (t, ln) in self.lines
                 if self.window is None or self.window[0] - pad <= t <= self.window[1] + pad]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(values, dist=None, device=None):
    """Element-wise maximum of a list of floats over all ranks (identity without a
    process group).  Every rank calls it at the same point."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def whole_job_value(kept_flops_per_rank, ms_per_step, world):
    """Whole-job TFLOP/s: every rank runs one replica of the workload."""
    return world * kept_flops_per_rank / (ms_per_step * 1e-3) / 1e12


def oracle_sample(w, target_s=10.0, seed=0, router="mean", budget=1, producer=False, compensate=None):
    """Time the fp64 oracle, as it stands, on a bounded sample of the workload: the
    full routing of head (b=0, h=0) and the attention of a seeded subset of that head's
    query blocks, sized to about `target_s` seconds.

    Throughput: routing one head costs t_sel and serves that head's kept FLOPs f_head;
    the sampled attention did f_sample kept FLOPs in t_attn.  So one kept FLOP costs
    t_sel / f_head + t_attn / f_sample seconds of the oracle."""
    import oracle
    q1, k1, v1 = (np.ascontiguousarray(x[:1, :1]) for x in (w.q, w.k, w.v))
    vl1 = np.ascontiguousarray(w.valid_len[:1])
    t0 = time.perf_counter()
    if producer:
        from workloads import make_norm_weights
        wq, wk = make_norm_weights(w.q.shape[3])
        pos1 = np.ascontiguousarray(w.positions[:1])
        rd = 3 * w.q.shape[3] // 4  # 96 for D = 128 (the page's setting), 48 for D = 64
        q1 = oracle.qk_norm_rope(q1, wq, pos1, rope_dim=rd)
        k1 = oracle.qk_norm_rope(k1, wk, pos1, rope_dim=rd)
    if router == "lse":
        idx, cnt = oracle.select_lse(q1, k1, vl1, w.sparsity, budget=budget)
    else:
        idx, cnt = oracle.select(q1, k1, vl1, w.sparsity)
    t_sel = time.perf_counter() - t0
    f_head = kept_flops(idx, cnt, vl1, w.D)
    L = int(vl1[0])
    nB0 = (L + 63) // 64
    order = np.random.default_rng(seed).permutation(nB0).astype(np.int32)
    # grow the sample (doubling) until one run takes about target_s / 2 or covers the head
    n, t_attn = 1, 0.0
    while True:
        t0 = time.perf_counter()
        if compensate:
            oracle.attention_compensated(q1, k1, v1, idx, cnt, vl1, qblocks=order[:n],
                                         order=1 if compensate == "first" else 0)
        else:
            oracle.attention(q1, k1, v1, idx, cnt, vl1, qblocks=order[:n])
        t_attn = time.perf_counter() - t0
        if t_attn >= target_s / 2 or n >= nB0:
            break
        n = min(nB0, max(2 * n, int(n * target_s / 2 / max(t_attn, 1e-3))))
    sel = order[:n]
    sub_cnt = np.zeros_like(cnt)
    sub_cnt[:, :, sel] = cnt[:, :, sel]
    f_sample = kept_flops(idx, sub_cnt, vl1, w.D) if n < nB0 else f_head
    sec_per_flop = t_sel / f_head + t_attn / f_sample
    return {"t_sel": t_sel, "t_attn": t_attn, "f_head": f_head, "f_sample": f_sample,
            "n_qblocks": n, "value": 1.0 / sec_per_flop / 1e12}


def token_features(w, make_hidden):
    """Token features of width H*D for the workload's tokens, in their order: the
    smooth-field features of the whole latent grid (make_hidden), picked at each token's
    (t, y, x) position; zero rows past each sample's length."""
    B, H, Npad, D = w.q.shape
    T, Hg, Wg = w.grid
    hid = make_hidden(B, w.grid, H * D)
    out = np.zeros((B, Npad, H * D), dtype=np.uint16)
    for b in range(B):
        L = int(w.valid_len[b])
        p = w.positions[b, :L].astype(np.int64)
        out[b, :L] = hid[b, (p[:, 0] * Hg + p[:, 1]) * Wg + p[:, 2]]
    return out


def pruned_workload(w, idx, valid_out, npad_out):
    """The workload's Q, K, V compacted to the kept tokens (idx, as the oracle lists them)."""
    import copy
    B, H, _, D = w.q.shape
    pw = copy.copy(w)
    pw.q, pw.k, pw.v = (np.zeros((B, H, npad_out, D), dtype=np.uint16) for _ in range(3))
    pw.positions = np.zeros((B, npad_out, 3), dtype=np.int32)
    for b in range(B):
        kb = int(valid_out[b])
        for dst, src in ((pw.q, w.q), (pw.k, w.k), (pw.v, w.v)):
            dst[b, :, :kb] = src[b][:, idx[b, :kb]]
        pw.positions[b, :kb] = w.positions[b, idx[b, :kb]]
    pw.valid_len = np.ascontiguousarray(valid_out, dtype=np.int32)
    return pw


TIE_REL = 1e-6   # score gap below which a routing difference is a tie (relative)


def parity_check(args, w, heads, o_h, lse_h, idx_h, cnt_h, n_qblocks=6, seed=0):
    """The GPU's results on `heads` of the timed workload against the fp64 oracle.

    Routing: every query-block row of each head, the oracle's kept set against the
    GPU's; a differing row is excused when every block in which they differ has an
    oracle score within TIE_REL of the oracle's k-th score.  Output: a seeded sample of
    query blocks per head (and the sample's last block), the GPU's bf16 output against
    the oracle fed the GPU's routing, over valid rows.  o_h, lse_h, idx_h, cnt_h: host
    arrays of the GPU results, one entry per head."""
    import oracle
    rows = mism = excused = 0
    err_max = err_sum = lse_max = 0.0
    n_out = 0
    for (b, h), og, lg, ig, cg in zip(heads, o_h, lse_h, idx_h, cnt_h):
        sl = lambda x: np.ascontiguousarray(x[b:b + 1, h:h + 1])
        q1, k1, v1 = sl(w.q), sl(w.k), sl(w.v)
        vl1 = np.ascontiguousarray(w.valid_len[b:b + 1])
        if args.producer:
            from workloads import make_norm_weights
            wq, wk = make_norm_weights(w.D)
            pos1 = np.ascontiguousarray(w.positions[b:b + 1])
            q1 = oracle.qk_norm_rope(q1, wq, pos1, rope_dim=3 * w.D // 4)
            k1 = oracle.qk_norm_rope(k1, wk, pos1, rope_dim=3 * w.D // 4)
        kmax = ig.shape[-1]
        if args.router == "lse":
            io, co, S = oracle.select_lse(q1, k1, vl1, w.sparsity, budget=args.budget, kmax=kmax, return_scores=True)
        else:
            io, co, _, _, S = oracle.select(q1, k1, vl1, w.sparsity, kmax=kmax, return_intermediates=True)
        L = int(vl1[0])
        nB = (L + 63) // 64
        for I in range(nB):
            rows += 1
            c = int(co[0, 0, I])
            a = set(io[0, 0, I, :c].tolist())
            g = set(ig[I, :int(cg[I])].tolist())
            if int(cg[I]) == c and a == g:
                continue
            row = S[0, 0, I, :nB]
            tau = np.sort(row)[::-1][c - 1]
            diff = (a - g) | (g - a)
            if int(cg[I]) == c and all(abs(row[j] - tau) <= TIE_REL * max(abs(row[j]), abs(tau)) for j in diff):
                excused += 1
            else:
                mism += 1
        rng = np.random.default_rng(seed + 7919 * b + h)
        qb = np.unique(np.concatenate([rng.choice(nB, min(n_qblocks, nB), replace=False), [nB - 1]])).astype(np.int32)
        ig4, cg4 = ig[None, None], cg[None, None]
        if args.compensate:
            o_ref, lse_ref = oracle.attention_compensated(q1, k1, v1, ig4, cg4, vl1, qblocks=qb,
                                                          order=1 if args.compensate == "first" else 0)
        else:
            o_ref, lse_ref = oracle.attention(q1, k1, v1, ig4, cg4, vl1, qblocks=qb)
        valid = np.isfinite(lse_ref[0, 0])
        e = np.abs(og[valid].astype(np.float64) - o_ref[0, 0][valid])
        err_max = max(err_max, float(e.max()))
        err_sum += float(e.sum())
        n_out += e.size
        lse_max = max(lse_max, float(np.abs(lg[valid] - lse_ref[0, 0][valid]).max()))
    return {"heads": [list(x) for x in heads], "mask_rows": rows, "mask_mismatch": mism, "mask_excused_ties": excused,
            "tie_rel": TIE_REL, "out_rows": int(n_out // w.D), "max_abs": err_max,
            "mean_abs": err_sum / max(n_out, 1), "lse_max_abs": lse_max,
            "tolerance": {"max_abs": 2e-2, "mean_abs": 2e-3},
            "ok": mism == 0 and err_max <= 2e-2 and err_sum / max(n_out, 1) <= 2e-3}


def cpu_baseline_from(sample, kind="oracle"):
    return {"value": sample["value"], "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": kind,
            "sample": (f"fp64 oracle on all host cores: routing of head (0,0) ({sample['t_sel']:.2f} s) "
                       f"+ attention of {sample['n_qblocks']} seeded query blocks of that head "
                       f"({sample['t_attn']:.2f} s); TFLOP/s = 1 / (t_route/F_head + t_attn/F_sample)")}


def workload_config(w, extra=None):
    c = {"workload": w.name, "B": w.B, "H": w.H, "D": w.D, "N": int(np.prod(w.grid)),
         "Npad": w.Npad, "valid_len": [int(x) for x in w.valid_len], "block": 64,
         "sparsity": w.sparsity, "grid_thw": list(w.grid), "parallelism": "replicas"}
    c.update(extra or {})
    return c


def router_config(args):
    c = {"router": "block mean"} if args.router == "mean" else {
        "router": "sub-block log-sum-exp (4 x 16 tokens)", "budget": args.budget}
    if args.producer:
        c["producer"] = "QK RMSNorm + 3D RoPE (rope_dim 3D/4, base 1e4, eps 1e-6) with fused block pooling"
    if args.compensate == "first":
        c["compensation"] = "dropped blocks by the first-order expansion of their exponentials about the mean key"
    elif args.compensate == "mean":
        c["compensation"] = "dropped blocks by their bf16 mean key and value, weighted by token count"
    return c


def run_reference(args):
    """The oracle as the reference arm, rank 0 only: every step is a bounded sample."""
    from workloads import CONFIGS, make_workload
    if int(os.environ.get("RANK", "0")) != 0:
        return
    w = make_workload(args.config, heads=1)
    per = []
    target = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for i in range(args.warmup + args.steps):
        s = oracle_sample(w, target_s=target, seed=i, router=args.router, budget=args.budget,
                          producer=args.producer, compensate=args.compensate)
        if i >= args.warmup:
            per.append(s)
    value = statistics.mean(s["value"] for s in per)
    t_step = statistics.mean(s["t_sel"] + s["t_attn"] for s in per)
    cb = cpu_baseline_from(per[-1])
    cb["value"] = value
    cfg = workload_config(w, {"H": CONFIGS[args.config]["H"], **router_config(args),
                              "sample": "each step: oracle routing of head (0,0) + attention of a "
                                        "seeded subset of its query blocks"})
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded smooth field + noise)",
            "config": cfg, "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args):
    import torch

    import video_dit_block_b200 as sba
    from workloads import make_workload

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    sba.set_attention_kernel(args.attn_kernel)
    w = make_workload(args.config)
    pair_kernel = args.attn_kernel == "cta_pair" and w.D == 128 and not args.compensate
    t = lambda x: torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    q, k, v = t(w.q), t(w.k), t(w.v)
    vl = torch.from_numpy(w.valid_len).to(dev)
    B, H, Npad, D = q.shape
    stream = torch.cuda.current_stream(dev)
    Npad_in = Npad
    if args.prune is not None:
        # token features of the workload's tokens (in their order), width H*D
        from workloads import make_hidden
        xf_host = token_features(w, make_hidden)
        x = t(xf_host)
        Npad = 64 * -(-sba.keep_token_count(Npad_in, args.prune) // 64)   # the pruned sequences' padded length
        pr_idx = torch.empty((B, Npad), dtype=torch.int32, device=dev)
        pr_vl = torch.empty((B,), dtype=torch.int32, device=dev)
        pr_ws = torch.empty(int(sba.lib().sba_token_prune_workspace_size(B, Npad_in)), dtype=torch.uint8, device=dev)
        qp, kp, vp = (torch.empty((B, H, Npad, D), dtype=torch.bfloat16, device=dev) for _ in range(3))
    lse_router = args.router == "lse"
    kmax = sba.keep_count_budget(Npad // 64, w.sparsity, args.budget) if lse_router else sba.kmax_for(Npad, w.sparsity)
    kv_idx = torch.empty((B, H, Npad // 64, kmax), dtype=torch.int32, device=dev)
    kv_cnt = torch.empty((B, H, Npad // 64), dtype=torch.int32, device=dev)
    wsz = sba.lse_workspace_size(B, H, Npad, D) if lse_router else sba.workspace_size(B, H, Npad, D)
    ws = torch.empty(wsz, dtype=torch.uint8, device=dev)
    o = torch.empty((B, H, Npad, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, Npad), dtype=torch.float32, device=dev)
    nQ = Npad // 64
    pair_order = torch.empty((B, H, 2 * ((nQ + 1) // 2)), dtype=torch.int32, device=dev)
    pws = torch.empty(int(sba.lib().sba_pair_workspace_size(B, H, Npad, 64)), dtype=torch.uint8, device=dev)

    def prep(qq=q, kk=k, vv=v, vll=vl, xx=None):
        """With --prune: saliency pruning of the step's tokens, then the compacted Q, K, V
        and valid lengths; otherwise the inputs as they are."""
        if args.prune is None:
            return qq, kk, vv, vll
        sba.token_prune(x if xx is None else xx, vll, args.prune, npad_out=Npad, idx=pr_idx, valid_out=pr_vl,
                        workspace=pr_ws, stream=stream)
        for src, dst in ((qq, qp), (kk, kp), (vv, vp)):
            sba.gather_tokens(src, pr_idx, pr_vl, out=dst, stream=stream)
        if args.producer:
            sba.gather_tokens(pos_src, pr_idx, pr_vl, out=pos, stream=stream)
        return qp, kp, vp, pr_vl

    if args.producer:
        if lse_router:
            raise SystemExit("--producer routes from block means: use the block-mean router")
        from workloads import make_norm_weights
        wq, wk = (t(x) for x in make_norm_weights(D))
        pos_src = torch.from_numpy(w.positions).to(dev)
        # with --prune, the pruned tokens' positions, gathered by each step's pruning
        pos = pos_src if args.prune is None else torch.empty((B, Npad, 3), dtype=torch.int32, device=dev)
        q_n, k_n = (torch.empty((B, H, Npad, D), dtype=torch.bfloat16, device=dev) for _ in range(2))
        q_m = torch.empty((B, H, Npad // 64, D), dtype=torch.float64, device=dev)
        k_m = torch.empty_like(q_m)

    def route(qq=q, kk=k, vll=vl, mid=None):
        """Routing (and, with --producer, the norm + RoPE before it); returns the Q, K
        the attention reads.  `mid`, an event, is recorded between the routing call
        and the query-block pairing."""
        if args.producer:
            sba.qk_norm_rope_pool(qq, wq, pos, vll, rope_dim=3 * D // 4, out=q_n, means=q_m, stream=stream)
            sba.qk_norm_rope_pool(kk, wk, pos, vll, rope_dim=3 * D // 4, out=k_n, means=k_m, stream=stream)
            sba.pool_select_means(q_m, k_m, vll, w.sparsity, kmax, kv_idx=kv_idx, kv_cnt=kv_cnt, workspace=ws,
                                  stream=stream)
            qq, kk = q_n, k_n
        elif lse_router:
            sba.pool_select_lse(qq, kk, vll, w.sparsity, budget=args.budget, kmax=kmax, kv_idx=kv_idx,
                                kv_cnt=kv_cnt, workspace=ws, stream=stream)
        else:
            sba.pool_select(qq, kk, vll, w.sparsity, kmax, kv_idx=kv_idx, kv_cnt=kv_cnt, workspace=ws,
                            stream=stream)
        if mid is not None:
            mid.record(stream)
        if not pair_kernel:  # the CTA-pair kernel tiles four adjacent query blocks itself
            sba.pair_query_blocks(kv_idx, kv_cnt, vll, pair_order=pair_order, workspace=pws, stream=stream)
        return qq, kk

    if args.compensate == "mean":
        cws = torch.empty(sba.mean_compensation_workspace_size(B, H, Npad, D), dtype=torch.uint8, device=dev)

    def attend(qq=q, kk=k, vv=v, vll=vl, out=o):
        if args.compensate == "first":
            sba.attention_compensated(qq, kk, vv, kv_idx, kv_cnt, vll, pair_order=pair_order, out=out, lse=lse,
                                      stream=stream)
        elif args.compensate == "mean":
            sba.attention_mean_compensated(qq, kk, vv, kv_idx, kv_cnt, vll, pair_order=pair_order, out=out,
                                           lse=lse, workspace=cws, stream=stream)
        else:
            sba.attention_paired(qq, kk, vv, kv_idx, kv_cnt, pair_order, vll, out=out, lse=lse, stream=stream)

    def step(qq=q, kk=k, vv=v, vll=vl, xx=None):
        qq, kk, vv, vll = prep(qq, kk, vv, vll, xx)
        qa, ka = route(qq, kk, vll)
        attend(qa, ka, vv, vll)

    def barrier():
        if dist is not None:
            dist.barrier()

    clocks = ClockSampler(local)
    clocks.start()  # sampling already when the timed region begins
    for _ in range(args.warmup):
        step()
    status = sba.device_status(stream)
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")
    vl_step = pr_vl.cpu().numpy() if args.prune is not None else w.valid_len
    f_step = kept_flops(kv_idx.cpu().numpy(), kv_cnt.cpu().numpy(), vl_step, D)

    # ---- timed region: K steps, events on the launching stream
    K = args.steps
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(5)) for _ in range(K)]
    barrier()
    torch.cuda.synchronize(dev)
    t_begin = time.monotonic()
    for i in range(K):
        ev[i][0].record(stream)
        qq, kk, vv, vll = prep()
        ev[i][3].record(stream)
        qa, ka = route(qq, kk, vll, mid=ev[i][4])
        ev[i][1].record(stream)
        attend(qa, ka, vv, vll)
        ev[i][2].record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark(t_begin, time.monotonic())
    clk = clocks.stop()
    barrier()
    total_ms = ev[0][0].elapsed_time(ev[-1][2])
    sel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    med_step = statistics.median(e[0].elapsed_time(e[2]) for e in ev)
    med_sel = statistics.median(e[0].elapsed_time(e[1]) for e in ev)
    med_attn = statistics.median(e[1].elapsed_time(e[2]) for e in ev)
    prune_ms = statistics.mean(e[0].elapsed_time(e[3]) for e in ev)
    med_call = statistics.median(e[3].elapsed_time(e[4]) for e in ev)  # the routing call alone
    med_pair = statistics.median(e[4].elapsed_time(e[1]) for e in ev)
    # the pages' micro-benchmark protocol: up to 10 rounds of consecutive steps, the
    # median of the rounds' mean step times
    n_rounds = min(10, K)
    per = K // n_rounds
    rounds = [ev[r * per:(r + 1) * per] for r in range(n_rounds)]
    rnd_step = statistics.median(statistics.mean(e[0].elapsed_time(e[2]) for e in rd) for rd in rounds)
    rnd_attn = statistics.median(statistics.mean(e[1].elapsed_time(e[2]) for e in rd) for rd in rounds)
    rnd_call = statistics.median(statistics.mean(e[3].elapsed_time(e[4]) for e in rd) for rd in rounds)
    if sba.device_status(stream) != 0:
        raise RuntimeError("device status error in the timed region")

    # ---- the same protocol with L2 flushed: before each round a buffer of 512 MB (four
    # times the L2) is written on the launching stream, then one step is timed; after
    # the warm region above and not part of `value`
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    fev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(5)) for _ in range(n_rounds)]
    barrier()
    torch.cuda.synchronize(dev)
    for r in range(n_rounds):
        flush.fill_(r + 1)  # torch's current stream is the launching stream
        fev[r][0].record(stream)
        qq, kk, vv, vll = prep()
        fev[r][3].record(stream)
        qa, ka = route(qq, kk, vll, mid=fev[r][4])
        fev[r][1].record(stream)
        attend(qa, ka, vv, vll)
        fev[r][2].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    del flush
    if sba.device_status(stream) != 0:
        raise RuntimeError("device status error in the L2-flushed rounds")
    fl_step = statistics.median(e[0].elapsed_time(e[2]) for e in fev)
    fl_attn = statistics.median(e[1].elapsed_time(e[2]) for e in fev)
    fl_call = statistics.median(e[3].elapsed_time(e[4]) for e in fev)

    (total_ms, attn_ms, sel_ms, med_step, med_sel, med_attn, prune_ms, med_call, med_pair, rnd_step, rnd_attn,
     rnd_call, fl_step, fl_attn, fl_call) = max_over_ranks(
        [total_ms, attn_ms, sel_ms, med_step, med_sel, med_attn, prune_ms, med_call, med_pair, rnd_step, rnd_attn,
         rnd_call, fl_step, fl_attn, fl_call], dist, dev)
    ms_step = total_ms / K
    value = whole_job_value(f_step, ms_step, world)

    # ---- the last timed step's results on two heads, for the parity check on rank 0
    par_heads = [(0, 0), (B - 1, H - 1)]
    par_data = None
    if rank == 0 and not args.no_parity:
        par_data = ([o[b, h].float().cpu().numpy() for b, h in par_heads],
                    [lse[b, h].cpu().numpy() for b, h in par_heads],
                    [kv_idx[b, h].cpu().numpy() for b, h in par_heads],
                    [kv_cnt[b, h].cpu().numpy() for b, h in par_heads])
        par_prune = (pr_idx.cpu().numpy(), pr_vl.cpu().numpy()) if args.prune is not None else None

    # ---- end to end through the public API with host buffers: every step uploads its
    # inputs from pinned host memory and downloads its output.  The steps are pipelined
    # the way a serving loop would run them: inputs and outputs are double-buffered on
    # the device, uploads run on one stream, compute on the launching stream and
    # downloads on a third, ordered by events, so step i+1's upload and step i-1's
    # download overlap step i's compute.  Timed from the first upload to the last
    # download.
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (z.cpu().pin_memory() for z in (q, k, v))
        vlh = vl.cpu().pin_memory()
        xh = x.cpu().pin_memory() if args.prune is not None else None
        oh = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        bufs = [(torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(vl),
                 torch.empty_like(x) if args.prune is not None else None) for _ in range(2)]
        outs = [o, torch.empty_like(o)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        in_done = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        out_done = [torch.cuda.Event() for _ in range(2)]
        Ke = max(4, K)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        e0.record(s_in)
        for i in range(Ke):
            bi_ = i % 2
            qd, kd, vd, vld, xd = bufs[bi_]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp_done[bi_])   # step i-2 has finished reading this buffer
                qd.copy_(qh, non_blocking=True)
                kd.copy_(kh, non_blocking=True)
                vd.copy_(vh, non_blocking=True)
                vld.copy_(vlh, non_blocking=True)
                if xd is not None:
                    xd.copy_(xh, non_blocking=True)
                in_done[bi_].record(s_in)
            stream.wait_event(in_done[bi_])
            if i >= 2:
                stream.wait_event(out_done[bi_])      # step i-2's output has been downloaded
            qq, kk, vv, vll = prep(qd, kd, vd, vld, xd)
            qa, ka = route(qq, kk, vll)
            attend(qa, ka, vv, vll, out=outs[bi_])
            comp_done[bi_].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[bi_])
                oh.copy_(outs[bi_], non_blocking=True)
                out_done[bi_].record(s_out)
        e1.record(s_out)
        torch.cuda.synchronize(dev)
        if sba.device_status(stream) != 0:
            raise RuntimeError("device status error in the end-to-end loop")
        e_ms = max_over_ranks([e0.elapsed_time(e1) / Ke], dist, dev)[0]
        bi = 3 * q.numel() * 2 + vl.numel() * 4 + (x.numel() * 2 if args.prune is not None else 0)
        e2e = {"value": whole_job_value(f_step, e_ms, world), "unit": "TFLOP/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": bi, "d2h_bytes_per_step": o.numel() * 2,
               "steps": Ke, "mode": "pipelined: double-buffered uploads, compute and downloads on three streams"}

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return
    peaks, src = load_peaks()
    tr = ATTN_TRAFFIC.get(w.name)
    traffic = (tr[0] if tr is not None and tr[1] == kernel_source_hash() and not args.compensate
               and not pair_kernel and args.prune is None else None)
    peak = float(peaks["bf16_tflops"])
    achieved = f_step / (attn_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded smooth field + noise, bf16; no weights involved)",
        "config": workload_config(w, {
            "l2": f"inputs {3 * q.numel() * 2 / 1e6:.0f} MB > 126 MB L2; no flush between steps "
                  "(median_ms.l2_flushed: a 512 MB write before each of its rounds)",
            "kmax": kmax, **router_config(args),
            **({"attention_kernel": "CTA pair (tcgen05 across two SMs)"} if pair_kernel else {})}),
        "pct_of_spec_bf16_peak": 100.0 * value / world / SPEC_BF16_TFLOPS,
        "attn_ms": attn_ms, "select_ms": sel_ms, "kept_tflop_per_step": f_step / 1e12,
        "median_ms": {"step": med_step, "select": med_sel, "attn": med_attn,
                      "step_tflops": f_step / (med_step * 1e-3) / 1e12 * world,
                      "rounds": {"n": n_rounds, "steps_each": per, "step": rnd_step, "attn": rnd_attn,
                                 "routing_call": rnd_call,
                                 "attn_tflops": f_step / (rnd_attn * 1e-3) / 1e12},
                      "l2_flushed": {"n": n_rounds, "flush_bytes": FLUSH_BYTES, "step": fl_step, "attn": fl_attn,
                                     "routing_call": fl_call,
                                     "step_tflops": f_step / (fl_step * 1e-3) / 1e12 * world,
                                     "attn_tflops": f_step / (fl_attn * 1e-3) / 1e12}},
        "roofline": {"bound": "tensor",
                     "kernel": "attn_pair_kernel<4>" if pair_kernel else
                     {"first": "attn_first_order_kernel", "mean": "attn_comp_kernel"}.get(args.compensate, "attn_kernel")
                     + ("<128,2>" if D == 128 else "<64,4>"),
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{src} bf16_tflops (burst): the timed region is K launches of "
                                    f"{attn_ms:.1f} ms, well short of the seconds-long loop of the sustained figure",
                     "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained", peak)),
                     "traffic": traffic},
        # per step: routing = pooling (Q and K in one launch) + key-norm maximum + fused
        # screen + finish + rest rows (the log-sum-exp router: the same pooling launch +
        # key-norm maximum + screen, only when blocks are dropped, + top-k); pairing =
        # bitmaps + proposals + the matching rounds and tile list in one launch (not with
        # the CTA-pair kernel); 1 attention
        # (--producer: 2 producer launches and 2 splits of the given means replace pooling)
        # (--compensate mean: 2 block-mean launches before the attention)
        # (--prune: norm + select + 3 gathers, and the positions' gather with --producer)
        "gpu_launches": ((3 + (1 if w.sparsity > 0 else 0) if lse_router else 5) + (3 if args.producer else 0)
                         + (0 if pair_kernel else 3) + 1 + (2 if args.compensate == "mean" else 0)
                         + (5 + (1 if args.producer else 0) if args.prune is not None else 0)) * K,
        "clocks": clk,
    }
    if not lse_router and not args.producer:
        # the routing call alone: it reads Q and K once (the block means it writes are
        # small beside them)
        qk_bytes = 2 * q.numel() * 2
        line["routing"] = {"pool_select_ms": med_call, "pair_ms": med_pair, "qk_bytes": qk_bytes,
                           "hbm_gbs": qk_bytes / (med_call * 1e-3) / 1e9,
                           "frac_of_hbm": qk_bytes / (med_call * 1e-3) / 1e9 / float(peaks["hbm_gbs"])}
    if e2e is not None:
        line["e2e"] = e2e
    if args.prune is not None:
        line["prune_ms"] = prune_ms
        line["config"]["pruning"] = {"ratio": args.prune, "features": f"bf16 [B, N, {x.shape[2]}] (H*D channels)",
                                     "valid_len_after": [int(z) for z in vl_step], "Npad_after": Npad}
        # the norm kernel reads the features once: its share of the pruning stage's time
        line["prune_feature_gbs"] = x.numel() * 2 / (prune_ms * 1e-3) / 1e9
    if par_data is not None:
        pw = w
        if args.prune is not None:
            import oracle
            io, vo, _ = oracle.token_prune(xf_host, w.valid_len, args.prune, npad_out=Npad)
            prune_exact = bool(np.array_equal(io, par_prune[0]) and np.array_equal(vo, par_prune[1]))
            pw = pruned_workload(w, io, vo, Npad)
        line["parity"] = parity_check(args, pw, par_heads, *par_data)
        if args.prune is not None:
            line["parity"]["prune_index_exact"] = prune_exact
            line["parity"]["ok"] = line["parity"]["ok"] and prune_exact
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_from(oracle_sample(w, target_s=15.0, router=args.router,
                                                               budget=args.budget, producer=args.producer,
                                                               compensate=args.compensate))
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def main():
    args = parse()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
