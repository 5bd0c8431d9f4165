#!/usr/bin/env python
"""Throughput of Thinformer Express prefill on B200 through the thin_attn C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl thin|reference] [--workload NAME]

One step = one thin_attn_forward of the whole path (batch thinning, HALVE
merges, attention) over the workload (default: express32k, B=1 H=32 T=32768
E=D=128 bf16, exact phase 1024, thin batch 1024, g=2) with q, k, v resident in
HBM.  Prints one JSON line on rank 0.  Multi-GPU (torchrun): the ranks hold
parts of one problem whose (b,h) slices are independent -- `--shard batch`
(default, weak scaling): rank r holds batch rows [rB, (r+1)B) of a problem with
N*B rows; `--shard heads` (strong scaling): rank r holds H/N heads of the
workload; `--shard seq` (strong scaling): rank r attends query rows
[r T/N, (r+1) T/N) (128-aligned) of every (b,h), each rank thinning all keys;
`--shard seqx`: the same ranges, each rank thinning only its own Express batches,
then one all-gather of the batch coresets (NCCL) before the merges and attention.
No collective on the data path; the random decisions are keyed on the whole
problem's (b,h); step time is the max over ranks of CUDA-event time.

--impl reference times the fp64 CPU oracle on the host cores (rank 0 only),
each step one head of the workload.
"""
import argparse
import datetime
import hashlib
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

import workloads as W  # noqa: E402

METRIC = "attention tokens/s (B·H·T) and ms/layer at S=32K causal; % of roofline"
UNIT = "tokens/s"


def args_():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="thin", choices=["thin", "reference"])
    p.add_argument("--workload", default="express32k", choices=sorted(W.WORKLOADS))
    p.add_argument("--shard", default="batch", choices=["batch", "heads", "seq", "seqx"],
                   help="N>1: batch rows of one larger problem per rank (weak) or the heads of one problem (strong)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-sdpa", action="store_true")
    p.add_argument("--no-per-workload", action="store_true",
                   help="N=1: skip the GPU-timed records of the other workloads")
    p.add_argument("--heads", type=int, default=0,
                   help="run the workload with this many heads instead of its own (small cases for profilers)")
    p.add_argument("--decode", action="store_true",
                   help="time token-by-token decoding of the workload through the Express decode cache "
                        "(causal workloads; prints its own JSON line)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "sm_max_mhz": d.get("sm_max_mhz", 1965.0), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def digitsum4(k):
    k = np.asarray(k, dtype=np.int64).copy()
    s = np.zeros_like(k)
    while np.any(k):
        s += k % 4
        k //= 4
    return s


def attention_work(w, plan, rows=None):
    """Algorithmic FLOPs and HBM bytes of one attention launch.

    FLOPs: 2 (E + D) per visible (query, key) pair.  Bytes: q read and out written
    once, plus every distinct key/value row read once (original tokens and coreset rows).
    ``rows=(q0, q1)``: a query-row shard's launch (its rows' pairs, q and out; the key/value rows
    are counted whole, an upper bound)."""
    BH = w.B * w.H
    es = 4 if w.dtype == "fp32" else 2
    if not w.causal:
        keys = plan["coreset_rows"] if plan["levels"] > 0 else w.S
        vis = np.full(w.T, keys, dtype=np.int64)
        kv_rows = keys
    elif w.cache == "A":
        # tokens [0, 4 n_out) exactly; batch (i, s): H_i and s - 1 thinned batches (n_out points each)
        # and its own tokens causally
        n_out = min(w.n_exact, w.T)
        ex = min(4 * n_out, w.T)
        parts = [np.arange(1, ex + 1, dtype=np.int64)]
        start, i = n_out * 4, 1
        while start < w.T:
            for s_ in range(1, 4):
                if start >= w.T:
                    break
                size = min(4 ** i * n_out, w.T - start)
                parts.append(s_ * n_out + np.arange(1, size + 1, dtype=np.int64))
                start += size
            i += 1
        vis = np.concatenate(parts)
        kv_rows = w.T + plan["n_nodes"] * plan["coreset_rows"]
    else:
        t = np.arange(w.T, dtype=np.int64)
        ne, b, c = min(w.n_exact, w.T), w.batch, plan["coreset_rows"]
        k = np.maximum(t - ne, 0) // b
        vis = np.where(t < ne, t + 1, ne + c * digitsum4(k) + (t - (ne + k * b) + 1))
        kv_rows = w.T + plan["n_nodes"] * c
    q0, q1 = rows if rows else (0, w.T)
    pairs = int(vis[q0:q1].sum())
    flops = 2.0 * (w.E + w.D) * pairs * BH
    bytes_ = es * BH * ((q1 - q0) * (w.E + w.D) + kv_rows * (w.E + w.D))
    return flops, bytes_, pairs


class Clocks:
    """SM clock and throttle reasons sampled through NVML every ~5 ms while the timed region runs.

    Reasons reported: hw_slowdown, hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
    (any sample with the bit set)."""

    BITS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40, "sw_power_cap": 0x4}

    def __init__(self, index):
        import threading
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(self._physical(index))
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # report, never fail the bench
            self.nv, self.err = None, f"nvml unavailable: {type(e).__name__}"
            return
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()

    @staticmethod
    def _physical(index):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            ids = [x for x in vis.split(",") if x.strip()]
            if index < len(ids) and ids[index].strip().isdigit():
                return int(ids[index])
        return index

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.reasons |= {k for k, b in self.BITS.items() if r & b}
            except Exception:
                pass
            time.sleep(0.005)

    def stop(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err], "samples": 0}
        self._stop.set()
        self.t.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


def cpu_baseline(w, seed_heads, budget_s=12.0, max_heads=8):
    """The fp64 oracle, as it stands, on a bounded sample: whole heads of the workload."""
    from oracle import express, express_a, thinformer
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    done, t_total = 0, 0.0
    for h in seed_heads[:max_heads]:
        q, k, v = W.make_qkv(w.with_(B=1), heads=[h])
        t0 = time.perf_counter()
        if w.causal:
            if w.cache == "A":
                express_a(q, k, v, w.n_exact, w.g, w.seed, heads=(w.H, [h]))
            else:
                express(q, k, v, w.n_exact, w.batch, w.g, w.seed, heads=(w.H, [h]))
        else:
            thinformer(q, k, v, w.g, w.seed, heads=(w.H, [h]))
        t_total += time.perf_counter() - t0
        done += 1
        if t_total >= budget_s:
            break
    return {"value": done * w.T / t_total, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{done} of {w.B * w.H} (b,h) slices, all {w.T} queries each: thinning + attention in fp64 numpy",
            "seconds": round(t_total, 3)}


def kernel_traffic(name):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source is unchanged since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path)).get(name)
    if not d:
        return None
    src = os.path.join(ROOT, d["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != d["sha256"]:
        return None
    return d["bytes_per_launch"]


KERNEL_SWITCHES = ("THIN_ATTN_PP", "THIN_ATTN_TC2P", "THIN_ATTN_TC1", "THIN_ATTN_TC2_PER_TILE", "THIN_ATTN_SIMT_ATTN",
                   "THIN_ATTN_OVERLAP")


def attention_traffic(w):
    """DRAM bytes per launch of the attention kernel the library picks for this workload, from the
    committed ncu summaries (Express 32K: the two-CTA kernel; Express 128K: the ping-pong kernel);
    None when another kernel is forced or the workload differs from the captured one."""
    if w.H != 32 or any(os.environ.get(k) for k in KERNEL_SWITCHES):
        return None
    return {"express32k": kernel_traffic("attention"),
            "express128k": kernel_traffic("attention_pp_express128k")}.get(w.name)


def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = W.WORKLOADS[a.workload]
    from oracle import express, express_a, thinformer
    heads = list(range(w.H)) * (1 + (a.steps + a.warmup) // max(1, w.H))
    times = []
    for i in range(a.warmup + a.steps):
        h = heads[i]
        q, k, v = W.make_qkv(w.with_(B=1), heads=[h])
        t0 = time.perf_counter()
        if w.causal:
            if w.cache == "A":
                express_a(q, k, v, w.n_exact, w.g, w.seed, heads=(w.H, [h]))
            else:
                express(q, k, v, w.n_exact, w.batch, w.g, w.seed, heads=(w.H, [h]))
        else:
            thinformer(q, k, v, w.g, w.seed, heads=(w.H, [h]))
        if i >= a.warmup:
            times.append(time.perf_counter() - t0)
    per = sum(times) / len(times)
    value = w.T / per
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": a.gpus, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": per * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": config_of(w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"one (b,h) slice per step ({w.T} queries, thinning + attention)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


class Shard:
    """This rank's part of the whole problem.

    ``batch`` (weak scaling): the whole problem has world * B batch rows and rank r holds rows
    [r B, (r+1) B) -- per-rank work fixed as the job grows.  ``heads`` (strong scaling): the whole
    problem is the workload itself and rank r holds heads [r H/N, (r+1) H/N).  Either way the
    handle's Philox counters are keyed on the whole problem's (b,h), so every rank computes exactly
    what a single run of the whole problem computes for its rows; no data crosses between ranks."""

    def __init__(self, w, world, rank, mode="batch"):
        if mode not in ("batch", "heads", "seq", "seqx"):
            raise ValueError(mode)
        if mode == "seqx" and w.mode != 1:
            raise ValueError("--shard seqx splits Express batch thinning: causal workloads with the batch cache only")
        self.split = mode == "seqx"
        mode = "seq" if mode == "seqx" else mode
        if mode == "heads" and w.H % world:
            raise ValueError(f"--shard heads needs H={w.H} divisible by the {world} ranks")
        self.mode, self.world, self.rank = mode, world, rank
        hl = w.H // world if mode == "heads" else w.H
        self.b0 = rank * w.B if mode == "batch" else 0
        self.h0 = rank * hl if mode == "heads" else 0
        self.local = w.with_(H=hl)                      # the shape this rank's handle holds
        self.heads = list(range(self.h0, self.h0 + hl))
        self.H_total = w.H
        self.global_batch = world * w.B if mode == "batch" else w.B
        self.whole_tokens = self.global_batch * w.H * w.T
        self.scaling = "weak" if mode == "batch" else "strong"
        self.parallelism = {"batch": "dp", "heads": "hp", "seq": "sp"}[mode] + ("x" if self.split else "") + str(world)
        self.q_range = (0, 0)
        if mode == "seq":
            # equal 128-aligned slices of the query rows, the last one ending at T
            step = -(-w.T // world // 128) * 128 if w.T >= 128 * world else 0
            q0, q1 = rank * step, (w.T if rank == world - 1 else (rank + 1) * step)
            if step == 0 or q0 >= q1 or q1 > w.T:
                raise ValueError(f"--shard seq needs T={w.T} >= 128 rows per rank")
            self.q_range = (q0, q1)

    @property
    def rows(self):
        """Query rows this rank attends (all of them unless --shard seq)."""
        return self.q_range if self.mode == "seq" else None

    @property
    def abi(self):
        """(b0, h0, H_total) of the handle's config."""
        return (self.b0, self.h0, self.H_total)

    def inputs(self, w):
        return W.make_qkv(w, heads=self.heads, b0=self.b0)


def max_over_ranks(x, dist, device):
    """Max of a per-rank scalar over all ranks (the step time the job is bound by)."""
    if dist is None:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def config_of(w):
    return {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "S": w.T if w.causal else w.S, "E": w.E, "D": w.D,
            "causal": w.causal, "cache": w.cache if w.causal else None, "g": w.g, "n_exact": w.n_exact,
            "batch": w.batch, "seed": w.seed,
            "l2": "inputs larger than L2 (no flush)" if 3 * w.B * w.H * w.T * w.E * 2 > 126e6 else
            "inputs smaller than L2"}


def run_decode(a):
    """Decode the whole workload one token per (b,h) and call through thin_attn_cache_decode.

    Timed with CUDA events from the end of the exact prefix to the last token.  Roofline: HBM, every
    visible key/value row read once per decoded token (the attention of a single query re-reads its
    whole key set) plus q read and out written -- the batch thinning and merges on completed batches
    are included in the time but not in these bytes."""
    import thinned_softmax_attention_b200 as TA
    w = W.WORKLOADS[a.workload]
    if not w.causal or w.cache != "B":
        raise SystemExit("--decode needs an Express workload with the 4-ary node cache")
    dev = torch.device("cuda", 0)
    q, k, v = (x.to(dev) for x in W.make_qkv(w))
    h = TA.ThinAttention(w.B, w.T, w.T, w.H, w.E, w.D, w.torch_dtype, n_exact=w.n_exact, batch=w.batch)
    plan = h.plan(True, w.g)
    cache = TA.ThinAttentionCache(w.B, w.H, w.E, w.D, w.torch_dtype, capacity=w.T, n_exact=w.n_exact,
                                  batch=w.batch, g=w.g, seed=w.seed)
    out = torch.empty(w.B, 1, w.H, w.D, dtype=w.torch_dtype, device=dev)
    ne, T = min(w.n_exact, w.T), w.T
    tail = min(256, T - ne)
    stream = torch.cuda.current_stream(dev)
    ev = {n: torch.cuda.Event(enable_timing=True) for n in ("start", "tail", "end")}
    clocks = Clocks(0)
    py_out = torch.empty(w.B, T - ne, w.H, w.D, dtype=w.torch_dtype, device=dev)   # B = 1: row views are contiguous
    for t in range(T):
        if t == ne:
            ev["start"].record(stream)
        if t == T - tail:
            ev["tail"].record(stream)
        cache.decode(q[:, t:t + 1], k[:, t:t + 1], v[:, t:t + 1], out=out if t < ne else py_out[:, t - ne:t - ne + 1])
    ev["end"].record(stream)
    torch.cuda.synchronize()
    cache.check()
    py_ms = ev["start"].elapsed_time(ev["end"])
    py_tail_ms = ev["tail"].elapsed_time(ev["end"]) / tail
    # the same tokens through thin_attn_cache_decode_n: the exact prefix in one call, then the rest in
    # one timed call (the library's per-token work without a Python round trip per token)
    cache2 = TA.ThinAttentionCache(w.B, w.H, w.E, w.D, w.torch_dtype, capacity=w.T, n_exact=w.n_exact,
                                   batch=w.batch, g=w.g, seed=w.seed)
    q2, k2, v2 = (x[:, ne:].contiguous() for x in (q, k, v))
    out2 = torch.empty_like(v2)
    if ne > 0:
        cache2.decode_n(q[:, :ne].contiguous(), k[:, :ne].contiguous(), v[:, :ne].contiguous())
    torch.cuda.synchronize()
    ev["start"].record(stream)
    cache2.decode_n(q2, k2, v2, out=out2)
    ev["end"].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    cache2.check()
    ms = ev["start"].elapsed_time(ev["end"])
    tail_ms = None
    n_tok = T - ne
    es = 4 if w.dtype == "fp32" else 2
    tt = np.arange(ne, T, dtype=np.int64)
    c, b = plan["coreset_rows"], w.batch
    kk = (tt - ne) // b
    vis = ne + c * digitsum4(kk) + (tt - (ne + kk * b) + 1)
    abytes = float(vis.sum() + 2 * n_tok) * (w.E + w.D) * es * w.B * w.H
    pk = peaks()
    gbs = abytes / (ms * 1e-3) / 1e9
    line = {"metric": "decode tokens/s (B*H tokens per decoded position) through the Express decode cache",
            "value": w.B * w.H * n_tok / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1, "higher_is_better": True,
            "dtype": w.dtype, "data": "synthetic", "config": config_of(w),
            "positions": [ne, T], "ms_per_position": round(ms / n_tok, 5),
            "entry": "thin_attn_cache_decode_n, all positions after the exact prefix in one call",
            "python_loop": {"ms_per_position": round(py_ms / n_tok, 5), "tail_ms_per_position": round(py_tail_ms, 5),
                            "entry": "ThinAttentionCache.decode, one Python call per position",
                            "value": w.B * w.H * n_tok / (py_ms * 1e-3)},
            "outputs_equal_python_loop": bool(torch.equal(out2, py_out)),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / pk["hbm_gbs"], 4), "algorithmic_bytes": abytes,
                         "note": "visible keys/values re-read per position; thinning and merges in the time only"},
            "clocks": clk}
    print(json.dumps(line))


def exact_reference_error(w, q, k, v, out, n_rows=128, max_b=4, max_h=4):
    """Approximation error of the computed output against exact softmax attention.

    Exact attention in fp64 by torch's SDPA on the host, on a seeded sample of query rows of up to
    ``max_b`` batch rows x ``max_h`` heads (outside any timed region).  Reported per (b,h) slice as
    max|o - o_exact| / max|o_exact| (worst slice), and per query row as max_d |o - o_exact| /
    max_d |o_exact| (worst row), with the mean over rows."""
    rng = np.random.default_rng(0)
    bs = list(range(min(w.B, max_b)))
    hs = sorted(set(np.linspace(0, w.H - 1, min(w.H, max_h)).round().astype(int).tolist()))
    rows = np.sort(rng.choice(w.T, min(n_rows, w.T), replace=False))
    S = k.shape[1]
    nb = len(bs)
    o = out[:nb, rows][:, :, hs].double().cpu()                        # (b, rows, h, D)
    qs = q[:nb, rows][:, :, hs].double().transpose(1, 2)               # (b, h, rows, E)
    ks = k[:nb, :, hs].double().transpose(1, 2)
    vs = v[:nb, :, hs].double().transpose(1, 2)
    mask = None
    if w.causal:
        mask = torch.as_tensor(np.arange(S)[None, :] <= rows[:, None])
    ex = torch.nn.functional.scaled_dot_product_attention(qs, ks, vs, attn_mask=mask, scale=w.scale)
    ex = ex.transpose(1, 2)                                            # (b, rows, h, D)
    d = (o - ex).abs()
    slice_err = (d.amax(dim=(1, 3)) / ex.abs().amax(dim=(1, 3))).max().item()
    row = d.amax(dim=3) / ex.abs().amax(dim=3)
    return {"vs": "exact softmax attention, fp64 (torch SDPA on the host)", "rows": len(rows),
            "batch_rows": bs, "heads": hs, "max_rel_per_slice": round(slice_err, 5),
            "max_rel_per_row": round(row.max().item(), 5), "mean_rel_per_row": round(row.mean().item(), 5)}


def attention_roofline(w, plan, attn_ms, pk, rows=None):
    """Roofline of the attention launch: bound by its arithmetic intensity against the ridge of the
    burst bf16 peak over HBM copy bandwidth.  The launch is timed alone, sub-second, at full clocks,
    so the burst peak is the denominator; the fraction of the sustained (power-capped) peak is
    reported beside it."""
    flops, abytes, pairs = attention_work(w, plan, rows)
    ridge = pk["bf16_tflops"] * 1e12 / (pk["hbm_gbs"] * 1e9)
    if w.dtype != "fp32" and flops / abytes >= ridge:
        achieved = flops / (attn_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(achieved / pk["bf16_tflops"], 4),
                "frac_sustained": round(achieved / pk["bf16_tflops_sustained"], 4),
                "peak_kind": f"bf16 dense burst ({pk['source']}); sustained {pk['bf16_tflops_sustained']}"}
    else:
        achieved = abytes / (attn_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 2), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / pk["hbm_gbs"], 4), "peak_kind": f"HBM copy ({pk['source']})"}
    roof.update({"kernel": "attention", "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": abytes,
                 "arithmetic_intensity": round(flops / abytes, 1), "ridge": round(ridge, 1),
                 "avg_launch_ms": round(attn_ms, 4)})
    return roof


def halving_roofline(w, h, ph, pk):
    """Halving launches, HBM-bound by their algorithmic bytes: every instance's n points read once and
    its n/2 survivors written once, 1.5 n (E+D) elements per instance.  Per launch from the live
    per-step CUDA events: the steps that ran in the persistent halving launch report its time on the
    first of them and 0 on the others, so they form one entry.  The headline is the launch that takes
    longest, beside the whole halving phase."""
    es = 4 if w.dtype == "fp32" else 2
    sp = h.profile_steps()
    tab = []
    for st in sp["steps"]:
        sb = st["n_inst"] * 3 * st["n"] // 2 * (w.E + w.D) * es
        kappa = st["n_inst"] * st["n"] * st["n"] // 2          # kernel evaluations of the instances' Grams
        sms = st["ms"] / max(1, sp["calls"])
        if sms == 0 and tab:
            tab[-1]["steps"].append({"n": st["n"], "n_inst": st["n_inst"]})
            tab[-1]["bytes"] += sb
            tab[-1]["kappa"] += kappa
            continue
        tab.append({"steps": [{"n": st["n"], "n_inst": st["n_inst"]}], "ms": round(sms, 4), "bytes": sb, "kappa": kappa})
    # The three floors of a halving launch: its Gram on the tensor cores (2 (E+D) flops per kernel
    # evaluation, at the burst bf16 peak), one exponential per evaluation on the MUFU pipes (16 per SM
    # per clock at the maximum SM clock, 148 SMs) and its algorithmic HBM bytes; the largest is the
    # launch's bound (HBM at every workload here).
    mufu_per_s = 148 * 16 * pk.get("sm_max_mhz", 1965.0) * 1e6
    for t in tab:
        terms = {"tensor_ms": t["kappa"] * 2 * (w.E + w.D) / (pk["bf16_tflops"] * 1e12) * 1e3,
                 "mufu_ms": t["kappa"] / mufu_per_s * 1e3,
                 "hbm_ms": t["bytes"] / (pk["hbm_gbs"] * 1e9) * 1e3}
        t["floors_ms"] = {k: round(v, 5) for k, v in terms.items()}
        t["frac"] = round(t["bytes"] / (t["ms"] * 1e-3) / 1e9 / pk["hbm_gbs"], 4) if t["ms"] > 0 else None
        t["kernel"] = (f"halving step n={t['steps'][0]['n']} x {t['steps'][0]['n_inst']} instances" if len(t["steps"]) == 1
                       else "persistent halving launch of " + " + ".join(f"{x['n_inst']} x {x['n']}" for x in t["steps"]))
    hbytes = sum(t["bytes"] for t in tab)
    hms = (ph["thin_ms"] + ph["merge_ms"]) / max(1, ph["calls"])
    top = max(tab, key=lambda t: t["ms"]) if tab else None
    if not top or top["ms"] <= 0:
        return None
    floors = top["floors_ms"]
    return {"bound": max(floors, key=floors.get)[:-3], "floors_ms": floors,
            "achieved": round(top["bytes"] / (top["ms"] * 1e-3) / 1e9, 1),
            "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": top["frac"], "kernel": top["kernel"],
            "algorithmic_bytes_per_launch": top["bytes"], "avg_launch_ms": top["ms"],
            "traffic": (None if w.name != "express32k" or w.H != 32 else
                        kernel_traffic("halving_sched") if len(top["steps"]) > 1 else
                        kernel_traffic("halving_fused_n64") if top["steps"][0]["n"] == 64 else None),
            "all_steps": {"achieved": round(hbytes / (hms * 1e-3) / 1e9, 1) if hms > 0 else None,
                          "frac": round(hbytes / (hms * 1e-3) / 1e9 / pk["hbm_gbs"], 4) if hms > 0 else None,
                          "bytes": hbytes, "ms": round(hms, 4)},
            "launches": tab}


L2_BYTES = 126e6


def timed_steps(step, steps, stream, flush):
    """CUDA-event time per step (ms).  With ``flush`` (a device buffer larger than L2) the buffer is
    rewritten before every step and each step is timed alone; otherwise the steps run back to back."""
    if flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps
    evs = []
    for _ in range(steps):
        flush.add_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / steps


def sdpa_ms(w, q, k, v, stream):
    """Exact attention at the same shape (PyTorch SDPA, the tensors' dtype), CUDA events, 3 runs."""
    try:
        qt, kt, vt = (x.transpose(1, 2) for x in (q, k, v))
        F = torch.nn.functional.scaled_dot_product_attention
        for _ in range(2):
            F(qt, kt, vt, is_causal=w.causal)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(3):
            F(qt, kt, vt, is_causal=w.causal)
        s1.record(stream)
        torch.cuda.synchronize()
        return round(s0.elapsed_time(s1) / 3, 4)
    except Exception as ex:  # report, do not fail the bench
        return f"unavailable: {type(ex).__name__}"


def measure_workload(TA, name, dev, steps, warmup):
    """One workload on this GPU alone: ms per layer (CUDA events, inputs resident in HBM), phases,
    the attention and halving rooflines and the approximation error against exact attention."""
    w = W.WORKLOADS[name]
    qc, kc, vc = W.make_qkv(w)
    q, k, v = (x.to(dev) for x in (qc, kc, vc))
    S = w.T if w.causal else w.S
    h = TA.ThinAttention(w.B, w.T, S, w.H, w.E, w.D, w.torch_dtype, n_exact=w.n_exact, batch=w.batch, device=dev.index)
    plan = h.plan(w.mode, w.g)
    h.reserve(w.mode, w.g)
    out = torch.empty(w.B, w.T, w.H, w.D, dtype=w.torch_dtype, device=dev)
    es = 4 if w.dtype == "fp32" else 2
    in_bytes = (q.numel() + k.numel() + v.numel()) * es
    flush = torch.empty(int(2 * L2_BYTES) // 4, dtype=torch.float32, device=dev) if in_bytes < L2_BYTES else None

    def step():
        h.forward(q, k, v, causal=w.mode, g=w.g, seed=w.seed, out=out)

    for _ in range(max(3, warmup)):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    h.profile(True)
    h.profile_read()
    ms = timed_steps(step, steps, stream, flush)
    h.profile(False)
    ph = h.profile_read()
    pk = peaks()
    attn_ms = ph["attn_ms"] / max(1, ph["calls"])
    rec = {"workload": name, "ms_per_layer": round(ms, 5), "tokens_per_s": w.B * w.H * w.T / (ms * 1e-3),
           "steps": steps, "l2": "flushed before every step (inputs smaller than L2)" if flush is not None else
           "inputs larger than L2 (no flush)",
           "phases_ms": {"thin_ms": round(ph["thin_ms"] / max(1, ph["calls"]), 4),
                         "merge_ms": round(ph["merge_ms"] / max(1, ph["calls"]), 4), "attn_ms": round(attn_ms, 4)},
           "roofline": dict(attention_roofline(w, plan, attn_ms, pk), traffic=attention_traffic(w)),
           "halving_roofline": halving_roofline(w, h, ph, pk),
           "gpu_launches_per_step": plan["kernel_launches"]}
    rec["approx_error"] = exact_reference_error(w, qc, kc, vc, out)
    rec["exact_sdpa_ms"] = sdpa_ms(w, q, k, v, stream)
    h.close()
    del q, k, v, out, flush
    torch.cuda.empty_cache()
    return rec


def main():
    a = args_()
    if a.impl == "reference":
        return run_reference(a)
    if a.decode:
        return run_decode(a)
    import thinned_softmax_attention_b200 as TA
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    wl = W.WORKLOADS[a.workload] if a.heads <= 0 else W.WORKLOADS[a.workload].with_(H=a.heads)
    shard = Shard(wl, world, rank, a.shard)
    w = shard.local
    qc, kc, vc = shard.inputs(w)
    q, k, v = (x.to(dev) for x in (qc, kc, vc))
    S = w.T if w.causal else w.S
    h = TA.ThinAttention(w.B, w.T, S, w.H, w.E, w.D, w.torch_dtype, n_exact=w.n_exact, batch=w.batch,
                         device=local, shard=shard.abi, q_range=shard.q_range, thin_split=shard.split)
    plan = h.plan(w.mode, w.g)
    h.reserve(w.mode, w.g)
    out = torch.empty(w.B, w.T, w.H, w.D, dtype=w.torch_dtype, device=dev)
    es = 4 if w.dtype == "fp32" else 2
    in_bytes = (q.numel() + k.numel() + v.numel()) * es
    flush = torch.empty(int(2 * L2_BYTES) // 4, dtype=torch.float32, device=dev) if in_bytes < L2_BYTES else None

    def step():
        if shard.split:
            # own batches, the coreset exchange (one all-gather over the ranks), merges + attention
            h.forward_phase(q, k, v, phase=1, g=w.g, seed=w.seed)
            if dist:
                TA.exchange_batch_coresets(h, w.g, dist)
            h.forward_phase(q, k, v, phase=2, g=w.g, seed=w.seed, out=out)
        else:
            h.forward(q, k, v, causal=w.mode, g=w.g, seed=w.seed, out=out)

    for _ in range(max(3, a.warmup)):
        step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = Clocks(local)
    time.sleep(0.02)
    h.profile(True)
    h.profile_read()
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize()
    step_ms = timed_steps(step, a.steps, stream, flush)
    if dist:
        dist.barrier()
    clk = clocks.stop()
    h.profile(False)
    ph = h.profile_read()
    ms = max_over_ranks(step_ms, dist, dev)
    value = shard.whole_tokens / (ms * 1e-3)

    pk = peaks()
    if shard.split:
        # a phased forward records no per-phase events: the step time is the measurement
        roof = {"unavailable": "per-phase times are not recorded for split-thinning forwards"}
        halving_roof = None
        phases = None
    else:
        attn_ms = ph["attn_ms"] / max(1, ph["calls"])
        roof = attention_roofline(w, plan, attn_ms, pk, shard.rows)
        roof["traffic"] = attention_traffic(w) if shard.rows is None else None
        halving_roof = halving_roofline(w, h, ph, pk)
        phases = {"thin_ms": round(ph["thin_ms"] / max(1, ph["calls"]), 4),
                  "merge_ms": round(ph["merge_ms"] / max(1, ph["calls"]), 4),
                  "attn_ms": round(attn_ms, 4)}

    e2e = None
    if not a.no_e2e and shard.rows is not None:
        # the host-buffer entry takes no query-row range: the inputs go in by pinned copies, this
        # rank's rows of out come back the same way, all on the timed stream
        q0, q1 = shard.rows
        qh, kh, vh = (x.pin_memory() for x in (qc, kc, vc))
        oh = torch.empty(w.B, q1 - q0, w.H, w.D, dtype=w.torch_dtype).pin_memory()

        def e2e_step():
            for dst, src in ((q, qh), (k, kh), (v, vh)):
                dst.copy_(src, non_blocking=True)
            step()
            oh.copy_(out[:, q0:q1], non_blocking=True)

        for _ in range(2):
            e2e_step()
        n_e2e = max(2, min(a.steps, 5))
        if dist:
            dist.barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        f1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(f0.elapsed_time(f1) / n_e2e, dist, dev)
        e2e = {"value": shard.whole_tokens / (ems * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": (q.numel() + k.numel() + v.numel()) * es,
               "d2h_bytes_per_step": oh.numel() * es, "ms_per_step": round(ems, 3)}
    elif not a.no_e2e:
        qh, kh, vh = (x.pin_memory() for x in (qc, kc, vc))
        oh = torch.empty(w.B, w.T, w.H, w.D, dtype=w.torch_dtype).pin_memory()
        for _ in range(2):
            h.forward_host(qh, kh, vh, oh, causal=w.mode, g=w.g, seed=w.seed)
        n_e2e = max(2, min(a.steps, 5))
        if dist:
            dist.barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(n_e2e):
            h.forward_host(qh, kh, vh, oh, causal=w.mode, g=w.g, seed=w.seed)
        f1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(f0.elapsed_time(f1) / n_e2e, dist, dev)
        e2e = {"value": shard.whole_tokens / (ems * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": (q.numel() + k.numel() + v.numel()) * es,
               "d2h_bytes_per_step": out.numel() * es, "ms_per_step": round(ems, 3)}

    sdpa = None
    if not a.no_sdpa and rank == 0:
        sdpa = sdpa_ms(w, q, k, v, stream)

    approx = None
    per_workload = None
    if rank == 0 and world == 1:
        approx = exact_reference_error(w, qc, kc, vc, out)
        if not a.no_per_workload:
            h.close()
            del q, k, v, out, flush
            torch.cuda.empty_cache()
            per_workload = {}
            for name in ("tiny", "vit", "biggan", "express128k"):
                if name != a.workload:
                    per_workload[name] = measure_workload(TA, name, dev, 10 if name == "express128k" else 20,
                                                          a.warmup)

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = cpu_baseline(w, list(range(w.H)))

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
            "warmup": max(3, a.warmup), "ms_per_step": ms, "higher_is_better": True, "scaling": shard.scaling,
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {**config_of(wl), "global_batch": shard.global_batch,
                       "parallelism": shard.parallelism, "heads_per_gpu": w.H},
            "ms_per_layer": ms, "phases_ms": phases, "roofline": roof, "halving_roofline": halving_roof,
            "approx_error": approx, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": plan["kernel_launches"] * a.steps, "clocks": clk, "exact_sdpa_ms": sdpa,
            "workspace_bytes": plan["workspace_bytes"], "per_workload": per_workload}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
