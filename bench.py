#!/usr/bin/env python
"""RecSA benchmark: decode queries/s (append + decode per step) and prefill
tokens/s on the Qwen3-4B-shaped layer at L = 524288, one B200 per rank.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl recsa|reference]

One step = one decode step of the whole hot path for the batch: recsa_append
of each sequence's new token (tree maintenance) then recsa_decode (level-wise
selection + shared-softmax gather attention).  Prefill (recsa_build over the
whole context, then recsa_prefill of every position) and a dense attention
comparator (torch SDPA, a library kernel) are measured once per run and
reported beside the main number.  Multi-GPU runs are independent replicas
(weak scaling): each rank serves its own batch; the time is the max over ranks.

The CPU oracle is executed only by the cpu_baseline leg and by --impl
reference (it is the reference arm: a float64 restatement of the method).
"""

from __future__ import annotations

import argparse
import hashlib
import json
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

from hierarchical_sparse_attention_recsa_b200 import counts, synth  # noqa: E402
from hierarchical_sparse_attention_recsa_b200 import recsa as R  # noqa: E402

METRIC = "decode queries/s and prefill tokens/s at L=524K on 1 B200; % of HBM roofline"
WORKLOAD = "qwen3-4b-524k"
NOMINAL_HBM_GBS = 8000.0     # roofline denominator named by the workload definition
ALU_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # fp32 FMA lanes x 2 x max SM clock


def bf16_peak():
    return peaks()[1]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------------------
# clocks sampler
# ---------------------------------------------------------------------------

class Clocks:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(),
                                 f"recsa_clocks_rank{device}_{os.getpid()}.csv")
        self.sel = []
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid).lower()
            rows = subprocess.run(["nvidia-smi", "--query-gpu=index,uuid",
                                   "--format=csv,noheader"], capture_output=True, text=True,
                                  timeout=20).stdout.strip().splitlines()
            for row in rows:
                idx, u = [x.strip() for x in row.split(",")]
                if uuid.replace("gpu-", "") in u.lower():
                    self.sel = ["-i", idx]
        except Exception:
            pass

    def start(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", *self.sel, "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            # wait for the first sample so that the timed region is covered
            t0 = time.time()
            while time.time() - t0 < 10 and os.path.getsize(self.path) == 0:
                time.sleep(0.05)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def geometry(w, batch, capacity) -> R.Geometry:
    return R.Geometry(head_dim=w.head_dim, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                      leaf_block=w.leaf_block, branching=w.branching, k=w.k, window=w.window,
                      batch=batch, capacity=capacity,
                      dtype=R.DTYPE_BF16 if w.dtype == torch.bfloat16 else R.DTYPE_F32,
                      rope_enabled=1, rope_base=w.rope_base)


def metric_for(name, L):
    if name == WORKLOAD:
        return METRIC
    return f"decode queries/s and prefill tokens/s at L={L} ({name}) on 1 B200; % of HBM roofline"


def elem_bytes(w):
    return 2 if w.dtype == torch.bfloat16 else 4


class L2Flush:
    """Write 256 MiB (twice the L2) before a timed region, then keep the GPU
    busy for ~100 us so that the host has queued the timed launch before the
    start event is reached: the events then bracket device time only, not the
    host's launch latency."""

    def __init__(self, mib=256, spin_cycles=200_000):
        self.buf = torch.empty(mib << 20, dtype=torch.uint8, device="cuda")
        self.spin = spin_cycles

    def __call__(self):
        self.buf.fill_(1)
        torch.cuda._sleep(self.spin)


DECODE_SOURCES = ["decode_cluster.cu", "rows.cuh", "pool.cuh", "recsa_internal.cuh"]
TRAFFIC_PROFILE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles",
                               "decode_cluster_kernel_qwen3-4b-524k_traffic.md")


def measured_traffic(workload, L, batch):
    """DRAM bytes per decode launch from the committed ncu capture of the same
    workload, or None when the workload differs or the kernel sources have
    changed since the capture (their sha256 no longer matches)."""
    if workload != WORKLOAD or L != synth.WORKLOADS[WORKLOAD].length or \
            batch != synth.WORKLOADS[WORKLOAD].batch or not os.path.exists(TRAFFIC_PROFILE):
        return None
    fields = {}
    for line in open(TRAFFIC_PROFILE):
        if ":" in line and line.split(":")[0] in ("traffic_bytes_per_launch", "source_sha256"):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    h = hashlib.sha256()
    csrc = os.path.join(os.path.dirname(os.path.abspath(R.__file__)), "csrc")
    for f in DECODE_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    if fields.get("source_sha256") != h.hexdigest() or "traffic_bytes_per_launch" not in fields:
        return None
    return float(fields["traffic_bytes_per_launch"])


VARIANT_SOURCES = ["zha_attend.cu", "decode_cluster.cu", "rows.cuh", "pool.cuh",
                   "recsa_internal.cuh"]
VARIANT_PROFILE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles",
                               "selection_variants_qwen3-4b-524k_traffic.md")


def measured_variant_traffic(leg, workload, L, batch):
    """DRAM bytes per launch of a selection-variant leg from the committed ncu
    capture of the same workload, or None (other workload, or the kernel
    sources changed since the capture)."""
    if workload != WORKLOAD or L != synth.WORKLOADS[WORKLOAD].length or \
            batch != synth.WORKLOADS[WORKLOAD].batch or not os.path.exists(VARIANT_PROFILE):
        return None
    fields = {}
    for line in open(VARIANT_PROFILE):
        if ":" in line and (line.startswith("traffic_bytes_per_launch[") or
                            line.startswith("source_sha256")):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    h = hashlib.sha256()
    csrc = os.path.join(os.path.dirname(os.path.abspath(R.__file__)), "csrc")
    for f in VARIANT_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    key = f"traffic_bytes_per_launch[{leg}]"
    if fields.get("source_sha256") != h.hexdigest() or key not in fields:
        return None
    return float(fields[key])


def elapsed(a, b):
    return a.elapsed_time(b)


def max_over_ranks(ms: float, world: int) -> float:
    """The largest of the ranks' device times (every rank calls it, in the same
    order); one rank: unchanged.  The tensor lives where the process group's
    backend communicates (CUDA for NCCL, host memory for gloo)."""
    if world == 1:
        return ms
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: int, world: int, ms: float) -> float:
    """Whole-job throughput: the units all ranks processed (weak scaling: the
    same number per rank) over the slowest rank's time."""
    return units_per_rank * world / (ms / 1e3)


def make_prefill_queries(w, K, q0, L, chunk=65536):
    Q = torch.empty((1, L - q0, w.n_q_heads, w.head_dim), dtype=w.dtype, device="cuda")
    for c0 in range(q0, L, chunk):
        n = min(chunk, L - c0)
        pos = (c0 + torch.arange(n, device="cuda", dtype=torch.int64))[None]
        q, _, _ = synth.make_queries(w, K[:1], pos, seed=100 + c0 // chunk)
        Q[:, c0 - q0:c0 - q0 + n] = q
    return Q


# ---------------------------------------------------------------------------
# RecSA arm
# ---------------------------------------------------------------------------

def run_recsa(args, rank, world, dev, cpu=None):
    w = synth.WORKLOADS[args.workload]
    if args.length:
        w = synth.Workload(**{**w.__dict__, "length": args.length})
    L, batch = w.length, w.batch
    K_steps, W_steps = args.steps, args.warmup
    n_stage = max(K_steps, W_steps)
    cap = L + max(512, n_stage + 1)
    hbm_gbs, bf16_tflops, peak_kind = peaks()
    torch.manual_seed(0)
    Kc, Vc, r = synth.make_kv(w, cap, seed=rank, device="cuda", batch=batch)
    r = r.contiguous()
    g = geometry(w, batch, cap)
    tree = torch.zeros(R.recsa_tree_bytes(g), dtype=torch.uint8, device="cuda")
    R.recsa_build(g, Kc, Vc, [L] * batch, r, 0, tree)
    # per-step inputs: queries at the new positions and the tokens to append
    pos = (L + torch.arange(n_stage, device="cuda", dtype=torch.int64))[None].expand(batch, -1)
    Qall, kind, _ = synth.make_queries(w, Kc, pos.contiguous(), seed=1 + rank)
    Qs = Qall.permute(1, 0, 2, 3).unsqueeze(2).contiguous()       # [step][batch][1][Hq][d]
    kn = Kc[:, :, L:L + n_stage].permute(2, 0, 1, 3).contiguous()  # [step][batch][Hkv][d]
    vn = Vc[:, :, L:L + n_stage].permute(2, 0, 1, 3).contiguous()
    O = torch.empty_like(Qs[0])
    lens = torch.full((batch,), L, dtype=torch.int64, device="cuda")
    lens0 = lens.clone()
    ti = R.recsa_trace_ints(g)
    traces = torch.zeros((K_steps, batch, 1, w.n_q_heads, ti), dtype=torch.int32, device="cuda")
    flush = L2Flush()
    stream = torch.cuda.current_stream()

    def step(i):
        R.recsa_decode_step(g, Qs[i], Kc, Vc, kn[i], vn[i], lens, r, 0, tree, 1, O)

    clocks = Clocks(dev)
    clocks.start()      # samples the warm-up, the timed steps and the e2e steps
    for i in range(W_steps):
        step(i)
    lens.copy_(lens0)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K_steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    for i in range(K_steps):
        flush()
        ev[i][0].record(stream)
        R.recsa_decode_step(g, Qs[i], Kc, Vc, kn[i], vn[i], lens, r, 0, tree, 1, O)
        ev[i][1].record(stream)
        # untimed: the same query decoded again with its selection trace, for accounting
        R.recsa_decode(g, Qs[i], Kc, Vc, tree, lens, 1, O, traces[i])
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    step_ms = sum(elapsed(e[0], e[1]) for e in ev)
    dec_ms = step_ms / K_steps
    # the same steps as two launches (recsa_append, then recsa_decode), for reference
    lens.copy_(lens0)
    ev3 = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K_steps)]
    torch.cuda.synchronize()
    for i in range(K_steps):
        flush()
        ev3[i][0].record(stream)
        R.recsa_append(g, Kc, Vc, kn[i], vn[i], lens, r, 0, tree)
        ev3[i][1].record(stream)
        R.recsa_decode(g, Qs[i], Kc, Vc, tree, lens, 1, O)
        ev3[i][2].record(stream)
    torch.cuda.synchronize()
    app_ms = sum(elapsed(e[0], e[1]) for e in ev3) / K_steps
    two_dec_ms = sum(elapsed(e[1], e[2]) for e in ev3) / K_steps
    step_ms = max_over_ranks(step_ms, world)
    value = job_rate(batch * K_steps, world, step_ms)

    # algorithmic bytes of the decode launches, from the traces
    tr = traces.cpu().numpy()
    acc = []
    for i in range(K_steps):
        lens_i = np.full(batch, L + i + 1)
        acc.append(counts.decode_bytes_from_trace(tr[i], lens_i, w.leaf_block, w.branching,
                                                  w.window, w.n_q_heads // w.n_kv_heads,
                                                  w.head_dim, elem_bytes(w), w.k))
    dec_bytes = float(np.mean([a["bytes"] for a in acc]))
    achieved = dec_bytes / (dec_ms / 1e3) / 1e9

    # end to end through the public API with host buffers
    def run_e2e():
        # Each step's inputs (Q, k_new, v_new) sit back to back in one pinned
        # host row and travel in one copy; the library gets views of the device
        # row (every part starts on a 16-byte boundary).
        esz = Qs.element_size()
        nq_, nk_ = Qs[0].numel(), kn[0].numel()
        row = nq_ + 2 * nk_
        host = torch.empty((K_steps, row), dtype=Qs.dtype).pin_memory()
        for i in range(K_steps):
            host[i, :nq_] = Qs[i].reshape(-1).cpu()
            host[i, nq_:nq_ + nk_] = kn[i].reshape(-1).cpu()
            host[i, nq_ + nk_:] = vn[i].reshape(-1).cpu()
        dev = torch.empty((row,), dtype=Qs.dtype, device="cuda")
        Qd = dev[:nq_].view(Qs[0].shape)
        knd = dev[nq_:nq_ + nk_].view(kn[0].shape)
        vnd = dev[nq_ + nk_:].view(vn[0].shape)
        assert (nq_ * esz) % 16 == 0 and (nk_ * esz) % 16 == 0
        Oh = torch.empty((K_steps,) + tuple(O.shape), dtype=O.dtype).pin_memory()
        lens.copy_(lens0)
        ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K_steps)]
        torch.cuda.synchronize()
        for i in range(K_steps):
            flush()
            ev2[i][0].record(stream)
            dev.copy_(host[i], non_blocking=True)
            R.recsa_decode_step(g, Qd, Kc, Vc, knd, vnd, lens, r, 0, tree, 1, O)
            Oh[i].copy_(O, non_blocking=True)
            ev2[i][1].record(stream)
        torch.cuda.synchronize()
        e2e_ms = sum(elapsed(a, b) for a, b in ev2)
        e2e_ms = max_over_ranks(e2e_ms, world)
        return {"value": job_rate(batch * K_steps, world, e2e_ms), "unit": "queries/s",
                "h2d_bytes_per_step": int(row * esz),
                "d2h_bytes_per_step": int(O.numel() * O.element_size())}

    e2e = None if args.only_decode else run_e2e()
    clk = clocks.stop()

    out = {
        "metric": metric_for(args.workload, L), "value": value, "unit": "queries/s",
        "n_gpus": world,
        "steps": K_steps, "warmup": W_steps, "ms_per_step": step_ms / K_steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32",
        "data": "synthetic: K,V ~ N(0,1) x per-channel LogNormal(0,0.5) scale, Q ~ N(0,1), "
                "1% planted needles, seeded",
        "config": {"workload": args.workload, "L": L, "batch": batch, "q_heads": w.n_q_heads,
                   "kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
                   "leaf_block": w.leaf_block, "branching": w.branching, "k": w.k,
                   "window": w.window, "levels": R.recsa_num_levels(g, L),
                   "step": "recsa_decode_step (append + decode in one launch) for the batch",
                   "l2": "flushed before every timed step (256 MiB write, outside the events; "
                         "the GPU is kept busy past the flush so the events bracket device "
                         "time, not host launch latency)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "kernel": "decode_cluster_kernel (fused step)",
                     "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                     "frac": achieved / hbm_gbs, "peak_kind": peak_kind,
                     "frac_of_8tbs": achieved / NOMINAL_HBM_GBS,
                     "bytes_per_launch": dec_bytes, "launch_ms": dec_ms,
                     "traffic": measured_traffic(args.workload, L, batch)},
        "decode_ms": dec_ms,
        "two_launches": {"append_ms": app_ms, "decode_ms": two_dec_ms,
                         "step_ms": app_ms + two_dec_ms},
        "e2e": e2e, "gpu_launches": K_steps, "clocks": clk,
    }
    del traces
    torch.cuda.empty_cache()
    if not args.no_prefill and args.workload != "decode-1m":
        out["prefill"] = run_prefill(args, w, Kc, Vc, r, cap, flush, stream, hbm_gbs)
        if not args.no_zha:
            out["zha_prefill"] = run_zha_prefill(args, w, Kc, Vc, r, cap, flush, stream)
    if not args.no_dense:
        out["dense"] = run_dense(args, w, Kc, Vc, Qs, cap, flush, stream, out.get("prefill"))
    if cpu is not None:
        out["cpu_baseline"] = cpu_baseline(cpu, seconds=args.cpu_seconds)
    cpu_leg = cpu
    if not args.no_zha:
        out["zha"] = run_variant(args, w, Kc, Vc, r, L, cap, Qs, flush, stream, hbm_gbs,
                                 peak_kind, R.MODE_ZHA, cpu_leg, leg="zha")
        out["zha_multiref"] = run_variant(args, w, Kc, Vc, r, L, cap, Qs, flush, stream,
                                          hbm_gbs, peak_kind, R.MODE_ZHA, cpu_leg,
                                          n_ref=ZHA_N_REF, leg="zha_multiref")
        out["zha_multiref_fp8"] = run_variant(args, w, Kc, Vc, r, L, cap, Qs, flush, stream,
                                              hbm_gbs, peak_kind, R.MODE_ZHA, None,
                                              n_ref=ZHA_N_REF, key_format=R.KEYS_FP8,
                                              leg="zha_multiref_fp8")
        out["zha_multiref_nvfp4"] = run_variant(args, w, Kc, Vc, r, L, cap, Qs, flush, stream,
                                                hbm_gbs, peak_kind, R.MODE_ZHA, None,
                                                n_ref=ZHA_N_REF, key_format=R.KEYS_NVFP4,
                                                leg="zha_multiref_nvfp4")
    if not args.no_group:
        out["group"] = run_variant(args, w, Kc, Vc, r, L, cap, Qs, flush, stream, hbm_gbs,
                                   peak_kind, R.MODE_GROUP, cpu_leg, leg="group")
    return out


ZHA_TOP_P = 0.9
ZHA_N_REF = 16     # reference queries per pooler in the pages' trained routers


def reference_queries(r, n_ref, seed=7):
    """n_ref reference queries: r, then n_ref - 1 more from its distribution
    (N(0, 1/d)), seeded; [n_ref, d] fp32 on r's device."""
    gen = torch.Generator().manual_seed(seed)
    d = r.shape[-1]
    extra = torch.randn((n_ref - 1, d), generator=gen) / d ** 0.5
    return torch.cat([r.reshape(1, d).float().cpu(), extra]).contiguous().to(r.device)


def run_variant(args, w, Kc, Vc, r, L, cap, Qs, flush, stream, hbm_gbs, peak_kind, mode, cpu,
                n_ref=1, key_format=0, leg=""):
    """A selection variant on the same cache: its own tree (same pooling),
    then the batch's decode queries at t = L - 1, timed per launch like the
    main decode.  MODE_ZHA: top-p expansion, exact tokens of the reached
    leaves and the window at true positions (the RoPE table covers every
    position), with n_ref reference queries per pooler and fp32 or FP8
    (key_format) summary keys.  MODE_GROUP: RecSA with one selection per KV
    group."""
    batch = Kc.shape[0]
    zha = mode == R.MODE_ZHA
    g = R.Geometry(head_dim=w.head_dim, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                   leaf_block=w.leaf_block, branching=w.branching, k=w.k, window=w.window,
                   batch=batch, capacity=cap,
                   dtype=R.DTYPE_BF16 if w.dtype == torch.bfloat16 else R.DTYPE_F32,
                   rope_enabled=1, rope_base=w.rope_base, mode=mode,
                   top_p=ZHA_TOP_P if zha else 0.0, n_ref=n_ref, key_format=key_format)
    tree = torch.zeros(R.recsa_tree_bytes(g), dtype=torch.uint8, device="cuda")
    refs = reference_queries(r, n_ref) if n_ref > 1 else r
    R.recsa_build(g, Kc, Vc, [L] * batch, refs, 0, tree)
    build = time_build(g, Kc, Vc, L, batch, refs, tree, flush, stream, w, n_ref) \
        if n_ref > 1 else None
    lens = torch.full((batch,), L, dtype=torch.int64, device="cuda")
    O = torch.empty_like(Qs[0])
    n = min(args.steps, Qs.shape[0])
    traces = torch.zeros((n, batch, 1, w.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                         device="cuda")
    for i in range(args.warmup):
        R.recsa_decode(g, Qs[i % Qs.shape[0]], Kc, Vc, tree, lens, 1, O)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
    torch.cuda.synchronize()
    for i in range(n):
        flush()
        ev[i][0].record(stream)
        R.recsa_decode(g, Qs[i], Kc, Vc, tree, lens, 1, O)
        ev[i][1].record(stream)
        R.recsa_decode(g, Qs[i], Kc, Vc, tree, lens, 1, O, traces[i])   # untimed, for counts
    torch.cuda.synchronize()
    dec_ms = sum(elapsed(a, b) for a, b in ev) / n
    tr = traces.cpu().numpy()
    G = w.n_q_heads // w.n_kv_heads
    d = w.head_dim   # stored bytes of one key row
    key_bytes = {R.KEYS_F32: 4 * d, R.KEYS_FP8: d + 4, R.KEYS_NVFP4: d // 2 + d // 16 + 4}[key_format]
    nb = [counts.decode_bytes_from_trace(tr[i], np.full(batch, L), w.leaf_block, w.branching,
                                         w.window, G, w.head_dim, elem_bytes(w), w.k,
                                         summary_values=not zha, keys_per_node=n_ref,
                                         key_row_bytes=key_bytes)["bytes"] for i in range(n)]
    kept = tr[..., 4 + 16:4 + 16 + R.recsa_num_levels(g, L)].astype(np.float64)
    nbytes = float(np.mean(nb))
    achieved = nbytes / (dec_ms / 1e3) / 1e9
    res = {"value": batch / (dec_ms / 1e3), "unit": "queries/s", "decode_ms": dec_ms,
           "kernel": "zha_attend_kernel (one CTA per query head)" if zha else
                     "decode_cluster_kernel (all G heads per CTA, one selection per KV group)",
           "kept_per_level_mean": [float(x) for x in kept.mean(axis=(0, 1, 2, 3))],
           "exact_tokens_mean": float(tr[..., 3].mean()),
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                        "frac": achieved / hbm_gbs, "peak_kind": peak_kind,
                        "bytes_per_launch": nbytes,
                        "traffic": measured_variant_traffic(leg, args.workload, L, batch)}}
    if build is not None:
        res["build"] = build
    if zha:
        res["top_p"] = ZHA_TOP_P
        res["n_ref"] = n_ref
        res["keys"] = {R.KEYS_F32: "fp32", R.KEYS_FP8: "fp8_e4m3 + fp32 row scale",
                       R.KEYS_NVFP4: "nvfp4 (e2m1, e4m3 per 16, fp32 per row)"}[key_format]
    del tree, traces
    torch.cuda.empty_cache()
    if cpu is not None:
        variant = ("zha" if n_ref == 1 else "zha_multiref") if zha else "group"
        res["cpu_baseline"] = cpu_baseline(cpu, seconds=min(args.cpu_seconds, 10.0),
                                           variant=variant)
    return res


def time_build(g, Kc, Vc, L, batch, refs, tree, flush, stream, w, n_ref, reps=3):
    """recsa_build of the batch's trees with n_ref reference queries (level 1
    on the tensor-core pooler: one read of K and V, the scores and the pooling
    as TF32 products with split fp32 operands).  HBM roofline over the K and V
    read; tensor fraction = TF32 flops (scores and pooling, each 2 x tokens x d
    x R x 2 operand parts, R padded to a multiple of 16) over the TF32 peak,
    taken as the measured bf16 peak x 1/2 (the nominal TF32 : BF16 ratio)."""
    ts = []
    for _ in range(reps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        R.recsa_build(g, Kc, Vc, [L] * batch, refs, 0, tree)
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(elapsed(e0, e1))
    ms = min(ts)
    hbm_gbs, bf16_tflops, peak_kind = peaks()
    kv = 2 * batch * w.n_kv_heads * L * w.head_dim * elem_bytes(w)
    nr = (n_ref + 15) // 16 * 16
    flops = 2 * 2 * 2 * float(batch * w.n_kv_heads * (L // w.leaf_block) * w.leaf_block) * \
        w.head_dim * nr
    tf32_peak = bf16_tflops / 2
    return {"ms": ms, "kernel": "leaf_multiref_tc_kernel + parent_kernel",
            "roofline": {"bound": "hbm", "achieved": kv / (ms / 1e3) / 1e9, "peak": hbm_gbs,
                         "unit": "GB/s", "frac": kv / (ms / 1e3) / 1e9 / hbm_gbs,
                         "peak_kind": peak_kind, "bytes": kv},
            "tensor": {"achieved": flops / (ms / 1e3) / 1e12, "peak": tf32_peak,
                       "unit": "TFLOP/s", "frac": flops / (ms / 1e3) / 1e12 / tf32_peak,
                       "peak_note": "tf32 = measured bf16 x 1/2 (nominal ratio)",
                       "flops": flops}}


def run_prefill(args, w, Kc, Vc, r, cap, flush, stream, hbm_gbs):
    """recsa_build over one sequence's L tokens, then recsa_prefill of the
    workload's query range (all L positions, or the last prefill_queries)."""
    L = w.length
    q0 = L - w.extra.get("prefill_queries", L)
    gp = geometry(w, 1, cap)
    K0, V0 = Kc[:1], Vc[:1]
    tree = torch.zeros(R.recsa_tree_bytes(gp), dtype=torch.uint8, device="cuda")
    Q = make_prefill_queries(w, Kc, q0, L)
    O = torch.empty_like(Q)
    chunk = 65536
    ws = None if args.no_window_ws else torch.empty(R.recsa_prefill_workspace_bytes(gp, chunk),
                                                    dtype=torch.uint8, device="cuda")

    def once():
        R.recsa_build(gp, K0, V0, [L], r, 0, tree)
        for c0 in range(q0, L, chunk):
            n = min(chunk, L - c0)
            R.recsa_prefill(gp, Q[:, c0 - q0:c0 - q0 + n], K0, V0, tree, c0, n,
                            O[:, c0 - q0:c0 - q0 + n], workspace=ws)

    once()
    torch.cuda.synchronize()
    times, build_t = [], []
    for _ in range(args.prefill_reps):
        flush()
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record(stream)
        R.recsa_build(gp, K0, V0, [L], r, 0, tree)
        e1.record(stream)
        for c0 in range(q0, L, chunk):
            n = min(chunk, L - c0)
            R.recsa_prefill(gp, Q[:, c0 - q0:c0 - q0 + n], K0, V0, tree, c0, n,
                            O[:, c0 - q0:c0 - q0 + n], workspace=ws)
        e2.record(stream)
        torch.cuda.synchronize()
        times.append(elapsed(e0, e2))
        build_t.append(elapsed(e0, e1))
    ms = min(times)
    t = np.arange(q0, L)
    ent, keys = counts.per_query_counts(t, w.leaf_block, w.branching, w.k, w.window,
                                        R.recsa_num_levels(gp, L))
    flops = float(2 * w.head_dim * (ent.sum() + keys.sum()) * w.n_q_heads)
    attend_ms = ms - min(build_t)
    kv_bytes = 2 * L * w.n_kv_heads * w.head_dim * elem_bytes(w)
    build_ms = min(build_t)
    # bytes the prefill touches (the workload definition's HBM roofline): the
    # sequence's K and V (every token is in some query's window or kept leaf),
    # every tree node (fp32 key and value), Q read and O written once
    nodes = sum(L // (w.leaf_block * w.branching ** l) for l in range(R.recsa_num_levels(gp, L)))
    tree_bytes = nodes * w.n_kv_heads * w.head_dim * 4 * 2
    qo_bytes = 2 * (L - q0) * w.n_q_heads * w.head_dim * elem_bytes(w)
    touched = kv_bytes + tree_bytes + qo_bytes
    del Q, O, tree
    torch.cuda.empty_cache()
    hbm_ach = touched / (attend_ms / 1e3) / 1e9
    return {"value": (L - q0) / (ms / 1e3), "unit": "tokens/s", "ms": ms,
            "reps": args.prefill_reps, "build_ms": build_ms, "attend_ms": attend_ms,
            "queries": L - q0, "q_start": q0, "tokens_built": L,
            "roofline": {"bound": "hbm", "kernel": PREFILL_KERNELS,
                         "achieved": hbm_ach, "peak": hbm_gbs, "unit": "GB/s",
                         "frac": hbm_ach / hbm_gbs, "frac_of_8tbs": hbm_ach / NOMINAL_HBM_GBS,
                         "bytes": touched, "bytes_kv": kv_bytes, "bytes_tree": tree_bytes,
                         "bytes_qo": qo_bytes, "traffic": None,
                         "note": "touched K/V, tree and Q/O over the prefill time (after the "
                                 "build); the path is compute-bound, see compute_roofline"},
            "tensor_roofline": {"bound": "tensor", "kernel": PREFILL_KERNELS,
                                "achieved": flops / (attend_ms / 1e3) / 1e12,
                                "peak": bf16_peak() / 2, "unit": "TFLOP/s",
                                "frac": flops / (attend_ms / 1e3) / 1e12 / (bf16_peak() / 2),
                                "peak_note": "TF32 = measured bf16 peak x 1/2 (nominal ratio): "
                                             "the window, tree-level and kept-leaf products run "
                                             "as TF32 tcgen05 MMAs; algorithmic flops as below",
                                "flops": flops},
            "compute_roofline": {"bound": "alu", "kernel": PREFILL_KERNELS,
                                 "achieved": flops / (attend_ms / 1e3) / 1e12,
                                 "peak": ALU_PEAK_TFLOPS, "unit": "TFLOP/s",
                                 "frac": flops / (attend_ms / 1e3) / 1e12 / ALU_PEAK_TFLOPS,
                                 "flops": flops,
                                 "flops_rule": "2 d (keys read + softmax entries) per query "
                                               "head, closed-form counts"},
            "build_roofline": {"bound": "hbm", "kernel": "leaf_kernel + parent_kernel",
                               "achieved": kv_bytes / (build_ms / 1e3) / 1e9,
                               "peak": hbm_gbs, "unit": "GB/s",
                               "frac": kv_bytes / (build_ms / 1e3) / 1e9 / hbm_gbs,
                               "tensor_pipe_frac": 0.0,
                               "tensor_note": "one reference query: the pooler scores each "
                                              "row with one dot product (a [B x d] by [d x 1] "
                                              "product) on CUDA cores; the tensor pipe is "
                                              "unused"}}


PREFILL_KERNELS = ("window_tc_kernel + score_tc_kernel + select_kernel + leaf_tc_kernel + "
                   "merge_kernel (window, tree levels and kept leaves on tcgen05)")


ZHA_PREFILL_QUERIES = 65536


def run_zha_prefill(args, w, Kc, Vc, r, cap, flush, stream):
    """ZHA routing (p = ZHA_TOP_P, fp32 keys) prefill of the last
    ZHA_PREFILL_QUERIES positions of one sequence: the window on
    window_tc_kernel, the routing and the leaves on zha_attend_kernel, which
    merges the window's partials (a bounded sample of the workload's full
    prefill).  ALU roofline with flops =
    2 d (summary keys scored + exact tokens) per query head, the counts taken
    from a traced prefill of 256 of the queries."""
    L = w.length
    nq = min(ZHA_PREFILL_QUERIES, L)
    q0 = L - nq
    g = R.Geometry(head_dim=w.head_dim, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                   leaf_block=w.leaf_block, branching=w.branching, k=w.k, window=w.window,
                   batch=1, capacity=cap,
                   dtype=R.DTYPE_BF16 if w.dtype == torch.bfloat16 else R.DTYPE_F32,
                   rope_enabled=1, rope_base=w.rope_base, mode=R.MODE_ZHA, top_p=ZHA_TOP_P)
    K0, V0 = Kc[:1], Vc[:1]
    tree = torch.zeros(R.recsa_tree_bytes(g), dtype=torch.uint8, device="cuda")
    R.recsa_build(g, K0, V0, [L], r, 0, tree)
    Q = make_prefill_queries(w, Kc, q0, L)
    O = torch.empty_like(Q)
    ws = torch.empty(R.recsa_prefill_workspace_bytes(g, nq), dtype=torch.uint8, device="cuda")
    R.recsa_prefill(g, Q, K0, V0, tree, q0, nq, O, workspace=ws)      # warm-up
    torch.cuda.synchronize()
    flush()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    R.recsa_prefill(g, Q, K0, V0, tree, q0, nq, O, workspace=ws)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = elapsed(e0, e1)
    ns = min(256, nq)
    trace = torch.zeros((1, ns, w.n_q_heads, R.recsa_trace_ints(g)), dtype=torch.int32,
                        device="cuda")
    R.recsa_prefill(g, Q[:, nq - ns:].contiguous(), K0, V0, tree, L - ns, ns,
                    O[:, nq - ns:].contiguous(), trace)
    tr = trace.cpu().numpy()
    per_head = float((tr[..., 2].astype(np.float64) + tr[..., 3]).mean())   # keys + exact
    flops = 2.0 * w.head_dim * per_head * nq * w.n_q_heads
    del Q, O, tree, trace, ws
    torch.cuda.empty_cache()
    return {"value": nq / (ms / 1e3), "unit": "tokens/s", "ms": ms, "queries": nq,
            "q_start": q0, "top_p": ZHA_TOP_P, "kernel": "window_tc_kernel + zha_attend_kernel",
            "sample": f"the last {nq} of {L} positions of one sequence",
            "roofline": {"bound": "alu", "achieved": flops / (ms / 1e3) / 1e12,
                         "peak": ALU_PEAK_TFLOPS, "unit": "TFLOP/s",
                         "frac": flops / (ms / 1e3) / 1e12 / ALU_PEAK_TFLOPS, "flops": flops,
                         "traffic": None}}


def run_dense(args, w, Kc, Vc, Qs, cap, flush, stream, prefill):
    """Dense attention on the same GPU with torch SDPA (library kernel)."""
    from torch.nn.attention import SDPBackend, sdpa_kernel
    L = w.length
    res = {"impl": "torch.nn.functional.scaled_dot_product_attention (flash/cuDNN/efficient)"}
    backends = [SDPBackend.FLASH_ATTENTION, SDPBackend.CUDNN_ATTENTION,
                SDPBackend.EFFICIENT_ATTENTION]
    try:
        Kd, Vd = Kc[:, :, :L], Vc[:, :, :L]
        q = Qs[0].permute(0, 2, 1, 3)               # [batch, Hq, 1, d]
        with sdpa_kernel(backends):
            for _ in range(3):
                torch.nn.functional.scaled_dot_product_attention(q, Kd, Vd, enable_gqa=True)
            ts = []
            for _ in range(10):
                flush()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                torch.nn.functional.scaled_dot_product_attention(q, Kd, Vd, enable_gqa=True)
                e1.record(stream)
                torch.cuda.synchronize()
                ts.append(elapsed(e0, e1))
        ms = statistics.median(ts)
        res["decode_ms"] = ms
        res["decode_queries_per_s"] = w.batch / (ms / 1e3)
        kv = 2 * Kd.numel() * Kd.element_size()
        hbm_gbs, _, peak_kind = peaks()
        res["decode_achieved_gbs"] = kv / (ms / 1e3) / 1e9
        res["decode_hbm_frac"] = res["decode_achieved_gbs"] / hbm_gbs
        res["decode_note"] = (f"reads all of K and V ({kv / 1e9:.2f} GB) once per step; "
                              f"fraction of {peak_kind} HBM bandwidth")
    except Exception as e:  # library kernel unavailable for this shape
        res["decode_error"] = str(e).splitlines()[0][:200]
    if prefill is not None and not args.no_dense_prefill and prefill.get("q_start", 0) == 0:
        try:
            Q = make_prefill_queries(w, Kc, 0, L).permute(0, 2, 1, 3)
            Kd, Vd = Kc[:1, :, :L], Vc[:1, :, :L]
            with sdpa_kernel(backends):
                torch.nn.functional.scaled_dot_product_attention(Q, Kd, Vd, is_causal=True,
                                                                 enable_gqa=True)
                flush()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                torch.nn.functional.scaled_dot_product_attention(Q, Kd, Vd, is_causal=True,
                                                                 enable_gqa=True)
                e1.record(stream)
                torch.cuda.synchronize()
            ms = elapsed(e0, e1)
            res["prefill_ms"] = ms
            res["prefill_tokens_per_s"] = L / (ms / 1e3)
            del Q
        except Exception as e:
            res["prefill_error"] = str(e).splitlines()[0][:200]
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------------------
# CPU oracle: cpu_baseline leg and the reference arm
# ---------------------------------------------------------------------------

class OracleDecode:
    """The float64 oracle on one KV head (G = 4 query heads) of the workload."""

    def __init__(self, workload=WORKLOAD, seed=0):
        import oracle
        self.oracle = oracle
        w = synth.WORKLOADS[workload]
        G = w.n_q_heads // w.n_kv_heads
        self.G = G
        self.w1 = synth.Workload(**{**w.__dict__, "n_q_heads": G, "n_kv_heads": 1, "batch": 1})
        L = w.length
        self.L = L
        n = 64
        K, V, r = synth.make_kv(self.w1, L + n, seed=seed, device="cpu", batch=1)
        self.K = K[0, 0].float().numpy()
        self.V = V[0, 0].float().numpy()
        pos = (L + torch.arange(n, dtype=torch.int64))[None]
        Q, _, _ = synth.make_queries(self.w1, K, pos, seed=1)
        self.Q = Q[0].float().numpy()
        self.geo = oracle.Geometry(w.head_dim, G, 1, w.leaf_block, w.branching, w.k, w.window,
                                   rope=True, rope_base=w.rope_base)
        self.tree = oracle.LazyTree(self.K, self.V, r.double().numpy(), w.leaf_block,
                                    w.branching)
        self.multi = oracle.LazyMultiTree(self.K, self.V,
                                          reference_queries(r, ZHA_N_REF).double().numpy(),
                                          w.leaf_block, w.branching)
        self.i = 0
        self.heads_per_query = w.n_q_heads
        # untimed: pool the nodes the first query visits (the oracle's tree build)
        self.query_heads(1)

    def query_heads(self, n_heads, variant=None):
        """Run n_heads (query, head) pairs (whole groups of G for "group"):
        RecSA, or the "zha" routing variant, or "group" shared selection."""
        done = 0
        while done < n_heads:
            i = self.i % self.Q.shape[0]
            t = self.L + i - 1
            h = done % self.G
            if variant == "group":
                self.oracle.group_traverse_and_attend(self.Q[i], t, self.K, self.V, self.tree,
                                                      self.geo)
                done += self.G
                self.i += 1
                continue
            if variant is None:
                self.oracle.traverse_and_attend(self.Q[i, h], t, self.K, self.V, self.tree,
                                                self.geo)
            else:
                src = self.multi if variant == "zha_multiref" else self.tree
                self.oracle.zha_route_and_attend(self.Q[i, h], t, self.K, self.V, src,
                                                 self.geo, ZHA_TOP_P)
            done += 1
            if h == self.G - 1:
                self.i += 1
        return done


def _single_thread():
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(1)
    except Exception:
        return None


# The oracle runs on every host core: one worker process per core, each a
# single-threaded numpy process over its own queries.  The pool is forked
# from the parent before CUDA is initialised (a process forked after CUDA
# initialisation cannot use it safely; the workers use only numpy), and the
# workers share the parent's oracle inputs copy-on-write.
_ORACLE = None
_LIMIT = None


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def _worker_init():
    global _LIMIT
    _LIMIT = _single_thread()


def _worker_time(arg):
    """One worker: `seconds` of (query, head) pairs of `variant`, starting at
    its own query; returns (query-heads, seconds)."""
    variant, seconds, idx = arg
    o = _ORACLE
    o.i = idx
    o.query_heads(o.G, variant)     # untimed: pool the nodes this worker visits first
    t0 = time.perf_counter()
    heads = 0
    while time.perf_counter() - t0 < seconds:
        heads += o.query_heads(o.G, variant)
    return heads, time.perf_counter() - t0


def _worker_steps(arg):
    """One worker's share of `n` reference-arm steps (G query heads each)."""
    n, idx = arg
    o = _ORACLE
    o.i = idx
    heads = 0
    for _ in range(n):
        heads += o.query_heads(o.G)
    return heads


class CpuPool:
    """The oracle's inputs and a fork pool of one worker per host core."""

    def __init__(self, workload):
        import multiprocessing
        global _ORACLE
        _ORACLE = OracleDecode(workload)
        self.oracle = _ORACLE
        self.cores = host_cores()
        self.pool = multiprocessing.get_context("fork").Pool(self.cores, initializer=_worker_init)

    def close(self):
        self.pool.terminate()
        self.pool.join()


def cpu_baseline(cpu: CpuPool, seconds=15.0, variant=None):
    o = cpu.oracle
    t0 = time.perf_counter()
    res = cpu.pool.map_async(_worker_time, [(variant, seconds, 5 * i)
                                            for i in range(cpu.cores)],
                             chunksize=1).get(timeout=seconds + 300)
    wall = time.perf_counter() - t0
    heads = sum(h for h, _ in res)
    dt = max(d for _, d in res)
    what = {None: "decode", "zha": f"ZHA decode (top-p {ZHA_TOP_P})",
            "zha_multiref": f"ZHA decode (top-p {ZHA_TOP_P}, {ZHA_N_REF} reference queries)",
            "group": "group-selection decode"}[variant]
    return {"value": heads / o.heads_per_query / dt, "unit": "queries/s", "cores": cpu.cores,
            "kind": "oracle",
            "sample": f"{heads} query-heads ({what} at t=L, one KV head's tree, G={o.G}) on "
                      f"{cpu.cores} worker processes (one per host core, single-threaded "
                      f"numpy) for {dt:.1f} s each ({wall:.1f} s wall); queries/s = "
                      f"query-heads/{o.heads_per_query}/s; each worker's first query (its "
                      "tree pooling) untimed"}


def run_reference(args, rank, world, cpu):
    if rank != 0:
        return None
    o = cpu.oracle
    n = cpu.cores
    cpu.pool.map_async(_worker_steps, [(max(args.warmup, 1), 5 * i) for i in range(n)],
                       chunksize=1).get(timeout=600)
    t0 = time.perf_counter()
    heads = 0
    for step in range(args.steps):
        heads += sum(cpu.pool.map_async(_worker_steps, [(1, 5 * i + args.warmup + step)
                                                        for i in range(n)],
                                        chunksize=1).get(timeout=300))
    dt = time.perf_counter() - t0
    value = heads / o.heads_per_query / dt
    return {"impl": "reference", "metric": metric_for(args.workload, o.L), "value": value,
            "unit": "queries/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic, seeded",
            "config": {"workload": args.workload, "L": o.L,
                       "step": f"{n} x {o.G} query heads of decode queries (one KV head's "
                               f"tree), one worker process per host core",
                       "parallelism": "rank 0 only"},
            "cpu_baseline": {"value": value, "unit": "queries/s", "cores": n, "kind": "oracle",
                             "sample": f"{args.steps} steps x {n} workers x {o.G} query heads; "
                                       f"queries/s = query-heads/{o.heads_per_query}/s"},
            "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="recsa", choices=["recsa", "reference"])
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(synth.WORKLOADS),
                    help="workload shape (the default is the headline 524K layer)")
    ap.add_argument("--prefill-reps", type=int, default=1)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-window-ws", action="store_true",
                    help="prefill without a workspace (window attended by the tree kernel)")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-dense-prefill", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-zha", action="store_true",
                    help="skip the ZHA routing-variant decode leg")
    ap.add_argument("--no-group", action="store_true",
                    help="skip the per-KV-group shared-selection decode leg")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--only-decode", action="store_true",
                    help="decode steps only (no prefill, dense, e2e or CPU legs); for profiling")
    ap.add_argument("--length", type=int, default=0,
                    help="override the context length (smaller cases for ncu captures)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.only_decode:
        args.no_prefill = args.no_dense = args.no_cpu = args.no_zha = args.no_group = True
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        cpu = CpuPool(args.workload) if rank == 0 else None
        try:
            out = run_reference(args, rank, world, cpu)
        finally:
            if cpu is not None:
                cpu.close()
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    # the oracle's worker pool is forked before CUDA is initialised
    cpu = CpuPool(args.workload) if rank == 0 and world == 1 and not args.no_cpu else None
    try:
        _run_gpu(args, rank, world, local, cpu)
    finally:
        if cpu is not None:
            cpu.close()


def _run_gpu(args, rank, world, local, cpu):
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    R.lib()
    out = run_recsa(args, rank, world, local, cpu)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
