#!/usr/bin/env python
"""Throughput of one block-diffusion denoising step on B200.

A step is the whole per-step hot path over one batch: bd_block_attn (the
current 32-token block over its block-level KV cache) followed by
bd_confidence_select (token shift, LM head, softmax statistics, unmask).
Metric: masked positions scored per second (every masked position of every
sequence gets its logits scored once per step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--tau T] [--sub-block S]

Under torchrun every rank runs an independent replica of the workload (the
batches are independent; no collective on the data path): weak scaling.
Inputs are synthetic and seeded (no dataset, no trained weights).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from decoding_bd_block_b200 import workloads as W  # noqa: E402

DEFAULT_WORKLOAD = W.QWEN7B_RAGGED.name
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
SELECT_KERNEL_SOURCES = ("decoding_bd_block_b200/csrc/select_tc.cu", "decoding_bd_block_b200/csrc/tc_common.cuh")


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(W.STEP_CONFIGS) + [W.MASK_ATTN.name, W.MASKED_CE.name])
    ap.add_argument("--tau", type=float, default=None)
    ap.add_argument("--sub-block", type=int, default=None)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--shared-clean", action="store_true",
                    help="mask attention: compute each sample's clean rows once for all its views "
                         "(bd_block_mask_attn_views)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--active-only", action="store_true",
                    help="score only the unmask rule's candidates (bd_confidence_select_active)")
    ap.add_argument("--eager", action="store_true",
                    help="launch every call from the host instead of replaying CUDA graphs")
    return ap.parse_args(argv)


# --------------------------------------------------------------------------
# distributed plumbing (one process per GPU; torchrun sets the env)
# --------------------------------------------------------------------------
class Dist:
    def __init__(self, backend: str):
        import torch.distributed as dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.dist = dist if self.world > 1 else None
        if self.dist is not None:
            import datetime
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=180))

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max(self, x: float, device=None) -> float:
        if self.dist is None:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def sum(self, x: float, device=None) -> float:
        if self.dist is None:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.SUM)
        return float(t.item())

    def close(self):
        if self.dist is not None:
            self.dist.destroy_process_group()


def active_bits(bits: int, sub_block: int) -> int:
    """Bit mask of the masked positions of the lowest sub-block that has one."""
    if not bits:
        return 0
    k0 = ((bits & -bits).bit_length() - 1) // sub_block * sub_block
    return bits & (((1 << sub_block) - 1) << k0)


def replica_throughput(dist: Dist, units: float, ms_rank: float, device=None):
    """Whole-job throughput of independent replicas: every rank processed
    `units` in `ms_rank` ms; the job's time is the slowest rank's.  Returns
    (ms, units summed over ranks per second)."""
    ms = dist.max(ms_rank, device)
    return ms, dist.sum(units, device) / (ms / 1e3)


# --------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.lines, self.proc = [], None
        if gpu_id is None:
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-i", gpu_id, "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()
        t0 = time.time()
        while not self.lines and time.time() - t0 < 5:
            time.sleep(0.02)

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append((time.time(), ln.strip()))

    def mark(self):
        return time.time()

    def stop(self, t0: float, t1: float):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = [ln.split(", ") for t, ln in self.lines if t0 - 0.15 <= t <= t1 + 0.25]
        rows = [r for r in rows if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def gpu_uuid(dev):
    try:
        import torch
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return None


class L2Flush:
    """The L2 flush between timed steps: write a buffer larger than L2, which
    evicts every line of the previous step, then read a second one, so that L2
    is left holding clean lines of unrelated data rather than dirty ones that
    the next step would write back to HBM while it runs (a step in a serving
    loop does not start behind a 256 MB memset)."""
    DESCRIPTION = (f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MB write, then a "
                   f"{L2_FLUSH_BYTES >> 20} MB read so that no dirty line is left)")

    def __init__(self, dev):
        import torch
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.sum()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


# Nominal per-GPU figures, for a second fraction beside the measured one:
# HBM3e bandwidth (HGX B200) and dense bf16 tensor throughput.
NOMINAL_PEAKS = {"GB/s": 7700.0, "TFLOP/s": 2250.0}


def with_nominal(roofline: dict) -> dict:
    """The roofline object with the fraction of the nominal peak of its unit
    (the part's data-sheet figure) added beside the measured one."""
    nom = NOMINAL_PEAKS.get(roofline.get("unit"))
    if nom is not None and roofline.get("achieved") is not None:
        roofline = dict(roofline, nominal_peak=nom, frac_of_nominal=roofline["achieved"] / nom)
    return roofline


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel's
    source is unchanged since it was captured (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(kernel)
    if not rec:
        return None
    h = hashlib.sha256()
    for src in rec.get("sources", []):
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != rec.get("source_sha256"):
        return None
    return rec.get("dram_bytes_per_launch")


def source_sha(paths):
    h = hashlib.sha256()
    for src in paths:
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


# --------------------------------------------------------------------------
# the oracle as a CPU baseline (test infrastructure, timed as it stands)
# --------------------------------------------------------------------------
def oracle_caches(cfg, a_in, seqs=None):
    """The oracle's cache (prefix K rotated at commit) of the given sequences:
    built once, outside any timed region, as the GPU arm's cache is."""
    import oracle as O
    seqs = range(cfg.batch) if seqs is None else seqs
    out = {}
    for s in seqs:
        c = O.OracleCache(1, cfg.n_heads_kv, cfg.head_dim, cfg.rope_theta)
        if a_in["prefix_len"][s]:
            c.commit(0, O.widen(a_in["prefix_k"][s], cfg.dtype),
                     O.widen(a_in["prefix_v"][s], cfg.dtype))
        out[s] = c
    return out


def oracle_step_sample(cfg, a_in, s_in, frac: float, tau: float, S: int, caches=None):
    """One oracle step on a bounded sample: block attention of the sequences
    in ``caches`` (all of them when None), and the LM-head statistics /
    selection over the first `frac` of the vocabulary.  Returns
    (attention seconds, LM-head seconds, vocabulary fraction actually used)."""
    import oracle as O
    t0 = time.perf_counter()
    if a_in is not None:
        caches = oracle_caches(cfg, a_in) if caches is None else caches
        for s, c in caches.items():
            O.block_attn_seq(c.k[0], c.v[0], O.widen(a_in["q"][s], cfg.dtype),
                             O.widen(a_in["k_blk"][s], cfg.dtype),
                             O.widen(a_in["v_blk"][s], cfg.dtype), cfg.rope_theta)
    t1 = time.perf_counter()
    if s_in is None:
        return t1 - t0, 0.0, 1.0
    Vs = max(1, int(round(cfg.vocab * frac)))
    O.confidence_select(s_in["h"], s_in["h_prev"], s_in["W"][:Vs], s_in["masked_bits"], tau, S,
                        s_in["tokens"], cfg.dtype)
    return t1 - t0, time.perf_counter() - t1, Vs / cfg.vocab


def full_step_seconds(parts):
    """Whole-step seconds estimated from sampled steps [(attention s, LM-head s,
    vocabulary fraction)]: the attention as timed, the LM-head time scaled to
    the full vocabulary (it is linear in the vocabulary rows)."""
    return sum(ta + tl / f for ta, tl, f in parts) / len(parts)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(cfg, a_in, s_in, tau, S, budget_s, got=None):
    """Time the oracle on the host on a bounded sample of the workload, and,
    when that sample is the whole step, compare the timed step's GPU outputs
    (``got``) with it.  Returns (cpu_baseline dict, parity dict or None).

    The sample is one whole oracle step (every sequence's block attention,
    the LM head over the full vocabulary, the selection) when a 2% probe
    predicts it fits in 3 x budget_s; otherwise a vocabulary fraction of the
    step sized to about budget_s, and no parity block."""
    import platform
    caches = oracle_caches(cfg, a_in) if a_in is not None else None
    probe = max(sum(oracle_step_sample(cfg, a_in, s_in, 0.02, tau, S, caches)[:2]), 1e-3)  # 2% of the vocab
    cpu = platform.processor() or platform.machine()
    n_pos = s_in["n_scored"] if s_in else 0
    if s_in is None or probe * 50 <= 3 * budget_s:  # (attention only: the probe was a whole step)
        t0 = time.perf_counter()
        ref = oracle_full_step(cfg, a_in, s_in, tau, S, caches)
        t = time.perf_counter() - t0
        base = {"value": (n_pos if s_in else cfg.batch * W.BLOCK * cfg.n_heads_q) / t,
                "unit": "masked positions scored/s" if s_in else "query rows/s",
                "cores": blas_threads(), "kind": "oracle",
                "sample": (f"one whole oracle step of workload {cfg.name}: block attention of all "
                           f"{cfg.batch} sequences"
                           + (f" + LM-head statistics over the full vocabulary and selection "
                              f"({n_pos} masked positions)" if s_in else "")
                           + f"; fp64 numpy on {cpu}")}
        return base, (parity_block(cfg, ref, got, tau, S) if got is not None else None)
    frac = float(min(1.0, max(0.02, 0.02 * budget_s / probe / 2)))
    parts, t_total = [], 0.0
    while t_total < budget_s * 0.5 or not parts:
        parts.append(oracle_step_sample(cfg, a_in, s_in, frac, tau, S, caches))
        t_total += sum(parts[-1][:2])
    return {"value": n_pos / full_step_seconds(parts), "unit": "masked positions scored/s",
            "cores": blas_threads(), "kind": "oracle",
            "sample": (f"{len(parts)} oracle step(s) of workload {cfg.name}: full block attention + "
                       f"LM-head statistics and selection over {parts[0][2]:.1%} of the vocabulary, "
                       f"the LM-head time scaled to the full vocabulary ({n_pos} masked positions "
                       f"per step); fp64 numpy on {cpu}")}, None


def oracle_full_step(cfg, a_in, s_in, tau, S, caches):
    """The oracle on the whole step: {s: block attention [32, Hq, d]} and the
    selection result of the full vocabulary (None without a select part)."""
    import oracle as O
    attn = {}
    if a_in is not None:
        for s, c in caches.items():
            attn[s] = O.block_attn_seq(c.k[0], c.v[0], O.widen(a_in["q"][s], cfg.dtype),
                                       O.widen(a_in["k_blk"][s], cfg.dtype),
                                       O.widen(a_in["v_blk"][s], cfg.dtype), cfg.rope_theta)
    sel = None
    if s_in is not None:
        sel = O.confidence_select(s_in["h"], s_in["h_prev"], s_in["W"], s_in["masked_bits"], tau, S,
                                  s_in["tokens"], cfg.dtype)
    return attn, sel


ATTN_TOL = {"f32": 1e-5, "bf16": 2e-2}  # max-abs bound of the attention outputs per storage type
PMAX_TOL = 1e-4                          # p_max agreement the threshold band needs


def parity_block(cfg, ref, got, tau, S):
    """The timed step's GPU outputs against the oracle's whole step.

    Decisions (unmask words) and tokens must be identical outside the
    positions the oracle flags as ambiguous; the flagged ones are counted.
    Attention: max-abs error against the oracle, with the stated bound."""
    attn_ref, sel = ref
    out = {"tau": tau, "sub_block": S}
    ok = True
    if attn_ref:
        err = max(float(np.abs(got["out"][s] - attn_ref[s]).max()) for s in attn_ref)
        out.update(attn_max_abs_err=err, attn_tol=ATTN_TOL[cfg.dtype],
                   attn_sequences=len(attn_ref))
        ok &= err <= ATTN_TOL[cfg.dtype]
    if sel is not None:
        bits = np.asarray(got["masked"], np.uint32)
        pos = dec = tok = 0
        bad_dec = bad_tok = bad_pmax = 0
        pmax_err = 0.0
        for s in range(len(bits)):
            b = int(bits[s])
            for i in range(W.BLOCK):
                if not (b >> i) & 1:
                    continue
                pos += 1
                pmax_err = max(pmax_err, abs(float(got["pmax"][s, i]) - float(sel["pmax"][s, i])))
                bad_pmax += abs(float(got["pmax"][s, i]) - float(sel["pmax"][s, i])) > PMAX_TOL
                if not sel["token_ambiguous"][s, i]:
                    bad_tok += int(got["argmax"][s, i]) != int(sel["argmax"][s, i])
            if sel["decision_ambiguous"][s]:
                continue
            dec += 1
            bad_dec += int(got["unmask"][s]) != int(sel["unmask"][s])
            for i in range(W.BLOCK):
                if not sel["token_ambiguous"][s, i]:
                    bad_tok += int(got["tokens"][s, i]) != int(sel["tokens"][s, i])
        out.update(sequences_checked=dec, positions_checked=pos,
                   decision_ambiguous=int(sel["decision_ambiguous"].sum()),
                   token_ambiguous=int(sel["token_ambiguous"].sum()),
                   decision_mismatches=bad_dec, token_mismatches=bad_tok,
                   pmax_max_abs_err=pmax_err, pmax_outside_tol=bad_pmax)
        ok &= bad_dec == 0 and bad_tok == 0 and bad_pmax == 0
    out["pass"] = bool(ok)
    return out


# --------------------------------------------------------------------------
# arms
# --------------------------------------------------------------------------
def reference_line(args, cfg_name, metric, unit, value, t, config, sample):
    """The JSON line of the reference arm (the oracle, timed on the host)."""
    return {
        "metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference", "config": dict(workload=cfg_name, **config),
        "cpu_baseline": {"value": value, "unit": unit, "kind": "oracle", "cores": blas_threads(),
                         "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def reference_budget(args):
    """Seconds of oracle work per step, so that the whole run ends in a few minutes."""
    return 150.0 / max(1, args.steps + args.warmup)


def run_reference(args, cfg, tau, S):
    a_in = W.make_attn_inputs(cfg)
    s_in = W.make_select_inputs(cfg) if cfg.hidden else None
    if s_in is None:  # attention only: a bounded number of whole sequences per step
        caches = oracle_caches(cfg, a_in, [0])
        t0 = time.perf_counter()
        oracle_step_sample(cfg, a_in, None, 0.0, tau, S, caches)
        probe = max(time.perf_counter() - t0, 1e-3)
        n_seq = int(min(cfg.batch, max(1, reference_budget(args) // probe)))
        caches = oracle_caches(cfg, a_in, range(n_seq))
        for _ in range(args.warmup):
            oracle_step_sample(cfg, a_in, None, 0.0, tau, S, caches)
        t = 0.0
        for _ in range(args.steps):
            t0 = time.perf_counter()
            oracle_step_sample(cfg, a_in, None, 0.0, tau, S, caches)
            t += time.perf_counter() - t0
        rows = n_seq * W.BLOCK * cfg.n_heads_q * args.steps
        line = reference_line(
            args, cfg.name, "query rows attended/s per denoise step (block attention only)",
            "query rows/s", rows / t, t, {"batch": cfg.batch, "sequences_per_step": n_seq},
            f"each step: the block attention of {n_seq} of the {cfg.batch} sequences of workload "
            f"{cfg.name} (the cache rotated once, before timing)")
        print(json.dumps(line), flush=True)
        return
    s_in["n_scored"] = int(sum(bin(int(b)).count("1") for b in s_in["masked_bits"]))
    caches = oracle_caches(cfg, a_in)
    probe = max(sum(oracle_step_sample(cfg, a_in, s_in, 0.02, tau, S, caches)[:2]), 1e-3)
    frac = float(min(1.0, max(0.002, 0.02 * reference_budget(args) / probe)))
    for _ in range(args.warmup):
        oracle_step_sample(cfg, a_in, s_in, frac, tau, S, caches)
    parts = [oracle_step_sample(cfg, a_in, s_in, frac, tau, S, caches) for _ in range(args.steps)]
    t_step = full_step_seconds(parts)
    line = reference_line(
        args, cfg.name, "masked positions scored/s per denoise step", "masked positions scored/s",
        s_in["n_scored"] / t_step, t_step * args.steps,
        {"batch": cfg.batch, "tau": tau, "sub_block": S, "vocab_fraction_per_step": parts[0][2]},
        f"each step: full block attention + LM-head statistics over {parts[0][2]:.2%} of the "
        f"vocabulary of workload {cfg.name}, the LM-head time scaled to the full vocabulary")
    print(json.dumps(line), flush=True)


def run_reference_mask_attn(args, cfg):
    """The oracle's 2L x 2L masked attention on a bounded sample of query rows."""
    import oracle as O
    t = W.make_mask_attn_inputs(cfg)
    q, k, v = (O.widen(t[x], cfg.dtype) for x in ("q", "k", "v"))
    rng = np.random.default_rng(0)
    per = probe_cost(lambda n: O.mask_attn(q, k, v, cfg.L, cfg.block, rows=np.arange(n)),
                     16)  # per query row over all views
    n_rows = int(min(2 * cfg.L, max(8, 0.5 * reference_budget(args) / per)))  # half: margin
    rows = np.sort(rng.choice(2 * cfg.L, n_rows, replace=False))
    for _ in range(args.warmup):
        O.mask_attn(q, k, v, cfg.L, cfg.block, rows=rows)
    tt = 0.0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        O.mask_attn(q, k, v, cfg.L, cfg.block, rows=rows)
        tt += time.perf_counter() - t0
    units = n_rows * cfg.n_seqs * cfg.n_heads_q * args.steps
    line = reference_line(
        args, cfg.name, "query rows attended/s (2L x 2L complementary-mask attention)",
        "query rows/s", units / tt, tt,
        {"views": cfg.n_seqs, "L": cfg.L, "block": cfg.block, "rows_per_view_per_step": n_rows},
        f"each step: {n_rows} of the {2 * cfg.L} query rows (all heads) of each of the "
        f"{cfg.n_seqs} views of workload {cfg.name}")
    print(json.dumps(line), flush=True)


def run_reference_ce(args, cfg):
    """The oracle's masked cross-entropy on a bounded sample of scored positions."""
    import oracle as O
    d = W.make_ce_inputs(cfg)
    pos = O.ce_positions(d["masked_bits"])
    per = probe_cost(lambda n: O.masked_ce(d["h"], d["W"], d["targets"], d["masked_bits"],
                                           cfg.dtype, positions=pos[:n]), 256)
    # whole chunks of 256 positions (the oracle's unit of work)
    n_pos = int(min(len(pos), max(256, 0.5 * reference_budget(args) / per // 256 * 256)))
    rng = np.random.default_rng(0)
    sample = [pos[i] for i in sorted(rng.choice(len(pos), n_pos, replace=False))]
    for _ in range(args.warmup):
        O.masked_ce(d["h"], d["W"], d["targets"], d["masked_bits"], cfg.dtype, positions=sample)
    tt = 0.0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        O.masked_ce(d["h"], d["W"], d["targets"], d["masked_bits"], cfg.dtype, positions=sample)
        tt += time.perf_counter() - t0
    line = reference_line(
        args, cfg.name, "masked positions' cross-entropy computed/s (training batch)",
        "scored positions/s", n_pos * args.steps / tt, tt,
        {"sequences": cfg.n_seqs, "L": cfg.L, "hidden": cfg.hidden, "vocab": cfg.vocab,
         "positions_per_step": n_pos},
        f"each step: the loss at {n_pos} of the {len(pos)} scored positions of workload {cfg.name}")
    print(json.dumps(line), flush=True)


def probe_cost(fn, n: int):
    """Seconds per unit of fn(n), fixed costs included (so a sample sized by it
    stays within its budget): one untimed call to warm up, one timed."""
    fn(n)
    t0 = time.perf_counter()
    fn(n)
    return max((time.perf_counter() - t0) / n, 1e-6)


def reference_rank0():
    """Under torchrun the reference arm runs on rank 0 only."""
    return int(os.environ.get("RANK", "0")) == 0


def run_ours(args, cfg, tau, S, dist: Dist):
    import torch

    from decoding_bd_block_b200 import bd
    from decoding_bd_block_b200.step import DecodeStep

    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    a_in = W.make_attn_inputs(cfg)
    s_in = W.make_select_inputs(cfg) if cfg.hidden else None
    step = DecodeStep(cfg, a_in, s_in, device=dev)
    if args.active_only and step.sel:
        # the kernels score only the candidates: count those as the units
        step.active_only = True
        step.n_scored = sum(bin(active_bits(int(b), S)).count("1") for b in step.masked_host)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        flush()
        step.run(tau, S)
    torch.cuda.synchronize(dev)
    # Kernels one step launches (counted on an eager step), then the step's
    # calls recorded once into CUDA graphs and replayed, as a serving loop
    # would: the timed region holds no host-side launch cost.
    n0 = bd.bd_kernel_launches()
    if step.attn:
        step.run_attn()
    n1 = bd.bd_kernel_launches()
    if step.sel:
        step.run_select(tau, S)
    per_step = bd.bd_kernel_launches() - n0
    sel_launches = per_step - (n1 - n0)
    graphs = None if args.eager else step.capture(tau, S, parts=("step", "attn", "select"))
    for _ in range(2):
        flush()
        if graphs:
            graphs["step"].replay()
        else:
            step.run(tau, S)
    torch.cuda.synchronize(dev)

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    launches0 = bd.bd_kernel_launches()
    dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    for i in range(K):
        flush()
        ev[i][0].record(stream)
        if graphs:
            graphs["step"].replay()
        else:
            step.run(tau, S)
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    t_wall1 = time.time()
    # the timed step's outputs, for the parity block (compared after timing)
    got = {"out": step.out.float().cpu().numpy() if step.attn else None}
    if step.sel:
        got.update(tokens=step.tokens.cpu().numpy(), unmask=step.unmask.cpu().numpy().view(np.uint32),
                   pmax=step.pmax.cpu().numpy(), argmax=step.argmax.cpu().numpy(),
                   masked=step.masked_host)
    # Per-call breakdown, outside the timed region: each call on its own
    # (one graph per call), L2 flushed before each step as above.
    n_bd = max(10, K // 4)
    evb = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_bd)]
    for i in range(n_bd):
        flush()
        evb[i][0].record(stream)
        if step.attn:
            graphs["attn"].replay() if graphs else step.run_attn()
        evb[i][1].record(stream)
        if step.sel:
            graphs["select"].replay() if graphs else step.run_select(tau, S)
        evb[i][2].record(stream)
    torch.cuda.synchronize(dev)
    launches = per_step * K if graphs else bd.bd_kernel_launches() - launches0
    clocks = sampler.stop(t_wall0, t_wall1)

    t_attn = [evb[i][0].elapsed_time(evb[i][1]) for i in range(n_bd)]
    t_sel = [evb[i][1].elapsed_time(evb[i][2]) for i in range(n_bd)]
    t_step = [ev[i][0].elapsed_time(ev[i][1]) for i in range(K)]
    ms_rank = float(np.mean(t_step))
    n_scored = step.n_scored if step.sel else 0
    unit_count = n_scored if step.sel else cfg.batch * W.BLOCK * cfg.n_heads_q
    ms, value = replica_throughput(dist, float(unit_count), ms_rank, dev)

    peaks, peak_kind = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    if step.sel:
        w_bytes = cfg.vocab * cfg.hidden * (2 if cfg.dtype == "bf16" else 4)
        rows_bytes = n_scored * cfg.hidden * (2 if cfg.dtype == "bf16" else 4)
        alg = w_bytes + rows_bytes
        t_dom = float(np.mean(t_sel)) / 1e3
        # one launch: the single-kernel select; else gather + LM head + merge
        dom = "select_fused" if sel_launches == 1 else "lmhead"
        traffic = recorded_traffic(dom)
        roofline = {"kernel": f"bd_confidence_select ({dom} kernel: vocab stream; whole call timed)",
                    "bound": "hbm", "achieved": alg / t_dom / 1e9, "peak": hbm, "unit": "GB/s",
                    "frac": alg / t_dom / 1e9 / hbm, "traffic": traffic,
                    "algorithmic_bytes_per_launch": alg, "peak_source": peak_kind}
    else:
        es = 2 if cfg.dtype == "bf16" else 4
        keys = float(np.sum(a_in["prefix_len"] + W.BLOCK))
        alg = keys * cfg.n_heads_kv * cfg.head_dim * 2 * es
        t_dom = float(np.mean(t_attn)) / 1e3
        roofline = {"kernel": "bd_block_attn (K/V stream; whole call timed)", "bound": "hbm",
                    "achieved": alg / t_dom / 1e9, "peak": hbm, "unit": "GB/s",
                    "frac": alg / t_dom / 1e9 / hbm, "traffic": recorded_traffic("attn"),
                    "algorithmic_bytes_per_launch": alg, "peak_source": peak_kind}

    e2e = None
    if not args.no_e2e and step.sel:
        e2e = measure_e2e(step, cfg, tau, S, flush, dev, dist, max(10, K // 4),
                          graphs["step"] if graphs else None)

    metric, unit = "masked positions scored/s per denoise step", "masked positions scored/s"
    if not step.sel:  # attention-only workload: units are (query head, block position) rows
        metric = "query rows attended/s per denoise step (block attention only)"
        unit = "query rows/s"
    elif step.active_only:
        metric = "candidate positions scored/s per denoise step (active sub-block only)"
        unit = "candidate positions scored/s"
    line = {
        "metric": metric,
        "value": value, "unit": unit, "n_gpus": dist.world,
        "steps": K, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
        "config": {"workload": cfg.name, "batch": cfg.batch, "n_heads_q": cfg.n_heads_q,
                   "n_heads_kv": cfg.n_heads_kv, "head_dim": cfg.head_dim,
                   "prefix_tokens": [int(x) for x in a_in["prefix_len"]],
                   "hidden": cfg.hidden, "vocab": cfg.vocab, "tau": tau, "sub_block": S,
                   "masked_positions_per_step": n_scored,
                   "l2": L2Flush.DESCRIPTION,
                   "parallelism": f"replicas x{dist.world} (independent batches)",
                   "launch": "eager" if args.eager else "CUDA graph replay of the C-ABI calls"},
        "breakdown_ms": {"bd_block_attn": float(np.mean(t_attn)),
                         "bd_confidence_select": float(np.mean(t_sel))},
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clocks,
        "timed_region_wall_s": t_wall1 - t_wall0,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        if s_in is not None:
            s_in["n_scored"] = n_scored
        line["cpu_baseline"], line["parity"] = cpu_baseline(
            cfg, a_in, s_in, tau, S, args.cpu_budget_s, None if step.active_only else got)
    if dist.rank == 0:
        line["roofline"] = with_nominal(line["roofline"])
        print(json.dumps(line), flush=True)


def measure_e2e(step, cfg, tau, S, flush, dev, dist, K, graph=None):
    """Same metric through the public API with the step's inputs on pinned host
    memory, as a serving loop runs it: every step's inputs (q, k_blk, v_blk,
    h, h_prev, mask bits, tokens) are copied from pinned host memory by one
    host-to-device copy on a second stream while the previous step computes
    (two device staging buffers); the step then copies its staging buffer
    into the step's arena (device to device), runs (the captured step graph,
    else eager calls) and reads back the tokens and unmask bits (one
    device-to-host copy).  Each step is timed from after the L2 flush that
    precedes it (as in the device-timed loop) to after its read-back, waiting
    for its own upload inside that window: any part of the upload that the
    previous step did not hide is counted."""
    import torch
    host_in = step.arena[:step.in_bytes].cpu().pin_memory()
    host_out = torch.empty(step.arena.numel() - step.out_off, dtype=torch.uint8).pin_memory()
    h2d = int(host_in.numel())
    d2h = int(host_out.numel())  # tokens and unmask bits (256-byte aligned within the arena)
    stream = torch.cuda.current_stream(dev)
    copy_stream = torch.cuda.Stream(dev)
    staging = [torch.empty(step.in_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    uploaded = [torch.cuda.Event() for _ in range(2)]  # host -> staging[b] done
    consumed = [torch.cuda.Event() for _ in range(2)]  # staging[b] -> arena done
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]

    def upload(b):
        with torch.cuda.stream(copy_stream):
            staging[b].copy_(host_in, non_blocking=True)
            uploaded[b].record(copy_stream)

    dist.barrier()
    torch.cuda.synchronize(dev)
    upload(0)
    for i in range(K):
        b = i % 2
        if i + 1 < K:  # the next step's inputs, once staging[1 - b] has been consumed
            if i >= 1:
                copy_stream.wait_event(consumed[1 - b])
            upload(1 - b)
        flush()
        ev[i][0].record(stream)
        stream.wait_event(uploaded[b])
        step.arena[:step.in_bytes].copy_(staging[b], non_blocking=True)
        consumed[b].record(stream)
        if graph is not None:
            graph.replay()
        else:
            step.run(tau, S)
        host_out.copy_(step.arena[step.out_off:], non_blocking=True)
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    ms_step = float(np.mean([e[0].elapsed_time(e[1]) for e in ev]))
    ms, value = replica_throughput(dist, float(step.n_scored), ms_step, dev)
    return {"value": value, "unit": "masked positions scored/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "launch": ("CUDA graph replay" if graph is not None else "eager C-ABI calls")
            + "; each step's host-to-device copy runs on a second stream during the previous step"}


def mask_pairs(L: int, D: int) -> int:
    """Allowed (query, key) pairs of the 2L x 2L training mask, per view and
    head: a noisy query of block b sees its own block's D noisy keys and the
    b D clean keys before it; a clean query of block b sees (b + 1) D clean
    keys.  Summed over the n = L / D blocks: D^2 (n^2 + n)."""
    n = L // D
    return D * D * (n * n + n)


def mask_clean_pairs(L: int, D: int) -> int:
    """The clean queries' share of mask_pairs: (b + 1) D^2 for block b,
    D^2 n (n + 1) / 2 in all.  They see clean keys only, so they are the same
    in every view of a sample."""
    n = L // D
    return D * D * n * (n + 1) // 2


def run_mask_attn(args, cfg, dist: Dist):
    """bd_block_mask_attn on the training-forward workload (2L x 2L mask)."""
    import torch

    from decoding_bd_block_b200 import bd
    from decoding_bd_block_b200.step import to_device

    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    t = W.make_mask_attn_inputs(cfg)
    q, k, v = (to_device(t[x], cfg.dtype, dev) for x in ("q", "k", "v"))
    out = torch.empty_like(q)
    shape = bd.make_shape(cfg.n_heads_q, cfg.n_heads_kv, cfg.head_dim, cfg.dtype)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)
    if args.shared_clean:
        call = lambda: bd.bd_block_mask_attn_views(shape, q, k, v, out, cfg.n_seqs, cfg.views,
                                                   cfg.L, cfg.block)
    else:
        call = lambda: bd.bd_block_mask_attn(shape, q, k, v, out, cfg.n_seqs, cfg.L, cfg.block)
    for _ in range(args.warmup):
        flush()
        call()
    torch.cuda.synchronize(dev)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    launches0 = bd.bd_kernel_launches()
    sampler = ClockSampler(gpu_uuid(dev))
    dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    for i in range(K):
        flush()
        ev[i][0].record(stream)
        call()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    clocks = sampler.stop(t_wall0, time.time())
    launches = bd.bd_kernel_launches() - launches0
    ms, rows_per_s = replica_throughput(dist, float(cfg.n_seqs * 2 * cfg.L * cfg.n_heads_q),
                                        float(np.mean([e[0].elapsed_time(e[1]) for e in ev])), dev)
    pairs = mask_pairs(cfg.L, cfg.block)
    flop = 4.0 * cfg.head_dim * cfg.n_heads_q * pairs * cfg.n_seqs
    if args.shared_clean:  # each sample's clean rows computed once, for all of its views
        flop -= (4.0 * cfg.head_dim * cfg.n_heads_q * mask_clean_pairs(cfg.L, cfg.block)
                 * (cfg.n_seqs - cfg.samples))
    peaks, peak_kind = measured_peaks()
    peak = float(peaks.get("bf16_tflops", 1590.0))
    ach = flop / (ms / 1e3) / 1e12
    line = {
        "metric": "query rows attended/s (2L x 2L complementary-mask attention)",
        "value": rows_per_s, "unit": "query rows/s", "n_gpus": dist.world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
        "config": {"workload": cfg.name, "views": cfg.n_seqs, "L": cfg.L, "block": cfg.block,
                   "n_heads_q": cfg.n_heads_q, "n_heads_kv": cfg.n_heads_kv,
                   "head_dim": cfg.head_dim, "allowed_pairs_per_view_head": pairs,
                   "clean_rows": (f"computed once per sample for its {cfg.views} views"
                                  if args.shared_clean else "computed for every view"),
                   "l2": L2Flush.DESCRIPTION},
        "roofline": {"kernel": "bd_block_mask_attn", "bound": "tensor", "achieved": ach,
                     "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
                     "traffic": recorded_traffic("mask_attn_views" if args.shared_clean
                                                 else "mask_attn"),
                     "algorithmic_flop_per_launch": flop, "peak_source": peak_kind},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if dist.rank == 0:
        line["roofline"] = with_nominal(line["roofline"])
        print(json.dumps(line), flush=True)


def run_masked_ce(args, cfg, dist: Dist):
    """bd_masked_ce on the training batch (16 sequences of 2048 positions)."""
    import torch

    from decoding_bd_block_b200 import bd
    from decoding_bd_block_b200.step import to_device

    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    d = W.make_ce_inputs(cfg)
    N, L = d["targets"].shape
    h = to_device(d["h"], cfg.dtype, dev)
    w = to_device(d["W"], cfg.dtype, dev)
    tg = torch.from_numpy(d["targets"]).to(dev)
    mb = torch.from_numpy(d["masked_bits"].view(np.int32)).to(dev)
    loss = torch.empty((N, L), dtype=torch.float32, device=dev)
    ls = torch.zeros(1, dtype=torch.float32, device=dev)
    ns = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = torch.empty(bd.bd_masked_ce_workspace_size(cfg.dtype, N, L, cfg.hidden, cfg.vocab),
                     dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)
    call = lambda: bd.bd_masked_ce(cfg.dtype, N, L, cfg.hidden, cfg.vocab, h, w, tg, mb, loss, ls,
                                   ns, ws)
    for _ in range(args.warmup):
        flush()
        call()
    torch.cuda.synchronize(dev)
    count = int(ns.item())
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    launches0 = bd.bd_kernel_launches()
    sampler = ClockSampler(gpu_uuid(dev))
    dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    for i in range(K):
        flush()
        ev[i][0].record(stream)
        call()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    clocks = sampler.stop(t_wall0, time.time())
    launches = bd.bd_kernel_launches() - launches0
    ms, value = replica_throughput(dist, float(count),
                                   float(np.mean([e[0].elapsed_time(e[1]) for e in ev])), dev)
    flop = 2.0 * count * cfg.vocab * cfg.hidden
    peaks, peak_kind = measured_peaks()
    peak = float(peaks.get("bf16_tflops", 1590.0))
    peak_sus = peaks.get("bf16_tflops_sustained")
    ach = flop / (ms / 1e3) / 1e12
    line = {
        "metric": "masked positions' cross-entropy computed/s (training batch)",
        "value": value, "unit": "scored positions/s", "n_gpus": dist.world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
        "config": {"workload": cfg.name, "sequences": N, "L": L, "hidden": cfg.hidden,
                   "vocab": cfg.vocab, "scored_positions": count,
                   "mean_loss": float(ls.item()) / max(count, 1),
                   "l2": L2Flush.DESCRIPTION},
        "roofline": {"kernel": "bd_masked_ce (LM head on tcgen05; whole call timed)",
                     "bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                     "frac": ach / peak, "traffic": recorded_traffic("masked_ce"),
                     "algorithmic_flop_per_launch": flop, "peak_source": peak_kind,
                     "frac_of_sustained_peak": (ach / float(peak_sus)) if peak_sus else None},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if dist.rank == 0:
        line["roofline"] = with_nominal(line["roofline"])
        print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.workload == W.MASK_ATTN.name:
        if args.impl == "reference":
            if reference_rank0():
                run_reference_mask_attn(args, W.MASK_ATTN)
            return 0
        dist = Dist("nccl")
        try:
            run_mask_attn(args, W.MASK_ATTN, dist)
        finally:
            dist.close()
        return 0
    if args.workload == W.MASKED_CE.name:
        if args.impl == "reference":
            if reference_rank0():
                run_reference_ce(args, W.MASKED_CE)
            return 0
        dist = Dist("nccl")
        try:
            run_masked_ce(args, W.MASKED_CE, dist)
        finally:
            dist.close()
        return 0
    cfg = W.STEP_CONFIGS[args.workload]
    tau = args.tau if args.tau is not None else cfg.taus[0]
    S = args.sub_block if args.sub_block is not None else cfg.sub_block
    if args.impl == "reference":
        if reference_rank0():
            run_reference(args, cfg, tau, S)
        return 0
    dist = Dist("nccl")
    try:
        run_ours(args, cfg, tau, S, dist)
    finally:
        dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
