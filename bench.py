"""Benchmark: confidence-scheduled speculative verification on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload c0|c1|c2|c3|c4] [--tau T]

One step = one pass of the whole hot path over one batch: the schedule
(prefix survival -> verify lengths) and the verification (softmax statistics,
accept test, correction/bonus draw), through the library's C ABI
(sv_schedule_verify: the schedule runs in the verification's first kernel;
workloads with fixed lengths call sv_verify).  The
default workload is the 256-row, 8-draft, 129280-token bf16 batch (per-row
temperature from {0, 0.6, 1.0}, lengths from the schedule with
conf ~ Beta(8,2), tau = 0.3).  Inputs are synthetic and seeded.  Workloads
whose inputs are under twice the L2 size are timed step by step with L2
flushed before each step.

Prints one JSON line (rank 0).  `value` is verified draft positions per
second over all ranks (sum of the scheduled lengths per step / device time,
max over ranks); `roofline` is the main verification kernel's bytes per
launch -- the logits the outcome depends on -- over its CUDA-event
duration; `e2e` repeats the measurement with the inputs in pinned host
memory and the host<->device copies inside the timed region;
`cpu_baseline` is the fp64 CPU oracle on all host cores and on one core;
`parity` checks the timed steps' outputs row by row against the oracle.
`--impl reference` times the oracle alone on the whole batch (rank 0;
other ranks exit).

Multi-GPU (torchrun): rows are independent, so every rank verifies its own
batch of B rows (Philox rows offset by rank * B) with no data-path
collective; NCCL carries only the barrier and the max-over-ranks timing.
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

import speculative_decoding_verification_93_b200 as sv  # noqa: E402
from speculative_decoding_verification_93_b200 import workloads  # noqa: E402
from speculative_decoding_verification_93_b200.sharding import max_over_ranks  # noqa: E402

METRIC = "verified draft positions/sec and achieved HBM GB/s (% of B200 peak) at B×K×V"
UNIT = "positions/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ["speculative_decoding_verification_93_b200/csrc/sv_verify.cu",
                  "speculative_decoding_verification_93_b200/csrc/sv_device.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "stream_kernel_traffic.json")
L2_BYTES = 126 << 20


def code_only(text: str) -> str:
    """C/C++/CUDA source with comments and whitespace outside string and
    character literals removed: what the compiler sees, so that editing a
    comment does not change the hash while any change of code does."""
    out = []
    i, n = 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif c.isspace():
            i += 1
        else:
            out.append(c)
            i += 1
    return "".join(out)


def kernel_hash() -> str:
    """Hash of the main kernel's code (comments and whitespace removed)."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        h.update(code_only(open(os.path.join(ROOT, f)).read()).encode())
        h.update(b"\0")
    return h.hexdigest()[:16]


def measured_hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def committed_traffic(workload: str):
    """DRAM bytes per launch of the main kernel from the committed ncu figures
    (a small JSON file keyed by workload), if they were taken on the current
    kernel code."""
    try:
        d = json.load(open(TRAFFIC_FILE))
    except (OSError, ValueError):
        return None
    if d.get("kernel_source_hash") != kernel_hash():
        return None
    w = d.get("workloads", {}).get(workload)
    return None if w is None else float(w["dram_bytes_per_launch"])


class ClockSampler:
    """nvidia-smi sampling during the timed region (clocks, throttle reasons)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(rows)}


def scheduled_bytes(lengths: np.ndarray, temperature: np.ndarray, V: int, esize: int,
                    has_draft: bool = True) -> int:
    """Logit bytes of every scheduled vector: per row
    esize * V * ((L + 1) target vectors + L draft vectors if T > 0)."""
    L = lengths.astype(np.int64)
    drafts = np.where((temperature > 0) & has_draft, L, 0)
    return int((esize * V * ((L + 1) + drafts)).sum())


def needed_bytes(accept: np.ndarray, lengths: np.ndarray, temperature: np.ndarray, V: int,
                 esize: int, has_draft: bool = True) -> int:
    """Logit bytes the outcome depends on, i.e. what verification must read
    once: target positions 0..a and, for sampled rows, draft positions
    0..min(a, L-1), where a is the accepted length (the first rejection, or
    L).  Positions after the first rejection never change the output."""
    a = accept.astype(np.int64)
    L = lengths.astype(np.int64)
    drafts = np.where((temperature > 0) & has_draft, np.minimum(a + 1, L), 0)
    return int((esize * V * ((a + 1) + drafts)).sum())


def oracle_leg(batch, gpu_lengths, results, budget_s: float, budget_1core_s: float,
               parity_budget_s: float, row_base: int = 0):
    """The CPU-baseline leg: the fp64 oracle, as it stands, on the host cores.

    1. All cores: whole passes over the batch, one per timed step's seed, in
       order, until ~budget_s of wall time.
    2. One core: the same rule on row blocks of the first step's seed until
       ~budget_1core_s.
    3. Parity of the timed steps: the GPU's outputs at each step's seed
       (``results``: list of (seed, out_tokens, out_accept)) are checked row
       by row against the oracle -- each row bit-exact or one of the
       oracle's tie-window outcomes -- until ~parity_budget_s.
    The oracle schedules on its own (rows on the schedule window may take
    either length).  Host copies of the logits are made once, untimed."""
    import oracle
    from oracle import compare as ocompare
    from speculative_decoding_verification_93_b200.workloads import to_host_logits
    zt = to_host_logits(batch.zt)
    zd = to_host_logits(batch.zd)
    tok = batch.tokens.cpu().numpy()
    tmp = batch.temperature.cpu().numpy()
    B = tok.shape[0]
    if batch.lengths is None:
        L0, Llo, Lhi = ocompare.schedule_span(batch.conf.cpu().numpy(), batch.tau)
    else:
        L0 = Llo = Lhi = batch.lengths.cpu().numpy()
    rid = np.arange(B, dtype=np.int64) + row_base
    nthreads = oracle.default_threads()
    seeds = [r[0] for r in results]

    positions, passes = 0, 0
    t0 = time.perf_counter()
    while True:
        oracle.verify(zt, zd, tok, L0, tmp, seeds[passes % len(seeds)], row_ids=rid,
                      nthreads=nthreads)
        passes += 1
        positions += int(L0.sum())
        el = time.perf_counter() - t0
        if el >= budget_s or passes >= 1000:
            break
    cpu = dict(value=round(positions / el, 1), unit=UNIT, cores=nthreads, kind="oracle",
               sample=f"{passes} full pass(es) over the {B}-row batch at the timed steps' "
                      f"seeds, {el:.1f} s wall, OpenMP over rows on {nthreads} threads")

    pos1, rows1 = 0, 0
    t0 = time.perf_counter()
    while True:
        r0 = rows1 % B
        r1 = min(B, r0 + 8)
        oracle.verify(zt[r0:r1], zd[r0:r1], tok[r0:r1], L0[r0:r1], tmp[r0:r1],
                      seeds[(rows1 // B) % len(seeds)], row_ids=rid[r0:r1], nthreads=1)
        pos1 += int(L0[r0:r1].sum())
        rows1 += r1 - r0
        el1 = time.perf_counter() - t0
        if el1 >= budget_1core_s or rows1 >= 1000 * B:
            break
    cpu["single_core"] = {"value": round(pos1 / el1, 1), "unit": UNIT, "cores": 1,
                          "sample": f"{rows1} rows in blocks of 8 (passes over the batch at "
                                    f"the timed steps' seeds), {el1:.1f} s"}

    tally = ocompare.Tally()
    checked = []
    t0 = time.perf_counter()
    for seed, g_tok, g_acc in results:
        tally.add(ocompare.check_rows(lambda idx: (zt[idx], zd[idx]), tok, tmp, seed, L0, Llo,
                                      Lhi, gpu_lengths, g_tok, g_acc, row_base=row_base,
                                      block=64, nthreads=nthreads))
        checked.append(seed)
        if time.perf_counter() - t0 >= parity_budget_s:
            break
    parity = dict(tally.summary(), steps_checked=len(checked),
                  seeds=f"{checked[0]}..{checked[-1]}",
                  rule="each row bit-exact against the oracle, or one of the oracle's outcomes "
                       "for decisions inside the tie windows (|u - min(1, ratio)| < 1e-5; draw "
                       "target within 1e-5 R of a CDF boundary; |S_i - tau| < 1e-6)")
    if tally.first_invalid:
        parity["first_invalid"] = tally.first_invalid
    return cpu, parity


def needs_flush(batch, esize) -> bool:
    """Inputs smaller than twice the L2 would be partly served from L2 by the
    next step: those workloads flush L2 before every timed step."""
    return (batch.zt.numel() + batch.zd.numel()) * esize < 2 * L2_BYTES


def workload_config(batch, lengths_np, esize):
    s = batch.spec
    dt = "bf16" if s.dtype == torch.bfloat16 else "fp32"
    inputs = (batch.zt.numel() + batch.zd.numel()) * esize
    l2 = (f"inputs {inputs / 1e9:.3f} GB < 2 x 126 MB L2: L2 flushed before every timed step "
          "(a 256 MB buffer written, then another read), each step timed alone with CUDA "
          "events" if needs_flush(batch, esize) else
          f"inputs {inputs / 1e9:.2f} GB > 126 MB L2 (no flush; steps back to back)")
    return {"workload": (f"{s.name}: B={int(batch.zt.shape[0])} K={s.K} V={s.V} {dt} logits; "
                         f"T per row from {list(s.temps)}; "
                         + (f"lengths from sv_schedule (conf~Beta{s.beta}, tau={batch.tau})"
                            if s.fixed_length is None else f"lengths={s.fixed_length}")),
            "B": int(batch.zt.shape[0]), "K": s.K, "V": s.V, "logits": dt,
            "tau": batch.tau if s.fixed_length is None else None,
            "mean_L": float(lengths_np.mean()),
            "l2": l2,
            "data_seed": s.data_seed}


def vocab_parallel_probe(batch, lengths, V, esize, sched_bytes, seed, steps, peak):
    """Vocabulary-parallel verification of the same batch, split over n = 1
    and n = 8 ranks: the time one rank spends in its three kernels
    (sv_vp_stats, sv_vp_decide, sv_vp_draw) for its slice, and the stats
    kernel's roofline.  One GPU stands in for the ranks: every slice's
    statistics are computed once to fill the gathered buffers, then rank 0's
    kernels are timed alone (collectives excluded: they need n GPUs).  L2 is
    flushed before every timed step (an eighth of the logits fits in L2)."""
    from speculative_decoding_verification_93_b200.vocab_parallel import shard_vocab
    dev = batch.zt.device
    B, K1, _ = batch.zt.shape
    K = K1 - 1
    # Read-only flush: fills L2 with clean lines (a write would leave dirty
    # lines that the timed kernel then has to write back).
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    res = {}
    for n in (1, 8):
        sl = []
        for r in range(n):
            v0, v1 = shard_vocab(V, n, r)
            zt_r = batch.zt[:, :, v0:v1].contiguous() if n > 1 else batch.zt
            zd_r = batch.zd[:, :, v0:v1].contiguous() if n > 1 else batch.zd
            sl.append((zt_r, zd_r, sv.vp_slice(zt_r, zd_r, V, v0, n, r)))
        nst = sv.sv_vp_stats_bytes(sl[0][2])
        stats_all = torch.empty(n * nst, dtype=torch.uint8, device=dev)
        stats_local = torch.empty(nst, dtype=torch.uint8, device=dev)
        mass_all = torch.empty(n * B, 2, dtype=torch.float32, device=dev)
        mass_local = torch.empty(B, 2, dtype=torch.float32, device=dev)
        ws = torch.empty(sv.sv_vp_workspace_bytes(sl[0][2]), dtype=torch.uint8, device=dev)
        ot = torch.empty(B, K1, dtype=torch.int32, device=dev)
        oa = torch.empty(B, dtype=torch.int32, device=dev)
        for r, (_, _, d) in enumerate(sl):
            sv.sv_vp_stats(d, batch.tokens, lengths, batch.temperature,
                           stats_all[r * nst:(r + 1) * nst])
        for r, (_, _, d) in enumerate(sl):
            sv.sv_vp_decide(d, stats_all, batch.tokens, lengths, batch.temperature, seed, ot, oa,
                            mass_all[r * B:(r + 1) * B], ws)
        d0 = sl[0][2]
        t_stats, t_step = [], []
        for i in range(steps + 3):
            flush.sum()
            a0 = torch.cuda.Event(enable_timing=True)
            a1 = torch.cuda.Event(enable_timing=True)
            a2 = torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            sv.sv_vp_stats(d0, batch.tokens, lengths, batch.temperature, stats_local)
            a1.record(stream)
            sv.sv_vp_decide(d0, stats_all, batch.tokens, lengths, batch.temperature, seed + i, ot,
                            oa, mass_local, ws)
            sv.sv_vp_draw(d0, mass_all, ot, ws)
            a2.record(stream)
            torch.cuda.synchronize()
            if i >= 3:
                t_stats.append(a0.elapsed_time(a1))
                t_step.append(a0.elapsed_time(a2))
        ms_stats = sum(t_stats) / len(t_stats)
        ms_step = sum(t_step) / len(t_step)
        v0, v1 = shard_vocab(V, n, 0)
        bytes_rank = sched_bytes * (v1 - v0) / V
        gbs = bytes_rank / (ms_stats / 1e3) / 1e9
        res[f"n{n}"] = {"slice_tokens": v1 - v0, "rank_ms_per_step": round(ms_step, 5),
                        "stats_kernel_ms": round(ms_stats, 5),
                        "stats_bytes_per_launch": int(bytes_rank),
                        "stats_gbs": round(gbs, 1), "stats_frac": round(gbs / peak, 4),
                        "exchange_bytes_per_rank": int(nst + B * 8 + B * K1 * 4)}
        del sl, stats_all
    res["note"] = ("one rank's kernels per step with the vocabulary split n ways; the three "
                   "collectives between them are not in these times (one GPU)")
    res["kernel"] = "sv::vp::vp_stats_kernel"
    res["launches_per_step"] = 4
    return res


def run_ours(args, rank, world, local_rank):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import torch.distributed as dist
    batch = workloads.make_batch(args.workload, device=dev, tau=args.tau,
                                 B=args.rows if args.rows > 0 else None,
                                 data_seed=workloads.SPECS[args.workload].data_seed + 1000 * rank)
    s = batch.spec
    B, K, V = int(batch.zt.shape[0]), s.K, s.V
    esize = 2 if s.dtype == torch.bfloat16 else 4
    dt = sv.SV_BF16 if esize == 2 else sv.SV_F32
    ws = torch.empty(sv.sv_verify_workspace_bytes(B, K, V, dt), dtype=torch.uint8, device=dev)
    out_tok = torch.empty(B, K + 1, dtype=torch.int32, device=dev)
    out_acc = torch.empty(B, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    lengths = torch.empty(B, dtype=torch.int32, device=dev)
    row_base = rank * B
    fixed = batch.lengths

    def step(i, zt, zd, tokens, temp, conf, ln):
        if fixed is None:
            sv.sv_schedule_verify(zt, zd, tokens, conf, batch.tau, ln, temp, args.seed + i, out_tok,
                                  out_acc, ws, status=status, row_base=row_base)
        else:
            sv.sv_verify(zt, zd, tokens, ln, temp, args.seed + i, out_tok, out_acc, ws,
                         status=status, row_base=row_base)

    ln_buf = lengths if fixed is None else fixed
    for i in range(args.warmup):
        step(i, batch.zt, batch.zd, batch.tokens, batch.temperature, batch.conf, ln_buf)
    torch.cuda.synchronize()
    lengths_np = ln_buf.cpu().numpy()
    temp_np = batch.temperature.cpu().numpy()
    positions = int(lengths_np.sum())
    sched_bytes = scheduled_bytes(lengths_np, temp_np, V, esize)

    # ---- device-timed region ------------------------------------------------
    clocks = ClockSampler(local_rank)
    if rank == 0:
        clocks.start()
    # Keep the GPU busy for --clock-load-s (about half a second) of untimed
    # steps while the sampler (one sample per 200 ms) starts, so its samples
    # see the load the timed region runs under; every rank runs the same
    # count.
    n_load = max(0, int(args.clock_load_s / 120e-6))
    for i in range(n_load):
        step(args.warmup + i, batch.zt, batch.zd, batch.tokens, batch.temperature, batch.conf,
             ln_buf)
    flush = needs_flush(batch, esize)
    if flush:
        # L2 flush between steps: write one 256 MB buffer, then read another,
        # so the step starts with none of its inputs in L2 and no dirty lines
        # left to write back.
        flush_w = torch.empty(64 << 20, dtype=torch.float32, device=dev)
        flush_r = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if flush:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for i in range(args.steps):
            flush_w.zero_()
            flush_r.sum()
            evs[i][0].record(stream)
            step(args.warmup + i, batch.zt, batch.zd, batch.tokens, batch.temperature,
                 batch.conf, ln_buf)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        ms_total = sum(a.elapsed_time(b) for a, b in evs)
    else:
        e0.record(stream)
        for i in range(args.steps):
            step(args.warmup + i, batch.zt, batch.zd, batch.tokens, batch.temperature,
                 batch.conf, ln_buf)
        e1.record(stream)
        torch.cuda.synchronize()
        ms_total = e0.elapsed_time(e1)
    if dist:
        dist.barrier()
    clk = clocks.stop() if rank == 0 else None
    ms_total = max_over_ranks(ms_total, dev)
    ms_step = ms_total / args.steps
    value = positions * world / (ms_step / 1e3)
    st = int(status.item())

    # ---- main-kernel duration: the same K steps again, with the library
    # recording CUDA events around the stream kernel on its launching stream
    # (kept out of the region above: an event between two launches stops them
    # from overlapping, which costs the step about 10 us) -------------------
    sv.sv_profile_begin(args.steps)
    torch.cuda.synchronize()
    need, results = [], []
    for i in range(args.steps):
        if flush:
            flush_w.zero_()
            flush_r.sum()
        step(args.warmup + i, batch.zt, batch.zd, batch.tokens, batch.temperature, batch.conf,
             ln_buf)
        acc_np = out_acc.cpu().numpy()
        need.append(needed_bytes(acc_np, lengths_np, temp_np, V, esize))
        # same seeds as the timed steps, so these are the timed steps' outputs
        results.append((args.seed + args.warmup + i, out_tok.cpu().numpy(), acc_np))
    torch.cuda.synchronize()
    kernel_ms = sv.sv_profile_read(args.steps)
    sv.sv_profile_begin(0)
    alg_bytes = sum(need) / len(need)

    # ---- the schedule alone (the step above runs it before each verification) --
    sched = None
    if rank == 0 and fixed is None:
        sch_len = torch.empty(B, dtype=torch.int32, device=dev)
        for _ in range(3):
            sv.sv_schedule(batch.conf, batch.tau, sch_len)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            sv.sv_schedule(batch.conf, batch.tau, sch_len)
        e1.record(stream)
        torch.cuda.synchronize()
        sched = {"kernel": "sv::schedule_kernel", "us_per_call": round(e0.elapsed_time(e1) /
                                                                       args.steps * 1e3, 2),
                 "rows": B, "positions": K, "bound": "launch latency (B threads)"}

    # ---- hardware-aware admission on the same confidences (next row of the
    # scheduler): a profiled speed table of the shape steps/s = s0/(1+n/n0) -------
    admit = None
    if rank == 0:
        n_tab = torch.arange(B * (K + 1) + 2, device=dev, dtype=torch.float32)
        speed_tab = (1000.0 / (1.0 + n_tab / (4.0 * B))).contiguous()
        adm_len = torch.empty(B, dtype=torch.int32, device=dev)
        adm_tau = torch.empty(1, dtype=torch.float32, device=dev)
        for _ in range(3):
            sv.sv_schedule_admit(batch.conf, speed_tab, adm_len, adm_tau)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            sv.sv_schedule_admit(batch.conf, speed_tab, adm_len, adm_tau)
        e1.record(stream)
        torch.cuda.synchronize()
        admit = {"kernel": "sv::admit_kernel", "us_per_call": round(e0.elapsed_time(e1) /
                                                                   args.steps * 1e3, 2),
                 "candidates": B * K, "admitted": int(adm_len.sum().item()),
                 "tau": round(float(adm_tau.item()), 6), "bound": "latency (one CTA)"}

    # ---- confidence-head calibration (per-position temperature scaling) on
    # synthetic held-out blocks: the fit that produces the confidences -------
    calib = None
    if rank == 0:
        hl, ha = workloads.sts_heldout(262144, K, seed=17)
        hlt = torch.from_numpy(hl).to(dev)
        hat = torch.from_numpy(ha).to(dev)
        hT = torch.empty(K, dtype=torch.float32, device=dev)
        hece = torch.empty(2, dtype=torch.float32, device=dev)
        hws = torch.empty(sv.sv_sts_workspace_bytes(262144, K), dtype=torch.uint8, device=dev)
        for _ in range(3):
            sv.sv_sts_fit(hlt, hat, hT, hece, hws)
        torch.cuda.synchronize()
        n_fit = max(1, min(args.steps, 10))
        e0.record(stream)
        for _ in range(n_fit):
            sv.sv_sts_fit(hlt, hat, hT, hece, hws)
        e1.record(stream)
        torch.cuda.synchronize()
        calib = {"kernel": "sv::sts_fit_kernel",
                 "us_per_call": round(e0.elapsed_time(e1) / n_fit * 1e3, 2),
                 "blocks": 262144, "positions": K,
                 "ece_before": round(float(hece[0].item()), 5),
                 "ece_after": round(float(hece[1].item()), 5),
                 "bound": "fp64 sigmoid per observed (block, position) and pass; grid barriers"}
        del hlt, hat, hws

    # ---- end-to-end through host buffers: sv_verify_host takes the inputs in
    # pinned host memory, schedules on the device, and copies to the device
    # only the logits the outcome depends on, one position level at a time
    # (rows leave once decided), then copies the outputs back ----------------
    e2e = None
    if not args.no_e2e:
        host = {n: getattr(batch, n).cpu().pin_memory() for n in
                ("zt", "zd", "tokens", "temperature", "conf")}
        h_tok = torch.empty(B, K + 1, dtype=torch.int32).pin_memory()
        h_acc = torch.empty(B, dtype=torch.int32).pin_memory()
        h_len = (fixed.cpu() if fixed is not None else torch.empty(B, dtype=torch.int32)).pin_memory()
        hws = torch.empty(sv.sv_verify_host_workspace_bytes(B, K, V, dt), dtype=torch.uint8,
                          device=dev)
        e2e_steps = max(1, min(args.steps, args.e2e_steps))
        h2d_seen, d2h_seen = [], []

        def e2e_step(i):
            h2d_seen.append(sv.sv_verify_host(
                host["zt"], host["zd"], host["conf"] if fixed is None else None, batch.tau,
                host["tokens"], host["temperature"], args.seed + i, h_tok, h_acc, h_len, hws,
                row_base=row_base, levelwise=True))
            # Device-to-host bytes: the lengths (when scheduled), then per verified
            # level the accept lengths and the tokens.  Level-wise outputs are on
            # the host when the call returns; a row is settled at level a + 1
            # (rejected) or max(L, 1) (done), and the levels run to the last one.
            a, L = h_acc.numpy(), h_len.numpy()
            levels = max(1, int(np.where(a < L, a + 1, np.maximum(L, 1)).max()))
            d2h_seen.append((B * 4 if fixed is None else 0) + levels * (B * 4 + B * (K + 1) * 4))

        e2e_step(0)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        e0.record(stream)
        for i in range(e2e_steps):
            e2e_step(i + 1)
        e1.record(stream)
        torch.cuda.synchronize()
        ms_e2e = e0.elapsed_time(e1)
        ms_e2e = max_over_ranks(ms_e2e, dev)
        d2h = sum(d2h_seen[1:]) / len(d2h_seen[1:])
        full = sum(host[n].numel() * host[n].element_size() for n in ("zt", "zd"))
        h2d_mean = sum(h2d_seen[1:]) / len(h2d_seen[1:])   # varies with each step's acceptances
        e2e = {"value": positions * world / (ms_e2e / e2e_steps / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": int(round(h2d_mean)), "d2h_bytes_per_step": int(round(d2h)),
               "steps": e2e_steps, "api": "sv_verify_host (levelwise)",
               "note": "inputs in pinned host memory; the schedule's lengths come back, then "
                       "position level l of the rows still undecided is copied and verified "
                       "(one synchronisation per level), so what crosses to the device is the "
                       "logits the outcome depends on plus one look-ahead position per "
                       f"rejecting row ({h2d_mean / full:.2f} of the {full / 1e9:.2f} GB "
                       "of logits, mean over the timed steps)"}
        del host, hws

    # ---- roofline of the main kernel ----------------------------------------
    peak, peak_src = measured_hbm_peak()
    kms = [t for t in kernel_ms if t > 0]
    avg_kernel_ms = sum(kms) / len(kms) if kms else float("nan")
    # achieved: the bytes the outcome depends on -- target positions 0..a and
    # draft positions 0..min(a, L-1) of sampled rows, a the accepted length --
    # each launch's own figure over that launch's duration, averaged.  Those
    # are the bytes verification must read once; positions after a row's
    # first rejection never change the output and the kernel skips them.
    # The bytes of every scheduled logit, read or not, are kept as a
    # secondary figure.
    achieved = (sum(nb / (t / 1e3) for nb, t in zip(need, kernel_ms) if t > 0) / len(kms) / 1e9
                if kms else float("nan"))
    achieved_sched = (sum(sched_bytes / (t / 1e3) for t in kernel_ms if t > 0) / len(kms) / 1e9
                      if kms else float("nan"))
    traffic = committed_traffic(args.workload if args.tau is None else
                                f"{args.workload}_tau{args.tau:g}")
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src ==
                "measured" else "fallback 6650 GB/s",
                "kernel": "sv::stream_kernel", "kernel_ms": round(avg_kernel_ms, 5),
                "algorithmic_bytes_per_launch": int(alg_bytes),
                "algorithmic_bytes": "logits the outcome depends on, each read once: target "
                                     "positions 0..a and draft positions 0..min(a, L-1) of "
                                     "sampled rows (a = accepted length); mean over the timed "
                                     "steps",
                "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
                "scheduled_bytes_per_launch": int(sched_bytes),
                "scheduled_bytes": "every scheduled logit once, elt*V*[(L_b+1) + L_b*(T_b>0)] "
                                   "per row; the kernel does not read the positions after a "
                                   "row's first rejection once it is known",
                "achieved_if_all_scheduled_read": round(achieved_sched, 1),
                "frac_if_all_scheduled_read": round(achieved_sched / peak, 4),
                "traffic_rate_gbs": (round(traffic / (avg_kernel_ms / 1e3) / 1e9, 1)
                                     if traffic else None),
                "step_gbs": round(alg_bytes / (ms_step / 1e3) / 1e9, 1),
                "kernel_timing": "CUDA events around each stream-kernel launch over a second "
                                 "timed pass of the same steps"}

    vocab = None
    if rank == 0 and world == 1 and not args.no_vocab:
        vocab = vocab_parallel_probe(batch, ln_buf, V, esize, sched_bytes, args.seed,
                                     min(args.steps, 20), peak)

    cpu = parity = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu, parity = oracle_leg(batch, lengths_np, results, args.cpu_seconds,
                                 args.cpu_1core_seconds, args.parity_seconds,
                                 row_base=row_base)

    if rank == 0:
        out = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
               "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
               "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
               "dtype": "f32", "data": "synthetic",
               "config": dict(workload_config(batch, lengths_np, esize),
                              parallelism=f"dp{world} (row shards, no collective)"),
               "e2e": e2e, "gpu_launches": args.steps * sv.sv_verify_launches(),
               "roofline": roofline, "cpu_baseline": cpu, "parity": parity, "clocks": clk,
               "schedule": sched,
               "admission": admit,
               "calibration": calib, "vocab_parallel": vocab,
               "device_status": st, "impl": "ours"}
        print(json.dumps(out), flush=True)
    del batch
    if dist:
        dist.barrier()


def run_reference(args, rank, world):
    """The oracle (fp64 CPU) timed as it stands on the host cores: each step is
    one bounded pass over a row sample of the same workload."""
    if rank != 0:
        return
    batch = workloads.make_batch(args.workload, device="cpu", tau=args.tau)
    s = batch.spec
    import oracle
    from speculative_decoding_verification_93_b200.workloads import to_host_logits
    if batch.lengths is None:
        lengths_np, _, _ = oracle.schedule(batch.conf.numpy(), batch.tau)
    else:
        lengths_np = batch.lengths.numpy()
    rows = np.arange(s.B if args.ref_rows <= 0 else min(s.B, args.ref_rows))
    zt = to_host_logits(batch.zt[: len(rows)])
    zd = to_host_logits(batch.zd[: len(rows)])
    tok = batch.tokens[: len(rows)].numpy()
    tmp = batch.temperature[: len(rows)].numpy()
    ln = lengths_np[: len(rows)]
    nthreads = oracle.default_threads()
    for i in range(args.warmup):
        oracle.verify(zt, zd, tok, ln, tmp, args.seed + i, nthreads=nthreads)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle.schedule(batch.conf[: len(rows)].numpy(), batch.tau)
        oracle.verify(zt, zd, tok, ln, tmp, args.seed + args.warmup + i, nthreads=nthreads)
    el = time.perf_counter() - t0
    positions = int(ln.sum())
    value = positions * args.steps / el
    esize = 2 if s.dtype == torch.bfloat16 else 4
    sample = (f"the whole {s.B}-row batch per step" if len(rows) == s.B else
              f"rows 0..{len(rows) - 1} of the {s.B}-row batch per step")
    out = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": dict(workload_config(batch, lengths_np, esize),
                          parallelism="host cores (OpenMP over rows)"),
           "impl": "reference",
           "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": nthreads,
                            "kind": "oracle", "sample": sample},
           "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="c2", choices=sorted(workloads.SPECS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-vocab", action="store_true")
    ap.add_argument("--clock-load-s", type=float, default=0.5,
                    help="seconds of untimed steps before the timed region, so the clock "
                         "sampler sees load (0 under a profiler)")
    ap.add_argument("--tau", type=float, default=None,
                    help="schedule threshold for workloads with scheduled lengths "
                         "(default: the workload's first)")
    ap.add_argument("--rows", type=int, default=0,
                    help="rows of the batch (0: the workload's own B); smaller batches of the "
                         "same workload for profiler captures")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--cpu-1core-seconds", type=float, default=5.0)
    ap.add_argument("--parity-seconds", type=float, default=15.0)
    ap.add_argument("--ref-rows", type=int, default=0,
                    help="rows of the batch the reference arm verifies per step (0: all)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
