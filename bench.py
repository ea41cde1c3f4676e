"""Benchmark: one SMC-SD round (score -> resample -> page-table remap) per step.

Workload: 256 sequences x 32 particles x (8+1) positions, V = 128256, bf16
target and draft logits (~37.8 GB read per round), systematic resampling and
a 128-page table remap for all 8192 particles.  Inputs are synthetic (seeded
generator, built on the device) and larger than L2, so no flush is needed.

Prints one JSON line (rank 0).  Multi-GPU: one process per GPU under torchrun;
each rank runs its own replica of the workload on disjoint sequences (weak
scaling, no collective on the data path; barrier + max-over-ranks timing).

On one GPU the line also carries `per_config`: the path's other
configurations (one SMC-SD sequence in fp32, the 64-sequence batch, standard
verification, dense and sparse Gumbel-top-k) timed on their own with L2
flushed (and hot where the inputs fit in L2), each with its clocks, its
algorithmic bytes against the copy peak and its own summary.
"""

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "verify+resample logit rows/s; achieved HBM TB/s as fraction of B200 peak"
WORKLOAD = "smc_scale"


KERNEL_SOURCES = ["resample_online_log_b200/csrc/smc.cu", "resample_online_log_b200/csrc/rows.cuh",
                  "resample_online_log_b200/csrc/common.cuh"]
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (the measured copy peak is the denominator of frac)
TRAFFIC_SUMMARY = "profiles/smc_kernel_smc_scale.md"


def _code_only(text):
    """Source text without comments and with whitespace runs collapsed, so that a
    comment-only edit keeps the hash (the compiled kernel is the same)."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def measured_traffic(B):
    """DRAM bytes (read + write) of one score-kernel launch over B sequences, from
    the committed ncu summary, if it was taken on the current kernel sources."""
    path = os.path.join(ROOT, TRAFFIC_SUMMARY)
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            if line.startswith("- ") and ":" in line:
                k, v = line[2:].split(":", 1)
                fields[k.strip()] = v.strip().strip("`")
    try:
        if fields.get("source_sha256") != kernel_source_hash():
            return None
        return float(fields["dram_bytes_per_sequence"]) * B
    except (KeyError, ValueError):
        return None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=timedelta(seconds=600))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _oracle_inputs(cfg, b, parts):
    """Host inputs of particles `parts` of sequence b of the workload (the seeded
    generator's exact values) and that sequence's page table."""
    from synth import gen
    rows = np.array([(b * cfg.N + n) * cfg.R + k for n in parts for k in range(cfg.R)])
    zt, zd = gen.gen_rows(cfg.seed, rows, cfg.V, cfg.sigma_z, cfg.L_head,
                          np.full(rows.shape, cfg.sigma_d_of_seq(b), dtype=np.float32), cfg.dtype)
    P, R = len(parts), cfg.R
    zt = zt.reshape(1, P, R, cfg.V)
    zd = zd.reshape(1, P, R, cfg.V)
    did = rows.reshape(P, R)[:, :cfg.K].reshape(-1)
    x = gen.draft_tokens_for_rows(cfg.seed, did, zd[:, :, :cfg.K].reshape(-1, cfg.V), cfg.tau)
    pt = gen.page_table(cfg.seed, cfg.B, cfg.N, cfg.P)[b:b + 1, parts]
    return dict(zT=zt, zD=zd, draft=x.reshape(1, P, cfg.K)), pt


def _oracle_round(cfg, h, pt):
    """The oracle's SMC-SD round (score -> resample -> remap) on the given particles."""
    import oracle
    o = oracle.smcsd_score(h["zT"], h["zD"], h["draft"], cfg.tau, cfg.seed, 1)
    r = oracle.smcsd_resample(o["logw"], cfg.seed, 1)
    oracle.kv_pagetable_remap(pt, r["ancestors"], num_pages=cfg.B * cfg.N * cfg.P,
                              tok_in=o["tokens"])
    return h["zT"].shape[1] * cfg.R


PARTS_PER_TASK = 8  # particles of one sequence per oracle process (72 row pairs)


def _oracle_proc(conn, b, n0):
    """One host core: generates its particles of the workload once, then runs the
    oracle's round on them on request, `reps` times or until `budget_s` seconds of
    compute, and answers (row pairs, seconds)."""
    from synth import gen
    cfg = gen.CONFIGS[WORKLOAD]
    h, pt = _oracle_inputs(cfg, b, list(range(n0, n0 + PARTS_PER_TASK)))
    conn.send("ready")
    while True:
        msg = conn.recv()
        if msg is None:
            break
        reps, budget_s = msg
        rows, t = 0, 0.0
        for _ in range(reps):
            t0 = time.perf_counter()
            rows += _oracle_round(cfg, h, pt)
            t += time.perf_counter() - t0
            if budget_s and t >= budget_s:
                break
        conn.send((rows, t))
    conn.close()


def oracle_cores():
    """Host cores the oracle baseline uses: all this process may run on (at most 32)."""
    return max(1, min(32, len(os.sched_getaffinity(0))))


class OracleCores:
    """One spawned process per host core, each holding 8 particles of its own
    sequence of the workload (process w: sequence w // 4, particles 8 (w % 4) ..)."""

    def __init__(self, cfg, workers):
        import multiprocessing as mp
        ctx = mp.get_context("spawn")
        per_seq = cfg.N // PARTS_PER_TASK
        self.conns, self.procs = [], []
        for w in range(workers):
            a, c = ctx.Pipe()
            pr = ctx.Process(target=_oracle_proc,
                             args=(c, w // per_seq, (w % per_seq) * PARTS_PER_TASK), daemon=True)
            pr.start()
            self.conns.append(a)
            self.procs.append(pr)
        for a in self.conns:
            assert a.recv() == "ready"

    def run(self, reps, budget_s=0.0):
        for a in self.conns:
            a.send((reps, budget_s))
        return [a.recv() for a in self.conns]

    def close(self):
        for a in self.conns:
            a.send(None)
        for pr in self.procs:
            pr.join(timeout=30)


def oracle_baseline(cfg, budget_s=10.0):
    """The oracle (as it stands) on every host core at once, each core on 8
    particles of its own sequence of the workload until `budget_s` seconds of
    compute; returns (row pairs/s of all cores together = total rows / the
    slowest core's time, cores, sample text)."""
    workers = oracle_cores()
    pool = OracleCores(cfg, workers)
    try:
        pool.run(1)  # warm
        res = pool.run(10 ** 6, budget_s)
    finally:
        pool.close()
    rows = sum(r for r, _ in res)
    t = max(s for _, s in res)
    sample = (f"{workers} processes x {PARTS_PER_TASK} particles x {cfg.R} row pairs "
              f"(V={cfg.V}) of the workload, {rows} row pairs, {t:.1f} s on the slowest core")
    return rows / t, workers, sample


def run_reference(args, rank, world):
    """--impl reference: the fp64 NumPy oracle on the host cores (rank 0 only).
    One step = the oracle's round on 8 particles (72 row pairs) per core, every
    core at once on its own particles of the workload."""
    if rank != 0:
        return
    from synth import gen
    cfg = gen.CONFIGS[WORKLOAD]
    workers = oracle_cores()
    pool = OracleCores(cfg, workers)
    try:
        for i in range(args.warmup):
            pool.run(1)
        rows, t_total = 0, 0.0
        for i in range(args.steps):
            t0 = time.perf_counter()
            res = pool.run(1)
            t_total += time.perf_counter() - t0
            rows += sum(r for r, _ in res)
    finally:
        pool.close()
    value = rows / t_total
    sample = (f"per step {workers} processes x {PARTS_PER_TASK} particles x {cfg.R} row pairs "
              f"(V={cfg.V}) of the workload, NumPy fp64")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "rows/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * t_total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": cfg.B, "N": cfg.N, "K": cfg.K, "V": cfg.V,
                   "logits": cfg.dtype, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "rows/s", "cores": workers, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local):
    import resample_online_log_b200 as lib
    from synth import device as sdev
    from synth import gen

    cfg = gen.CONFIGS[WORKLOAD]
    if args.sequences:  # a smaller case of the same workload (profiling)
        cfg = gen.SynthConfig(**{**cfg.__dict__, "B": args.sequences})
    if rank:  # disjoint synthetic sequences per replica
        cfg = gen.SynthConfig(**{**cfg.__dict__, "seed": cfg.seed + 1000 * rank})
    B, N, R, K, V, P = cfg.B, cfg.N, cfg.R, cfg.K, cfg.V, cfg.P
    dev = "cuda"
    d = sdev.gen_config_device(cfg)
    zT, zD, x = d["zT"], d["zD"], d["draft"]
    pt = torch.from_numpy(gen.page_table(cfg.seed, B, N, P)).to(dev)
    logw = torch.empty((B, N), dtype=torch.float64, device=dev)
    bonus = torch.empty((B, N), dtype=torch.int32, device=dev)
    tv = torch.empty((B, N, R), dtype=torch.float32, device=dev)
    toks = torch.empty((B, N, R), dtype=torch.int32, device=dev)
    anc = torch.empty((B, N), dtype=torch.int32, device=dev)
    W = torch.empty((B, N), dtype=torch.float64, device=dev)
    ess = torch.empty((B,), dtype=torch.float64, device=dev)
    pt_out = torch.empty_like(pt)
    tok_out = torch.empty_like(toks)
    refcnt = torch.empty((B * N * P,), dtype=torch.int32, device=dev)
    err = torch.zeros((1,), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    ev_pairs = []

    def step(i, record=False):
        rnd = i + 1
        if record:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        lib.smcsd_score(zT, zD, x, cfg.tau, cfg.seed, rnd, logw, bonus, tv_out=tv, tokens_out=toks,
                        dev_err=err)
        if record:
            e1.record(stream)
            ev_pairs.append((e0, e1))
        lib.smcsd_resample(logw, cfg.seed, rnd, anc, w_out=W, ess_out=ess, dev_err=err)
        lib.kv_pagetable_remap(pt, anc, pt_out, tok_in=toks, tok_out=tok_out, page_refcnt=refcnt,
                               num_pages=B * N * P, dev_err=err)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(args.warmup + i, record=True)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    clocks = clk.stop()
    ms_local = t0.elapsed_time(t1)
    ms = max_over_ranks(ms_local, world)
    score_ms = statistics.mean(a.elapsed_time(b) for a, b in ev_pairs)
    score_ms = max_over_ranks(score_ms, world)
    assert int(err.item()) == 0, f"device error word {int(err.item())}"
    ess_n = (ess / N).cpu().numpy()

    rows_per_step = B * N * R
    value = rows_per_step * world * args.steps / (ms * 1e-3)
    esize = 2 if cfg.dtype == "bf16" else 4
    alg_bytes = (2 * rows_per_step * V * esize + B * N * K * 4      # logits + draft tokens
                 + B * N * (8 + 4) + rows_per_step * (4 + 4))       # logw, bonus, tv, tokens
    hbm_peak, peak_kind = peaks()
    achieved = alg_bytes / (score_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "rows/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD if not args.sequences else f"{WORKLOAD}[B={B}]",
                   "B": B, "N": N, "K": K, "V": V, "logits": cfg.dtype,
                   "tau": cfg.tau, "pages_per_particle": P, "parallelism": f"replicas{world}",
                   "l2": f"inputs ({2 * rows_per_step * V * esize / 1e9:.1f} GB) larger than L2; no flush"},
        "hbm_TBps_score": achieved / 1e3,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": measured_traffic(B), "kernel": "smc_kernel",
                     "peak_kind": peak_kind, "score_ms": score_ms,
                     "algorithmic_bytes": alg_bytes,
                     "frac_of_nominal_8TBps": achieved / NOMINAL_HBM_GBS},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
        "ess_over_N": {"mean": float(ess_n.mean()), "min": float(ess_n.min()),
                       "max": float(ess_n.max())},
    }
    # End to end through the public API with host buffers (pinned), one replica.
    if args.e2e_steps > 0:
        h_zT = torch.empty(zT.shape, dtype=zT.dtype, pin_memory=True)
        h_zD = torch.empty(zD.shape, dtype=zD.dtype, pin_memory=True)
        h_x = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
        h_pt = pt.cpu().pin_memory()
        h_zT.copy_(zT)
        h_zD.copy_(zD)
        h_x.copy_(x)
        outs = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                for t in (logw, bonus, anc, pt_out, tok_out)]
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.e2e_steps):
            zT.copy_(h_zT, non_blocking=True)
            zD.copy_(h_zD, non_blocking=True)
            x.copy_(h_x, non_blocking=True)
            pt.copy_(h_pt, non_blocking=True)
            step(1000 + i)
            for o, t in zip(outs, (logw, bonus, anc, pt_out, tok_out)):
                o.copy_(t, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        h2d = sum(t.numel() * t.element_size() for t in (h_zT, h_zD, h_x, h_pt))
        d2h = sum(t.numel() * t.element_size() for t in outs)
        line["e2e"] = {"value": rows_per_step * world * args.e2e_steps / (e2e_ms * 1e-3),
                       "unit": "rows/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "steps": args.e2e_steps}
        del h_zT, h_zD
    if rank == 0 and world == 1 and args.configs:
        line["per_config"] = per_config(args, hbm_peak, peak_kind)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample = oracle_baseline(gen.CONFIGS[WORKLOAD], budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": v, "unit": "rows/s", "cores": cores, "kind": "oracle",
                                "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)


PER_CONFIGS = ("smc_small", "smc_batch", "verify", "topk_dense", "topk_sparse", "draft", "ngram",
               "bandit")


def per_config(args, hbm_peak, peak_kind):
    """The path's other configurations, each timed on its own (one GPU): kernel
    time (mean and median of `args.config_steps` launches, L2 flushed before
    each by writing 256 MB, plus hot timings where the inputs fit in L2), the
    algorithmic bytes against the copy-bandwidth peak, the SM clocks sampled
    while it ran, and the configuration's own summary (ESS of the SMC rounds,
    the verify accepted-length histogram by draft-noise third)."""
    import resample_online_log_b200 as lib
    from synth import device as sdev
    from synth import gen

    dev = "cuda"
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # 2x L2
    err = torch.zeros((1,), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    wanted = [c for c in args.configs.split(",") if c]
    out = {}

    def timed(call, flush_l2, n):
        for i in range(max(3, args.warmup)):
            call(i)
        torch.cuda.synchronize()
        clk = ClockSampler(torch.cuda.current_device())
        clk.start()
        time.sleep(0.2)
        ts = []
        for i in range(n):
            if flush_l2:
                flush.add_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            call(100 + i)
            e1.record(stream)
            ts.append((e0, e1))
        torch.cuda.synchronize()
        clocks = clk.stop()
        ms = [a.elapsed_time(b) for a, b in ts]
        assert int(err.item()) == 0, f"device error word {int(err.item())}"
        return statistics.mean(ms), statistics.median(ms), clocks

    def entry(ms, med, alg, units, unit_name, clocks, extra):
        ach = alg / (ms * 1e-3) / 1e9
        return {"ms_mean": ms, "ms_median": med, "algorithmic_bytes": alg,
                "achieved_GBps": ach, "frac": ach / hbm_peak, "peak": hbm_peak,
                "peak_kind": peak_kind, unit_name: units / (ms * 1e-3), "clocks": clocks, **extra}

    n = args.config_steps
    for name in wanted:
        if name in ("smc_small", "smc_batch"):
            cfg = gen.CONFIGS[name]
            d = sdev.gen_config_device(cfg)
            B, N, R, K, V, P = cfg.B, cfg.N, cfg.R, cfg.K, cfg.V, cfg.P
            pt = torch.from_numpy(gen.page_table(cfg.seed, B, N, P)).to(dev)
            logw = torch.empty((B, N), dtype=torch.float64, device=dev)
            bonus = torch.empty((B, N), dtype=torch.int32, device=dev)
            tv = torch.empty((B, N, R), dtype=torch.float32, device=dev)
            toks = torch.empty((B, N, R), dtype=torch.int32, device=dev)
            anc = torch.empty((B, N), dtype=torch.int32, device=dev)
            ess = torch.empty((B,), dtype=torch.float64, device=dev)
            pt_out, tok_out = torch.empty_like(pt), torch.empty_like(toks)

            def rnd(i):
                lib.smcsd_score(d["zT"], d["zD"], d["draft"], cfg.tau, cfg.seed, i, logw, bonus,
                                tv_out=tv, tokens_out=toks, dev_err=err)
                lib.smcsd_resample(logw, cfg.seed, i, anc, ess_out=ess, dev_err=err)
                lib.kv_pagetable_remap(pt, anc, pt_out, tok_in=toks, tok_out=tok_out, dev_err=err)
            esize = 2 if cfg.dtype == "bf16" else 4
            alg = (2 * B * N * R * V * esize + B * N * K * 4 + B * N * 12 + B * N * R * 8
                   + 2 * B * N * P * 4 + 2 * B * N * R * 4)
            ms, med, clocks = timed(rnd, True, n)
            ess_n = (ess / N).cpu().numpy()
            extra = {"config": {"B": B, "N": N, "K": K, "V": V, "logits": cfg.dtype, "tau": cfg.tau,
                                "step": "score -> resample -> page-table remap", "l2": "flushed"},
                     "ess_over_N": {"mean": float(ess_n.mean()), "min": float(ess_n.min()),
                                    "max": float(ess_n.max())}}
            if 2 * B * N * R * V * esize < (60 << 20):  # fits in L2: the hot figure too
                hms, hmed, _ = timed(rnd, False, n)
                extra["hot_ms_mean"], extra["hot_ms_median"] = hms, hmed
            out[name] = entry(ms, med, alg, B * N * R, "rows_per_s", clocks, extra)
            del d
        elif name == "verify":
            cfg = gen.CONFIGS["verify"]
            d = sdev.gen_config_device(cfg)
            B, K, V = cfg.B, cfg.K, cfg.V
            acc = torch.empty((B,), dtype=torch.int32, device=dev)
            toks = torch.empty((B, K + 1), dtype=torch.int32, device=dev)
            tv = torch.empty((B, K), dtype=torch.float32, device=dev)

            def ver(i):
                lib.sd_verify_reject(d["zT"], d["zD"], d["draft"], cfg.tau, cfg.seed, i, acc, toks,
                                     tv_out=tv, dev_err=err)
            alg = ((2 * K + 1) * V * 2 + K * 4 + 4 + (K + 1) * 4 + K * 4) * B
            ms, med, clocks = timed(ver, True, n)
            hms, hmed, _ = timed(ver, False, n)
            a = acc.cpu().numpy()
            thirds = [(0, 43), (43, 86), (86, 128)]
            hist = {f"sigma_{sd}": np.bincount(a[lo:hi], minlength=K + 1).tolist()
                    for (lo, hi), sd in zip(thirds, cfg.sigma_d)}
            out[name] = entry(ms, med, alg, B * (K + 1), "target_rows_per_s", clocks,
                              {"config": {"B": B, "K": K, "V": V, "logits": cfg.dtype, "tau": cfg.tau,
                                          "l2": "flushed; hot_* without the flush"},
                               "hot_ms_mean": hms, "hot_ms_median": hmed,
                               "accepted_len_hist_by_draft_noise": hist})
            del d
        elif name in ("topk_dense", "topk_sparse"):
            cfg = gen.CONFIGS["topk"]
            rows, V, k = cfg.B, cfg.V, cfg.topk
            idx = torch.empty((rows, k), dtype=torch.int32, device=dev)
            if name == "topk_dense":
                z = sdev.gen_config_device(cfg)["z"]
                sc = torch.empty((rows, k), dtype=torch.float32, device=dev)
                lp = torch.empty((rows, k), dtype=torch.float32, device=dev)

                def tk(i):
                    lib.gumbel_topk(z, k, cfg.tau, cfg.seed, i, idx, score_out=sc, logp_out=lp,
                                    dev_err=err)
                alg = rows * (V * 2 + k * 12)
                ms, med, clocks = timed(tk, True, n)
                out[name] = entry(ms, med, alg, rows, "rows_per_s", clocks,
                                  {"config": {"rows": rows, "V": V, "k": k, "logits": cfg.dtype,
                                              "tau": cfg.tau, "l2": "flushed"}})
                del z
            else:
                six, spr = gen.sparse_rows(cfg.seed, rows, cfg.sparse_L, V)
                ix = torch.from_numpy(six).to(dev)
                pr = torch.from_numpy(spr.astype(np.float32)).to(dev)

                def tks(i):
                    lib.gumbel_topk_sparse(ix, pr, k, cfg.tau, cfg.seed, i, idx, dev_err=err)
                alg = rows * (cfg.sparse_L * 8 + k * 4)
                ms, med, clocks = timed(tks, True, n)
                hms, hmed, _ = timed(tks, False, n)
                out[name] = entry(ms, med, alg, rows, "rows_per_s", clocks,
                                  {"config": {"rows": rows, "L": cfg.sparse_L, "k": k, "tau": cfg.tau,
                                              "l2": "flushed; hot_* without the flush"},
                                   "hot_ms_mean": hms, "hot_ms_median": hmed})
        elif name == "draft":
            # the draft step's sampler over every draft row of the smc_batch round
            cfg = gen.CONFIGS["smc_batch"]
            d = sdev.gen_config_device(cfg)
            zD = d["zD"].reshape(-1, cfg.V)
            rows = zD.shape[0]
            toks = torch.empty((rows,), dtype=torch.int32, device=dev)
            lq = torch.empty((rows,), dtype=torch.float32, device=dev)

            def dr(i):
                lib.sd_draft_sample(zD, cfg.tau, cfg.seed, i, toks, logq_out=lq, dev_err=err)
            alg = rows * (cfg.V * 2 + 8)
            ms, med, clocks = timed(dr, True, n)
            out[name] = entry(ms, med, alg, rows, "rows_per_s", clocks,
                              {"config": {"rows": rows, "V": cfg.V, "logits": cfg.dtype,
                                          "tau": cfg.tau, "l2": "flushed",
                                          "rows_from": "smc_batch draft tensor"}})
            del d
        elif name == "ngram":
            # STAND store: 512 observed positions of a 152064-entry vocabulary,
            # bigram contexts drawn Zipf(1.2) from 2048 n-grams, top-10 rows
            import dataclasses
            cfg = dataclasses.replace(gen.CONFIGS["topk"], B=512)
            U, V, k, nn, cap = cfg.B, cfg.V, 10, 2, 1 << 16
            z = sdev.gen_config_device(cfg)["z"]
            rng = np.random.default_rng(cfg.seed)
            pool = rng.integers(0, V, size=(2048, nn)).astype(np.int32)
            ctx = torch.from_numpy(pool[np.minimum(rng.zipf(1.2, size=U) - 1, 2047)]).to(dev)
            oi = torch.empty((U, k), dtype=torch.int32, device=dev)
            op = torch.empty((U, k), dtype=torch.float32, device=dev)
            tab = lib.NgramTable(cap, k, max_update=U)

            def obs(i):
                lib.ngram_observe_topk(z, k, cfg.tau, oi, op, dev_err=err)
            alg_o = U * (V * 2 + k * 8)
            ms, med, clocks = timed(obs, True, n)
            out["ngram_observe"] = entry(ms, med, alg_o, U, "rows_per_s", clocks,
                                         {"config": {"rows": U, "V": V, "k": k, "logits": cfg.dtype,
                                                     "tau": cfg.tau, "l2": "flushed"}})

            def upd(i):
                tab.update(ctx, oi, op, dev_err=err)
            # reads: contexts and rows; the rows of every touched n-gram read and written
            alg_u = U * (nn * 4 + k * 8) + 2 * U * (8 + 4 + k * 8)
            ms, med, clocks = timed(upd, False, n)
            out["ngram_update"] = entry(ms, med, alg_u, U, "observations_per_s", clocks,
                                        {"config": {"observations": U, "n": nn, "k": k,
                                                    "capacity": cap, "distinct_ngrams": 2048,
                                                    "l2": "hot (kilobyte-scale inputs)"}})
            li = torch.empty((U, k), dtype=torch.int32, device=dev)
            lp_ = torch.empty((U, k), dtype=torch.float32, device=dev)
            cnt = torch.empty((U,), dtype=torch.int32, device=dev)

            def look(i):
                tab.lookup(ctx, li, lp_, count_out=cnt, dev_err=err)
            alg_l = U * (nn * 4 + 8 + 4 + k * 8) + U * (k * 8 + 4)
            ms, med, clocks = timed(look, False, n)
            out["ngram_lookup"] = entry(ms, med, alg_l, U, "queries_per_s", clocks,
                                        {"config": {"queries": U, "n": nn, "k": k, "capacity": cap,
                                                    "l2": "hot (kilobyte-scale inputs)"}})
            del z
        elif name == "bandit":
            # MetaSD-UCB round for 4096 sequences, 8 drafters, K = 5, BD reward
            B, M, K = 4096, 8, 5
            tvb = torch.rand((B, K), device=dev)
            arm = torch.full((B,), -1, dtype=torch.int32, device=dev)
            pulls = torch.zeros((B, M), dtype=torch.int32, device=dev)
            sums = torch.zeros((B, M), dtype=torch.float64, device=dev)

            def ban(i):
                lib.sd_metasd_ucb(arm, pulls, sums, arm, K, tv=tvb, c=2.0, dev_err=err)
            alg = B * (K * 4 + 4 + 4) + 2 * B * M * 12
            ms, med, clocks = timed(ban, False, n)
            out[name] = entry(ms, med, alg, B, "sequences_per_s", clocks,
                              {"config": {"B": B, "M": M, "K": K, "reward": "BD",
                                          "l2": "hot (kilobyte-scale inputs)"}})
        torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sequences", type=int, default=0,
                    help="run B sequences of the workload instead of all 256 (profiling)")
    ap.add_argument("--configs", default=",".join(PER_CONFIGS),
                    help="the other configurations timed into per_config (empty: none)")
    ap.add_argument("--config-steps", type=int, default=20)
    ap.add_argument("--per-config-only", action="store_true",
                    help="print only the per_config object (one GPU)")
    args = ap.parse_args()
    if args.per_config_only:
        hbm_peak, peak_kind = peaks()
        print(json.dumps({"per_config": per_config(args, hbm_peak, peak_kind)}), flush=True)
        return
    rank, world, local = dist_init()
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
