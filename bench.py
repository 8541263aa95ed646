"""Benchmark: chain verification of the B=512, K=8, V=151936 bfloat16 workload (top-k 50,
temperature 0.8) on N GPUs, one process per GPU (weak scaling: every rank verifies its
own batch; no collective on the data path).

One step = one spec_verify_chain call over one batch (row statistics + accept scan +
draw). Prints one JSON line (rank 0). `--impl reference` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import specgen  # noqa: E402

METRIC = "verified draft positions/sec and achieved HBM GB/s (fraction of 8 TB/s)"
UNIT = "positions/s"
L2_NOTE = "inputs larger than L2 (126 MB); no flush between steps"


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def workload(cfg: specgen.ChainConfig, greedy: bool) -> dict:
    name = f"chain_B{cfg.B}_K{cfg.K}_V{cfg.V}_{cfg.dtype}_T{0.0 if greedy else cfg.temp:g}"
    if not greedy:
        name += (f"_topk{cfg.top_k}" if cfg.top_k else "") + \
            (f"_topp{cfg.top_p:g}" if cfg.top_p < 1 else "")
    name += f"_zipf{cfg.zipf:g}" if cfg.zipf else ""
    return {"workload": name, "B": cfg.B, "K": cfg.K,
            "V": cfg.V, "logits": cfg.dtype, "temperature": 0.0 if greedy else cfg.temp,
            "top_k": 0 if greedy else cfg.top_k, "top_p": cfg.top_p, "l2": L2_NOTE}


def algorithmic_bytes(cfg, greedy: bool) -> int:
    """One read of every logit row the step must read: B*(2K+1) rows (B*(K+1) greedy)."""
    rows = cfg.B * ((cfg.K + 1) if greedy else (2 * cfg.K + 1))
    return rows * cfg.V * (2 if cfg.dtype == "bf16" else 4)


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


def kernel_code(src: str) -> str:
    """The source without its // comments and blank lines: what the counters depend on."""
    lines = (ln.split("//", 1)[0].rstrip() for ln in src.splitlines())
    return "\n".join(ln for ln in lines if ln.strip())


def read_profile_traffic(name: str):
    """Per-launch DRAM traffic (read + write bytes) of the row-statistics kernel for this
    workload, from the committed ncu summary; None if there is none or the kernel code
    (comments aside) has changed since the counters were taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)
        with open(os.path.join(ROOT, "draft_token_verification_spec_b200", "csrc",
                               "stream.cuh")) as f:
            sha = hashlib.sha256(kernel_code(f.read()).encode()).hexdigest()[:16]
    except (OSError, ValueError):
        return None
    if rec.get("stream_cuh_sha256_16") != sha:
        return None
    return rec.get("traffic", {}).get(name)


def max_over_ranks(x: float, device, world: int) -> float:
    """The largest x over all ranks (device-timed durations: the job ends with the slowest)."""
    if world <= 1:
        return float(x)
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(B: int, K: int, world: int, steps: int, ms_max: float) -> float:
    """Verified draft positions per second over the whole job: every rank verifies B*K
    positions per step, and the job takes the slowest rank's time."""
    return B * K * world * steps / (ms_max / 1e3)


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix=f"clocks_gpu{self.index}_", suffix=".csv")
            self.fh = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}",
                                          f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "50"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"samples": 0}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.fh.close()
        if os.environ.get("SPEC_CLOCKS_CSV"):  # keep the raw samples where the caller asks
            import shutil
            shutil.copyfile(self.path, os.environ["SPEC_CLOCKS_CSV"])
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 9:
                    continue
                try:
                    sm.append(float(p[1]))
                    mx = max(mx, float(p[2]))
                except ValueError:
                    continue
                for n, v in zip(names, p[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx or None,
                "reasons": sorted(reasons), "samples": len(sm)}


def _events(n):
    import torch
    pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(n)]
    for a, b in pairs:  # torch creates an event on its first record; the library re-records it
        a.record()
        b.record()
    return pairs


def time_calls(step, steps: int, warmup: int):
    """Device time of `steps` calls of step() after `warmup` untimed ones: (total ms, the
    row-statistics stage of each call in ms, from the library's timing hook)."""
    import torch

    import draft_token_verification_spec_b200 as sv

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    pairs = _events(steps)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(steps):
        sv.spec_set_row_kernel_events(*pairs[i])
        step()
    end.record()
    torch.cuda.synchronize()
    sv.spec_set_row_kernel_events(None, None)
    return start.elapsed_time(end), [a.elapsed_time(b) for a, b in pairs]


def roofline_entry(alg: int, row_ms: float, kernel: str = "stream_rows_kernel") -> dict:
    peaks, peak_src = measured_peaks()
    achieved = alg / (row_ms / 1e3) / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
            "peak_source": peak_src + " (STREAM-style copy)",
            "frac_of_8TBs": round(achieved / 8000.0, 4), "kernel": kernel,
            "kernel_ms": round(row_ms, 4), "algorithmic_bytes": alg}


def chain_device_inputs(cfg, greedy, dev):
    """Generator logits and uniforms on the device, and drafter tokens x_i ~ transformed q_i
    (temperature 0: the draft argmax) drawn with the library's own transform and draw."""
    import torch

    import draft_token_verification_spec_b200 as sv

    target, draft = specgen.chain_logits(cfg)
    u = specgen.chain_uniforms(cfg)
    pick = specgen.drafter_uniforms(cfg)

    def to_dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    tg, dg, ug = to_dev(target), to_dev(draft), to_dev(u)
    if greedy:
        xg = dg.float().argmax(dim=2).to(torch.int32).contiguous()
    else:
        probs, _ = sv.spec_logits_to_probs(dg, cfg.temp, cfg.top_k, cfg.top_p, with_entropy=False)
        xg = sv.spec_residual_sample(probs.view(-1, cfg.V), None,
                                     to_dev(pick).view(-1)).view(cfg.B, cfg.K)
        del probs
    torch.cuda.synchronize()
    return target, draft, u, tg, dg, ug, xg


def per_config_chain(cfg, greedy, args, dev) -> dict:
    """One workload timed like the headline (same steps and warm-up), device-resident
    inputs, plus the oracle on the host cores over a bounded sample."""
    import torch

    import draft_token_verification_spec_b200 as sv

    _, _, _, tg, dg, ug, xg = chain_device_inputs(cfg, greedy, dev)
    temp = 0.0 if greedy else cfg.temp
    acc = torch.empty(cfg.B, dtype=torch.int32, device=dev)
    out = torch.empty((cfg.B, cfg.K + 1), dtype=torch.int32, device=dev)
    ws = torch.empty(sv.spec_workspace_size(cfg.B, cfg.K, cfg.V), dtype=torch.uint8, device=dev)

    def step():
        sv.spec_verify_chain(tg, None if greedy else dg, xg, ug, temp, cfg.top_k, cfg.top_p,
                             accepted_len=acc, out_tokens=out, workspace=ws)

    ms, row_ms = time_calls(step, args.steps, args.warmup)
    accl = acc.cpu().numpy()
    assert accl.min() >= 0 and sv.spec_get_device_status(ws) == 0, cfg.name
    row = float(np.mean(row_ms))
    res = {"workload": workload(cfg, greedy)["workload"], "metric_unit": UNIT,
           "value": cfg.B * cfg.K * args.steps / (ms / 1e3), "ms_per_step": ms / args.steps,
           "row_stage_ms": round(row, 4),
           "roofline": {**roofline_entry(algorithmic_bytes(cfg, greedy), row),
                        "traffic": read_profile_traffic(workload(cfg, greedy)["workload"])},
           "mean_accepted_len": float(accl.mean())}
    del tg, dg, ug, xg, ws
    torch.cuda.empty_cache()
    if not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(cfg, greedy, budget_s=4.0)
    return res


def tree_streamed_rows(parent) -> int:
    """Logit rows of one batch row that typical acceptance reads: the rows of nodes with a
    child (a node's row is read only to test its children)."""
    par = np.asarray(parent)
    return int(np.unique(par[1:][(par[1:] >= 0)]).size)


def per_config_tree(cfg, args, dev) -> dict:
    """The MEDUSA-tree workload under typical acceptance: verified positions = B * (N - 1)
    candidate nodes per call."""
    import torch

    import draft_token_verification_spec_b200 as sv

    logits, toks, par = specgen.tree_inputs(cfg)
    lg = torch.from_numpy(logits.view(np.int16)).to(dev).view(torch.bfloat16)
    tk, pa = torch.from_numpy(toks).to(dev), torch.from_numpy(par).to(dev)
    path = torch.empty((cfg.B, cfg.N), dtype=torch.int32, device=dev)
    plen = torch.empty(cfg.B, dtype=torch.int32, device=dev)
    ws = torch.empty(sv.spec_workspace_size(cfg.B, cfg.N, cfg.V), dtype=torch.uint8, device=dev)

    def step():
        sv.spec_verify_tree_typical(lg, tk, pa, cfg.eps, cfg.delta, best_path=path,
                                    accepted_len=plen, workspace=ws)

    ms, row_ms = time_calls(step, args.steps, args.warmup)
    lens = plen.cpu().numpy()
    assert lens.min() >= 1 and sv.spec_get_device_status(ws) == 0
    row = float(np.mean(row_ms))
    alg = cfg.B * tree_streamed_rows(par) * cfg.V * 2
    res = {"workload": cfg.name, "metric_unit": UNIT,
           "value": cfg.B * (cfg.N - 1) * args.steps / (ms / 1e3), "ms_per_step": ms / args.steps,
           "row_stage_ms": round(row, 4), "roofline": roofline_entry(alg, row),
           "mean_accepted_len": float(lens.mean())}
    if not args.no_cpu_baseline:
        import oracle
        threads = os.cpu_count() or 1
        t0 = time.perf_counter()
        oracle.verify_tree_typical(logits, toks, par, cfg.eps, cfg.delta, threads=threads)
        dt = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": cfg.B * (cfg.N - 1) / dt, "unit": UNIT, "cores": threads,
                               "kind": "oracle",
                               "sample": f"all {cfg.B} batch rows, {threads} threads, {dt:.2f}s"}
    return res


def run_ours(args, cfg, greedy, rank, world):
    import torch

    import draft_token_verification_spec_b200 as sv

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    sv.lib()  # fail loudly if the CUDA library is missing
    t0 = time.time()
    target, draft, u, tg, dg, ug, xg = chain_device_inputs(cfg, greedy, dev)
    log(f"[rank {rank}] generated inputs in {time.time() - t0:.1f}s")
    temp = 0.0 if greedy else cfg.temp
    acc = torch.empty(cfg.B, dtype=torch.int32, device=dev)
    out = torch.empty((cfg.B, cfg.K + 1), dtype=torch.int32, device=dev)
    ws = torch.empty(sv.spec_workspace_size(cfg.B, cfg.K, cfg.V), dtype=torch.uint8, device=dev)

    def step():
        sv.spec_verify_chain(tg, None if greedy else dg, xg, ug, temp, cfg.top_k, cfg.top_p,
                             accepted_len=acc, out_tokens=out, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = sv.spec_get_device_status(ws)
    assert status == 0, f"device status {status}"
    accl = acc.cpu().numpy()
    assert accl.min() >= 0, "error rows in the benchmark batch"

    pairs = _events(args.steps)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.2)
    start.record()
    for i in range(args.steps):
        sv.spec_set_row_kernel_events(*pairs[i])
        step()
    end.record()
    torch.cuda.synchronize()
    clock_info = clocks.stop()
    sv.spec_set_row_kernel_events(None, None)
    if world > 1:
        torch.distributed.barrier()
    ms = start.elapsed_time(end)
    row_ms = [a.elapsed_time(b) for a, b in pairs]
    ms_max = max_over_ranks(ms, dev, world)
    value = job_value(cfg.B, cfg.K, world, args.steps, ms_max)

    # end to end through the same call: pinned host inputs in, results out, every step
    e2e_steps = max(3, min(args.steps, 10))
    h_t = torch.from_numpy(target.view(np.int16)).pin_memory() if target.dtype == np.uint16 \
        else torch.from_numpy(target).pin_memory()
    h_d = torch.from_numpy(draft.view(np.int16)).pin_memory() if draft.dtype == np.uint16 \
        else torch.from_numpy(draft).pin_memory()
    h_x = xg.cpu().pin_memory()
    h_u = torch.from_numpy(u).pin_memory()
    h_acc = torch.empty(cfg.B, dtype=torch.int32).pin_memory()
    h_out = torch.empty((cfg.B, cfg.K + 1), dtype=torch.int32).pin_memory()
    tg_raw = tg.view(torch.int16) if tg.dtype == torch.bfloat16 else tg
    dg_raw = dg.view(torch.int16) if dg.dtype == torch.bfloat16 else dg
    h2d = h_t.numel() * h_t.element_size() + (0 if greedy else h_d.numel() * h_d.element_size()) \
        + h_x.numel() * 4 + h_u.numel() * 4
    d2h = h_acc.numel() * 4 + h_out.numel() * 4
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(e2e_steps):
        tg_raw.copy_(h_t, non_blocking=True)
        if not greedy:
            dg_raw.copy_(h_d, non_blocking=True)
        xg.copy_(h_x, non_blocking=True)
        ug.copy_(h_u, non_blocking=True)
        step()
        h_acc.copy_(acc, non_blocking=True)
        h_out.copy_(out, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev, world)
    e2e_value = job_value(cfg.B, cfg.K, world, 1, e2e_ms)

    # the row kernel, the exact finisher (candidate modes only), the double-precision top-p
    # placement (exact normalisers and re-collection, top-p without top-k) and the
    # per-batch-row kernel
    candidates = not greedy and ((0 < cfg.top_k < cfg.V) or cfg.top_p < 1.0)
    refined = not greedy and cfg.top_p < 1.0 and not (0 < cfg.top_k < cfg.V)
    kernels_per_step = 2 + (1 if candidates else 0) + (2 if refined else 0)
    row_avg_ms = float(np.mean(row_ms))
    alg = algorithmic_bytes(cfg, greedy)
    traffic = read_profile_traffic(workload(cfg, greedy)["workload"])
    del h_t, h_d
    return {
        "value": value, "ms_per_step": ms_max / args.steps,
        "roofline": {**roofline_entry(alg, row_avg_ms), "traffic": traffic},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "steps": e2e_steps},
        "gpu_launches": kernels_per_step * args.steps,
        "clocks": clock_info,
        "acceptance": {"mean_accepted_len": float(accl.mean()),
                       "emitted_per_round": float(accl.mean() + 1),
                       "histogram": np.bincount(accl, minlength=cfg.K + 1).tolist()},
        # one read of every logit row, per verified draft position (the minimum the step
        # must move), and what the row kernel's counted DRAM traffic gives per position
        "bytes_per_position": {"algorithmic": alg / (cfg.B * cfg.K),
                               "counted": (None if traffic is None
                                           else traffic / (cfg.B * cfg.K))},
    }


def oracle_drafts(cfg, target, draft, B, greedy):
    import oracle

    pick = specgen.drafter_uniforms(cfg, B)
    if greedy:
        lf = specgen.bf16_bits_to_f32(draft) if draft.dtype == np.uint16 else draft
        return np.argmax(lf, axis=2).astype(np.int32)
    toks = np.empty((B, cfg.K), np.int32)
    for b in range(B):
        probs = oracle.transform_rows(draft[b], cfg.temp, cfg.top_k, cfg.top_p)[0]
        toks[b] = oracle.residual_sample(probs.astype(np.float32), None, pick[b])[0]
    return toks


def time_oracle(cfg, greedy, rows: int, threads: int):
    """Seconds the oracle takes to verify `rows` batch rows of the workload."""
    import oracle

    target, draft = specgen.chain_logits(cfg, rows)
    u = specgen.chain_uniforms(cfg, rows)
    toks = oracle_drafts(cfg, target, draft, rows, greedy)
    t0 = time.perf_counter()
    oracle.verify_chain(target, None if greedy else draft, toks, u, 0.0 if greedy else cfg.temp,
                        cfg.top_k, cfg.top_p, threads=threads)
    return time.perf_counter() - t0


def cpu_baseline(cfg, greedy, budget_s: float = 15.0) -> dict:
    threads = os.cpu_count() or 1
    rows = max(1, threads)
    dt = time_oracle(cfg, greedy, rows, threads)
    grow = int(min(cfg.B, max(rows, rows * budget_s / max(dt, 1e-3) / 2)))
    if grow > rows:
        rows, dt = grow, time_oracle(cfg, greedy, grow, threads)
    return {"value": rows * cfg.K / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"first {rows} of {cfg.B} batch rows ({rows * cfg.K} positions), "
                      f"{threads} threads over batch rows, {dt:.1f}s"}


def per_config_lstate(cfg, args, dev) -> dict:
    """Linear-attention state commit after verification: the factors of the round's steps,
    then the commit of each sequence's accepted prefix to its state, in place. Timed with
    CUDA events around each commit (the factor kernel is reported beside it)."""
    import torch

    import draft_token_verification_spec_b200 as sv

    state, alpha, beta, keys, values, steps = specgen.linear_state_inputs(cfg)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    st, al, be, k, v, n = d(state), d(alpha), d(beta), d(keys), d(values), d(steps)
    w, u, g = sv.spec_linear_state_factors(al, be, k, v)
    torch.cuda.synchronize()
    ev = _events(args.steps)
    fev = _events(args.steps)
    for _ in range(args.warmup):
        sv.spec_commit_linear_state(st, k, w, u, g, n)
    torch.cuda.synchronize()
    for i in range(args.steps):
        fev[i][0].record()
        sv.spec_linear_state_factors(al, be, k, v, w, u, g)
        fev[i][1].record()
        ev[i][0].record()
        sv.spec_commit_linear_state(st, k, w, u, g, n)
        ev[i][1].record()
    torch.cuda.synchronize()
    ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    fms = float(np.mean([a.elapsed_time(b) for a, b in fev]))
    committed = int((steps > 0).sum())
    S = cfg.K + 1
    alg = committed * cfg.H * cfg.dk * cfg.dv * 4 * 2 + \
        int(steps.sum()) * cfg.H * (2 * cfg.dk + cfg.dv) * 4
    res = {"workload": cfg.name, "metric_unit": "committed steps/s",
           "value": float(steps.sum()) / (ms / 1e3), "ms_per_step": ms,
           "factors_ms": round(fms, 4), "mean_steps": float(steps.mean()), "steps_per_round": S,
           "roofline": roofline_entry(alg, ms, kernel="lstate_commit_kernel")}
    del st, al, be, k, v, n, w, u, g
    torch.cuda.empty_cache()
    if not args.no_cpu_baseline:
        import oracle
        threads = os.cpu_count() or 1
        rows = min(cfg.B, 4 * threads)
        t0 = time.perf_counter()
        oracle.linear_state_replay(state[:rows], alpha[:rows], beta[:rows], keys[:rows],
                                   values[:rows], steps[:rows], threads=threads)
        dt = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": float(steps[:rows].sum()) / dt,
                               "unit": "committed steps/s", "cores": threads, "kind": "oracle",
                               "sample": f"first {rows} of {cfg.B} sequences (step-by-step "
                                         f"replay), {threads} threads, {dt:.2f}s"}
    return res


def per_config_lmhead(cfg, args, dev) -> list:
    """Chain verification from hidden states: the LM-head products of the target and draft
    models on the tensor cores with the top-k statistics in their epilogue, then the
    verification from those lists (spec_verify_chain_lmhead), at the configuration's top-k
    and at temperature 0. Timed with CUDA events around each call; the roofline counts the
    two products' FLOPs against the whole call."""
    import torch

    import draft_token_verification_spec_b200 as sv

    ht, hd, wt, wd = specgen.lmhead_inputs(cfg)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(
        torch.bfloat16)
    Ht, Hd, Wt, Wd = bf(ht), bf(hd), bf(wt), bf(wd)
    B, K, V, d = cfg.B, cfg.K, cfg.V, cfg.d
    # the drafter's tokens: x_i ~ its top-k distribution at temperature T (or its argmax),
    # from a plain bf16 product and torch sampling (input preparation, not timed)
    g = torch.Generator(device=dev)
    g.manual_seed(cfg.seed)
    ld = (Hd.reshape(-1, d) @ Wd.T).float()
    vals, idx = torch.topk(ld, cfg.top_k, dim=1)
    pick = torch.multinomial(torch.softmax(vals / cfg.temp, dim=1), 1, generator=g)
    x_s = idx.gather(1, pick).view(B, K).to(torch.int32)
    x_g = ld.argmax(dim=1).view(B, K).to(torch.int32)
    del ld, vals, idx
    u = torch.from_numpy(specgen.dyadic_uniforms(specgen.rng(cfg.seed, specgen.S_ACCEPT),
                                                 (B, K + 1))).to(dev)
    peaks, peak_src = measured_peaks()
    steps = max(3, min(args.steps, 20))
    out = []
    for temp, top_k, x in ((cfg.temp, cfg.top_k, x_s), (0.0, 0, x_g)):
        ws = torch.empty(sv.spec_lmhead_workspace_size(B, K, V, d, top_k), dtype=torch.uint8,
                         device=dev)
        acc = torch.empty(B, dtype=torch.int32, device=dev)
        toks = torch.empty((B, K + 1), dtype=torch.int32, device=dev)

        def call():
            sv.spec_verify_chain_lmhead(Ht, None if temp == 0 else Hd, Wt,
                                        None if temp == 0 else Wd, x, u, temp, top_k,
                                        accepted_len=acc, out_tokens=toks, workspace=ws)

        for _ in range(max(3, args.warmup)):
            call()
        torch.cuda.synchronize()
        ev = _events(steps)
        for i in range(steps):
            ev[i][0].record()
            call()
            ev[i][1].record()
        torch.cuda.synchronize()
        ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
        rows = B * (K + 1) + (0 if temp == 0 else B * K)
        flops = 2.0 * rows * V * d
        tf = flops / (ms / 1e3) / 1e12
        name = cfg.name if temp > 0 else cfg.name.replace(f"_T{cfg.temp:g}_topk{cfg.top_k}", "_T0")
        res = {"workload": name, "metric_unit": "positions/s",
               "value": B * K / (ms / 1e3), "ms_per_step": ms,
               "mean_accepted_len": float(acc.float().mean()),
               "roofline": {"bound": "tensor", "achieved": round(tf, 1),
                            "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                            "frac": round(tf / peaks["bf16_tflops"], 4),
                            "peak_source": peak_src + " (cuBLAS bf16 GEMM, burst)",
                            "kernel": "lmhead_topk_kernel (whole call timed)",
                            "kernel_ms": round(ms, 4), "algorithmic_flops": flops}}
        if not args.no_cpu_baseline and temp > 0:
            import oracle
            threads = os.cpu_count() or 1
            t0 = time.perf_counter()
            lt = oracle.lmhead_logits(ht[:1].reshape(-1, d), wt, threads=threads)
            lq = oracle.lmhead_logits(hd[:1].reshape(-1, d), wd, threads=threads)
            oracle.verify_chain(lt.reshape(1, K + 1, V), lq.reshape(1, K, V),
                                x[:1].cpu().numpy(), u[:1].cpu().numpy(),
                                float(np.float32(temp)), top_k)
            dt = time.perf_counter() - t0
            res["cpu_baseline"] = {"value": K / dt, "unit": "positions/s", "cores": threads,
                                   "kind": "oracle",
                                   "sample": f"1 of {B} sequences (double LM-head products "
                                             f"and verification), {threads} threads, "
                                             f"{dt:.1f}s"}
        out.append(res)
        del ws
    del Ht, Hd, Wt, Wd
    torch.cuda.empty_cache()
    return out


def per_config_all(args) -> list:
    """Every other workload, one entry each (1 GPU): the three other chain workloads, the
    temperature-0 variants of the two that have one, the MEDUSA tree, the linear-attention
    state commit, and verification from hidden states (LM head fused; sampling and
    temperature 0)."""
    import torch

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    out = []
    for cfg, greedy in [(specgen.CFG1, False), (specgen.CFG2, False), (specgen.CFG2, True),
                        (specgen.CFG3, False), (specgen.CFG5, True)]:
        out.append(per_config_chain(cfg, greedy, args, dev))
        log(f"per-config {out[-1]['workload']}: {out[-1]['ms_per_step']:.4f} ms")
    out.append(per_config_tree(specgen.CFG4, args, dev))
    out.append(per_config_lstate(specgen.LSTATE, args, dev))
    out.extend(per_config_lmhead(specgen.LMHEAD, args, dev))
    return out


def run_reference(args, cfg, greedy) -> dict:
    """The oracle, as it stands, on the host cores: each step verifies a bounded sample."""
    import oracle

    threads = os.cpu_count() or 1
    wave = time_oracle(cfg, greedy, threads, threads)  # one batch row per thread
    waves = int(150.0 / max(1, args.steps + args.warmup) / max(wave, 1e-4))
    per_step = min(cfg.B, threads * max(1, waves))
    target, draft = specgen.chain_logits(cfg, per_step)
    u = specgen.chain_uniforms(cfg, per_step)
    toks = oracle_drafts(cfg, target, draft, per_step, greedy)
    temp = 0.0 if greedy else cfg.temp

    def step():
        oracle.verify_chain(target, None if greedy else draft, toks, u, temp, cfg.top_k,
                            cfg.top_p, threads=threads)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = per_step * cfg.K * args.steps / dt
    sample = (f"first {per_step} of {cfg.B} batch rows per step ({per_step * cfg.K} positions), "
              f"{threads} threads over batch rows")
    return {"value": value, "ms_per_step": dt / args.steps * 1e3,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=5, choices=sorted(specgen.CHAIN_CONFIGS))
    ap.add_argument("--greedy", action="store_true", help="temperature-0 variant")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the batch size (smaller cases for profiler captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the headline workload")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"
    cfg = specgen.CHAIN_CONFIGS[args.config]
    if args.batch:
        cfg = dataclasses.replace(cfg, B=args.batch)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    base = {"metric": METRIC, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "data": "synthetic (seeded generator; no dataset)",
            "config": workload(cfg, args.greedy)}

    if args.impl == "reference":
        if rank != 0:
            return
        res = run_reference(args, cfg, args.greedy)
        print(json.dumps({**base, "impl": "reference", "dtype": "f64", **res}), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        res = run_ours(args, cfg, args.greedy, rank, world)
        if rank == 0:
            line = {**base, "dtype": "f32", "value": res.pop("value"),
                    "ms_per_step": res.pop("ms_per_step"), **res}
            if not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline(cfg, args.greedy)
            if world == 1 and not args.no_per_config and args.config == 5 and not args.greedy \
                    and not args.batch:
                line["per_config"] = per_config_all(args)
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
