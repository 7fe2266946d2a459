"""Benchmark of the hashed N-gram embedding forward on B200: one JSON line.

Headline workload: the full-scale layer, V0 = 131072, D = 4096, N = 5, K = 2 (8 sub-tables of
width 512, V_{n,k} ~ 7.27M primes: 59.6 GB of bf16 sub-tables + 1.07 GB E_0 + 33.5 MB W),
prefill of 8 sequences x 4096 Zipf(1.1) tokens. A step is one call of the C ABI's
ngram_embed_fwd over the whole batch (context + hash, gather, projection, E_0 add, scale),
inputs resident in HBM; the L2 is flushed (a 256 MB write) between timed steps, outside
the timed events.

The same line carries, as sub-objects: the other prefill workloads (D = 2048, N = 3, K = 2;
D = 4096, N = 5, K = 2 with varied lengths), each with its own roofline; speculative decode
(1000 steps of 256 sequences x 5 ids through the N-gram cache) on the full-scale layer and
on the D = 4096, N = 3, K = 4 layer; the backward pass (D = 2048 layer); the LayerNorm
amplification; the hash statistics sweep; and the fp64 CPU oracle's rate on the host cores.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

N > 1 (launched under torch.distributed.run): each rank runs its own batch of the same
size (data parallel, no collective on the data path), `value` = all ranks' tokens / the
slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import configs, gen, workloads  # noqa: E402

METRIC = "N-gram embed tokens/s (prefill & decode) + % of tensor/HBM roofline, 1 B200"
UNIT = "tokens/s"
WORKLOADS = {
    "full_scale_prefill": configs.FULL_SCALE,
    "prefill_d2048": configs.PREFILL_D2048,
    "prefill_varlen_d4096": configs.PREFILL_D4096_VARLEN,
    # small cases of the prefill kernel shapes for profiler captures: the same tokens and
    # layer widths over ~1-3.5 GB of tables (still far above the 126 MB L2)
    "profile_d2048": configs.PREFILL_D2048.with_(
        name="profile_bf16_D2048_N3_K2_small",
        V_nk=tuple(configs.primes_from(270000 + 131072 // 2, 4))),
    "profile_full_scale": configs.FULL_SCALE.with_(
        name="profile_full_scale_bf16_D4096_N5_K2_small",
        V_nk=tuple(configs.primes_from(300000 + 131072 // 2, 8))),
    # the backward's shapes (T = 32768, D = 2048) over ~100k-row sub-tables: with the fp32
    # gradient tables about 3 GB held, for multi-pass captures (--profile-backward)
    "profile_d2048_bwd": configs.PREFILL_D2048.with_(
        name="profile_bwd_bf16_D2048_N3_K2_small",
        V_nk=tuple(configs.primes_from(100000, 4))),
}
HEADLINE = "full_scale_prefill"
# the other prefill workloads, measured in the same run (each with its own roofline)
SUB_PREFILL = ("prefill_varlen_d4096", "prefill_d2048")
DECODE_WORKLOADS = {
    "full_scale_decode": configs.FULL_SCALE_DECODE,
    "spec_decode": configs.SPEC_DECODE,
    # small case of the spec_decode kernel shapes for profiler captures: 8 sub-tables of
    # ~300k rows (2.5 GB, still far above the 126 MB L2)
    "profile_decode": configs.SPEC_DECODE.with_(
        name="profile_spec_decode_bf16_D4096_N3_K4_small",
        V_nk=tuple(configs.primes_from(300000 + 131072 // 2, 8))),
}
L2_FLUSH_BYTES = 256 << 20
TRAFFIC_RECORDS = os.path.join("profiles", "traffic_records.json")


# the projection kernels' device code, stage counts and tile shapes
PROJECTION_SOURCES = ("common.cuh", "proj_sm100.cuh", "proj_sm100_pair.cuh")


def code_only(text: str) -> str:
    """C++ source with its comments and blank lines removed and trailing spaces cut: what
    the compiler sees of it (these sources hold no comment markers inside string literals)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip())


def kernel_source_hash(read=None) -> str:
    """sha256 over the projection kernels' sources, comments removed: a profile's counters
    describe the kernels of the code they were taken from, and only those. `read(name)`
    returns a source's text (default: the working tree)."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "hashed_gram_embedding_horner_b200", "csrc")
    for name in PROJECTION_SOURCES:
        text = read(name) if read else open(os.path.join(csrc, name), encoding="utf-8").read()
        h.update(name.encode())
        h.update(code_only(text).encode())
    return h.hexdigest()


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of `kernel` at
    `workload`, from the committed record of ncu captures, if it was taken from these
    sources; else None. A record taken on a smaller case of the same kernel shape carries
    the factor that scales it to one launch of `workload` (the units the launches process)."""
    path = os.path.join(ROOT, TRAFFIC_RECORDS)
    if not os.path.exists(path):
        return None
    try:
        records = json.load(open(path))["records"]
    except (ValueError, KeyError):
        return None
    src = kernel_source_hash()
    for rec in records:
        if rec.get("kernel") == kernel and rec.get("workload") == workload and rec.get("source_sha256") == src:
            return float(rec["bytes_per_launch"]) * float(rec.get("scale_to_workload", 1.0))
    return None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples, each stamped with the host time it
    arrived, so that a summary covers only a window in which the GPU was busy."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.samples = []  # (host time, line)
        self.marks = {}

    def _read(self):
        for ln in self.proc.stdout:
            if ln.strip():
                self.samples.append((time.time(), ln))

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def mark(self, name):
        self.marks[name] = time.time()

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
            self.reader.join(timeout=5)

    def summary(self, start="load_start", end="load_end"):
        """Median SM clock over the samples taken between the two marks (the whole run if
        either is missing), the throttle reasons seen then or in the timed region."""
        t0, t1 = self.marks.get(start), self.marks.get(end)
        r0, r1 = self.marks.get("timed_start"), self.marks.get("timed_end")
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, ln in self.samples:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            in_load = t0 is None or t1 is None or t0 <= ts <= t1
            in_timed = r0 is not None and r1 is not None and r0 <= ts <= r1
            if not (in_load or in_timed):
                continue
            try:
                clk = float(f[1])
                mx = float(f[2])
            except ValueError:
                continue
            if in_load:
                sm.append(clk)
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        out = {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
               "samples": len(sm)}
        if t0 is not None and t1 is not None:
            out["window_s"] = round(t1 - t0, 3)
            out["what"] = ("median of the samples taken while the timed step ran again back to back for a "
                           "second after the timed measurements (those alone are shorter than the sampling "
                           "interval); reasons from both")
        return out


def rank_config(cfg, rank: int):
    """Rank r's batch under data parallelism: the same shape and tables, its own token
    stream (rank 0 runs the configured workload)."""
    return cfg if rank == 0 else cfg.with_(seed=cfg.seed + 7919 * rank)


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's number (device times are reduced with MAX over ranks)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def tokens_per_step(cfg) -> int:
    return cfg.num_seqs * cfg.seq_len if cfg.seq_len else cfg.extras.get("total_tokens")


# ------------------------------------------------------------------ reference arm: the oracle

class OracleSampler:
    """Times the fp64 CPU oracle (exact hash + Eq. 3 combine) on bounded samples of a
    prefill workload's tokens; the table rows a sample reads are regenerated beforehand,
    outside the timed part."""

    def __init__(self, cfg):
        import oracle
        from synth.tables import host_W
        self.oracle, self.cfg = oracle, cfg
        self.tokens, self.offsets = workloads.prefill_tokens(cfg)
        self.windows = oracle.context_windows(cfg.N, self.tokens, self.offsets)
        self.W = host_W(cfg)
        self.rng = np.random.default_rng(0)

    def run(self, n: int) -> float:
        """Seconds of oracle work for n sampled tokens (hash + combine)."""
        from synth.tables import host_rows
        cfg, o = self.cfg, self.oracle
        rows = np.sort(self.rng.choice(len(self.tokens), size=n, replace=False))
        win = self.windows[rows]
        t0 = time.perf_counter()
        idx = o.hash_indices(cfg.V0, cfg.N, cfg.K, cfg.V_nk, win)
        t_hash = time.perf_counter() - t0
        e0 = host_rows(cfg, gen.TAG_E0, self.tokens[rows], cfg.D, cfg.e_std)
        sub = np.stack([host_rows(cfg, gen.TAG_SUBTABLE0 + s, idx[:, s], cfg.d, cfg.e_std) for s in range(cfg.S)], 1)
        t1 = time.perf_counter()
        o.combine(cfg.D, cfg.S, e0, sub, self.W)
        return t_hash + time.perf_counter() - t1

    def size_for(self, budget_s: float, max_tokens: int) -> int:
        """Tokens that take about `budget_s` of oracle time (from a short calibration run)."""
        n = max(self.oracle.num_threads(), 8)
        dt = self.run(n)
        return int(min(max_tokens, max(n, n * budget_s / max(dt, 1e-6) * 0.8)))


def oracle_sample_rate(cfg, budget_s: float = 15.0, max_tokens: int = 32768):
    """The oracle's tokens/s on one bounded sample of the workload (the cpu_baseline)."""
    s = OracleSampler(cfg)
    n = s.size_for(budget_s, max_tokens)
    dt = s.run(n)
    return {"value": n / dt, "unit": UNIT, "cores": s.oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} tokens sampled from the workload (exact hash + fp64 Eq. 3), {dt:.1f} s"}


def run_reference(args, cfg):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    s = OracleSampler(cfg)
    n = s.size_for(args.ref_step_seconds, 2048)
    times = []
    for i in range(args.warmup + args.steps):
        dt = s.run(n)
        if i >= args.warmup:
            times.append(dt)
    sec = float(np.mean(times))
    value = n / sec
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        # each step is one timed sample of `sample_tokens_per_step` tokens of the workload
        "ms_per_step": 1e3 * sec, "sample_tokens_per_step": n,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_block(cfg, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": s.oracle.num_threads(), "kind": "oracle",
                         "sample": f"{n} tokens sampled from the workload per step (exact hash + fp64 Eq. 3), "
                                   f"{sec:.2f} s per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_block(cfg, args):
    return {"workload": cfg.name, "V0": cfg.V0, "D": cfg.D, "N": cfg.N, "K": cfg.K, "V_nk": list(cfg.V_nk),
            "tokens_per_step": tokens_per_step(cfg), "num_seqs": cfg.num_seqs, "token_dist": f"zipf({cfg.zipf_alpha})",
            "tables_gb": round(cfg.table_bytes() / 1e9, 2), "parallelism": f"dp{args.gpus}",
            "l2": "flushed between timed steps (256 MB write)"}


def events(n):
    import torch
    return [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]


def kernel_of_form(form: str) -> str:
    if form.startswith("cta_pair_columns"):
        return "proj_sm100_cols_kernel"
    if form.startswith("cta_pair"):
        return "proj_sm100_pair_kernel"
    return {"one_cta": "proj_sm100_kernel", "one_cta_stream_k": "proj_sm100_kernel",
            "cuda_cores": "proj_simt_kernel"}[form]


# ------------------------------------------------------------------ prefill

def run_prefill(ne, cfg, tables, args, dev, flush, world, rank, clock_gpu=None, e2e=True):
    """Time `args.steps` whole-layer steps of a prefill workload (L2 flushed between steps),
    then its dominant kernel alone (the projection) and the hash, and, if `e2e`, the same
    call with host buffers (H2D of the inputs and D2H of the output inside the timed region).
    Returns (result dict, output tensor, workspace, plan)."""
    import torch
    E0, E, W = tables
    stream = torch.cuda.current_stream()
    tokens_h, offsets_h = workloads.prefill_tokens(rank_config(cfg, rank))
    T = len(tokens_h)
    tokens = torch.from_numpy(tokens_h).to(dev)
    offsets = torch.from_numpy(offsets_h).to(dev)
    plan = ne.ngram_embed_plan_create(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, ne.NGRAM_BF16)
    ws = ne.new_workspace(plan, T)
    out = torch.empty((T, cfg.D), dtype=torch.bfloat16, device=dev)

    def step():
        ne.ngram_embed_fwd(plan, tokens, offsets, E0, E, W, out, ws, stream=stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if ne.ngram_embed_get_status(ws) != 0:
        raise RuntimeError(f"device status {ne.status_names(ne.ngram_embed_get_status(ws))}")

    clk = ClockSampler(clock_gpu) if clock_gpu is not None else None
    if clk:
        clk.__enter__()
    ev = events(args.steps)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    if clk:
        clk.mark("timed_start")
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    total_ms = float(np.sum([a.elapsed_time(b) for a, b in ev]))
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / args.steps

    # the dominant kernel alone: the projection (gather + tcgen05 GEMM + epilogue) from
    # precomputed indices; and the hash alone. CUDA events on the launching stream.
    idx = torch.empty((T, cfg.S), dtype=torch.int32, device=dev)
    ne.ngram_hash_indices(plan, tokens, offsets, idx, ws, stream=stream)
    pe, hs = events(args.steps), events(args.steps)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        hs[i][0].record(stream)
        ne.ngram_hash_indices(plan, tokens, offsets, idx, ws, stream=stream)
        hs[i][1].record(stream)
        flush.fill_((i + 1) & 0xFF)
        pe[i][0].record(stream)
        ne.ngram_embed_project(plan, tokens, idx, E0, E, W, out, ws, stream=stream)
        pe[i][1].record(stream)
    torch.cuda.synchronize()
    if clk:
        clk.mark("timed_end")
        # the clock under this load, after every timed number: the same step back to back
        # for about a second (the timed steps alone are shorter than the sampling interval)
        clk.mark("load_start")
        t_end = time.time() + 1.0
        while time.time() < t_end:
            for _ in range(8):
                step()
            torch.cuda.synchronize()
        clk.mark("load_end")
        clk.__exit__(None, None, None)
    proj_ms = float(np.mean([a.elapsed_time(b) for a, b in pe]))
    hash_ms = float(np.mean([a.elapsed_time(b) for a, b in hs]))
    pk = peaks()
    flops = 2.0 * T * cfg.D * cfg.D
    achieved = flops / (proj_ms / 1e3) / 1e12
    form = ne.ngram_embed_plan_kernel_form(plan, T)
    kernel = kernel_of_form(form)
    algo_bytes = T * (2 * cfg.D * 2 + 4) + cfg.D * cfg.D * 2
    res = {
        "workload": cfg.name, "tokens_per_step": T, "steps": args.steps, "ms_per_step": ms_per_step,
        "value": world * T / (ms_per_step / 1e3), "unit": UNIT, "tables_gb": round(cfg.table_bytes() / 1e9, 2),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / pk["bf16_tflops"], "traffic": profiled_traffic(kernel, cfg.name),
                     "kernel": kernel + " (" + form + "): fused sub-row gather + tcgen05 projection + E_0 add + scale",
                     "kernel_ms": proj_ms, "peak_source": pk["source"] + " (burst)",
                     "layer_frac": (flops / (ms_per_step / 1e3) / 1e12) / pk["bf16_tflops"],
                     "hash_kernel_ms": hash_ms, "flops_per_launch": flops, "algorithmic_bytes": algo_bytes},
    }
    if clk:
        res["clocks"] = clk.summary()
    if e2e:
        # end to end through the C ABI with host buffers: H2D inputs, fwd, D2H output
        tok_pin = torch.from_numpy(tokens_h).pin_memory()
        off_pin = torch.from_numpy(offsets_h).pin_memory()
        out_pin = torch.empty((T, cfg.D), dtype=torch.bfloat16).pin_memory()
        tok_d, off_d = torch.empty_like(tokens), torch.empty_like(offsets)
        ee = events(args.steps)
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            ee[i][0].record(stream)
            tok_d.copy_(tok_pin, non_blocking=True)
            off_d.copy_(off_pin, non_blocking=True)
            ne.ngram_embed_fwd(plan, tok_d, off_d, E0, E, W, out, ws, stream=stream)
            out_pin.copy_(out, non_blocking=True)
            ee[i][1].record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in ee])), world, dev)
        res["e2e"] = {"value": world * T / (e2e_ms / 1e3), "unit": UNIT,
                      "h2d_bytes_per_step": tokens.numel() * 4 + offsets.numel() * 4,
                      "d2h_bytes_per_step": out.numel() * 2}
    res["device_status"] = ne.ngram_embed_get_status(ws)
    return res, out, ws, plan, (tokens, idx)


def run_layernorm(ne, plan, out, ws, args, flush):
    """Embedding amplification by LayerNorm over the layer output (HBM-bound: the output read
    once from HBM, written once), in place, L2 flushed before each launch."""
    import torch
    stream = torch.cuda.current_stream()
    ln_ev = events(args.steps)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        ln_ev[i][0].record(stream)
        ne.ngram_embed_layernorm(plan, out, out, ws, eps=1e-5, stream=stream)
        ln_ev[i][1].record(stream)
    torch.cuda.synchronize()
    ln_ms = float(np.mean([a.elapsed_time(b) for a, b in ln_ev]))
    ln_bytes = 2 * out.numel() * out.element_size()
    pk = peaks()
    return {"layernorm_ms": ln_ms, "bytes": ln_bytes, "gbs": ln_bytes / (ln_ms / 1e3) / 1e9,
            "frac_hbm": ln_bytes / (ln_ms / 1e3) / 1e9 / pk["hbm_gbs"], "tokens": out.shape[0], "D": out.shape[1]}


# ------------------------------------------------------------------ decode (speculative, ring cache)

def run_decode(ne, cfg, tables, steps: int, warmup: int, dev, rank: int = 0, extras: bool = True):
    """Speculative decode: per step, every sequence brings 5 ids (x0 + 4 drafts); the layer
    reads each sequence's context from the N-gram cache ring, then the accepted prefix
    (1 + a ids, a ~ U{0..4}) is committed. `steps` steps are captured in one CUDA graph and
    replayed; the L2 is not flushed between steps (steady state: W stays L2-resident, the
    tens of GB of sub-tables do not)."""
    import torch
    E0, E, W = tables
    ds = workloads.DecodeStream(rank_config(cfg, rank))  # this rank's streams; tables shared
    B, P, C = ds.B, ds.P, cfg.ring_capacity
    T = B * P
    plan = ne.ngram_embed_plan_create(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, ne.NGRAM_BF16)
    ws = ne.new_workspace(plan, T)
    cache = ne.Cache.empty(B, C, device=dev)
    ne.ngram_cache_reset(plan, cache, ws)
    dev_i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
    ids, poff = ds.prompts()
    for start in range(0, cfg.prompt_max + 1, C):
        chunk = [ids[poff[b] + start: min(poff[b + 1], poff[b] + start + C)] for b in range(B)]
        off = gen.offsets_from_lengths([len(c) for c in chunk])
        flat = np.concatenate(chunk).astype(np.int32) if off[-1] else np.zeros(1, np.int32)
        ne.ngram_cache_append(plan, cache, dev_i32(flat), dev_i32(off), ws)
    n_total = warmup + 2 * steps
    tok_all = dev_i32(np.stack([ds.step_tokens(i) for i in range(n_total)]))
    cnt_all = dev_i32(np.stack([1 + ds.accept_lengths(i) for i in range(n_total)]))
    offsets = dev_i32(ds.step_offsets())
    out = torch.empty((T, cfg.D), dtype=torch.bfloat16, device=dev)

    def step(i, stream):
        # commit the previous step's accepted ids (fused with this step's hashing), then the layer
        ne.ngram_embed_fwd_step(plan, tok_all[i], offsets, E0, E, W, out, ws, cache,
                                commit_tokens=tok_all[i - 1] if i > 0 else None, commit_stride=P,
                                commit_counts=cnt_all[i - 1] if i > 0 else None, stream=stream)

    cur = torch.cuda.current_stream()
    for i in range(warmup):
        step(i, cur)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    graphs = []
    for rep in range(2):  # two graphs: one warm-up replay, one timed
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for i in range(warmup + rep * steps, warmup + (rep + 1) * steps):
                step(i, s)
        graphs.append(g)
    torch.cuda.synchronize()
    graphs[0].replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        a.record(s)
        graphs[1].replay()
        b.record(s)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    status = ne.ngram_embed_get_status(ws)
    del graphs
    pk = peaks()
    flops = 2.0 * T * cfg.D * cfg.D
    form = ne.ngram_embed_plan_kernel_form(plan, T)
    dense = "dense" in form
    res = {
        "workload": cfg.name, "steps": steps, "tokens_per_step": T, "ms_per_step": ms / steps,
        "value": steps * T / (ms / 1e3), "unit": UNIT, "graph": True,
        # commit + hash (+ the dense-A forms' sub-row gather into G) in one launch, the projection
        "gpu_launches_per_step": 2,
        "layer_tflops": flops / (ms / steps / 1e3) / 1e12,
        "layer_frac": flops / (ms / steps / 1e3) / 1e12 / pk["bf16_tflops"],
        "kernel_form": form,
    }
    if not extras:
        res["device_status"] = status
        return res
    # The projection alone at this shape, and the stand-alone hash and gather stages. Each is
    # timed as `n` launches on `n` different steps' inputs captured in one CUDA graph (so
    # host launch overhead is not in the number and the sub-rows are not L2 hits from the
    # launch before), averaged over the replay.
    n_k = min(20, n_total)
    idx_all = torch.empty((n_k, T, cfg.S), dtype=torch.int32, device=dev)
    for i in range(n_k):
        ne.ngram_hash_indices(plan, tok_all[i], offsets, idx_all[i], ws, cache=cache)
    G = torch.empty((T, cfg.D), dtype=torch.bfloat16, device=dev)

    def timed(fn):
        gs = torch.cuda.Stream()
        gs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(gs):
            for i in range(3):
                fn(i, gs)
        torch.cuda.current_stream().wait_stream(gs)
        gg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gg, stream=gs):
            for i in range(n_k):
                fn(i, gs)
        torch.cuda.synchronize()
        gg.replay()
        torch.cuda.synchronize()
        res_ms = []
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(gs):
                e0.record(gs)
                gg.replay()
                e1.record(gs)
            torch.cuda.synchronize()
            res_ms.append(e0.elapsed_time(e1) / n_k)
        del gg
        return float(np.median(res_ms))

    proj_ms = timed(lambda i, st: ne.ngram_embed_project(plan, tok_all[i], idx_all[i], E0, E, W, out, ws, stream=st))
    hash_ms = timed(lambda i, st: ne.ngram_hash_indices(plan, tok_all[i], offsets, idx_all[n_k - 1 - i], ws,
                                                        cache=cache, stream=st))
    # the step's table lookups as the dense-A form runs them: its 8 sub-rows per token (8 KiB)
    # copied from the sub-tables into G (written back, 8 KiB); the E_0 rows are read by the
    # projection's epilogue
    gather_ms = timed(lambda i, st: ne.ngram_embed_gather(plan, idx_all[i], E, G, ws, stream=st))
    gather_bytes = T * cfg.S * cfg.d * 2 * 2  # rows read + rows written
    # Draft-phase embedding cache: a verify call whose 5 in-step embeddings were all
    # computed while drafting (all hits), and the last draft call of a step (4 hits and the
    # new draft's miss per sequence), against the plain forward of the same 1280 tokens.
    dc = ne.DraftCache.empty(plan, B, P, device=dev)
    ne.ngram_draft_cache_reset(plan, dc, ws)
    dws = ne.new_draft_workspace(plan, T, device=dev)
    tok_v = tok_all[0]
    tok_alt = tok_all[0].clone().view(B, P)
    tok_alt[:, P - 1] = (tok_alt[:, P - 1] + 1) % cfg.V0
    tok_alt = tok_alt.view(-1)
    ne.ngram_embed_fwd_draft(plan, tok_v, offsets, E0, E, W, out, dws, cache, dc)
    hits_d = torch.zeros(1, dtype=torch.int32, device=dev)
    verify_ms = timed(lambda i, st: ne.ngram_embed_fwd_draft(plan, tok_v, offsets, E0, E, W, out, dws, cache, dc,
                                                             hits=hits_d, stream=st))
    alt = [tok_v, tok_alt]
    draft_ms = timed(lambda i, st: ne.ngram_embed_fwd_draft(plan, alt[i & 1], offsets, E0, E, W, out, dws, cache, dc,
                                                            stream=st))
    plain_ms = timed(lambda i, st: ne.ngram_embed_fwd(plan, tok_all[i], offsets, E0, E, W, out, ws, cache=cache,
                                                      stream=st))
    hit_rate = hits_d.item() / (T * (3 + 4 * n_k))  # timed(): 3 eager calls, then 1 + 3 replays of n_k
    kernel = kernel_of_form(form)
    traffic = profiled_traffic(kernel, cfg.name)
    res.update({
        "projection": {"ms": proj_ms, "tflops": flops / (proj_ms / 1e3) / 1e12,
                       "frac": flops / (proj_ms / 1e3) / 1e12 / pk["bf16_tflops"],
                       "what": "ngram_embed_project: " + ("sub-row gather into G + dense-A tcgen05 projection"
                                                          if dense else "fused row gather + tcgen05 projection")},
        # the step's dominant kernel against both rooflines: its FLOPs at the bf16 peak, and the
        # DRAM bytes an ncu capture of it moved (one launch at this shape) over its time here
        "roofline": {"bound": "tensor", "kernel": kernel + " (" + form + ")", "kernel_ms": proj_ms,
                     "achieved": flops / (proj_ms / 1e3) / 1e12, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": flops / (proj_ms / 1e3) / 1e12 / pk["bf16_tflops"], "traffic": traffic,
                     "dram_gbs": None if traffic is None else traffic / (proj_ms / 1e3) / 1e9,
                     "dram_frac_hbm": None if traffic is None else traffic / (proj_ms / 1e3) / 1e9 / pk["hbm_gbs"],
                     "algorithmic_bytes": T * (2 * cfg.D * 2 + 4) + cfg.D * cfg.D * 2},
        "hash_ms": hash_ms,
        "gather_stage": {
            "what": ("gather_kernel, as the step runs it: the sub-rows copied into G" if dense else
                     "gather_kernel alone (the sub-rows copied into G); not a kernel of this step, whose "
                     "projection gathers its rows itself"),
            "ms": gather_ms, "bytes": gather_bytes, "gbs": gather_bytes / (gather_ms / 1e3) / 1e9,
            "frac_hbm": gather_bytes / (gather_ms / 1e3) / 1e9 / pk["hbm_gbs"]},
        "draft_cache": {"verify_all_hits_ms": verify_ms, "draft_step_4_of_5_hits_ms": draft_ms,
                        "plain_forward_ms": plain_ms, "verify_hit_rate": hit_rate},
        "device_status": status,
    })
    return res


def tables_for(cfg, held):
    """The device tables of `cfg`: the ones already held when they are identical, else freshly
    filled ones (the held ones are released first)."""
    import torch
    from synth.tables import device_tables
    if held[0] is not None and configs.same_tables(held[0], cfg):
        return held[1]
    held[0] = held[1] = None
    torch.cuda.empty_cache()
    t = device_tables(cfg)
    held[0], held[1] = cfg, t
    return t


# ------------------------------------------------------------------ our arm

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-step-seconds", type=float, default=4.0)
    ap.add_argument("--no-decode", action="store_true", help="skip the speculative-decode measurements")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward (training) measurement")
    ap.add_argument("--no-stats", action="store_true", help="skip the hash-statistics sweep")
    ap.add_argument("--no-sub", action="store_true", help="skip the other prefill workloads")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--decode-workload", default=None, choices=sorted(DECODE_WORKLOADS),
                    help="with --decode-only: the one decode workload to run")
    ap.add_argument("--decode-only", action="store_true",
                    help="only the speculative-decode measurement (one JSON line with the decode object)")
    ap.add_argument("--profile-backward", action="store_true",
                    help="with --profile-only: also run the backward (all three gradients) as many times")
    ap.add_argument("--profile-only", action="store_true",
                    help="warm up, run --steps forward calls back to back and exit (for profiler captures)")
    args = ap.parse_args()
    cfg = WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, cfg)
        return

    import torch
    import torch.distributed as dist

    import hashed_gram_embedding_horner_b200 as ne
    from synth.tables import device_tables

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    held = [None, None]  # (config, tables) currently on the device

    if args.decode_only:
        names = [args.decode_workload] if args.decode_workload else ["full_scale_decode", "spec_decode"]
        dec = {}
        for name in names:
            dcfg = DECODE_WORKLOADS[name]
            d = run_decode(ne, dcfg, tables_for(dcfg, held), args.decode_steps, max(args.warmup, 3), dev, rank=rank)
            d["ms_per_step"] = max_over_ranks(d["ms_per_step"], world, dev)
            d["value"] = world * d["tokens_per_step"] / (d["ms_per_step"] / 1e3)
            dec[dcfg.name] = d
        if rank == 0:
            print(json.dumps({"decode_only": True, "decode": dec}), flush=True)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return

    if args.profile_only:
        E0, E, W = device_tables(cfg)
        tokens_h, offsets_h = workloads.prefill_tokens(cfg)
        tokens, offsets = torch.from_numpy(tokens_h).to(dev), torch.from_numpy(offsets_h).to(dev)
        plan = ne.ngram_embed_plan_create(cfg.V0, cfg.D, cfg.N, cfg.K, cfg.V_nk, ne.NGRAM_BF16)
        ws = ne.new_workspace(plan, len(tokens_h))
        out = torch.empty((len(tokens_h), cfg.D), dtype=torch.bfloat16, device=dev)
        for _ in range(max(args.warmup, 3) + args.steps):
            ne.ngram_embed_fwd(plan, tokens, offsets, E0, E, W, out, ws, stream=stream)
        torch.cuda.synchronize()
        bwd_status = None
        if args.profile_backward:
            T = len(tokens_h)
            idx = torch.empty((T, cfg.S), dtype=torch.int32, device=dev)
            ne.ngram_hash_indices(plan, tokens, offsets, idx, ws, stream=stream)
            del out, E0
            g_out = (torch.randn((T, cfg.D), device=dev) * 0.01).to(torch.bfloat16)
            dE = [torch.zeros((v, cfg.d), dtype=torch.float32, device=dev) for v in cfg.V_nk]
            dW = torch.zeros((cfg.D, cfg.D), dtype=torch.float32, device=dev)
            dE0 = torch.zeros((cfg.V0, cfg.D), dtype=torch.float32, device=dev)
            bws = ne.new_bwd_workspace(plan, T, device=dev)
            for _ in range(max(args.warmup, 3) + args.steps):
                ne.ngram_embed_bwd(plan, tokens, idx, g_out, bws, E_nk=E, W_stacked=W, dE0=dE0, dE_nk=dE, dW=dW,
                                   stream=stream)
            torch.cuda.synchronize()
            bwd_status = ne.ngram_embed_get_status(bws)
        print(json.dumps({"profile_only": cfg.name, "steps": args.steps,
                          "status": ne.ngram_embed_get_status(ws), "backward_status": bwd_status}), flush=True)
        return

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    # --- the headline workload: the whole layer, its dominant kernel, end to end, LayerNorm
    head, out, ws, plan, _ = run_prefill(ne, cfg, tables_for(cfg, held), args, dev, flush, world, rank,
                                         clock_gpu=local)
    amplification = run_layernorm(ne, plan, out, ws, args, flush)
    del out, ws

    # --- speculative decode: the headline layer's decode half first (its tables are held)
    decode = None
    if not args.no_decode:
        decode = {}
        for name in ("full_scale_decode", "spec_decode"):
            dcfg = DECODE_WORKLOADS[name]
            d = run_decode(ne, dcfg, tables_for(dcfg, held), args.decode_steps, max(args.warmup, 3), dev, rank=rank)
            d["ms_per_step"] = max_over_ranks(d["ms_per_step"], world, dev)
            d["value"] = world * d["tokens_per_step"] / (d["ms_per_step"] / 1e3)
            decode[dcfg.name] = d

    # --- the other prefill workloads, each with its own roofline (the varlen D = 4096 layer
    # draws the same tables as the spec-decode layer above, so they are not filled again)
    sub = {}
    backward = None
    if not args.no_sub:
        for name in SUB_PREFILL:
            scfg = WORKLOADS[name]
            r, sout, sws, splan, (stok, sidx) = run_prefill(ne, scfg, tables_for(scfg, held), args, dev, flush,
                                                            world, rank, e2e=False)
            sub[scfg.name] = r
            del sout, sws
            if name == "prefill_d2048" and not args.no_backward:
                backward = run_backward(ne, scfg, held[1], splan, stok, sidx, args, dev, flush)
    held[0] = held[1] = None
    torch.cuda.empty_cache()

    # --- hash statistics (section 3.2.2, Fig. 3b): collisions of the 2-gram hash for table
    # sizes swept over [30, 33] V0 (denser next to the multiples of V0), on 100 Zipf
    # sequences of 4096 tokens
    stats = None
    if not args.no_stats and rank == 0:
        stats = run_hash_stats(ne, cfg, dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample_rate(cfg)

    if rank == 0:
        line = {
            "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_block(cfg, argparse.Namespace(gpus=world)),
            "roofline": head["roofline"],
            "cpu_baseline": cpu,
            "e2e": head["e2e"],
            "gpu_launches": 2 * args.steps,
            "prefill_other_workloads": sub,
            "decode": decode,
            "backward": backward,
            "hash_stats": stats,
            "amplification": amplification,
            "clocks": head.get("clocks"),
            "device_status": head["device_status"],
            "impl": "ours",
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_backward(ne, cfg, tables, plan, tokens, idx, args, dev, flush):
    """Parameter gradients for a random bf16 dL/de, fp32 gradient tables accumulated in
    place; two tcgen05 GEMMs of 2 T D^2 FLOPs each dominate."""
    import torch
    E0, E, W = tables
    stream = torch.cuda.current_stream()
    T = tokens.numel()
    g_out = (torch.randn((T, cfg.D), device=dev) * 0.01).to(torch.bfloat16)
    dE0 = torch.zeros((cfg.V0, cfg.D), dtype=torch.float32, device=dev)
    dE = [torch.zeros((v, cfg.d), dtype=torch.float32, device=dev) for v in cfg.V_nk]
    dW = torch.zeros((cfg.D, cfg.D), dtype=torch.float32, device=dev)
    bws = ne.new_bwd_workspace(plan, T, device=dev)
    bwd = lambda: ne.ngram_embed_bwd(plan, tokens, idx, g_out, bws, E_nk=E, W_stacked=W, dE0=dE0, dE_nk=dE,
                                     dW=dW, stream=stream)
    for _ in range(2):
        bwd()
    torch.cuda.synchronize()
    bw_ev = events(max(3, args.steps // 4))
    for i, (e0, e1) in enumerate(bw_ev):
        flush.fill_(i & 0xFF)
        e0.record(stream)
        bwd()
        e1.record(stream)
    torch.cuda.synchronize()
    bw_ms = float(np.mean([a.elapsed_time(b) for a, b in bw_ev]))
    bw_flops = 4.0 * T * cfg.D * cfg.D
    pk = peaks()
    res = {"workload": cfg.name, "ms": bw_ms, "tokens_per_s": T / (bw_ms / 1e3),
           "tflops": bw_flops / (bw_ms / 1e3) / 1e12, "frac": bw_flops / (bw_ms / 1e3) / 1e12 / pk["bf16_tflops"],
           "device_status": ne.ngram_embed_get_status(bws)}
    del g_out, dE0, dE, dW, bws
    torch.cuda.empty_cache()
    return res


def run_hash_stats(ne, cfg, dev):
    import torch
    stream = torch.cuda.current_stream()
    V0 = cfg.V0
    s_tok = torch.from_numpy(gen.zipf_tokens(cfg.seed + 99, 100 * 4096, V0).astype(np.int32)).to(dev)
    s_off = torch.from_numpy(gen.offsets_from_lengths([4096] * 100)).to(dev)
    moduli = sorted({int(V0 * (30 + k * 0.05)) for k in range(61)} |
                    {m * V0 + dd for m in (30, 31, 32, 33) for dd in (-3, -1, 1, 3)})
    ne.ngram_hash_stats(V0, 2, s_tok, s_off, moduli[:2])  # warm-up
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    distinct, rows = ne.ngram_hash_stats(V0, 2, s_tok, s_off, moduli, stream=stream)
    t1.record(stream)
    torch.cuda.synchronize()
    st_ms = t0.elapsed_time(t1)
    coll = np.array([distinct - r for r in rows])
    near = np.array([min(abs(v - m * V0) for m in (30, 31, 32, 33)) <= 3 for v in moduli])
    return {"ms": st_ms, "windows": int(s_tok.numel()), "moduli": len(moduli),
            "windows_per_s": s_tok.numel() * len(moduli) / (st_ms / 1e3), "distinct_2grams": distinct,
            "collisions_near_multiples_median": float(np.median(coll[near])),
            "collisions_elsewhere_median": float(np.median(coll[~near]))}


if __name__ == "__main__":
    main()
