"""Benchmark of the attention hot path on B200.

One step = one causal GQA prefill (B=2, Hq=32, Hkv=8, S=8192, D=128, the shape of
a Llama-3-8B / Mistral layer) followed by one paged GQA decode (64 sequences,
lengths uniform in [512, 8192], Hq=32, Hkv=8, D=128, 16-token pages from a
shared pool in random order). Inputs are seeded synthetic bf16 N(0, 1) data
resident in HBM. L2 is flushed before every timed step (a 256 MiB write, then a 256 MiB read of
another buffer, so that no dirty line of the flush is written back inside the timed region).
Kernels are timed with CUDA events on the launching stream.

value = prefill TFLOP/s (algorithmic FLOPs: 4*D per visible (query, key) pair,
causal diagonal counted exactly); the decode's KV-read GB/s is reported beside
it. With --gpus N under torchrun every rank runs its own copy of the workload
(independent problems, weak scaling); times are the max over ranks.

--impl reference times the float64 CPU oracle (test infrastructure) on a
bounded sample of the same workload, on rank 0 only.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from attention_online_softmax_fwd_b200 import inputs as gen  # noqa: E402

METRIC = "prefill attn TFLOPS & paged-decode KV-read GB/s, % of B200 roofline"
PREFILL_CFG = "gqa_prefill_llama3_8b"
DECODE_CFG = "paged_gqa_decode"
DECODE_SPLIT = 256
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


def prefill_flops(B, Hq, S, D, causal=True):
    pairs = S * (S + 1) // 2 if causal else S * S
    return 4.0 * D * B * Hq * pairs


def decode_bytes(seq_lens, Hq, Hkv, D, max_pages, kv_elem_bytes=2):
    """Algorithmic bytes: every cached K and V row once, plus q, o, lse, tables."""
    toks = int(sum(seq_lens))
    n = len(seq_lens)
    kv = toks * Hkv * D * kv_elem_bytes * 2
    return kv + n * Hq * D * 2 * 2 + n * Hq * 4 + n * max_pages * 4 + n * 4


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_profile_traffic():
    """Per-launch DRAM bytes of the prefill and decode kernels from the committed ncu summary."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f)
    return {}


def physical_gpu_id(local):
    """The nvidia-smi --id of CUDA device ``local``: its UUID when torch reports one
    (right under any CUDA_VISIBLE_DEVICES mapping), else the entry of
    CUDA_VISIBLE_DEVICES, else the index itself."""
    try:
        uuid = str(torch.cuda.get_device_properties(local).uuid)
        if uuid and uuid != "None":
            return uuid if uuid.startswith(("GPU-", "MIG-")) else "GPU-" + uuid
    except (AttributeError, RuntimeError, AssertionError):
        pass
    visible = [x.strip() for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
    if local < len(visible):
        return visible[local]
    return str(local)


class ClockSampler:
    """nvidia-smi clocks/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, fallback=None):
        self.index = index
        self.fallback = fallback
        self.proc = None
        self.lines = []

    def _spawn(self, gpu_id):
        return subprocess.Popen(
            ["nvidia-smi", f"--id={gpu_id}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader", "-lms", "100"],
            stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)

    def start(self):
        try:
            self.proc = self._spawn(self.index)
            time.sleep(0.2)
            if self.proc.poll() is not None and self.fallback is not None:   # id not accepted
                self.index = self.fallback
                self.proc = self._spawn(self.index)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1].split()[0]))
                smax.append(float(parts[2].split()[0]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm), "gpu": str(self.index)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def dist_max(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------- CPU oracle timing

def oracle_sample(n_prefill_heads=2, n_decode_seqs=4, seed_shift=0):
    """Time the float64 oracle on a bounded sample of the workload.

    Prefill: ``n_prefill_heads`` (b, hq) heads of the GQA config, all 8192 query
    rows each. Decode: ``n_decode_seqs`` sequences of the decode config, all
    query heads. Returns (prefill TFLOP/s, decode GB/s, seconds, description).
    """
    from oracle import attn_oracle as orc
    pc = gen.CONFIGS[PREFILL_CFG]
    q, k, v = gen.prefill_inputs(1, pc["Hq"], pc["Hkv"], pc["S"], pc["D"], pc["seed"])
    heads = [(0, (seed_shift * 7 + 5 * i) % pc["Hq"]) for i in range(n_prefill_heads)]
    t0 = time.perf_counter()
    orc.prefill(q, k, v, True, gen.attn_scale(pc["D"]), heads=heads)
    tp = time.perf_counter() - t0
    fl = prefill_flops(1, len(heads), pc["S"], pc["D"])
    dc = gen.CONFIGS[DECODE_CFG]
    cache = gen.paged_decode_inputs(dc["N"], dc["Hq"], dc["Hkv"], dc["D"], dc["page_size"], dc["len_lo"],
                                    dc["len_hi"], seed=dc["seed"], poison=False)
    seqs = [(seed_shift * 3 + 9 * i) % dc["N"] for i in range(n_decode_seqs)]
    t0 = time.perf_counter()
    orc.decode_paged(cache.q, cache.k_pages, cache.v_pages, cache.block_table, cache.seq_lens,
                     dc["page_size"], gen.attn_scale(dc["D"]), seqs=seqs)
    td = time.perf_counter() - t0
    lens = [int(cache.seq_lens[s]) for s in seqs]
    by = decode_bytes(lens, dc["Hq"], dc["Hkv"], dc["D"], cache.max_pages)
    desc = (f"{len(heads)} of {pc['B'] * pc['Hq']} (b,hq) heads of the GQA prefill (all {pc['S']} rows each); "
            f"{len(seqs)} of {dc['N']} decode sequences")
    return fl / tp / 1e12, by / td / 1e9, tp + td, desc


def cpu_threads():
    return torch.get_num_threads(), os.cpu_count()


def run_reference(args, world, rank):
    if rank != 0:
        return
    for i in range(args.warmup):
        oracle_sample(1, 2, seed_shift=i)
    tfl, gbs, secs = [], [], 0.0
    desc = ""
    for i in range(args.steps):
        a, b, s, desc = oracle_sample(1, 2, seed_shift=100 + i)
        tfl.append(a)
        gbs.append(b)
        secs += s
    value = statistics.mean(tfl)
    cores = cpu_threads()[1]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{PREFILL_CFG}+{DECODE_CFG}", "sample_per_step": desc},
        "decode": {"value": statistics.mean(gbs), "unit": "GB/s"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------- GPU arm

def run_gpu(args, world, rank, local):
    import attention_online_softmax_fwd_b200 as ab
    from attention_online_softmax_fwd_b200 import binding
    binding.load_library()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    pc = gen.CONFIGS[PREFILL_CFG]
    dc = gen.CONFIGS[DECODE_CFG]
    B, Hq, Hkv, S, D = pc["B"], pc["Hq"], pc["Hkv"], pc["S"], pc["D"]
    q_h, k_h, v_h = gen.prefill_inputs(B, Hq, Hkv, S, D, pc["seed"] + 1000 * rank)
    cache = gen.paged_decode_inputs(dc["N"], dc["Hq"], dc["Hkv"], dc["D"], dc["page_size"], dc["len_lo"],
                                    dc["len_hi"], seed=dc["seed"] + 1000 * rank, poison=False)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, S), dtype=torch.float32, device=dev)
    dq, dkp, dvp = cache.q.to(dev), cache.k_pages.to(dev), cache.v_pages.to(dev)
    dbt, dsl = cache.block_table.to(dev), cache.seq_lens.to(dev)
    do = torch.empty_like(dq)
    dlse = torch.empty((dc["N"], dc["Hq"]), dtype=torch.float32, device=dev)
    ws = torch.empty(ab.decode_workspace_bytes(dc["N"], dc["Hq"], dc["D"], cache.max_pages, dc["page_size"],
                                               DECODE_SPLIT), dtype=torch.uint8, device=dev)
    scale = gen.attn_scale(D)
    flush = L2Flush(dev)

    def prefill_call():
        ab.prefill(q, k, v, causal=True, scale=scale, out=o, lse=lse)

    def decode_call():
        ab.decode_paged(dq, dkp, dvp, dbt, dsl, scale=scale, split_tokens=DECODE_SPLIT, out=do, lse=dlse,
                        workspace=ws)

    for _ in range(args.warmup):
        flush()
        prefill_call()
        decode_call()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(physical_gpu_id(local), fallback=str(local))
    clocks.start()
    time.sleep(0.3)
    dist_barrier(world)
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for i in range(args.steps):
        flush()
        ev[i][0].record(stream)
        prefill_call()
        ev[i][1].record(stream)
        decode_call()
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    dist_barrier(world)
    wall = time.perf_counter() - wall0
    clk = clocks.stop()
    pre_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    dec_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    pre_ms = dist_max(pre_ms, world)
    dec_ms = dist_max(dec_ms, world)
    step_ms = pre_ms + dec_ms

    # ---- end to end through the public API: pinned host inputs in, results back to host
    q_p, k_p, v_p = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
    o_p = torch.empty(q_h.shape, dtype=torch.bfloat16).pin_memory()
    lse_p = torch.empty((B, Hq, S), dtype=torch.float32).pin_memory()
    dq_p, dbt_p, dsl_p = cache.q.pin_memory(), cache.block_table.pin_memory(), cache.seq_lens.pin_memory()
    do_p = torch.empty(cache.q.shape, dtype=torch.bfloat16).pin_memory()
    dlse_p = torch.empty((dc["N"], dc["Hq"]), dtype=torch.float32).pin_memory()
    h2d_pre = sum(t.numel() * t.element_size() for t in (q_p, k_p, v_p))
    d2h_pre = o_p.numel() * 2 + lse_p.numel() * 4
    h2d_dec = sum(t.numel() * t.element_size() for t in (dq_p, dbt_p, dsl_p))
    d2h_dec = do_p.numel() * 2 + dlse_p.numel() * 4

    def e2e_step():
        q.copy_(q_p, non_blocking=True); k.copy_(k_p, non_blocking=True); v.copy_(v_p, non_blocking=True)
        prefill_call()
        o_p.copy_(o, non_blocking=True); lse_p.copy_(lse, non_blocking=True)
        ee = torch.cuda.Event(enable_timing=True)
        ee.record(stream)
        dq.copy_(dq_p, non_blocking=True); dbt.copy_(dbt_p, non_blocking=True); dsl.copy_(dsl_p, non_blocking=True)
        decode_call()
        do_p.copy_(do, non_blocking=True); dlse_p.copy_(dlse, non_blocking=True)
        return ee

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    e2e_pre, e2e_dec = [], []
    for i in range(args.steps):
        flush()
        e0 = torch.cuda.Event(enable_timing=True)
        e2 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e1 = e2e_step()
        e2.record(stream)
        e2.synchronize()
        e2e_pre.append(e0.elapsed_time(e1))
        e2e_dec.append(e1.elapsed_time(e2))
    e2e_pre_ms = dist_max(statistics.mean(e2e_pre), world)
    e2e_dec_ms = dist_max(statistics.mean(e2e_dec), world)

    # ---- parity spot check of this run's output (cheap invariant: finite, LSE >= row max bound)
    finite = bool(torch.isfinite(o.float()).all().item() and torch.isfinite(do.float()).all().item())

    peaks, peak_src = load_peaks()
    traffic = load_profile_traffic()
    fl = prefill_flops(B, Hq, S, D)
    by = decode_bytes(cache.seq_lens.tolist(), dc["Hq"], dc["Hkv"], dc["D"], cache.max_pages)
    pre_tfs = fl / (pre_ms * 1e-3) / 1e12
    dec_gbs = by / (dec_ms * 1e-3) / 1e9
    value = pre_tfs * world

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": f"{PREFILL_CFG}+{DECODE_CFG}",
            "prefill": {"B": B, "Hq": Hq, "Hkv": Hkv, "S": S, "D": D, "causal": True, "seed": pc["seed"]},
            "decode": {"num_seqs": dc["N"], "Hq": dc["Hq"], "Hkv": dc["Hkv"], "D": dc["D"],
                       "page_size": dc["page_size"], "len_range": [dc["len_lo"], dc["len_hi"]],
                       "split_tokens": DECODE_SPLIT, "tokens": int(cache.seq_lens.sum()), "seed": dc["seed"]},
            "l2": "flushed before every timed step (256 MiB write, then 256 MiB read of another buffer)",
            "parallelism": f"replica x{world}" if world > 1 else "single GPU",
        },
        "prefill": {"ms": pre_ms, "tflops": pre_tfs, "flops_per_launch": fl,
                    "frac_of_spec_2250": pre_tfs / SPEC_PEAKS["bf16_tflops"]},
        "decode": {"ms": dec_ms, "value": dec_gbs * world, "unit": "GB/s", "bytes_per_call": by,
                   "frac_of_spec_8000": dec_gbs / SPEC_PEAKS["hbm_gbs"]},
        "roofline": {"bound": "tensor", "kernel": "prefill_kernel<128,causal>", "achieved": pre_tfs,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": pre_tfs / peaks["bf16_tflops"],
                     "peak_source": f"{peak_src} bf16 burst", "traffic": traffic.get("prefill_bytes_per_launch")},
        "roofline_decode": {"bound": "hbm", "kernel": "decode_heads_kernel<128,4,4>+decode_merge_kernel",
                            "achieved": dec_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": dec_gbs / peaks["hbm_gbs"], "peak_source": f"{peak_src} HBM copy",
                            "traffic": traffic.get("decode_bytes_per_call")},
        "e2e": {"value": fl / (e2e_pre_ms * 1e-3) / 1e12 * world, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d_pre + h2d_dec, "d2h_bytes_per_step": d2h_pre + d2h_dec,
                "prefill_ms": e2e_pre_ms, "decode_ms": e2e_dec_ms,
                "decode_gbs": by / (e2e_dec_ms * 1e-3) / 1e9 * world},
        "gpu_launches": 3 * args.steps,
        "clocks": clk,
        "wall_s_timed_region": wall,
        "outputs_finite": finite,
    }
    if rank == 0 and world == 1 and not args.no_extras:
        line["decode_fp8"] = fp8_decode_report(dev, peaks, cache, flush)
        line["chunked_prefill_paged"] = chunked_prefill_report(dev, peaks)
        line["mha_prefill"] = mha_prefill_report(dev, peaks)
    if rank == 0 and world == 1 and not args.no_blasst:
        line["blasst_long_context"] = blasst_long_context_report(dev, peaks)
        line["decode_skip_nothing_skipped"] = skip_overhead_report(dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tfs, gbs, secs, desc = oracle_sample(int(args.cpu_heads), 4)
        line["cpu_baseline"] = {"value": tfs, "unit": "TFLOP/s", "cores": cpu_threads()[0], "kind": "oracle",
                                "sample": desc, "decode_gbs": gbs, "seconds": secs}
    if rank == 0:
        print(json.dumps(line), flush=True)


def fp8_decode_report(dev, peaks, cache, flush, reps=10):
    """The decode workload above with its page pools stored as FP8 E4M3 codes
    (one scale per pool): same sequences, split and query; half the cache bytes."""
    import attention_online_softmax_fwd_b200 as ab
    dc = gen.CONFIGS[DECODE_CFG]
    kc, ks = gen.quantize_pool_e4m3(cache.k_pages)
    vc, vs = gen.quantize_pool_e4m3(cache.v_pages)
    args = [t.to(dev) for t in (cache.q, kc, vc)]
    bt, sl = cache.block_table.to(dev), cache.seq_lens.to(dev)
    o = torch.empty_like(args[0])
    lse = torch.empty((dc["N"], dc["Hq"]), dtype=torch.float32, device=dev)
    ws = torch.empty(ab.decode_workspace_bytes(dc["N"], dc["Hq"], dc["D"], cache.max_pages, dc["page_size"],
                                               DECODE_SPLIT), dtype=torch.uint8, device=dev)
    scale = gen.attn_scale(dc["D"])
    stream = torch.cuda.current_stream(dev)

    def call():
        ab.decode_paged_fp8(args[0], args[1], args[2], ks, vs, bt, sl, scale=scale, split_tokens=DECODE_SPLIT,
                            out=o, lse=lse, workspace=ws)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    ms = statistics.mean(ts)
    by = decode_bytes(cache.seq_lens.tolist(), dc["Hq"], dc["Hkv"], dc["D"], cache.max_pages, kv_elem_bytes=1)
    gbs = by / (ms * 1e-3) / 1e9
    return {"workload": f"{DECODE_CFG} with E4M3 K/V pools, split {DECODE_SPLIT}",
            "kernel": "decode_heads_kernel<128,4,4,fp8>+decode_merge_kernel", "ms": ms, "gbs": gbs,
            "bytes_per_call": by, "frac_of_measured_hbm": gbs / peaks["hbm_gbs"],
            "traffic": load_profile_traffic().get("decode_fp8_bytes_per_call"),
            "frac_of_spec_8000": gbs / SPEC_PEAKS["hbm_gbs"],
            "tokens_per_s": int(cache.seq_lens.sum()) / (ms * 1e-3)}


def chunked_prefill_report(dev, peaks, reps=5):
    """Chunked prefill over the paged cache: 4 sequences, 2048 new tokens each
    after cached prefixes of 0, 2048, 4096 and 6144 tokens (Hq 32, Hkv 8, D 128,
    16-token pages). FLOPs: 4 D per visible (query, key) pair."""
    import attention_online_softmax_fwd_b200 as ab
    B, Sq, Hq, Hkv, D, ps = 4, 2048, 32, 8, 128, 16
    lens = [2048, 4096, 6144, 8192]
    c = gen.paged_prefill_inputs(B, Sq, Hq, Hkv, D, ps, lens, seed=1006)
    args = [t.to(dev) for t in (c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens)]
    scale = gen.attn_scale(D)
    pairs = sum(Sq * (L - Sq) + Sq * (Sq + 1) // 2 for L in lens)
    fl = 4.0 * D * Hq * pairs
    flush = L2Flush(dev)
    o = torch.empty_like(args[0])
    ms, _ = _timed(lambda: ab.prefill_paged(*args, scale=scale, out=o), dev, reps, flush)
    tf = fl / (ms * 1e-3) / 1e12
    return {"workload": "B4 Sq2048 after prefixes 0/2048/4096/6144, Hq32 Hkv8 D128, 16-token pages",
            "ms": ms, "tflops": tf, "flops": fl, "frac_of_measured_bf16": tf / peaks["bf16_tflops"],
            "l2": "flushed before every launch"}


def mha_prefill_report(dev, peaks, reps=20):
    """The MHA causal prefill shaped like a 7B Llama-2 layer (B=4, Hq=Hkv=32,
    S=2048, D=128): 137.4 GFLOP per launch, L2 flushed before each launch."""
    import attention_online_softmax_fwd_b200 as ab
    c = gen.CONFIGS["mha_prefill_llama2_7b"]
    B, Hq, Hkv, S, D = c["B"], c["Hq"], c["Hkv"], c["S"], c["D"]
    q, k, v = [t.to(dev) for t in gen.prefill_inputs(B, Hq, Hkv, S, D, c["seed"])]
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, S), dtype=torch.float32, device=dev)
    scale = gen.attn_scale(D)
    flush = L2Flush(dev)
    ms = _timed(lambda: ab.prefill(q, k, v, causal=True, scale=scale, out=o, lse=lse), dev, reps, flush)[0]
    fl = prefill_flops(B, Hq, S, D)
    tf = fl / (ms * 1e-3) / 1e12
    return {"workload": "mha_prefill_llama2_7b B4 Hq32 Hkv32 S2048 D128 causal", "kernel": "prefill_kernel<128,causal>",
            "ms": ms, "tflops": tf, "flops_per_launch": fl, "frac_of_measured_bf16": tf / peaks["bf16_tflops"],
            "frac_of_spec_2250": tf / SPEC_PEAKS["bf16_tflops"], "l2": "flushed before every launch"}


class L2Flush:
    """Evicts the timed work's inputs from L2 (126 MB) between timed iterations: writes a
    256 MiB buffer, then reads another 256 MiB buffer, so that L2 is left holding clean lines
    of unrelated data and the timed kernels pay no write-back of the flush's own dirty lines."""

    def __init__(self, dev):
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(64 << 20, dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.sum()


def _timed(fn, dev, reps, flush=None):
    """Median CUDA-event time (ms) of ``fn`` on the current stream, after one warm-up call."""
    stream = torch.cuda.current_stream(dev)
    out = fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        if flush is not None:
            flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        out = fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    return statistics.median(ts), out


def _decode_kept_bytes(mask, seq_lens, G, D, rows_per_unit, page_size, max_pages):
    """Algorithmic bytes of a tile-skip decode: every cached K row, and the V rows
    of the 64-token tiles that some query head of their KV head keeps."""
    m = mask.cpu()
    if rows_per_unit == "head":
        n, hq, t = m.shape
        m = m.view(n, hq // G, G, t)
        kept = ((m == 0).any(dim=2))                     # a KV head's tile is loaded if one of its heads keeps it
    else:
        kept = (m == 0)
    toks = 0
    L = [int(x) for x in seq_lens]
    for b, Lb in enumerate(L):
        for t in range(-(-Lb // 64)):
            n_tok = min(64, Lb - 64 * t)
            toks += n_tok * int(kept[b, :, t].sum())
    return sum(L) * kept.shape[1] * D * 2, toks * D * 2    # (K bytes, kept V bytes)


def _skip_decode_line(ab, dargs, lam, split, rows, lens, G, D, page_size, max_pages, dense_bytes, dms0, do0,
                      scale, dev, reps, flush, ws):
    """One tile-skip decode configuration: timed without the decision mask (a fill kernel
    the caller would not run), then run once more with it for the statistics."""
    N, Hq, _ = dargs[0].shape
    Hkv = dargs[1].shape[2]
    ms, _ = _timed(lambda: ab.decode_paged_blasst(*dargs, lam, scale=scale, split_tokens=split, rows_per_unit=rows,
                                                  skip_mask=False, workspace=ws), dev, reps, flush)
    do, _, dmask = ab.decode_paged_blasst(*dargs, lam, scale=scale, split_tokens=split, rows_per_unit=rows,
                                          workspace=ws)
    dvis = dmask != 2
    _, v_kept = _decode_kept_bytes(dmask, lens, G, D, rows, page_size, max_pages)
    v_all = sum(lens) * Hkv * D * 2
    kept_bytes = dense_bytes - v_all + v_kept      # q, o, lse and tables included
    return {"ms": ms, "passes": ab.binding.decode_skip_passes(N, Hq, Hkv, max_pages, page_size, split),
            "skipped_frac": float(((dmask == 1) & dvis).sum().item() / dvis.sum().item()),
            "bytes_kept": kept_bytes, "v_bytes_saved_frac": 1.0 - v_kept / v_all,
            "gbs_on_kept_bytes": kept_bytes / (ms * 1e-3) / 1e9,
            "max_abs_err_vs_dense": float((do.float() - do0.float()).abs().max().item()),
            "speedup_vs_dense": dms0 / ms}


def blasst_long_context_report(dev, peaks, reps=5):
    """Long-context BLASST workload (B=1, Hq=32, Hkv=8, S=32768, D=128, 64-key tiles,
    lambda in {0, 0.1, 0.3}): prefill, and the decode of the last row over the paged
    cache at split_tokens = 2048 (the decision split of the workload; 256 and one
    split over the whole sequence as extra lines), for the recipe input (4u on every
    64th key) and a single dominant key (12u on key 0); then the dominant-key pattern
    over a batch of 8 x 16384 tokens. Reports times, the number of passes over K,
    skipped fractions, the kept-tile bytes the decode reads, the error against
    lambda = 0 and the speedup over the dense path (the dense decode at split 256,
    its fastest here)."""
    import attention_online_softmax_fwd_b200 as ab
    c = gen.CONFIGS["blasst_long_context"]
    B, Hq, Hkv, S, D = c["B"], c["Hq"], c["Hkv"], c["S"], c["D"]
    G = Hq // Hkv
    scale = gen.attn_scale(D)
    fl = prefill_flops(B, Hq, S, D)
    flush = L2Flush(dev)
    ws = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
    report = {"workload": "blasst_long_context B1 Hq32 Hkv8 S32768 D128, tiles of 64 keys",
              "decode_note": "decode bytes = every K row + V rows of kept (KV head, tile) pairs; L2 flushed; "
                             "timed without the decision-mask output",
              "prefill_note": "prefill speedup against the dense kernel on the same input"}
    for name, amp, period, seed in (("recipe", 4.0, 64, c["seed"]), ("dominant_key", 12.0, S, c["seed"] + 7)):
        q_h, k_h, v_h = gen.peaked_prefill_inputs(B, Hq, Hkv, S, D, seed, amp=amp, period=period)
        cache = gen.paged_from_contiguous(q_h[:, S - 1], k_h, v_h, page_size=c["page_size"], seed=c["seed"] + 1,
                                          poison=False)
        dargs = [t.to(dev) for t in (cache.q, cache.k_pages, cache.v_pages, cache.block_table, cache.seq_lens)]
        q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
        del q_h, k_h, v_h
        sec = {"prefill": {}, "decode": {}}
        ms0, (o0, _) = _timed(lambda: ab.prefill(q, k, v, causal=True, scale=scale), dev, 3)
        sec["prefill"]["0.0"] = {"ms": ms0, "tflops": fl / (ms0 * 1e-3) / 1e12}
        dense_bytes = decode_bytes([S], Hq, Hkv, D, cache.max_pages)
        dms0, (do0, _) = _timed(lambda: ab.decode_paged(*dargs, scale=scale, split_tokens=256, workspace=ws), dev,
                                reps, flush)
        sec["decode"]["0.0"] = {"ms": dms0, "split": 256, "gbs": dense_bytes / (dms0 * 1e-3) / 1e9,
                                "frac_of_measured_hbm": dense_bytes / (dms0 * 1e-3) / 1e9 / peaks["hbm_gbs"]}
        for lam in (0.1, 0.3):
            cnt = torch.zeros(1, dtype=torch.int64, device=dev)
            ms, (o, _, mask) = _timed(lambda: ab.prefill_blasst(q, k, v, lam, causal=True, scale=scale,
                                                                 skipped_tiles=cnt), dev, 3)
            vis = mask != 2
            err = (o.float() - o0.float()).abs()
            sec["prefill"][str(lam)] = {
                "ms": ms, "tflops_dense_equiv": fl / (ms * 1e-3) / 1e12,
                "skipped_frac": float(((mask == 1) & vis).sum().item() / vis.sum().item()),
                "max_abs_err_vs_dense": float(err.max().item()), "mean_abs_err_vs_dense": float(err.mean().item()),
                "speedup_vs_dense": ms0 / ms}
            for split in (2048, 256, S):
                for rows in ("group", "head"):
                    sec["decode"][f"{lam}_split{split}_{rows}"] = _skip_decode_line(
                        ab, dargs, lam, split, rows, [S], G, D, c["page_size"], cache.max_pages, dense_bytes, dms0,
                        do0, scale, dev, reps, flush, ws)
        report[name] = sec
        del q, k, v, dargs

    # The same dominant-key pattern over a batch of 8 sequences of 16384 tokens (537 MB of K/V):
    # enough bytes that the decode is bound by HBM rather than by latency, so that the V rows the
    # skip does not read show up in the time. Split 16384 is one decision walk per sequence.
    cache = gen.peaked_decode_batch(8, Hq, Hkv, 16384, D, c["seed"] + 9, amp=12.0, page_size=c["page_size"])
    dargs = [t.to(dev) for t in (cache.q, cache.k_pages, cache.v_pages, cache.block_table, cache.seq_lens)]
    lens = [16384] * 8
    dense_bytes = decode_bytes(lens, Hq, Hkv, D, cache.max_pages)
    dense = {sp: _timed(lambda: ab.decode_paged(*dargs, scale=scale, split_tokens=sp, workspace=ws), dev, reps,
                        flush) for sp in (128, 256)}
    best = min(dense, key=lambda sp: dense[sp][0])
    dms0, (do0, _) = dense[best]
    batch = {"workload": "8 sequences x 16384 tokens, 12u on key 0 of each and on every query, Hq32 Hkv8 D128",
             "0.0": {"ms": dms0, "split": best, "gbs": dense_bytes / (dms0 * 1e-3) / 1e9,
                     "ms_by_split": {str(sp): dense[sp][0] for sp in dense}}}
    for lam in (0.1, 0.3):
        for split in (256, 2048, 16384):
            for rows in ("group", "head"):
                batch[f"{lam}_split{split}_{rows}"] = _skip_decode_line(
                    ab, dargs, lam, split, rows, lens, G, D, c["page_size"], cache.max_pages, dense_bytes, dms0,
                    do0, scale, dev, reps, flush, ws)
    report["dominant_key_decode_batch"] = batch
    return report


def skip_overhead_report(dev, reps=5):
    """The tile-skip decode with nothing skipped (lambda = 1e-6 on the N(0, 1) batch of
    64 sequences of 512..8192 tokens, split 256: one pass over K) against the dense
    decode on the same batch: the cost of deciding every tile and gating its V rows."""
    import attention_online_softmax_fwd_b200 as ab
    dc = gen.CONFIGS["paged_gqa_decode"]
    cache = gen.paged_decode_inputs(dc["N"], dc["Hq"], dc["Hkv"], dc["D"], dc["page_size"], dc["len_lo"],
                                    dc["len_hi"], seed=dc["seed"], poison=False)
    dargs = [t.to(dev) for t in (cache.q, cache.k_pages, cache.v_pages, cache.block_table, cache.seq_lens)]
    scale = gen.attn_scale(dc["D"])
    flush = L2Flush(dev)
    ws = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
    dms, _ = _timed(lambda: ab.decode_paged(*dargs, scale=scale, split_tokens=256, workspace=ws), dev, reps, flush)
    out = {"workload": "paged_gqa_decode (64 sequences, 512..8192 tokens, Hq32 Hkv8 D128), split 256",
           "dense_ms": dms}
    for lam in (1e-6, 0.3):
        cnt = torch.zeros(1, dtype=torch.int64, device=dev)
        ms, _ = _timed(lambda: ab.decode_paged_blasst(*dargs, lam, scale=scale, split_tokens=256, skip_mask=False,
                                                      workspace=ws, skipped_tiles=cnt), dev, reps, flush)
        out[str(lam)] = {"ms": ms, "time_vs_dense": ms / dms, "skipped_decisions": int(cnt.item()) // (reps + 1),
                         "passes": ab.binding.decode_skip_passes(dc["N"], dc["Hq"], dc["Hkv"], cache.max_pages,
                                                                 dc["page_size"], 256)}
    return out


PROFILE_CASES = ("skip_decode_one_pass", "skip_decode_two_pass", "dense_decode_batch", "single_seq_decode",
                 "mha_prefill", "chunked_prefill")


def run_profile_case(name, dev, calls=5):
    """A few launches of one workload, for an ncu capture of its kernels (nothing is timed or
    printed but a line naming the case):
      skip_decode_one_pass  the paged GQA decode batch (64 sequences of 512..8192 tokens),
                            lambda = 0.3, split 256, group decisions: one pass over K
      skip_decode_two_pass  8 x 16384 tokens with one dominant key each, lambda = 0.3, one
                            split per sequence, group decisions: two passes
      dense_decode_batch    the same 8 x 16384 tokens, dense, split 256
      single_seq_decode     the 32768-token BLASST sequence's last row, dense, split 256
      mha_prefill           the MHA prefill B4 Hq=Hkv=32 S2048 D128, causal
      chunked_prefill       the chunked prefill over 16-token pages: 4 x 2048 new tokens after
                            cached prefixes of 0, 2048, 4096 and 6144 tokens, Hq 32 Hkv 8 D128"""
    import attention_online_softmax_fwd_b200 as ab
    scale = gen.attn_scale(128)
    ws = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
    if name == "mha_prefill":
        c = gen.CONFIGS["mha_prefill_llama2_7b"]
        q, k, v = [t.to(dev) for t in gen.prefill_inputs(c["B"], c["Hq"], c["Hkv"], c["S"], c["D"], c["seed"])]
        fn = lambda: ab.prefill(q, k, v, causal=True, scale=scale)
    elif name == "chunked_prefill":
        c = gen.paged_prefill_inputs(4, 2048, 32, 8, 128, 16, [2048, 4096, 6144, 8192], seed=1006)
        args = [t.to(dev) for t in (c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens)]
        fn = lambda: ab.prefill_paged(*args, scale=scale)
    else:
        if name == "skip_decode_one_pass":
            dc = gen.CONFIGS["paged_gqa_decode"]
            cache = gen.paged_decode_inputs(dc["N"], dc["Hq"], dc["Hkv"], dc["D"], dc["page_size"], dc["len_lo"],
                                            dc["len_hi"], seed=dc["seed"], poison=False)
        elif name == "single_seq_decode":
            c = gen.CONFIGS["blasst_long_context"]
            q_h, k_h, v_h = gen.peaked_prefill_inputs(1, c["Hq"], c["Hkv"], c["S"], c["D"], c["seed"] + 7, amp=12.0,
                                                      period=c["S"])
            cache = gen.paged_from_contiguous(q_h[:, -1], k_h, v_h, page_size=c["page_size"], seed=c["seed"] + 1,
                                              poison=False)
        else:
            cache = gen.peaked_decode_batch(8, 32, 8, 16384, 128, gen.CONFIGS["blasst_long_context"]["seed"] + 9,
                                            amp=12.0, page_size=16)
        d = [t.to(dev) for t in (cache.q, cache.k_pages, cache.v_pages, cache.block_table, cache.seq_lens)]
        if name == "skip_decode_one_pass":
            fn = lambda: ab.decode_paged_blasst(*d, 0.3, scale=scale, split_tokens=256, skip_mask=False, workspace=ws)
        elif name == "skip_decode_two_pass":
            fn = lambda: ab.decode_paged_blasst(*d, 0.3, scale=scale, split_tokens=16384, skip_mask=False,
                                                workspace=ws)
        else:
            fn = lambda: ab.decode_paged(*d, scale=scale, split_tokens=256, workspace=ws)
    for _ in range(calls):
        fn()
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": name, "calls": calls}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-blasst", action="store_true", help="skip the long-context BLASST report")
    ap.add_argument("--no-extras", action="store_true", help="skip the FP8-decode and chunked-prefill reports")
    ap.add_argument("--cpu-heads", type=int, default=8)
    ap.add_argument("--profile-case", choices=PROFILE_CASES, default=None,
                    help="run a few launches of one workload for an ncu capture, and nothing else")
    args = ap.parse_args()
    if args.profile_case:
        run_profile_case(args.profile_case, torch.device("cuda:0"))
        return
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_gpu(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
