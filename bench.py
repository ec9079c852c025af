"""Benchmark: 200K-token prefill of one 8-layer group with index sharing.

One step = layer_group_forward over 8 layers with pattern FSSSFSSS (one
indexer per four layers): 2 fused indexer + top-k launches and 8 sparse
attention launches on a 200000-token sequence (H_I=32, d_I=128, top-2048,
GQA 32 query / 4 KV heads, d=128, bf16; output bf16).  The same group with
pattern FFFFFFFF (every layer indexes) is timed alongside for the indexer
time ratio.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

N > 1 runs under torchrun: every rank runs its own independent sequence
(replicas, weak scaling; the path has no cross-GPU exchange), the step
time is the max over ranks and `value` counts the tokens of all ranks.
Rank 0 prints one JSON line.  `--impl reference` times the CPU oracle on
the host cores on a bounded sample of rows of the same workload.
`--case cp` splits ONE sequence over the torchrun ranks instead
(context-parallel prefill: zig-zag row blocks, an all-gather of the keys
each step, strong scaling).
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill tok/s at 200K ctx (indexer+top-k+sparse attn), % roofline"
L, H_I, D_I, TOPK = 200000, 32, 128, 2048
HQ, HKV, DH = 32, 4, 128
PATTERN = "FSSSFSSS"
ALL_F = "FFFFFFFF"
N_LAYERS = 8
WORKLOAD = (f"prefill L={L}, batch 1, 8 layers {PATTERN} (1 indexer per 4 layers; all-F timed too), "
            f"indexer H_I={H_I} d_I={D_I} bf16 top-{TOPK}, sparse attention GQA {HQ}Q/{HKV}KV d={DH} bf16, "
            f"bf16 output")


# Per-layer noise of the structured generator.  The top-2048 of 200K tokens (1 %) reacts more to
# layer noise than the small test shapes do: at 0.2 adjacent layers share ~61 % of their
# selections, below the pages' 70-100 % band; 0.12 puts them at ~78 % (measured, reported by
# the run as adjacent_layer_overlap).  The 1M-token chunk (top-2048 of up to 1M) uses 0.1.
SIGMA_200K = 0.12
SIGMA_1M = 0.1


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p["bf16_tflops_sustained"], "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ----------------------------------------------------------- algorithmic work
def gathered_rows(L_, k):
    """sum_t min(k, t+1): KV rows one attention launch gathers per KV head."""
    return k * (k + 1) // 2 + max(0, L_ - k) * k


def attn_bytes(L_=L, k=TOPK):
    return gathered_rows(L_, k) * HKV * (DH + DH) * 2


def indexer_flops(L_=L):
    return 2 * H_I * D_I * L_ * (L_ + 1) // 2


# ------------------------------------------------------------------ clocks
class ClockSampler:
    def __init__(self, index, path):
        self.path = path
        self.p = None
        try:
            self.f = open(path, "w")
            self.p = subprocess.Popen(
                ["nvidia-smi", f"--id={index}",
                 "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        sm.sort()
        med = sm[len(sm) // 2] if sm else None
        return {"sm_mhz": med, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- GPU arm
def adjacent_overlap(layers, dev, rows=2048):
    """Mean top-k overlap of adjacent layers' own selections (the pages report 70-100%) over the
    last `rows` query rows: each layer's indexer runs on them alone, idx_overlap counts the
    shared indices."""
    import torch
    from long_context_dsa_b200 import dsa

    p0 = L - rows
    sel = []
    for Lh in layers[:4]:
        sel.append(dsa.idx_score_topk(Lh["q_I"][:, p0:].contiguous(), Lh["k_I"], Lh["w"][:, p0:].contiguous(),
                                      TOPK, q_pos0=p0))
    fr = [float(dsa.idx_overlap(sel[l], sel[l + 1]).double().mean().item()) / TOPK for l in range(len(sel) - 1)]
    torch.cuda.synchronize()
    return {"rows": f"last {rows} of {L}", "layers": "0-1, 1-2, 2-3", "values": [round(x, 4) for x in fr],
            "mean": round(sum(fr) / len(fr), 4)}


def pattern_search(layers, dev, rows=2048, n_f=2):
    """The F/S search on this workload: every layer's own selection over the last `rows` query
    rows (calibration rows), all pairwise overlaps, then the greedy pattern with n_f F layers."""
    import time

    import numpy as np
    import torch
    from long_context_dsa_b200 import dsa

    torch.cuda.synchronize()
    t0 = time.perf_counter()
    p0 = L - rows
    sel = [dsa.idx_score_topk(Lh["q_I"][:, p0:].contiguous(), Lh["k_I"], Lh["w"][:, p0:].contiguous(), TOPK,
                              q_pos0=p0) for Lh in layers]
    n = len(layers)
    ov = np.zeros((n, n))
    for f in range(n):
        for j in range(f + 1, n):
            ov[f, j] = float(dsa.idx_overlap(sel[f], sel[j]).double().mean().item()) / TOPK
    pattern = dsa.layer_pattern_search(ov, n_f)
    sec = time.perf_counter() - t0
    return {"calibration_rows": f"last {rows} of {L}", "n_f": n_f, "pattern": pattern,
            "mean_overlap_of_s_layers": round(float(np.mean([ov[max(i for i in range(j + 1) if pattern[i] == 'F'), j]
                                                            for j in range(n) if pattern[j] == "S"])), 4),
            "seconds": round(sec, 3)}


def attn_traffic():
    """DRAM bytes of one full 200K sparse-attention launch (layer 0 of the warm-up step), from ncu
    (dram__bytes_read.sum 22.01 GB + dram__bytes_write.sum 1.64 GB; one pass, no replay), taken on
    the current kernel.  Rows run KV head by KV head, so one head's K/V (102 MB) stays in L2 while
    its rows gather from it.  Update with the capture when the kernel changes."""
    return round(22.01e9 + 1.64e9)


def stratified_random_indices(L_, k, dev, seed, rows_per_chunk=8192):
    """Top-k-shaped index rows that defeat the workload's cross-query reuse: row t with t+1 > k
    takes one uniformly random token from each of k equal strata of [0, t] (distinct, ascending);
    shorter rows take every token, then -1.  Seeded, drawn on the device in row chunks."""
    import torch

    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    out = torch.empty((1, L_, k), dtype=torch.int32, device=dev)
    i = torch.arange(k, device=dev, dtype=torch.int64)
    for r0 in range(0, L_, rows_per_chunk):
        r1 = min(L_, r0 + rows_per_chunk)
        n = torch.arange(r0, r1, device=dev, dtype=torch.int64)[:, None] + 1      # tokens 0..t
        lo = (i[None, :] * n) // k
        hi = ((i[None, :] + 1) * n) // k
        u = torch.rand((r1 - r0, k), generator=g, device=dev, dtype=torch.float64)
        pick = lo + (u * (hi - lo).double()).long()
        pick = torch.minimum(pick, hi - 1)
        short = n <= k                                                               # every token, then -1
        full = torch.where(i[None, :] < n, i[None, :], torch.full_like(pick, -1))
        out[0, r0:r1] = torch.where(short, full, pick).int()
    return out


def attention_random_indices(layers, dev, stream, o_buf, ws, reps=3):
    """The prefill workload's sparse attention (layer 0's Q/K/V, bf16 output, the bench's launch
    configuration) on stratified random top-2048 rows instead of the indexer's selections: nearby
    queries no longer share selections, so the gather leans on HBM instead of L2."""
    import torch
    from long_context_dsa_b200 import dsa

    idx = stratified_random_indices(L, TOPK, dev, seed=77)
    Lh = layers[0]
    dsa.sparse_attn_topk(Lh["Q"], Lh["K"], Lh["V"], idx, o_dtype=torch.bfloat16, out=o_buf, workspace=ws,
                         stream=stream)
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        dsa.sparse_attn_topk(Lh["Q"], Lh["K"], Lh["V"], idx, o_dtype=torch.bfloat16, out=o_buf, workspace=ws,
                             stream=stream)
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    dsa.check_status(ws)
    del idx
    torch.cuda.empty_cache()
    return sum(ts) / len(ts)


def run_gpu(args, rank, world, local_rank):
    import torch
    from long_context_dsa_b200 import dsa, replicas

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    hbm, bf16_burst, bf16_sus, peak_src = peaks()

    barrier = replicas.barrier

    # ---- inputs (seeded; each rank its own sequence)
    layers = make_layers(dev, rank)
    for Lh in layers:
        Lh["O"] = torch.empty((1, L, HQ, DH), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()
    shape = dsa.group_shape(1, L, 0, L, H_I, D_I, HQ, HKV, DH, DH, TOPK, o_dtype=dsa.DSA_BF16)
    ws = torch.zeros(dsa.layer_group_forward_workspace_size(shape), dtype=torch.uint8, device=dev)
    cache = dsa.IndexCache(torch.empty((1, L, TOPK), dtype=torch.int32, device=dev))

    def make_events():
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(3 * N_LAYERS)]
        for e in evs:
            e.record(stream)
        return evs

    def step(pattern, evs=None):
        return dsa.layer_group_forward(shape, layers, pattern, cache, workspace=ws, events=evs)

    for _ in range(args.warmup):
        step(PATTERN)
    torch.cuda.synchronize()
    dsa.check_status(ws)

    # ---- timed region: K steps of the shared-index group
    step_evs = [make_events() for _ in range(args.steps)]
    import tempfile
    clk = ClockSampler(local_rank, os.path.join(args.clocks_dir or tempfile.gettempdir(), f"clocks_rank{rank}.csv"))
    barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    launches = 0
    for i in range(args.steps):
        st = step(PATTERN, step_evs[i])
        launches += st.indexer_launches + st.attention_launches
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = clk.stop()
    dsa.check_status(ws)
    ms_local = t0.elapsed_time(t1)
    idx_ms, attn_ms = [], []
    for evs in step_evs:
        for l in range(N_LAYERS):
            if PATTERN[l] == "F":
                idx_ms.append(evs[3 * l].elapsed_time(evs[3 * l + 1]))
            attn_ms.append(evs[3 * l + 1].elapsed_time(evs[3 * l + 2]))

    # ---- the same attention on indices without cross-query reuse (HBM-bound gather)
    rnd_ms = attention_random_indices(layers, dev, stream, layers[0]["O"], ws)

    # ---- all-F group (indexer ratio), untimed for `value`
    allf_evs = make_events()
    step(ALL_F)
    torch.cuda.synchronize()
    allf_evs = make_events()
    step(ALL_F, allf_evs)
    torch.cuda.synchronize()
    dsa.check_status(ws)
    allf_idx = [allf_evs[3 * l].elapsed_time(allf_evs[3 * l + 1]) for l in range(N_LAYERS)]
    allf_step = allf_evs[0].elapsed_time(allf_evs[-1])
    overlap = adjacent_overlap(layers, dev)
    search = pattern_search(layers, dev)

    # ---- end to end through the public API from pinned host memory
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, layers, shape, cache, ws, dev, stream, world)

    # ---- max over ranks
    ms = replicas.max_over_ranks(ms_local, dev)
    ms_per_step = ms / args.steps
    idx_avg = sum(idx_ms) / len(idx_ms)
    attn_avg = sum(attn_ms) / len(attn_ms)
    value = replicas.job_throughput(L, world, ms_per_step)

    abytes = attn_bytes()
    dram = attn_traffic()
    iflops = indexer_flops()
    t_idx = 2 * iflops / (bf16_sus * 1e12)
    t_gather = N_LAYERS * abytes / (hbm * 1e9)
    step_roof_s = max(t_idx, t_gather)
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded structured generator; no dataset or trained weights)",
        "config": {"workload": WORKLOAD, "seq_len": L, "global_batch": world, "layers": N_LAYERS,
                   "pattern": PATTERN, "topk": TOPK, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (q_I 1.6 GB, Q 1.6 GB per layer); no flush needed"},
        "roofline": {
            "bound": "hbm", "kernel": "sparse_attn_kernel (gathered K/V rows)",
            "achieved": round(dram / (attn_avg / 1e3) / 1e9, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(dram / (attn_avg / 1e3) / 1e9 / hbm, 4), "traffic": dram,
            "peak_source": f"{peak_src} hbm_gbs",
            "achieved_basis": "DRAM bytes of one full-size launch (ncu dram__bytes_read+write) / average "
                              "launch time in the timed region",
            "algorithmic_bytes_per_launch": abytes, "avg_launch_ms": round(attn_avg, 3),
            "gathered_gbs_equiv": round(abytes / (attn_avg / 1e3) / 1e9, 1),
            "gathered_frac_equiv": round(abytes / (attn_avg / 1e3) / 1e9 / hbm, 4),
            "gathered_note": "algorithmic gathered bytes (sum_t min(k,t+1) x Hkv x 2d x 2 B) / launch time: above "
                             "HBM peak because every token is gathered by many queries and L2 serves the repeats "
                             "(DRAM moves ~3 % of the gathered bytes); the kernel is bound by instruction issue and "
                             "latency (57 % of issue slots used), not by DRAM or by the gather path: a pure "
                             "16-byte cp.async copy through the same per-warp rings, with the same 2048-key units "
                             "in the same KV-head order and ascending index lists, moves 19.1 TB/s of random rows "
                             "of a 200K-token pool on this GPU"},
        "attention_random_indices": {
            "kernel": "sparse_attn_kernel, same shape and launch configuration, stratified random top-2048 rows",
            "avg_launch_ms": round(rnd_ms, 3),
            "achieved": round(abytes / (rnd_ms / 1e3) / 1e9, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(abytes / (rnd_ms / 1e3) / 1e9 / hbm, 4),
            "note": "each token is still gathered by ~2000 queries over the launch, so L2 keeps part of the "
                    "410 MB K/V; with no shared selections between neighbours the DRAM share is far higher"},
        "indexer_roofline": {
            "bound": "tensor", "kernel": "indexer_topk_kernel (fused scores + top-k)",
            "achieved": round(iflops / (idx_avg / 1e3) / 1e12, 1), "peak": bf16_sus, "unit": "TFLOP/s",
            "frac": round(iflops / (idx_avg / 1e3) / 1e12 / bf16_sus, 4),
            "peak_source": f"{peak_src} bf16_tflops_sustained (kernel inside a long step)",
            "frac_of_burst": round(iflops / (idx_avg / 1e3) / 1e12 / bf16_burst, 4),
            "algorithmic_flops_per_launch": iflops, "avg_launch_ms": round(idx_avg, 3)},
        "step_roofline": {"t_indexer_s": round(t_idx, 4), "t_gather_s": round(t_gather, 4),
                          "bound_s": round(step_roof_s, 4),
                          "frac": round(step_roof_s / (ms_per_step / 1e3), 4),
                          "note": "the step's roofline: max(indexer FLOPs at tensor peak, gathered bytes at HBM "
                                  "peak); the gathered bytes are largely L2 hits here (see roofline), so this bound "
                                  "is not tight and a fraction near 1 does not mean the step is at its limit"},
        "index_sharing": {"all_f_step_ms": round(allf_step, 3), "shared_step_ms": round(ms_per_step, 3),
                          "all_f_indexer_ms": round(sum(allf_idx), 3),
                          "shared_indexer_ms": round(sum(idx_ms) / args.steps, 3),
                          "indexer_time_ratio": round(sum(allf_idx) / (sum(idx_ms) / args.steps), 3),
                          "adjacent_layer_overlap": overlap},
        "pattern_search": search,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if e2e is not None:
        out["e2e"] = e2e
    return out, layers


def run_e2e(args, layers, shape, cache, ws, dev, stream, world=1):
    """Same metric through the public API with host buffers: every step copies its inputs
    host->device from pinned memory and reads every layer's output back.  Copies overlap the
    compute: inputs stream in on one copy stream layer by layer, each layer starts when its own
    inputs have landed (F layers write the group's index cache with idx_score_topk, every layer
    reads it via idx_cache_get and runs sparse_attn_topk), and each output streams back on a
    second copy stream as soon as it is written."""
    import torch
    from long_context_dsa_b200 import dsa, replicas

    names_f = ("q_I", "k_I", "w", "Q", "K", "V")
    names_s = ("Q", "K", "V")
    host_in, host_out = [], []
    for l, Lh in enumerate(layers):
        names = names_f if PATTERN[l] == "F" else names_s
        host_in.append({n: torch.empty_like(Lh[n], device="cpu").pin_memory() for n in names})
        for n in names:
            host_in[-1][n].copy_(Lh[n])
        host_out.append(torch.empty_like(Lh["O"], device="cpu").pin_memory())
    h2d = sum(t.numel() * t.element_size() for d in host_in for t in d.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    steps = max(1, min(args.steps, 2))
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def one():
        start = torch.cuda.Event()
        start.record(stream)
        s_in.wait_event(start)
        landed = []  # per layer: (indexer inputs in, attention inputs in)
        with torch.cuda.stream(s_in):
            for l, Lh in enumerate(layers):
                evs = []
                for group in (("q_I", "k_I", "w"), ("Q", "K", "V")):
                    for n in group:
                        if n in host_in[l]:
                            Lh[n].copy_(host_in[l][n], non_blocking=True)
                    e = torch.cuda.Event()
                    e.record(s_in)
                    evs.append(e)
                landed.append(evs)
        for l, Lh in enumerate(layers):
            if PATTERN[l] == "F":
                stream.wait_event(landed[l][0])
                dsa.idx_score_topk(Lh["q_I"], Lh["k_I"], Lh["w"], TOPK, out=cache.buf, workspace=ws, stream=stream)
                cache.put(l, PATTERN)
            stream.wait_event(landed[l][1])
            idx = dsa.idx_cache_get(cache, l, PATTERN)
            dsa.sparse_attn_topk(Lh["Q"], Lh["K"], Lh["V"], idx, o_dtype=torch.bfloat16, out=Lh["O"], workspace=ws,
                                 stream=stream)
            done = torch.cuda.Event()
            done.record(stream)
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                host_out[l].copy_(Lh["O"], non_blocking=True)
        end = torch.cuda.Event()
        end.record(s_out)
        stream.wait_event(end)

    one()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    replicas.barrier()
    a.record(stream)
    for _ in range(steps):
        one()
    b.record(stream)
    torch.cuda.synchronize()
    dsa.check_status(ws)
    ms = replicas.max_over_ranks(a.elapsed_time(b) / steps, dev)
    return {"value": round(replicas.job_throughput(L, world, ms), 1), "unit": "tok/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": round(ms, 3),
            "note": "pinned host inputs copied in and every layer's bf16 output read back inside the timed "
                    "region, the copies overlapped with the compute on two copy streams"}


# ------------------------------------------------------------ CPU oracle arm
def make_layers(dev, rank=0, keep_indexer_all=True):
    """The workload's seeded inputs on `dev` (the GPU arm and the oracle sample draw the same bytes)."""
    import torch
    from long_context_dsa_b200 import synth

    from long_context_dsa_b200 import replicas

    seed = replicas.rank_seed(1000, rank)
    gen = synth.StructuredIndexer("prefill200k", 1, L, H_I, D_I, r=32, base_std=1.0, noise_std=SIGMA_200K,
                                  device=dev, seed=seed)
    layers = []
    for l in range(N_LAYERS):
        Lh = {}
        if keep_indexer_all or PATTERN[l] == "F":
            Lh["q_I"], Lh["k_I"], Lh["w"] = gen.layer(l)
        Lh["Q"], Lh["K"], Lh["V"] = synth.attention_inputs("prefill200k", l, 1, L, L, HQ, HKV, DH, DH,
                                                           device=dev, seed=seed)
        layers.append(Lh)
    del gen
    return layers


def oracle_sample(layers, n_rows: int, seed: int = 0):
    """Time the oracle on `n_rows` query rows of the workload (spread over t, last row included) and
    extrapolate to the full step by algorithmic work.  `layers` holds the workload's inputs (any
    device); only the sampled rows and the keys are copied to the host, outside the timed parts.
    Returns (tok/s, extrapolated seconds, sample text, threads, measured seconds)."""
    import numpy as np
    import torch

    import oracle

    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[L - 1], rng.integers(0, L, n_rows - 1)]))
    t_idx = t_att = 0.0
    work_idx = work_att = 0.0
    sel = {}
    def f64(x):  # exact widening to the oracle's working precision, outside the timed parts
        return x.detach().to("cpu", torch.float64).numpy()

    for l in range(N_LAYERS):
        Lh = layers[l]
        if PATTERN[l] == "F":
            k = f64(Lh["k_I"][0])
            for t in rows:
                q = f64(Lh["q_I"][0, t:t + 1])
                w = f64(Lh["w"][0, t:t + 1])
                a = time.perf_counter()
                sc = oracle.indexer_scores(q, k[:t + 1], w, q_pos0=t)
                sel[t] = oracle.topk_select(sc, TOPK, q_pos0=t)
                t_idx += time.perf_counter() - a
                work_idx += t + 1
            del k
        K, V = f64(Lh["K"][0]), f64(Lh["V"][0])
        for t in rows:
            Q = f64(Lh["Q"][0, t:t + 1])
            a = time.perf_counter()
            oracle.sparse_attention(Q, K, V, sel[t])
            t_att += time.perf_counter() - a
            work_att += min(TOPK, t + 1)
    n_f = PATTERN.count("F")
    # seconds per candidate key of one F layer, per gathered row of one layer
    per_idx = t_idx / work_idx
    per_att = t_att / work_att
    total = per_idx * n_f * (L * (L + 1) / 2) + per_att * N_LAYERS * gathered_rows(L, TOPK)
    threads = cpu_info()["cores"]
    sample = (f"{len(rows)} query rows (seeded, spread over t, last row included) through the {PATTERN} group: "
              f"indexer+top-k on {n_f} F layers and attention on {N_LAYERS} layers; "
              f"{t_idx + t_att:.1f} s measured, extrapolated by algorithmic work "
              f"(sum of t+1 for the indexer, sum of min(k,t+1) for attention)")
    return L / total, total, sample, threads, t_idx + t_att


def cpu_info():
    """Host cores this process may run on, the CPU model and numpy's BLAS thread count (the
    oracle's matrix products run in numpy's BLAS; everything else is single-threaded numpy)."""
    cores = len(os.sched_getaffinity(0))
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    blas = None
    try:
        import numpy  # noqa: F401  (loads the BLAS library threadpoolctl inspects)
        import threadpoolctl
        info = [p for p in threadpoolctl.threadpool_info() if p.get("user_api") == "blas"]
        if info:
            blas = {"library": info[0].get("internal_api"), "threads": info[0].get("num_threads")}
    except Exception:
        pass
    return {"cores": cores, "cpu_model": model, "blas": blas}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import torch
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    layers = make_layers(dev, keep_indexer_all=False)
    vals, measured = [], 0.0
    for i in range(args.warmup + args.steps):
        v, total, sample, threads, meas = oracle_sample(layers, args.ref_rows, seed=i)
        if i >= args.warmup:
            vals.append(v)
            measured += meas
    value = sum(vals) / len(vals)
    return {"metric": METRIC, "impl": "reference", "value": round(value, 3), "unit": "tok/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(L / value * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "seq_len": L, "pattern": PATTERN},
            "cpu_baseline": {"value": round(value, 3), "unit": "tok/s", "cores": threads, "kind": "oracle",
                             "sample": sample, "host": cpu_info()},
            "e2e": {"value": round(value, 3), "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_profile_case(args):
    """Small single-kernel launches for ncu captures: the last 2048 queries of the 200K prefill
    through the fused indexer, and the last 4096 queries through sparse attention, both against
    the full 200K-token caches (so L2 sees the real key / KV footprint)."""
    import torch
    from long_context_dsa_b200 import dsa, synth

    dev = torch.device("cuda", 0)
    nq_i, nq_a = 2048, 4096
    gen = synth.StructuredIndexer("prof", 1, L, H_I, D_I, r=32, base_std=1.0, noise_std=SIGMA_200K,
                                device=dev, seed=7)
    q, k, w = gen.layer(0)
    del gen
    q = q[:, L - nq_i:].contiguous()
    w = w[:, L - nq_i:].contiguous()
    Q, K, V = synth.attention_inputs("prof", 0, 1, nq_a, L, HQ, HKV, DH, DH, device=dev, seed=7)
    ws = torch.zeros(dsa.idx_score_topk_workspace_size(1, nq_a, L - nq_a, L, H_I, D_I, TOPK), dtype=torch.uint8,
                     device=dev)
    idx_i = torch.empty((1, nq_i, TOPK), dtype=torch.int32, device=dev)
    O = torch.empty((1, nq_a, HQ, DH), dtype=torch.bfloat16, device=dev)
    # attention indices: a fresh selection of the last 4096 rows with the same indexer
    qa = synth.StructuredIndexer("prof", 1, L, H_I, D_I, r=32, base_std=1.0, noise_std=SIGMA_200K,
                                device=dev, seed=7)
    qa_q, _, qa_w = qa.layer(0)
    del qa
    idx_a = dsa.idx_score_topk(qa_q[:, L - nq_a:].contiguous(), k, qa_w[:, L - nq_a:].contiguous(), TOPK,
                               q_pos0=L - nq_a, workspace=ws)
    del qa_q, qa_w
    torch.cuda.synchronize()
    t_i, t_a = [], []
    for it in range(args.warmup + args.steps):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record()
        dsa.idx_score_topk(q, k, w, TOPK, q_pos0=L - nq_i, out=idx_i, workspace=ws)
        e[1].record()
        dsa.sparse_attn_topk(Q, K, V, idx_a, o_dtype=torch.bfloat16, out=O, workspace=ws)
        e[2].record()
        torch.cuda.synchronize()
        if it >= args.warmup:
            t_i.append(e[0].elapsed_time(e[1]))
            t_a.append(e[1].elapsed_time(e[2]))
    dsa.check_status(ws)
    fl = 2 * H_I * D_I * sum(range(L - nq_i + 1, L + 1))
    by = nq_a * TOPK * HKV * 2 * DH * 2
    ti, ta = min(t_i), min(t_a)
    print(json.dumps({"case": "profile", "indexer_ms": ti, "indexer_tflops": fl / ti / 1e9,
                      "attn_ms": ta, "attn_gathered_gbs": by / ta / 1e6,
                      "indexer_queries": nq_i, "attn_queries": nq_a, "n_kv": L}))


def run_profile_paged(args):
    """Small paged decode case for ncu captures of the gather attention: 64 sequences of 12500
    tokens in shuffled 64-token pages (K/V pools 0.8 GB each in bf16, larger than L2), random
    top-2048 selections, GQA 32/4, d=128.  Each iteration launches the bf16-cache kernel, then
    the fp8-cache kernel on the same cache quantized to E4M3 + per-row scales."""
    import numpy as np
    import torch
    from long_context_dsa_b200 import dsa, synth

    dev = torch.device("cuda", 0)
    B, P, Lseq = 64, 64, 12500
    rng = np.random.default_rng(4000)
    lens = np.full(B, Lseq, np.int32)
    max_pages = (Lseq + P - 1) // P
    num_pages = B * max_pages
    table = torch.from_numpy(rng.permutation(num_pages).astype(np.int32).reshape(B, max_pages)).to(dev)
    seq = torch.from_numpy(lens).to(dev)
    idx = torch.from_numpy(np.stack([np.sort(rng.choice(Lseq, size=TOPK, replace=False))
                                     for _ in range(B)]).astype(np.int32)).to(dev)
    Kp = synth.normal((num_pages, P, HKV, DH), synth.seed_for(4000, "profpaged", "K"), dev, dtype=torch.bfloat16)
    Vp = synth.normal((num_pages, P, HKV, DH), synth.seed_for(4000, "profpaged", "V"), dev, dtype=torch.bfloat16)
    Q = synth.normal((B, HQ, DH), synth.seed_for(4000, "profpaged", "Q"), dev, dtype=torch.bfloat16)
    K8, ks = synth.quantize_e4m3_rows(Kp)
    V8, vs = synth.quantize_e4m3_rows(Vp)
    ws = torch.zeros(dsa.sparse_attn_topk_workspace_size(B, 1, num_pages * P, HQ, HKV, DH, DH, TOPK),
                     dtype=torch.uint8, device=dev)
    O = torch.empty((B, HQ, DH), dtype=torch.bfloat16, device=dev)
    t_b, t_8 = [], []
    for it in range(args.warmup + args.steps):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record()
        dsa.sparse_attn_topk_paged(Q, Kp, Vp, table, seq, idx, o_dtype=torch.bfloat16, out=O, workspace=ws)
        e[1].record()
        dsa.sparse_attn_topk_paged_e4m3(Q, K8, ks, V8, vs, table, seq, idx, o_dtype=torch.bfloat16, out=O,
                                        workspace=ws)
        e[2].record()
        torch.cuda.synchronize()
        if it >= args.warmup:
            t_b.append(e[0].elapsed_time(e[1]))
            t_8.append(e[1].elapsed_time(e[2]))
    # steady state: 10 back-to-back calls per event pair behind an untimed one, so the host's
    # launch work overlaps the GPU (a single call after a synchronize times the host too)
    def burst(fn, n=10):
        fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n
    tb = min(burst(lambda: dsa.sparse_attn_topk_paged(Q, Kp, Vp, table, seq, idx, o_dtype=torch.bfloat16, out=O,
                                                      workspace=ws)) for _ in range(3))
    t8 = min(burst(lambda: dsa.sparse_attn_topk_paged_e4m3(Q, K8, ks, V8, vs, table, seq, idx,
                                                           o_dtype=torch.bfloat16, out=O, workspace=ws))
             for _ in range(3))
    dsa.check_status(ws)
    by = B * TOPK * HKV * DH * 2          # K and V codes gathered (bf16: twice this)
    print(json.dumps({"case": "profile_paged", "bf16_ms": tb, "bf16_gathered_gbs": 2 * by / tb / 1e6,
                      "fp8_ms": t8, "fp8_gathered_gbs": by / t8 / 1e6, "fp8_over_bf16": t8 / tb,
                      "single_call_bf16_ms": min(t_b), "single_call_fp8_ms": min(t_8)}))


def run_profile_latent(args):
    """Small latent-attention case for ncu captures: 1024 query rows with 64 heads against a
    262144-token latent cache (302 MB, larger than L2), stratified random top-2048 rows, bf16
    output -- the tensor-core latent kernel (one unit per row)."""
    import torch
    from long_context_dsa_b200 import dsa, synth

    dev = torch.device("cuda", 0)
    n_kv, nq, hq = 1 << 18, 1024, 64
    Q, KV, _ = synth.attention_inputs("proflat", 0, 1, nq, n_kv, hq, 1, 576, None, device=dev, seed=8)
    idx = stratified_random_indices(n_kv, TOPK, dev, seed=8)[:, n_kv - nq:].contiguous()
    O = torch.empty((1, nq, hq, 512), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(dsa.sparse_attn_topk_workspace_size(1, nq, n_kv, hq, 1, 576, 512, TOPK), dtype=torch.uint8,
                     device=dev)
    ts = []
    for it in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dsa.sparse_attn_topk(Q, KV, None, idx, d_v=512, o_dtype=torch.bfloat16, out=O, workspace=ws)
        b.record()
        torch.cuda.synchronize()
        if it >= args.warmup:
            ts.append(a.elapsed_time(b))
    dsa.check_status(ws)
    by = nq * TOPK * 576 * 2
    fl = nq * TOPK * hq * 2 * (576 + 512)
    t = min(ts)
    print(json.dumps({"case": "profile_latent", "ms": t, "gathered_gbs": by / t / 1e6, "tflops": fl / t / 1e9}))


def run_profile_decode1m(args):
    """One-query fp8 decode indexer at a 1048577-token cache (H_I=64, d_I=128, top-2048) for ncu
    captures: the split decode kernel writing the row's score keys and histogram, then the bin select."""
    import torch
    from long_context_dsa_b200 import dsa, synth

    dev = torch.device("cuda", 0)
    n = (1 << 20) + 1
    gen = synth.StructuredIndexer("profdec1m", 1, n, 64, D_I, r=32, base_std=1.0, noise_std=SIGMA_1M, device=dev,
                                  seed=9)
    q, w = gen.queries(0, n - 1, n)
    k8, ks = synth.quantize_e4m3_rows(gen.keys(0))
    q8, qs = synth.quantize_e4m3_rows(q)
    del gen
    ws = torch.zeros(dsa.idx_score_topk_workspace_size(1, 1, n - 1, n, 64, D_I, TOPK, dsa.DSA_E4M3),
                     dtype=torch.uint8, device=dev)
    out = torch.empty((1, 1, TOPK), dtype=torch.int32, device=dev)
    ts = []
    for it in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dsa.idx_score_topk(q8, k8, w, TOPK, q_pos0=n - 1, q_scale=qs, k_scale=ks, out=out, workspace=ws)
        b.record()
        torch.cuda.synchronize()
        if it >= args.warmup:
            ts.append(a.elapsed_time(b))
    dsa.check_status(ws)
    print(json.dumps({"case": "profile_decode1m", "ms": min(ts), "key_gbs": n * (D_I + 4) / min(ts) / 1e6}))


def run_profile_decode(args):
    """One decode indexer call of the batched decode shape for ncu captures: 64 sequences, one
    query each at the end of a 200000-token bf16 key cache (H_I=32, d_I=128, top-2048): the split
    decode kernel writing every row's score keys and histogram, then the bin select."""
    import torch
    from long_context_dsa_b200 import dsa, synth

    dev = torch.device("cuda", 0)
    B, Lc = 64, 200000
    gen = synth.StructuredIndexer("decode200k", B, Lc, H_I, D_I, r=32, base_std=1.0, noise_std=SIGMA_200K,
                                  device=dev, seed=2000)
    q, w = gen.queries(0, Lc - 1, Lc)
    k = gen.keys(0)
    del gen
    ws = torch.zeros(dsa.idx_score_topk_workspace_size(B, 1, Lc - 1, Lc, H_I, D_I, TOPK), dtype=torch.uint8,
                     device=dev)
    out = torch.empty((B, 1, TOPK), dtype=torch.int32, device=dev)
    ts = []
    for it in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dsa.idx_score_topk(q, k, w, TOPK, q_pos0=Lc - 1, out=out, workspace=ws)
        b.record()
        torch.cuda.synchronize()
        if it >= args.warmup:
            ts.append(a.elapsed_time(b))
    dsa.check_status(ws)
    print(json.dumps({"case": "profile_decode", "ms": min(ts), "key_gbs": B * Lc * D_I * 2 / min(ts) / 1e6}))


def run_decode(args, dev):
    """Decode step: 64 sequences, one new token each, at a 200000-token cache; 4 layers FSSS
    (H_I=32, d_I=128, top-2048; attention 32 query / 4 KV heads, d=128)."""
    import torch
    from long_context_dsa_b200 import dsa, synth

    B, Lc, pat = 64, 200000, "FSSS"
    gen = synth.StructuredIndexer("decode200k", B, Lc, H_I, D_I, r=32, base_std=1.0, noise_std=SIGMA_200K,
                                  device=dev,
                                  seed=2000)
    layers = []
    for l in range(4):
        Lh = {}
        Lh["q_I"], Lh["w"] = gen.queries(l, Lc - 1, Lc)
        Lh["k_I"] = gen.keys(l)
        Lh["Q"], Lh["K"], Lh["V"] = synth.attention_inputs("decode200k", l, B, 1, Lc, HQ, HKV, DH, DH, device=dev,
                                                           seed=2000)
        Lh["O"] = torch.empty((B, 1, HQ, DH), dtype=torch.bfloat16, device=dev)
        layers.append(Lh)
    del gen
    shape = dsa.group_shape(B, 1, Lc - 1, Lc, H_I, D_I, HQ, HKV, DH, DH, TOPK, o_dtype=dsa.DSA_BF16)
    ws = torch.zeros(dsa.layer_group_forward_workspace_size(shape), dtype=torch.uint8, device=dev)
    cache = dsa.IndexCache(torch.empty((B, 1, TOPK), dtype=torch.int32, device=dev))
    sel = [dsa.idx_score_topk(layers[l]["q_I"], layers[l]["k_I"], layers[l]["w"], TOPK, q_pos0=Lc - 1)
           for l in (0, 1)]
    overlap = round(float(dsa.idx_overlap(sel[0], sel[1]).double().mean().item()) / TOPK, 4)
    del sel
    res = {}
    for p in (pat, "FFFF"):
        for _ in range(3):
            dsa.layer_group_forward(shape, layers, p, cache, workspace=ws)
        torch.cuda.synchronize()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(12)]
        for e in evs:
            e.record()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = 10
        t0.record()
        for _ in range(n - 1):
            dsa.layer_group_forward(shape, layers, p, cache, workspace=ws)
        dsa.layer_group_forward(shape, layers, p, cache, workspace=ws, events=evs)
        t1.record()
        torch.cuda.synchronize()
        dsa.check_status(ws)
        ms = t0.elapsed_time(t1) / n
        idx_ms = sum(evs[3 * l].elapsed_time(evs[3 * l + 1]) for l in range(4))
        att_ms = sum(evs[3 * l + 1].elapsed_time(evs[3 * l + 2]) for l in range(4))
        res[p] = (ms, idx_ms, att_ms)
    ms, idx_ms, att_ms = res[pat]
    graph_ms = decode_graph_ms(lambda: [dsa.layer_group_forward(shape, layers, pat, cache, workspace=ws)
                                        for _ in range(10)], 10, ws)
    kbytes = B * Lc * D_I * 2  # the key cache one F layer scans
    abytes = B * TOPK * HKV * 2 * DH * 2
    del layers
    torch.cuda.empty_cache()
    return {"workload": f"decode B={B} at a {Lc}-token cache, 4 layers {pat}, H_I={H_I} d_I={D_I} top-{TOPK}, "
                        f"GQA {HQ}Q/{HKV}KV d={DH}",
            "tok_per_s": round(B / (ms / 1e3), 1), "ms_per_step": round(ms, 4),
            "graph_tok_per_s": _finite(B / (graph_ms / 1e3), 1), "graph_ms_per_step": _finite(graph_ms, 4),
            "indexer_ms": round(idx_ms, 4), "attention_ms": round(att_ms, 4),
            "indexer_gbs": round(kbytes / (idx_ms / 1e3) / 1e9, 1),
            "attention_gathered_gbs": round(4 * abytes / (att_ms / 1e3) / 1e9, 1),
            "adjacent_layer_overlap": overlap,
            "all_f_ms_per_step": round(res["FFFF"][0], 4),
            "all_f_tok_per_s": round(B / (res["FFFF"][0] / 1e3), 1)}


def run_decode_mha(args, dev):
    """Decode with 32 KV heads (MHA, the config's head count) at B = 8: the 200K cache of 64 such
    sequences would not fit one GPU (210 GB per layer).  4 layers FSSS, top-2048."""
    import torch
    from long_context_dsa_b200 import dsa, synth

    B, Lc, Hkv = 8, 200000, 32
    gen = synth.StructuredIndexer("decodemha", B, Lc, H_I, D_I, r=32, base_std=1.0, noise_std=SIGMA_200K,
                                  device=dev,
                                  seed=5000)
    layers = []
    for l in range(4):
        Lh = {}
        Lh["q_I"], Lh["w"] = gen.queries(l, Lc - 1, Lc)
        Lh["k_I"] = gen.keys(l)
        Lh["Q"], Lh["K"], Lh["V"] = synth.attention_inputs("decodemha", l, B, 1, Lc, HQ, Hkv, DH, DH, device=dev,
                                                           seed=5000)
        Lh["O"] = torch.empty((B, 1, HQ, DH), dtype=torch.bfloat16, device=dev)
        layers.append(Lh)
    del gen
    shape = dsa.group_shape(B, 1, Lc - 1, Lc, H_I, D_I, HQ, Hkv, DH, DH, TOPK, o_dtype=dsa.DSA_BF16)
    ws = torch.zeros(dsa.layer_group_forward_workspace_size(shape), dtype=torch.uint8, device=dev)
    cache = dsa.IndexCache(torch.empty((B, 1, TOPK), dtype=torch.int32, device=dev))
    for _ in range(3):
        dsa.layer_group_forward(shape, layers, "FSSS", cache, workspace=ws)
    torch.cuda.synchronize()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(12)]
    for e in evs:
        e.record()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = 10
    a.record()
    for i in range(n):
        dsa.layer_group_forward(shape, layers, "FSSS", cache, workspace=ws, events=evs if i == n - 1 else None)
    b.record()
    torch.cuda.synchronize()
    dsa.check_status(ws)
    ms = a.elapsed_time(b) / n
    att_ms = sum(evs[3 * l + 1].elapsed_time(evs[3 * l + 2]) for l in range(4))
    abytes = B * TOPK * Hkv * 2 * DH * 2
    del layers
    torch.cuda.empty_cache()
    return {"workload": f"decode B={B} at a {Lc}-token cache, 4 layers FSSS, MHA {HQ}Q/{Hkv}KV d={DH}, top-{TOPK}",
            "tok_per_s": round(B / (ms / 1e3), 1), "ms_per_step": round(ms, 4),
            "attention_ms": round(att_ms, 4),
            "attention_gathered_gbs": round(4 * abytes / (att_ms / 1e3) / 1e9, 1)}


def run_mtp(args, dev):
    """Multi-token (speculative) decode: 64 sequences verify 4 draft tokens each at a 200000-token
    cache, 4 layers FSSS.  Shared: the F layer selects once, for the last draft token, and all 4
    tokens attend through that selection (each causally up to its own position).  Unshared: one
    selection per token (4 indexer launches) and per-token attention."""
    import torch
    from long_context_dsa_b200 import dsa, synth

    B, Lc, m, nl = 64, 200000, 4, 4
    p0 = Lc - m
    gen = synth.StructuredIndexer("mtp200k", B, Lc, H_I, D_I, r=32, base_std=1.0, noise_std=SIGMA_200K,
                                  device=dev,
                                  seed=3000)
    q_all, w_all = gen.queries(0, p0, Lc)
    k_I = gen.keys(0)
    del gen
    q_last, w_last = q_all[:, m - 1:].contiguous(), w_all[:, m - 1:].contiguous()
    q_tok = [q_all[:, j:j + 1].contiguous() for j in range(m)]
    w_tok = [w_all[:, j:j + 1].contiguous() for j in range(m)]
    att = [synth.attention_inputs("mtp200k", l, B, m, Lc, HQ, HKV, DH, DH, device=dev, seed=3000) for l in range(nl)]
    Q_tok = [[Q[:, j:j + 1].contiguous() for j in range(m)] for (Q, _, _) in att]
    O = torch.empty((B, m, HQ, DH), dtype=torch.bfloat16, device=dev)
    O1 = [torch.empty((B, 1, HQ, DH), dtype=torch.bfloat16, device=dev) for _ in range(m)]
    idx_s = torch.empty((B, 1, TOPK), dtype=torch.int32, device=dev)
    idx_u = [torch.empty((B, 1, TOPK), dtype=torch.int32, device=dev) for _ in range(m)]
    need = [dsa.idx_score_topk_workspace_size(B, 1, p0 + j, Lc, H_I, D_I, TOPK) for j in range(m)]
    need += [dsa.sparse_attn_topk_workspace_size(B, n, Lc, HQ, HKV, DH, DH, TOPK) for n in (1, m)]
    ws = torch.zeros(max(need), dtype=torch.uint8, device=dev)

    def shared():
        dsa.idx_score_topk(q_last, k_I, w_last, TOPK, q_pos0=Lc - 1, out=idx_s, workspace=ws)
        for (Q, K, V) in att:
            dsa.sparse_attn_topk_shared(Q, K, V, idx_s, m, p0, o_dtype=torch.bfloat16, out=O, workspace=ws)

    def unshared():
        for j in range(m):
            dsa.idx_score_topk(q_tok[j], k_I, w_tok[j], TOPK, q_pos0=p0 + j, out=idx_u[j], workspace=ws)
        for l, (Q, K, V) in enumerate(att):
            for j in range(m):
                dsa.sparse_attn_topk(Q_tok[l][j], K, V, idx_u[j], o_dtype=torch.bfloat16, out=O1[j], workspace=ws)

    res = {}
    for name, fn in (("shared", shared), ("unshared", unshared)):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = 10
        a.record()
        for _ in range(n):
            fn()
        b.record()
        torch.cuda.synchronize()
        dsa.check_status(ws)
        res[name] = a.elapsed_time(b) / n
    del att, Q_tok, k_I
    torch.cuda.empty_cache()
    return {"workload": f"multi-token decode: B={B} sequences verify {m} draft tokens at a {Lc}-token cache, "
                        f"{nl} layers FSSS, H_I={H_I} d_I={D_I} top-{TOPK}, GQA {HQ}Q/{HKV}KV d={DH}",
            "shared_ms_per_step": round(res["shared"], 4),
            "shared_tok_per_s": round(B * m / (res["shared"] / 1e3), 1),
            "unshared_ms_per_step": round(res["unshared"], 4),
            "unshared_tok_per_s": round(B * m / (res["unshared"] / 1e3), 1),
            "speedup": round(res["unshared"] / res["shared"], 3)}


def run_paged(args, dev):
    """Serving-style decode: 64 sequences of different lengths (seeded, 100K-200K tokens) whose
    k_I and K/V caches sit in a shared pool of 64-token pages in shuffled order; one new token each,
    4 layers FSSS (paged decode indexer once, paged gather attention on every layer)."""
    import numpy as np
    import torch
    from long_context_dsa_b200 import dsa, synth

    B, Lmax, P, nl = 64, 200000, 64, 4
    rng = np.random.default_rng(4000)
    lens = rng.integers(100000, Lmax + 1, size=B).astype(np.int32)
    pages = (lens + P - 1) // P
    num_pages = int(pages.sum())
    max_pages = int(pages.max())
    perm = torch.from_numpy(rng.permutation(num_pages).astype(np.int64)).to(dev)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    rows = []  # pool row of every cached token, sequence by sequence
    off = 0
    for b in range(B):
        table[b, :pages[b]] = torch.arange(off, off + pages[b], dtype=torch.int32)
        off += int(pages[b])
    table = table.to(dev)
    table = torch.where(table >= 0, perm[table.clamp(min=0).long()].int(), table)
    for b in range(B):
        t = torch.arange(int(lens[b]), device=dev)
        rows.append(table[b, t // P].long() * P + t % P)

    def to_pool(x):  # [B, Lmax, ...] contiguous cache -> [num_pages * P, ...] pool
        pool = torch.zeros((num_pages * P,) + tuple(x.shape[2:]), dtype=x.dtype, device=dev)
        for b in range(B):
            pool[rows[b]] = x[b, :int(lens[b])]
        return pool

    gen = synth.StructuredIndexer("paged200k", B, Lmax, H_I, D_I, r=32, base_std=1.0, noise_std=SIGMA_200K,
                                  device=dev,
                                  seed=4000)
    k_pool = to_pool(gen.keys(0)).view(num_pages, P, D_I)
    q = torch.stack([gen.queries(0, int(n) - 1, int(n))[0][b, 0] for b, n in enumerate(lens)]).contiguous()
    w = torch.stack([gen.w[b, int(n) - 1] for b, n in enumerate(lens)]).contiguous()
    del gen
    layers = []
    for l in range(nl):
        _, K, V = synth.attention_inputs("paged200k", l, B, 1, Lmax, HQ, HKV, DH, DH, device=dev, seed=4000)
        Kp = to_pool(K).view(num_pages, P, HKV, DH)
        del K
        Vp = to_pool(V).view(num_pages, P, HKV, DH)
        del V
        Q = synth.normal((B, HQ, DH), synth.seed_for(4000, "paged200k", l, "Qdec"), dev, dtype=torch.bfloat16)
        layers.append((Q, Kp, Vp))
        torch.cuda.empty_cache()
    seq = torch.from_numpy(lens).to(dev)
    idx = torch.empty((B, TOPK), dtype=torch.int32, device=dev)
    O = torch.empty((B, HQ, DH), dtype=torch.bfloat16, device=dev)
    max_len = int(lens.max())
    ws = torch.zeros(max(dsa.idx_score_topk_paged_workspace_size(B, max_len, H_I, D_I, TOPK),
                         dsa.sparse_attn_topk_workspace_size(B, 1, num_pages * P, HQ, HKV, DH, DH, TOPK)),
                     dtype=torch.uint8, device=dev)

    def step(evs=None):
        if evs:
            evs[0].record()
        dsa.idx_score_topk_paged(q, k_pool, table, seq, w, TOPK, max_len, out=idx, workspace=ws)
        if evs:
            evs[1].record()
        for (Q, Kp, Vp) in layers:
            dsa.sparse_attn_topk_paged(Q, Kp, Vp, table, seq, idx, o_dtype=torch.bfloat16, out=O, workspace=ws)
        if evs:
            evs[2].record()

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    n = 10
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(n):
        step(evs if i == n - 1 else None)
    b.record()
    torch.cuda.synchronize()
    dsa.check_status(ws)
    ms = a.elapsed_time(b) / n
    kbytes = int(lens.sum()) * D_I * 2
    attn_ms = evs[1].elapsed_time(evs[2])
    idx_ms = evs[0].elapsed_time(evs[1])

    # the same step with the K/V cache stored as E4M3 codes + one scale per (token, KV head)
    layers8 = []
    for i in range(nl):
        Q, Kp, Vp = layers[i]
        layers[i] = None
        K8, ks = synth.quantize_e4m3_rows(Kp)
        del Kp
        torch.cuda.empty_cache()
        V8, vs = synth.quantize_e4m3_rows(Vp)
        del Vp
        torch.cuda.empty_cache()
        layers8.append((Q, K8, ks, V8, vs))

    def step8(evs=None):
        if evs:
            evs[0].record()
        dsa.idx_score_topk_paged(q, k_pool, table, seq, w, TOPK, max_len, out=idx, workspace=ws)
        if evs:
            evs[1].record()
        for (Q, K8, ks, V8, vs) in layers8:
            dsa.sparse_attn_topk_paged_e4m3(Q, K8, ks, V8, vs, table, seq, idx, o_dtype=torch.bfloat16, out=O,
                                            workspace=ws)
        if evs:
            evs[2].record()

    for _ in range(3):
        step8()
    torch.cuda.synchronize()
    a.record()
    for i in range(n):
        step8(evs if i == n - 1 else None)
    b.record()
    torch.cuda.synchronize()
    dsa.check_status(ws)
    ms8 = a.elapsed_time(b) / n
    attn8_ms = evs[1].elapsed_time(evs[2])
    gathered = B * TOPK * HKV * 2 * DH * nl           # K and V rows of every selected token (all lengths >= k)
    del layers8, k_pool
    torch.cuda.empty_cache()
    return {"workload": f"paged decode: B={B} sequences of {int(lens.min())}-{int(lens.max())} tokens "
                        f"(mean {int(lens.mean())}) in shuffled {P}-token pages, 4 layers FSSS, "
                        f"H_I={H_I} d_I={D_I} top-{TOPK}, GQA {HQ}Q/{HKV}KV d={DH}",
            "tok_per_s": round(B / (ms / 1e3), 1), "ms_per_step": round(ms, 4),
            "indexer_ms": round(idx_ms, 4),
            "attention_ms": round(attn_ms, 4),
            "attention_gathered_gbs": round(2 * gathered / (attn_ms / 1e3) / 1e9, 1),
            "indexer_gbs": round(kbytes / (idx_ms / 1e3) / 1e9, 1),
            "fp8_kv": {"tok_per_s": round(B / (ms8 / 1e3), 1), "ms_per_step": round(ms8, 4),
                       "attention_ms": round(attn8_ms, 4),
                       "attention_gathered_gbs": round(gathered / (attn8_ms / 1e3) / 1e9, 1),
                       "cache": "E4M3 codes + fp32 scale per (token, KV head), quantized from the bf16 cache"}}


def run_ctx1m(args, dev):
    """The last 8192-token chunk of a 1M-token chunked prefill: fp8 indexer (H_I=64, d_I=128,
    per-token scales) on 2 of 8 layers (FSSSFSSS), latent attention (576-dim rows, 512-dim values,
    64 query heads) on all 8, against the full 1048576-token caches."""
    import torch
    from long_context_dsa_b200 import dsa, synth

    L1, C, H1, HQ1 = 1 << 20, 8192, 64, 64
    p0 = L1 - C
    gen = synth.StructuredIndexer("ctx1m", 1, L1, H1, D_I, r=32, base_std=1.0, noise_std=SIGMA_1M, device=dev,
                                  seed=3000)
    layers = []
    for l in range(N_LAYERS):
        Lh = {}
        if PATTERN[l] == "F" or l == 1:  # layer 1's own indexer inputs: the overlap check only
            q, w = gen.queries(l, p0, L1)
            Lh["q_I"], Lh["q_scale"] = synth.quantize_e4m3_rows(q)
            Lh["k_I"], Lh["k_scale"] = synth.quantize_e4m3_rows(gen.keys(l))
            Lh["w"] = w
        Lh["Q"], Lh["K"], _ = synth.attention_inputs("ctx1m", l, 1, C, L1, HQ1, 1, 576, None, device=dev, seed=3000)
        Lh["O"] = torch.empty((1, C, HQ1, 512), dtype=torch.bfloat16, device=dev)
        layers.append(Lh)
    del gen
    shape = dsa.group_shape(1, C, p0, L1, H1, D_I, HQ1, 1, 576, 512, TOPK, idx_dtype=dsa.DSA_E4M3,
                            o_dtype=dsa.DSA_BF16)
    ws = torch.zeros(dsa.layer_group_forward_workspace_size(shape), dtype=torch.uint8, device=dev)
    cache = dsa.IndexCache(torch.empty((1, C, TOPK), dtype=torch.int32, device=dev))
    dsa.layer_group_forward(shape, layers, PATTERN, cache, workspace=ws)
    torch.cuda.synchronize()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(3 * N_LAYERS)]
    for e in evs:
        e.record()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    dsa.layer_group_forward(shape, layers, PATTERN, cache, workspace=ws, events=evs)
    t1.record()
    torch.cuda.synchronize()
    dsa.check_status(ws)
    ms = t0.elapsed_time(t1)
    idx_ms = [evs[3 * l].elapsed_time(evs[3 * l + 1]) for l in range(N_LAYERS) if PATTERN[l] == "F"]
    att_ms = [evs[3 * l + 1].elapsed_time(evs[3 * l + 2]) for l in range(N_LAYERS)]
    iflops = 2 * H1 * D_I * sum(range(p0 + 1, L1 + 1))
    abytes = C * TOPK * 576 * 2
    sel = [dsa.idx_score_topk(layers[l]["q_I"], layers[l]["k_I"], layers[l]["w"], TOPK, q_pos0=p0,
                              q_scale=layers[l]["q_scale"], k_scale=layers[l]["k_scale"]) for l in (0, 1)]
    overlap = round(float(dsa.idx_overlap(sel[0], sel[1]).double().mean().item()) / TOPK, 4)
    del layers, sel
    torch.cuda.empty_cache()
    # whole 1M prefill estimate: indexer work grows with the chunk's position, attention does not
    n_chunks = L1 // C
    idx_avg = sum(idx_ms) / len(idx_ms)
    est_s = (sum(att_ms) * n_chunks + idx_avg * 2 * sum((c * C + C / 2) / (p0 + C / 2) for c in range(n_chunks))) / 1e3
    return {"workload": f"last {C}-token chunk of a {L1}-token chunked prefill, 8 layers {PATTERN}, fp8 e4m3 "
                        f"indexer H_I={H1} d_I={D_I} top-{TOPK}, latent attention 576/512 with {HQ1} heads",
            "chunk_ms": round(ms, 3), "chunk_tok_per_s": round(C / (ms / 1e3), 1),
            "indexer_ms_per_f_layer": round(idx_avg, 3),
            "indexer_fp8_tflops": round(iflops / (idx_avg / 1e3) / 1e12, 1),
            # no measured fp8 peak: the measured sustained bf16 peak x the nominal fp8/bf16 ratio (4.5/2.25)
            "indexer_fp8_frac": round(iflops / (idx_avg / 1e3) / 1e12 / (2 * peaks()[2]), 4),
            "indexer_fp8_peak_source": "2 x measured bf16_tflops_sustained (nominal fp8/bf16 ratio)",
            "attention_ms_per_layer": round(sum(att_ms) / len(att_ms), 3),
            "attention_gathered_gbs": round(abytes / (sum(att_ms) / len(att_ms) / 1e3) / 1e9, 1),
            "adjacent_layer_overlap": overlap,
            "full_prefill_estimate_s": round(est_s, 2),
            "full_prefill_estimate_tok_per_s": round(L1 / est_s, 1)}


def run_prefill16k(args, dev):
    """The 16K-token prefill group: L=16384, batch 1, 4 layers FSSS, H_I=64 d_I=128 bf16 indexer,
    top-2048, attention 32 query / 32 KV heads (MHA), d=128, bf16 output."""
    import torch
    from long_context_dsa_b200 import dsa, synth

    L2, H2, HQ2, HKV2, pat = 16384, 64, 32, 32, "FSSS"
    gen = synth.StructuredIndexer("prefill16k", 1, L2, H2, D_I, r=32, base_std=1.0, noise_std=0.2, device=dev,
                                  seed=6000)
    layers = []
    for l in range(4):
        Lh = {}
        Lh["q_I"], Lh["k_I"], Lh["w"] = gen.layer(l)
        Lh["Q"], Lh["K"], Lh["V"] = synth.attention_inputs("prefill16k", l, 1, L2, L2, HQ2, HKV2, DH, DH,
                                                           device=dev, seed=6000)
        Lh["O"] = torch.empty((1, L2, HQ2, DH), dtype=torch.bfloat16, device=dev)
        layers.append(Lh)
    del gen
    shape = dsa.group_shape(1, L2, 0, L2, H2, D_I, HQ2, HKV2, DH, DH, TOPK, o_dtype=dsa.DSA_BF16)
    ws = torch.zeros(dsa.layer_group_forward_workspace_size(shape), dtype=torch.uint8, device=dev)
    cache = dsa.IndexCache(torch.empty((1, L2, TOPK), dtype=torch.int32, device=dev))
    sel = [dsa.idx_score_topk(layers[l]["q_I"], layers[l]["k_I"], layers[l]["w"], TOPK) for l in (0, 1)]
    overlap = round(float(dsa.idx_overlap(sel[0][:, TOPK:].contiguous(), sel[1][:, TOPK:].contiguous()).double().mean().item())
                    / TOPK, 4)
    del sel
    for _ in range(3):
        dsa.layer_group_forward(shape, layers, pat, cache, workspace=ws)
    torch.cuda.synchronize()
    n = 5
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(12)]
    for e in evs:
        e.record()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(n):
        dsa.layer_group_forward(shape, layers, pat, cache, workspace=ws, events=evs if i == n - 1 else None)
    b.record()
    torch.cuda.synchronize()
    dsa.check_status(ws)
    ms = a.elapsed_time(b) / n
    idx_ms = evs[0].elapsed_time(evs[1])
    att_ms = [evs[3 * l + 1].elapsed_time(evs[3 * l + 2]) for l in range(4)]
    hbm, _, bf16_sus, _ = peaks()
    iflops = 2 * H2 * D_I * L2 * (L2 + 1) // 2
    abytes = gathered_rows(L2, TOPK) * HKV2 * 2 * DH * 2
    roof_s = iflops / (bf16_sus * 1e12) + 4 * abytes / (hbm * 1e9)
    del layers
    torch.cuda.empty_cache()
    return {"workload": f"prefill L={L2}, batch 1, 4 layers {pat}, indexer H_I={H2} d_I={D_I} bf16 top-{TOPK}, "
                        f"attention MHA {HQ2}Q/{HKV2}KV d={DH} bf16, bf16 output",
            "tok_per_s": round(L2 / (ms / 1e3), 1), "ms_per_step": round(ms, 3),
            "indexer_ms": round(idx_ms, 3),
            "indexer_tflops": round(iflops / (idx_ms / 1e3) / 1e12, 1),
            "attention_ms_per_layer": round(sum(att_ms) / 4, 3),
            "attention_gathered_gbs": round(abytes / (sum(att_ms) / 4 / 1e3) / 1e9, 1),
            "roofline_ms": round(roof_s * 1e3, 2),
            "roofline_tok_per_s": round(L2 / roof_s, 1),
            "roofline_note": "indexer FLOPs at sustained bf16 + gathered bytes at HBM peak; the 268 MB K/V of a "
                             "layer is largely L2-resident, so the gather can beat its HBM time",
            "adjacent_layer_overlap": overlap}


def _ctx1m_caches(dev, n_kv, n_layers=N_LAYERS, seed=3000):
    """The 1M-context caches: fp8 indexer keys (+ per-token scales) of the F layers and one latent
    [1, n_kv, 576] bf16 cache per layer."""
    import torch
    from long_context_dsa_b200 import synth

    gen = synth.StructuredIndexer("ctx1m", 1, n_kv, 64, D_I, r=32, base_std=1.0, noise_std=SIGMA_1M, device=dev,
                                  seed=seed)
    keys = {}
    for l in range(n_layers):
        if PATTERN[l] == "F":
            keys[l] = synth.quantize_e4m3_rows(gen.keys(l))
    lat = []
    for l in range(n_layers):
        _, KV, _ = synth.attention_inputs("ctx1m", l, 1, 1, n_kv, 64, 1, 576, None, device=dev, seed=seed)
        lat.append(KV)
        torch.cuda.empty_cache()
    return gen, keys, lat


def _finite(x, nd):
    """x rounded to nd places, or None when it is not a finite number."""
    import math
    return round(x, nd) if math.isfinite(x) else None


def decode_graph_ms(run_steps, steps, ws, reps=5):
    """Capture `run_steps` (issues `steps` decode steps through the library on the current stream)
    into one CUDA graph, replay it and return ms per step (CUDA events around the replays)."""
    import torch
    from long_context_dsa_b200 import dsa

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run_steps()  # warm every launch path on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            run_steps()
    except Exception as e:  # reported, not fatal: the eager numbers stand on their own
        torch.cuda.synchronize()
        print(f"decode graph capture failed: {e}", file=sys.stderr)
        return float("nan")
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    dsa.check_status(ws)
    ms = a.elapsed_time(b) / (reps * steps)
    del g
    return ms


def run_decode1m(args, dev):
    """Decode after the 1M-token prefill: 32 steps, batch 1, the new token at positions 1048576 ..
    1048607 (the cache grows from 1048577 to 1048608 tokens); 8 layers FSSSFSSS, fp8 indexer H_I=64
    d_I=128 top-2048 (split decode kernel), latent attention 64 heads (split ranges + merge)."""
    import torch
    from long_context_dsa_b200 import dsa, synth

    L1, steps, H1, HQ1 = 1 << 20, 32, 64, 64
    n_max = L1 + steps
    gen, keys, lat = _ctx1m_caches(dev, n_max)
    qi = {}
    for l in keys:
        q, w = gen.queries(l, L1, n_max)                     # the 32 decode tokens' indexer queries
        q8, qs = synth.quantize_e4m3_rows(q)
        qi[l] = (q8, qs, w)
    del gen
    Qd = [synth.normal((1, steps, HQ1, 576), synth.seed_for(3000, "dec1m", l, "Q"), dev, dtype=torch.bfloat16)
          for l in range(N_LAYERS)]
    O = torch.empty((1, 1, HQ1, 512), dtype=torch.bfloat16, device=dev)
    shape0 = dsa.group_shape(1, 1, n_max - 1, n_max, H1, D_I, HQ1, 1, 576, 512, TOPK, idx_dtype=dsa.DSA_E4M3,
                             o_dtype=dsa.DSA_BF16)
    ws = torch.zeros(dsa.layer_group_forward_workspace_size(shape0), dtype=torch.uint8, device=dev)
    cache = dsa.IndexCache(torch.empty((1, 1, TOPK), dtype=torch.int32, device=dev))

    def step(s, evs=None):
        n_kv = L1 + s + 1
        shape = dsa.group_shape(1, 1, n_kv - 1, n_kv, H1, D_I, HQ1, 1, 576, 512, TOPK, idx_dtype=dsa.DSA_E4M3,
                                o_dtype=dsa.DSA_BF16)
        layers = []
        for l in range(N_LAYERS):
            Lh = {"Q": Qd[l][:, s:s + 1], "K": lat[l][:, :n_kv], "V": None, "O": O}
            if l in keys:
                q8, qs, w = qi[l]
                Lh.update(q_I=q8[:, s:s + 1], q_scale=qs[:, s:s + 1], w=w[:, s:s + 1],
                          k_I=keys[l][0][:, :n_kv], k_scale=keys[l][1][:, :n_kv])
            layers.append(Lh)
        return dsa.layer_group_forward(shape, layers, PATTERN, cache, workspace=ws, events=evs)

    for s in range(3):
        step(s)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3 * N_LAYERS)] for _ in range(steps)]
    for es in evs:
        for e in es:
            e.record()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for s in range(steps):
        step(s, evs[s])
    b.record()
    torch.cuda.synchronize()
    dsa.check_status(ws)
    ms = a.elapsed_time(b) / steps
    idx_ms = sum(es[3 * l].elapsed_time(es[3 * l + 1]) for es in evs for l in range(N_LAYERS)) / steps
    att_ms = sum(es[3 * l + 1].elapsed_time(es[3 * l + 2]) for es in evs for l in range(N_LAYERS)) / steps
    # the same 32 steps captured once into a CUDA graph and replayed: at batch 1 a step is ~20 small
    # launches, so the host's launch rate matters; the graph removes it
    graph_ms = decode_graph_ms(lambda: [step(s) for s in range(steps)], steps, ws)
    hbm = peaks()[0]
    n_f = PATTERN.count("F")
    kbytes = n_f * (L1 + steps // 2) * (D_I + 4)            # fp8 keys + fp32 scales per F layer
    abytes = N_LAYERS * TOPK * 576 * 2                      # the selected latent rows of every layer
    bound_s = (kbytes + abytes) / (hbm * 1e9)
    del lat, keys, qi, Qd
    torch.cuda.empty_cache()
    return {"workload": f"{steps} decode steps after a {L1}-token prefill, batch 1, 8 layers {PATTERN}, fp8 e4m3 "
                        f"indexer H_I={H1} d_I={D_I} top-{TOPK}, latent attention 576/512 with {HQ1} heads",
            "tok_per_s": round(1e3 / ms, 1), "ms_per_step": round(ms, 4),
            "indexer_ms_per_step": round(idx_ms, 4), "attention_ms_per_step": round(att_ms, 4),
            "graph_tok_per_s": _finite(1e3 / graph_ms, 1), "graph_ms_per_step": _finite(graph_ms, 4),
            "hbm_bound_ms_per_step": round(bound_s * 1e3, 4),
            "frac_of_hbm_bound": round(bound_s * 1e3 / ms, 4),
            "graph_frac_of_hbm_bound": _finite(bound_s * 1e3 / graph_ms, 4),
            "bound_note": "fp8 keys + scales of the 2 F layers and 2048 latent rows of each of 8 layers, read "
                          "once at measured HBM bandwidth"}


def run_ctx1m_full(args, dev):
    """The whole 1M-token chunked prefill, measured: 128 chunks of 8192 query rows, each chunk one
    layer_group_forward over 8 layers FSSSFSSS (fp8 indexer H_I=64 on the 2 F layers, latent attention
    with 64 heads on all 8) against the caches up to the chunk's end.  Keys and latent caches are the
    full 1M-token tensors; every chunk's indexer queries are its own rows; the attention queries of one
    chunk per layer are reused by every chunk (they set no control flow)."""
    import torch
    from long_context_dsa_b200 import dsa, synth

    L1, C, H1, HQ1 = 1 << 20, 8192, 64, 64
    n_chunks = L1 // C
    gen, keys, lat = _ctx1m_caches(dev, L1)
    qi = {}
    for l in keys:
        q8 = torch.empty((1, L1, H1, D_I), dtype=torch.uint8, device=dev)
        qs = torch.empty((1, L1, H1), dtype=torch.float32, device=dev)
        for c in range(n_chunks):
            q, _ = gen.queries(l, c * C, (c + 1) * C)
            q8[:, c * C:(c + 1) * C], qs[:, c * C:(c + 1) * C] = synth.quantize_e4m3_rows(q)
        qi[l] = (q8, qs, gen.w.contiguous())
    del gen
    torch.cuda.empty_cache()
    Qc = [synth.normal((1, C, HQ1, 576), synth.seed_for(3000, "ctx1m_full", l, "Q"), dev, dtype=torch.bfloat16)
          for l in range(N_LAYERS)]
    Oc = [torch.empty((1, C, HQ1, 512), dtype=torch.bfloat16, device=dev) for _ in range(N_LAYERS)]
    shape_max = dsa.group_shape(1, C, L1 - C, L1, H1, D_I, HQ1, 1, 576, 512, TOPK, idx_dtype=dsa.DSA_E4M3,
                                o_dtype=dsa.DSA_BF16)
    ws = torch.zeros(dsa.layer_group_forward_workspace_size(shape_max), dtype=torch.uint8, device=dev)
    cache = dsa.IndexCache(torch.empty((1, C, TOPK), dtype=torch.int32, device=dev))

    def chunk(c, evs=None):
        p0, n_kv = c * C, (c + 1) * C
        shape = dsa.group_shape(1, C, p0, n_kv, H1, D_I, HQ1, 1, 576, 512, TOPK, idx_dtype=dsa.DSA_E4M3,
                                o_dtype=dsa.DSA_BF16)
        layers = []
        for l in range(N_LAYERS):
            Lh = {"Q": Qc[l], "K": lat[l][:, :n_kv], "V": None, "O": Oc[l]}
            if l in qi:
                q8, qs, w = qi[l]
                Lh.update(q_I=q8[:, p0:n_kv], q_scale=qs[:, p0:n_kv], w=w[:, p0:n_kv],
                          k_I=keys[l][0][:, :n_kv], k_scale=keys[l][1][:, :n_kv])
            layers.append(Lh)
        return dsa.layer_group_forward(shape, layers, PATTERN, cache, workspace=ws, events=evs)

    chunk(0)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3 * N_LAYERS)] for _ in range(n_chunks)]
    for es in evs:
        for e in es:
            e.record()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for c in range(n_chunks):
        chunk(c, evs[c])
    b.record()
    torch.cuda.synchronize()
    dsa.check_status(ws)
    ms = a.elapsed_time(b)
    idx_ms = sum(es[3 * l].elapsed_time(es[3 * l + 1]) for es in evs for l in range(N_LAYERS))
    att_ms = sum(es[3 * l + 1].elapsed_time(es[3 * l + 2]) for es in evs for l in range(N_LAYERS))
    iflops = PATTERN.count("F") * 2 * H1 * D_I * L1 * (L1 + 1) // 2
    abytes = N_LAYERS * gathered_rows(L1, TOPK) * 576 * 2
    del lat, keys, qi, Qc, Oc
    torch.cuda.empty_cache()
    return {"workload": f"{L1}-token chunked prefill in {n_chunks} chunks of {C}, 8 layers {PATTERN}, fp8 e4m3 "
                        f"indexer H_I={H1} d_I={D_I} top-{TOPK}, latent attention 576/512 with {HQ1} heads",
            "seconds": round(ms / 1e3, 3), "tok_per_s": round(L1 / (ms / 1e3), 1),
            "indexer_s": round(idx_ms / 1e3, 3), "attention_s": round(att_ms / 1e3, 3),
            "indexer_fp8_tflops": round(iflops / (idx_ms / 1e3) / 1e12, 1),
            "attention_gathered_gbs": round(abytes / (att_ms / 1e3) / 1e9, 1)}


def run_cp(args, rank, world, local_rank):
    """Context-parallel prefill of ONE 200K-token sequence split over the ranks (strong
    scaling): every rank owns two zig-zag blocks of query rows, the keys (k_I of the F
    layers, K and V of every layer) are all-gathered inside each step, then each rank runs
    the layer group on its blocks as chunks of prefill.  With one rank the gather is the
    local buffer itself and the step is the sequence in two chunks."""
    import torch
    from long_context_dsa_b200 import context_parallel as cp
    from long_context_dsa_b200 import dsa, replicas

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    plan = cp.make_plan(L, world, rank)
    full = make_layers(dev, rank=0, keep_indexer_all=False)   # the same sequence on every rank
    layers, local_keys, gbufs = [], [], []
    for Lh in full:
        d = {n: cp.local_rows(Lh[n], plan) for n in ("q_I", "w", "Q") if n in Lh}
        d["O"] = torch.empty((2, plan.blk, HQ, DH), dtype=torch.bfloat16, device=dev)
        kl = {n: cp.local_rows(Lh[n], plan) for n in ("k_I", "K", "V") if n in Lh}
        layers.append(d)
        local_keys.append(kl)
        gbufs.append({n: (torch.empty((2 * world, plan.blk) + tuple(t.shape[2:]), dtype=t.dtype, device=dev)
                          if world > 1 else None) for n, t in kl.items()})
    del full
    torch.cuda.empty_cache()
    gather_bytes = sum(t.numel() * t.element_size() for kl in local_keys for t in kl.values()) * (world - 1)
    ws = torch.zeros(cp.workspace_size(plan, H_I, D_I, HQ, HKV, DH, DH, TOPK, o_dtype=dsa.DSA_BF16),
                     dtype=torch.uint8, device=dev)
    cache_buf = torch.empty((2, plan.blk, TOPK), dtype=torch.int32, device=dev)

    def step():
        for d, kl, gb in zip(layers, local_keys, gbufs):
            for n, t in kl.items():
                d[n] = cp.allgather_keys(t, plan, out=gb[n])
        return cp.layer_group_forward(plan, layers, PATTERN, cache_buf, ws, H_I, D_I, HQ, HKV, DH, DH, TOPK,
                                      o_dtype=dsa.DSA_BF16, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    dsa.check_status(ws)
    replicas.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    launches = 0
    for _ in range(args.steps):
        n_idx, n_attn = step()
        launches += n_idx + n_attn
    t1.record(stream)
    torch.cuda.synchronize()
    replicas.barrier()
    dsa.check_status(ws)
    ms = replicas.max_over_ranks(t0.elapsed_time(t1), dev) / args.steps
    work = [cp.indexer_work(cp.make_plan(L, world, r)) for r in range(world)]
    return {"metric": METRIC, "value": round(L / (ms / 1e3), 1), "unit": "tok/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded structured generator; no dataset or trained weights)",
            "config": {"workload": WORKLOAD + "; one sequence split over the ranks in zig-zag blocks",
                       "seq_len": L, "global_batch": 1, "layers": N_LAYERS, "pattern": PATTERN, "topk": TOPK,
                       "parallelism": f"context-parallel x{world}", "rows_per_block": plan.blk,
                       "l2": "inputs larger than L2; no flush needed"},
            "gpu_launches": launches,
            "all_gather_bytes_per_rank_per_step": gather_bytes,
            "indexer_work_max_over_mean": round(max(work) / (sum(work) / world), 5)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--ref-rows", type=int, default=24)
    ap.add_argument("--cpu-rows", type=int, default=24, help="oracle rows for cpu_baseline (0 = skip)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--clocks-dir", default=None, help="keep the sampled clock log (clocks_rank<r>.csv) here")
    ap.add_argument("--no-extra", action="store_true", help="skip the decode and 1M-chunk measurements")
    ap.add_argument("--case", default="bench",
                    choices=["bench", "profile", "profile_paged", "decode", "decode_mha", "ctx1m", "mtp", "paged",
                             "prefill16k", "decode1m", "ctx1m_full", "profile_latent", "profile_decode1m", "profile_decode",
                             "cp"],
                    help="profile: small single-kernel launches for ncu captures; decode / ctx1m / ...: only "
                         "that extra measurement, printed as one JSON line; cp: one 200K sequence split over "
                         "the torchrun ranks (context-parallel prefill, strong scaling)")
    args = ap.parse_args()
    if args.case == "profile":
        run_profile_case(args)
        return
    if args.case == "profile_paged":
        run_profile_paged(args)
        return
    if args.case == "profile_decode":
        run_profile_decode(args)
        return
    if args.case == "profile_latent":
        run_profile_latent(args)
        return
    if args.case == "profile_decode1m":
        run_profile_decode1m(args)
        return
    extra_cases = {"decode": run_decode, "decode_mha": run_decode_mha, "ctx1m": run_ctx1m, "mtp": run_mtp,
                   "paged": run_paged, "prefill16k": run_prefill16k, "decode1m": run_decode1m,
                   "ctx1m_full": run_ctx1m_full}
    if args.case in extra_cases:
        import torch
        dev = torch.device("cuda", 0)
        fn = extra_cases[args.case]
        print(json.dumps({"case": args.case, **fn(args, dev)}), flush=True)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local_rank))
    if args.case == "cp":
        out = run_cp(args, rank, world, local_rank)
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps(out), flush=True)
        return
    out, layers = run_gpu(args, rank, world, local_rank)
    if rank == 0 and args.cpu_rows > 0:
        v, total, sample, threads, meas = oracle_sample(layers, args.cpu_rows)
        out["cpu_baseline"] = {"value": round(v, 3), "unit": "tok/s", "cores": threads, "kind": "oracle",
                               "sample": sample, "host": cpu_info()}
    del layers
    if not args.no_extra and world == 1:  # the extra measurements are single-GPU cases
        import torch
        torch.cuda.empty_cache()
        dev = torch.device("cuda", local_rank)
        out["decode"] = run_decode(args, dev)
        out["decode_mha32_b8"] = run_decode_mha(args, dev)
        out["multi_token_decode"] = run_mtp(args, dev)
        out["paged_decode"] = run_paged(args, dev)
        out["context_1m_tail_chunk"] = run_ctx1m(args, dev)
        out["prefill_16k"] = run_prefill16k(args, dev)
        out["decode_after_1m"] = run_decode1m(args, dev)
        out["context_1m_full_prefill"] = run_ctx1m_full(args, dev)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
