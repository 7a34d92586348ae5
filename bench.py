#!/usr/bin/env python
"""Benchmark of the DSA decode step (indexer -> top-k -> sparse MLA) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode32k]
    python bench.py --impl reference ...        # the fp64 CPU oracle arm

One step = one pass of the whole hot path over one batch of the workload
(decode32k: one 32K-context sequence; batched: 32 ragged sequences; fp8: 4
sequences at 128K with an e4m3 indexer cache).  Inputs are seeded synthetic
data drawn on the device; the timed region replays CUDA graphs that hold
exactly K steps, each step reading its own copy of the caches (copies rotate
over more than 3x the L2 size, so every step starts with a cold L2).

Prints one JSON line (rank 0).  Multi-GPU (torchrun): every rank runs its own
replica (the path shards by sequence and has no exchange step), the timed
region is bracketed by barriers and the max over ranks is used.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "DSA decode steps/s @32K ctx (indexer+top-k+sparse MLA); % HBM roofline"
UNIT = "steps/s"
L2_BYTES_DEFAULT = 126 * 1024 * 1024


# ---------------------------------------------------------------- algorithmic work

def stage_bytes(wl, end_pos):
    """Algorithmic HBM bytes per step, per stage and for the whole step.

    Only what the method must move: the indexer key cache (+ e4m3 scales),
    q_I and w, the selected latent rows (576 bf16 each), q and the output.
    Scores and indices are intermediates; the per-stage figures include the
    stage's own output so that each kernel's roofline is stated on what it
    must write."""
    H, k = wl.H, wl.topk
    fp8 = wl.idx_dtype == "e4m3"
    key_row = 128 + 4 if fp8 else 256
    qi = 64 * 128 * (1 if fp8 else 2)
    out_b = 4 if wl.out_dtype == "f32" else 2
    T = wl.T
    idx = topk_b = mla = step = 0
    short = T == 1 and max(end_pos) <= k  # the decode step skips indexer and selection
    for E in end_pos:
        valid_sum = sum(min(E, E - T + t + 1) for t in range(T))
        keff_sum = sum(min(k, E - T + t + 1) for t in range(T))
        idx += E * key_row + T * (qi + 256) + valid_sum * 4
        topk_b += valid_sum * 4 + T * k * 4
        mla += keff_sum * 1152 + T * H * (576 * 2 + 512 * out_b)
        step += (0 if short else E * key_row + T * (qi + 256)) + keff_sum * 1152 + T * H * (576 * 2 + 512 * out_b)
    return {"indexer": idx, "topk": topk_b, "sparse_mla": mla, "step": step}


def oracle_work(wl, end_pos):
    """Multiply-adds of one oracle step (indexer 64*128 per key, MLA H*(576+512) per kept key)."""
    T = wl.T
    w = 0
    for E in end_pos:
        for t in range(T):
            L = E - T + t + 1
            w += L * 8192 + min(wl.topk, L) * wl.H * 1088
    return w


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock, its maximum and the clock-event (throttle) reasons of one GPU,
    sampled every few milliseconds on a background thread through NVML while
    the timed region runs; falls back to `nvidia-smi -lms` when NVML is
    unavailable."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device, period_s=0.005):
        self.device = device
        self.period = period_s
        self.samples = []      # (sm_mhz, max_mhz, reasons_mask)
        self.thread = None
        self.proc = None
        self.stop_flag = False

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.device.index or 0)

    def start(self):
        import threading
        try:
            import pynvml
            h = self._nvml_handle()
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)

            def sample():
                try:
                    self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), mx,
                                         int(get_reasons(h))))
                except Exception:
                    pass

            def loop():
                while not self.stop_flag:
                    sample()
                    time.sleep(self.period)

            self._sample = sample
            sample()  # one sample as the region starts, however short it is
            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        try:  # fallback: nvidia-smi polling
            self.path = os.path.join(ROOT, "gpurun_out", f".clocks_{os.getpid()}.csv")
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.device.index or 0), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=2)
            self._sample()  # and one as it ends
            sm = [x[0] for x in self.samples]
            reasons = sorted({name for _, _, m in self.samples for bit, name in self.REASONS.items() if m & bit})
            return {"sm_mhz": statistics.median(sm) if sm else None,
                    "sm_max_mhz": self.samples[0][1] if self.samples else None,
                    "reasons": reasons, "samples": len(sm), "source": "nvml"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        try:
            os.remove(self.path)
        except OSError:
            pass
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "source": "nvidia-smi"}


# ---------------------------------------------------------------- distributed plumbing

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_max(x: float, world: int, device=None) -> float:
    """Max of a host float over ranks (identity when world == 1)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(steps_per_rank: int, world: int, max_seconds: float) -> float:
    """Whole-job throughput: every rank's steps over the slowest rank's time."""
    return steps_per_rank * world / max_seconds


# ---------------------------------------------------------------- CPU (oracle) timing

def oracle_step_inputs(wl, inp_cpu, budget_work):
    """A bounded sample of one step for the oracle: whole sequences while they
    fit the budget, else a prefix of one sequence's keys (topk and kept rows
    scaled with it).  Returns (sample Inputs, fraction of the full step's work)."""
    from sparse_attention_04_b200 import inputs as I
    full = oracle_work(wl, inp_cpu.end_pos)
    seqs, acc = [], 0
    for b, E in enumerate(inp_cpu.end_pos):
        wk = oracle_work(wl, [E])
        if acc + wk > budget_work and seqs:
            break
        seqs.append(b)
        acc += wk
    if acc <= budget_work:
        eps = [inp_cpu.end_pos[b] for b in seqs]
        sub_wl = I.Workload(wl.name, len(seqs), wl.T, None, None, wl.topk, wl.H, wl.idx_dtype, wl.scale,
                            wl.out_dtype, wl.seed)
        return _slice(inp_cpu, sub_wl, seqs, eps), acc / full
    # one sequence is already over budget: keep a prefix of m-th of its keys
    E = inp_cpu.end_pos[0]
    m = max(1, math.ceil(oracle_work(wl, [E]) / budget_work))
    E2 = max(wl.T, E // m)
    k2 = max(1, wl.topk // m)
    sub_wl = I.Workload(wl.name, 1, wl.T, None, None, k2, wl.H, wl.idx_dtype, wl.scale, wl.out_dtype, wl.seed)
    sub = _slice(inp_cpu, sub_wl, [0], [E2])
    return sub, oracle_work(sub_wl, [E2]) / full


def _slice(inp, wl, seqs, eps):
    import torch
    from sparse_attention_04_b200.inputs import Inputs
    off = inp.offsets.tolist()
    cat = lambda t: torch.cat([t[off[b]:off[b] + e] for b, e in zip(seqs, eps)]).contiguous()
    new_off = [0]
    for e in eps:
        new_off.append(new_off[-1] + e)
    ks = None if inp.k_scale is None else cat(inp.k_scale)
    # the T query rows of a truncated sequence are its last T positions
    return Inputs(wl, eps, torch.tensor(new_off, dtype=torch.int32), inp.q_idx[seqs].contiguous(),
                  inp.w[seqs].contiguous(), cat(inp.k_idx), ks, inp.q[seqs].contiguous(), cat(inp.kv))


def time_oracle(wl, inp_cpu, n_steps, seconds_per_step_budget):
    """Runs n_steps oracle steps on a bounded sample; returns (full steps/s, cores, sample text)."""
    import oracle
    # calibrate the oracle's multiply-add rate on a small slice
    probe_wl_inp, frac0 = oracle_step_inputs(wl, inp_cpu, 2e8)
    t0 = time.perf_counter()
    oracle.decode_step(probe_wl_inp)
    rate = oracle_work(probe_wl_inp.wl, probe_wl_inp.end_pos) / max(time.perf_counter() - t0, 1e-6)
    sample, frac = oracle_step_inputs(wl, inp_cpu, max(1e6, rate * seconds_per_step_budget))
    t0 = time.perf_counter()
    for _ in range(n_steps):
        oracle.decode_step(sample)
    dt = time.perf_counter() - t0
    per_full_step = dt / n_steps / frac
    text = (f"{n_steps} oracle step(s) on {len(sample.end_pos)} sequence(s) with end_pos {sample.end_pos[:4]}"
            f"{'...' if len(sample.end_pos) > 4 else ''}, topk {sample.wl.topk}; time scaled by "
            f"{1 / frac:.2f} (multiply-add count of the full step / the sample's)")
    return 1.0 / per_full_step, oracle.num_threads(), text


# ---------------------------------------------------------------- native arm

def load_peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        return {}


def hbm_peak_of(peaks):
    try:
        return float(peaks["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def measure_decode(args, wl, dev, stream, world, K, W, peaks, with_e2e):
    """Times exactly K decode steps of workload `wl` (CUDA graphs replayed on
    `stream`, every step on its own cold cache copy), then the stages one by
    one.  Returns a dict with the step rate, the per-stage times and
    rooflines, the clock record of the timed region and (with_e2e) the
    end-to-end leg."""
    import torch
    from sparse_attention_04_b200 import _lib, api
    from sparse_attention_04_b200 import inputs as I

    base = I.make_inputs(wl, dev)
    E = base.end_pos
    max_e = max(E)
    sb = stage_bytes(wl, E)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size or L2_BYTES_DEFAULT
    n_copies = max(2, math.ceil(3 * l2 / sb["step"]))
    per_copy = sum(t.numel() * t.element_size() for t in
                   (base.k_idx, base.kv, base.q_idx, base.w, base.q) + ((base.k_scale,) if base.k_scale is not None else ()))
    free, _ = torch.cuda.mem_get_info(dev)
    n_copies = max(2, min(n_copies, int(0.5 * free // per_copy)))
    clone = lambda t: None if t is None else t.clone()
    copies = [base] + [I.Inputs(wl, E, base.offsets, clone(base.q_idx), clone(base.w), clone(base.k_idx),
                                clone(base.k_scale), clone(base.q), clone(base.kv)) for _ in range(n_copies - 1)]
    step = api.DecodeStep(wl.B, max_e, wl.topk, wl.H,
                          torch.float32 if wl.out_dtype == "f32" else torch.bfloat16, dev)
    rows = base.rows

    def one_step(c):
        x = copies[c % n_copies]
        step(x.q_idx, x.w, x.k_idx, x.k_scale, x.q, x.kv, x.offsets, rows, wl.scale)

    one_step(0)
    torch.cuda.synchronize()
    if int(step.status.item()) != 0:
        raise SystemExit(f"{wl.name}: device status " + _lib.status_string(int(step.status.item())))

    G = min(K, args.graph_steps)

    def capture(n, start):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                one_step(start + i)
        return g

    graph_main = capture(G, 0)
    graph_rem = capture(K % G, 0) if K % G else None
    graph_warm = capture(min(W, G), 0) if W > 0 else None
    launches_per_step = _lib.decode_step_launches(wl.B, max_e, wl.topk, wl.H)

    # ---- warm-up (untimed): W steps, then one replay of every graph the
    # timed region replays, so that no graph's first launch (its upload to
    # the device) falls inside the events
    for _ in range(max(1, W // max(1, min(W, G)))):
        if graph_warm is not None:
            graph_warm.replay()
    graph_main.replay()
    if graph_rem is not None:
        graph_rem.replay()
    torch.cuda.synchronize()

    # ---- timed region: exactly K steps (clocks sampled throughout)
    if world > 1:
        torch.distributed.barrier()
    clocks = ClockSampler(dev)
    clocks.start()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(K // G):
            graph_main.replay()
        if graph_rem is not None:
            graph_rem.replay()
        ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    elapsed = ev0.elapsed_time(ev1) / 1e3
    t_max = reduce_max(elapsed, world, dev)
    value = aggregate_value(K, world, t_max)
    ms_per_step = t_max / K * 1e3

    # ---- per-stage durations (same kernels, events between stages, in a graph)
    n_prof = min(64, max(8, K))
    ld = step.ld
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)] for _ in range(n_prof)]
    ws_mla = step.workspace[_lib.decode_step_workspace_layout(wl.B, max_e, wl.topk, wl.H)[3]:]
    g_prof = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_prof, stream=stream):
        for i in range(n_prof):
            x = copies[i % n_copies]
            evs[i][0].record()
            _lib.indexer_scores(x.q_idx, x.w, x.k_idx, x.k_scale, x.offsets, wl.B, 1, rows, step.scores, ld,
                                status=step.status)
            evs[i][1].record()
            _lib.topk(step.scores, ld, x.offsets, wl.B, 1, wl.topk, step.indices, status=step.status)
            evs[i][2].record()
            _lib.sparse_mla(x.q, x.kv, x.offsets, step.indices, wl.B, 1, wl.H, wl.topk, wl.scale, rows,
                            step.out, lse=step.lse, workspace=ws_mla, status=step.status)
            evs[i][3].record()
    clocks_st = ClockSampler(dev)
    clocks_st.start()
    g_prof.replay()
    g_prof.replay()
    torch.cuda.synchronize()
    clk_st = clocks_st.stop()
    names = ["indexer", "topk", "sparse_mla"]
    stage_s = {n: sum(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(n_prof)) / n_prof / 1e3
               for j, n in enumerate(names)}
    if max_e <= wl.topk:
        # short context: the step runs the attention alone (over every
        # position), so its whole time is the attention stage
        names = ["sparse_mla"]
        stage_s = {"sparse_mla": ms_per_step / 1e3}
    dominant = max(stage_s, key=stage_s.get)
    hbm_peak, peak_src = hbm_peak_of(peaks)
    achieved = sb[dominant] / stage_s[dominant] / 1e9
    traffic = load_traffic(wl.name, dominant)
    roofline = {"bound": "hbm", "kernel": dominant, "achieved": round(achieved, 1), "peak": hbm_peak,
                "unit": "GB/s", "frac": round(achieved / hbm_peak, 4), "traffic": traffic,
                "peak_source": peak_src,
                "stage_us": {n: round(v * 1e6, 3) for n, v in stage_s.items()},
                "stage_frac": {n: round(sb[n] / stage_s[n] / 1e9 / hbm_peak, 4) for n in names},
                "step_frac": round(sb["step"] * (value / world) / 1e9 / hbm_peak, 4),
                "stage_clocks": clk_st}
    res = {"value": value, "ms_per_step": ms_per_step, "roofline": roofline, "clocks": clk, "end_pos": E,
           "n_copies": n_copies, "bytes_per_step": sb["step"], "launches": launches_per_step * K,
           "indexer_keys_per_s": round(sum(E) / stage_s["indexer"], 1) if "indexer" in stage_s else None}
    if with_e2e:
        res["e2e"] = run_e2e(args, wl, copies, n_copies, step, stream, dev, K, G, world)
    del g_prof, graph_main, graph_rem, graph_warm, copies
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def decode_config(wl, end_pos, world):
    """The `config` object of a decode line (both arms print the same one)."""
    E = end_pos
    return {"workload": wl.name, "B": wl.B, "end_pos": E if len(E) <= 4 else {"min": min(E), "max": max(E),
                                                                               "sum": sum(E)},
            "topk": wl.topk, "heads": wl.H, "indexer": f"64x128 {wl.idx_dtype}",
            "parallelism": f"replicas x{world}",
            "l2": "cold: every step reads its own copy of the caches, copies rotating over > 3x L2",
            "algorithmic_bytes_per_step": stage_bytes(wl, E)["step"]}


def run_native(args, rank, world, local):
    import torch
    from sparse_attention_04_b200 import inputs as I

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    wl = I.WORKLOADS[args.workload]
    if wl.T != 1:
        run_prefill_only(args, rank, world, dev)
        return
    peaks = load_peaks()
    K, W = args.steps, args.warmup
    stream = torch.cuda.Stream(dev)
    main = measure_decode(args, wl, dev, stream, world, K, W, peaks, with_e2e=True)
    E = main["end_pos"]

    # the other decode workloads, same measurement (no end-to-end leg)
    extra = {}
    if not args.no_extra and args.workload == "decode32k":
        for name in ("batched", "fp8"):
            r = measure_decode(args, I.WORKLOADS[name], dev, stream, world, K, W, peaks, with_e2e=False)
            ewl = I.WORKLOADS[name]
            extra[name] = {"workload": name, "B": ewl.B, "indexer": f"64x128 {ewl.idx_dtype}",
                           "end_pos": r["end_pos"] if len(r["end_pos"]) <= 4 else
                           {"min": min(r["end_pos"]), "max": max(r["end_pos"]), "sum": sum(r["end_pos"])},
                           "steps_per_s": round(r["value"], 2), "ms_per_step": round(r["ms_per_step"], 6),
                           "algorithmic_bytes_per_step": r["bytes_per_step"],
                           "step_frac": r["roofline"]["step_frac"], "stage_us": r["roofline"]["stage_us"],
                           "indexer_keys_per_s": r["indexer_keys_per_s"], "roofline": r["roofline"],
                           "clocks": r["clocks"], "l2": f"cold: {r['n_copies']} rotating cache copies",
                           "gpu_launches": r["launches"]}

    prefill = prestage = None
    if not args.no_prefill:
        clocks = ClockSampler(dev)
        clocks.start()
        prefill = run_prefill(dev, stream, peaks)
        prefill["clocks"] = clocks.stop()
        clocks = ClockSampler(dev)
        clocks.start()
        prestage = run_prestage(dev, stream, peaks)
        prestage["clocks"] = clocks.stop()

    line = {"metric": METRIC, "value": round(main["value"], 2), "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": round(main["ms_per_step"], 6), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if wl.idx_dtype == "bf16" else "e4m3+bf16",
            "data": "synthetic (seeded N(0,1) bf16 caches and queries)",
            "config": decode_config(wl, E, world),
            "cache_copies": main["n_copies"], "roofline": main["roofline"], "e2e": main["e2e"], "gpu_launches": main["launches"],
            "clocks": main["clocks"], "indexer_keys_per_s": main["indexer_keys_per_s"]}
    line.update(extra)
    if prefill is not None:
        line["prefill_indexer"] = prefill
    if prestage is not None:
        line["indexer_prestage"] = prestage
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = I.make_inputs(wl, "cpu")
        v, cores, text = time_oracle(wl, base, n_steps=3, seconds_per_step_budget=args.cpu_seconds / 3)
        line["cpu_baseline"] = {"value": round(v, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": text}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(args, wl, copies, n_copies, step, stream, dev, K, G, world):
    """End to end through the public API (api.HostDecodeStep over the C ABI):
    per step the new token's inputs go host -> device from pinned memory (q_I
    in bf16, w, the new indexer key and latent row by a copy kernel, q by the
    copy engine on a side stream while the indexer and the selection run),
    dsa_cache_append writes the key (e4m3-quantised for the e4m3 cache) and
    latent row into each sequence's last cache row, dsa_quantize_queries
    turns q_I into codes for the e4m3 indexer, the indexer, selection and
    attention run, and the output comes back device -> host by a copy
    kernel.  One CUDA graph of steps; each step starts after the previous
    one has finished."""
    import torch
    from sparse_attention_04_b200 import api
    B, H = wl.B, wl.H
    hs = api.HostDecodeStep(B, max(copies[0].end_pos), wl.topk, H, wl.idx_dtype, step.out.dtype, dev)
    g = torch.Generator().manual_seed(wl.seed + 100)
    hs.host_q_idx.copy_(torch.randn(B, 1, 64, 128, generator=g).to(torch.bfloat16))
    hs.host_w.copy_(copies[0].w.cpu().reshape(B, 1, 64))
    hs.host_q.copy_(torch.randn(B, 1, H, 576, generator=g).to(torch.bfloat16))
    hs.host_k_new.copy_(torch.randn(B, 1, 128, generator=g).to(torch.bfloat16))
    hs.host_kv_new.copy_(torch.randn(B, 1, 576, generator=g).to(torch.bfloat16))
    h2d, d2h = hs.h2d_bytes, hs.d2h_bytes

    def e2e_step(i):
        x = copies[i % n_copies]
        hs(x.k_idx, x.k_scale, x.kv, x.offsets, x.rows, wl.scale)

    Ge = min(G, 256)
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr, stream=stream):
        for i in range(Ge):
            e2e_step(i)
    gr.replay()
    torch.cuda.synchronize()
    reps = max(1, K // Ge)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(reps):
            gr.replay()
        ev1.record(stream)
    torch.cuda.synchronize()
    t = reduce_max(ev0.elapsed_time(ev1) / 1e3, world, dev)
    return {"value": round(aggregate_value(reps * Ge, world, t), 2), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "note": "caches stay resident; per step the new token's q_I bf16, w, key and latent row go in by a "
                    "copy kernel over PCIe and q by the copy engine beside the indexer, dsa_cache_append writes "
                    "the new rows (e4m3 keys quantised), the output comes out by a copy kernel; each step after "
                    "the previous one"}


def prefill_indexer_flops(T, E):
    """Useful indexer flops of one causal prefill: 2*64*128 per (query, visible key)."""
    return 2 * 64 * 128 * sum(min(E, E - T + t + 1) for t in range(T))


def run_prefill(dev, stream, peaks, reps=20):
    """Causal 4K prefill (B=1, T=4096): the indexer against the bf16 tensor
    peak, and the whole staged path (indexer, top-k, sparse MLA) for context.

    Three copies of the inputs and of the score matrix rotate between
    launches (about 400 MB in all, above 3x L2).  Events on the launching
    stream bracket a CUDA graph of `reps` launches."""
    import torch
    from sparse_attention_04_b200 import _lib
    from sparse_attention_04_b200 import inputs as I
    wl = I.WORKLOADS["prefill4k"]
    B, T, H, k = wl.B, wl.T, wl.H, wl.topk
    E = wl.end_pos
    n_copies = 3
    copies = [I.make_inputs(wl, dev)]
    for _ in range(n_copies - 1):
        c = copies[0]
        copies.append(I.Inputs(wl, c.end_pos, c.offsets, c.q_idx.clone(), c.w.clone(), c.k_idx.clone(), None,
                               c.q, c.kv))
    ld = (E + 3) // 4 * 4
    scores = [torch.empty((B * T, ld), dtype=torch.float32, device=dev) for _ in range(n_copies)]
    indices = torch.empty((B * T, k), dtype=torch.int32, device=dev)
    out = torch.empty((B, T, H, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, T, H), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = torch.empty(max(16, _lib.sparse_mla_workspace_size(B, T, H, k)), dtype=torch.uint8, device=dev)

    def indexer(i):
        x = copies[i % n_copies]
        _lib.indexer_scores(x.q_idx, x.w, x.k_idx, None, x.offsets, B, T, x.rows, scores[i % n_copies], ld,
                            status=status)

    def staged(i):
        x = copies[i % n_copies]
        indexer(i)
        _lib.topk(scores[i % n_copies], ld, x.offsets, B, T, k, indices, status=status)
        _lib.sparse_mla(x.q, x.kv, x.offsets, indices, B, T, H, k, wl.scale, x.rows, out, lse=lse, workspace=ws,
                        status=status)

    def timed(fn, n):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                fn(i)
        g.replay()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            ev0.record(stream)
            g.replay()
            ev1.record(stream)
        torch.cuda.synchronize()
        return ev0.elapsed_time(ev1) / 1e3 / n

    def select(i):
        x = copies[i % n_copies]
        _lib.topk(scores[i % n_copies], ld, x.offsets, B, T, k, indices, status=status)

    def attend(i):
        x = copies[i % n_copies]
        _lib.sparse_mla(x.q, x.kv, x.offsets, indices, B, T, H, k, wl.scale, x.rows, out, lse=lse, workspace=ws,
                        status=status)

    t_idx = timed(indexer, reps)
    t_all = timed(staged, max(2, reps // 4))
    t_sel = timed(select, reps)       # the score copies were all written above
    t_att = timed(attend, max(2, reps // 4))
    if int(status.item()) != 0:
        raise SystemExit("prefill: device status " + _lib.status_string(int(status.item())))
    flops = prefill_indexer_flops(T, E)
    try:
        peak, src = float(peaks["bf16_tflops"]), "measured (burst)"
    except Exception:
        peak, src = 1590.0, "fallback"
    achieved = flops / t_idx / 1e12
    # attention: 2*H*(576 + 512) flops per kept (row, key); row t keeps min(t + 1, k) keys
    att_flops = 2 * H * (576 + 512) * sum(min(E - T + t + 1, k) for t in range(T))
    att = att_flops / t_att / 1e12
    return {"workload": "prefill4k", "kernel": "indexer", "bound": "tensor", "us": round(t_idx * 1e6, 2),
            "flops": flops, "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "peak_source": src,
            "staged_step_us": round(t_all * 1e6, 1),
            "stages_us": {"indexer": round(t_idx * 1e6, 1), "topk": round(t_sel * 1e6, 1),
                          "sparse_mla": round(t_att * 1e6, 1)},
            "attention": {"kernel": "sparse_mla", "bound": "tensor", "flops": att_flops, "achieved": round(att, 1),
                          "peak": peak, "unit": "TFLOP/s", "frac": round(att / peak, 4),
                          "traffic": load_traffic("prefill4k", "sparse_mla")},
            "note": "causal lower triangle only; 3 rotating input and score copies"}


def run_prestage(dev, stream, peaks, reps=20):
    """The indexer pre-stage (rotary embedding + Hadamard rotation) over the
    queries of the causal 4K prefill: 4096 rows x 64 heads of 128 bf16, read
    and written once (128 MiB per launch), against the HBM copy peak.  Three
    copies rotate (384 MiB, above 3x L2)."""
    import torch
    from sparse_attention_04_b200 import _lib
    n_rows, V, L, n_copies = 4096, 64, 4096, 3
    g = torch.Generator(device=dev).manual_seed(3)
    xs = [torch.randn(n_rows, V, 128, generator=g, device=dev).to(torch.bfloat16) for _ in range(n_copies)]
    ys = [torch.empty_like(x) for x in xs]
    pos = torch.arange(n_rows, dtype=torch.int32, device=dev)
    theta = 10000.0 ** (-torch.arange(32, dtype=torch.float64, device=dev) / 32)
    ang = torch.arange(L, dtype=torch.float64, device=dev)[:, None] * theta[None]
    rc, rs = torch.cos(ang).float().contiguous(), torch.sin(ang).float().contiguous()
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    with torch.cuda.stream(stream):
        for i in range(3):
            _lib.indexer_prestage(xs[i], pos, rc, rs, y=ys[i], status=status, stream=stream)
        torch.cuda.synchronize()
        gph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gph, stream=stream):
            for i in range(reps):
                _lib.indexer_prestage(xs[i % n_copies], pos, rc, rs, y=ys[i % n_copies], status=status,
                                      stream=stream)
        gph.replay()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        gph.replay()
        ev1.record(stream)
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise SystemExit("prestage: device status " + _lib.status_string(int(status.item())))
    t = ev0.elapsed_time(ev1) / 1e3 / reps
    nbytes = 2 * n_rows * V * 128 * 2
    try:
        peak, src = float(peaks["hbm_gbs"]), "measured"
    except Exception:
        peak, src = 6650.0, "fallback"
    achieved = nbytes / t / 1e9
    return {"workload": "prefill4k queries (4096 x 64 x 128 bf16)", "kernel": "rope_hadamard", "bound": "hbm",
            "us": round(t * 1e6, 2), "bytes": nbytes, "achieved": round(achieved, 1), "peak": peak,
            "unit": "GB/s", "frac": round(achieved / peak, 4), "peak_source": src,
            "vectors_per_s": round(n_rows * V / t, 1)}


def run_prefill_only(args, rank, world, dev):
    """`--workload prefill4k`: the causal prefill indexer alone, as its own JSON line."""
    import torch
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        peaks = {}
    stream = torch.cuda.Stream(dev)
    clocks = ClockSampler(dev)
    clocks.start()
    res = run_prefill(dev, stream, peaks, reps=max(1, args.steps))
    clk = clocks.stop()
    t_max = reduce_max(res["us"] * 1e-6, world, dev)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        line = {"metric": "DSA causal prefill indexer TFLOP/s (T=4096, lower triangle)",
                "value": round(res["flops"] * world / t_max / 1e12, 1), "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": 3, "ms_per_step": round(t_max * 1e3, 4),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded N(0,1) bf16)", "config": {"workload": "prefill4k", "B": 1, "T": 4096,
                                                                     "end_pos": 4096, "heads": 64},
                "roofline": dict({k: res[k] for k in ("bound", "achieved", "peak", "unit", "frac", "peak_source")},
                                 traffic=load_traffic("prefill4k", "indexer")),
                "prefill_indexer": res, "clocks": clk}
        print(json.dumps(line), flush=True)


def load_traffic(workload, kernel):
    """DRAM bytes per launch from the committed ncu summary for this kernel and
    workload, if one exists for the current kernel version; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(path))
        return d.get(workload, {}).get(kernel)
    except Exception:
        return None


# ---------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    """The fp64 oracle, as it stands, on the host cores (rank 0 only)."""
    if rank != 0:
        return
    from sparse_attention_04_b200 import inputs as I
    wl = I.WORKLOADS[args.workload]
    inp = I.make_inputs(wl, "cpu")
    budget = max(0.002, args.reference_seconds / max(1, args.steps + args.warmup))
    import oracle
    # calibrate the multiply-add rate on a sample large enough that fixed
    # costs do not dominate, then run whole steps when they fit the budget
    sample, frac = oracle_step_inputs(wl, inp, 2e8)
    t0 = time.perf_counter()
    oracle.decode_step(sample)
    rate = oracle_work(sample.wl, sample.end_pos) / max(time.perf_counter() - t0, 1e-6)
    sample, frac = oracle_step_inputs(wl, inp, max(1e5, rate * budget))
    for _ in range(args.warmup):
        oracle.decode_step(sample)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.decode_step(sample)
    dt = time.perf_counter() - t0
    value = args.steps * frac / dt
    text = (f"each step: the oracle on {len(sample.end_pos)} sequence(s), end_pos {sample.end_pos[:4]}, "
            f"topk {sample.wl.topk}; scaled by {1 / frac:.2f} (multiply-add count of the full step / the sample's)")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 / value, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1))", "config": decode_config(wl, inp.end_pos, world),
            "same_config": frac >= 1.0,
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": text},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--workload", default="decode32k", choices=["decode32k", "batched", "fp8", "tiny", "prefill4k", "decode2k"])
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--graph-steps", type=int, default=500)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--reference-seconds", type=float, default=120.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the causal 4K prefill indexer measurement")
    ap.add_argument("--no-extra", action="store_true", help="skip the batched and fp8 decode measurements")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    rank, world, local = dist_env()
    if world != args.gpus and world != 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_native(args, rank, world, local)


if __name__ == "__main__":
    main()
