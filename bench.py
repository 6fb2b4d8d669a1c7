#!/usr/bin/env python
"""Benchmark: MLA decode over a paged latent cache on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload long|dsv3|ragged|retrofit|tiny|prefill] [--cache bf16|fp8]

A step is one pass of the whole decode path -- absorb-in, split-KV decode, and
the log-sum-exp combine fused with absorb-out (mla_combine_absorb_out; with
--unfused the two run as separate calls) -- over one batch of the workload (default:
batch 16, 128 heads, 65536 cached tokens per sequence, d_c 512, d_R 64,
page_size 64, shuffled page table). Inputs (1.2 GB of latent cache) exceed the
126 MB L2, so no flush is needed between steps. With N GPUs each rank runs its
own replica (no collective on the data path; weak scaling) and the time is the
maximum over ranks. One JSON line is printed by rank 0.

--cache fp8 keeps the latent cache as E4M3 codes with one fp32 scale per token
(k_R stays bf16) and decodes with mla_decode_splitkv_fp8: 644 instead of 1152
bytes of HBM traffic per cached token (d_c 512 workloads only; reported under
its own metric name, not the bf16 headline).

--workload prefill times the decompress branch instead: a step is one prefill
of batch 8 x 4096 prompt tokens (decompression of K_nope / V, then causal
attention), reported as query tokens/s against the bf16 tensor roofline.

--impl reference times the fp64 CPU oracle on the host cores instead (each
step a bounded sample of the same workload) and prints the same line with
"impl": "reference".
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode KV-tokens/s per B200 (bf16) + % of HBM/tensor roofline vs CPU oracle"
FP8_METRIC = ("MLA decode KV-tokens/s per B200 (E4M3 latent cache, bf16 products) + % of HBM/tensor "
              "roofline vs CPU oracle")
UNIT = "KV-tokens/s"
PREFILL_METRIC = "MLA prefill (decompress branch) query tokens/s per B200 (bf16) + % of tensor roofline"
PREFILL_UNIT = "query-tokens/s"
FALLBACK_HBM_GBS = 6650.0
# the decode launch of every EV_EVERY-th timed step is bracketed by CUDA events
EV_EVERY = 8
# working set per step kept above three times the 126 MB L2
L2_FLUSH_BYTES = 3 * 126 * 1024 * 1024
FALLBACK_BF16_TFLOPS = 1590.0

# DRAM bytes per launch of the decode kernel from an ncu capture, keyed by
# (sha256 of the kernel source it was taken on, workload, cache format);
# reported only while the source is unchanged.
TRAFFIC = {
    # decode_pair_kernel<false>, long (B16 L65536): 1,213,058,560 read + 8,914,432 written
    # (captured on source d4f9909abe7a9ad4; the only change since is one comment)
    ('b438ad938357535c', "long", "bf16"): 1221972992,
    # decode_pair_kernel<true>, long, E4M3 cache: 679,790,080 read + 6,549,760 written
    ('b438ad938357535c', "long", "fp8"): 686339840,
}


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (smaller cases for profiling)")
    ap.add_argument("--cache", choices=["bf16", "fp8"], default="bf16",
                    help="latent cache format (fp8: E4M3 codes + per-token scales)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--unfused", action="store_true",
                    help="run combine and absorb-out as two calls instead of the fused one")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    return ap.parse_args()


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0


def _sustained_tflops():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"


def _src_hash():
    h = hashlib.sha256()
    for f in ("decode.cuh", "common.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "mla_latent_kv_18_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _workload_desc(w, lens):
    return (f"{w.name}: batch {w.batch}, n_q {w.n_q}, heads {w.heads}, d_nope {w.d_nope}, "
            f"d_c {w.d_latent}, d_R {w.d_rope}, page {w.page_size}, "
            f"seq {'U[%d,%d]' % w.ragged if w.ragged else w.seq_len}, "
            f"{'identity' if w.table == 'identity' else 'shuffled'} page table")


class ClockSampler:
    """Samples SM clock and clock-event reasons via NVML during the run (read only)."""

    def __init__(self, index, period_s=0.005):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                util = nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                self.samples.append((time.time(), mhz, reasons, util))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        nv = self.nv
        win = [s for s in self.samples if t0 <= s[0] <= t1] or self.samples[-5:]
        names = {
            "gpu_idle": getattr(nv, "nvmlClocksEventReasonGpuIdle", 0x1),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        seen = set()
        for s in win:
            for k, bit in names.items():
                if s[2] & bit and k != "gpu_idle":
                    seen.add(k)
        return {"sm_mhz": statistics.median([s[1] for s in win]) if win else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(seen), "samples": len(win)}


def _max_over_ranks(values, world, device):
    """Elementwise maximum of a list of floats over all ranks (the job's time is
    its slowest rank's). Identity for one rank; needs an initialised process
    group otherwise (nccl with a CUDA device, gloo with "cpu")."""
    if world == 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def _job_value(world, tokens_per_step, steps, ms):
    """Whole-job throughput: every rank processes its own batch (weak scaling),
    over the slowest rank's time in ms."""
    return world * tokens_per_step * steps / (ms / 1e3)


def _dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _prefill_flops(w, lens):
    """Algorithmic FLOPs of one prefill: decompression (two [L x d_c] x [d_c x 128]
    products per head) and causal attention (192-wide scores, 128-wide values over
    the visible keys only)."""
    dk = 2.0 * float(sum(int(L) for L in lens)) * w.d_latent * w.heads * (w.d_nope + w.d_v)
    vis = float(sum(int(L) * w.n_q - w.n_q * (w.n_q - 1) // 2 for L in lens))
    at = 2.0 * w.heads * vis * ((w.d_nope + w.d_rope) + w.d_v)
    return dk, at


def _prefill_oracle_sample(w, inp, seed, queries=None):
    """The fp64 oracle's decompress branch on one random (sequence, head) pair per
    host thread (the oracle runs one pair per thread), with all queries of each pair
    or `queries` random ones. Returns (query-token rate, threads, description)."""
    import numpy as np
    import oracle
    args = [inp[k] for k in ("q_c", "q_r", "ckv_pool", "kr_pool", "block_table", "seq_lens",
                             "w_uk", "w_uv")]
    rng = np.random.default_rng(seed)
    B, M, H = w.batch, w.n_q, w.heads
    cores = oracle.num_threads()
    pairs = rng.choice(B * H, size=min(cores, B * H), replace=False)
    sel = []
    for ph in pairs:
        b, h = divmod(int(ph), H)
        qs = np.arange(M) if queries is None else np.sort(rng.choice(M, size=queries,
                                                                     replace=False))
        sel.append((b * M + qs.astype(np.int64)) * H + h)
    sel = np.concatenate(sel)
    t0 = time.perf_counter()
    oracle.prefill_decompress(*args, sel=sel)
    dt = time.perf_counter() - t0
    desc = (f"{len(pairs)} random (sequence, head) pairs, one per host thread, "
            f"{'all %d' % M if queries is None else queries} queries of each, fp64 "
            f"decompress-branch oracle (decompression of the pair's whole sequence included), "
            f"{dt:.1f} s; query tokens counted as rows / heads")
    return len(sel) / H / dt, cores, desc


def run_reference(a):
    """Times the fp64 CPU oracle on bounded samples of the workload."""
    world, rank, _ = _dist_init()
    if rank != 0:
        return 0
    import numpy as np
    import oracle
    from mla_latent_kv_18_b200.inputs import make_inputs, workload
    w = workload(a.workload, **({"batch": a.batch} if a.batch > 0 else {}))
    if w.name == "prefill":
        inp = make_inputs(w, seed=0)
        lens = inp["seq_lens"].numpy()
        cores = oracle.num_threads()
        for i in range(a.warmup):
            _prefill_oracle_sample(w, inp, 100 + i, queries=8)
        t0 = time.perf_counter()
        for i in range(a.steps):
            _prefill_oracle_sample(w, inp, i, queries=8)
        dt = time.perf_counter() - t0
        npairs = min(cores, w.batch * w.heads)
        value = a.steps * npairs * 8 / w.heads / dt
        line = {"impl": "reference", "metric": PREFILL_METRIC, "value": value,
                "unit": PREFILL_UNIT, "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup,
                "ms_per_step": 1e3 * dt / max(1, a.steps), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": _workload_desc(w, lens), "batch": w.batch,
                           "seq_len": w.seq_len, "heads": w.heads,
                           "parallelism": "oracle on host cores"},
                "cpu_baseline": {"value": value, "unit": PREFILL_UNIT, "cores": cores,
                                 "kind": "oracle",
                                 "sample": f"per step: {npairs} random (sequence, head) pairs, 8 "
                                           "random queries of each, through the fp64 "
                                           "decompress-branch oracle"},
                "e2e": {"value": value, "unit": PREFILL_UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0
    inp = make_inputs(w, seed=0)
    cores = oracle.num_threads()
    R = w.n_q * w.heads
    rng = np.random.default_rng(0)
    args = [inp[k] for k in ("q_c", "q_r", "ckv_pool", "kr_pool", "block_table", "seq_lens",
                             "w_uk", "w_uv")]
    lens = inp["seq_lens"].numpy()

    def step():
        sel = rng.choice(w.batch * R, size=cores, replace=False)
        oracle.decode_absorbed(*args, sel=sel)
        return float(sum(lens[s // R] for s in sel)) / R

    for _ in range(a.warmup):
        step()
    t0 = time.perf_counter()
    tokens = sum(step() for _ in range(a.steps))
    dt = time.perf_counter() - t0
    value = tokens / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * dt / a.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": _workload_desc(w, lens), "batch": w.batch,
                       "seq_len": w.seq_len or list(w.ragged), "heads": w.heads,
                       "parallelism": "oracle on host cores"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{cores} random (sequence, head) rows per step, each the "
                                       "full absorbed fp64 oracle over the sequence's tokens"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def _quantize_pool(api, d, dims, dev):
    """The E4M3 cache (codes, scales) of every slot of the bf16 c_KV pool, written by
    the library's quantiser through an identity page table (k_R rewritten unchanged)."""
    import torch
    pool = d["ckv_pool"]
    pages = pool.shape[0]
    codes, scales = api.alloc_fp8_cache(pages, pool.shape[2], dev)
    table = torch.arange(pages, dtype=torch.int32, device=dev)[None]
    pos = torch.arange(pages * 64, dtype=torch.int32, device=dev)
    seq = torch.zeros_like(pos)
    api.append_kv_fp8(pool.view(-1, pool.shape[2]), d["kr_pool"].view(-1, d["kr_pool"].shape[2]),
                      seq, pos, codes, scales, d["kr_pool"], table, dims, theta=0.0)
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    return codes, scales


def cpu_baseline(w, inp, target_s):
    """Oracle (absorbed fp64 path, all host cores) on a bounded sample of rows."""
    import numpy as np
    import oracle
    cores = oracle.num_threads()
    R = w.n_q * w.heads
    lens = inp["seq_lens"].numpy()
    args = [inp[k] for k in ("q_c", "q_r", "ckv_pool", "kr_pool", "block_table", "seq_lens",
                             "w_uk", "w_uv")]
    rng = np.random.default_rng(1)
    n = cores
    t0 = time.perf_counter()
    sel = rng.choice(w.batch * R, size=n, replace=False)
    oracle.decode_absorbed(*args, sel=sel)
    dt = time.perf_counter() - t0
    if dt < target_s / 2:
        n = int(min(w.batch * R, max(n, n * target_s / max(dt, 1e-3))))
        sel = rng.choice(w.batch * R, size=n, replace=False)
        t0 = time.perf_counter()
        oracle.decode_absorbed(*args, sel=sel)
        dt = time.perf_counter() - t0
    tokens = float(sum(lens[s // R] for s in sel)) / R
    return {"value": tokens / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n} random (sequence, head) rows of the workload, full absorbed fp64 "
                      f"oracle over each row's tokens, {dt:.1f} s; KV-tokens counted as "
                      "rows x tokens / rows-per-sequence"}


def main():
    a = _args()
    if a.impl == "reference":
        return run_reference(a)

    import torch
    import torch.distributed as dist
    world, rank, local = _dist_init()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=120), device_id=dev)

    from mla_latent_kv_18_b200 import build as mla_build
    mla_build.build()
    from mla_latent_kv_18_b200 import api
    from mla_latent_kv_18_b200.inputs import make_inputs, to_device, workload

    w = workload(a.workload, **({"batch": a.batch} if a.batch > 0 else {}))
    inp = make_inputs(w, seed=rank)
    d = to_device(inp, dev)
    lens = inp["seq_lens"].numpy()
    if w.name == "prefill":
        return main_prefill(a, w, inp, d, lens, world, rank, local, dev)
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    T = api.tile_tokens(dims)
    total_tiles = int(sum((int(L) + T - 1) // T for L in lens))
    dec = api.Decoder(dims, w.batch, d["block_table"].shape[1], total_tiles, dev)
    stream = torch.cuda.current_stream()
    tokens_per_step = float(lens.sum())
    fp8 = a.cache == "fp8"
    if fp8:
        assert w.d_latent == 512, "the E4M3 decode serves d_c 512 workloads"
        d["codes"], d["scales"] = _quantize_pool(api, d, dims, dev)
        del d["ckv_pool"]
    # Model state of one layer: the latent cache and the two absorbed weights. When
    # it fits in L2, the steps walk over several layers' copies (a model's layers
    # each own a cache and weights), so that no step finds its operands in L2.
    state_keys = (("codes", "scales") if fp8 else ("ckv_pool",)) + ("kr_pool", "w_uk", "w_uv")
    layer_bytes = sum(d[k].numel() * d[k].element_size() for k in state_keys)
    n_layers = max(1, math.ceil(L2_FLUSH_BYTES / layer_bytes))
    layers = [d] + [{k: d[k].clone() for k in state_keys} for _ in range(n_layers - 1)]
    cursor = [0]

    def step(ev=None, x=None, out=None):
        x = d if x is None else x            # this step's inputs (q_c, q_r, table, lengths)
        out = dec.out if out is None else out
        m = layers[cursor[0] % n_layers]     # this step's layer (cache and weights)
        cursor[0] += 1
        api.absorb_q(x["q_c"], x["q_r"], m["w_uk"], dims, out=dec.q)
        if ev is not None:
            ev[0].record(stream)
        if fp8:
            api.decode_splitkv_fp8(dec.q, m["codes"], m["scales"], m["kr_pool"], x["block_table"],
                                   x["seq_lens"], dims, dec.num_parts, workspace=dec.workspace)
        else:
            api.decode_splitkv(dec.q, m["ckv_pool"], m["kr_pool"], x["block_table"], x["seq_lens"],
                               dims, dec.num_parts, workspace=dec.workspace)
        if ev is not None:
            ev[1].record(stream)
        if a.unfused:
            api.combine(dec.workspace, x["seq_lens"], dec.max_pages, dims, dec.num_parts,
                        o_lat=dec.o_lat, lse_out=dec.lse)
            api.absorb_out(dec.o_lat, m["w_uv"], dims, out=out)
        else:
            api.combine_absorb_out(dec.workspace, x["seq_lens"], dec.max_pages, dims,
                                   dec.num_parts, m["w_uv"], out=out, lse_out=dec.lse)

    def barrier():
        if world > 1:
            dist.barrier()

    sampler = ClockSampler(local).start()
    for _ in range(max(3, a.warmup)):
        step()
    torch.cuda.synchronize()
    assert api.get_device_error() == 0

    # the decode launch is bracketed by events on every EV_EVERY-th step only: an
    # event between two kernels stops the next one from being launched early
    # (programmatic dependent launch), which the other steps keep
    evs = {i: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for i in range(0, a.steps, EV_EVERY)}
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    start.record(stream)
    for i in range(a.steps):
        step(evs.get(i))
    end.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    barrier()
    ms = start.elapsed_time(end)
    decode_ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in evs.values())
    assert api.get_device_error() == 0

    # end to end through the same calls: every step's inputs come from pinned
    # host memory and its output goes back to pinned host memory, as a serving
    # loop would run it: inputs and outputs double-buffered, the copies on a
    # second stream overlapping the neighbouring steps' compute.
    keys = ("q_c", "q_r", "block_table", "seq_lens")
    h = {k: inp[k].pin_memory() for k in keys}
    h_out = [torch.empty(dec.out.shape, dtype=dec.out.dtype).pin_memory() for _ in range(2)]
    xbuf = [{k: torch.empty_like(d[k]) for k in keys} for _ in range(2)]
    obuf = [torch.empty_like(dec.out) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in h.values())
    d2h = h_out[0].numel() * h_out[0].element_size()
    cstream = torch.cuda.Stream(device=dev)
    loaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    drained = [torch.cuda.Event() for _ in range(2)]
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_steps = max(1, a.steps // 2)

    def load(i):
        j = i % 2
        with torch.cuda.stream(cstream):
            if i >= 2:
                cstream.wait_event(computed[j])   # step i-2 has finished reading buffer j
            for k in keys:
                xbuf[j][k].copy_(h[k], non_blocking=True)
            loaded[j].record(cstream)

    barrier()
    torch.cuda.synchronize()
    e_start.record(stream)
    cstream.wait_event(e_start)   # the copies belong to the timed region too
    load(0)
    for i in range(e_steps):
        j = i % 2
        if i + 1 < e_steps:
            load(i + 1)
        stream.wait_event(loaded[j])
        if i >= 2:
            stream.wait_event(drained[j])         # step i-2's output has left buffer j
        step(x=xbuf[j], out=obuf[j])
        computed[j].record(stream)
        with torch.cuda.stream(cstream):
            cstream.wait_event(computed[j])
            h_out[j].copy_(obuf[j], non_blocking=True)
            drained[j].record(cstream)
    stream.wait_stream(cstream)
    e_end.record(stream)
    torch.cuda.synchronize()
    # the same with every copy in series with the compute (no overlap), fewer steps
    s_steps = max(1, a.steps // 10)
    s_start, s_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    s_start.record(stream)
    for _ in range(s_steps):
        for k in keys:
            xbuf[0][k].copy_(h[k], non_blocking=True)
        step(x=xbuf[0], out=obuf[0])
        h_out[0].copy_(obuf[0], non_blocking=True)
    s_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    e_ms = e_start.elapsed_time(e_end)
    sampler.stop()

    s_ms = s_start.elapsed_time(s_end)
    ms, e_ms, decode_ms, s_ms = _max_over_ranks([ms, e_ms, decode_ms, s_ms], world, dev)
    value = _job_value(world, tokens_per_step, a.steps, ms)
    e2e_value = _job_value(world, tokens_per_step, e_steps, e_ms)
    e2e_serial = _job_value(world, tokens_per_step, s_steps, s_ms)

    hbm, tflops, src = _peaks()
    R = w.n_q * w.heads
    kv_bytes = tokens_per_step * ((w.d_latent + 4 + 2 * w.d_rope) if fp8 else (w.d_latent + w.d_rope) * 2)
    q_bytes = w.batch * R * (w.d_latent + w.d_rope) * 2
    alg_bytes = kv_bytes + q_bytes
    vis = sum(sum(int(L) - w.n_q + i + 1 for i in range(w.n_q)) for L in lens)
    alg_flops = vis * w.heads * (2 * (w.d_latent + w.d_rope) + 2 * w.d_latent)
    achieved = alg_bytes / (decode_ms / 1e3) / 1e9
    tr = TRAFFIC.get((_src_hash(), w.name, a.cache))
    roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "traffic": tr, "kernel": ("decode_pair_kernel<true>" if fp8 else
                                                              "decode_pair_kernel<false>")
            if w.d_latent == 512 else "decode_single_kernel",
            "peak_source": f"{src} (MEASURED_PEAKS.json hbm_gbs)" if src == "measured" else src,
            "algorithmic_bytes_per_launch": alg_bytes,
            "decode_ms_per_launch": decode_ms,
            "tensor_achieved_tflops": alg_flops / (decode_ms / 1e3) / 1e12,
            "tensor_peak_tflops": tflops,
            "tensor_frac": alg_flops / (decode_ms / 1e3) / 1e12 / tflops}

    clocks = sampler.summary(wall0, wall1)
    line = {"metric": FP8_METRIC if fp8 else METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": ms / a.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": _workload_desc(w, lens), "batch": w.batch,
                       "seq_len": w.seq_len or list(w.ragged), "heads": w.heads,
                       "kv_tokens_per_step": tokens_per_step, "num_parts": dec.num_parts,
                       "cache": ("E4M3 c_KV codes + fp32 per-token scales, bf16 k_R (644 B/token)"
                                 if fp8 else "bf16 c_KV and k_R (1152 B/token)"),
                       "l2": ("inputs larger than L2 (latent cache %.2f GB), no flush" % (kv_bytes / 1e9)
                              if n_layers == 1 else
                              "inputs larger than L2: steps cycle over %d layers' copies of the "
                              "latent cache and weights (%.2f GB in all), no flush"
                              % (n_layers, n_layers * layer_bytes / 1e9)),
                       "layers": n_layers,
                       "parallelism": "replicas" if world > 1 else "single",
                       "step_calls": ["mla_absorb_q",
                                      "mla_decode_splitkv_fp8" if fp8 else "mla_decode_splitkv"] +
                                     (["mla_combine", "mla_absorb_out"] if a.unfused
                                      else ["mla_combine_absorb_out"])},
            "roofline": roof,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "copies": "pinned host buffers; inputs and output double-buffered, copies on a "
                              "second stream overlapping the neighbouring steps' compute",
                    "serial_value": e2e_serial,
                    "d2h_bytes_per_step": d2h},
            "clocks": clocks,
            "gpu_launches": (4 if a.unfused else 3) * a.steps}
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, inp, a.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main_prefill(a, w, inp, d, lens, world, rank, local, dev):
    """One step = one prefill of the workload through the decompress branch:
    mla_decompress_kv then mla_prefill_attention."""
    import torch
    import torch.distributed as dist
    from mla_latent_kv_18_b200 import api
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    B, max_pages = d["block_table"].shape
    M, H = w.n_q, w.heads
    ws = api.alloc_prefill_workspace(dims, B, max_pages, dev)
    out = torch.empty(B, M, H, w.d_v, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, M, H, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    tokens_per_step = float(B * M)

    def step(ev=None, x=None, o=None):
        x = d if x is None else x
        o = out if o is None else o
        if ev is not None:
            ev[0].record(stream)
        api.decompress_kv(d["ckv_pool"], x["block_table"], x["seq_lens"], d["w_uk"], d["w_uv"],
                          dims, workspace=ws)
        if ev is not None:
            ev[1].record(stream)
        api.prefill_attention(x["q_c"], x["q_r"], d["kr_pool"], x["block_table"], x["seq_lens"],
                              dims, ws, out=o, lse=lse)
        if ev is not None:
            ev[2].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()

    sampler = ClockSampler(local).start()
    for _ in range(max(3, a.warmup)):
        step()
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(a.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    start.record(stream)
    for i in range(a.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    barrier()
    assert api.get_device_error() == 0
    ms = start.elapsed_time(end)
    dk_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    at_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)

    # end to end: q_c, q_r, table and lengths from pinned host memory, the output back
    # to pinned host memory, double-buffered with the copies on a second stream
    keys = ("q_c", "q_r", "block_table", "seq_lens")
    h = {k: inp[k].pin_memory() for k in keys}
    h_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    xbuf = [{k: torch.empty_like(d[k]) for k in keys} for _ in range(2)]
    obuf = [torch.empty_like(out) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in h.values())
    d2h = h_out[0].numel() * h_out[0].element_size()
    cstream = torch.cuda.Stream(device=dev)
    loaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    drained = [torch.cuda.Event() for _ in range(2)]
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_steps = max(1, min(a.steps // 2, 10))

    def load(i):
        j = i % 2
        with torch.cuda.stream(cstream):
            if i >= 2:
                cstream.wait_event(computed[j])
            for k in keys:
                xbuf[j][k].copy_(h[k], non_blocking=True)
            loaded[j].record(cstream)

    barrier()
    torch.cuda.synchronize()
    e_start.record(stream)
    cstream.wait_event(e_start)
    load(0)
    for i in range(e_steps):
        j = i % 2
        if i + 1 < e_steps:
            load(i + 1)
        stream.wait_event(loaded[j])
        if i >= 2:
            stream.wait_event(drained[j])
        step(x=xbuf[j], o=obuf[j])
        computed[j].record(stream)
        with torch.cuda.stream(cstream):
            cstream.wait_event(computed[j])
            h_out[j].copy_(obuf[j], non_blocking=True)
            drained[j].record(cstream)
    stream.wait_stream(cstream)
    e_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    sampler.stop()
    assert api.get_device_error() == 0
    e_ms = e_start.elapsed_time(e_end)
    ms, e_ms, dk_ms, at_ms = _max_over_ranks([ms, e_ms, dk_ms, at_ms], world, dev)
    value = _job_value(world, tokens_per_step, a.steps, ms)
    e2e_value = _job_value(world, tokens_per_step, e_steps, e_ms)

    _, burst, bsrc = _peaks()
    sust, ssrc = _sustained_tflops()
    dk_fl, at_fl = _prefill_flops(w, lens)
    achieved = at_fl / (at_ms / 1e3) / 1e12
    roof = {"bound": "tensor", "achieved": achieved, "peak": sust, "unit": "TFLOP/s",
            "frac": achieved / sust, "traffic": None, "kernel": "prefill_attn_kernel",
            "peak_source": (f"{ssrc} (MEASURED_PEAKS.json bf16_tflops_sustained: the kernel "
                            "runs back to back for seconds)"),
            "frac_of_burst_peak": achieved / burst,
            "algorithmic_flops_per_launch": at_fl, "attention_ms_per_launch": at_ms,
            "decompress_kernel": {"ms_per_launch": dk_ms, "algorithmic_flops_per_launch": dk_fl,
                                  "achieved_tflops": dk_fl / (dk_ms / 1e3) / 1e12,
                                  "frac": dk_fl / (dk_ms / 1e3) / 1e12 / sust}}
    line = {"metric": PREFILL_METRIC, "value": value, "unit": PREFILL_UNIT, "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms / a.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": _workload_desc(w, lens), "batch": B, "seq_len": w.seq_len,
                       "query_tokens_per_sequence": M, "heads": H,
                       "step_tflop": (dk_fl + at_fl) / 1e12,
                       "l2": "inputs larger than L2 (q_c + q_r %.2f GB, decompressed K/V %.2f GB), "
                             "no flush" % ((d["q_c"].numel() + d["q_r"].numel()) * 2 / 1e9,
                                           ws.numel() / 1e9),
                       "parallelism": "replicas" if world > 1 else "single",
                       "step_calls": ["mla_decompress_kv", "mla_prefill_attention"]},
            "roofline": roof,
            "e2e": {"value": e2e_value, "unit": PREFILL_UNIT, "h2d_bytes_per_step": h2d,
                    "copies": "pinned host buffers; inputs and output double-buffered, copies on a "
                              "second stream overlapping the neighbouring steps' compute",
                    "d2h_bytes_per_step": d2h},
            "clocks": sampler.summary(wall0, wall1),
            "gpu_launches": 2 * a.steps}
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        v, cores, desc = _prefill_oracle_sample(w, inp, 1)
        line["cpu_baseline"] = {"value": v, "unit": PREFILL_UNIT, "cores": cores,
                                "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
