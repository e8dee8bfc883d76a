#!/usr/bin/env python
"""Benchmark of the SemKV mixed-precision KV-cache hot path on B200.

Default workload (the headline line): generation-time quantization on a Llama-3.1-8B-shaped
model, batch 16, 32 layers, 8 KV heads, 32 query heads, head_dim 128, a 32768-token prefill per
sequence, group 64, L_hi 8 / L_lo 5, p 0.25.  One step = one generated token per sequence in every
layer: semkv_append_decode per layer (the token is quantized at the precision its score earns
against the unit's threshold and appended, then GQA decode attention reads the packed cache,
appended token included), the 32 calls captured as one CUDA graph.  The prefill that builds the
cache (semkv_assign_precision + semkv_quantize_pack of every layer) is timed in the same run.

Also reported in the same run (keys of the JSON line):
  per_kernel.prefill_*  selection and quantize/pack GB/s of the 32-layer prefill
  per_kernel.decode_32L the 32 decode_attention calls alone, over the cache the timed steps left
  extras.llama8b_32L    decode attention of all 32 layers per step over a 131072-token cache
                        (B1, G128, L 6/5, p 0.5), the 32 calls as one CUDA graph
  extras.llama8b_1L     one layer (B1, T32768, G64, L 8/5, p 0.25): select + quantize + append_decode
                        as one graph, the per-call split and the quantizer variants
  sweep                 the Mistral-7B-shaped cache (B8, T32768, Student-t values, Zipf(1.0) scores)
                        at 45 points (level pair x p x G): storage ratio against fp16 from the
                        cache's buffer sizes, and decode GB/s

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl semkv|reference] [--workload NAME]

Under torchrun (N > 1) every rank runs the same per-GPU workload on its own data (independent
units, no collective on the data path: weak scaling); the time is the max over ranks.
Throughput unit: GB/s of algorithmic bytes (what the method must move: fp16 K/V read once by the
prefill, packed codes + fp16 scale/zero written once and read once per decode, scores, queries,
bitmap/rank).
"""
from __future__ import annotations

import argparse
import concurrent.futures
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn HBM GB/s & %roofline over packed mixed-precision KV; quantize GB/s"
L2_FLUSH_BYTES = 512 << 20  # > 126 MB L2
HEADLINES = ("gen", "llama8b_32L", "llama8b_1L")


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["semkv", "reference"], default="semkv")
    ap.add_argument("--workload", choices=HEADLINES, default="gen")
    ap.add_argument("--layers", type=int, default=0, help="layers of the multi-layer workloads (0: all)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="only the headline workload")
    ap.add_argument("--profile", action="store_true", help="few steps, no clocks/e2e/cpu/extras (for ncu)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------- algorithmic bytes


def radix_words(L: int, n: int = 128) -> int:
    k = 0
    p = 1
    while p * L <= 2 ** 32:
        p *= L
        k += 1
    return -(-n // k)


def record_bytes(w, L: int, Lv: int | None = None) -> int:
    """K + V record of one token in a segment: the K words of its row, its share of the V column
    words, and the fp16 scale/zero pair per group of each."""
    Lv = Lv or L
    return 4 * radix_words(L, w.D) + 4 * radix_words(Lv) * w.D // 128 + 2 * 4 * (w.D // w.G)


# the quantizer variants timed beside the one-layer step (recent window of the selection; clipped
# range; V level counts of their own for the hi and lo segments)
WINDOW, CLIP, V_LEVELS = 128, 0.9, (4, 2)
# kernels one decode call launches when both segments hold tiles: the hi and lo decode grids, then
# the merge (the committed ncu launch lists show the same kernels)
DECODE_KERNELS_PER_CALL = 3


def alg_bytes(w, T: int, n_hi: int, new_hi: int = 0, appended: bool = False, v_levels=None) -> dict:
    """Algorithmic bytes of one layer, per hot-path step (what the method must move).  With
    `appended`, one generated token per unit follows the prefill (`new_hi` of them on the L_hi grid)
    and the decode reads the cache including it.  v_levels: the V level counts of the two segments,
    when they differ from the K ones."""
    units = w.B * w.H
    lv_hi, lv_lo = v_levels or (w.L_hi, w.L_lo)
    rec_hi, rec_lo = record_bytes(w, w.L_hi, lv_hi), record_bytes(w, w.L_lo, lv_lo)
    cache = units * (n_hi * rec_hi + (T - n_hi) * rec_lo)
    bitmap_rank = units * 2 * 4 * ((T + 31) // 32)
    q = w.B * w.Hq * w.D * 2
    new = new_hi * rec_hi + (units - new_hi) * rec_lo if appended else 0
    return {
        "select": units * 4 * T + bitmap_rank,
        "quantize": units * T * w.D * 2 * 2 + bitmap_rank + cache,
        # the new token's k, v rows and score read, its record written
        "append": units * (w.D * 2 * 2 + 4) + new if appended else 0,
        # the running rule also reads every stored score key and writes the new one
        "append_running": units * (w.D * 2 * 2 + 4) + new + units * 4 * (T + 1) if appended else 0,
        "decode": cache + new + q,
        "cache": cache,
    }


def gen_steps_bytes(w, nh0, nl0, nh1, nl1, steps: int) -> dict:
    """Algorithmic bytes of `steps` generation steps over all layers, from each layer's segment
    counts summed over its units before (nh0, nl0) and after (nh1, nl1) them.  Per step and layer:
    every unit's new k, v rows and score read and its record written (append), then the records of
    every cached token, the new one included, and the fp16 queries read (decode).  The split of the
    new tokens between the grids is taken evenly over the steps (exact in total)."""
    units = w.B * w.H
    rec_hi, rec_lo = record_bytes(w, w.L_hi), record_bytes(w, w.L_lo)
    q = w.B * w.Hq * w.D * 2
    dec = app = 0.0
    for a, b, c, d in zip(nh0, nl0, nh1, nl1):
        dh, dl = c - a, d - b
        assert dh + dl == units * steps, "every unit appends one token per step"
        # step j (1..steps) attends over a + j dh/steps hi and b + j dl/steps lo tokens
        dec += rec_hi * (steps * a + dh * (steps + 1) / 2) + rec_lo * (steps * b + dl * (steps + 1) / 2)
        dec += steps * q
        app += steps * units * (w.D * 2 * 2 + 4) + dh * rec_hi + dl * rec_lo
    return {"decode": dec, "append": app, "total": dec + app}


def decode_bytes_now(w, nh, nl) -> float:
    """Bytes one decode of every layer reads, from the layers' summed segment counts."""
    q = w.B * w.Hq * w.D * 2
    return sum(a * record_bytes(w, w.L_hi) + b * record_bytes(w, w.L_lo) + q for a, b in zip(nh, nl))


def storage_ratio(D: int, G: int, L_hi: int, L_lo: int, p: float, T: int, B: int = 1, H: int = 1) -> float:
    """Storage reduction against fp16 of one layer's cache (K and V at 2 bytes per value), from the
    buffer sizes the library reports for it (semkv_cache_bytes: code words, scale/zero pairs and the
    precision bitmap; a pure host call)."""
    from mixed_precision_kv_semkv_b200 import _lib

    _, ch, cl, tc = _lib.semkv_capacities(T, p)
    s = _lib.CacheStruct(B=B, H=H, Hq=H, D=D, G=G, L_hi=L_hi, L_lo=L_lo, cap_hi=ch, cap_lo=cl, T_cap=tc)
    sizes = dict(zip(_lib.BUF_NAMES, _lib.semkv_cache_bytes(s)))
    packed = sum(sizes[n] for n in ("k_hi", "v_hi", "kz_hi", "vz_hi", "k_lo", "v_lo", "kz_lo", "vz_lo", "bitmap"))
    return B * H * T * D * 2 * 2 / packed


# ---------------------------------------------------------------- ranks (one process per GPU)


def rank_env() -> tuple[int, int, int]:
    """(world size, rank, local rank) from the torchrun environment (1, 0, 0 without it)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(rank: int) -> int:
    """Each rank draws its own independent units (weak scaling: the per-GPU work is fixed)."""
    return 1000003 * rank


def max_over_ranks(value: float, dist=None, device="cpu") -> float:
    """The slowest rank's value (used for the timed region); no data-path collective."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world: int, step_bytes: float, steps: int, total_ms: float) -> float:
    """Whole-job GB/s: every rank moves step_bytes per step; time = the max over ranks."""
    return world * step_bytes * steps / (total_ms * 1e-3) / 1e9


# ---------------------------------------------------------------- clocks


class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.index)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 8]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- the oracle on the host cores


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


class OracleGen:
    """Units of the generation workload on the host, run by the oracle as it stands.

    The units' prefill (selection + quantize/pack, one layer) is built first; each `step` then runs
    one generation step of every unit -- the oracle's append of the unit's next generated token,
    its dequantization of the whole cache and its attention of the g query heads -- with the units
    spread over a pool of threads, one per host core (the oracle's C routines run without the
    interpreter lock).  Inputs come from the seeded generator; nothing here is timed but `step`
    and `prefill_seconds`."""

    def __init__(self, w, n_units: int, steps: int, threads: int, T: int | None = None):
        import numpy as np

        import oracle
        from mixed_precision_kv_semkv_b200 import synth

        self.np, self.oracle, self.synth, self.w = np, oracle, synth, w
        self.T = w.T if T is None else T
        B = max(1, -(-n_units // w.H))
        self.units = [(b, h) for b in range(B) for h in range(w.H)][:n_units]
        self.threads = threads
        self.pool = concurrent.futures.ThreadPoolExecutor(max_workers=threads)
        d = synth.layer_cpu(w, 0, B=B, T=self.T)
        gen = synth.gen_steps_cpu(w, d["K"], 0, 0, steps)
        self.d, self.gen = d, gen
        self.g = w.Hq // w.H
        n_hi = oracle.n_hi(w.p, self.T)
        self.tiles = (-(-(n_hi + steps) // 128), -(-(self.T - n_hi + steps) // 128))
        self.T_cap = -(-(self.T + steps) // 32) * 32
        t0 = time.perf_counter()
        self.states = list(self.pool.map(self._prefill, self.units))
        self.prefill_seconds = time.perf_counter() - t0
        rec_hi, rec_lo = record_bytes(w, w.L_hi), record_bytes(w, w.L_lo)
        n = len(self.units)
        # bytes of the timed prefill: scores and fp16 K/V read, records and bitmap/rank written
        self.prefill_bytes = n * (4 * self.T + self.T * w.D * 2 * 2 + n_hi * rec_hi + (self.T - n_hi) * rec_lo
                                  + 2 * 2 * 4 * ((self.T + 31) // 32))
        self.step_i = 0

    def _prefill(self, bh):
        b, h = bh
        o, w = self.oracle, self.w
        bm, rk, nh, tau, _ = o.select(self.d["scores"][b, h], w.p)
        hi, lo, _ = o.quantize_pack_unit(self.d["K"][b, h].view(self.np.uint16), self.d["V"][b, h].view(self.np.uint16),
                                         bm, w.G, w.L_hi, w.L_lo, *self.tiles)
        return o.UnitState(self.T_cap, bm, rk, nh, self.T - nh, tau, hi, lo)

    def _unit_step(self, args):
        (b, h), st, i, fp64 = args
        o, w, np = self.oracle, self.w, self.np
        nh_before = st.n_hi
        o.append_unit(st, self.gen["k"][i, b, h].view(np.uint16), self.gen["v"][i, b, h].view(np.uint16),
                      float(self.gen["scores"][i, b, h]), w.G, w.L_hi, w.L_lo)
        T = st.n_hi + st.n_lo
        Kh, Vh = o.dequantize_unit(T, w.D, w.G, w.L_hi, w.L_lo, st.bitmap, st.hi, st.lo)
        q = self.gen["q"][i, b, h * self.g:(h + 1) * self.g].view(np.uint16)
        (o.attention_fp64 if fp64 else o.attention_f32)(q, Kh, Vh, self.synth.sm_scale(w.D))
        rec_hi, rec_lo = record_bytes(w, w.L_hi), record_bytes(w, w.L_lo)
        new_rec = rec_hi if st.n_hi > nh_before else rec_lo
        # append: k, v rows and score read, the record written; decode: every record and the queries
        return (w.D * 2 * 2 + 4) + new_rec + st.n_hi * rec_hi + st.n_lo * rec_lo + self.g * w.D * 2

    def step(self, fp64: bool = False) -> tuple[float, float]:
        """One generation step of every unit; (seconds, algorithmic bytes)."""
        i = self.step_i
        self.step_i += 1
        t0 = time.perf_counter()
        nbytes = sum(self.pool.map(self._unit_step, [(u, st, i, fp64) for u, st in zip(self.units, self.states)]))
        return time.perf_counter() - t0, float(nbytes)

    def close(self):
        self.pool.shutdown()


def oracle_gen_baseline(w, seconds_target: float = 15.0, max_steps: int = 20, n_units: int | None = None):
    """The oracle timed on the host's cores on a bounded sample of the generation workload: one
    layer's units (one per core, up to 64), each running generation steps (append + dequantize +
    attention of its g heads), until about `seconds_target` of wall time."""
    cores = host_cores()
    n = n_units or max(w.H, min(64, cores))
    og = OracleGen(w, n, max_steps + 1, threads=min(cores, n))
    try:
        secs = nbytes = secs64 = nbytes64 = 0.0
        steps = 0
        s64, b64 = og.step(fp64=True)  # the parity variant (fp64 attention), one step
        secs64, nbytes64 = s64, b64
        while steps < max_steps and secs < seconds_target:
            s, b = og.step(fp64=False)
            secs += s
            nbytes += b
            steps += 1
    finally:
        og.close()
    return {"gbs": nbytes / secs / 1e9, "gbs_fp64": nbytes64 / secs64 / 1e9, "seconds": secs, "steps": steps,
            "units": n, "threads": og.threads, "prefill_gbs": og.prefill_bytes / og.prefill_seconds / 1e9,
            "sample": f"{n} units (batch row x kv head) of one layer of workload {w.name}, T={og.T}: the prefill "
                      f"(select + quantize/pack), then {steps} generation steps (append + dequantize + fp32-"
                      f"accumulate attention) timed; fp64 attention (the parity variant) one step; units spread "
                      f"over {og.threads} threads"}


# ---------------------------------------------------------------- reference arm


def workload_config(w, world: int) -> dict:
    """The `config` of both arms' JSON lines: the workload, named by what it is and its sizes."""
    shape = (f"B{w.B} H{w.H} Hq{w.Hq} D{w.D}, G{w.G}, L {w.L_hi}/{w.L_lo}, p {w.p}")
    if w.name == "gen":
        text = (f"gen: Llama-3.1-8B-shaped generation, {w.layers} layers, {shape}, {w.T}-token prefill; "
                f"step = one generated token per sequence in every layer")
        step = "semkv_append_decode per layer (append-quantize at the running threshold + GQA decode), one graph"
    elif w.name == "llama8b_32L":
        text = f"llama8b_32L: Llama-3.1-8B-shaped cache, {w.layers} layers, {shape}, T{w.T}"
        step = "semkv_decode_attention per layer, one graph"
    else:
        text = f"{w.name}: Llama-3.1-8B-shaped layer, {shape}, T{w.T}"
        step = ("assign_precision + quantize_pack + append_decode (append_token of one generated token per unit "
                "and decode_attention in one pass)")
    return {"workload": text, "parallelism": f"dp{world} (independent units)", "step": step}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from mixed_precision_kv_semkv_b200 import synth

    w = synth.WORKLOADS["gen"]
    cores = host_cores()
    steps = max(1, min(args.steps, 10))
    warm = max(0, min(args.warmup, 3))
    n = max(w.H, min(32, cores))
    og = OracleGen(w, n, steps + warm + 1, threads=min(cores, n))
    try:
        for _ in range(warm):
            og.step()
        secs = byts = 0.0
        for _ in range(steps):
            s, b = og.step()
            secs += s
            byts += b
    finally:
        og.close()
    gbs = byts / secs / 1e9
    sample = (f"{n} units (batch row x kv head) of one layer per step, T={w.T}: append + dequantize + fp32-"
              f"accumulate attention, units over {og.threads} threads")
    line = {"metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus, "steps": steps, "warmup": warm,
            "ms_per_step": secs / steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic", "impl": "reference",
            "config": dict(workload_config(w, args.gpus), sample=sample),
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": og.threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm: shared pieces


class Gpu:
    """Per-process GPU context: device, stream, L2 flush buffer, rank info."""

    def __init__(self, args):
        import torch

        self.torch = torch
        self.args = args
        self.world, self.rank, self.local = rank_env()
        torch.cuda.set_device(self.local)
        self.dist = None
        if self.world > 1:
            import datetime

            import torch.distributed as dist

            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", self.local))
            self.dist = dist
        self.stream = torch.cuda.current_stream()
        self.flush_buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device="cuda")
        self.flush_sink = torch.empty((), dtype=torch.int64, device="cuda")
        self.seed = rank_seed(self.rank)

    def flush(self):
        """Evict the L2: write 512 MB, then read back the first half of it, so that the next kernel
        finds a cold L2 holding no dirty lines (it does not pay for writing back the flush)."""
        self.flush_buf.zero_()
        self.torch.sum(self.flush_buf[: L2_FLUSH_BYTES // 8], dim=0, out=self.flush_sink)

    def event(self):
        return self.torch.cuda.Event(enable_timing=True)

    def graph(self, fn):
        fn()  # eager once: module loading and kernel attributes happen outside capture
        self.torch.cuda.synchronize()
        g = self.torch.cuda.CUDAGraph()
        with self.torch.cuda.graph(g, capture_error_mode="relaxed"):
            fn()
        return g

    def time_graph(self, g, reps: int, before=(), flush: bool = True) -> float:
        """Average ms of one replay of g (events around it on the launching stream), each rep after
        an optional L2 flush and the untimed graphs `before`."""
        pairs = []
        for _ in range(reps):
            if flush:
                self.flush()
            for b in before:
                b.replay()
            e0, e1 = self.event(), self.event()
            e0.record(self.stream)
            g.replay()
            e1.record(self.stream)
            pairs.append((e0, e1))
        self.torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in pairs) / reps


def hbm_peak():
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return float(peaks["hbm_gbs"]), "measured"
    except (OSError, ValueError, KeyError):
        return 6650.0, "fallback"


def captured_traffic(name: str, kernel_key: str):
    """DRAM bytes per launch of a kernel from the committed ncu capture, if its sources are
    unchanged since (profiles/traffic_<name>.json holds the sources' sha256)."""
    try:
        import hashlib

        prof = json.load(open(os.path.join(ROOT, "profiles", f"traffic_{name}.json")))
        m = hashlib.sha256()
        for f in prof["sources"][kernel_key]:
            m.update(open(os.path.join(ROOT, f), "rb").read())
        if m.hexdigest() == prof["source_sha256"][kernel_key]:
            return prof[kernel_key]
    except (OSError, ValueError, KeyError):
        pass
    return None


def counts(caches):
    """Per layer: (sum of n_hi over units, sum of n_lo over units) (synchronizes)."""
    nh = [int(c.bufs["n_hi"].sum().item()) for c in caches]
    nl = [int(c.bufs["n_lo"].sum().item()) for c in caches]
    return nh, nl


def prefill_layer(gpu, w, cache, d, T, warm: bool = False):
    """semkv_assign_precision then semkv_quantize_pack of one layer, each timed after an L2 flush;
    returns (select ms, quantize ms).  With `warm`, both calls run once untimed first (they write
    the same cache again): the first launch of a kernel loads its module, which must not be timed."""
    from mixed_precision_kv_semkv_b200 import semkv_assign_precision, semkv_quantize_pack

    if warm:
        semkv_assign_precision(cache, d["scores"], T, w.p)
        semkv_quantize_pack(cache, d["K"], d["V"], T)
    gpu.flush()
    e = [gpu.event() for _ in range(3)]
    e[0].record(gpu.stream)
    semkv_assign_precision(cache, d["scores"], T, w.p)
    e[1].record(gpu.stream)
    gpu.flush()  # the quantization reads the fp16 rows from HBM, not from L2
    e[1].synchronize()
    e1b = gpu.event()
    e1b.record(gpu.stream)
    semkv_quantize_pack(cache, d["K"], d["V"], T)
    e[2].record(gpu.stream)
    e[2].synchronize()
    return e[0].elapsed_time(e[1]), e1b.elapsed_time(e[2])


# ---------------------------------------------------------------- GPU arm: generation workload


def run_gen(gpu, w, K: int, W: int, want_e2e: bool):
    """The generation workload: prefill of every layer, then K timed generation steps (each one
    graph of the layers' append_decode calls), plus the decode calls alone and, optionally, the
    end-to-end steps with host buffers."""
    torch = gpu.torch
    from mixed_precision_kv_semkv_b200 import SemkvCache, semkv_append_decode, semkv_decode_attention, synth

    layers = gpu.args.layers or w.layers
    E = min(K, 10) if want_e2e else 0
    S = 1 + W + K + E  # generated tokens per unit: the eager capture step, warm-up, timed, end-to-end
    T, U = w.T, w.B * w.H
    caches, t_sel, t_q = [], [], []
    pool_k = torch.empty((S, layers, w.B, w.H, w.D), dtype=torch.float16, device="cuda")
    pool_v = torch.empty_like(pool_k)
    pool_s = torch.empty((S, layers, w.B, w.H), dtype=torch.float32, device="cuda")
    pool_q = torch.empty((S, layers, w.B, w.Hq, w.D), dtype=torch.float16, device="cuda")
    for layer in range(layers):
        d = synth.layer_gpu(w, gpu.seed, layer=layer)
        cache = SemkvCache.for_prefill(w.B, w.H, w.Hq, w.G, w.L_hi, w.L_lo, T, w.p, extra=S)
        ts, tq = prefill_layer(gpu, w, cache, d, T, warm=layer == 0)
        t_sel.append(ts)
        t_q.append(tq)
        gen = synth.gen_steps_gpu(w, d["K"], gpu.seed, layer, S)
        pool_k[:, layer] = gen["k"]
        pool_v[:, layer] = gen["v"]
        pool_s[:, layer] = gen["scores"]
        pool_q[:, layer] = gen["q"]
        caches.append(cache)
        del d, gen
    torch.cuda.synchronize()
    assert all(c.status() == 0 for c in caches), "device status after the prefill"
    nh_pre, nl_pre = counts(caches)
    nb_layer = alg_bytes(w, T, nh_pre[0] // U)
    prefill = {"select_ms": sum(t_sel), "quantize_ms": sum(t_q),
               "select_gbs": layers * nb_layer["select"] / (sum(t_sel) * 1e-3) / 1e9,
               "quantize_gbs": sum(alg_bytes(w, T, nh // U)["quantize"] for nh in nh_pre) / (sum(t_q) * 1e-3) / 1e9}
    torch.cuda.empty_cache()

    cur_k, cur_v, cur_s, cur_q = (torch.empty_like(x[0]) for x in (pool_k, pool_v, pool_s, pool_q))
    out = torch.empty((layers, w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    ws = caches[0].workspace()
    scale = synth.sm_scale(w.D)
    si = [0]  # next generated token of the pool

    def stage(i):
        cur_k.copy_(pool_k[i])
        cur_v.copy_(pool_v[i])
        cur_s.copy_(pool_s[i])
        cur_q.copy_(pool_q[i])

    def step_calls():
        for layer in range(layers):
            semkv_append_decode(caches[layer], cur_k[layer], cur_v[layer], cur_s[layer], cur_q[layer], scale,
                                out[layer], ws)

    stage(0)
    step_graph = gpu.graph(step_calls)  # the eager call appends pool token 0
    si[0] = 1
    for _ in range(W):
        stage(si[0])
        si[0] += 1
        step_graph.replay()
    torch.cuda.synchronize()
    assert all(c.status() == 0 for c in caches), "device status after the warm-up"
    nh0, nl0 = counts(caches)

    clocks = Clocks(gpu.local)
    if not gpu.args.profile:
        clocks.start()
        time.sleep(0.3)
    if gpu.dist is not None:
        gpu.dist.barrier()
    torch.cuda.synchronize()
    evs = []
    for _ in range(K):
        stage(si[0])  # this step's generated tokens into the graph's input buffers (untimed)
        si[0] += 1
        e0, e1 = gpu.event(), gpu.event()
        e0.record(gpu.stream)
        step_graph.replay()
        e1.record(gpu.stream)
        evs.append((e0, e1))
    torch.cuda.synchronize()
    if gpu.dist is not None:
        gpu.dist.barrier()
    ck = clocks.stop() if not gpu.args.profile else {}
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = max_over_ranks(sum(step_ms), gpu.dist, "cuda")
    nh1, nl1 = counts(caches)
    assert all(c.status() == 0 for c in caches), "device status after the timed steps"
    nb = gen_steps_bytes(w, nh0, nl0, nh1, nl1, K)

    # the decode calls alone (graph of the layers' decode_attention), over the cache as it is now
    def decode_calls():
        for layer in range(layers):
            semkv_decode_attention(caches[layer], cur_q[layer], scale, out[layer], ws)

    dec_graph = gpu.graph(decode_calls)
    dec_ms = gpu.time_graph(dec_graph, reps=min(max(K, 3), 20), flush=False)
    dec_bytes = decode_bytes_now(w, nh1, nl1)

    e2e = None
    if E:
        hk, hv, hs, hq = (x[si[0]:si[0] + E].cpu().pin_memory() for x in (pool_k, pool_v, pool_s, pool_q))
        hout = torch.empty(out.shape, dtype=torch.float32).pin_memory()
        nh2, nl2 = counts(caches)
        torch.cuda.synchronize()
        e0, e1 = gpu.event(), gpu.event()
        e0.record(gpu.stream)
        for i in range(E):
            cur_k.copy_(hk[i], non_blocking=True)
            cur_v.copy_(hv[i], non_blocking=True)
            cur_s.copy_(hs[i], non_blocking=True)
            cur_q.copy_(hq[i], non_blocking=True)
            step_graph.replay()
            hout.copy_(out, non_blocking=True)
        e1.record(gpu.stream)
        e1.synchronize()
        el = max_over_ranks(e0.elapsed_time(e1), gpu.dist, "cuda")
        nh3, nl3 = counts(caches)
        nbe = gen_steps_bytes(w, nh2, nl2, nh3, nl3, E)
        h2d = sum(x[0].numel() * x[0].element_size() for x in (hk, hv, hs, hq))
        e2e = {"value": gpu.world * nbe["total"] / (el * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": hout.numel() * 4, "ms_per_step": el / E,
               "path": "per step: pinned host -> device copies of the step's generated k, v, scores and queries "
                       "(all layers), the step's graph, device -> pinned host copy of every layer's attention "
                       "output"}
        si[0] += E
    assert all(c.status() == 0 for c in caches), "device status at the end"
    del step_graph, dec_graph
    res = {"total_ms": total_ms, "step_bytes": nb["total"] / K, "bytes": nb, "step_ms": step_ms, "clocks": ck,
           "prefill": prefill, "decode_ms": dec_ms, "decode_bytes": dec_bytes, "layers": layers, "e2e": e2e,
           "launches_per_step": layers * DECODE_KERNELS_PER_CALL, "T_end": T + si[0]}
    caches.clear()
    del pool_k, pool_v, pool_s, pool_q, ws, out
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------- GPU arm: 32-layer decode


def run_decode_layers(gpu, w, K: int, W: int):
    """A multi-layer cache (one prefill per layer), then K timed steps of one graph holding every
    layer's semkv_decode_attention."""
    torch = gpu.torch
    from mixed_precision_kv_semkv_b200 import SemkvCache, semkv_decode_attention, synth

    layers = gpu.args.layers or w.layers
    caches, qs, t_sel, t_q = [], [], [], []
    for layer in range(layers):
        d = synth.layer_gpu(w, gpu.seed, layer=layer)
        cache = SemkvCache.for_prefill(w.B, w.H, w.Hq, w.G, w.L_hi, w.L_lo, w.T, w.p)
        ts, tq = prefill_layer(gpu, w, cache, d, w.T, warm=layer == 0)
        t_sel.append(ts)
        t_q.append(tq)
        caches.append(cache)
        qs.append(d["q"].clone())
        del d
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    assert all(c.status() == 0 for c in caches)
    nh, nl = counts(caches)
    out = torch.empty((layers, w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    ws = caches[0].workspace()
    scale = synth.sm_scale(w.D)

    def calls():
        for layer in range(layers):
            semkv_decode_attention(caches[layer], qs[layer], scale, out[layer], ws)

    g = gpu.graph(calls)
    for _ in range(W):
        g.replay()
    ms = gpu.time_graph(g, reps=K, flush=False)  # the step reads every layer's cache: far more than L2
    byts = decode_bytes_now(w, nh, nl)
    U = w.B * w.H
    peak, _ = hbm_peak()
    res = {"ms_per_step": ms, "gbs": byts / (ms * 1e-3) / 1e9, "frac": byts / (ms * 1e-3) / 1e9 / peak,
           "bytes_per_step": byts, "steps": K, "layers": layers,
           "prefill_select_gbs": sum(alg_bytes(w, w.T, a // U)["select"] for a in nh) / (sum(t_sel) * 1e-3) / 1e9,
           "prefill_quantize_gbs": sum(alg_bytes(w, w.T, a // U)["quantize"] for a in nh) / (sum(t_q) * 1e-3) / 1e9,
           "launches_per_step": layers * DECODE_KERNELS_PER_CALL}
    assert all(c.status() == 0 for c in caches)
    del g
    caches.clear()
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------- GPU arm: one-layer step and variants


def run_one_layer(gpu, w, K: int, W: int, variants: bool = True):
    """One layer: select + quantize + append_decode as one graph, timed over K steps with an L2
    flush between them; the per-call split and (with `variants`) the quantizer variants, each call
    from a graph of its own."""
    torch = gpu.torch
    from mixed_precision_kv_semkv_b200 import (SemkvCache, semkv_append_decode, semkv_append_token,
                                               semkv_append_token_running, semkv_assign_precision,
                                               semkv_capacities, semkv_decode_attention, semkv_quantize_pack, synth)

    T = w.T
    d = synth.layer_gpu(w, seed=gpu.seed)
    K_, V_, S_, q = d["K"], d["V"], d["scores"], d["q"]
    gen = synth.gen_steps_gpu(w, K_, seed=gpu.seed, layer=0, steps=1)
    kn, vn, sn = (gen[x][0].contiguous() for x in ("k", "v", "scores"))
    # room for the recent-window variant below; the step itself runs the plain selection
    cache = SemkvCache.for_prefill(w.B, w.H, w.Hq, w.G, w.L_hi, w.L_lo, T, w.p, extra=1, window=WINDOW)
    cache.struct.window = 0
    ws = cache.workspace()
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    out_s = torch.empty_like(out)
    scale = synth.sm_scale(w.D)
    calls = [lambda: semkv_assign_precision(cache, S_, T, w.p),
             lambda: semkv_quantize_pack(cache, K_, V_, T),
             lambda: semkv_append_token(cache, kn, vn, sn),
             lambda: semkv_decode_attention(cache, q, scale, out_s, ws)]
    names = ("select", "quantize", "append", "decode_in_step")
    for c in calls:
        c()
    torch.cuda.synchronize()
    n_hi0 = semkv_capacities(T, w.p)[0]
    new_hi = int((cache.bufs["n_hi"] - n_hi0).sum().item())
    nb = alg_bytes(w, T, n_hi0, new_hi, appended=True)
    step_bytes = nb["select"] + nb["quantize"] + nb["append"] + nb["decode"]
    fused_call = lambda: semkv_append_decode(cache, kn, vn, sn, q, scale, out, ws)  # noqa: E731
    calls[0]()
    calls[1]()
    fused_call()
    torch.cuda.synchronize()
    assert torch.equal(out, out_s), "append+decode in one pass differs from append then decode"
    step_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(step_graph, capture_error_mode="relaxed"):
        calls[0]()
        calls[1]()
        fused_call()
    graphs = []
    for c in calls:
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, capture_error_mode="relaxed"):
            c()
        graphs.append(gr)
    for _ in range(max(W, 3)):
        gpu.flush()
        step_graph.replay()
    torch.cuda.synchronize()
    step_ms = gpu.time_graph(step_graph, reps=K)
    # the append after a fresh prefill each time (its segment and T_cap have room for one token)
    t_call = [gpu.time_graph(g, reps=min(K, 300), before=graphs[:2] if i == 2 else ()) for i, g in enumerate(graphs)]
    per_kernel = {nm: {"ms": t, "gbs": nb[nm.replace("_in_step", "")] / (t * 1e-3) / 1e9}
                  for nm, t in zip(names, t_call)}
    # the fused call and the running append on their own, each after a fresh prefill
    run_call = lambda: semkv_append_token_running(cache, kn, vn, sn, w.p)  # noqa: E731
    graphs[0].replay()
    graphs[1].replay()
    run_graph = gpu.graph(run_call)
    graphs[0].replay()
    graphs[1].replay()
    fused_graph = gpu.graph(fused_call)
    t_run = gpu.time_graph(run_graph, reps=min(K, 300), before=graphs[:2])
    t_fused = gpu.time_graph(fused_graph, reps=min(K, 300), before=graphs[:2])
    graphs[0].replay()
    graphs[1].replay()
    graphs[2].replay()
    t_dec_cold = gpu.time_graph(graphs[3], reps=min(K, 200))
    per_kernel.update({
        "decode_l2_cold": {"ms": t_dec_cold, "gbs": nb["decode"] / (t_dec_cold * 1e-3) / 1e9},
        "append_running": {"ms": t_run, "gbs": nb["append_running"] / (t_run * 1e-3) / 1e9},
        "append_decode": {"ms": t_fused, "gbs": (nb["append"] + nb["decode"]) / (t_fused * 1e-3) / 1e9},
    })
    if variants:
        cache.struct.window = WINDOW
        win_graph = gpu.graph(calls[0])
        cache.struct.window = 0
        calls[0]()
        cache.struct.clip = CLIP
        clip_graph = gpu.graph(calls[1])
        cache.struct.clip = 0.0
        torch.cuda.synchronize()
        t_win = gpu.time_graph(win_graph, reps=min(K, 300))
        t_clip = gpu.time_graph(clip_graph, reps=min(K, 300), before=(graphs[0],))
        cache.struct.L_hi_v, cache.struct.L_lo_v = V_LEVELS
        calls[0]()
        kvq_graph = gpu.graph(calls[1])
        out_v = torch.empty_like(out)
        kv_decode = lambda: semkv_decode_attention(cache, q, scale, out_v, ws)  # noqa: E731
        kvd_graph = gpu.graph(kv_decode)
        cache.struct.L_hi_v, cache.struct.L_lo_v = 0, 0
        t_kvq = gpu.time_graph(kvq_graph, reps=min(K, 300), before=(graphs[0],))
        t_kvd = gpu.time_graph(kvd_graph, reps=min(K, 300), before=(graphs[0], kvq_graph))
        nb_kv = alg_bytes(w, T, n_hi0, v_levels=V_LEVELS)
        cache.struct.k_per_channel = 1
        calls[0]()
        kpq_graph = gpu.graph(calls[1])
        kpd_graph = gpu.graph(kv_decode)
        cache.struct.k_per_channel = 0
        t_kpq = gpu.time_graph(kpq_graph, reps=min(K, 300), before=(graphs[0],))
        t_kpd = gpu.time_graph(kpd_graph, reps=min(K, 300), before=(graphs[0], kpq_graph))
        kpc_range_bytes = w.B * w.H * T * w.D * 2  # the grid pass reads K once more
        per_kernel.update({
            f"select_window{WINDOW}": {"ms": t_win, "gbs": nb["select"] / (t_win * 1e-3) / 1e9},
            f"quantize_clip{CLIP}": {"ms": t_clip, "gbs": nb["quantize"] / (t_clip * 1e-3) / 1e9},
            "quantize_v_levels{}_{}".format(*V_LEVELS): {"ms": t_kvq, "gbs": nb_kv["quantize"] / (t_kvq * 1e-3) / 1e9},
            "decode_v_levels{}_{}".format(*V_LEVELS): {"ms": t_kvd, "gbs": nb_kv["decode"] / (t_kvd * 1e-3) / 1e9},
            "quantize_k_per_channel": {"ms": t_kpq,
                                       "gbs": (nb["quantize"] + kpc_range_bytes) / (t_kpq * 1e-3) / 1e9},
            "decode_k_per_channel": {"ms": t_kpd, "gbs": nb["decode"] / (t_kpd * 1e-3) / 1e9},
        })
    torch.cuda.synchronize()
    assert cache.status() == 0, f"device status {cache.status()}"
    peak, _ = hbm_peak()
    res = {"ms_per_step": step_ms, "gbs": step_bytes / (step_ms * 1e-3) / 1e9, "step_bytes": step_bytes,
           "per_kernel": per_kernel, "quantize_frac": per_kernel["quantize"]["gbs"] / peak,
           "decode_frac": per_kernel["decode_l2_cold"]["gbs"] / peak,
           "timing": "step = one CUDA graph of select, quantize and append_decode, L2 flushed (512 MB written, 256 MB of it read back) "
                     "between steps; per_kernel = each call from a graph of its own, L2 flushed before it"}
    del graphs, step_graph
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------- GPU arm: precision sweep


def run_sweep(gpu, w, reps: int = 20):
    """The Mistral-7B-shaped cache (one layer: batch 8, 8 KV heads, T 32768) at every (level pair,
    p, G) point: prefill, then the decode timed over an L2-cold cache; the storage ratio against
    fp16 comes from the cache's buffer sizes."""
    torch = gpu.torch
    from mixed_precision_kv_semkv_b200 import (SemkvCache, semkv_assign_precision, semkv_decode_attention,
                                               semkv_quantize_pack, synth)

    d = synth.layer_gpu(w, gpu.seed, layer=0)
    T = w.T
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    scale = synth.sm_scale(w.D)
    peak, _ = hbm_peak()
    fp16_bytes = w.B * w.H * T * w.D * 2 * 2
    pts = []
    for (Lh, Ll) in synth.SWEEP_PAIRS:
        for p in synth.SWEEP_P:
            for G in synth.SWEEP_G:
                cache = SemkvCache.for_prefill(w.B, w.H, w.Hq, G, Lh, Ll, T, p)
                semkv_assign_precision(cache, d["scores"], T, p)
                semkv_quantize_pack(cache, d["K"], d["V"], T)
                ws = cache.workspace()
                g = gpu.graph(lambda: semkv_decode_attention(cache, d["q"], scale, out, ws))  # noqa: B023
                ms = gpu.time_graph(g, reps=reps)
                nh = int(cache.bufs["n_hi"].sum().item())
                nl = int(cache.bufs["n_lo"].sum().item())
                assert cache.status() == 0
                wq = type(w)(w.name, w.B, w.H, w.Hq, T, G, Lh, Ll, p)
                byts = nh * record_bytes(wq, Lh) + nl * record_bytes(wq, Ll) + w.B * w.Hq * w.D * 2
                gbs = byts / (ms * 1e-3) / 1e9
                ratio = fp16_bytes / cache.packed_bytes
                assert abs(ratio - storage_ratio(w.D, G, Lh, Ll, p, T, B=w.B, H=w.H)) < 1e-12
                pts.append({"L_hi": Lh, "L_lo": Ll, "p": p, "G": G, "ratio_vs_fp16": ratio,
                            "decode_ms": ms, "decode_gbs": gbs, "decode_frac": gbs / peak})
                del g, cache, ws
    del d
    torch.cuda.empty_cache()
    return pts


# ---------------------------------------------------------------- GPU arm: the JSON line


def run_semkv(args):
    gpu = Gpu(args)
    torch = gpu.torch
    from mixed_precision_kv_semkv_b200 import build, synth

    build.build()
    w = synth.WORKLOADS[args.workload]
    K = 3 if args.profile else args.steps
    W = max(args.warmup, 3)
    want_e2e = not (args.no_e2e or args.profile)
    peak, peak_kind = hbm_peak()
    extras, per_kernel, sweep = {}, {}, None

    if w.name == "gen":
        r = run_gen(gpu, w, K, W, want_e2e)
        value = weak_scaling_value(gpu.world, r["step_bytes"], K, r["total_ms"])
        ms_step = r["total_ms"] / K
        layer_ms = ms_step / r["layers"]
        layer_bytes = r["step_bytes"] / r["layers"]
        dom_name = "semkv_append_decode per layer (k_decode_i8 hi + lo grids, k_decode_merge)"
        ach = layer_bytes / (layer_ms * 1e-3) / 1e9
        per_kernel = {
            "append_decode_layer": {"ms": layer_ms, "gbs": ach},
            "decode_32L": {"ms": r["decode_ms"], "gbs": r["decode_bytes"] / (r["decode_ms"] * 1e-3) / 1e9,
                           "frac": r["decode_bytes"] / (r["decode_ms"] * 1e-3) / 1e9 / peak},
            "prefill_select": {"ms": r["prefill"]["select_ms"], "gbs": r["prefill"]["select_gbs"]},
            "prefill_quantize": {"ms": r["prefill"]["quantize_ms"], "gbs": r["prefill"]["quantize_gbs"],
                                 "frac": r["prefill"]["quantize_gbs"] / peak},
        }
        dec_gbs = per_kernel["decode_32L"]["gbs"]
        launches = r["launches_per_step"] * K
        clocks, e2e = r["clocks"], r["e2e"]
        traffic = captured_traffic("gen", "append_decode")
        cfg_extra = {"l2": "not flushed: a step reads far more than the 126 MB L2",
                     "generated_tokens": f"T grows from {w.T} (prefill) to {r['T_end']} over the run",
                     "timing": "per step: CUDA events around one replay of the step graph; the step's generated "
                               "tokens are staged into the graph's input buffers before the first event"}
        steps_ms = r["step_ms"]
    elif w.name == "llama8b_32L":
        r = run_decode_layers(gpu, w, K, W)
        value = weak_scaling_value(gpu.world, r["bytes_per_step"], K, max_over_ranks(r["ms_per_step"] * K, gpu.dist,
                                                                                      "cuda"))
        ms_step = r["ms_per_step"]
        dom_name = "semkv_decode_attention per layer (k_decode_i8 hi + lo grids, k_decode_merge)"
        ach = r["gbs"]
        dec_gbs = r["gbs"]
        launches = r["launches_per_step"] * K
        clocks, e2e, traffic, steps_ms = {}, None, captured_traffic("llama8b_32L", "decode"), None
        cfg_extra = {"l2": "not flushed: a step reads far more than the 126 MB L2"}
    else:
        r = run_one_layer(gpu, w, K, W)
        value = weak_scaling_value(gpu.world, r["step_bytes"], K, max_over_ranks(r["ms_per_step"] * K, gpu.dist,
                                                                                 "cuda"))
        ms_step = r["ms_per_step"]
        per_kernel = r["per_kernel"]
        dom = max(("select", "quantize", "append_decode"), key=lambda k: per_kernel[k]["ms"])
        dom_name = {"select": "semkv_assign_precision (k_select_cluster)",
                    "quantize": "semkv_quantize_pack (k_quantize_fast)",
                    "append_decode": "semkv_append_decode (k_decode_i8 x 2 + k_decode_merge)"}[dom]
        ach = per_kernel[dom]["gbs"]
        dec_gbs = per_kernel["decode_l2_cold"]["gbs"]
        launches = (2 + DECODE_KERNELS_PER_CALL) * K
        clocks, e2e, traffic, steps_ms = {}, None, captured_traffic(w.name, dom), None
        cfg_extra = {"l2": "flushed between steps (512 MB written, then 256 MB of it read back: a cold L2 with no dirty lines)", "timing": r["timing"]}

    if w.name == "gen" and not (args.no_extras or args.profile):
        extras["llama8b_32L"] = run_decode_layers(gpu, synth.WORKLOADS["llama8b_32L"], min(K, 50), W)
        extras["llama8b_1L"] = run_one_layer(gpu, synth.WORKLOADS["llama8b_1L"], min(max(K, 20), 400), W)
        sweep = run_sweep(gpu, synth.WORKLOADS["mistral_sweep"])

    cpu = None
    if gpu.rank == 0 and gpu.world == 1 and not args.no_cpu_baseline and not args.profile:
        c = oracle_gen_baseline(synth.WORKLOADS["gen"])
        cpu = {"value": c["gbs"], "unit": "GB/s", "cores": c["threads"], "kind": "oracle", "sample": c["sample"],
               "value_fp64_attention": c["gbs_fp64"], "prefill_gbs": c["prefill_gbs"]}

    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": gpu.world, "steps": K, "warmup": W,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "decode: u8 codes x s8/u8 fixed-point limbs on the integer tensor cores (queries as three s8 "
                 "limbs of a 20-bit image, P' = p s_V as three u8 limbs of a 22-bit image per tile), s32 "
                 "accumulate, f32 softmax; quantize: binary32 IEEE",
        "data": "synthetic",
        "config": dict(workload_config(w, gpu.world), **cfg_extra),
        "per_kernel": per_kernel,
        "roofline": {"bound": "hbm", "kernel": dom_name, "achieved": ach, "peak": peak, "unit": "GB/s",
                     "frac": ach / peak, "peak_kind": peak_kind, "traffic": traffic, "frac_of_8000": ach / 8000.0},
        "decode_roofline": {"achieved": dec_gbs, "peak": peak, "frac": dec_gbs / peak,
                            "frac_of_8000": dec_gbs / 8000.0},
        "clocks": clocks, "e2e": e2e, "cpu_baseline": cpu, "gpu_launches": launches,
    }
    if steps_ms:
        line["step_ms_min_median_max"] = [min(steps_ms), statistics.median(steps_ms), max(steps_ms)]
    if extras:
        line["extras"] = extras
    if sweep is not None:
        line["sweep"] = sweep
    if gpu.rank == 0:
        print(json.dumps(line), flush=True)
    if gpu.dist is not None:
        gpu.dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_semkv(args)


if __name__ == "__main__":
    sys.exit(main())
