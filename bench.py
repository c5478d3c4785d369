#!/usr/bin/env python
"""Indexer throughput on B200: query-key pairs scored and selected per second.

A step is one pass of the whole hot path over one batch of a workload: append the step's
new keys to the indexer K cache (quantising them for an FP8 cache), quantise the queries
(FP8), score every causal (query, key) pair (tensor-core logits with the fused ReLU /
head-weighted sum / causal mask) and select the top 2048 keys per query.

The headline line is the long FP8 prefill (1 sequence of 65536 tokens, H_I=64, d_I=128,
E4M3 with a per-token scale, top_k=2048), the largest single-GPU workload.  The line's
"configs" block carries the same measurement for the decode batch (32 x 32768 keys, bf16),
the bf16 prefill (L=16384) and the ragged FP8 decode (16 sequences of 4096..131072 keys,
2 queries each), each with its own roofline, e2e and CPU-oracle baseline.  Steps are
captured in CUDA graphs and replayed; every workload's inputs exceed the 126 MB L2, so no
flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank processes its own copy-shaped workload (its own seed: weak
scaling, no collective on the data path); the time is the max over ranks and `value`
counts the pairs of all ranks.  `--impl reference` times the fp64 CPU oracle on a bounded
sample of the headline workload.
"""

from __future__ import annotations

import argparse
import contextlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "indexer query-key pairs scored+selected/sec (prefill & decode); % of roofline"
UNIT = "pairs/s"
WORKLOADS = {
    "decode": "decode batch: 32 seqs x 32768 keys, H_I=64, d_I=128, bf16, top_k=2048, 1 query/seq",
    "prefill": "prefill: 1 seq L=16384, H_I=64, d_I=128, bf16, 1% outlier keys x4, causal, top_k=2048",
    "prefill8": "long prefill FP8: 1 seq L=65536, H_I=64, d_I=128, E4M3 + per-token scale, causal, top_k=2048",
    "decode8": "ragged decode FP8: 16 seqs, lengths U[4096,131072], 2 queries/seq, H_I=64, d_I=128, top_k=2048",
    "tiny": "tiny prefill: 1 seq L=512, H_I=4, d_I=64, bf16, top_k=32",
}
HEADLINE = "prefill8"                       # the largest single-GPU workload
SUBCONFIGS = ("decode", "prefill", "decode8")
# steps captured per CUDA graph: short decode steps are batched, long prefill steps go one by one
GRAPH_STEPS = {"decode": 50, "decode8": 50, "prefill": 1, "prefill8": 1, "tiny": 50}
E2E_STEPS = {"decode": 200, "decode8": 200, "prefill": 20, "prefill8": 10, "tiny": 50}
MIN_TIMED_S = 1.0                           # sub-configurations time at least this long


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40, help="timed steps of the headline workload")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--kernel-samples", type=int, default=12,
                    help="graph replays whose profiled step gives the median kernel times")
    ap.add_argument("--cpu-seconds", type=float, default=4.0, help="oracle CPU work per workload for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-side", action="store_true", help="skip the after-selection / RoPE / compressed sections")
    ap.add_argument("--workload", choices=["all", "decode", "prefill", "prefill8", "decode8", "tiny"], default="all",
                    help="all (the default): the headline plus the per-config blocks; one name: that workload alone")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="profiling only: run a prefill workload at this sequence length instead")
    ap.add_argument("--profile-steps", type=int, default=0,
                    help="profiling only: run this many untimed steps of the workload and exit (no JSON line); "
                         "the command ncu wraps to capture single kernels")
    ap.add_argument("--only", choices=["rope"], default=None,
                    help="profiling only: time one side section alone (rope: the fused RoPE kernels at prefill "
                         "size) and print its figures as JSON, without the decode workload")
    ap.add_argument("--reps", type=int, default=10, help="launches per kernel in --only")
    return ap.parse_args()


# ----------------------------------------------------------------------------- multi-rank aggregation

def max_over_ranks(x: float, dist=None) -> float:
    """The slowest rank's value (the job's time); x itself without a process group."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(pairs_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: the pairs every rank scored and selected per second of the slowest rank."""
    return pairs_per_rank * world / (ms_per_step * 1e-3)


# ----------------------------------------------------------------------------- workload

def workload(rank: int, name: str):
    """The workload each rank processes; ranks draw different seeds (weak scaling)."""
    from sparse_attention_token_02_b200 import workloads as W
    make = {"decode": W.decode, "prefill": W.prefill, "prefill8": W.prefill8, "decode8": W.decode8,
            "tiny": W.tiny}[name]
    wl = make()
    return W.scaled(wl, seed=wl.seed + 1000 * rank) if rank else wl


def host_inputs(wl):
    from sparse_attention_token_02_b200 import workloads as W
    return W.make_inputs(wl)


# ----------------------------------------------------------------------------- oracle timing (CPU baseline)

def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        return os.cpu_count() or 1


class OracleRows:
    """The oracle's work for one query row of a workload, as a step does it per token: for an
    FP8 cache, quantise the token's own key row (the append) and its query (the oracle's
    codec); then score the query against keys 0..p and take the top-k.

    The history keys the scores read are inputs, already in the cache when a step runs; for
    the timing they are the bf16 source values decoded to fp64 (the fp64 contraction costs the
    same whatever the values are), so that a sample of rows does not first have to run the
    slow reference codec over the whole cache."""

    def __init__(self, wl, inp):
        import oracle
        self.oracle, self.wl, self.inp = oracle, wl, inp
        self.fp8 = wl.dtype == "fp8"
        self.row_seq = np.repeat(np.arange(wl.num_seqs), wl.q_lens)
        self.row_pos = np.concatenate([np.arange(L - n, L) for L, n in zip(wl.seq_lens, wl.q_lens)])
        self._keys = {}

    def keys(self, b):
        if b not in self._keys:
            self._keys[b] = self.oracle.bf16_bits_to_f64(self.inp["k_bits"][b])
        return self._keys[b]

    def prepare(self, r: int):
        """Everything row r needs that is an input, not oracle work: its sequence's key values,
        its query bits and head weights (drawn here when the inputs are generated lazily)."""
        b, p = int(self.row_seq[r]), int(self.row_pos[r])
        self.keys(b)
        return self.inp["q_bits"][r], self.inp["w"][r], self.inp["k_bits"][b][p: p + 1]

    def row(self, r: int, n_keys: int | None = None, prepared=None) -> int:
        """The oracle on packed row r (its first n_keys keys if given); returns the pairs scored."""
        o = self.oracle
        b, p = int(self.row_seq[r]), int(self.row_pos[r])
        n = p + 1 if n_keys is None else min(p + 1, n_keys)
        bits, w, kbits = prepared if prepared is not None else self.prepare(r)
        if self.fp8:
            o.quantize_rows(o.bf16_bits_to_f64(kbits).astype(np.float32))          # the token's key (append)
            codes, sc = o.quantize_rows(o.bf16_bits_to_f64(bits.reshape(1, -1)).astype(np.float32))
            qv = (o.e4m3_decode(codes) * np.float64(sc[0])).reshape(bits.shape)
        else:
            qv = o.bf16_bits_to_f64(bits)
        s = o.row_scores(qv, self.keys(b)[:n], np.asarray(w, dtype=np.float64))
        o.topk_row(s, self.wl.top_k)
        return n


def oracle_baseline(wl, inp, seconds: float, threads: int | None = None, seed: int = 0) -> dict:
    """Times the fp64 oracle on whole query rows of the workload, taken in a seeded random
    order, until `seconds` of oracle time have passed (or every row is done); the rate is the
    sampled rows' pairs per second, which is the whole workload's rate when the rows are a
    sample of it ("extrapolated" says so)."""
    from threadpoolctl import threadpool_limits
    orc = OracleRows(wl, inp)
    T = wl.total_q
    order = np.random.default_rng(seed).permutation(T)
    busy = pairs = rows = 0
    limit = threadpool_limits(limits=threads) if threads else contextlib.nullcontext()
    with limit:
        cores = _blas_threads()
        t_prep = 0.0
        for r in order:
            t = time.perf_counter()
            prep = orc.prepare(int(r))                        # inputs: drawn before timing
            t_prep += time.perf_counter() - t
            t = time.perf_counter()
            pairs += orc.row(int(r), prepared=prep)
            busy += time.perf_counter() - t
            rows += 1
            if busy >= seconds or t_prep >= max(30.0, 6 * seconds):   # bounded: the bench must end in minutes
                break
    extrapolated = rows < T
    per_row = ("quantise the token's key and query (oracle codec), scores, top-k" if wl.dtype == "fp8"
               else "scores, top-k")
    sample = (f"{rows} of {T} query rows ({'seeded random order, ' if extrapolated else ''}{pairs} pairs, "
              f"{busy:.1f} s of numpy fp64 oracle; per row: {per_row})")
    return {"value": pairs / busy, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
            "extrapolated": extrapolated, "model": cpu_model()}


def cpu_baselines(name, wl, inp, seconds) -> dict:
    """cpu_baseline of one workload: the oracle on the host's BLAS threads, plus one thread
    on the tiny and decode-batch workloads."""
    out = oracle_baseline(wl, inp, seconds)
    if name in ("tiny", "decode"):
        one = oracle_baseline(wl, inp, seconds / 2, threads=1)
        out["threads_1"] = {"value": one["value"], "sample": one["sample"], "extrapolated": one["extrapolated"]}
    return out


def run_reference(args):
    """The oracle as the reference arm, on the headline workload: each step is a bounded
    sample of it (a few whole query rows, in a seeded random order), sized so that warm-up
    plus all steps take about two and a half minutes."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    name = HEADLINE if args.workload == "all" else args.workload
    wl = workload(0, name)
    inp = reference_inputs(wl)
    orc = OracleRows(wl, inp)
    order = np.random.default_rng(1).permutation(wl.total_q)
    prep = orc.prepare(int(order[0]))
    t = time.perf_counter()
    orc.row(int(order[0]), prepared=prep)
    row_s = max(time.perf_counter() - t, 1e-6)
    budget = 150.0 / max(1, args.steps + args.warmup)
    rows_per_step = max(1, min(wl.total_q, int(budget / row_s)))
    secs, pairs, i = [], 0, 1
    for s in range(args.warmup + args.steps):
        rows = [int(order[(i + j) % len(order)]) for j in range(rows_per_step)]
        i += rows_per_step
        preps = [orc.prepare(r) for r in rows]             # inputs: drawn before the step's timing
        t = time.perf_counter()
        n = 0
        for r, pr in zip(rows, preps):
            n += orc.row(r, prepared=pr)
        if s >= args.warmup:
            secs.append(time.perf_counter() - t)
            pairs += n
    value = pairs / sum(secs)
    sample = (f"per step {rows_per_step} whole query row(s) of the workload in a seeded random order "
              f"(numpy fp64 oracle: scores + top-k; {len(secs)} steps, {sum(secs):.1f} s), "
              f"extrapolated to the workload by pair count")
    info = {"value": value, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle", "sample": sample,
            "model": cpu_model()}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(secs),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOADS[name], "sample": sample},
            "cpu_baseline": info,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def reference_inputs(wl):
    """Host inputs of a workload; for the long prefill only the key rows and the query / weight
    rows the reference arm can reach are drawn (any rows of a tensor regenerate alone)."""
    from sparse_attention_token_02_b200 import workloads as W
    if wl.total_q <= 20000:
        return W.make_inputs(wl)

    n = W.CHUNK_ROWS
    T = wl.total_q
    return {"k_bits": [W.f32_to_bf16_bits(W.key_rows(wl, b)) for b in range(wl.num_seqs)],
            "q_bits": _ChunkRows(lambda c: W.f32_to_bf16_bits(W.query_rows(wl, c * n, min(T, (c + 1) * n))), n),
            "w": _ChunkRows(lambda c: W.weight_rows(wl, c * n, min(T, (c + 1) * n)), n)}


class _ChunkRows:
    """Rows of a generated tensor, drawn a chunk of rows at a time on first use."""

    def __init__(self, fn, rows_per_chunk):
        self.fn, self.n, self.cache = fn, rows_per_chunk, {}

    def __getitem__(self, r):
        c, i = divmod(int(r), self.n)
        if c not in self.cache:
            self.cache[c] = self.fn(c)
        return self.cache[c][i]


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples (every 200 ms) over the whole run; summary() gives the samples of
    one timed region by wall-clock time."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_uuid: str | None):
        self.lines = []
        self.proc = None
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if device_uuid:
            cmd += ["-i", device_uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def close(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        self.proc = None

    def summary(self, t_begin: float, t_end: float):
        """Median SM clock, max clock and active throttle reasons of the samples taken between
        the wall-clock times t_begin and t_end."""
        if not self.lines and self.proc is None:
            return None
        import datetime
        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in list(self.lines):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                clk, mx = float(parts[2]), float(parts[3])
            except ValueError:
                continue
            if not (t_begin - 0.1 <= ts <= t_end + 0.1):
                continue
            sm.append(clk)
            try:
                power.append(float(parts[4]))
            except ValueError:
                pass
            for n, v in zip(names, parts[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ----------------------------------------------------------------------------- roofline denominators

def peaks():
    """Roofline denominators: the measured copy bandwidth and cuBLAS bf16 GEMM
    rates (FP8 taken as 2x bf16, the nominal dense ratio), else the recipe's fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        hbm, b, bs, kind = float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        hbm, b, bs, kind = 6650.0, 1590.0, 1400.0, "fallback"
    return {"hbm": hbm, "bf16_burst": b, "bf16_sustained": bs, "fp8_burst": 2 * b, "fp8_sustained": 2 * bs,
            "kind": kind}


PROFILE_NAMES = {"decode": "decode_bf16", "prefill": "prefill_bf16", "prefill8": "prefill_fp8",
                 "decode8": "decode8_fp8", "tiny": "tiny_bf16"}


def profiled_traffic(name: str):
    """DRAM bytes per launch of a workload's logits kernel from the committed ncu summary
    profiles/logits_<workload>_traffic.md, or None when there is none or the kernel source
    changed since those counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"logits_{PROFILE_NAMES[name]}_traffic.md")
    src = os.path.join(ROOT, "sparse_attention_token_02_b200", "csrc", "kernels_logits.cu")
    try:
        text = open(path).read()
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
        fields = dict(ln.split(":", 1) for ln in text.splitlines() if ":" in ln and not ln.startswith("#"))
        if fields.get("kernels_logits_sha256", "").strip() != sha:
            return None
        return float(fields["dram_bytes_per_launch"].strip())
    except Exception:
        return None


# ----------------------------------------------------------------------------- side measurements

# Before a launch timed alone, the GPU spins this many cycles (about 150 us) after the L2
# flush, so the host has enqueued the start event, the launch and the end event before the
# device reaches them: the events then bracket device time only, not the host's call overhead.
_HOST_LEAD_CYCLES = 300_000


def after_select_timings(api, hx, stream, dev, reps=10):
    """Latent-row gather (bf16 c^KV, d_c = 512 per cached token, synthetic) at the step's
    selection, and the in-place sort of the selection; CUDA events around each launch.  Before
    each launch a 256 MB buffer is read (not written): that evicts the inputs from the L2
    without leaving dirty lines whose write-back would fall into the timed launch."""
    import torch
    wl = hx.wl
    with torch.cuda.stream(stream):
        latent = torch.empty(wl.total_k, 512, dtype=torch.bfloat16, device=dev)
        latent.view(torch.int16).random_()
        base = api.selection_row_base(hx.seq_lens, hx.q_lens, hx.k_base, device=dev)
        out = torch.empty(wl.total_q, wl.top_k, 512, dtype=torch.bfloat16, device=dev)
        flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
        idx0, sc0 = hx.out_idx.clone(), hx.out_score.clone()
    res = {}
    for name in ("gather", "sort"):
        total = 0.0
        for it in range(reps + 1):                   # the first launch (module load, set-up) is not timed
            with torch.cuda.stream(stream):
                flush.max()
                i2, s2 = idx0.clone(), sc0.clone()
                torch.cuda._sleep(_HOST_LEAD_CYCLES)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            if name == "gather":
                api.dsa_gather_rows(latent, idx0, base, out=out, stream=stream)
            else:
                api.dsa_sort_selection(i2, s2, stream=stream)
            e1.record(stream)
            stream.synchronize()
            total += e0.elapsed_time(e1) if it else 0.0
        res[name] = total / reps
    api.dsa_check_device_errors(stream)
    valid = int((idx0 >= 0).sum().item())
    moved = valid * 1024 + idx0.numel() * (4 + 1024) + base.numel() * 8   # reads of rows + idx, all writes
    pk = peaks()
    gbs = moved / (res["gather"] * 1e-3) / 1e9
    del latent, out, flush
    return {"gather_latent": {"ms": res["gather"], "rows": int(idx0.numel()), "row_bytes": 1024,
                              "bytes": moved, "achieved_gbs": gbs, "frac_of_hbm": gbs / pk["hbm"]},
            "sort_selection": {"ms": res["sort"], "rows": int(idx0.shape[0]), "top_k": int(idx0.shape[1])}}


def rope_timings(api, stream, dev, reps=10):
    """The fused RoPE kernels at prefill size (16384 tokens, H_I = 64, d_I = 128): queries
    rotated and quantised to E4M3, and 65536 key rows rotated and quantised into an FP8 cache;
    CUDA events around each launch after a 256 MB L2-evicting read."""
    import torch
    T, H, d, n = 16384, 64, 128, 65536
    with torch.cuda.stream(stream):
        q = torch.randn(T, H, d, device=dev).to(torch.bfloat16)
        pos_q = torch.arange(T, dtype=torch.int32, device=dev)
        k = torch.randn(n, d, device=dev).to(torch.bfloat16)
        pos_k = torch.arange(n, dtype=torch.int32, device=dev)
        rows = torch.arange(n, dtype=torch.int64, device=dev)
        cache = api.IndexerKCache.empty(n, d, True, device=dev)
        codes = torch.empty(T, H, d, dtype=torch.uint8, device=dev)
        scale = torch.empty(T, dtype=torch.float32, device=dev)
        flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    res = {}
    for name in ("queries", "keys"):
        total = 0.0
        for it in range(reps + 1):                   # the first launch (module load, set-up) is not timed
            with torch.cuda.stream(stream):
                flush.max()
                torch.cuda._sleep(_HOST_LEAD_CYCLES)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            if name == "queries":
                api.dsa_rope_queries(q, pos_q, fp8=True, rope_dim=64, interleaved=False, out=codes, scale=scale,
                                     stream=stream)
            else:
                api.dsa_indexer_kcache_append_rope(cache, k, rows, pos_k, rope_dim=64, interleaved=False, stream=stream)
            e1.record(stream)
            stream.synchronize()
            total += e0.elapsed_time(e1) if it else 0.0
        res[name] = total / reps
    api.dsa_check_device_errors(stream)
    hbm = peaks()["hbm"]
    qb = T * H * d * 2 + T * 4 + T * H * d + T * 4          # bf16 in, positions, codes + scales out
    kb = n * d * 2 + n * 12 + n * d + n * 4                 # bf16 in, positions + rows, codes + scales out
    out = {}
    for name, b in (("queries", qb), ("keys", kb)):
        gbs = b / (res[name] * 1e-3) / 1e9
        out[name] = {"ms": res[name], "bytes": b, "achieved_gbs": gbs, "frac_of_hbm": gbs / hbm}
    out["config"] = "16384 queries x 64 heads / 65536 keys, d_I=128, rope_dim 64 (half pairs), FP8 out"
    del q, k, cache, codes, flush
    return out


def compressed_timings(api, hx, stream, dev, m=4, reps=10):
    """Decode over an m-compressed key cache with the decode batch's shape (block keys
    synthetic N(0, 1) bf16, one row per m tokens); CUDA events around each call after a
    256 MB L2-evicting read."""
    import torch
    wl = hx.wl
    blocks = [L // m for L in wl.seq_lens]
    base = np.concatenate([[0], np.cumsum(blocks)[:-1]]).astype(np.int64)
    with torch.cuda.stream(stream):
        cache = api.IndexerKCache.empty(int(sum(blocks)), wl.d, False, device=dev)
        keys = torch.randn(int(sum(blocks)), wl.d, device=dev).to(torch.bfloat16)
        api.dsa_indexer_kcache_append(cache, keys, torch.arange(int(sum(blocks)), dtype=torch.int64, device=dev),
                                      stream=stream)
        flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
        oi = torch.empty(wl.total_q, wl.top_k, dtype=torch.int32, device=dev)
        os_ = torch.empty(wl.total_q, wl.top_k, dtype=torch.float32, device=dev)
    call = lambda: api.dsa_indexer_decode_compressed(hx.q, cache, hx.w, hx.seq_lens, hx.q_lens, m, wl.top_k,
                                                     k_base=base, out_idx=oi, out_score=os_, stream=stream)
    call()
    total = 0.0
    for _ in range(reps):
        with torch.cuda.stream(stream):
            flush.max()
            torch.cuda._sleep(_HOST_LEAD_CYCLES)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        stream.synchronize()
        total += e0.elapsed_time(e1)
    api.dsa_check_device_errors(stream)
    ms = total / reps
    pairs = sum((L - n + j + 1) // m for L, n in zip(wl.seq_lens, wl.q_lens) for j in range(n))
    kbytes = int(sum(blocks)) * wl.d * 2
    hbm = peaks()["hbm"]
    del cache, keys, flush
    out = {"m": m, "ms": ms, "pairs": pairs, "pairs_per_s": pairs / (ms * 1e-3),
           "key_bytes": kbytes, "frac_of_hbm": kbytes / (ms * 1e-3) / 1e9 / hbm,
           "note": "eager call (logits + top-k); the decode kernels with each query's limit at its last block"}
    out["prefill"] = compressed_prefill_timing(api, stream, dev, m, reps)
    return out


def compressed_prefill_timing(api, stream, dev, m=4, reps=5, L=16384, H=64, d=128, top_k=2048):
    """Prefill over an m-compressed cache: one sequence of L tokens, every token a query
    (bf16, H_I = 64, d_I = 128, synthetic N(0, 1) block keys and queries, softmaxed w);
    CUDA events around each call after a 256 MB L2-evicting read."""
    import torch
    nb = L // m
    with torch.cuda.stream(stream):
        cache = api.IndexerKCache.empty(nb, d, False, device=dev)
        keys = torch.randn(nb, d, device=dev).to(torch.bfloat16)
        api.dsa_indexer_kcache_append(cache, keys, torch.arange(nb, dtype=torch.int64, device=dev), stream=stream)
        q = (torch.randn(L, H, d, device=dev) / d ** 0.5).to(torch.bfloat16)
        w = torch.softmax(torch.randn(L, H, device=dev), dim=1)
        flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
        oi = torch.empty(L, top_k, dtype=torch.int32, device=dev)
        os_ = torch.empty(L, top_k, dtype=torch.float32, device=dev)
    call = lambda: api.dsa_indexer_prefill_compressed(q, cache, w, (L,), m, top_k, out_idx=oi, out_score=os_,
                                                      stream=stream)
    call()
    total = 0.0
    for _ in range(reps):
        with torch.cuda.stream(stream):
            flush.max()
            torch.cuda._sleep(_HOST_LEAD_CYCLES)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        stream.synchronize()
        total += e0.elapsed_time(e1)
    api.dsa_check_device_errors(stream)
    ms = total / reps
    pairs = sum((p + 1) // m for p in range(L))
    flops = 2.0 * pairs * H * d
    del cache, keys, q, flush
    return {"L": L, "m": m, "ms": ms, "pairs": pairs, "pairs_per_s": pairs / (ms * 1e-3),
            "tflops": flops / (ms * 1e-3) / 1e12, "note": "logits + top-k, causal over complete blocks"}


# ----------------------------------------------------------------------------- our path

class Harness:
    """Device state and one step of the hot path for a workload.

    decode : the step appends each sequence's newest q_len keys (re-written in place),
             quantises the queries (FP8), then scores + selects (dsa_indexer_decode).
    prefill: the step appends every key of the sequence (quantising for FP8),
             quantises the queries (FP8), then scores + selects (dsa_indexer_prefill).
    """

    def __init__(self, wl, inp, dev, stream):
        import torch
        from sparse_attention_token_02_b200 import api
        self.api, self.wl, self.dev, self.stream = api, wl, dev, stream
        self.fp8 = wl.dtype == "fp8"
        self.decode = wl.kind == "decode"
        L = np.array(wl.seq_lens, dtype=np.int64)
        self.k_base = np.concatenate([[0], np.cumsum(L)[:-1]]).astype(np.int64)
        self.seq_lens, self.q_lens = list(wl.seq_lens), list(wl.q_lens)
        T, H, d = wl.total_q, wl.H, wl.d
        bf = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
        with torch.cuda.stream(stream):
            self.cache = api.IndexerKCache.empty(wl.total_k, d, self.fp8, device=dev)
            k_all = bf(np.concatenate(inp["k_bits"])).to(dev)
            api.dsa_indexer_kcache_append(self.cache, k_all, torch.arange(wl.total_k, dtype=torch.int64, device=dev),
                                          stream=stream)
            if self.decode:
                # the step's new keys: the newest q_len rows of each sequence
                rows = np.concatenate([self.k_base[b] + np.arange(L[b] - n, L[b]) for b, n in enumerate(self.q_lens)])
                self.k_step_host = bf(np.concatenate(inp["k_bits"])[rows])
                self.rows_host = torch.from_numpy(rows.astype(np.int64))
                del k_all
            else:
                self.k_step_host = bf(np.concatenate(inp["k_bits"]))
                self.rows_host = torch.arange(wl.total_k, dtype=torch.int64)
            self.k_step = self.k_step_host.to(dev)
            self.rows = self.rows_host.to(dev)
            self.q_src_host = bf(inp["q_bits"])
            self.q_src = self.q_src_host.to(dev)
            self.w_host = torch.from_numpy(inp["w"])
            self.w = self.w_host.to(dev)
            if self.fp8:
                self.q = torch.empty(T, H, d, dtype=torch.uint8, device=dev)
                self.q_scale = torch.empty(T, dtype=torch.float32, device=dev)
            else:
                self.q, self.q_scale = self.q_src, None
            self.out_idx = torch.empty(T, wl.top_k, dtype=torch.int32, device=dev)
            self.out_score = torch.empty(T, wl.top_k, dtype=torch.float32, device=dev)
        stream.synchronize()

    def step(self, k_step=None, q_src=None, w=None):
        api, s, wl = self.api, self.stream, self.wl
        k_step = self.k_step if k_step is None else k_step
        q_src = self.q_src if q_src is None else q_src
        w = self.w if w is None else w
        api.dsa_indexer_kcache_append(self.cache, k_step, self.rows, stream=s)
        if self.fp8:
            api.dsa_quantize_rows_fp8(q_src.view(q_src.shape[0], -1), dst=self.q.view(self.q.shape[0], -1),
                                      scale=self.q_scale, stream=s)
        q = self.q if self.fp8 else q_src
        if self.decode:
            api.dsa_indexer_decode(q, self.cache, w, self.seq_lens, self.q_lens, wl.top_k, q_scale=self.q_scale,
                                   k_base=self.k_base, out_idx=self.out_idx, out_score=self.out_score, stream=s)
        else:
            api.dsa_indexer_prefill(q, self.cache, w, self.seq_lens, wl.top_k, q_scale=self.q_scale,
                                    q_lens=self.q_lens, k_base=self.k_base, out_idx=self.out_idx,
                                    out_score=self.out_score, stream=s)

    # algorithmic work of the dominant (logits) kernel per step
    def logits_bytes(self):
        wl = self.wl
        esz = 1 if self.fp8 else 2
        k_bytes = wl.total_k * wl.d * esz + (wl.total_k * 4 if self.fp8 else 0)
        q_bytes = wl.total_q * wl.H * wl.d * esz + (wl.total_q * 4 if self.fp8 else 0)
        return k_bytes + q_bytes + wl.total_q * wl.H * 4

    def logits_flops(self):
        return 2.0 * self.wl.pairs * self.wl.H * self.wl.d


def measure(name, hx, args, steps, world, dist, clocks, wl, inp, rank):
    """One workload's block: device-timed steps in CUDA graphs, median kernel times,
    roofline of the logits kernel, end-to-end steps from pinned host memory, CPU baseline."""
    import torch
    api, stream, dev = hx.api, hx.stream, hx.dev
    G = GRAPH_STEPS[name]

    # uncaptured warm-up (also plans the batch once)
    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            hx.step()
    api.dsa_check_device_errors(stream)

    # capture G steps; the middle one carries kernel-timing events (events between kernels
    # would keep the next kernel from starting its prologue early, so the other steps have none)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    with torch.cuda.stream(stream):
        for e in ev:
            e.record(stream)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    n0 = api.dsa_kernel_launch_count()
    with torch.cuda.graph(graph, stream=stream, capture_error_mode="relaxed"):
        for g in range(G):
            if g == G // 2:
                api.dsa_set_profile_events(*ev)
            hx.step()
            api.dsa_set_profile_events(None, None, None)
    launches_per_step = (api.dsa_kernel_launch_count() - n0) / G
    with torch.cuda.stream(stream):
        graph.replay()
    stream.synchronize()
    api.dsa_check_device_errors(stream)

    if steps is None:
        # sub-configurations: at least MIN_TIMED_S of timed work, a whole number of graphs
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            t0.record(stream)
            graph.replay()
            t1.record(stream)
        stream.synchronize()
        est = t0.elapsed_time(t1) / G
        steps = max(args.steps, int(math.ceil(MIN_TIMED_S * 1e3 / max(est, 1e-3))))
        steps = max(steps, G)
        steps = int(max_over_ranks(steps, dist if world > 1 else None))   # every rank replays the same count
    replays = int(math.ceil(steps / G))
    K = replays * G

    # timed region
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    wall0 = time.time()
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(replays):
            graph.replay()
        t1.record(stream)
    torch.cuda.synchronize(dev)
    wall1 = time.time()
    if world > 1:
        dist.barrier()
    ms_total = max_over_ranks(t0.elapsed_time(t1), dist if world > 1 else None)
    ms_step = ms_total / K
    clk = clocks.summary(wall0, wall1) if clocks is not None else None

    # kernel times: the profiled step of each of `kernel-samples` further replays
    lg, tk = [], []
    for _ in range(max(10, args.kernel_samples)):
        with torch.cuda.stream(stream):
            graph.replay()
        stream.synchronize()
        lg.append(ev[0].elapsed_time(ev[1]))
        tk.append(ev[1].elapsed_time(ev[2]))
    logits_ms, topk_ms = statistics.median(lg), statistics.median(tk)
    api.dsa_check_device_errors(stream)
    del graph

    e2e = e2e_block(name, hx, dist, world)

    # roofline of the dominant (logits) kernel
    pk = peaks()
    if hx.decode:
        alg = hx.logits_bytes()
        achieved = alg / (logits_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                "frac": achieved / pk["hbm"], "traffic": profiled_traffic(name),
                "peak_source": f"{pk['kind']} hbm_gbs (copy)", "alg_bytes_per_launch": alg}
    else:
        alg = hx.logits_flops()
        achieved = alg / (logits_ms * 1e-3) / 1e12
        peak = pk["fp8_sustained"] if hx.fp8 else pk["bf16_sustained"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": profiled_traffic(name),
                "peak_source": (f"{pk['kind']} bf16_tflops_sustained (the kernel runs inside a long loop)" +
                                (" x 2, the nominal FP8 / bf16 dense ratio" if hx.fp8 else "")),
                "alg_flops_per_launch": alg,
                "frac_of_burst_peak": achieved / (pk["fp8_burst"] if hx.fp8 else pk["bf16_burst"])}
    roof.update({"kernel": f"logits ({wl.kind}, {wl.dtype})", "kernel_ms": logits_ms,
                 "kernel_ms_samples": len(lg), "kernel_ms_spread": [min(lg), max(lg)]})
    step_bytes = hx.logits_bytes()
    block = {
        "workload": WORKLOADS[name], "pairs_per_step_per_gpu": wl.pairs, "steps": K, "graph_steps": G,
        "ms_per_step": ms_step, "value": job_value(wl.pairs, world, ms_step), "unit": UNIT,
        "dtype": "fp8_e4m3" if hx.fp8 else "bf16",
        "step": ("kcache_append + " + ("quantise q + " if hx.fp8 else "") +
                 ("decode" if hx.decode else "prefill") + " (logits + top-k)"),
        "roofline": roof,
        "kernels_ms": {"logits": logits_ms, "topk": topk_ms, "samples": len(lg)},
        "step_frac_of_hbm": (step_bytes / (ms_step * 1e-3) / 1e9 / pk["hbm"]) if hx.decode else None,
        "e2e": e2e,
        "gpu_launches": int(round(launches_per_step * K)),
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        block["cpu_baseline"] = cpu_baselines(name, wl, inp, args.cpu_seconds)
    else:
        block["cpu_baseline"] = None
    return block


def e2e_block(name, hx, dist, world):
    """End to end from pinned host memory: every step uploads its inputs and reads its
    selection back, through the library's one-call host step (dsa_indexer_decode_host /
    dsa_indexer_prefill_host with a completion event: the uploads of a step overlap the
    kernels of the previous one, its read-back those of the next).  Steps are enqueued back
    to back; the events bracket all of them, the end event after the last read-back."""
    import torch
    api, stream, dev = hx.api, hx.stream, hx.dev
    k_h, q_h, w_h = hx.k_step_host.pin_memory(), hx.q_src_host.pin_memory(), hx.w_host.pin_memory()
    oi_h = torch.empty(hx.out_idx.shape, dtype=torch.int32, pin_memory=True)
    os_h = torch.empty(hx.out_score.shape, dtype=torch.float32, pin_memory=True)
    rows_h = hx.rows_host.pin_memory()
    done = [torch.cuda.Event(), torch.cuda.Event()]
    last = [None]
    batch = api.host_batch(hx.seq_lens, hx.q_lens, hx.k_base)   # built once, like a serving loop's metadata

    def e2e_step():
        ev = done[0] if last[0] is not done[0] else done[1]
        if hx.decode:
            api.dsa_indexer_decode_host(q_h, w_h, k_h, rows_h, hx.cache, batch, None, hx.wl.top_k,
                                        oi_h, os_h, stream=stream, done_event=ev)
        else:
            api.dsa_indexer_prefill_host(q_h, w_h, k_h, rows_h, hx.cache, batch, hx.wl.top_k,
                                         oi_h, os_h, stream=stream, done_event=ev)
        last[0] = ev

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    E = E2E_STEPS[name]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    stream.synchronize()                     # the first upload (on the library's copy stream) starts after e0
    h0 = time.perf_counter()
    for _ in range(E):
        e2e_step()
    host_us = (time.perf_counter() - h0) * 1e6 / E   # host time to enqueue one step (the API call)
    if last[0] is not None:
        stream.wait_event(last[0])           # every read-back has completed (one copy stream, in order)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / E, dist if world > 1 else None)
    api.dsa_check_device_errors(stream)
    h2d = sum(t.numel() * t.element_size() for t in (k_h, q_h, w_h)) + (rows_h.numel() * 8 if hx.decode else 0)
    d2h = sum(t.numel() * t.element_size() for t in (oi_h, os_h))
    pairs = hx.wl.pairs * world
    return {"value": pairs / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": e2e_ms, "steps": E, "host_enqueue_us_per_step": host_us,
            "path": ("dsa_indexer_decode_host_async" if hx.decode else "dsa_indexer_prefill_host_async") +
                    " (one C-ABI call per step: uploads, append, quantise, score + select, read-back; library copy "
                    "streams, two device slots)"}


def run_ours(args):
    import torch
    import torch.distributed as dist

    from sparse_attention_token_02_b200 import api

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.Stream(device=dev)

    head = HEADLINE if args.workload == "all" else args.workload

    if args.profile_steps > 0:
        wl = workload(rank, head)
        if args.seq_len and wl.kind == "prefill":
            from sparse_attention_token_02_b200 import workloads as W
            wl = W.scaled(wl, seq_lens=(args.seq_len,), q_lens=(args.seq_len,))
        hx = Harness(wl, host_inputs(wl), dev, stream)
        with torch.cuda.stream(stream):
            for _ in range(args.profile_steps):
                hx.step()
        api.dsa_check_device_errors(stream)
        if world > 1:
            dist.destroy_process_group()
        return 0

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    time.sleep(0.5)

    names = [head] + (list(SUBCONFIGS) if args.workload == "all" else [])
    blocks, side = {}, {}
    for name in names:
        wl = workload(rank, name)
        inp = host_inputs(wl)
        hx = Harness(wl, inp, dev, stream)
        blocks[name] = measure(name, hx, args, args.steps if name == head else None, world, dist, clocks, wl,
                               inp, rank)
        if name == "decode" and not args.no_side:
            # the selection's consumers and the fused RoPE / compressed-cache calls (outside the
            # timed steps), each launch timed alone after an L2 flush
            side["after_select"] = after_select_timings(api, hx, stream, dev)
            side["rope_fused"] = rope_timings(api, stream, dev)
            side["compressed_decode"] = compressed_timings(api, hx, stream, dev)
        del hx, inp
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
    clocks.close()
    if args.workload == "all" and rank == 0 and world == 1 and not args.no_cpu_baseline:
        wl = workload(0, "tiny")
        tiny_cpu = cpu_baselines("tiny", wl, host_inputs(wl), args.cpu_seconds)
    else:
        tiny_cpu = None

    if world > 1:
        dist.barrier()
    if rank == 0:
        hb = blocks[head]
        line = {
            "metric": METRIC, "value": hb["value"], "unit": UNIT, "n_gpus": world, "steps": hb["steps"],
            "warmup": args.warmup, "ms_per_step": hb["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": hb["dtype"], "data": "synthetic",
            "config": {"workload": WORKLOADS[head], "pairs_per_step_per_gpu": hb["pairs_per_step_per_gpu"],
                       "l2": "inputs larger than L2 (126 MB), no flush",
                       "step": hb["step"] + f", CUDA graphs of {hb['graph_steps']} step(s)",
                       "parallelism": f"{world} independent ranks (each its own workload: weak scaling)"},
            "roofline": hb["roofline"],
            "kernels_ms": hb["kernels_ms"],
            "cpu_baseline": hb["cpu_baseline"],
            "e2e": hb["e2e"],
            "gpu_launches": hb["gpu_launches"],
            "clocks": hb["clocks"],
            "configs": {n: b for n, b in blocks.items() if n != head},
        }
        if tiny_cpu is not None:
            line["tiny_cpu_baseline"] = tiny_cpu
        line.update(side)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_only(args):
    import torch

    from sparse_attention_token_02_b200 import api
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.Stream(device=dev)
    if args.only == "rope":
        print(json.dumps({"rope_fused": rope_timings(api, stream, dev, reps=args.reps)}), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.only:
        return run_only(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
