#!/usr/bin/env python
"""Indexer throughput on B200: query-key pairs scored and selected per second.

A step is one pass of the whole hot path over the decode-batch workload
(32 sequences x 32768 cached keys, H_I=64, d_I=128, bf16, top_k=2048, one query per
sequence): append the step's new keys to the cache, score every (query, key) pair
(tensor-core logits + fused ReLU / head-weighted sum), select the top 2048 per
query.  Steps are captured in a CUDA graph and replayed; the K cache (268 MB) is
larger than L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank processes its own 32 sequences (weak scaling, no
collective on the data path); the time is the max over ranks and `value` counts
the pairs of all ranks.  `--impl reference` times the fp64 CPU oracle on a
bounded sample of the same workload.
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
WORKLOAD = WORKLOADS["decode"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--graph-steps", type=int, default=50, help="steps captured per CUDA graph")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU work for the oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=["decode", "prefill", "prefill8", "decode8", "tiny"], default="decode",
                    help="decode (the default) is the measured workload; the others are for profiling")
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

def workload(rank: int, name: str = "decode"):
    """The workload each rank processes; ranks draw different seeds (weak scaling)."""
    from sparse_attention_token_02_b200 import workloads as W
    make = {"decode": W.decode, "prefill": W.prefill, "prefill8": W.prefill8, "decode8": W.decode8,
            "tiny": W.tiny}[name]
    wl = make()
    return W.scaled(wl, seed=wl.seed + 1000 * rank) if rank else wl


def host_inputs(wl):
    from sparse_attention_token_02_b200 import workloads as W
    return W.make_inputs(wl)


# ----------------------------------------------------------------------------- oracle timing

def _oracle_cores():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        return os.cpu_count() or 1


def _oracle_row(wl, inp, b, n_keys):
    """One decode row of sequence b restricted to its first n_keys keys, through the oracle."""
    import oracle
    kv = oracle.bf16_bits_to_f64(inp["k_bits"][b][:n_keys])
    qv = oracle.bf16_bits_to_f64(inp["q_bits"][b: b + 1])
    res = oracle.decode_oracle(qv, [kv], inp["w"][b: b + 1].astype(np.float64), [n_keys], 1, wl.top_k)
    assert res["idx"].shape == (1, wl.top_k)
    return n_keys


def oracle_sample(wl, inp, seconds: float):
    """Times the fp64 oracle on whole decode rows of this workload until `seconds` pass."""
    pairs = rows = b = 0
    t0 = time.perf_counter()
    while True:
        pairs += _oracle_row(wl, inp, b, wl.seq_lens[b])
        rows += 1
        b = (b + 1) % wl.num_seqs
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": pairs / dt, "unit": UNIT, "cores": _oracle_cores(), "kind": "oracle",
            "sample": f"{rows} whole decode rows of {wl.seq_lens[0]} keys (numpy fp64 oracle, {dt:.1f} s)"}


def run_reference(args):
    """The oracle as the reference arm: each step is a bounded sample of the workload
    (whole rows when the step budget allows, else a row's first keys, at least top_k+1),
    sized so that warm-up plus all steps take about two and a half minutes."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = workload(0)
    inp = host_inputs(wl)
    L = wl.seq_lens[0]
    t = time.perf_counter()
    _oracle_row(wl, inp, 0, L)
    row_s = time.perf_counter() - t
    budget = 150.0 / max(1, args.steps + args.warmup)
    if budget >= row_s:
        rows_per_step, keys = max(1, min(wl.num_seqs, int(budget / row_s))), L
    else:
        rows_per_step, keys = 1, int(min(L, max(wl.top_k + 1, L * budget / row_s)))
    secs, pairs = [], 0
    b = 0
    for i in range(args.warmup + args.steps):
        t = time.perf_counter()
        n = 0
        for _ in range(rows_per_step):
            n += _oracle_row(wl, inp, b, keys)
            b = (b + 1) % wl.num_seqs
        if i >= args.warmup:
            secs.append(time.perf_counter() - t)
            pairs += n
    value = pairs / sum(secs)
    sample = (f"per step {rows_per_step} decode row(s) x {keys} keys of the workload "
              f"(numpy fp64 oracle; {len(secs)} steps, {sum(secs):.1f} s)")
    info = {"value": value, "unit": UNIT, "cores": _oracle_cores(), "kind": "oracle", "sample": sample}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(secs),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "sample": sample},
            "cpu_baseline": info,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
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

    def stop(self, t_begin: float, t_end: float):
        """Summary of the samples taken between the wall-clock times t_begin and t_end."""
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        import datetime
        sm, mx, reasons, n_all = [], None, set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                clk, mx = float(parts[2]), float(parts[3])
            except ValueError:
                continue
            n_all += 1
            if not (t_begin - 0.1 <= ts <= t_end + 0.1):
                continue
            sm.append(clk)
            for n, v in zip(names, parts[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0, "samples_total": n_all}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- our path

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


def profiled_traffic():
    """DRAM bytes per launch of the decode logits kernel from the committed ncu summary,
    or None when the kernel source changed since those counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "logits_decode_bf16_traffic.md")
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

    wl = workload(rank, args.workload)
    if args.seq_len and wl.kind == "prefill":
        from sparse_attention_token_02_b200 import workloads as W
        wl = W.scaled(wl, seq_lens=(args.seq_len,), q_lens=(args.seq_len,))
    inp = host_inputs(wl)
    hx = Harness(wl, inp, dev, stream)

    if args.profile_steps > 0:
        with torch.cuda.stream(stream):
            for _ in range(args.profile_steps):
                hx.step()
        api.dsa_check_device_errors(stream)
        if world > 1:
            dist.destroy_process_group()
        return 0

    # uncaptured warm-up (also plans the batch once)
    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            hx.step()
    api.dsa_check_device_errors(stream)

    # capture G steps; the middle one carries kernel-timing events (events between kernels
    # would keep the next kernel from starting its prologue early, so the other steps have none)
    G = max(1, min(args.graph_steps, args.steps))
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
    replays = max(1, args.steps // G)
    K = replays * G
    with torch.cuda.stream(stream):
        graph.replay()
    stream.synchronize()
    api.dsa_check_device_errors(stream)

    # timed region
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    time.sleep(0.5)
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
    clk = clocks.stop(wall0, wall1)
    ms_total = t0.elapsed_time(t1)
    # kernel times of the profiled step of the last replay in the timed region
    logits_ms = ev[0].elapsed_time(ev[1])
    topk_ms = ev[1].elapsed_time(ev[2])
    api.dsa_check_device_errors(stream)
    ms_total = max_over_ranks(ms_total, dist if world > 1 else None)
    ms_step = ms_total / K
    pairs_step = wl.pairs * world
    value = job_value(wl.pairs, world, ms_step)

    # end to end from pinned host buffers: upload the step's inputs, run, read the result back
    k_h, q_h, w_h = hx.k_step_host.pin_memory(), hx.q_src_host.pin_memory(), hx.w_host.pin_memory()
    k_d, q_d, w_d = torch.empty_like(hx.k_step), torch.empty_like(hx.q_src), torch.empty_like(hx.w)
    oi_h = torch.empty(hx.out_idx.shape, dtype=torch.int32, pin_memory=True)
    os_h = torch.empty(hx.out_score.shape, dtype=torch.float32, pin_memory=True)

    rows_h = hx.rows_host.pin_memory()

    # Each step uploads its inputs from pinned host memory and reads its selection back.
    # Decode goes through the library's one-call host step (dsa_indexer_decode_host with a
    # completion event: the read-back of a step overlaps the kernels of the next); prefill
    # copies around the device call.  Steps are enqueued back to back (the host does not wait
    # for each one); the events below bracket all of them, the end event placed after the
    # last step's read-back has completed.
    done = [torch.cuda.Event(), torch.cuda.Event()]
    last = [None]
    batch = api.host_batch(hx.seq_lens, hx.q_lens, hx.k_base)   # built once, like a serving loop's metadata

    def e2e_step():
        if hx.decode:
            ev = done[0] if last[0] is not done[0] else done[1]
            api.dsa_indexer_decode_host(q_h, w_h, k_h, rows_h, hx.cache, batch, None, hx.wl.top_k,
                                        oi_h, os_h, stream=stream, done_event=ev)
            last[0] = ev
            return
        with torch.cuda.stream(stream):
            k_d.copy_(k_h, non_blocking=True)
            q_d.copy_(q_h, non_blocking=True)
            w_d.copy_(w_h, non_blocking=True)
            hx.step(k_step=k_d, q_src=q_d, w=w_d)
            oi_h.copy_(hx.out_idx, non_blocking=True)
            os_h.copy_(hx.out_score, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    E = max(1, args.e2e_steps if hx.decode else min(args.e2e_steps, 10))
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

    # the selection's consumers (outside the timed step): the latent-row gather the sparse
    # attention makes and the sorted order, each launch timed alone after an L2 flush
    after = after_select_timings(api, hx, stream, dev) if hx.decode else None
    rope = rope_timings(api, stream, dev) if hx.decode else None
    comp = compressed_timings(api, hx, stream, dev) if hx.decode and not hx.fp8 else None

    # roofline of the dominant kernel (the logits kernel)
    pk = peaks()
    if hx.decode:
        alg = hx.logits_bytes()
        achieved = alg / (logits_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                "frac": achieved / pk["hbm"], "traffic": profiled_traffic() if args.workload == "decode" else None,
                "peak_source": f"{pk['kind']} hbm_gbs", "alg_bytes_per_launch": alg}
    else:
        alg = hx.logits_flops()
        achieved = alg / (logits_ms * 1e-3) / 1e12
        peak = pk["fp8_sustained"] if hx.fp8 else pk["bf16_sustained"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": None,
                "peak_source": (f"{pk['kind']} bf16_tflops_sustained" + (" x 2 (FP8/bf16 nominal ratio)" if hx.fp8 else "")),
                "alg_flops_per_launch": alg,
                "frac_of_burst_peak": achieved / (pk["fp8_burst"] if hx.fp8 else pk["bf16_burst"])}
    roof.update({"kernel": f"logits ({wl.kind}, {wl.dtype})", "kernel_ms": logits_ms})

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload == "decode":
        cpu = oracle_sample(wl, inp, args.cpu_seconds)

    if world > 1:
        dist.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8_e4m3" if hx.fp8 else "bf16", "data": "synthetic",
            "config": {"workload": WORKLOADS[args.workload], "pairs_per_step_per_gpu": wl.pairs,
                       "l2": "inputs larger than L2 (126 MB), no flush",
                       "step": ("kcache_append + " + ("quantise q + " if hx.fp8 else "") +
                                ("decode" if hx.decode else "prefill") + " (logits + top-k), CUDA graph of %d steps" % G),
                       "parallelism": f"{world} independent ranks (sequences sharded)"},
            "roofline": roof,
            "kernels_ms": {"logits": logits_ms, "topk": topk_ms},
            "cpu_baseline": cpu,
            "e2e": {"value": pairs_step / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "host_enqueue_us_per_step": host_us},
            "gpu_launches": int(round(launches_per_step * K)),
            "clocks": clk,
        }
        if after is not None:
            line["after_select"] = after
        if rope is not None:
            line["rope_fused"] = rope
        if comp is not None:
            line["compressed_decode"] = comp
        print(json.dumps(line), flush=True)
    del graph
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
