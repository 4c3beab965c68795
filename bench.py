#!/usr/bin/env python3
"""Benchmark of the Shannonic INT8 codec hot path on B200.

One step = the whole hot path over one batch of synthetic input resident in HBM:
histogram → range DP + tANS tables → encode → decode (four C-ABI calls into libshn.so).
Default workload: the INT8 KV cache [32 layers, K/V, batch 8, 8 kv heads, seq 4096, head_dim 128]
(2 GiB, one table per layer×K/V), K=16, L=128, 4096-symbol chunks, 4 states per chunk.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload kv|weight|sweep]

Multi-GPU (torchrun): every rank codes its own KV cache (seeded by rank) with no data-path
collective — weak scaling; the time is the max over ranks.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from entropy_coded_lossless_b200 import inputs  # noqa: E402

METRIC = "tANS decode/encode GB/s (INT8 side), % of HBM roofline; bits/symbol vs H"
UNIT = "GB/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="kv",
                    choices=["kv", "weight", "sweep", "activations", "int4", "regen", "sweepgrid"],
                    help="regen: time table regeneration only; sweepgrid: rate and time over the whole "
                         "entropy x chunk x K x L grid of the 1 GiB sweep")
    ap.add_argument("--cpu-sample-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-fused", action="store_true", help="skip the fused decode+dequantise measurement (kv)")
    ap.add_argument("--no-offload", action="store_true", help="skip the host offload/reload measurement (kv)")
    ap.add_argument("--no-configs", action="store_true",
                    help="kv: skip the other configurations (1, 2 with plain tANS, 4, and 5 at four entropies)")
    ap.add_argument("--segments", type=int, default=0, help="kv workload: use only the first N segments")
    ap.add_argument("--entropy", type=float, default=5.3, choices=[2.0, 4.0, 5.3, 7.9], help="sweep workload")
    ap.add_argument("--sweep-bytes", type=int, default=1 << 30, help="sweep workload: stream length (default 1 GiB)")
    ap.add_argument("--K", type=int, default=None, help="override the workload's range count")
    ap.add_argument("--log2L", type=int, default=None, help="override the workload's log2 state count")
    ap.add_argument("--chunk-symbols", type=int, default=None)
    ap.add_argument("--states", type=int, default=None, help="interleaved states per chunk")
    ap.add_argument("--profile-only", action="store_true",
                    help="run compress + decode twice untimed and exit (the case profiles/ captures)")
    return ap.parse_args()


def apply_overrides(p, args):
    for key, val in (("K", args.K), ("log2L", args.log2L), ("chunk_symbols", args.chunk_symbols),
                     ("states_per_chunk", args.states)):
        if val is not None:
            p[key] = val


def workload(name, device, seed_offset=0, n_segments=0, entropy=5.3, sweep_bytes=1 << 30):
    """(int8 tensor, segments, params dict, description)."""
    if name == "kv":
        segs = inputs.kv_cache_segments()
        if n_segments and n_segments < len(segs):
            seg = segs[0][1]
            segs = segs[:n_segments]
            x = torch.empty(n_segments * seg, dtype=torch.int8, device=device)
            for i in range(n_segments):
                x[i * seg:(i + 1) * seg] = inputs.kv_cache_segment_int8(i // 2, i % 2, seed=2 + seed_offset,
                                                                        device=device)
            desc = f"kv_cache_int8 first {n_segments} of 64 layer x K/V segments ({n_segments * seg} bytes)"
        else:
            x = inputs.kv_cache_int8(seed=2 + seed_offset, device=device)
            desc = "kv_cache_int8[32,2,8,8,4096,128] (2 GiB, 64 segments = layer x K/V)"
    elif name == "weight":
        x = inputs.weight_like_int8(seed=1 + seed_offset, device=device)
        segs = [(0, x.numel())]
        desc = "weight_like_int8[4096,1024] (per-row absmax, 1% outliers x8)"
    elif name == "int4":
        x = inputs.int4_weight_like(seed=6 + seed_offset, device=device)
        segs = [(0, x.numel())]
        desc = "int4_weight_like[4096,4096] (group-64 absmax INT4, one value per byte)"
    elif name == "activations":
        x, segs, _ = inputs.activation_batch_int8(1024, 65536, seed=3 + seed_offset, device=device)
        desc = "1024 activation tensors x 65536 INT8 (per-tensor tables)"
    else:
        x = inputs.sweep_stream_int8(entropy, n=sweep_bytes, seed=4 + seed_offset, device=device)
        segs = [(0, x.numel())]
        desc = f"{sweep_bytes} bytes of truncated discrete Laplace, H={entropy} bits"
    return x, segs, dict(K=16, log2L=7, chunk_symbols=4096, states_per_chunk=4), desc


def kernel_launches_per_step(segs, p_dict) -> int:
    """Kernels one step launches through the four calls, following the library's batching: a
    histogram launch per 512 segments; the table build (plus the LG-table fill from 256 tables on);
    per encoder batch (at most 512 consecutive segments of one kind, where segments of at most 64
    chunks, empty ones included, are the small kind) a slot-coding launch and a header launch; the
    three-launch scan and the slot compaction once; the decoder's check and decode launches."""
    n = len(segs)
    if n == 0:
        return 0
    launches = -(-n // 512) + 1 + (1 if n >= 256 else 0) + 3 + 1 + 2
    batches, count, kind = 0, 0, None
    for _, length in segs:
        small = -(-length // p_dict["chunk_symbols"]) <= 64
        if batches == 0 or count == 512 or small != kind:
            batches, count, kind = batches + 1, 0, small
        count += 1
    return launches + 2 * batches


# seed of each workload's generator (rank r of a multi-GPU run adds r)
WORKLOAD_SEED = {"kv": 2, "weight": 1, "int4": 6, "activations": 3, "sweep": 4}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def max_over_ranks(value: float, device) -> float:
    """Max of a per-rank float over the process group (identity without one)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return value
    t = torch.tensor([value], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_rank: int, world: int, ms_per_step: float) -> float:
    """Weak scaling: every rank codes its own bytes_per_rank each step; time is the max over ranks."""
    return world * bytes_per_rank / (ms_per_step * 1e-3) / 1e9


# DRAM bytes (read + write) per symbol of each kernel, from the ncu captures of that kernel on the
# INT8 KV cache (K=16, L=128, C=4096, S=4; 768 MiB for the coder kernels, 256 MiB for the
# histogram and table build; the bytes grow in proportion to the symbols), with the digest of the
# kernel's source file (comments removed) at capture time: if the code has changed since, the figure
# is stale and the bench reports traffic as null.
MEASURED_TRAFFIC = {
    "decode_kernel": {
        "bytes_per_symbol": 1.8686,
        "source": "decode.cu",
        "sha256_prefix": "4ba1ae6f524ade66"
    },
    "encode_write_kernel": {
        "bytes_per_symbol": 2.0253,
        "source": "encode.cu",
        "sha256_prefix": "d5136af6dad60ad2"
    },
    "histogram_kernel": {
        "bytes_per_symbol": 1.0125,
        "source": "histogram.cu",
        "sha256_prefix": "48178df8a53eb610"
    },
    "build_tables_kernel": {
        "bytes_per_symbol": 0.0003,
        "source": "build_tables.cu",
        "sha256_prefix": "687e0c81ec448e3a"
    },
    "encode_compact_kernel": {
        "bytes_per_symbol": 1.7239,
        "source": "encode.cu",
        "sha256_prefix": "d5136af6dad60ad2"
    }
}


def source_digest(path):
    """sha256 prefix of a CUDA source with comments and blank lines removed, so that editing a
    comment does not invalidate a capture of the kernel."""
    import hashlib
    import re

    txt = open(path).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    txt = re.sub(r"//[^\n]*", "", txt)
    txt = "\n".join(ln.strip() for ln in txt.splitlines() if ln.strip())
    return hashlib.sha256(txt.encode()).hexdigest()[:16]


def measured_traffic(kernels, n_symbols):
    """Total DRAM bytes of the given kernels for n_symbols, or None if any capture is stale."""
    total = 0.0
    for k in kernels:
        m = MEASURED_TRAFFIC[k]
        if source_digest(os.path.join(ROOT, "entropy_coded_lossless_b200", "csrc", m["source"])) != m["sha256_prefix"]:
            return None
        total += m["bytes_per_symbol"] * n_symbols
    return total


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """SM clock and clock-event (throttle) reasons of this process's GPU, read through NVML every
    2 ms on a host thread (read-only queries; nothing is set). window() keeps the samples of the
    timed region and summary() reports their median SM clock, the maximum clock and every reason
    seen active. Falls back to nvidia-smi at 100 ms when NVML is unavailable."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, device):
        self.device = device
        self.samples = []  # (host time, sm MHz, reasons bitmask)
        self.max_mhz = None
        self.source = None
        self._stop = threading.Event()
        self._thread = None
        self._proc = None

    def _nvml_handle(self):
        import pynvml

        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.device)
        bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
        return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons

            def loop():
                while not self._stop.is_set():
                    try:
                        self.samples.append((time.time(), float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                             int(get_reasons(h))))
                    except Exception:
                        pass
                    time.sleep(0.002)

            self.source = "nvml, 2 ms"
        except Exception:
            loop = self._smi_loop
            self.source = "nvidia-smi, 100 ms"
        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()
        return self

    def _smi_loop(self):
        idx = torch.cuda.current_device() if self.device is None else torch.device(self.device).index or 0
        try:
            self._proc = subprocess.Popen(
                ["nvidia-smi", f"--id={idx}", "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except Exception:
            return
        for line in self._proc.stdout:
            parts = [v.strip() for v in line.split(",")]
            try:
                self.max_mhz = float(parts[1])
                self.samples.append((time.time(), float(parts[0]), int(parts[2], 16)))
            except (ValueError, IndexError):
                continue
            if self._stop.is_set():
                break

    def window(self, t0, t1):
        """Keep only the samples taken between host times t0 and t1."""
        self.samples = [v for v in self.samples if t0 <= v[0] <= t1]

    def __exit__(self, *a):
        self._stop.set()
        if self._proc is not None:
            self._proc.terminate()
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0, "source": self.source}
        seen = 0
        for _, _, r in self.samples:
            seen |= r
        return {"sm_mhz": statistics.median(v[1] for v in self.samples), "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(v[1] for v in self.samples),
                "reasons": [n for n, bit in self.REASONS if seen & bit], "samples": len(self.samples),
                "source": self.source}


def stream_rate(stream_np, segs, p, hist, mask=None):
    """RP (payload bits/symbol), total bits/symbol and H from the stream and histograms (host, fp64).
    mask: segments to count (default all; the total then still covers the whole stream)."""
    hdr = np.frombuffer(stream_np[:64].tobytes(), dtype="<u8")
    index_off, payload_off = int(hdr[5]), int(hdr[6])
    n_segs = len(segs)
    descs = np.frombuffer(stream_np[64:64 + 32 * n_segs].tobytes(), dtype="<u4").reshape(n_segs, 8)
    total_chunks = int(hdr[4])
    index = np.frombuffer(stream_np[index_off:index_off + 4 * total_chunks].tobytes(), dtype="<u4").astype(np.int64)
    words = np.frombuffer(stream_np[payload_off:].tobytes()[: (len(stream_np) - payload_off) // 4 * 4], dtype="<u4")
    payload_bits = 0
    sel = [s for s in range(n_segs) if mask is None or mask[s]]
    for s in sel:
        first = int(descs[s, 7])
        nch = -(-segs[s][1] // p["chunk_symbols"])
        start_w = int(descs[s, 4] | (descs[s, 5] << 32)) // 4
        pay_words = int(descs[s, 6])
        if nch == 0:
            continue
        ends = np.append(index[first + 1:first + nch], pay_words)
        last = words[start_w + ends - 1].astype(np.int64)
        hb = np.floor(np.log2(np.maximum(last, 1))).astype(np.int64)
        T = 32 * (ends - 1) + hb  # sentinel position = bits before it
        T -= 32 * np.append(0, ends[:-1])
        payload_bits += int(T.sum()) - nch * p["states_per_chunk"] * p["log2L"]
    n = sum(segs[s][1] for s in sel)
    h = hist.reshape(-1, 256).astype(np.float64)
    ent = 0.0
    for s in sel:
        row = h[s]
        tot = row.sum()
        if tot > 0:
            q = row[row > 0] / tot
            ent += float(-(q * np.log2(q)).sum()) * tot
    H = ent / n
    rp = payload_bits / n
    return {"payload": rp, "total": 8.0 * len(stream_np) / n, "entropy": H, "diff_pct": (rp - H) / H * 100.0}


def theorem1_terms(stream_np, hist, R, mask=None):
    """Shannonic §4, Theorem 1, per run: the code length closed form CL = H(P) + D_KL(P||Q) + sum_k P_k w_k
    of every segment, from its histogram (host fp64) and the table record its stream carries (f, lo),
    averaged over all symbols. P_k is the share of values in range k, Q_k = f_k / L the share of tANS
    states it got, w_k = ceil(log2 |range k|) its offset width. With H the histogram entropy and
    H(p|P) = H - H(P) the entropy left inside the ranges, the payload rate decomposes as
        RP - H = D_KL(P||Q)                      (state-count quantisation, L finite)
               + [sum_k P_k w_k - H(p|P)]        (fixed-width offsets, K ranges)
               + [RP - CL]                       (the spread: tANS against its ideal Q)."""
    hdr = np.frombuffer(stream_np[:64].tobytes(), dtype="<u4")
    n_segs, K, tb = int(hdr[2]), int(hdr[3] & 0xFFFF), int(hdr[5])
    L = 1 << R
    h = hist.reshape(-1, 256).astype(np.float64)
    rec0 = 64 + 32 * n_segs
    acc = {"H": 0.0, "HP": 0.0, "DKL": 0.0, "offset": 0.0}
    n_all = 0.0
    for s in range(n_segs):
        row = h[s]
        n = row.sum()
        if n == 0 or (mask is not None and not mask[s]):
            continue
        rec = stream_np[rec0 + tb * s: rec0 + tb * s + 3 * K]
        f = np.frombuffer(rec[:2 * K].tobytes(), dtype="<u2").astype(np.float64)
        lo = rec[2 * K:3 * K].astype(np.int64)
        hi = np.append(lo[1:], 256)
        Pk = np.array([row[a:b].sum() for a, b in zip(lo, hi)]) / n
        w = np.array([int(b - a - 1).bit_length() for a, b in zip(lo, hi)], dtype=np.float64)
        nz = Pk > 0
        q = row[row > 0] / n
        acc["H"] += n * float(-(q * np.log2(q)).sum())
        acc["HP"] += n * float(-(Pk[nz] * np.log2(Pk[nz])).sum())
        acc["DKL"] += n * float((Pk[nz] * np.log2(Pk[nz] / (f[nz] / L))).sum())
        acc["offset"] += n * float((Pk * w).sum())
        n_all += n
    t = {k: v / n_all for k, v in acc.items()} if n_all else {k: 0.0 for k in acc}
    t["H_given_P"] = t["H"] - t["HP"]
    t["CL"] = t["HP"] + t["DKL"] + t["offset"]
    t["offset_excess"] = t["offset"] - t["H_given_P"]
    return {"H": t["H"], "H_P": t["HP"], "D_KL_P_Q": t["DKL"], "offset_bits": t["offset"],
            "H_p_given_P": t["H_given_P"], "offset_excess": t["offset_excess"], "CL": t["CL"]}


def rate_report(stream_np, segs, p, hist, mask=None):
    """stream_rate plus the Theorem-1 terms and the spread's excess RP - CL."""
    r = stream_rate(stream_np, segs, p, hist, mask)
    t = theorem1_terms(stream_np, hist, p["log2L"], mask)
    t["spread_excess"] = r["payload"] - t["CL"]
    r["theorem1"] = t
    return r


def oracle_matches(x_dev, segs, p, gpu_stream_np, cores, stream=None):
    """CPU-baseline leg: whether the oracle's SHN1 stream of the whole workload (all host threads)
    is byte-identical to the GPU's. `stream` is the oracle stream if one was already made."""
    import oracle

    if stream is None:
        xs = x_dev.view(torch.uint8).cpu().numpy()
        stream, _ = oracle.encode(xs, p["K"], p["log2L"], p["states_per_chunk"], p["chunk_symbols"], segments=segs,
                                  threads=cores)
    return bool(stream.size == gpu_stream_np.size and np.array_equal(stream, gpu_stream_np))


def cpu_baseline(x_dev, segs, p, budget_s, full_n, gpu_stream_np=None):
    """The CPU oracle as it stands (encode + decode, all host threads) on a bounded sample of the
    same workload: whole segments, as many as fit the time budget (at least one). With the GPU's
    stream of the whole workload it also reports whether the oracle's stream is byte-identical to
    it (reusing the timed sample's stream when the sample is the whole workload)."""
    import oracle

    cores = oracle.cpu_count()
    o0, n0 = segs[0]
    one = x_dev[o0:o0 + n0].cpu().numpy()
    t = time.perf_counter()
    s, _ = oracle.encode(one, p["K"], p["log2L"], p["states_per_chunk"], p["chunk_symbols"], threads=cores)
    rc, _ = oracle.decode(s, threads=cores)
    dt1 = time.perf_counter() - t
    # one thread, on a slice of the first segment (about a second of work)
    m = min(one.size, max(p["chunk_symbols"], int(one.size * min(1.0, 1.0 / max(dt1 * cores, 1e-3)))))
    t = time.perf_counter()
    s1, _ = oracle.encode(one[:m], p["K"], p["log2L"], p["states_per_chunk"], p["chunk_symbols"], threads=1)
    oracle.decode(s1, threads=1)
    one_thread_gbs = m / (time.perf_counter() - t) / 1e9
    k = max(1, min(len(segs), int(budget_s / max(dt1, 1e-3))))
    sample = [segs[i] for i in range(k)]
    xs = np.concatenate([x_dev[o:o + n].cpu().numpy() for o, n in sample])
    local = []
    off = 0
    for _, n in sample:
        local.append((off, n))
        off += n
    t = time.perf_counter()
    s, _ = oracle.encode(xs, p["K"], p["log2L"], p["states_per_chunk"], p["chunk_symbols"], segments=local,
                         threads=cores)
    rc, y = oracle.decode(s, threads=cores)
    dt = time.perf_counter() - t
    assert rc == 0 and np.array_equal(y, xs.view(np.uint8))
    del y
    nbytes = xs.size
    out = {"value": nbytes / dt / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle", "cpu_model": cpu_model(),
           "sample": f"{k} of {len(segs)} segments ({nbytes} bytes): histogram+DP+tables+encode+decode, "
                     f"{dt:.1f} s on {cores} host threads",
           "one_thread": {"value": one_thread_gbs, "unit": UNIT, "sample": f"first {m} bytes of segment 0"}}
    if gpu_stream_np is not None:
        whole = local == [(o, n) for o, n in segs]  # the sample is the workload, laid out the same way
        del xs
        out["oracle_identical"] = oracle_matches(x_dev, segs, p, gpu_stream_np, cores, stream=s if whole else None)
    return out


def run_regen(args):
    """Per-round table regeneration on the GPU (histogram + range selection + tables, every segment),
    at the two tensor sizes of the pages' preprocessing table: 51 MB (ResNet-50 weights, one table per
    ~13 MB tensor) and 8.7 GB (Gemma-2-9B weights, one table per ~21.75 MB tensor)."""
    from entropy_coded_lossless_b200 import shn

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    p = shn.CodecParams(16, 7, 4096, 4)
    cases = []
    for name, n, seg, paper_s in (("ResNet-50-sized weights", 51_000_000, 12_750_000, 0.052),
                                  ("Gemma-2-9B-sized weights", 8_700_000_000, 21_750_000, 15.4)):
        x = inputs.laplace_int8(n, 7.258, seed=7, device=dev)
        segs = shn.Segments([(o, min(seg, n - o)) for o in range(0, n, seg)])  # marshalled once
        codec_hist = torch.zeros(len(segs) * 256, dtype=torch.int64, device=dev)
        tables = shn.empty_aligned(len(segs) * shn.TABLE_BYTES, dev)
        stream = torch.cuda.current_stream()

        def regen():
            shn.shn_histogram(x, segs, codec_hist)
            shn.shn_build_tables(codec_hist, len(segs), p, tables)

        for _ in range(max(3, args.warmup)):
            regen()
        torch.cuda.synchronize()
        ts = []
        for _ in range(max(5, min(args.steps, 20))):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            regen()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        ms = statistics.median(ts)
        cases.append({"tensor": name, "bytes": n, "tables": len(segs), "gpu_ms": ms,
                      "paper_cpu_s": paper_s, "paper_hw": "Intel i9-10920X, 4 threads (context only)"})
        del x
        torch.cuda.empty_cache()
    print(json.dumps({"metric": "table regeneration time (histogram + DP range selection + tANS tables)",
                      "value": cases[-1]["gpu_ms"], "unit": "ms", "n_gpus": 1, "higher_is_better": False,
                      "dtype": "u8", "data": "synthetic", "config": {"workload": "regen", "K": 16, "L": 128},
                      "cases": cases}), flush=True)


def run_sweepgrid(args):
    """Every point of the 1 GiB sweep (H x C x K x L, 108 points): payload and total bits/value
    against the entropy, and the median encode/decode time of 3 runs (inputs > L2)."""
    from entropy_coded_lossless_b200 import shn

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    pts, cur_h, x = [], None, None
    for pt in inputs.sweep_points():
        if pt["H"] != cur_h:
            del x
            torch.cuda.empty_cache()
            x = inputs.sweep_stream_int8(pt["H"], seed=4, device=dev)
            cur_h = pt["H"]
        segs = [(0, x.numel())]
        p_dict = dict(K=pt["K"], log2L=int(pt["L"]).bit_length() - 1, chunk_symbols=pt["C"], states_per_chunk=4)
        p = shn.CodecParams(**p_dict)
        codec = shn.Codec(segs, p, device=dev)
        out = torch.empty(x.numel(), dtype=torch.uint8, device=dev)
        codec.histogram(x)
        codec.build()
        te, td = [], []
        for _ in range(3):
            a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            a.record(stream)
            codec.encode(x)
            b.record(stream)
            codec.decode(codec.stream_buf, codec.stream_buf.numel(), out)
            c.record(stream)
            torch.cuda.synchronize()
            te.append(a.elapsed_time(b))
            td.append(b.elapsed_time(c))
        ok = codec.status("enc")[0] == 0 and codec.status("dec")[0] == 0 and torch.equal(out, x.view(torch.uint8))
        nbytes = int(codec.out_bytes.item())
        rate = stream_rate(codec.stream_buf[:nbytes].cpu().numpy(), segs, p_dict, codec.hist.cpu().numpy())
        pts.append({"H": pt["H"], "C": pt["C"], "K": pt["K"], "L": pt["L"], "payload": rate["payload"],
                    "total": rate["total"], "entropy": rate["entropy"], "diff_pct": rate["diff_pct"],
                    "encode_ms": statistics.median(te), "decode_ms": statistics.median(td), "correct": bool(ok)})
        del codec, out
    print(json.dumps({"metric": "bits/symbol vs H and codec time over the 1 GiB sweep grid", "value":
                      sum(1 for q in pts if q["K"] == 16 and q["L"] == 128 and q["diff_pct"] <= 1.0),
                      "unit": "points with K=16, L=128 within 1% of H", "n_gpus": 1, "higher_is_better": True,
                      "dtype": "u8", "data": "synthetic", "config": {"workload": "sweepgrid"}, "points": pts}),
          flush=True)


def config_workloads(dev):
    """The other configurations, in the order they are measured: (name, description, tensor,
    segments, params, families or None). Drawn on the device from the same seeds the tests use."""
    b53 = inputs.LAPLACE_B_FOR_ENTROPY[5.3]
    base = dict(K=16, log2L=7, chunk_symbols=4096, states_per_chunk=4)
    yield ("config1_laplace_65536", "65,536 i.i.d. truncated discrete Laplace (H = 5.3 bits), seed 0",
           inputs.laplace_int8(65536, b53, seed=0, device=dev), None, dict(base), None)
    w = inputs.weight_like_int8(seed=1, device=dev)
    yield ("config2_weight_like_4096x1024", "weight-like [4096,1024], per-row absmax, 1% outliers x8, seed 1",
           w, None, dict(base), None)
    yield ("config2_plain_tans_L1024", "the same weight tensor, plain tANS: K = 256 identity ranges, L = 1024",
           w, None, dict(base, K=256, log2L=10), None)
    del w
    x, segs, fam = inputs.activation_batch_int8(1024, 65536, seed=3, device=dev)
    yield ("config4_activations_1024x65536", "1024 activation tensors x 65,536, per-tensor tables, seed 3",
           x, segs, dict(base), fam)
    del x
    for H in (2.0, 4.0, 5.3, 7.9):
        yield (f"config5_1GiB_H{H}", f"1 GiB truncated discrete Laplace, H = {H} bits, seed 4",
               inputs.sweep_stream_int8(H, seed=4, device=dev), None, dict(base), None)


def measure_config(shn, x, segs, p_dict, dev, stream, peak, reps=10, warmup=3):
    """Median CUDA-event time of each stage over `reps` runs of histogram -> tables -> encode ->
    decode (L2 flushed by a 256 MiB write before every run when the workload is below 256 MiB),
    the rate report, and whether the round trip is exact. Returns (dict, GPU stream on the host)."""
    p = shn.CodecParams(**p_dict)
    codec = shn.Codec(segs, p, device=dev)
    n = codec.n_symbols
    out = torch.empty(n, dtype=torch.uint8, device=dev)
    comp_cap = codec.stream_buf.numel()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if n < (1 << 28) else None
    names = ("histogram", "build", "encode", "decode")
    times = {k: [] for k in names}
    for r in range(warmup + reps):
        if flush is not None:
            flush.zero_()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        ev[0].record(stream)
        codec.histogram(x)
        ev[1].record(stream)
        codec.build()
        ev[2].record(stream)
        codec.encode(x)
        ev[3].record(stream)
        codec.decode(codec.stream_buf, comp_cap, out)
        ev[4].record(stream)
        torch.cuda.synchronize()
        if r >= warmup:
            for i, k in enumerate(names):
                times[k].append(ev[i].elapsed_time(ev[i + 1]))
    xb = x.view(torch.uint8).reshape(-1)
    expect = torch.cat([xb[o:o + m] for o, m in segs])
    ok = codec.status("enc")[0] == 0 and codec.status("dec")[0] == 0 and torch.equal(out, expect)
    del expect
    nbytes = int(codec.out_bytes.item())
    stream_np = codec.stream_buf[:nbytes].cpu().numpy()
    hist = codec.hist.cpu().numpy()
    st = {k: statistics.median(v) for k, v in times.items()}
    res = {"symbols": n, "segments": len(segs), "K": p.K, "L": 1 << p.log2L, "chunk_symbols": p.chunk_symbols,
           "states_per_chunk": p.states_per_chunk, "stream_bytes": nbytes, "correct": bool(ok),
           "ms": st, "step_ms": sum(st.values()),
           "encode_gbs_int8": n / (st["encode"] * 1e-3) / 1e9, "decode_gbs_int8": n / (st["decode"] * 1e-3) / 1e9,
           "encode_frac": (n + nbytes) / (st["encode"] * 1e-3) / 1e9 / peak,
           "decode_frac": (n + nbytes) / (st["decode"] * 1e-3) / 1e9 / peak,
           "timing": f"median of {reps} runs after {warmup} warm-up runs"
                     + ("; L2 flushed before each run" if flush is not None else "; inputs larger than L2"),
           "bits_per_symbol": rate_report(stream_np, segs, p_dict, hist)}
    del codec, out, flush
    return res, stream_np, hist


def rate_grid(shn, x, segs, dev, grid=((16, 8), (16, 9), (16, 10), (32, 8), (32, 10), (16, 12))):
    """Payload rate against the entropy at larger state counts (and K = 32) for a workload that
    misses 1 % of H at K = 16, L = 128: histogram, tables and encode on the GPU, rate and Theorem-1
    terms on the host."""
    pts = []
    for K, R in grid:
        p_dict = dict(K=K, log2L=R, chunk_symbols=4096, states_per_chunk=4)
        codec = shn.Codec(segs, shn.CodecParams(**p_dict), device=dev)
        codec.compress(x)
        ok = codec.status("enc")[0] == 0
        nbytes = int(codec.out_bytes.item())
        r = rate_report(codec.stream_buf[:nbytes].cpu().numpy(), segs, p_dict, codec.hist.cpu().numpy())
        t = r["theorem1"]
        pts.append({"K": K, "L": 1 << R, "ok": bool(ok), "payload": r["payload"], "entropy": r["entropy"],
                    "diff_pct": r["diff_pct"], "D_KL_P_Q": t["D_KL_P_Q"], "offset_excess": t["offset_excess"],
                    "spread_excess": t["spread_excess"]})
        del codec
    return pts


def run_configs(shn, dev, stream, peak, cpu_check):
    """Every configuration besides the headline one, measured on this GPU; with cpu_check the CPU
    baseline leg also compares each GPU stream with the oracle's, byte for byte."""
    res = {}
    cores = None
    for name, desc, x, segs, p_dict, fam in config_workloads(dev):
        if segs is None:
            segs = [(0, x.numel())]
        r, stream_np, hist = measure_config(shn, x, segs, p_dict, dev, stream, peak)
        r["workload"] = desc
        if fam is not None:  # per family of activation tensor
            names = ["laplace", "gaussian", "relu_gaussian"]
            r["by_family"] = {names[f]: rate_report(stream_np, segs, p_dict, hist, mask=[v == f for v in fam])
                              for f in range(3)}
        if p_dict["K"] != 256 and r["bits_per_symbol"]["diff_pct"] > 1.0:  # where K = 16, L = 128 misses 1 % of H
            r["rate_grid"] = rate_grid(shn, x, segs, dev)
        if cpu_check:
            import oracle

            cores = cores or oracle.cpu_count()
            t = time.perf_counter()
            r["oracle_identical"] = oracle_matches(x, segs, p_dict, stream_np, cores)
            r["oracle_check_s"] = time.perf_counter() - t
        res[name] = r
        del x, stream_np
        torch.cuda.empty_cache()
    return res


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    x, segs, p, desc = workload(args.workload, "cpu", entropy=args.entropy, sweep_bytes=args.sweep_bytes)
    apply_overrides(p, args)
    import oracle

    cores = oracle.cpu_count()
    # each step: a bounded sample (whole segments) of the workload, histogram → tables → encode → decode
    o0, n0 = segs[0]
    one = x[o0:o0 + n0].numpy()
    t = time.perf_counter()
    s, _ = oracle.encode(one, p["K"], p["log2L"], p["states_per_chunk"], p["chunk_symbols"], threads=cores)
    oracle.decode(s, threads=cores)
    dt1 = time.perf_counter() - t
    per_step_budget = 120.0 / max(1, args.steps + args.warmup)
    k = max(1, min(len(segs), int(per_step_budget / max(dt1, 1e-3))))
    sample = segs[:k]
    xs = np.concatenate([x[o:o + n].numpy() for o, n in sample])
    local, off = [], 0
    for _, n in sample:
        local.append((off, n))
        off += n

    def step():
        s, _ = oracle.encode(xs, p["K"], p["log2L"], p["states_per_chunk"], p["chunk_symbols"], segments=local,
                             threads=cores)
        rc, y = oracle.decode(s, threads=cores)
        assert rc == 0

    for _ in range(args.warmup):
        step()
    t = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t) / args.steps
    v = xs.size / dt / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u8", "data": "synthetic",
            "config": {"workload": desc, "K": p["K"], "L": 1 << p["log2L"], "chunk_symbols": p["chunk_symbols"],
                       "states_per_chunk": p["states_per_chunk"], "sample_segments": k,
                       "seed": WORKLOAD_SEED.get(args.workload)},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "cpu_model": cpu_model(),
                             "sample": f"{k} of {len(segs)} segments per step ({xs.size} bytes)"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "regen":
        return run_regen(args)
    if args.workload == "sweepgrid":
        return run_sweepgrid(args)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    from entropy_coded_lossless_b200 import shn

    x, segs, p_dict, desc = workload(args.workload, dev, seed_offset=rank, n_segments=args.segments,
                                     entropy=args.entropy, sweep_bytes=args.sweep_bytes)
    apply_overrides(p_dict, args)
    p = shn.CodecParams(**p_dict)
    codec = shn.Codec(segs, p, device=dev)
    n = codec.n_symbols
    out = torch.empty(n, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    comp_cap = codec.stream_buf.numel()
    if args.profile_only:
        # (kv: also the fused bf16 decode after each INT8 decode, so its launches can be captured too)
        scales = y16 = None
        if args.workload == "kv":
            scales = torch.cat([inputs.kv_cache_segment_int8_and_scales(i // 2, i % 2, seed=2 + rank, device=dev)[1]
                                for i in range(len(segs))])
            y16 = torch.empty(n, dtype=torch.bfloat16, device=dev)
        for _ in range(2):
            codec.compress(x)
            codec.decode(codec.stream_buf, comp_cap, out)
            if y16 is not None:
                shn.shn_decode_bf16(codec.stream_buf, comp_cap, p, scales, 7, codec.work_dec, y16)
        torch.cuda.synchronize()
        ok = codec.status("enc")[0] == 0 and codec.status("dec")[0] == 0 and torch.equal(out, x.view(torch.uint8))
        print(json.dumps({"profile_case": desc, "symbols": n, "stream_bytes": int(codec.out_bytes.item()),
                          "correct": bool(ok)}))
        if world > 1:
            torch.distributed.destroy_process_group()
        sys.exit(0 if ok else 3)

    stage_names = ("histogram", "build", "encode", "decode")
    stage_ms = {k: 0.0 for k in stage_names}

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        codec.histogram(x)
        if evs:
            evs[1].record(stream)
        codec.build()
        if evs:
            evs[2].record(stream)
        codec.encode(x)
        if evs:
            evs[3].record(stream)
        codec.decode(codec.stream_buf, comp_cap, out)
        if evs:
            evs[4].record(stream)

    # events for every timed step, read only after the last one (no host sync inside the region)
    evs_all = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    # a workload that fits in L2 is timed with L2 flushed before every step (a 256 MiB write outside
    # the stage events); its step time is then the sum of the stage events
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if n < (1 << 28) else None
    with ClockSampler(dev) as clk:
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        h0 = time.time()
        t0.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.zero_()
            step(evs_all[i])
        t1.record(stream)
        torch.cuda.synchronize()
        h1 = time.time()
        time.sleep(0.15)
    clk.window(h0, h1)
    for evs in evs_all:
        for i, k in enumerate(stage_names):
            stage_ms[k] += evs[i].elapsed_time(evs[i + 1])
    if world > 1:
        torch.distributed.barrier()
    ms_region = t0.elapsed_time(t1) if flush is None else sum(stage_ms.values())
    ms_total = max_over_ranks(ms_region, dev)
    ms_step = ms_total / args.steps

    # correctness of the timed work
    est, edet = codec.status("enc")
    dst, ddet = codec.status("dec")
    ok = est == 0 and dst == 0 and torch.equal(out, x.view(torch.uint8))
    nbytes = int(codec.out_bytes.item())
    stream_np = codec.stream_buf[:nbytes].cpu().numpy()
    rate = rate_report(stream_np, segs, p_dict, codec.hist.cpu().numpy())
    if args.workload == "int4":  # bits per weight as the pages count them: codes + one 32-bit scale per 64
        rate["total_with_group_scales"] = rate["total"] + 32 / 64
        rate["int4_alone_with_group_scales"] = 4 + 32 / 64

    # e2e through the C ABI with host buffers: every step copies its input from pinned host memory,
    # runs the four calls and copies its stream and status words back. Steps are software-pipelined
    # over three streams (H2D, compute, D2H; double-buffered device input and stream), so one step's
    # D2H overlaps the next step's H2D on the other copy engine.
    e2e = None
    if not args.no_e2e:
        h_in = torch.empty(n, dtype=torch.int8, pin_memory=True)
        h_in.copy_(x.cpu())
        h_out = [torch.empty(comp_cap, dtype=torch.uint8, pin_memory=True) for _ in range(2)]
        h_st = [torch.empty(16, dtype=torch.uint8, pin_memory=True) for _ in range(2)]
        codecs = [codec, shn.Codec(segs, p, device=dev)]
        outs = [out, torch.empty_like(out)]
        x_e = [torch.empty_like(x) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        for b in range(2):  # all buffers start free
            ev_comp[b].record(stream)
            ev_out[b].record(stream)

        def e2e_step(i):
            b = i & 1
            cd = codecs[b]
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_comp[b])  # step i-2 no longer reads x_e[b]
                x_e[b].copy_(h_in, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])  # step i-2's stream has left the device
            cd.histogram(x_e[b], stream)
            cd.build(stream)
            cd.encode(x_e[b], stream)
            cd.decode(cd.stream_buf, comp_cap, outs[b], stream)
            ev_comp[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b])
                h_out[b][:nbytes].copy_(cd.stream_buf[:nbytes], non_blocking=True)
                h_st[b][:8].copy_(cd.work_enc[:8], non_blocking=True)
                h_st[b][8:16].copy_(cd.work_dec[:8], non_blocking=True)
                ev_out[b].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ksteps = max(2, args.steps)  # the same K steps as the device-timed figure
        e0.record(stream)
        s_in.wait_event(e0)
        for i in range(ksteps):
            e2e_step(i)
        stream.wait_stream(s_out)
        e1.record(stream)
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(e0.elapsed_time(e1) / ksteps, dev)
        e2e_ok = all(bool(torch.equal(h_out[b][:nbytes], h_out[0][:nbytes])) for b in range(2)) and \
            all(int(h_st[b].view(torch.int32)[0]) == 0 and int(h_st[b].view(torch.int32)[2]) == 0 for b in range(2))
        e2e = {"value": whole_job_gbs(n, world, ms_e2e), "unit": UNIT, "h2d_bytes_per_step": n,
               "d2h_bytes_per_step": nbytes + 16, "ms_per_step": ms_e2e, "correct": e2e_ok,
               "what": "pinned H2D input + shn_histogram + shn_build_tables + shn_encode + shn_decode + D2H stream/status; "
                       "steps pipelined over H2D / compute / D2H streams (double-buffered)"}

    # Decode fused with the KV cache's dequantisation (bf16 = int8 x scale per head_dim group of 128),
    # against the unfused path a user would otherwise run: shn_decode, then a PyTorch dequantisation.
    fused = None
    if args.workload == "kv" and not args.segments and not args.no_fused:
        scales = inputs.kv_cache_scales(seed=2 + rank, device=dev)
        y16 = torch.empty(n, dtype=torch.bfloat16, device=dev)

        def run_fused():
            shn.shn_decode_bf16(codec.stream_buf, comp_cap, p, scales, 7, codec.work_dec, y16)

        def run_unfused():
            codec.decode(codec.stream_buf, comp_cap, out)
            return (out.view(torch.int8).view(-1, 128).float() * scales[:, None]).to(torch.bfloat16).reshape(-1)

        def timed(fn, reps=5):
            fn()
            torch.cuda.synchronize()
            ts = []
            for _ in range(reps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                r = fn()
                b.record(stream)
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b))
            return sorted(ts)[len(ts) // 2], r

        ms_f, _ = timed(run_fused)
        fused_ok = codec.status("dec")[0] == 0
        ms_u, y_ref = timed(run_unfused)
        fused_ok = fused_ok and torch.equal(y16.view(torch.int16), y_ref.view(torch.int16))
        del y_ref
        torch.cuda.empty_cache()
        fused = {"what": "shn_decode_bf16: decode + bf16 dequantisation (scale per 128 values) in one kernel",
                 "ms": ms_f, "gbs_int8": n / (ms_f * 1e-3) / 1e9,
                 "alg_bytes_per_launch": nbytes + 2 * n + 4 * (n >> 7),
                 "unfused_ms": ms_u, "unfused": "shn_decode then (int8.float() * scale).to(bfloat16) in PyTorch",
                 "speedup_vs_unfused": ms_u / ms_f, "matches_unfused": bool(fused_ok)}

    # Compressed offload to host memory and pipelined reload (8 streams of 8 segments each), against
    # plain pinned copies of the INT8 tensor over the same link.
    offl = None
    if args.workload == "kv" and not args.segments and not args.no_offload:
        ends = list(range(8, len(segs) + 1, 8))
        batches = [segs[a:b] for a, b in zip([0] + ends[:-1], ends)]
        owork = shn.empty_aligned(shn.offload_workspace_bytes(p, segs, ends), dev)
        h_all = torch.empty(comp_cap + 16 * len(batches), dtype=torch.uint8, pin_memory=True)
        h_raw = torch.empty(n, dtype=torch.uint8, pin_memory=True)
        wrk = shn.empty_aligned(256, dev)
        back = torch.empty(n, dtype=torch.uint8, device=dev)
        copy_stream = torch.cuda.Stream(dev)
        placed = {}

        segs_c = shn.Segments(segs)  # marshalled once

        def do_offload():  # blocks until the last batch is encoded; the copies finish on copy_stream
            placed["offs"], placed["sizes"] = shn.shn_offload(x, segs_c, ends, p, owork, h_all, stream, copy_stream)
            stream.wait_stream(copy_stream)

        do_offload()
        torch.cuda.synchronize()
        sizes = placed["sizes"]
        hosts = [h_all[o:o + b] for o, b in zip(placed["offs"], sizes)]
        offsets = np.cumsum([0] + [sum(ln for _, ln in b) for b in batches])[:-1].tolist()
        staging = shn.empty_aligned(2 * max(-(-v // 16) * 16 for v in sizes), dev, 16)

        def do_reload():
            shn.shn_decode_from_host(hosts, sizes, p, staging, wrk, back, offsets, stream, copy_stream)

        def ev_time(fn, reps=3):
            fn()
            torch.cuda.synchronize()
            ts = []
            for _ in range(reps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b))
            return sorted(ts)[len(ts) // 2]

        ms_off = ev_time(do_offload)
        ms_rel = ev_time(do_reload)
        reload_ok = shn.shn_get_device_status(wrk)[0] == 0 and torch.equal(back, x.view(torch.uint8))
        ms_d2h = ev_time(lambda: h_raw.copy_(x.view(torch.uint8), non_blocking=True))
        ms_h2d = ev_time(lambda: back.copy_(h_raw, non_blocking=True))
        comp = sum(sizes)
        offl = {"what": "shn_offload: 8 streams of 8 segments, each copied to pinned host memory by the copy engine "
                        "while the next encodes; shn_decode_from_host copying them back while the previous decodes",
                "compressed_bytes": comp, "int8_bytes": n,
                "offload_ms": ms_off, "offload_gbs_int8": n / (ms_off * 1e-3) / 1e9,
                "reload_ms": ms_rel, "reload_gbs_int8": n / (ms_rel * 1e-3) / 1e9,
                "raw_d2h_ms": ms_d2h, "raw_h2d_ms": ms_h2d,
                "offload_vs_raw": ms_d2h / ms_off, "reload_vs_raw": ms_h2d / ms_rel,
                "reload_correct": bool(reload_ok)}
        del hosts, h_all, h_raw, staging, back, owork

    if rank == 0:
        peak, peak_kind = measured_peaks()
        if fused is not None:
            fused["achieved_gbs"] = fused["alg_bytes_per_launch"] / (fused["ms"] * 1e-3) / 1e9
            fused["frac"] = fused["achieved_gbs"] / peak
        stages = {}
        for k, v in stage_ms.items():
            ms = v / args.steps
            stages[k] = {"ms": ms, "gbs_int8": n / (ms * 1e-3) / 1e9 if ms > 0 else None}
        alg = {"histogram": n, "build": 0, "encode": n + nbytes, "decode": n + nbytes}
        dom = max(("encode", "decode", "histogram"), key=lambda k: stages[k]["ms"])
        if offl is not None:
            # Shannonic §6, when compression pays: sender encodes, the link carries CSR of the bytes,
            # the receiver decodes, one after the other; with every rate INT8-side that is
            # CSR < 1 - R_link (1/R_enc + 1/R_dec). R_enc covers histogram + tables + encode.
            ms_enc = stages["histogram"]["ms"] + stages["build"]["ms"] + stages["encode"]["ms"]
            ms_dec = stages["decode"]["ms"]
            csr = offl["compressed_bytes"] / n
            cond = {"csr": csr, "r_enc_gbs": n / ms_enc / 1e6, "r_dec_gbs": n / ms_dec / 1e6}
            for d in ("d2h", "h2d"):
                r_link = n / offl[f"raw_{d}_ms"] / 1e6
                csr_max = 1.0 - r_link * (1.0 / cond["r_enc_gbs"] + 1.0 / cond["r_dec_gbs"])
                cond[d] = {"r_link_gbs": r_link, "csr_max": csr_max, "pays": bool(csr < csr_max)}
            offl["latency_condition"] = cond

        kernels_of = {"decode": ["decode_kernel"], "encode": ["encode_write_kernel", "encode_compact_kernel"],
                      "histogram": ["histogram_kernel"]}

        def roof(k):
            ms = stages[k]["ms"]
            a = alg[k] / (ms * 1e-3) / 1e9
            return {"bound": "hbm", "achieved": a, "peak": peak, "unit": "GB/s", "frac": a / peak,
                    "traffic": measured_traffic(kernels_of[k], n), "kernel": "+".join(kernels_of[k]),
                    "alg_bytes_per_launch": alg[k], "peak_kind": peak_kind,
                    "timing": "CUDA events around the C-ABI call on the launching stream, mean over the timed steps"}

        launches_per_step = kernel_launches_per_step(segs, p_dict)
        line = {
            "metric": METRIC,
            "value": whole_job_gbs(n, world, ms_step),
            "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "u8",
            "data": "synthetic",
            "config": {"workload": desc, "K": p.K, "L": 1 << p.log2L, "chunk_symbols": p.chunk_symbols,
                       "states_per_chunk": p.states_per_chunk, "bytes_per_gpu": n,
                       "seed": None if WORKLOAD_SEED.get(args.workload) is None else WORKLOAD_SEED[args.workload] + rank,
                       "l2": "inputs larger than L2 (input, stream and output each > 126 MB per step)"
                       if flush is None else "L2 flushed (256 MiB write) before every step; step time = sum of stage events",
                       "parallelism": f"replicas x{world} (independent segments per rank)"},
            "step": "histogram + DP/tables + encode + decode (value = INT8 bytes per step / step time)",
            "stages": stages,
            "roofline": roof(dom),
            "roofline_decode": roof("decode"),
            "roofline_encode": roof("encode"),
            "bits_per_symbol": rate,
            "stream_bytes": nbytes,
            "correct": bool(ok),
            "clocks": clk.summary(),
            "decode_bf16_fused": fused,
            "offload": offl,
            "gpu_launches": launches_per_step * args.steps,
            "e2e": e2e,
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(x, segs, p_dict, args.cpu_sample_seconds, n, gpu_stream_np=stream_np)
            line["oracle_identical"] = line["cpu_baseline"]["oracle_identical"]
        if args.workload == "kv" and not args.segments and not args.no_configs:
            del x, out, codec
            torch.cuda.empty_cache()
            line["configs"] = run_configs(shn, dev, stream, peak, cpu_check=not args.no_cpu_baseline and world == 1)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    if not ok:
        sys.exit(3)


if __name__ == "__main__":
    main()
