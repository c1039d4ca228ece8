"""Benchmark: quantized paged KV append + decode attention on B200.

One step = append one new token per sequence (quantise + store) and run the
decode attention over every sequence's cache (all steps of the hot path), with
the prefix already in the cache and all inputs resident in HBM.  The headline
workload is INT8-G64 (batch 8, lengths uniform in [1024, 8192], 8 kv-heads,
32 query heads, head_dim 256, 64-token pages); the other formats' workloads are
reported under "formats", and the chunked-prefill workload (append a 512-token
chunk per sequence + causal attention of its queries, against the tensor-core
roofline) under "prefill".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--quick]
                    [--prefill-only]

N > 1: launched by torchrun, one rank per GPU; every rank runs its own replica
(the path has no exchange step), timings are the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_paged_kv_03_b200 import inputs as I   # noqa: E402

METRIC = "quantized-KV paged decode attention: HBM GB/s, % of peak, tokens/s per format"
HEADLINE_CONFIG = 1
L2_FLUSH_BYTES = 256 << 20


def make_l2_flush(torch):
    """Flush the L2 between timed calls: write a buffer larger than L2, then read
    another one, so the timed call starts with a cold L2 that holds no dirty lines
    (whose write-back would otherwise compete with the call's first reads)."""
    wbuf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    rbuf = torch.zeros(L2_FLUSH_BYTES // 8, dtype=torch.float64, device="cuda")

    def flush():
        wbuf.fill_(1)
        rbuf.sum()
    return flush


# From an ncu capture of the fused step's decode_kernel launch on the headline
# workload: DRAM bytes read + written per launch.  It describes the kernel built
# from the sources with this digest only (null for any other build).
HEADLINE_TRAFFIC = {"bytes": 127_864_013 + 4_574_703,
                    "sources_sha256": "91cf11454ddfe22d953ee2ab311bce4d567f51e7b855c816619a04313cb59c68"}
KERNEL_SOURCES = ("kvq_decode.cu", "kvq_common.cuh", "kvq_quant.cuh", "kvq_internal.h")


# The same for the chunked-prefill kernel on its workload.
PREFILL_TRAFFIC = {"bytes": 173_958_912 + 38_617_515,
                   "sources_sha256": "317fa9a46181eca3319643d4c7bc3ffde291a7a013326c6d7185427ff47037b8"}
PREFILL_SOURCES = ("kvq_prefill.cu", "kvq_prefill.h", "kvq_tc.cuh", "kvq_common.cuh")


def kernel_digest(files=KERNEL_SOURCES) -> str:
    """sha256 of a kernel's sources with comments and whitespace removed:
    edits to comments keep a recorded capture valid, code edits void it."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "quantized_paged_kv_03_b200", "csrc", f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()


def headline_traffic(config: int, batch) -> int | None:
    """The captured traffic when it applies to this run (same kernel, same workload)."""
    if config != HEADLINE_CONFIG or batch is not None:
        return None
    return HEADLINE_TRAFFIC["bytes"] if kernel_digest() == HEADLINE_TRAFFIC["sources_sha256"] else None


def prefill_traffic() -> int | None:
    ok = kernel_digest(PREFILL_SOURCES) == PREFILL_TRAFFIC["sources_sha256"]
    return PREFILL_TRAFFIC["bytes"] if ok else None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------- accounting

def decode_bytes(w: I.Workload, token_bytes: int, out_bytes_per_elem: int = 4) -> int:
    """Algorithmic bytes of one decode: KV pages read + q + out + block table + seq_lens."""
    kv = int(w.seq_lens.astype(np.int64).sum()) * w.H * token_bytes
    pages = int(((w.seq_lens.astype(np.int64) + w.P - 1) // w.P).sum())
    return kv + w.B * w.Hq * w.D * 2 + w.B * w.Hq * w.D * out_bytes_per_elem + pages * 4 + w.B * 4


def append_bytes(n_tokens: int, w: I.Workload, token_bytes: int) -> int:
    """Algorithmic bytes of one append: bf16 K and V read, codes + scales written, slots."""
    return n_tokens * w.H * (2 * w.D * 2 + token_bytes) + 8 * n_tokens


# ---------------------------------------------------------------- clocks

class ClockSampler:
    def __init__(self, path):
        self.path, self.proc = path, None

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,"
                 "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
                 "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                 "clocks_event_reasons.sw_power_cap", "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self, device_index=0):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9 or not f[1].isdigit():
                continue
            if int(f[0]) != device_index:
                continue
            rows.append(f)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [int(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": int(rows[0][2]), "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- GPU arm

class Arm:
    """One workload on the GPU: cache with the prefix appended, step inputs in HBM."""

    def __init__(self, cfg: int, fmt: str, seed_offset: int = 0, batch: int | None = None):
        import torch
        import quantized_paged_kv_03_b200 as K
        self.torch, self.K = torch, K
        spec = I.CONFIGS[cfg]
        seed = I.SEED_BASE + cfg + 1000 * seed_offset
        self.w = w = I.make_workload(cfg, fmt=fmt, seed=seed, B=batch)
        self.fmt = fmt
        self.tb = K.token_bytes(fmt, w.D)
        scales = None
        if fmt == "fp8_tensor":
            scales = [(I.tensor_amax(w.k) / 448.0 or 1.0, I.tensor_amax(w.v) / 448.0 or 1.0)]
        self.scales = scales
        self.cache = K.KVCache(fmt, w.D, w.H, w.P, w.num_pages, 1, 0, scales)
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
        kp, vp, sp = w.prefix()
        step = 1 << 20
        for i in range(0, len(sp), step):     # bulk prefill, untimed
            self.cache.append(0, dev(kp[i:i + step]).view(torch.bfloat16),
                              dev(vp[i:i + step]).view(torch.bfloat16), dev(sp[i:i + step]))
        # a bulk append to time on its own: the prefix's first rows again (same
        # slots, same codes), at most 2^18 tokens
        na = min(len(sp), 1 << 18)
        self.app_k = dev(kp[:na]).view(torch.bfloat16)
        self.app_v = dev(vp[:na]).view(torch.bfloat16)
        self.app_s = dev(sp[:na])
        self.bulk_tokens = na
        del kp, vp
        kn, vn, sn = w.new_tokens()
        self.h_k, self.h_v, self.h_s = kn, vn, sn
        self.k_new = dev(kn).view(torch.bfloat16)
        self.v_new = dev(vn).view(torch.bfloat16)
        self.slots = dev(sn)
        self.q = dev(w.q).view(torch.bfloat16)
        self.bt = dev(w.block_table)
        self.sl = dev(w.seq_lens)
        self.out = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
        self.ws = self.cache.workspace(w.B, w.Hq, w.max_seq_len)
        self.dec_bytes = decode_bytes(w, self.tb)
        self.app_bytes = append_bytes(w.B, w, self.tb)
        self.bulk_bytes = append_bytes(self.bulk_tokens, w, self.tb)
        self.qerr = self.quant_error()
        self.w.k = self.w.v = None     # host copies no longer needed
        torch.cuda.synchronize()

    def quant_error(self, n_samples: int = 3):
        """Quantisation error, for information: one fused step's outputs against
        fp64 attention over the unquantised bf16 K/V (the values a BF16 cache
        holds), on sampled (sequence, kv-head) pairs -- the shortest, the
        longest and a middle-length sequence, kv-head 0 and the last kv-head."""
        torch, w = self.torch, self.w
        self.step()
        out = self.out.double()
        G = w.Hq // w.H
        order = np.argsort(w.seq_lens, kind="stable")
        seqs = sorted({int(order[0]), int(order[len(order) // 2]), int(order[-1])})[:n_samples]
        bf16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(
            torch.bfloat16).double()
        worst_max, worst_rms = 0.0, 0.0
        for b in seqs:
            rows = slice(int(w.starts[b]), int(w.starts[b + 1]))
            for h in sorted({0, w.H - 1}):
                k, v = bf16(w.k[rows, h]), bf16(w.v[rows, h])
                q = bf16(w.q[b, h * G:(h + 1) * G])
                ref = torch.softmax((q @ k.T) / np.sqrt(w.D), dim=-1) @ v
                err = out[b, h * G:(h + 1) * G] - ref
                worst_max = max(worst_max, float(err.abs().max() / v.abs().max()))
                worst_rms = max(worst_rms, float(err.norm() / ref.norm()))
                del k, v
        return {"max_abs_over_max_abs_v": round(worst_max, 6), "rel_rms": round(worst_rms, 6)}

    def step(self):
        """One decode step, one launch: append each sequence's new token and attend."""
        self.cache.append_decode(0, self.k_new, self.v_new, self.q, self.bt, self.sl, self.w.max_seq_len,
                                 out=self.out, workspace=self.ws)

    def bulk_append(self):
        self.cache.append(0, self.app_k, self.app_v, self.app_s)

    def decode_only(self):
        self.cache.decode_attention(0, self.q, self.bt, self.sl, self.w.max_seq_len, out=self.out,
                                    workspace=self.ws)

    def run(self, steps: int, warmup: int, flush, fn=None):
        """Device-timed calls (CUDA events on the launching stream), L2 flushed
        before each call outside the events.  Returns milliseconds per call."""
        torch = self.torch
        fn = fn or self.step
        for _ in range(warmup):
            flush()
            fn()
        torch.cuda.synchronize()
        s = torch.cuda.current_stream()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for i in range(steps):
            flush()
            ev[i][0].record(s)
            fn()
            ev[i][1].record(s)
        torch.cuda.synchronize()
        return np.array([e[0].elapsed_time(e[1]) for e in ev])

    def run_e2e(self, steps: int, warmup: int, flush):
        """Same step through the public API from pinned host memory: H2D of the
        step's inputs, append, decode, D2H of the output, all inside the events.
        The inputs (new K and V rows, q, block table, seq_lens) sit in one pinned
        host buffer, each part 256-byte aligned, and go over in one copy into one
        device buffer whose parts the call takes as its arguments."""
        torch = self.torch
        parts = [np.ascontiguousarray(a) for a in (self.h_k, self.h_v, self.w.q, self.w.block_table, self.w.seq_lens)]
        offs, off = [], 0
        for a in parts:
            offs.append(off)
            off = (off + a.nbytes + 255) & ~255
        hbuf = torch.zeros(off, dtype=torch.uint8).pin_memory()
        hnp = hbuf.numpy()
        for a, o in zip(parts, offs):
            hnp[o:o + a.nbytes] = a.reshape(-1).view(np.uint8)
        dbuf = torch.empty(off, dtype=torch.uint8, device="cuda")

        def part(i, like):
            return dbuf[offs[i]:offs[i] + parts[i].nbytes].view(like.dtype).view(like.shape)

        k, v, q = part(0, self.k_new), part(1, self.v_new), part(2, self.q)
        bt, sl = part(3, self.bt), part(4, self.sl)
        hout = torch.empty(self.out.shape, dtype=torch.float32).pin_memory()
        h2d = sum(a.nbytes for a in parts)
        d2h = hout.numel() * 4
        s = torch.cuda.current_stream()

        def one():
            dbuf.copy_(hbuf, non_blocking=True)
            self.cache.append_decode(0, k, v, q, bt, sl, self.w.max_seq_len, out=self.out, workspace=self.ws)
            hout.copy_(self.out, non_blocking=True)

        for _ in range(warmup):
            flush()
            one()
        torch.cuda.synchronize()
        ts = []
        for _ in range(steps):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(s)
            one()
            b.record(s)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return np.array(ts), h2d, d2h


# ---------------------------------------------------------------- prefill arm

def prefill_flops(seq_lens, q_lens, Hq: int, D: int) -> int:
    """Algorithmic FLOPs of a chunked-prefill attention: 4 * D per (query row,
    visible key) -- q.k and p.v, a multiply and an add per dimension each.
    Query token i of a chunk of n sees L - n + i + 1 keys (causal)."""
    keys = 0
    for L, n in zip(seq_lens, q_lens):
        first = int(L) - int(n) + 1
        k = np.arange(first, first + int(n), dtype=np.int64)
        keys += int(k[k > 0].sum())
    return 4 * D * Hq * keys


class PrefillArm:
    """The chunked-prefill workload on the GPU: the prefix of every sequence in
    the cache, the chunk's K/V rows, slots and queries resident in HBM.  One
    step = append the chunk (kvq_append) + the causal attention of its queries
    (kvq_prefill_attention)."""

    def __init__(self, seed_offset: int = 0):
        import torch
        import quantized_paged_kv_03_b200 as K
        self.torch = torch
        spec, n = I.PREFILL, I.PREFILL_CHUNK
        self.w = w = I.make_workload(spec, seed=I.PREFILL_SEED + 1000 * seed_offset)
        fmt = spec.formats[0]
        self.cache = K.KVCache(fmt, w.D, w.H, w.P, w.num_pages)
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
        pre, pre_s, ch, ch_s = [], [], [], []
        for b in range(w.B):
            L, s0 = int(w.seq_lens[b]), int(w.starts[b])
            pre.append(np.arange(s0, s0 + L - n))
            pre_s.append(w.slots(b, 0, L - n))
            ch.append(np.arange(s0 + L - n, s0 + L))
            ch_s.append(w.slots(b, L - n, L))
        pre, pre_s, ch = np.concatenate(pre), np.concatenate(pre_s), np.concatenate(ch)
        step = 1 << 18
        for i in range(0, len(pre), step):     # the prefix, untimed
            r = pre[i:i + step]
            self.cache.append(0, dev(w.k[r]).view(torch.bfloat16), dev(w.v[r]).view(torch.bfloat16),
                              dev(pre_s[i:i + step]))
        self.k_ch = dev(w.k[ch]).view(torch.bfloat16)
        self.v_ch = dev(w.v[ch]).view(torch.bfloat16)
        self.s_ch = dev(np.concatenate(ch_s))
        self.q_lens = np.full(w.B, n, np.int64)
        hq, cu = I.prefill_queries(w, self.q_lens)
        self.q, self.cu = dev(hq).view(torch.bfloat16), dev(cu)
        self.bt, self.sl = dev(w.block_table), dev(w.seq_lens)
        self.out = torch.empty((int(cu[-1]), w.Hq, w.D), dtype=torch.float32, device="cuda")
        self.max_q = n
        self.chunk_tokens = int(len(ch))
        self.flops = prefill_flops(w.seq_lens, self.q_lens, w.Hq, w.D)
        self.tb = K.token_bytes(fmt, w.D)
        self.kv_bytes = int(w.seq_lens.astype(np.int64).sum()) * w.H * self.tb
        self.app_bytes = append_bytes(self.chunk_tokens, w, self.tb)
        self.append_chunk()
        torch.cuda.synchronize()
        self.w.k = self.w.v = None

    def append_chunk(self):
        self.cache.append(0, self.k_ch, self.v_ch, self.s_ch)

    def attend(self):
        self.cache.prefill_attention(0, self.q, self.cu, self.bt, self.sl, self.max_q, out=self.out)

    def step(self):
        self.append_chunk()
        self.attend()

    run = Arm.run

    def report(self, steps: int, warmup: int, flush, peak_tflops: float, peak_kind: str):
        step_ms = float(self.run(steps, warmup, flush).mean())
        att_ms = float(self.run(steps, warmup, flush, fn=self.attend).mean())
        app_ms = float(self.run(steps, warmup, flush, fn=self.append_chunk).mean())
        w = self.w
        tflops = self.flops / (att_ms * 1e-3) / 1e12
        return {
            "workload": I.PREFILL.name,
            "step_ms": round(step_ms, 5),
            "chunk_tokens_per_s": round(self.chunk_tokens / (step_ms * 1e-3), 1),
            "attention_ms": round(att_ms, 5), "attention_TFLOPs": round(tflops, 1),
            "append_GBps": round(self.app_bytes / (app_ms * 1e-3) / 1e9, 1),
            "flops_per_launch": self.flops,
            "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": peak_tflops,
                         "unit": "TFLOP/s", "frac": round(tflops / peak_tflops, 4), "traffic": prefill_traffic(),
                         "kernel": "prefill_ws_kernel (tcgen05, warp-specialised)", "peak_source": f"{peak_kind} bf16_tflops"},
            "gpu_launches_per_step": 2,
        }


def load_tensor_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return float(json.load(open(p))["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


# ---------------------------------------------------------------- oracle arm

def oracle_sample(cfg: int, fmt: str, budget_s: float = 12.0, threads: int | None = None):
    """Time the CPU oracle (as it stands) on a bounded sample of one step of the
    workload: the step's appends plus the decode of as many (sequence, kv-head)
    jobs as fit in about `budget_s`; returns GB/s of the same algorithmic bytes."""
    from concurrent.futures import ThreadPoolExecutor
    import oracle as O
    threads = threads or min(32, os.cpu_count() or 1)
    w = I.make_workload(cfg, fmt=fmt)
    f = {v: k for k, v in O.FORMAT_NAMES.items()}[fmt]
    tb = O.token_bytes(f, w.D)
    G = w.Hq // w.H
    scale = 1.0 / np.sqrt(w.D)
    # per-job inputs prepared outside the timing: bf16 rows of each (b, h)
    jobs = [(b, h) for b in range(w.B) for h in range(w.H)]
    rng = np.random.default_rng(0)
    rng.shuffle(jobs)

    def job(bh):
        b, h = bh
        rows = slice(int(w.starts[b]), int(w.starts[b + 1]))
        kc, ks = O.quantize_rows(f, False, w.k[rows, h])
        vc, vs = O.quantize_rows(f, True, w.v[rows, h])
        kd = O.dequant_rows(f, False, kc, ks, w.D)
        vd = O.dequant_rows(f, True, vc, vs, w.D)
        q = O.bf16_bits_to_f64(w.q[b, h * G:(h + 1) * G])
        O.attend(q, kd, vd, O.is_rotated(f, False), O.is_rotated(f, True), scale)
        return int(w.seq_lens[b])

    t0 = time.perf_counter()
    done_tokens = 0
    done = 0
    with ThreadPoolExecutor(threads) as ex:
        # cycle through the step's jobs until the time budget is used (at least one pass)
        while done < len(jobs) or time.perf_counter() - t0 < budget_s:
            batch = [jobs[(done + i) % len(jobs)] for i in range(threads)]
            done_tokens += sum(ex.map(job, batch))
            done += len(batch)
    dt = time.perf_counter() - t0
    # bytes of the decode work done (the quantisation of the rows stands in for
    # the step's append of those rows and is not counted)
    nbytes = done_tokens * tb + done * G * w.D * (2 + 4)
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{done} (seq, kv-head) jobs of {I.CONFIGS[cfg].name}, {done_tokens} tokens, {dt:.1f} s"}


def cpu_baseline(cfg: int, fmt: str, budget_s: float = 12.0, single_s: float = 6.0):
    """The oracle on all host threads (up to 32) and on one thread, with the
    host's core count."""
    many = oracle_sample(cfg, fmt, budget_s=budget_s)
    one = oracle_sample(cfg, fmt, budget_s=single_s, threads=1)
    many["nproc"] = os.cpu_count()
    many["single_thread"] = {"value": one["value"], "cores": 1, "sample": one["sample"]}
    return many


# ---------------------------------------------------------------- main

def format_entry(step_gbs, peak, dec_gbs, app_gbs, tokens_s, step_ms, qerr):
    """One workload/format of the `formats` map: step GB/s (fused append +
    decode), its fraction of the peak, decode-only GB/s, bulk-append GB/s,
    tokens/s (sequences per second of the step), step ms and the quantisation
    error against fp64 attention over the bf16 inputs (max / rel. RMS)."""
    return {"step_GBps": round(step_gbs, 1), "frac": round(step_gbs / peak, 3),
            "decode_GBps": round(dec_gbs, 1), "append_GBps": round(app_gbs, 1),
            "tokens_per_s": round(tokens_s, 1), "step_ms": round(step_ms, 4),
            "qerr": [qerr["max_abs_over_max_abs_v"], qerr["rel_rms"]]}


def dist_setup(n):
    if n <= 1:
        return 0, 1, None
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(n)))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    return rank, world, dist


def max_over_ranks(x: float, dist, device="cuda") -> float:
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, dist, device="cuda") -> float:
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def whole_job_rate(units_this_rank: float, ms_this_rank: float, dist, device="cuda"):
    """Units processed by all ranks / the slowest rank's time (per second), and
    that time: each rank runs its own replica (weak scaling)."""
    ms = max_over_ranks(ms_this_rank, dist, device)
    total = sum_over_ranks(units_this_rank, dist, device)
    return total / (ms * 1e-3), ms


def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    fmt = I.CONFIGS[HEADLINE_CONFIG].formats[0]
    budget = max(2.0, 10.0 * args.steps / max(1, args.steps + args.warmup))
    vals = []
    last = None
    for _ in range(args.warmup):
        oracle_sample(HEADLINE_CONFIG, fmt, budget_s=1.0)
    for _ in range(args.steps):
        last = oracle_sample(HEADLINE_CONFIG, fmt, budget_s=budget)
        vals.append(last["value"])
    v = float(np.mean(vals))
    one = oracle_sample(HEADLINE_CONFIG, fmt, budget_s=budget, threads=1)
    spec = I.CONFIGS[HEADLINE_CONFIG]
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": spec.name, "format": fmt},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": last["cores"], "nproc": os.cpu_count(),
                             "kind": "oracle", "sample": last["sample"],
                             "single_thread": {"value": one["value"], "cores": 1, "sample": one["sample"]}},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def prefill_only(args):
    """One JSON line with the prefill object alone (rank 0, one GPU)."""
    import torch
    from quantized_paged_kv_03_b200 import build
    build.build()
    flush = make_l2_flush(torch)
    tpk, tkind = load_tensor_peak()
    clocks_path = os.path.join(tempfile.gettempdir(), f"kvq_bench_clocks_{os.getpid()}_prefill.csv")
    arm = PrefillArm()
    clk = ClockSampler(clocks_path).__enter__()
    rep = arm.report(args.steps, args.warmup, flush, tpk, tkind)
    clk.__exit__(None, None, None)
    rep["clocks"] = clk.summary(0)
    print(json.dumps({"prefill": rep}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--quick", action="store_true", help="headline workload only")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle baseline")
    ap.add_argument("--config", type=int, default=HEADLINE_CONFIG,
                    help="workload index for the headline line (profiling a single kernel)")
    ap.add_argument("--format", default=None, help="format of that workload (default: its first)")
    ap.add_argument("--batch", type=int, default=None, help="fewer sequences (small profiling case)")
    ap.add_argument("--prefill-only", action="store_true",
                    help="time the chunked-prefill workload alone (profiling the prefill kernel)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return reference_arm(args)
    if args.prefill_only:
        return prefill_only(args)

    import torch
    from quantized_paged_kv_03_b200 import build
    rank, world, dist = dist_setup(args.gpus)
    if rank == 0:
        build.build()
    if dist is not None:
        dist.barrier()
    peak, peak_kind = load_peaks()
    flush = make_l2_flush(torch)

    spec = I.CONFIGS[args.config]
    fmt = args.format or spec.formats[0]
    arm = Arm(args.config, fmt, seed_offset=rank, batch=args.batch)
    clocks_path = os.path.join(tempfile.gettempdir(), f"kvq_bench_clocks_{os.getpid()}_r{rank}.csv")
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clk = ClockSampler(clocks_path).__enter__()     # sampled over every timed section below
    t_wall = time.perf_counter()
    step_t = arm.run(args.steps, args.warmup, flush)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    t_wall = time.perf_counter() - t_wall
    dec_t = arm.run(args.steps, args.warmup, flush, fn=arm.decode_only)
    app_ms = max_over_ranks(float(arm.run(args.steps, args.warmup, flush, fn=arm.bulk_append).mean()), dist)
    step_ms = float(step_t.mean())
    step_bytes = arm.dec_bytes + arm.app_bytes
    bytes_per_s, step_ms_max = whole_job_rate(step_bytes, step_ms, dist)
    value = bytes_per_s / 1e9
    tokens, _ = whole_job_rate(arm.w.B, step_ms, dist)
    dec_ms_max = max_over_ranks(float(dec_t.mean()), dist)
    total_bytes = sum_over_ranks(step_bytes, dist)
    step_gbs = step_bytes / (step_ms_max * 1e-3) / 1e9     # the step is one launch of the fused kernel

    e2e_ts, h2d, d2h = arm.run_e2e(max(5, args.steps // 2), args.warmup, flush)
    e2e_ms = max_over_ranks(float(e2e_ts.mean()), dist)
    dec_gbs = arm.dec_bytes / (dec_ms_max * 1e-3) / 1e9

    formats = {}
    if not args.quick:
        for cfg in (0, 2, 3, 4):
            for f in I.CONFIGS[cfg].formats:
                a = Arm(cfg, f, seed_offset=rank)
                sm = max_over_ranks(float(a.run(args.steps, args.warmup, flush).mean()), dist)
                dm = max_over_ranks(float(a.run(args.steps, args.warmup, flush, fn=a.decode_only).mean()), dist)
                am = max_over_ranks(float(a.run(args.steps, args.warmup, flush, fn=a.bulk_append).mean()), dist)
                sb = a.dec_bytes + a.app_bytes
                formats[f"{I.CONFIGS[cfg].name}/{f}"] = format_entry(
                    sb / (sm * 1e-3) / 1e9, peak, a.dec_bytes / (dm * 1e-3) / 1e9,
                    a.bulk_bytes / (am * 1e-3) / 1e9, a.w.B / (sm * 1e-3), sm, a.qerr)
                del a
                torch.cuda.empty_cache()

    prefill = None
    if not args.quick:
        tpk, tkind = load_tensor_peak()
        pa = PrefillArm(seed_offset=rank)
        prefill = pa.report(args.steps, args.warmup, flush, tpk, tkind)
        if dist is not None:
            # whole job: every rank's chunk over the slowest rank's time
            att_tf, att_ms = whole_job_rate(pa.flops / 1e12, prefill["attention_ms"], dist)
            tok_s, step_ms = whole_job_rate(pa.chunk_tokens, prefill["step_ms"], dist)
            prefill.update(attention_ms=round(att_ms, 5), attention_TFLOPs=round(att_tf, 1),
                           step_ms=round(step_ms, 5), chunk_tokens_per_s=round(tok_s, 1),
                           scope=f"whole job, {world} replicas; roofline per GPU")
        del pa
        torch.cuda.empty_cache()

    clk.__exit__(None, None, None)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(args.config, fmt)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms_max, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16-mma/f32-acc", "data": "synthetic",
            "config": {"workload": spec.name, "format": fmt, "batch": arm.w.B,
                       "n_kv_heads": arm.w.H, "n_q_heads": arm.w.Hq, "head_dim": arm.w.D,
                       "page_size": arm.w.P, "kv_tokens": int(arm.w.seq_lens.sum()),
                       "step": "append 1 token/seq + decode, one fused launch",
                       "l2": "flushed before every step (256 MiB write + 256 MiB read), outside the events",
                       "parallelism": f"replicas x{world}"},
            "tokens_per_s": round(tokens, 1),
            "pct_of_peak": round(100 * value / peak, 2),
            "decode_only_GBps": round(dec_gbs, 1),
            "append_GBps": round(arm.bulk_bytes / (app_ms * 1e-3) / 1e9, 1),
            "roofline": {"bound": "hbm", "achieved": round(step_gbs, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(step_gbs / peak, 4), "traffic": headline_traffic(args.config, args.batch),
                         "kernel": "decode_kernel (fused append)", "peak_source": f"{peak_kind} hbm_gbs"},
            "e2e": {"value": round(total_bytes / (e2e_ms * 1e-3) / 1e9 if world > 1 else
                                   step_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                    "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": int(d2h)},
            "gpu_launches": args.steps,
            "clocks": clk.summary(int(os.environ.get("LOCAL_RANK", "0"))),
            "wall_s_timed_region": round(t_wall, 3),
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        if prefill is not None:
            line["prefill"] = prefill
        # last, so that a truncated tail of the line still shows every format
        line["formats"] = {f"{spec.name}/{fmt}": format_entry(step_gbs, peak, dec_gbs,
                                                              arm.bulk_bytes / (app_ms * 1e-3) / 1e9,
                                                              tokens, step_ms_max, arm.qerr), **formats}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
