"""Seeded synthetic inputs for the KV-cache append, decode and chunked-prefill paths.

This module draws random numbers and shapes them; it holds none of the
method's arithmetic (no rotation, no scales, no codes).  Tests feed the same
arrays to the CUDA library and to the CPU oracle; the benchmark feeds them to
the library.

Recipe (stand-ins for the workloads the pages describe; the pages publish no
dataset for this path):
  * values: numpy ``Generator(PCG64)`` standard normals in fp32, multiplied by
    a per-channel factor, rounded to bf16 (round to nearest even);
  * outlier channels: per kv-head, exactly round(p * D) channels chosen without
    replacement, the same channels in K and V, scaled by the factor;
  * log-uniform channel std: per (kv-head, channel), drawn separately for K and V;
  * sequence lengths: uniform integers, or a clipped lognormal;
  * block tables: each sequence's pages are a slice of one random permutation
    of the page pool, so consecutive pages are not adjacent in memory;
  * the last token of every sequence is the step's new token (appended during
    the step, then attended to); the others are the prefix;
  * chunked prefill: the last n tokens of a sequence are the chunk, its query
    rows N(0, 1) bf16 like the decode queries (``prefill_queries``).
Every stream is a child of ``SeedSequence([seed, stream_id, ...])`` so results do
not depend on the thread count.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

FORMATS = {"bf16": 0, "fp8_row256": 1, "int8_g64": 2, "nvfp4_g16": 3, "k8v4": 4,
           "mxfp8_g32": 5, "fp8_tensor": 6}


@dataclass(frozen=True)
class ConfigSpec:
    name: str
    formats: tuple
    B: int
    n_kv_heads: int
    n_q_heads: int
    head_dim: int
    page_size: int
    lengths: tuple            # ("fixed", L) | ("uniform", lo, hi) | ("lognormal", median, sigma, lo, hi)
    outlier_frac: float = 0.0
    outlier_gain: float = 1.0
    loguniform_std: tuple = ()  # (lo, hi) per-channel std, K and V drawn separately
    page_size_by_format: dict = field(default_factory=dict)


# The five workloads (sizes, value distributions and formats as specified for
# this path).  Index 0 is the small case; index 1 is the headline decode case.
CONFIGS = [
    ConfigSpec("fp8_row256_tiny", ("fp8_row256",), B=1, n_kv_heads=1, n_q_heads=1,
               head_dim=256, page_size=64, lengths=("fixed", 256)),
    ConfigSpec("int8_g64_b8_u1k8k", ("int8_g64",), B=8, n_kv_heads=8, n_q_heads=32,
               head_dim=256, page_size=64, lengths=("uniform", 1024, 8192),
               outlier_frac=0.02, outlier_gain=20.0),
    ConfigSpec("nvfp4_g16_b32_32k", ("nvfp4_g16",), B=32, n_kv_heads=4, n_q_heads=24,
               head_dim=256, page_size=64, lengths=("fixed", 32768),
               outlier_frac=0.01, outlier_gain=16.0),
    ConfigSpec("k8v4_b1_256k", ("k8v4",), B=1, n_kv_heads=4, n_q_heads=24,
               head_dim=256, page_size=64, lengths=("fixed", 262144),
               loguniform_std=(0.1, 10.0)),
    ConfigSpec("mxfp8_fp8t_bf16_b256_lognormal", ("mxfp8_g32", "fp8_tensor", "bf16"), B=256,
               n_kv_heads=8, n_q_heads=64, head_dim=128, page_size=64,
               lengths=("lognormal", 4096, 1.0, 512, 16384),
               outlier_frac=0.02, outlier_gain=20.0,
               page_size_by_format={"mxfp8_g32": 128}),
]

SEED_BASE = 20261200

# Chunked-prefill workload: the shape and value recipe of the INT8-G64 decode
# workload above (8 kv-heads, 32 query heads, head_dim 256, 64-token pages, 2 %
# of channels x20), with 4 sequences of 8192 cached tokens whose last
# PREFILL_CHUNK tokens are the chunk being prefilled.
PREFILL = ConfigSpec("int8_g64_prefill_b4_8k_chunk512", ("int8_g64",), B=4, n_kv_heads=8, n_q_heads=32,
                     head_dim=256, page_size=64, lengths=("fixed", 8192),
                     outlier_frac=0.02, outlier_gain=20.0)
PREFILL_CHUNK = 512
PREFILL_SEED = SEED_BASE + 500


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (r >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(seed: int, *stream) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *stream])))


def seq_lengths(spec: ConfigSpec, seed: int, B: int | None = None) -> np.ndarray:
    B = spec.B if B is None else B
    r = _rng(seed, 1)
    kind = spec.lengths[0]
    if kind == "fixed":
        L = np.full(B, spec.lengths[1], np.int64)
    elif kind == "uniform":
        L = r.integers(spec.lengths[1], spec.lengths[2], endpoint=True, size=B)
    elif kind == "lognormal":
        med, sigma, lo, hi = spec.lengths[1:]
        L = np.clip(np.rint(np.exp(np.log(med) + sigma * r.standard_normal(B))), lo, hi)
    else:
        raise ValueError(kind)
    return L.astype(np.int32)


def channel_gains(spec: ConfigSpec, seed: int, H: int, D: int):
    """Per-(kv-head, channel) multipliers for K and V, fp32 [H, D] each."""
    gk = np.ones((H, D), np.float32)
    gv = np.ones((H, D), np.float32)
    r = _rng(seed, 2)
    if spec.outlier_frac > 0:
        n = int(round(spec.outlier_frac * D))
        for h in range(H):
            ch = r.choice(D, size=n, replace=False)
            gk[h, ch] = spec.outlier_gain
            gv[h, ch] = spec.outlier_gain
    if spec.loguniform_std:
        lo, hi = spec.loguniform_std
        gk = np.exp(r.uniform(np.log(lo), np.log(hi), size=(H, D))).astype(np.float32)
        gv = np.exp(r.uniform(np.log(lo), np.log(hi), size=(H, D))).astype(np.float32)
    return gk, gv


@dataclass
class Workload:
    spec: ConfigSpec
    fmt: str
    seed: int
    B: int
    H: int            # kv heads
    Hq: int
    D: int
    P: int
    seq_lens: np.ndarray      # int32 [B], lengths after the step's append
    block_table: np.ndarray   # int32 [B, max_pages]; unused entries are -1
    num_pages: int
    k: np.ndarray             # uint16 bf16 bits [sum(seq_lens), H, D], sequence-major
    v: np.ndarray
    q: np.ndarray             # uint16 bf16 bits [B, Hq, D]
    starts: np.ndarray        # int64 [B+1] row offsets of each sequence in k / v

    @property
    def max_pages(self) -> int:
        return self.block_table.shape[1]

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max()) if self.B else 0

    def slots(self, b: int, t0: int, t1: int) -> np.ndarray:
        t = np.arange(t0, t1)
        return self.block_table[b][t // self.P].astype(np.int64) * self.P + t % self.P

    def prefix(self):
        """(k, v, slot_mapping) of every token except each sequence's last."""
        rows, slots = [], []
        for b in range(self.B):
            L = int(self.seq_lens[b])
            if L > 1:
                rows.append(np.arange(self.starts[b], self.starts[b] + L - 1))
                slots.append(self.slots(b, 0, L - 1))
        if not rows:
            e = np.zeros((0, self.H, self.D), np.uint16)
            return e, e.copy(), np.zeros(0, np.int64)
        idx = np.concatenate(rows)
        return self.k[idx], self.v[idx], np.concatenate(slots)

    def new_tokens(self):
        """(k, v, slot_mapping) of each sequence's last token: the step's append."""
        last = self.starts[1:] - 1
        slots = np.array([self.slots(b, int(self.seq_lens[b]) - 1, int(self.seq_lens[b]))[0]
                          for b in range(self.B)], np.int64)
        return self.k[last], self.v[last], slots


_CHUNK_ROWS = 4096


def _fill_normals(out: np.ndarray, seed: int, stream: tuple, gain: np.ndarray):
    """out[...] = bf16(gain * N(0,1)) for a block of rows [n, H, D]."""
    x = _rng(seed, *stream).standard_normal(out.shape, dtype=np.float32)
    x *= gain
    out[...] = bf16_bits(x)


def make_workload(cfg: int | ConfigSpec, fmt: str | None = None, seed: int | None = None,
                  B: int | None = None, seq_lens: np.ndarray | None = None,
                  threads: int | None = None, page_slack: int = 0) -> Workload:
    """Build the seeded workload of a config (optionally with fewer sequences or
    other lengths, for tests that need a smaller case of the same shape)."""
    spec = CONFIGS[cfg] if isinstance(cfg, int) else cfg
    cfg_index = CONFIGS.index(spec) if spec in CONFIGS else 99
    fmt = spec.formats[0] if fmt is None else fmt
    seed = SEED_BASE + cfg_index if seed is None else seed
    if seq_lens is None:
        seq_lens = seq_lengths(spec, seed, B)
    seq_lens = np.asarray(seq_lens, np.int32)
    B = len(seq_lens)
    H, Hq, D = spec.n_kv_heads, spec.n_q_heads, spec.head_dim
    P = spec.page_size_by_format.get(fmt, spec.page_size)

    pages = [(int(L) + P - 1) // P for L in seq_lens]
    num_pages = sum(pages) + page_slack
    perm = _rng(seed, 3).permutation(num_pages).astype(np.int32)
    max_pages = max(pages) if pages else 1
    bt = np.full((B, max(1, max_pages)), -1, np.int32)
    o = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[o:o + n]
        o += n

    starts = np.zeros(B + 1, np.int64)
    starts[1:] = np.cumsum(seq_lens)
    T = int(starts[-1])
    k = np.empty((T, H, D), np.uint16)
    v = np.empty((T, H, D), np.uint16)
    gk, gv = channel_gains(spec, seed, H, D)
    # one independent stream per (sequence, K|V, block of _CHUNK_ROWS rows)
    jobs = [(b, which, c) for b in range(B) for which in (0, 1)
            for c in range(0, int(seq_lens[b]), _CHUNK_ROWS)]

    def run(job):
        b, which, c = job
        lo = starts[b] + c
        hi = min(starts[b + 1], lo + _CHUNK_ROWS)
        dst = (k if which == 0 else v)[lo:hi]
        _fill_normals(dst, seed, (4, b, which, c), gk if which == 0 else gv)

    threads = threads or min(32, os.cpu_count() or 1)
    if threads > 1 and T * H * D > (1 << 22):
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(run, jobs))
    else:
        for j in jobs:
            run(j)
    q = bf16_bits(_rng(seed, 5).standard_normal((B, Hq, D), dtype=np.float32))
    return Workload(spec, fmt, seed, B, H, Hq, D, P, seq_lens, bt, num_pages, k, v, q, starts)


def prefill_queries(w: Workload, q_lens, seed: int | None = None):
    """Query rows of a prefill chunk: q_lens[b] tokens of sequence b (its last
    q_lens[b] tokens when q_lens[b] <= seq_lens[b]).  Returns (q, cu_q_lens):
    bf16 bits [sum(q_lens), Hq, D], N(0, 1) like the decode queries, and the
    int32 row offsets [B + 1] of each sequence's rows."""
    q_lens = np.asarray(q_lens, np.int64)
    cu = np.zeros(len(q_lens) + 1, np.int32)
    cu[1:] = np.cumsum(q_lens)
    r = _rng(w.seed if seed is None else seed, 6)
    q = bf16_bits(r.standard_normal((int(cu[-1]), w.Hq, w.D), dtype=np.float32))
    return q, cu


@dataclass
class MLAWorkload:
    """An MLA latent-cache decode case: one cached row of DC + DR values per
    token (no kv-head dimension), Hq query rows per sequence."""
    seed: int
    B: int
    Hq: int
    DC: int
    DR: int
    P: int
    seq_lens: np.ndarray      # int32 [B]
    block_table: np.ndarray   # int32 [B, max_pages], -1 past each sequence
    num_pages: int
    rows: np.ndarray          # bf16 bits [T, DC + DR], sequences back to back
    q: np.ndarray             # bf16 bits [B, Hq, DC + DR]
    starts: np.ndarray        # int64 [B + 1] first row of each sequence

    def slots(self) -> np.ndarray:
        """Cache slot of every row (page of the block table x P + offset)."""
        out = np.empty(int(self.starts[-1]), np.int64)
        for b in range(self.B):
            t = np.arange(int(self.seq_lens[b]))
            out[self.starts[b]:self.starts[b + 1]] = self.block_table[b, t // self.P].astype(np.int64) * self.P + t % self.P
        return out


def make_mla_workload(seq_lens, Hq: int, seed: int, DC: int = 512, DR: int = 64, P: int = 64,
                      outlier_frac: float = 0.02, outlier_gain: float = 20.0) -> MLAWorkload:
    """Seeded MLA latent rows and queries: standard normals rounded to bf16,
    with round(outlier_frac * (DC + DR)) outlier channels scaled by
    outlier_gain (the same channels for every token); the queries N(0, 1).
    Block tables as in make_workload: slices of one random page permutation."""
    seq_lens = np.asarray(seq_lens, np.int32)
    B, W = len(seq_lens), DC + DR
    pages = [(int(L) + P - 1) // P for L in seq_lens]
    num_pages = max(1, sum(pages))
    perm = _rng(seed, 3).permutation(num_pages).astype(np.int32)
    bt = np.full((B, max(1, max(pages) if pages else 1)), -1, np.int32)
    o = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[o:o + n]
        o += n
    starts = np.zeros(B + 1, np.int64)
    starts[1:] = np.cumsum(seq_lens)
    gain = np.ones(W, np.float32)
    n_out = int(round(outlier_frac * W))
    if n_out:
        gain[_rng(seed, 7).choice(W, n_out, replace=False)] = outlier_gain
    x = _rng(seed, 8).standard_normal((int(starts[-1]), W), dtype=np.float32) * gain
    q = _rng(seed, 9).standard_normal((B, Hq, W), dtype=np.float32)
    return MLAWorkload(seed, B, Hq, DC, DR, P, seq_lens, bt, num_pages, bf16_bits(x), bf16_bits(q), starts)


def tensor_amax(x_bf16: np.ndarray) -> float:
    """Largest magnitude of a bf16 tensor (input statistic for a static scale)."""
    if x_bf16.size == 0:
        return 0.0
    return float(np.abs(bf16_to_f32(x_bf16)).max())
