"""CPU oracle for the quantized paged KV cache (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
path (``quantized_paged_kv_03_b200``) never imports it, and this package never
imports the product path.

The arithmetic lives in ``kvq_oracle.c`` (plain C, fp32 where the method fixes
fp32, fp64 for attention); this module only marshals numpy arrays and adds the
paged-cache bookkeeping (slot mapping on append, block table on decode) in
plain numpy indexing.

Pages cited:
  [NInfer]     "NInfer KV Cache 量化指南：BF16、INT8、FP8、NVFP4 与 K8V4 五种格式怎么选"
               -- 64-token pages (the paging remark), asymmetric K/V
               encodings, the per-token byte table and the format paragraphs.
  [TokenSpeed] "TokenSpeed量化实战：fp8、NVFP4与KV缓存压缩如何省下50%显存"
               -- mxfp8 with ``--block-size 128``.
  [llama.cpp]  "llama.cpp 引入 FP8 KV Cache,降低本地推理显存占用"
               -- "为什么压缩 KV Cache": M_KV = 2 x B x L x H_kv x S x d_head.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

BF16, FP8_ROW256, INT8_G64, NVFP4_G16, K8V4, MXFP8_G32, FP8_TENSOR = range(7)
FORMAT_NAMES = {BF16: "bf16", FP8_ROW256: "fp8_row256", INT8_G64: "int8_g64",
                NVFP4_G16: "nvfp4_g16", K8V4: "k8v4", MXFP8_G32: "mxfp8_g32",
                FP8_TENSOR: "fp8_tensor"}
FLAG_NO_ROTATE = 1
CODE_E4M3, CODE_E2M1, CODE_INT8, CODE_FP16, CODE_UE4M3 = range(5)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-ffp-contract=off",
                               "-fno-fast-math", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, u32, f32, f64 = (ctypes.c_int, ctypes.c_int64, ctypes.c_uint32,
                                   ctypes.c_float, ctypes.c_double)
        sig = {
            "or_f32_to_f16": (ctypes.c_uint16, [f32]),
            "or_f32_to_e4m3": (ctypes.c_uint8, [f32]),
            "or_f32_to_e2m1": (ctypes.c_uint8, [f32]),
            "or_f32_to_ue4m3": (ctypes.c_uint8, [f32]),
            "or_f32_to_int8": (ctypes.c_int8, [f32]),
            "or_f16_to_f64": (f64, [ctypes.c_uint16]),
            "or_e4m3_to_f64": (f64, [ctypes.c_uint8]),
            "or_e2m1_to_f64": (f64, [ctypes.c_uint8]),
            "or_mx_exponent": (i32, [f32]),
            "or_encode": (None, [i32, P, i64, P]),
            "or_encode_bits": (None, [i32, u32, i64, P]),
            "or_fwht256": (None, [P]),
            "or_hadamard_entry": (f64, [i32, i32, i32]),
            "or_is_rotated": (i32, [i32, i32, ctypes.c_uint]),
            "or_row_bytes": (i32, [i32, i32, i32, P, P]),
            "or_quantize_rows": (i32, [i32, i32, ctypes.c_uint, f32, i32, i64, P, P, P]),
            "or_dequant_rows": (i32, [i32, i32, f32, i32, i64, P, P, P]),
            "or_attend": (i32, [i32, i64, i32, P, i32, i32, P, P, f64, P]),
            "or_mla_attend": (i32, [i32, i32, i64, i32, P, P, f64, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


# ------------------------------------------------------------------ scalars

def f32_to_f16_bits(x: float) -> int:
    return int(lib().or_f32_to_f16(float(x)))


def f32_to_e4m3(x: float) -> int:
    return int(lib().or_f32_to_e4m3(float(x)))


def f32_to_e2m1(x: float) -> int:
    return int(lib().or_f32_to_e2m1(float(x)))


def f32_to_int8(x: float) -> int:
    return int(lib().or_f32_to_int8(float(x)))


def e4m3_value(c: int) -> float:
    return float(lib().or_e4m3_to_f64(int(c)))


def e2m1_value(c: int) -> float:
    return float(lib().or_e2m1_to_f64(int(c)))


def f16_value(h: int) -> float:
    return float(lib().or_f16_to_f64(int(h)))


def mx_exponent(amax: float) -> int:
    return int(lib().or_mx_exponent(float(amax)))


def code_width(code: int) -> int:
    return 2 if code == CODE_FP16 else 1


def encode(code: int, x: np.ndarray) -> np.ndarray:
    """Element codes of fp32 values x (fp16: little-endian byte pairs)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.size * code_width(code), np.uint8)
    lib().or_encode(code, _ptr(x), x.size, _ptr(out))
    return out


def encode_bits(code: int, start: int, n: int, threads: int = 1) -> np.ndarray:
    """Codes of the fp32 bit patterns start .. start+n-1 (threads split the range)."""
    w = code_width(code)
    out = np.empty(n * w, np.uint8)
    if threads <= 1 or n < 1 << 16:
        lib().or_encode_bits(code, start & 0xFFFFFFFF, n, _ptr(out))
        return out
    step = -(-n // threads)
    base = out.ctypes.data

    def run(i):
        lo = i * step
        cnt = min(step, n - lo)
        if cnt > 0:
            lib().or_encode_bits(code, (start + lo) & 0xFFFFFFFF, cnt,
                                 ctypes.c_void_p(base + lo * w))

    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(run, range(threads)))
    return out


# ----------------------------------------------------------------- Hadamard

def fwht256(x: np.ndarray) -> np.ndarray:
    """fp32 normalised Hadamard-256 of one row, in the butterfly order the
    format fixes (ascending stages, then x 1/16)."""
    y = np.array(x, dtype=np.float32, copy=True).reshape(256)
    lib().or_fwht256(_ptr(y))
    return y


def hadamard(n: int = 256) -> np.ndarray:
    """Normalised Sylvester Hadamard matrix, fp64, from its entry definition."""
    L = lib()
    return np.array([[L.or_hadamard_entry(n, i, j) for j in range(n)] for i in range(n)])


# --------------------------------------------------------------- row codecs

def is_rotated(fmt: int, is_v: bool, flags: int = 0) -> bool:
    return bool(lib().or_is_rotated(fmt, int(is_v), flags))


def row_bytes(fmt: int, is_v: bool, D: int):
    """(code bytes, scale bytes) of one stored row, or None if invalid."""
    cb, sb = ctypes.c_int(), ctypes.c_int()
    if lib().or_row_bytes(fmt, int(is_v), D, ctypes.byref(cb), ctypes.byref(sb)) < 0:
        return None
    return cb.value, sb.value


def token_bytes(fmt: int, D: int) -> int:
    """K+V bytes per token per kv-head ([NInfer] per-token table)."""
    k, v = row_bytes(fmt, False, D), row_bytes(fmt, True, D)
    return sum(k) + sum(v)


def quantize_rows(fmt: int, is_v: bool, x_bf16: np.ndarray, flags: int = 0,
                  tensor_scale: float = 1.0):
    """Quantise rows of bf16 bit patterns [..., D] -> (codes, scales) uint8 arrays
    of shape [n, code_bytes] and [n, scale_bytes]."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    D = x.shape[-1]
    n = x.size // D
    cb, sb = row_bytes(fmt, is_v, D)
    codes = np.zeros((n, cb), np.uint8)
    scales = np.zeros((n, sb), np.uint8)
    rc = lib().or_quantize_rows(fmt, int(is_v), flags, float(tensor_scale), D, n, _ptr(x),
                                _ptr(codes), _ptr(scales))
    if rc != 0:
        raise ValueError("oracle quantize_rows: invalid format/size")
    return codes, scales


def dequant_rows(fmt: int, is_v: bool, codes: np.ndarray, scales: np.ndarray, D: int,
                 tensor_scale: float = 1.0) -> np.ndarray:
    """Stored rows -> fp64 values [n, D] in the stored (rotated) domain."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    n = codes.shape[0]
    out = np.empty((n, D), np.float64)
    rc = lib().or_dequant_rows(fmt, int(is_v), float(tensor_scale), D, n, _ptr(codes),
                               _ptr(scales), _ptr(out))
    if rc != 0:
        raise ValueError("oracle dequant_rows: invalid format/size")
    return out


def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, k_rot: bool, v_rot: bool,
           scale: float) -> np.ndarray:
    """fp64 attention of G query rows q [G, D] over L rows k, v [L, D]."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    G, D = q.shape
    L = k.shape[0]
    out = np.empty((G, D), np.float64)
    if lib().or_attend(D, L, G, _ptr(q), int(k_rot), int(v_rot), _ptr(k), _ptr(v),
                       float(scale), _ptr(out)) != 0:
        raise ValueError("oracle attend: invalid sizes")
    return out


def mla_attend(q: np.ndarray, kv: np.ndarray, DC: int, scale: float) -> np.ndarray:
    """fp64 MLA latent attention (absorbed form) of G query rows q [G, DC + DR]
    over L cached rows kv [L, DC + DR]: scores from the latent and rotary parts,
    values = the latent part.  Returns [G, DC]."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    kv = np.ascontiguousarray(kv, dtype=np.float64)
    G, W = q.shape
    L = kv.shape[0]
    if kv.shape[1] != W or not 0 < DC <= W:
        raise ValueError("oracle mla_attend: row widths differ")
    out = np.empty((G, DC), np.float64)
    if lib().or_mla_attend(DC, W - DC, L, G, _ptr(q), _ptr(kv), float(scale), _ptr(out)) != 0:
        raise ValueError("oracle mla_attend: invalid sizes")
    return out


def bf16_bits_to_f64(x: np.ndarray) -> np.ndarray:
    return (np.asarray(x, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ------------------------------------------------------------- paged cache

class PagedCache:
    """Plain paged store: for each (page, row-in-page, kv-head) the logical code
    and scale bytes of K and V.  [NInfer]: 64-token pages with independently
    encoded K and V; [TokenSpeed]: mxfp8 uses 128-token blocks."""

    def __init__(self, fmt: int, D: int, n_kv_heads: int, page_size: int, num_pages: int,
                 flags: int = 0, k_scale: float = 1.0, v_scale: float = 1.0):
        self.fmt, self.D, self.H, self.P, self.num_pages = fmt, D, n_kv_heads, page_size, num_pages
        self.flags, self.k_scale, self.v_scale = flags, k_scale, v_scale
        kcb, ksb = row_bytes(fmt, False, D)
        vcb, vsb = row_bytes(fmt, True, D)
        nslots = num_pages * page_size
        self.kc = np.zeros((nslots, n_kv_heads, kcb), np.uint8)
        self.ks = np.zeros((nslots, n_kv_heads, ksb), np.uint8)
        self.vc = np.zeros((nslots, n_kv_heads, vcb), np.uint8)
        self.vs = np.zeros((nslots, n_kv_heads, vsb), np.uint8)

    def append(self, k_bf16: np.ndarray, v_bf16: np.ndarray, slot_mapping: np.ndarray):
        """Write tokens [T, H, D] at slots; a negative slot skips the token."""
        slots = np.asarray(slot_mapping, np.int64)
        keep = slots >= 0
        if not keep.any():
            return
        kq = quantize_rows(self.fmt, False, k_bf16[keep], self.flags, self.k_scale)
        vq = quantize_rows(self.fmt, True, v_bf16[keep], self.flags, self.v_scale)
        T = int(keep.sum())
        s = slots[keep]
        self.kc[s] = kq[0].reshape(T, self.H, -1)
        self.ks[s] = kq[1].reshape(T, self.H, -1)
        self.vc[s] = vq[0].reshape(T, self.H, -1)
        self.vs[s] = vq[1].reshape(T, self.H, -1)

    def slots_of(self, block_table_row: np.ndarray, seq_len: int) -> np.ndarray:
        t = np.arange(seq_len)
        return np.asarray(block_table_row, np.int64)[t // self.P] * self.P + t % self.P

    def dequant(self, slots: np.ndarray, h: int):
        """fp64 K and V rows of kv-head h at the given slots (stored domain)."""
        k = dequant_rows(self.fmt, False, self.kc[slots, h], self.ks[slots, h], self.D, self.k_scale)
        v = dequant_rows(self.fmt, True, self.vc[slots, h], self.vs[slots, h], self.D, self.v_scale)
        return k, v

    def decode_one(self, q_bf16: np.ndarray, block_table_row: np.ndarray, seq_len: int,
                   h_kv: int, heads: list, scale: float) -> np.ndarray:
        """Attention for the given query heads (rows of q [Hq, D]) that share
        kv-head h_kv, over tokens [0, seq_len) of one sequence."""
        slots = self.slots_of(block_table_row, seq_len)
        k, v = self.dequant(slots, h_kv)
        q = bf16_bits_to_f64(q_bf16[heads])
        return attend(q, k, v, is_rotated(self.fmt, False, self.flags),
                      is_rotated(self.fmt, True, self.flags), scale)

    def decode(self, q_bf16: np.ndarray, block_table: np.ndarray, seq_lens: np.ndarray,
               scale: float | None = None, threads: int = 1) -> np.ndarray:
        """Full decode step: q [B, Hq, D] bf16 bits -> out [B, Hq, D] fp64.
        Query head h reads kv-head h // (Hq / H_kv)."""
        B, Hq, D = q_bf16.shape
        G = Hq // self.H
        scale = 1.0 / np.sqrt(D) if scale is None else scale
        out = np.zeros((B, Hq, D), np.float64)

        def run(job):
            b, h = job
            heads = list(range(h * G, (h + 1) * G))
            out[b, h * G:(h + 1) * G] = self.decode_one(q_bf16[b], block_table[b], int(seq_lens[b]),
                                                         h, heads, scale)

        jobs = [(b, h) for b in range(B) for h in range(self.H) if seq_lens[b] > 0]
        if threads <= 1:
            for j in jobs:
                run(j)
        else:
            with ThreadPoolExecutor(threads) as ex:
                list(ex.map(run, jobs))
        return out


    def prefill(self, q_bf16: np.ndarray, cu_q_lens: np.ndarray, block_table: np.ndarray,
                seq_lens: np.ndarray, scale: float | None = None, threads: int = 1) -> np.ndarray:
        """Causal attention of a chunk of query tokens per sequence over the
        cache (the multi-token form of the attention over the quantized pages,
        [NInfer] "causal_cache"), plain definition:
          q [Tq, Hq, D] bf16 bits; rows cu_q_lens[b] .. cu_q_lens[b+1]-1 are the
          n_b query tokens of sequence b, in order.  Query token i of sequence b
          sits at position pos = seq_lens[b] - n_b + i (the chunk is the last n_b
          tokens of the sequence) and attends the cached tokens [0, pos], the
          token itself included; query head h reads kv-head h // (Hq / H_kv).
          A row with pos < 0 has no keys: its output is zero.
        Returns out [Tq, Hq, D] fp64."""
        Tq, Hq, D = q_bf16.shape
        G = Hq // self.H
        cu = np.asarray(cu_q_lens, np.int64)
        B = len(cu) - 1
        scale = 1.0 / np.sqrt(D) if scale is None else scale
        out = np.zeros((Tq, Hq, D), np.float64)
        k_rot = is_rotated(self.fmt, False, self.flags)
        v_rot = is_rotated(self.fmt, True, self.flags)

        def run(job):
            b, h = job
            n, L = int(cu[b + 1] - cu[b]), int(seq_lens[b])
            k, v = self.dequant(self.slots_of(block_table[b], L), h)
            heads = slice(h * G, (h + 1) * G)
            for i in range(n):
                pos = L - n + i
                if pos < 0:
                    continue
                row = int(cu[b]) + i
                q = bf16_bits_to_f64(q_bf16[row, heads])
                out[row, heads] = attend(q, k[:pos + 1], v[:pos + 1], k_rot, v_rot, scale)

        jobs = [(b, h) for b in range(B) for h in range(self.H)
                if cu[b + 1] > cu[b] and seq_lens[b] > 0]
        if threads <= 1:
            for j in jobs:
                run(j)
        else:
            with ThreadPoolExecutor(threads) as ex:
                list(ex.map(run, jobs))
        return out


def kv_elements(B: int, L: int, H_kv: int, S: int, d_head: int) -> int:
    """[llama.cpp] M_KV = 2 x B x L x H_kv x S x d_head (elements, K and V)."""
    return 2 * B * L * H_kv * S * d_head


# ------------------------------------------------------ MLA latent cache

class MLAPagedCache:
    """Paged store of an MLA latent cache: one row of DC + DR values per token
    (latent, then rotary key), no kv-head dimension -- every query head reads
    the same row.  Stored as BF16 (the row's bits) or as FP8-E4M3 with one
    per-tensor scale over the whole row ([TokenSpeed] fp8 KV switch, used with
    its trtllm_mla backend).  Widths and the absorbed form: DeepSeek-V2 report,
    "Multi-Head Latent Attention" (DC = 512, DR = 64); pages of page_size
    tokens as in [NInfer]'s paging remark."""

    def __init__(self, fmt: int, num_pages: int, page_size: int = 64, DC: int = 512, DR: int = 64,
                 tensor_scale: float = 1.0):
        if fmt not in (BF16, FP8_TENSOR):
            raise ValueError("MLA latent cache: BF16 or FP8 per-tensor only")
        self.fmt, self.P, self.num_pages, self.DC, self.DR = fmt, page_size, num_pages, DC, DR
        self.scale = tensor_scale
        cb, _ = row_bytes(fmt, False, DC + DR)
        self.codes = np.zeros((num_pages * page_size, cb), np.uint8)

    def row_bytes(self) -> int:
        return self.codes.shape[1]

    def append(self, rows_bf16: np.ndarray, slot_mapping: np.ndarray):
        """Write latent rows [T, DC + DR] (bf16 bits) at slots; a negative slot skips."""
        slots = np.asarray(slot_mapping, np.int64)
        keep = slots >= 0
        if not keep.any():
            return
        x = np.ascontiguousarray(rows_bf16[keep], np.uint16)
        codes, _ = quantize_rows(self.fmt, False, x[:, None, :], 0, self.scale)
        self.codes[slots[keep]] = codes.reshape(len(x), -1)

    def dequant(self, slots: np.ndarray) -> np.ndarray:
        empty = np.zeros((len(slots), 0), np.uint8)
        return dequant_rows(self.fmt, False, np.ascontiguousarray(self.codes[slots]), empty,
                            self.DC + self.DR, self.scale)

    def decode(self, q_bf16: np.ndarray, block_table: np.ndarray, seq_lens: np.ndarray,
               scale: float) -> np.ndarray:
        """q [B, Hq, DC + DR] bf16 bits (absorbed latent query, then rotary
        query) -> latent outputs [B, Hq, DC] fp64; a zero-length sequence
        gives zero rows.  `scale` is the model's softmax scale (for the
        DeepSeek-V2 shape 1/sqrt(128 + 64), the width of a head's un-absorbed
        query), not 1/sqrt(DC + DR)."""
        B, Hq, W = q_bf16.shape
        if W != self.DC + self.DR:
            raise ValueError("MLA decode: query width differs from the cache rows")
        out = np.zeros((B, Hq, self.DC), np.float64)
        for b in range(B):
            n = int(seq_lens[b])
            if n <= 0:
                continue
            t = np.arange(n)
            slots = np.asarray(block_table[b], np.int64)[t // self.P] * self.P + t % self.P
            out[b] = mla_attend(bf16_bits_to_f64(q_bf16[b]), self.dequant(slots), self.DC, scale)
        return out
