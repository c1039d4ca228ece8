"""Helpers shared by the GPU parity tests: feed one seeded workload to the
CUDA library and to the CPU oracle, and compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
import quantized_paged_kv_03_b200 as K
from quantized_paged_kv_03_b200 import build
from quantized_paged_kv_03_b200 import inputs as I

# Attention tolerance: |out_gpu - out_oracle| <= 2e-3 * max|V| per element,
# max|V| over the (sequence, kv-head)'s bf16 V rows.
ATTN_TOL = 2e-3

_built = False


def ensure_built():
    global _built
    if not _built:
        build.build()
        _built = True


def dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    return dev(bits.astype(np.uint16)).view(torch.bfloat16)


def tensor_scales(w: I.Workload):
    """Per-tensor fp8 scales from the inputs' amax (static calibration)."""
    return (I.tensor_amax(w.k) / 448.0 or 1.0, I.tensor_amax(w.v) / 448.0 or 1.0)


def gpu_cache(w: I.Workload, fmt: str, flags: int = 0, scales=None, extra_pages: int = 0):
    ensure_built()
    ts = [scales] if scales is not None else None
    return K.KVCache(fmt, w.D, w.H, w.P, w.num_pages + extra_pages, 1, flags, ts)


def oracle_cache(w: I.Workload, fmt: str, flags: int = 0, scales=(1.0, 1.0)):
    return O.PagedCache(K.FORMATS[fmt], w.D, w.H, w.P, w.num_pages, flags, scales[0], scales[1])


def append_all(c: K.KVCache, oc, w: I.Workload):
    """Append the prefix, then the step's new tokens, to both caches."""
    kp, vp, sp = w.prefix()
    kn, vn, sn = w.new_tokens()
    for k, v, s in ((kp, vp, sp), (kn, vn, sn)):
        if len(s):
            c.append(0, bf16_dev(k), bf16_dev(v), dev(s))
            if oc is not None:
                oc.append(k, v, s)


def all_slots(w: I.Workload) -> np.ndarray:
    return np.concatenate([w.slots(b, 0, int(w.seq_lens[b])) for b in range(w.B)])


def gpu_decode(c: K.KVCache, w: I.Workload, out_fp32=True, scale=0.0, seq_lens=None, block_table=None):
    sl = w.seq_lens if seq_lens is None else seq_lens
    bt = w.block_table if block_table is None else block_table
    out = c.decode_attention(0, bf16_dev(w.q), dev(bt.astype(np.int32)), dev(sl.astype(np.int32)),
                             int(max(1, sl.max())), out_fp32=out_fp32, softmax_scale=scale)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64)


def vmax_per_head(w: I.Workload) -> np.ndarray:
    """max |V| over each (sequence, kv-head): [B, H]."""
    m = np.zeros((w.B, w.H))
    vf = np.abs(I.bf16_to_f32(w.v))
    for b in range(w.B):
        if w.seq_lens[b] > 0:
            m[b] = vf[w.starts[b]:w.starts[b + 1]].max(axis=(0, 2))
    return m


def attn_errors(got: np.ndarray, want: np.ndarray, w: I.Workload):
    """(max error / (tol * max|V|) over all elements, max abs error)."""
    G = w.Hq // w.H
    vm = np.repeat(vmax_per_head(w), G, axis=1)[:, :, None]
    err = np.abs(got - want)
    ratio = err / (ATTN_TOL * np.maximum(vm, 1e-30))
    return float(ratio.max()), float(err.max())
