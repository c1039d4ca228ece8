"""Dynamic-range parity: the decode, fused append + decode and chunked-prefill
kernels against the oracle on inputs far from unit magnitude.

Two of the formats are chosen for their range ("TokenSpeed量化实战", the
--kv-cache-dtype table: mxfp8 has the better dynamic range; "llama.cpp 引入
FP8 KV Cache", section on FP8's gains and error bounds: FP8 has the wider
range), and every format's scales are stored in a format of their own (fp16,
UE4M3, UE8M0, fp32).  The kernels feed fp16 operands to the tensor cores, so
these cases check that no step on the GPU path loses a value's range that the
stored format keeps: K and V (separately and together) scaled by 1e-3 ... 1e-5,
V near the top of the bf16 range, K scaled up with q scaled down by the same
power of two, MX group exponents near -20 and +12, and V scales that differ by
2^10 inside a page and from page to page.  The gate is the one of every
attention test: |out_gpu - out_oracle| <= 2e-3 * max|V| of the (sequence,
kv-head), per element."""
import numpy as np
import pytest
import torch

import quantized_paged_kv_03_b200 as K
from quantized_paged_kv_03_b200 import inputs as I
from kvq_testutil import (ATTN_TOL, attn_errors, bf16_dev, dev, gpu_cache, gpu_decode, oracle_cache,
                          tensor_scales, vmax_per_head)


def scaled(bits, factor):
    """bf16 values times `factor` (an array broadcast over the rows, or a number),
    rounded back to bf16."""
    return I.bf16_bits(I.bf16_to_f32(bits) * np.asarray(factor, np.float32))


# one small case per format: format, value-distribution config, D, P, H_kv, Hq
FORMATS = [
    ("fp8_row256", 0, 256, 64, 2, 8),
    ("int8_g64", 1, 256, 64, 2, 8),
    ("nvfp4_g16", 2, 256, 64, 2, 12),
    ("k8v4", 3, 256, 64, 2, 12),
    ("mxfp8_g32", 4, 128, 128, 2, 16),
    ("fp8_tensor", 4, 128, 64, 2, 16),
    ("bf16", 4, 128, 64, 2, 16),
]
FMT_IDS = [f[0] for f in FORMATS]


def workload(cfg, D, P, lengths, H, Hq, seed):
    base = I.CONFIGS[cfg]
    spec = I.ConfigSpec("t", base.formats, B=len(lengths), n_kv_heads=H, n_q_heads=Hq,
                        head_dim=D, page_size=P, lengths=("fixed", 1),
                        outlier_frac=base.outlier_frac, outlier_gain=base.outlier_gain,
                        loguniform_std=base.loguniform_std)
    return I.make_workload(spec, fmt="x", seed=seed, seq_lens=np.array(lengths))


def ranged(fmt_case, lengths, kf=1.0, vf=1.0, qf=1.0, seed=31, shape=None):
    """A workload of the format's case with K, V and q rescaled; `shape`, if
    given, edits (k, v) further (per channel or per token)."""
    fmt, cfg, D, P, H, Hq = fmt_case
    w = workload(cfg, D, P, lengths, H, Hq, seed)
    w.k, w.v, w.q = scaled(w.k, kf), scaled(w.v, vf), scaled(w.q, qf)
    if shape is not None:
        w.k, w.v = shape(w)
    return w


def caches(fmt, w):
    scales = tensor_scales(w) if fmt == "fp8_tensor" else (1.0, 1.0)
    flags = K.FLAG_NO_ROTATE if w.D != 256 else 0
    c = gpu_cache(w, fmt, flags, scales if fmt == "fp8_tensor" else None)
    oc = oracle_cache(w, fmt, flags, scales)
    return c, oc


def all_slots(w):
    return np.concatenate([w.slots(b, 0, int(w.seq_lens[b])) for b in range(w.B)])


def decode_check(fmt, w):
    c, oc = caches(fmt, w)
    s = all_slots(w)
    c.append(0, bf16_dev(w.k), bf16_dev(w.v), dev(s))
    oc.append(w.k, w.v, s)
    got = gpu_decode(c, w)
    want = oc.decode(w.q, w.block_table, w.seq_lens, threads=8)
    assert np.isfinite(got).all()
    ratio, err = attn_errors(got, want, w)
    assert ratio <= 1.0, f"{fmt}: max err {err:.3g} = {ratio:.3f} x tolerance"
    assert c.read_device_status() == 0


# ---------------------------------------------------------------- decode

@pytest.mark.gpu
@pytest.mark.parametrize("which", ["k", "v", "kv"])
@pytest.mark.parametrize("factor", [1e-3, 1e-4, 1e-5])
@pytest.mark.parametrize("case", FORMATS, ids=FMT_IDS)
def test_decode_small_values(case, factor, which):
    w = ranged(case, [300, 77], kf=factor if "k" in which else 1.0, vf=factor if "v" in which else 1.0)
    decode_check(case[0], w)


@pytest.mark.gpu
@pytest.mark.parametrize("kf,vf,qf", [(1.0, 1e4, 1.0), (1.0, 1e30, 1.0), (2.0 ** 20, 1.0, 2.0 ** -20),
                                      (1.0, 1.0, 1e-4)],
                         ids=["v_1e4", "v_1e30", "k_2^20_q_2^-20", "q_1e-4"])
@pytest.mark.parametrize("case", FORMATS, ids=FMT_IDS)
def test_decode_large_values_and_small_queries(case, kf, vf, qf):
    w = ranged(case, [300, 77], kf=kf, vf=vf, qf=qf)
    decode_check(case[0], w)


def mx_group_exponents(w):
    """Groups of 32 channels alternately scaled towards MX exponent -20 and +12
    (a group amax near 2^1.5 has exponent -7)."""
    g = np.where((np.arange(w.D) // 32) % 2 == 0, 2.0 ** -13, 2.0 ** 19).astype(np.float32)
    return scaled(w.k, g), scaled(w.v, g)


@pytest.mark.gpu
@pytest.mark.parametrize("qf", [2.0 ** -19], ids=["q_2^-19"])
def test_decode_mx_group_exponents(qf):
    w = ranged(FORMATS[4], [300, 77], qf=qf, shape=mx_group_exponents)
    decode_check("mxfp8_g32", w)


def v_groups_in_one_page(w):
    """In the second page of every sequence, V's odd scale groups (of 64
    channels, covering each format's group) are 2^10 larger than the rest."""
    v = w.v.copy()
    g = np.where((np.arange(w.D) // 64) % 2 == 1, 2.0 ** 10, 1.0).astype(np.float32)
    for b in range(w.B):
        lo, hi = int(w.starts[b]) + w.P, min(int(w.starts[b]) + 2 * w.P, int(w.starts[b + 1]))
        if hi > lo:
            v[lo:hi] = scaled(v[lo:hi], g)
    return w.k, v


def v_pages_alternate(w):
    """V of every odd page 2^10 larger than V of the even pages: the running
    reference of the decode warps (and of the prefill blocks) has to rise
    mid-sequence."""
    v = w.v.copy()
    for b in range(w.B):
        t = np.arange(int(w.seq_lens[b]))
        rows = int(w.starts[b]) + t[(t // w.P) % 2 == 1]
        v[rows] = scaled(v[rows], 2.0 ** 10)
    return w.k, v


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [v_groups_in_one_page, v_pages_alternate], ids=["groups", "pages"])
@pytest.mark.parametrize("case", FORMATS, ids=FMT_IDS)
def test_decode_v_scales_spread_by_2_10(case, shape):
    # four 5000-token sequences: more page-units than CTAs, so a CTA walks
    # several pages and a warp's reference meets larger scales after smaller ones
    w = ranged(case, [5000, 5000, 3000, 130], shape=shape, seed=37)
    decode_check(case[0], w)


# ---------------------------------------------------------------- fused append + decode

@pytest.mark.gpu
@pytest.mark.parametrize("kf,vf", [(1e-5, 1e-5), (1.0, 1e4)], ids=["kv_1e-5", "v_1e4"])
@pytest.mark.parametrize("case", [FORMATS[1], FORMATS[3], FORMATS[4], FORMATS[5]],
                         ids=["int8_g64", "k8v4", "mxfp8_g32", "fp8_tensor"])
def test_fused_step_range(case, kf, vf):
    fmt = case[0]
    w = ranged(case, [700, 129, 64], kf=kf, vf=vf, seed=41)
    c, oc = caches(fmt, w)
    kp, vp, sp = w.prefix()
    kn, vn, sn = w.new_tokens()
    c.append(0, bf16_dev(kp), bf16_dev(vp), dev(sp))
    oc.append(kp, vp, sp)
    oc.append(kn, vn, sn)
    got = c.append_decode(0, bf16_dev(kn), bf16_dev(vn), bf16_dev(w.q), dev(w.block_table),
                          dev(w.seq_lens), w.max_seq_len)
    torch.cuda.synchronize()
    got = got.cpu().numpy().astype(np.float64)
    for a, b in zip(c.read_rows(0, dev(sn)), (oc.kc[sn], oc.ks[sn], oc.vc[sn], oc.vs[sn])):
        assert np.array_equal(a.cpu().numpy(), b)
    ratio, err = attn_errors(got, oc.decode(w.q, w.block_table, w.seq_lens, threads=8), w)
    assert ratio <= 1.0, f"{fmt}: max err {err:.3g} = {ratio:.3f} x tolerance"
    assert c.read_device_status() == 0


# ---------------------------------------------------------------- chunked prefill

def prefill_check(fmt, w, q_lens):
    c, oc = caches(fmt, w)
    s = all_slots(w)
    c.append(0, bf16_dev(w.k), bf16_dev(w.v), dev(s))
    oc.append(w.k, w.v, s)
    q, cu = I.prefill_queries(w, q_lens)
    q = scaled(q, w.qf)
    out = c.prefill_attention(0, bf16_dev(q), dev(cu), dev(w.block_table), dev(w.seq_lens), int(max(q_lens)))
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    want = oc.prefill(q, cu, w.block_table, w.seq_lens)
    assert np.isfinite(got).all()
    G = w.Hq // w.H
    seq_of_row = np.repeat(np.arange(w.B), np.diff(cu))
    tol = ATTN_TOL * np.repeat(vmax_per_head(w)[seq_of_row], G, axis=1)[:, :, None]
    ratio = float((np.abs(got - want) / np.maximum(tol, 1e-30)).max())
    assert ratio <= 1.0, f"{fmt}: {ratio:.3f} x tolerance"
    assert c.read_device_status() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("kf,vf,qf", [(1e-4, 1e-4, 1.0), (1.0, 1e-5, 1.0), (1e-5, 1.0, 1.0),
                                      (1.0, 1e4, 1.0), (1.0, 1e30, 1.0), (2.0 ** 20, 1.0, 2.0 ** -20),
                                      (1.0, 1.0, 1e-4)],
                         ids=["kv_1e-4", "v_1e-5", "k_1e-5", "v_1e4", "v_1e30", "k_2^20_q_2^-20", "q_1e-4"])
@pytest.mark.parametrize("case", FORMATS, ids=FMT_IDS)
def test_prefill_range(case, kf, vf, qf):
    w = ranged(case, [300, 150], kf=kf, vf=vf, seed=43)
    w.qf = qf
    prefill_check(case[0], w, [100, 150])


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [v_groups_in_one_page, v_pages_alternate], ids=["groups", "pages"])
@pytest.mark.parametrize("case", FORMATS, ids=FMT_IDS)
def test_prefill_v_scales_spread_by_2_10(case, shape):
    w = ranged(case, [700, 260], shape=shape, seed=47)
    w.qf = 1.0
    prefill_check(case[0], w, [160, 130])


@pytest.mark.gpu
def test_prefill_mx_group_exponents():
    w = ranged(FORMATS[4], [300, 150], shape=mx_group_exponents, seed=43)
    w.qf = 2.0 ** -19
    prefill_check("mxfp8_g32", w, [100, 150])
