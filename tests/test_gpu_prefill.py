"""Chunked-prefill attention parity: the CUDA kernel against the oracle's
fp64 causal attention over the oracle's own cache, within 2e-3 * max|V| per
element, for every format, page sizes that give every key-tile size (16, 32,
64 tokens; whole-page and split-page copies), GQA groups that do not divide
the 128-row query block, several query blocks per sequence, chunks longer
than the cached sequence (zero rows), empty chunks, bf16 output and a grid
sized below the longest chunk."""
import numpy as np
import pytest
import torch

import quantized_paged_kv_03_b200 as K
from quantized_paged_kv_03_b200 import inputs as I
from kvq_testutil import (ATTN_TOL, append_all, bf16_dev, dev, gpu_cache, oracle_cache,
                          tensor_scales, vmax_per_head)


def workload(cfg, D, P, lengths, H, Hq, seed=21):
    base = I.CONFIGS[cfg]
    spec = I.ConfigSpec("t", base.formats, B=len(lengths), n_kv_heads=H, n_q_heads=Hq,
                        head_dim=D, page_size=P, lengths=("fixed", 1),
                        outlier_frac=base.outlier_frac, outlier_gain=base.outlier_gain,
                        loguniform_std=base.loguniform_std)
    return I.make_workload(spec, fmt="x", seed=seed, seq_lens=np.array(lengths))


def build_case(fmt, cfg, D, P, lengths, H, Hq, seed=21):
    w = workload(cfg, D, P, lengths, H, Hq, seed)
    scales = tensor_scales(w) if fmt == "fp8_tensor" else (1.0, 1.0)
    flags = K.FLAG_NO_ROTATE if D != 256 else 0   # the Hadamard is 256-point
    c = gpu_cache(w, fmt, flags, scales if fmt == "fp8_tensor" else None)
    oc = oracle_cache(w, fmt, flags, scales)
    append_all(c, oc, w)
    return w, c, oc


def gpu_prefill(c, w, q, cu, max_q_len=None, out_fp32=True, scale=0.0, block_table=None, seq_lens=None):
    bt = w.block_table if block_table is None else block_table
    sl = w.seq_lens if seq_lens is None else seq_lens
    out = c.prefill_attention(0, bf16_dev(q), dev(cu.astype(np.int32)), dev(bt.astype(np.int32)),
                              dev(sl.astype(np.int32)), max_q_len, out_fp32=out_fp32,
                              softmax_scale=scale)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64)


def check(got, want, w, cu):
    """max error over all elements, in units of 2e-3 * max|V| of the row's
    (sequence, kv-head)."""
    G = w.Hq // w.H
    vm = vmax_per_head(w)                                   # [B, H]
    seq_of_row = np.repeat(np.arange(w.B), np.diff(cu))
    tol = ATTN_TOL * np.repeat(vm[seq_of_row], G, axis=1)[:, :, None]
    ratio = np.abs(got - want) / np.maximum(tol, 1e-30)
    return float(ratio.max()) if ratio.size else 0.0


CASES = [
    # format, value-distribution config, D, P, seq_lens, chunk lengths, H_kv, Hq
    ("int8_g64", 1, 256, 64, [700, 300, 64, 5], [200, 300, 1, 8], 2, 8),
    ("nvfp4_g16", 2, 256, 64, [500, 130], [130, 129], 2, 12),
    ("k8v4", 3, 256, 64, [400], [150], 1, 6),
    ("fp8_row256", 0, 256, 16, [90, 33], [40, 33], 2, 4),
    ("mxfp8_g32", 4, 128, 128, [600, 129], [100, 129], 2, 16),
    ("fp8_tensor", 4, 128, 32, [300, 70], [64, 70], 2, 8),
    ("bf16", 4, 128, 64, [260, 17], [100, 17], 2, 16),
    ("bf16", 0, 256, 64, [200], [200], 1, 3),
    ("int8_g64", 1, 128, 48, [250], [120], 1, 4),
    ("nvfp4_g16", 2, 256, 256, [600], [300], 1, 6),
    ("nvfp4_g16", 2, 128, 64, [333, 65], [90, 65], 2, 6),
    ("mxfp8_g32", 4, 256, 64, [180], [77], 1, 2),
    ("fp8_tensor", 4, 256, 64, [150], [150], 1, 1),
    ("int8_g64", 1, 256, 128, [1000, 1], [512, 1], 2, 8),   # 16 query blocks in one sequence
]


@pytest.mark.gpu
@pytest.mark.parametrize("fmt,cfg,D,P,lengths,q_lens,H,Hq", CASES)
def test_prefill_matches_oracle(fmt, cfg, D, P, lengths, q_lens, H, Hq):
    w, c, oc = build_case(fmt, cfg, D, P, lengths, H, Hq)
    q, cu = I.prefill_queries(w, q_lens)
    got = gpu_prefill(c, w, q, cu)
    want = oc.prefill(q, cu, w.block_table, w.seq_lens, threads=8)
    ratio = check(got, want, w, cu)
    assert ratio <= 1.0, f"{fmt}: max err = {ratio:.3f} x tolerance"
    # rows before the first cached token (chunk longer than the sequence) are zero
    for b, (L, n) in enumerate(zip(lengths, q_lens)):
        if n > L:
            assert not got[cu[b]:cu[b] + n - L].any()
    assert c.read_device_status() == 0


@pytest.mark.gpu
def test_prefill_grid_below_the_longest_chunk_and_bf16_output():
    # max_q_len = 64 sizes the grid for 2 query blocks per (sequence, kv-head);
    # the 400-token chunk (12.5 blocks at G = 4) is still computed in full.
    w, c, oc = build_case("int8_g64", 1, 256, 64, [900, 70], 2, 8)
    q, cu = I.prefill_queries(w, [400, 0])
    want = oc.prefill(q, cu, w.block_table, w.seq_lens, threads=8)
    got = gpu_prefill(c, w, q, cu, max_q_len=64)
    assert check(got, want, w, cu) <= 1.0
    full = gpu_prefill(c, w, q, cu)
    assert np.array_equal(got, full)        # same rows, same arithmetic, any grid
    ob = gpu_prefill(c, w, q, cu, out_fp32=False)
    assert np.abs(ob - got).max() <= 2 ** -8 * np.abs(got).max()
    assert c.read_device_status() == 0


@pytest.mark.gpu
def test_prefill_custom_scale_and_empty_sequences():
    # attend over shorter prefixes of the cached sequences: none for sequence 0
    # (and no chunk), 2 tokens for a 3-token chunk in sequence 2
    w, c, oc = build_case("fp8_row256", 0, 256, 64, [150, 150, 150], 1, 2)
    sl = np.array([0, 150, 2], np.int32)
    q, cu = I.prefill_queries(w, [0, 60, 3])
    want = oc.prefill(q, cu, w.block_table, sl, scale=0.2)
    got = gpu_prefill(c, w, q, cu, scale=0.2, seq_lens=sl)
    assert check(got, want, w, cu) <= 1.0
    assert not got[cu[2]].any()
    assert got[cu[2] + 1:].any()
    assert c.read_device_status() == 0


@pytest.mark.gpu
def test_prefill_bad_page_id_is_recorded():
    w, c, oc = build_case("int8_g64", 1, 256, 64, [200], 1, 4)
    q, cu = I.prefill_queries(w, [20])
    bt = w.block_table.copy()
    bt[0, 1] = w.num_pages + 5
    gpu_prefill(c, w, q, cu, block_table=bt)
    assert c.read_device_status(clear=True) & K.STATUS_BAD_PAGE
    assert c.read_device_status() == 0


@pytest.mark.gpu
def test_prefill_full_size_workload_sampled_rows():
    """The benchmark's chunked-prefill workload in the launch configuration the
    benchmark times (4 x 8192 cached tokens, 512-token chunks, the grid sized by
    max_q_len = 512): sampled query rows against the oracle, row by row."""
    import oracle as O
    spec, n = I.PREFILL, I.PREFILL_CHUNK
    w = I.make_workload(spec, seed=I.PREFILL_SEED)
    c = gpu_cache(w, "int8_g64")
    oc = oracle_cache(w, "int8_g64")
    append_all(c, oc, w)
    q, cu = I.prefill_queries(w, np.full(w.B, n))
    got = gpu_prefill(c, w, q, cu, max_q_len=n)
    G = w.Hq // w.H
    f = K.FORMATS["int8_g64"]
    worst = 0.0
    for b in (0, w.B - 1):
        L = int(w.seq_lens[b])
        for h in (0, w.H - 1):
            k, v = oc.dequant(oc.slots_of(w.block_table[b], L), h)
            vmax = np.abs(I.bf16_to_f32(w.v[w.starts[b]:w.starts[b + 1], h])).max()
            for i in (0, 1, n // 2, n - 1):
                pos = L - n + i
                row = int(cu[b]) + i
                qr = O.bf16_bits_to_f64(q[row, h * G:(h + 1) * G])
                want = O.attend(qr, k[:pos + 1], v[:pos + 1], O.is_rotated(f, False), O.is_rotated(f, True),
                                1.0 / np.sqrt(w.D))
                err = np.abs(got[row, h * G:(h + 1) * G] - want).max() / (ATTN_TOL * vmax)
                worst = max(worst, err)
    assert worst <= 1.0, worst
    assert c.read_device_status() == 0
