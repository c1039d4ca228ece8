"""Decode-attention parity: the CUDA split-K paged GQA kernel against the
oracle's fp64 attention over the oracle's own cache, within
2e-3 * max|V| per element, for every format, over ragged multi-page
sequences, GQA groups 1..12, head_dim 128/256, several CTA splits per
sequence, bf16 output, empty sequences and bad page ids."""
import numpy as np
import pytest
import torch

import quantized_paged_kv_03_b200 as K
from quantized_paged_kv_03_b200 import inputs as I
from kvq_testutil import (append_all, attn_errors, bf16_dev, dev, gpu_cache, gpu_decode,
                          oracle_cache, tensor_scales, vmax_per_head)


def workload(cfg, D, P, lengths, H, Hq, seed=11):
    base = I.CONFIGS[cfg]
    spec = I.ConfigSpec("t", base.formats, B=len(lengths), n_kv_heads=H, n_q_heads=Hq,
                        head_dim=D, page_size=P, lengths=("fixed", 1),
                        outlier_frac=base.outlier_frac, outlier_gain=base.outlier_gain,
                        loguniform_std=base.loguniform_std)
    return I.make_workload(spec, fmt="x", seed=seed, seq_lens=np.array(lengths))


CASES = [
    # format, value-distribution config, D, P, lengths, H_kv, Hq
    ("fp8_row256", 0, 256, 64, [256], 1, 1),
    ("fp8_row256", 0, 256, 64, [1, 17, 64, 65, 300], 2, 8),
    ("int8_g64", 1, 256, 64, [1100, 63, 1, 700], 2, 8),
    ("nvfp4_g16", 2, 256, 64, [900, 333], 2, 12),
    ("k8v4", 3, 256, 64, [2000], 2, 12),
    ("mxfp8_g32", 4, 128, 128, [600, 129, 1], 2, 16),
    ("fp8_tensor", 4, 128, 64, [512, 77], 2, 16),
    ("bf16", 4, 128, 64, [300, 2], 2, 16),
    ("bf16", 0, 256, 64, [200], 1, 3),
    ("int8_g64", 1, 256, 64, [5000], 1, 24),     # G = 24: three 8-head blocks
    ("nvfp4_g16", 2, 128, 64, [700, 65, 3], 2, 6),   # 4-bit code words span two q lanes
    ("int8_g64", 1, 128, 64, [400, 64], 2, 4),
    # pages staged in 64-token units (128 and 256 tokens) and whole small pages
    ("int8_g64", 1, 256, 128, [300, 129, 64, 1], 2, 8),
    ("nvfp4_g16", 2, 256, 256, [700, 255, 1], 1, 6),
    ("fp8_tensor", 4, 128, 32, [100, 33, 1], 2, 8),
    ("k8v4", 3, 256, 128, [500, 130], 1, 6),
]


def run_case(fmt, cfg, D, P, lengths, H, Hq, out_fp32=True, seed=11):
    w = workload(cfg, D, P, lengths, H, Hq, seed)
    scales = tensor_scales(w) if fmt == "fp8_tensor" else (1.0, 1.0)
    flags = K.FLAG_NO_ROTATE if D != 256 else 0   # the Hadamard is 256-point
    c = gpu_cache(w, fmt, flags, scales if fmt == "fp8_tensor" else None)
    oc = oracle_cache(w, fmt, flags, scales)
    append_all(c, oc, w)
    got = gpu_decode(c, w, out_fp32=out_fp32)
    want = oc.decode(w.q, w.block_table, w.seq_lens, threads=8)
    return w, c, got, want


@pytest.mark.gpu
@pytest.mark.parametrize("fmt,cfg,D,P,lengths,H,Hq", CASES)
def test_decode_matches_oracle(fmt, cfg, D, P, lengths, H, Hq):
    w, c, got, want = run_case(fmt, cfg, D, P, lengths, H, Hq)
    ratio, err = attn_errors(got, want, w)
    assert ratio <= 1.0, f"{fmt}: max err {err:.3g} = {ratio:.3f} x tolerance"
    assert c.read_device_status() == 0


@pytest.mark.gpu
def test_decode_bf16_output_and_repeat_calls_are_identical():
    w, c, got, want = run_case("int8_g64", 1, 256, 64, [3000, 5], 2, 8)
    # second and third calls reuse the (self-resetting) workspace
    again = gpu_decode(c, w)
    assert np.array_equal(got, again)
    ob = gpu_decode(c, w, out_fp32=False)
    assert np.abs(ob - got).max() <= 2 ** -8 * np.abs(got).max()


@pytest.mark.gpu
def test_decode_single_token_returns_stored_v():
    """seq_len = 1: softmax weight 1, so out = the stored V row (un-rotated)."""
    w, c, got, want = run_case("fp8_row256", 0, 256, 64, [1, 1], 1, 4)
    ratio, _ = attn_errors(got, want, w)
    assert ratio <= 0.1


@pytest.mark.gpu
def test_decode_empty_sequence_gives_zero_rows():
    w = workload(1, 256, 64, [130, 0, 64], 2, 8)
    c = gpu_cache(w, "int8_g64")
    oc = oracle_cache(w, "int8_g64")
    slots = np.concatenate([w.slots(b, 0, int(w.seq_lens[b])) for b in range(w.B)])
    c.append(0, bf16_dev(w.k), bf16_dev(w.v), dev(slots))
    oc.append(w.k, w.v, slots)
    got = gpu_decode(c, w)
    assert not got[1].any()
    want = oc.decode(w.q, w.block_table, w.seq_lens)
    vm = np.repeat(vmax_per_head(w), 4, axis=1)[:, :, None]
    for b in (0, 2):
        assert (np.abs(got[b] - want[b]) <= 2e-3 * vm[b]).all()


@pytest.mark.gpu
def test_decode_flags_bad_page_ids_without_faulting():
    w = workload(1, 256, 64, [200], 1, 4)
    c = gpu_cache(w, "int8_g64")
    append_all(c, None, w)
    bt = w.block_table.copy()
    bt[0, 1] = w.num_pages + 100            # out of range: replaced by page 0 and recorded
    gpu_decode(c, w, block_table=bt)
    assert c.read_device_status(clear=True) & K.STATUS_BAD_PAGE


@pytest.mark.gpu
def test_decode_many_sequences_balanced_split():
    """Lognormal lengths over a batch of 64: ranges of page-heads cross
    sequence boundaries in every CTA."""
    spec = I.CONFIGS[4]
    lens = I.seq_lengths(spec, 5, 64) // 8
    w = workload(4, 128, 128, list(lens), 2, 16, seed=5)
    c = gpu_cache(w, "mxfp8_g32")
    oc = oracle_cache(w, "mxfp8_g32")
    append_all(c, oc, w)
    got = gpu_decode(c, w)
    want = oc.decode(w.q, w.block_table, w.seq_lens, threads=8)
    ratio, err = attn_errors(got, want, w)
    assert ratio <= 1.0, err


@pytest.mark.gpu
@pytest.mark.parametrize("fmt,cfg,D,P,lengths,H,Hq", [
    ("int8_g64", 1, 256, 64, [1, 64, 65, 700, 1100], 2, 8),
    ("nvfp4_g16", 2, 256, 64, [333, 900], 2, 12),
    ("k8v4", 3, 256, 64, [2000, 129], 2, 12),
    ("mxfp8_g32", 4, 128, 128, [600, 128, 1], 2, 16),
    ("fp8_tensor", 4, 128, 64, [512, 77], 2, 16),
    ("bf16", 4, 128, 64, [300, 2], 2, 16),
    ("int8_g64", 1, 256, 256, [700, 193, 64], 1, 8),
    # one 330 000-token sequence on one kv-head: every CTA's range holds about
    # 17 of the segment's units, so the new token is quantised when its unit
    # arrives rather than at the segment start (the INT8 kernel's other path)
    pytest.param("int8_g64", 1, 256, 64, [330000], 1, 4, id="int8_g64-long_ranges")])
def test_fused_append_decode_equals_append_then_decode(fmt, cfg, D, P, lengths, H, Hq):
    """kvq_append_decode stores the same codes as kvq_append and returns the
    same output as kvq_decode_attention run after it."""
    w = workload(cfg, D, P, lengths, H, Hq, seed=13)
    scales = tensor_scales(w) if fmt == "fp8_tensor" else (1.0, 1.0)
    sc = scales if fmt == "fp8_tensor" else None
    kp, vp, sp = w.prefix()
    kn, vn, sn = w.new_tokens()
    ref = gpu_cache(w, fmt, 0, sc)
    fused = gpu_cache(w, fmt, 0, sc)
    for c in (ref, fused):
        c.append(0, bf16_dev(kp), bf16_dev(vp), dev(sp))
    ref.append(0, bf16_dev(kn), bf16_dev(vn), dev(sn))
    want = gpu_decode(ref, w)
    q, bt, sl = bf16_dev(w.q), dev(w.block_table), dev(w.seq_lens)
    got = fused.append_decode(0, bf16_dev(kn), bf16_dev(vn), q, bt, sl, w.max_seq_len)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy().astype(np.float64), want)
    for a, b in zip(ref.read_rows(0, dev(sn)), fused.read_rows(0, dev(sn))):
        assert torch.equal(a, b)
    # and against the oracle
    oc = oracle_cache(w, fmt, 0, scales)
    oc.append(kp, vp, sp)
    oc.append(kn, vn, sn)
    ratio, err = attn_errors(got.cpu().numpy().astype(np.float64),
                             oc.decode(w.q, w.block_table, w.seq_lens, threads=8), w)
    assert ratio <= 1.0, err
    assert fused.read_device_status() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("fmt,cfg,H,lengths", [("k8v4", 3, 1, [24000]), ("int8_g64", 1, 1, [12000, 9000])],
                         ids=["one_segment_296_parts", "two_segments"])
def test_decode_segment_cut_into_many_groups(fmt, cfg, H, lengths):
    """A single long sequence on one kv-head is cut across every CTA of the
    grid (hundreds of parts): its parts are merged in groups of 16 and the
    groups merged again, by whichever CTAs finish last.  The result must match
    the oracle and be bit-identical on a repeat call (a fixed merge order,
    counters left at zero)."""
    w, c, got, want = run_case(fmt, cfg, 256, 64, lengths, H, 6)
    ratio, err = attn_errors(got, want, w)
    assert ratio <= 1.0, f"{fmt}: max err {err:.3g} = {ratio:.3f} x tolerance"
    again = gpu_decode(c, w)
    assert np.array_equal(got, again)
    assert c.read_device_status() == 0
