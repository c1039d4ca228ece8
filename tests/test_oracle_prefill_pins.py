"""Pins for the oracle's chunked-prefill attention (``PagedCache.prefill``):
each check ties it to something outside the oracle -- torch's scaled-dot-product
attention with its lower-right causal mask (the convention for a query chunk
that ends the key sequence), scipy's Hadamard matrix, brute-force perturbation
of single cached tokens -- so that an off-by-one in the positions, a dropped
diagonal, a wrong kv-head for a query head, a row taken from the wrong sequence
or a missing rotation fails here.  CPU only."""
import numpy as np
import scipy.linalg
import torch
import torch.nn.functional as F
from torch.nn.attention.bias import causal_lower_right

import oracle as O
from quantized_paged_kv_03_b200 import inputs as I


def small_workload(fmt, D, P, lengths, H, Hq, seed=3, outlier=0.0):
    spec = I.ConfigSpec("pin", (fmt,), B=len(lengths), n_kv_heads=H, n_q_heads=Hq, head_dim=D,
                        page_size=P, lengths=("fixed", 1), outlier_frac=outlier, outlier_gain=8.0)
    return I.make_workload(spec, fmt=fmt, seed=seed, seq_lens=np.array(lengths))


def filled_cache(w, fmt_id, flags=0):
    oc = O.PagedCache(fmt_id, w.D, w.H, w.P, w.num_pages, flags)
    for b in range(w.B):
        L = int(w.seq_lens[b])
        rows = slice(int(w.starts[b]), int(w.starts[b]) + L)
        oc.append(w.k[rows], w.v[rows], w.slots(b, 0, L))
    return oc


def sdpa(q, k, v, G, mask=None, causal=False, scale=None):
    """torch fp64 attention: q [n, Hq, D], k, v [L, H, D] -> [n, Hq, D]."""
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(k).permute(1, 0, 2)[None].repeat_interleave(G, dim=1)
    vt = torch.from_numpy(v).permute(1, 0, 2)[None].repeat_interleave(G, dim=1)
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, is_causal=causal, scale=scale)
    return o[0].permute(1, 0, 2).numpy()


def bf16_f64(bits):
    return I.bf16_to_f32(bits).astype(np.float64)


def test_prefill_matches_sdpa_with_lower_right_causal_mask():
    # BF16 stores K bit for bit and V as fp16 (numpy's float16 cast is the same
    # nearest-even rounding), so the attention is torch's over those values.
    lengths, q_lens = [37, 50, 1, 16], [37, 12, 1, 5]
    w = small_workload("bf16", 128, 16, lengths, H=2, Hq=6)
    oc = filled_cache(w, O.BF16)
    q, cu = I.prefill_queries(w, q_lens)
    got = oc.prefill(q, cu, w.block_table, w.seq_lens)
    for b, (L, n) in enumerate(zip(lengths, q_lens)):
        rows = slice(int(w.starts[b]), int(w.starts[b]) + L)
        k = bf16_f64(w.k[rows])
        v = I.bf16_to_f32(w.v[rows]).astype(np.float16).astype(np.float64)
        want = sdpa(bf16_f64(q[cu[b]:cu[b + 1]]), k, v, G=3, mask=causal_lower_right(n, L))
        np.testing.assert_allclose(got[cu[b]:cu[b + 1]], want, rtol=1e-10, atol=1e-12)


def test_prefill_of_a_whole_prompt_is_standard_causal_attention():
    L = 70
    w = small_workload("bf16", 128, 64, [L], H=1, Hq=2)
    oc = filled_cache(w, O.BF16)
    q, cu = I.prefill_queries(w, [L])
    got = oc.prefill(q, cu, w.block_table, w.seq_lens, scale=0.3)
    k = bf16_f64(w.k)
    v = I.bf16_to_f32(w.v).astype(np.float16).astype(np.float64)
    want = sdpa(bf16_f64(q), k, v, G=2, causal=True, scale=0.3)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def test_prefill_of_rotated_formats_is_attention_over_rotated_back_rows():
    # NVFP4-G16 rotates K and V by the normalised Hadamard-256; scipy's Sylvester
    # matrix / 16 rotates the stored rows back, and torch does the attention.
    lengths, q_lens = [90, 33], [20, 33]
    w = small_workload("nvfp4_g16", 256, 32, lengths, H=2, Hq=4, outlier=0.02)
    oc = filled_cache(w, O.NVFP4_G16)
    q, cu = I.prefill_queries(w, q_lens)
    got = oc.prefill(q, cu, w.block_table, w.seq_lens)
    Hm = scipy.linalg.hadamard(256).astype(np.float64) / 16.0
    for b, (L, n) in enumerate(zip(lengths, q_lens)):
        slots = oc.slots_of(w.block_table[b], L)
        kv = [oc.dequant(slots, h) for h in range(w.H)]
        k = np.stack([kd @ Hm for kd, _ in kv], axis=1)
        v = np.stack([vd @ Hm for _, vd in kv], axis=1)
        want = sdpa(bf16_f64(q[cu[b]:cu[b + 1]]), k, v, G=2, mask=causal_lower_right(n, L))
        np.testing.assert_allclose(got[cu[b]:cu[b + 1]], want, rtol=1e-9, atol=1e-11)


def test_one_token_chunks_equal_decode():
    lengths = [300, 1, 65]
    w = small_workload("int8_g64", 256, 64, lengths, H=2, Hq=8, outlier=0.02)
    oc = filled_cache(w, O.INT8_G64)
    q, cu = I.prefill_queries(w, [1, 1, 1])
    got = oc.prefill(q, cu, w.block_table, w.seq_lens)
    want = oc.decode(q, w.block_table, w.seq_lens)
    np.testing.assert_array_equal(got, want)


def test_each_row_sees_exactly_its_prefix():
    # Overwrite the cached K/V of one token at position p: rows whose position is
    # below p keep their bits, rows at or after p change.
    L, n, p = 40, 10, 35
    w = small_workload("fp8_row256", 256, 16, [L], H=1, Hq=2)
    oc = filled_cache(w, O.FP8_ROW256)
    q, cu = I.prefill_queries(w, [n])
    before = oc.prefill(q, cu, w.block_table, w.seq_lens)
    other = small_workload("fp8_row256", 256, 16, [1], H=1, Hq=2, seed=99)
    oc.append(other.k, other.v, w.slots(0, p, p + 1))
    after = oc.prefill(q, cu, w.block_table, w.seq_lens)
    pos = L - n + np.arange(n)
    for i in range(n):
        if pos[i] < p:
            np.testing.assert_array_equal(after[i], before[i])
        else:
            assert np.abs(after[i] - before[i]).max() > 1e-6, i


def test_rows_before_the_first_cached_token_are_zero():
    # A chunk longer than the cached sequence: its first n - L rows would sit
    # before position 0 and attend nothing; the rest equal the chunk of length L.
    L, n = 5, 8
    w = small_workload("int8_g64", 256, 16, [L], H=1, Hq=3)
    oc = filled_cache(w, O.INT8_G64)
    q, cu = I.prefill_queries(w, [n])
    got = oc.prefill(q, cu, w.block_table, w.seq_lens)
    assert not got[:n - L].any()
    tail = oc.prefill(np.ascontiguousarray(q[n - L:]), np.array([0, L], np.int32),
                      w.block_table, w.seq_lens)
    np.testing.assert_array_equal(got[n - L:], tail)
