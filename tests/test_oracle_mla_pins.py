"""Pins for the oracle's MLA latent-cache decode (the absorbed form over one
shared row of latent + rotary-key values per token).  Each check ties it to
something outside the oracle: the fp8 memory figure of the TokenSpeed page,
torch's scaled-dot-product attention over the expanded per-head keys and
values that the latent stands for (the DeepSeek-V2 definition), and closed-form
special cases.  A dropped rotary term, a wrong value slice, a wrong scale or a
wrong slot fails one of them.  CPU only."""
import json
import os

import numpy as np
import pytest
import torch

import oracle as O
from quantized_paged_kv_03_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
DC, DR, D_NOPE, D_V = 512, 64, 128, 128     # DeepSeek-V2 report, MLA section
SCALE = 1.0 / np.sqrt(D_NOPE + DR)


def fp8_cache(w, scale=None):
    amax = float(np.abs(I.bf16_to_f32(w.rows)).max())
    c = O.MLAPagedCache(O.FP8_TENSOR, w.num_pages, w.P, DC, DR, scale or amax / 448.0)
    c.append(w.rows, w.slots())
    return c


def test_fp8_latent_row_is_half_of_bf16_as_the_page_prints():
    g = json.load(open(os.path.join(GOLDEN, "kv_cache_dtype_memory.json")))["memory_relative_to_bf16"]
    bf = O.MLAPagedCache(O.BF16, 1, 64, DC, DR).row_bytes()
    f8 = O.MLAPagedCache(O.FP8_TENSOR, 1, 64, DC, DR).row_bytes()
    assert bf == 2 * (DC + DR) == 1152 and f8 == DC + DR == 576
    assert f8 / bf == g["fp8/fp8_e4m3"]


@pytest.mark.parametrize("fmt", [O.BF16, O.FP8_TENSOR])
def test_one_token_returns_its_latent(fmt):
    w = I.make_mla_workload([1, 1], Hq=3, seed=21)
    c = O.MLAPagedCache(fmt, w.num_pages, w.P, DC, DR, 0.05)
    c.append(w.rows, w.slots())
    out = c.decode(w.q, w.block_table, w.seq_lens, SCALE)
    for b in range(w.B):
        lat = c.dequant(w.slots()[b:b + 1])[0, :DC]
        assert np.array_equal(out[b], np.broadcast_to(lat, (w.Hq, DC)))


def test_absorbed_latent_attention_equals_expanded_attention():
    """The latent decode, mapped back through W_UV, equals standard attention of
    each head over its own keys [W_UK c_t, r_t] and values W_UV c_t (torch SDPA
    in fp64), with the query's latent part q_lat = W_UK^T q_nope."""
    w = I.make_mla_workload([77], Hq=4, seed=22)
    c = fp8_cache(w)
    kv = c.dequant(w.slots())                                  # [L, DC + DR]
    r = np.random.default_rng(5)
    W_UK = r.standard_normal((w.Hq, D_NOPE, DC)) / np.sqrt(DC)
    W_UV = r.standard_normal((w.Hq, D_V, DC)) / np.sqrt(DC)
    q_nope = r.standard_normal((w.Hq, D_NOPE)) * 3.0
    q_rope = r.standard_normal((w.Hq, DR)) * 3.0
    q_lat = np.einsum("hnc,hn->hc", W_UK, q_nope)
    o_lat = O.mla_attend(np.concatenate([q_lat, q_rope], 1), kv, DC, SCALE)
    got = np.einsum("hvc,hc->hv", W_UV, o_lat)

    lat, rope = torch.from_numpy(kv[:, :DC]), torch.from_numpy(kv[:, DC:])
    for h in range(w.Hq):
        K = torch.cat([lat @ torch.from_numpy(W_UK[h]).T, rope], 1)        # [L, 192]
        V = lat @ torch.from_numpy(W_UV[h]).T                             # [L, 128]
        Q = torch.from_numpy(np.concatenate([q_nope[h], q_rope[h]]))[None]
        want = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None], scale=SCALE)[0, 0]
        vmax = float(V.abs().max())
        assert np.abs(got[h] - want.numpy()).max() <= 1e-12 * vmax, h
    # the rotary part matters here: without it the outputs move well beyond rounding
    o_nr = O.mla_attend(np.concatenate([q_lat, 0 * q_rope], 1), kv, DC, SCALE)
    assert np.abs(o_nr - o_lat).max() > 1e-3


def test_without_rotary_part_it_is_one_head_attention_with_k_equal_v():
    w = I.make_mla_workload([130], Hq=2, seed=23)
    c = fp8_cache(w)
    kv = c.dequant(w.slots())
    q = I.bf16_to_f32(w.q[0]).astype(np.float64)
    q[:, DC:] = 0.0
    got = O.mla_attend(q, kv, DC, SCALE)
    want = O.attend(q[:, :DC], kv[:, :DC], kv[:, :DC], False, False, SCALE)
    assert np.abs(got - want).max() <= 1e-12 * np.abs(kv[:, :DC]).max()


def test_equal_latents_give_that_latent_whatever_the_scores():
    # a convex combination of equal rows is the row: catches values taken from
    # the wrong columns (the rotary part) or weights that do not sum to one
    r = np.random.default_rng(7)
    row = r.standard_normal(DC)
    kv = np.concatenate([np.tile(row, (40, 1)), r.standard_normal((40, DR)) * 4], 1)
    q = r.standard_normal((5, DC + DR))
    got = O.mla_attend(q, kv, DC, 0.3)
    assert np.abs(got - row).max() <= 1e-13 * np.abs(row).max()


def test_paged_store_equals_contiguous_rows():
    w = I.make_mla_workload([300, 1, 64, 65], Hq=3, seed=24)
    c = fp8_cache(w)
    out = c.decode(w.q, w.block_table, w.seq_lens, SCALE)
    kv_all = O.dequant_rows(O.FP8_TENSOR, False, O.quantize_rows(
        O.FP8_TENSOR, False, w.rows[:, None, :], 0, c.scale)[0], np.zeros((len(w.rows), 0), np.uint8),
        DC + DR, c.scale)
    for b in range(w.B):
        rows = kv_all[w.starts[b]:w.starts[b + 1]]
        want = O.mla_attend(I.bf16_to_f32(w.q[b]).astype(np.float64), rows, DC, SCALE)
        assert np.array_equal(out[b], want), b
    assert len(set(w.block_table[w.block_table >= 0].tolist())) == int((w.block_table >= 0).sum())


def test_empty_sequence_gives_zero_rows():
    w = I.make_mla_workload([0, 5], Hq=2, seed=25)
    c = fp8_cache(w)
    out = c.decode(w.q, w.block_table, w.seq_lens, SCALE)
    assert not out[0].any() and out[1].any()
