"""Append parity: the codes and scale bytes the CUDA append kernel stores must
equal the oracle's bit for bit, for every format, on seeded inputs shaped like
the workloads (outlier channels, log-uniform channel std), over several pages
with ragged tails, plus the skip / out-of-range slot rules and exact round
trips of grid-valued rows."""
import numpy as np
import pytest
import torch

import oracle as O
import quantized_paged_kv_03_b200 as K
from quantized_paged_kv_03_b200 import inputs as I
from kvq_testutil import (all_slots, append_all, bf16_dev, dev, gpu_cache, oracle_cache,
                          tensor_scales)

CASES = [
    # (format, config index for the value distribution, head_dim, page_size, lengths)
    ("fp8_row256", 0, 256, 64, [256, 3]),
    ("int8_g64", 1, 256, 64, [1, 77, 200]),
    ("nvfp4_g16", 2, 256, 64, [130, 64]),
    ("k8v4", 3, 256, 64, [191, 5]),
    ("mxfp8_g32", 4, 128, 128, [300, 1]),
    ("fp8_tensor", 4, 128, 64, [129, 64]),
    ("bf16", 4, 128, 64, [100, 33]),
    ("bf16", 0, 256, 64, [70]),
    ("int8_g64", 4, 128, 64, [70, 9]),        # unrotated-capable D=128 needs NO_ROTATE
    ("nvfp4_g16", 0, 256, 32, [45]),
    ("mxfp8_g32", 1, 256, 64, [80]),
    ("fp8_tensor", 1, 256, 64, [80]),
]


def workload(cfg, D, P, lengths, seed=7, H=2, Hq=4):
    base = I.CONFIGS[cfg]
    spec = I.ConfigSpec("t", base.formats, B=len(lengths), n_kv_heads=H, n_q_heads=Hq,
                        head_dim=D, page_size=P, lengths=("fixed", 1),
                        outlier_frac=base.outlier_frac, outlier_gain=base.outlier_gain,
                        loguniform_std=base.loguniform_std)
    return I.make_workload(spec, fmt="x", seed=seed, seq_lens=np.array(lengths))


@pytest.mark.gpu
@pytest.mark.parametrize("fmt,cfg,D,P,lengths", CASES)
def test_append_codes_bit_exact(fmt, cfg, D, P, lengths):
    flags = K.FLAG_NO_ROTATE if (D != 256 and fmt in ("int8_g64", "nvfp4_g16", "k8v4")) else 0
    w = workload(cfg, D, P, lengths)
    scales = tensor_scales(w) if fmt == "fp8_tensor" else (1.0, 1.0)
    c = gpu_cache(w, fmt, flags, scales if fmt == "fp8_tensor" else None)
    oc = oracle_cache(w, fmt, flags, scales)
    append_all(c, oc, w)
    slots = all_slots(w)
    kc, ks, vc, vs = [t.cpu().numpy() for t in c.read_rows(0, dev(slots))]
    assert np.array_equal(kc, oc.kc[slots]), "K codes"
    assert np.array_equal(ks, oc.ks[slots]), "K scales"
    assert np.array_equal(vc, oc.vc[slots]), "V codes"
    assert np.array_equal(vs, oc.vs[slots]), "V scales"
    # stored values: code x scale (exact in fp32 except an fp32 per-tensor scale)
    kd, vd = [t.cpu().numpy().astype(np.float64) for t in c.dequant(0, dev(slots))]
    for h in range(w.H):
        ok, ov = oc.dequant(slots, h)
        if fmt == "fp8_tensor":
            assert np.allclose(kd[:, h], ok, rtol=2 ** -23, atol=0)
            assert np.allclose(vd[:, h], ov, rtol=2 ** -23, atol=0)
        else:
            assert np.array_equal(kd[:, h], ok)
            assert np.array_equal(vd[:, h], ov)


@pytest.mark.gpu
def test_append_skips_negative_and_flags_out_of_range_slots():
    w = workload(1, 256, 64, [64], H=1, Hq=1)
    c = gpu_cache(w, "int8_g64")
    k, v = bf16_dev(w.k), bf16_dev(w.v)
    slots = w.slots(0, 0, 64).copy()
    c.append(0, k, v, dev(slots))
    before = [t.cpu().numpy() for t in c.read_rows(0, dev(slots))]
    bad = slots.copy()
    bad[:10] = -1
    bad[10] = w.num_pages * w.P + 5          # out of range: skipped and recorded
    k2 = bf16_dev(w.k[::-1].copy())
    c.append(0, k2, k2, dev(bad))
    assert c.read_device_status(clear=True) & K.STATUS_BAD_SLOT
    assert c.read_device_status() == 0
    after = [t.cpu().numpy() for t in c.read_rows(0, dev(slots))]
    for a, b in zip(before, after):
        assert np.array_equal(a[:11], b[:11])          # skipped rows untouched
        assert not np.array_equal(a[11:], b[11:])      # the others rewritten


@pytest.mark.gpu
def test_grid_valued_rows_round_trip_exactly():
    """Rows whose values are code x scale with the group amax on the top code
    come back unchanged through append + dequant (rotation off)."""
    r = np.random.default_rng(3)
    e4 = np.array([(1 + m / 8) * 2.0 ** (e - 7) for e in range(1, 16) for m in range(8)
                   if not (e == 15 and m == 7)])
    D, P = 256, 64
    rows = []
    for t in range(P):
        c = r.choice(np.concatenate([e4, -e4]), size=D)
        c[t % D] = 448.0
        rows.append(c * 2.0 ** r.integers(-6, 3))
    x = np.array(rows, np.float32)[:, None, :]
    bits = I.bf16_bits(x)
    assert np.array_equal(I.bf16_to_f32(bits), x)
    c = K.KVCache("fp8_row256", D, 1, P, 2, flags=K.FLAG_NO_ROTATE)
    slots = np.arange(P, 2 * P, dtype=np.int64)
    c.append(0, bf16_dev(bits), bf16_dev(bits), dev(slots))
    kd, vd = c.dequant(0, dev(slots))
    assert np.array_equal(kd.cpu().numpy()[:, 0], x[:, 0])
    assert np.array_equal(vd.cpu().numpy()[:, 0], x[:, 0])


@pytest.mark.gpu
def test_zero_rows_and_tiny_rows():
    """All-zero rows store zero codes and scales; rows whose scale underflows
    fp16 store +0 codes (both sides follow the same rule)."""
    D, P = 256, 64
    x = np.zeros((4, 1, D), np.float32)
    x[1, 0, :] = 1e-30
    x[2, 0, 5] = -3e-38
    x[3, 0, :] = np.linspace(-1e4, 1e4, D)
    bits = I.bf16_bits(x)
    slots = np.arange(4, dtype=np.int64)
    for fmt in ("fp8_row256", "int8_g64", "nvfp4_g16", "k8v4", "mxfp8_g32"):
        c = K.KVCache(fmt, D, 1, P, 1)
        c.append(0, bf16_dev(bits), bf16_dev(bits), dev(slots))
        oc = O.PagedCache(K.FORMATS[fmt], D, 1, P, 1)
        oc.append(bits, bits, slots)
        got = [t.cpu().numpy() for t in c.read_rows(0, dev(slots))]
        for g, want in zip(got, (oc.kc, oc.ks, oc.vc, oc.vs)):
            assert np.array_equal(g, want[slots]), fmt
