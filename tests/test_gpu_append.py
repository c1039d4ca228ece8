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


@pytest.mark.gpu
@pytest.mark.parametrize("D", [256, 128])
def test_int8_codes_on_rounding_ties(D):
    """INT8 rows whose quotients value / scale land exactly on half-integers
    (each 64-group's amax is 127 x 2^j, so its fp16 scale is 2^j, and the other
    values are (k + 1/2) x 2^j): the codes must equal the oracle's, which
    rounds the correctly rounded quotient half to even."""
    r = np.random.default_rng(11)
    P, n = 64, 48
    rows = []
    for t in range(n):
        j = int(r.integers(-20, 12))
        k = r.integers(0, 127, size=D).astype(np.float64)
        x = (k + 0.5) * r.choice([-1.0, 1.0], size=D)
        x[(np.arange(D) % 64) == (t % 64)] = 127.0          # one amax per group
        rows.append(x * 2.0 ** j)
    x = np.array(rows, np.float32)[:, None, :]
    bits = I.bf16_bits(x)
    assert np.array_equal(I.bf16_to_f32(bits), x)             # every value is a bf16 value
    slots = np.arange(n, dtype=np.int64) + P
    c = K.KVCache("int8_g64", D, 1, P, 2, flags=K.FLAG_NO_ROTATE)
    c.append(0, bf16_dev(bits), bf16_dev(bits), dev(slots))
    oc = O.PagedCache(K.FORMATS["int8_g64"], D, 1, P, 2, flags=K.FLAG_NO_ROTATE)
    oc.append(bits, bits, slots)
    got = [t.cpu().numpy() for t in c.read_rows(0, dev(slots))]
    for g, want in zip(got, (oc.kc, oc.ks, oc.vc, oc.vs)):
        assert np.array_equal(g, want[slots])
    codes = oc.kc[slots].view(np.int8).astype(np.int64)
    assert (np.abs(codes) % 2 == 0).sum() > 0.4 * codes.size   # ties went to even codes


def e4m3_midpoints():
    """Every rounding boundary of E4M3 up to 448, subnormal range included:
    midpoints of consecutive grid values, as float64."""
    g = [j * 2.0 ** -9 for j in range(8)]                                  # subnormals
    g += [(1 + m / 8) * 2.0 ** e for e in range(-6, 9) for m in range(8)]  # normals
    g = np.array(sorted(v for v in g if v <= 448.0))
    return (g[1:] + g[:-1]) / 2


E2M1_MIDPOINTS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", ["nvfp4_g16", "fp8_row256", "fp8_tensor", "k8v4"])
def test_codes_on_grid_rounding_boundaries(fmt):
    """Rows whose quotients value / scale land exactly on the encoder's rounding
    boundaries (midpoints of the E2M1 or E4M3 grid, E4M3's subnormal range
    included), or one bf16 step beside them: every code must equal the
    oracle's, which rounds the correctly rounded quotient to nearest even.
    Rotation is off so that the quotients are the constructed ones."""
    r = np.random.default_rng(17)
    D, P, n = 256, 64, 40
    mids = {"fp8_row256": e4m3_midpoints(), "fp8_tensor": e4m3_midpoints(), "nvfp4_g16": E2M1_MIDPOINTS}
    top = {"fp8_row256": 448.0, "fp8_tensor": 448.0, "nvfp4_g16": 6.0}
    group = {"fp8_row256": 256, "fp8_tensor": 256, "nvfp4_g16": 16}

    def rows(kind, pow2):
        out = []
        for t in range(n):
            j = pow2[t]
            m = r.choice(mids[kind], size=D)
            m = m * r.choice([-1.0, 1.0], size=D)
            beside = r.random(D) < 0.3                           # one bf16 step off the boundary
            m = np.where(beside, m * (1 + r.choice([-1.0, 1.0], size=D) * 2.0 ** -7), m)
            m[(np.arange(D) % group[kind]) == (t % group[kind])] = top[kind]   # each group's amax
            out.append(m * 2.0 ** j)
        x = np.array(out, np.float32)[:, None, :]
        bits = I.bf16_bits(x)
        return bits

    if fmt == "k8v4":
        kb = rows("fp8_row256", r.integers(-12, 8, size=n))
        vb = rows("nvfp4_g16", r.integers(-9, 8, size=n))
        scales = None
    elif fmt == "fp8_tensor":
        kb = rows(fmt, np.zeros(n, int))
        vb = rows(fmt, np.full(n, -3))
        scales = (1.0, 0.125)          # the tensor scales put the quotients on the boundaries
    else:
        lo, hi = (-9, 8) if fmt == "nvfp4_g16" else (-12, 8)
        kb = rows(fmt, r.integers(lo, hi, size=n))
        vb = rows(fmt, r.integers(lo, hi, size=n))
        scales = None
    slots = np.arange(n, dtype=np.int64) + P
    c = K.KVCache(fmt, D, 1, P, 2, 1, K.FLAG_NO_ROTATE, [scales] if scales else None)
    c.append(0, bf16_dev(kb), bf16_dev(vb), dev(slots))
    sk, sv = scales if scales else (1.0, 1.0)
    oc = O.PagedCache(K.FORMATS[fmt], D, 1, P, 2, K.FLAG_NO_ROTATE, sk, sv)
    oc.append(kb, vb, slots)
    got = [t.cpu().numpy() for t in c.read_rows(0, dev(slots))]
    for g, want, name in zip(got, (oc.kc, oc.ks, oc.vc, oc.vs), ("K codes", "K scales", "V codes", "V scales")):
        assert np.array_equal(g, want[slots]), name
