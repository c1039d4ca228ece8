"""Pins for the CPU oracle: each check ties an oracle function to something
outside itself (the pages' byte table, closed forms, brute force over a format's
grid, textbook library routines), so that a dropped term, a wrong sign, index
or operand order in the oracle fails here.  CPU only."""
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.special
import torch

import oracle as O
from quantized_paged_kv_03_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
NAMES = {"bf16": O.BF16, "int8_g64": O.INT8_G64, "fp8_row256": O.FP8_ROW256,
         "nvfp4_g16": O.NVFP4_G16, "k8v4": O.K8V4, "mxfp8_g32": O.MXFP8_G32,
         "fp8_tensor": O.FP8_TENSOR}


# ------------------------------------------------------------ byte table

def test_token_bytes_match_the_pages_table():
    g = json.load(open(os.path.join(GOLDEN, "token_bytes.json")))
    D = g["head_dim"]
    for name, want in g["bytes_per_token"].items():
        assert O.token_bytes(NAMES[name], D) == want, name
    # "≈51% / ≈50% / ≈28% / ≈39%" of BF16 (the table truncates: 528/1024 = 51.6%)
    for name, pct in (("int8_g64", 51), ("fp8_row256", 50), ("nvfp4_g16", 28), ("k8v4", 39)):
        assert math.floor(100 * O.token_bytes(NAMES[name], D) / 1024) == pct
    # the NVFP4 paragraph's capacity figure (about 3.5x): context at fixed memory grows by 1024 / 288
    r = O.token_bytes(O.BF16, D) / O.token_bytes(O.NVFP4_G16, D)
    assert 3.4 < r < 3.6


def test_token_bytes_of_the_d128_formats_follow_their_definitions():
    # [TokenSpeed]: mxfp8 = fp8 codes + one UE8M0 byte per 32 head_dim values;
    # [FP8-KV] per-tensor fp8 = codes only; BF16 = 2 bytes per value.
    D = 128
    assert O.token_bytes(O.MXFP8_G32, D) == 2 * (D + D // 32) == 264
    assert O.token_bytes(O.FP8_TENSOR, D) == 2 * D == 256
    assert O.token_bytes(O.BF16, D) == 4 * D == 512
    # "0.5x of BF16" ignoring scale bytes
    assert 2 * D / (4 * D) == 0.5


def test_kv_size_formula_matches_bf16_bytes():
    # [llama.cpp] M_KV = 2 B L H_kv S d_head elements; BF16 stores 2 bytes each.
    B, L, H, S, d = 3, 2, 4, 100, 256
    elems = O.kv_elements(B, L, H, S, d)
    assert elems * 2 == O.token_bytes(O.BF16, d) * B * L * H * S


# ------------------------------------------------------------ grids

def e4m3_grid():
    """All finite non-negative E4M3 values with their codes, from the format
    definition (bias 7, 3 mantissa bits, S.1111.111 is NaN)."""
    vals, codes = [], []
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            v = (m / 8) * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
            vals.append(v)
            codes.append((e << 3) | m)
    return np.array(vals), np.array(codes)


def e2m1_grid():
    vals = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    return vals, np.arange(8)


def brute_nearest(x, vals, codes, sign_bit):
    """Nearest grid value, ties to the even code, saturating; sign kept."""
    a = np.abs(x.astype(np.float64))[:, None]
    d = np.abs(a - vals[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = (d == best)
    # among tied candidates prefer an even code
    even = cand & ((codes[None, :] & 1) == 0)
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    c = codes[pick]
    c = np.where(a[:, 0] > vals.max(), codes[vals.argmax()], c)
    neg = np.signbit(x)
    return (c | np.where(neg, sign_bit, 0)).astype(np.uint8)


def sample_f32(n, seed):
    r = np.random.default_rng(seed)
    a = (r.standard_normal(n) * np.exp2(r.integers(-14, 12, n))).astype(np.float32)
    b = r.integers(0, 2 ** 32, n, dtype=np.uint64).astype(np.uint32).view(np.float32)
    b = b[np.isfinite(b)]
    return np.concatenate([a, b])


def e4m3_edge_values():
    vals, _ = e4m3_grid()
    mids = (vals[1:] + vals[:-1]) / 2
    extra = [448, 464, 465, 480, 1e6, 2.0 ** -10, 2.0 ** -9, 3 * 2.0 ** -11, 0.0]
    x = np.concatenate([vals, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9), extra])
    x = x.astype(np.float32)
    return np.concatenate([x, -x])


def test_e4m3_encoder_is_nearest_even_saturating():
    vals, codes = e4m3_grid()
    x = np.concatenate([e4m3_edge_values(), sample_f32(200000, 1)])
    want = brute_nearest(x, vals, codes, 0x80)
    got = O.encode(O.CODE_E4M3, x)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (x[bad[:5]], got[bad[:5]], want[bad[:5]])
    # closed-form spot values
    assert O.f32_to_e4m3(448.0) == 0x7E and O.f32_to_e4m3(1e9) == 0x7E
    assert O.f32_to_e4m3(-0.0) == 0x80 and O.f32_to_e4m3(2.0 ** -9) == 0x01


def test_e4m3_encoder_agrees_with_torch_in_range():
    x = sample_f32(100000, 2)
    x = x[np.abs(x) < 464]
    t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.encode(O.CODE_E4M3, x), t)


def test_e4m3_and_e2m1_decoders():
    allc = np.arange(256, dtype=np.uint8)
    finite = (allc & 0x7F) != 0x7F
    t = torch.from_numpy(allc[finite]).view(torch.float8_e4m3fn).float().numpy()
    d = np.array([O.e4m3_value(c) for c in allc[finite]])
    assert np.array_equal(d, t.astype(np.float64))
    tab = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    for c in range(16):
        v = tab[c & 7] * (-1 if c & 8 else 1)
        assert O.e2m1_value(c) == v


def test_e2m1_encoder_is_nearest_even_saturating():
    vals, codes = e2m1_grid()
    mids = (vals[1:] + vals[:-1]) / 2
    x = np.concatenate([vals, mids, np.nextafter(mids, 0), np.nextafter(mids, 9), [7, 100, 1e30]])
    x = np.concatenate([x, -x]).astype(np.float32)
    x = np.concatenate([x, sample_f32(100000, 3)])
    want = brute_nearest(x, vals, codes, 0x8)
    got = O.encode(O.CODE_E2M1, x)
    assert np.array_equal(got, want)
    # ties: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4
    for v, code in ((0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5, 6), (6, 7)):
        assert O.f32_to_e2m1(v) == code


def test_fp16_encoder_matches_numpy_and_saturates():
    x = sample_f32(300000, 4)
    x = np.concatenate([x, np.float32([65504, 65519.99, 65520, 1e6, -1e6, 2.0 ** -25, 2.0 ** -24 * 1.5])])
    got = O.encode(O.CODE_FP16, x).view(np.uint16)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16)
    ref = np.where(np.isinf(ref), np.copysign(np.float16(65504), ref), ref).astype(np.float16)
    assert np.array_equal(got, ref.view(np.uint16))
    for h in (0x0001, 0x3C00, 0x7BFF, 0x8400, 0x03FF):
        assert O.f16_value(h) == float(np.uint16(h).view(np.float16))


def test_int8_and_mx_exponent():
    x = sample_f32(100000, 5)
    x = np.concatenate([x, np.float32([126.5, 127.5, -127.5, -128.7, 0.5, 1.5, -0.5, 2.5])])
    got = O.encode(O.CODE_INT8, x).view(np.int8)
    assert np.array_equal(got, np.clip(np.rint(x.astype(np.float64)), -127, 127).astype(np.int8))
    for a in (1.0, 448.0, 449.0, 1e-3, 3.0e-41, 2.0 ** 100, 0.999):
        want = math.frexp(a)[1] - 1 - 8
        assert O.mx_exponent(a) == max(-127, min(127, want))
    assert O.mx_exponent(0.0) == -127


# ------------------------------------------------------------ Hadamard

def test_hadamard_matrix_is_orthonormal_sylvester():
    H = O.hadamard(256)
    assert np.array_equal(H, scipy.linalg.hadamard(256) / 16.0)
    assert np.array_equal(H @ H.T, np.eye(256))


def test_fwht_of_unit_vectors_is_a_hadamard_column():
    Hs = scipy.linalg.hadamard(256).astype(np.float64) / 16
    for i in (0, 1, 7, 128, 200, 255):
        e = np.zeros(256, np.float32)
        e[i] = 1.0
        assert np.array_equal(O.fwht256(e).astype(np.float64), Hs[:, i])


def test_fwht_value_bound_involution_and_dot_invariance():
    r = np.random.default_rng(6)
    Hs = scipy.linalg.hadamard(256).astype(np.float64) / 16
    for _ in range(20):
        x = I.bf16_to_f32(I.bf16_bits(r.standard_normal(256).astype(np.float32) * 3))
        y = O.fwht256(x).astype(np.float64)
        exact = Hs @ x.astype(np.float64)
        # 8 rounded add/sub stages on partial sums bounded by ||x||_1
        assert np.max(np.abs(y - exact)) <= 8 * 2.0 ** -24 * np.abs(x).sum() / 16 * 16
        back = O.fwht256(y.astype(np.float32)).astype(np.float64)
        assert np.max(np.abs(back - x)) <= 1e-5 * np.abs(x).max()
        k = r.standard_normal(256)
        assert abs((Hs @ x) @ (Hs @ k) - x @ k) < 1e-10


# ------------------------------------------------------------ rows

def rows_for(fmt, D, is_v, n=8, seed=7, gain=1.0):
    r = np.random.default_rng(seed)
    return I.bf16_bits(r.standard_normal((n, D)).astype(np.float32) * gain)


def test_grid_valued_rows_round_trip_exactly():
    r = np.random.default_rng(8)
    vals, _ = e4m3_grid()
    D = 256
    # FP8 row-256: codes on the e4m3 grid, one at +-448, scale 2^-5 * 1.25
    s = 1.25 * 2.0 ** -5
    c = r.choice(np.concatenate([vals, -vals]), size=D)
    c[17] = -448.0
    x = I.bf16_bits((c * s).astype(np.float32))
    for fmt, is_v in ((O.FP8_ROW256, False), (O.FP8_ROW256, True), (O.K8V4, False)):
        codes, scales = O.quantize_rows(fmt, is_v, x, O.FLAG_NO_ROTATE)
        assert scales.view(np.uint16)[0, 0] == np.float16(s).view(np.uint16)
        back = O.dequant_rows(fmt, is_v, codes, scales, D)
        assert np.array_equal(back[0], c * s)
    # INT8-G64: integers with +-127 in every group, power-of-two scale per group
    ci = r.integers(-127, 128, D).astype(np.float64)
    ci[::64] = 127
    sg = np.repeat(2.0 ** np.array([-3, 0, -6, 2]), 64)
    x = I.bf16_bits((ci * sg).astype(np.float32))
    codes, scales = O.quantize_rows(O.INT8_G64, False, x, O.FLAG_NO_ROTATE)
    assert np.array_equal(codes.view(np.int8)[0], ci.astype(np.int8))
    assert np.array_equal(O.dequant_rows(O.INT8_G64, False, codes, scales, D)[0], ci * sg)
    # NVFP4-G16: e2m1 grid with a 6 in every group, ue4m3 scales
    g4 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    cf = r.choice(np.concatenate([g4, -g4]), size=D)
    cf[::16] = -6
    s16 = np.repeat(r.choice(vals[1:40], size=16), 16)
    x = I.bf16_bits((cf * s16).astype(np.float32))
    for fmt in (O.NVFP4_G16, O.K8V4):
        codes, scales = O.quantize_rows(fmt, True, x, O.FLAG_NO_ROTATE)
        assert np.array_equal(O.dequant_rows(fmt, True, codes, scales, D)[0], cf * s16)
    # MXFP8-G32 at D=128: e4m3 grid values x 2^E with 448 in each group
    D = 128
    cm = r.choice(np.concatenate([vals, -vals]), size=D)
    cm[::32] = 448
    E = np.repeat(np.array([-10, 0, 3, -1]), 32)
    x = I.bf16_bits((cm * 2.0 ** E).astype(np.float32))
    codes, scales = O.quantize_rows(O.MXFP8_G32, False, x)
    assert np.array_equal(scales[0], (np.array([-10, 0, 3, -1]) + 127).astype(np.uint8))
    assert np.array_equal(O.dequant_rows(O.MXFP8_G32, False, codes, scales, D)[0], cm * 2.0 ** E)
    # per-tensor FP8 with a given scale
    x = I.bf16_bits((cm * 0.375).astype(np.float32))
    codes, scales = O.quantize_rows(O.FP8_TENSOR, True, x, 0, 0.375)
    assert np.array_equal(O.dequant_rows(O.FP8_TENSOR, True, codes, scales, D, 0.375)[0], cm * 0.375)
    # BF16: K is the bit pattern, V the fp16 of the same value
    x = rows_for(O.BF16, 128, False)
    kc, _ = O.quantize_rows(O.BF16, False, x)
    assert np.array_equal(kc.view(np.uint16), x)
    vc, _ = O.quantize_rows(O.BF16, True, x)
    assert np.array_equal(vc.view(np.uint16), I.bf16_to_f32(x).astype(np.float16).view(np.uint16))


def test_scales_are_rounded_amax_over_qmax():
    r = np.random.default_rng(9)
    x = I.bf16_bits((r.standard_normal((16, 256)) * 3).astype(np.float32))
    xf = I.bf16_to_f32(x)
    _, s = O.quantize_rows(O.FP8_ROW256, False, x)
    want = (np.abs(xf).max(axis=1) / np.float32(448)).astype(np.float16)
    assert np.array_equal(s.view(np.uint16)[:, 0], want.view(np.uint16))
    _, s = O.quantize_rows(O.INT8_G64, True, x)             # V of INT8 is not rotated
    want = (np.abs(xf.reshape(16, 4, 64)).max(axis=2) / np.float32(127)).astype(np.float16)
    assert np.array_equal(s.view(np.uint16), want.view(np.uint16))
    _, s = O.quantize_rows(O.NVFP4_G16, True, x, O.FLAG_NO_ROTATE)
    a = torch.from_numpy(np.abs(xf.reshape(16, 16, 16)).max(axis=2) / np.float32(6))
    assert np.array_equal(s, a.to(torch.float8_e4m3fn).view(torch.uint8).numpy())


def test_groups_are_independent():
    x = rows_for(O.INT8_G64, 256, False, n=1)
    y = x.copy()
    y[0, 130] = I.bf16_bits(np.float32([500.0]))[0]
    a = O.quantize_rows(O.INT8_G64, True, x)
    b = O.quantize_rows(O.INT8_G64, True, y)
    assert np.array_equal(a[0][0, :128], b[0][0, :128]) and np.array_equal(a[1][0, :4], b[1][0, :4])
    assert not np.array_equal(a[1][0, 4:6], b[1][0, 4:6])


def test_zero_rows_store_zero():
    x = np.zeros((1, 256), np.uint16)
    for fmt in (O.FP8_ROW256, O.INT8_G64, O.NVFP4_G16, O.K8V4):
        for is_v in (False, True):
            c, s = O.quantize_rows(fmt, is_v, x)
            assert not c.any() and not s.any()
    c, s = O.quantize_rows(O.MXFP8_G32, False, np.zeros((1, 128), np.uint16))
    assert not c.any() and not s.any()


@pytest.mark.parametrize("fmt,k_rot,v_rot", [
    (O.INT8_G64, True, False), (O.NVFP4_G16, True, True), (O.K8V4, False, True),
    (O.FP8_ROW256, False, False), (O.BF16, False, False)])
def test_which_tensors_are_rotated(fmt, k_rot, v_rot):
    """[NInfer]: INT8 rotates K; NVFP4 rotates K and V; K8V4's V is NVFP4."""
    Hs = scipy.linalg.hadamard(256) / 16.0
    x = rows_for(fmt, 256, False, n=4, gain=1.0)
    xf = I.bf16_to_f32(x).astype(np.float64)
    for is_v, rot in ((False, k_rot), (True, v_rot)):
        c, s = O.quantize_rows(fmt, is_v, x)
        d = O.dequant_rows(fmt, is_v, c, s, 256)
        plain = d @ Hs if rot else d          # H symmetric: un-rotate by H
        err = np.abs(plain - xf).max()
        assert err < 0.35 * np.abs(xf).max(), (fmt, is_v, err)
        assert O.is_rotated(fmt, is_v) == rot


def test_nibble_order_low_nibble_is_even_element():
    # reading: element 2i in bits 0..3 of byte i, element 2i+1 in bits 4..7
    x = np.zeros((1, 256), np.float32)
    x[0, 0] = 6.0
    x[0, 1] = -1.0
    c, s = O.quantize_rows(O.NVFP4_G16, False, I.bf16_bits(x), O.FLAG_NO_ROTATE)
    assert s[0, 0] == 0x38     # ue4m3(6 / 6) = 1.0
    assert c[0, 0] == (0x7 | (0xA << 4))


# ------------------------------------------------------------ attention

def test_attention_single_token_returns_v():
    r = np.random.default_rng(10)
    q = r.standard_normal((3, 256))
    k = r.standard_normal((1, 256))
    v = r.standard_normal((1, 256))
    out = O.attend(q, k, v, False, False, 1 / 16)
    assert np.array_equal(out, np.repeat(v, 3, axis=0))
    Hs = scipy.linalg.hadamard(256) / 16.0
    out = O.attend(q, k, v @ Hs, True, True, 1 / 16)     # stored V row = H v
    assert np.allclose(out, np.repeat(v, 3, axis=0), atol=1e-12)


def test_attention_constant_keys_average_values():
    r = np.random.default_rng(11)
    q = r.standard_normal((2, 128))
    k = np.repeat(r.standard_normal((1, 128)), 37, axis=0)
    v = r.standard_normal((37, 128))
    out = O.attend(q, k, v, False, False, 0.3)
    assert np.allclose(out, np.repeat(v.mean(axis=0, keepdims=True), 2, axis=0), atol=1e-13)


@pytest.mark.parametrize("D,G,L,k_rot,v_rot", [(256, 1, 5, False, False), (256, 6, 130, True, True),
                                                (256, 4, 64, True, False), (128, 8, 200, False, False),
                                                (256, 6, 77, False, True)])
def test_attention_brute_force(D, G, L, k_rot, v_rot):
    r = np.random.default_rng(D + G + L)
    q = r.standard_normal((G, D))
    k = r.standard_normal((L, D)) * 2
    v = r.standard_normal((L, D))
    Hs = scipy.linalg.hadamard(D) / np.sqrt(D)
    kk = k @ Hs.T if k_rot else k              # stored rows are H k
    vv = v @ Hs.T if v_rot else v
    scale = 1 / np.sqrt(D)
    p = scipy.special.softmax(scale * (q @ k.T), axis=1)
    want = p @ v
    got = O.attend(q, kk, vv, k_rot, v_rot, scale)
    assert np.allclose(got, want, atol=1e-12, rtol=1e-10)


def test_paged_cache_matches_contiguous_attention():
    spec = I.ConfigSpec("t", ("int8_g64",), B=3, n_kv_heads=2, n_q_heads=6, head_dim=256,
                        page_size=64, lengths=("fixed", 1))
    w = I.make_workload(spec, seq_lens=np.array([1, 70, 129]), seed=5)
    c = O.PagedCache(O.INT8_G64, 256, 2, 64, w.num_pages)
    kp, vp, sp = w.prefix()
    c.append(kp, vp, sp)
    kn, vn, sn = w.new_tokens()
    sn2 = sn.copy()
    sn2[0] = -1                                   # skipped token
    c.append(kn, vn, sn2)
    assert not c.kc[sn[0]].any()
    c.append(kn[:1], vn[:1], sn[:1])
    out = c.decode(w.q, w.block_table, w.seq_lens)
    for b in range(3):
        rows = np.arange(w.starts[b], w.starts[b + 1])
        for h in range(2):
            kc, ks = O.quantize_rows(O.INT8_G64, False, w.k[rows, h])
            vc, vs = O.quantize_rows(O.INT8_G64, True, w.v[rows, h])
            kd = O.dequant_rows(O.INT8_G64, False, kc, ks, 256)
            vd = O.dequant_rows(O.INT8_G64, True, vc, vs, 256)
            q = O.bf16_bits_to_f64(w.q[b, 3 * h:3 * h + 3])
            want = O.attend(q, kd, vd, True, False, 1 / 16)
            assert np.array_equal(out[b, 3 * h:3 * h + 3], want)
