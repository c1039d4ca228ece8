"""Parity at the workloads' full sizes, run the way bench.py runs them (bulk
prefix append, one-token-per-sequence step append, decode with the planned
persistent grid): for sampled (sequence, kv-head) pairs the stored codes and
scales must equal the oracle's bit for bit and the attention outputs must be
within 2e-3 * max|V| of the oracle's fp64 attention.  The samples include the
longest and the shortest sequence of each batch."""
import numpy as np
import pytest
import torch

import oracle as O
import quantized_paged_kv_03_b200 as K
from quantized_paged_kv_03_b200 import inputs as I
from kvq_testutil import ATTN_TOL, bf16_dev, dev, ensure_built, tensor_scales

CASES = [(1, "int8_g64"), (2, "nvfp4_g16"), (3, "k8v4"), (4, "mxfp8_g32"), (4, "fp8_tensor"), (4, "bf16")]
_workloads = {}


def workload(cfg, fmt):
    """The config's seeded inputs with the page table of this format's page size
    (one full-size workload is kept in host memory at a time)."""
    spec = I.CONFIGS[cfg]
    key = (cfg, spec.page_size_by_format.get(fmt, spec.page_size))
    if key not in _workloads:
        _workloads.clear()
        _workloads[key] = I.make_workload(cfg, fmt=fmt)
    return _workloads[key]


def run_gpu(w: I.Workload, fmt: str, scales):
    """Bench-shaped run: bulk prefix append, step append, decode (fp32 out)."""
    c = K.KVCache(fmt, w.D, w.H, w.P, w.num_pages, 1, 0, [scales] if fmt == "fp8_tensor" else None)
    kp, vp, sp = w.prefix()
    step = 1 << 20
    for i in range(0, len(sp), step):
        c.append(0, bf16_dev(kp[i:i + step]), bf16_dev(vp[i:i + step]), dev(sp[i:i + step]))
    del kp, vp
    kn, vn, sn = w.new_tokens()
    c.append(0, bf16_dev(kn), bf16_dev(vn), dev(sn))
    out = c.decode_attention(0, bf16_dev(w.q), dev(w.block_table), dev(w.seq_lens), w.max_seq_len)
    torch.cuda.synchronize()
    return c, out.cpu().numpy().astype(np.float64)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg,fmt", CASES)
def test_full_size_sampled_parity(cfg, fmt):
    ensure_built()
    w = workload(cfg, fmt)
    scales = tensor_scales(w) if fmt == "fp8_tensor" else (1.0, 1.0)
    c, out = run_gpu(w, fmt, scales)
    assert c.read_device_status() == 0
    f = K.FORMATS[fmt]
    G = w.Hq // w.H
    order = np.argsort(w.seq_lens)
    seqs = sorted({int(order[0]), int(order[-1]), int(order[len(order) // 2])})
    rng = np.random.default_rng(cfg)
    for b in seqs:
        L = int(w.seq_lens[b])
        rows = np.arange(w.starts[b], w.starts[b + 1])
        slots = w.slots(b, 0, L)
        kc, ks, vc, vs = [t.cpu().numpy() for t in c.read_rows(0, dev(slots))]
        for h in sorted({0, int(rng.integers(w.H))}):
            okc, oks = O.quantize_rows(f, False, w.k[rows, h], 0, scales[0])
            ovc, ovs = O.quantize_rows(f, True, w.v[rows, h], 0, scales[1])
            assert np.array_equal(kc[:, h], okc) and np.array_equal(ks[:, h], oks), (fmt, b, h, "K")
            assert np.array_equal(vc[:, h], ovc) and np.array_equal(vs[:, h], ovs), (fmt, b, h, "V")
            kd = O.dequant_rows(f, False, okc, oks, w.D, scales[0])
            vd = O.dequant_rows(f, True, ovc, ovs, w.D, scales[1])
            q = O.bf16_bits_to_f64(w.q[b, h * G:(h + 1) * G])
            want = O.attend(q, kd, vd, O.is_rotated(f, False), O.is_rotated(f, True), 1 / np.sqrt(w.D))
            vmax = float(np.abs(I.bf16_to_f32(w.v[rows, h])).max())
            err = np.abs(out[b, h * G:(h + 1) * G] - want).max()
            assert err <= ATTN_TOL * vmax, (fmt, b, h, err, ATTN_TOL * vmax)
