"""Failure paths of the kernels, made on purpose without faulting the GPU.

Every pipeline wait in the decode and prefill kernels is bounded: when a
stage copy or a tensor-core result does not arrive within the limit, the
kernel records bit 2 of the device status word, stops starting new work,
waits (with the default limit) for the copies and tensor-core operations it
has already issued, frees its tensor memory and returns.  These tests lower
the limit to zero polls through the test surface (kvq_debug_set_wait_polls),
so that the first wait gives up at once, and check that the call returns,
that the status word says so, and that the next call with the default limit
on the same cache is correct again -- the context stays usable.  Bad page
ids and slots are covered by the parity tests."""
import numpy as np
import pytest
import torch

import quantized_paged_kv_03_b200 as K
from quantized_paged_kv_03_b200 import inputs as I
from kvq_testutil import append_all, bf16_dev, dev, gpu_cache, gpu_decode, oracle_cache, attn_errors


def workload(cfg, D, P, lengths, H, Hq, seed=51):
    base = I.CONFIGS[cfg]
    spec = I.ConfigSpec("t", base.formats, B=len(lengths), n_kv_heads=H, n_q_heads=Hq,
                        head_dim=D, page_size=P, lengths=("fixed", 1),
                        outlier_frac=base.outlier_frac, outlier_gain=base.outlier_gain,
                        loguniform_std=base.loguniform_std)
    return I.make_workload(spec, fmt="x", seed=seed, seq_lens=np.array(lengths))


class zero_wait_limit:
    """Every wait of the launches inside the block gives up at once."""

    def __enter__(self):
        self.prev = K.set_wait_polls(0)

    def __exit__(self, *exc):
        K.set_wait_polls(-1)


@pytest.mark.gpu
@pytest.mark.parametrize("fmt,cfg,D,P,H,Hq", [("int8_g64", 1, 256, 64, 2, 8),
                                             ("nvfp4_g16", 2, 256, 256, 1, 6),
                                             ("mxfp8_g32", 4, 128, 128, 2, 16)])
def test_decode_wait_that_gives_up_is_reported_and_recovers(fmt, cfg, D, P, H, Hq):
    w = workload(cfg, D, P, [1100, 300, 5], H, Hq)
    c = gpu_cache(w, fmt, 0 if D == 256 else K.FLAG_NO_ROTATE)
    append_all(c, None, w)
    good = gpu_decode(c, w)
    assert c.read_device_status() == 0
    with zero_wait_limit():
        gpu_decode(c, w)                      # returns: gpu_decode synchronises
    assert c.read_device_status(clear=True) & K.STATUS_WAIT_TIMEOUT
    assert np.array_equal(gpu_decode(c, w), good)
    assert c.read_device_status() == 0


@pytest.mark.gpu
def test_fused_step_wait_that_gives_up_is_reported_and_recovers():
    w = workload(1, 256, 64, [700, 129, 64], 2, 8)
    ref = gpu_cache(w, "int8_g64")
    c = gpu_cache(w, "int8_g64")
    kp, vp, sp = w.prefix()
    kn, vn, sn = w.new_tokens()
    for x in (ref, c):
        x.append(0, bf16_dev(kp), bf16_dev(vp), dev(sp))
    ref.append(0, bf16_dev(kn), bf16_dev(vn), dev(sn))
    want = gpu_decode(ref, w)
    args = (0, bf16_dev(kn), bf16_dev(vn), bf16_dev(w.q), dev(w.block_table), dev(w.seq_lens), w.max_seq_len)
    with zero_wait_limit():
        c.append_decode(*args)
        torch.cuda.synchronize()
    assert c.read_device_status(clear=True) & K.STATUS_WAIT_TIMEOUT
    got = c.append_decode(*args)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy().astype(np.float64), want)
    assert c.read_device_status() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("fmt,cfg,D,P,H,Hq", [("int8_g64", 1, 256, 64, 2, 8), ("bf16", 4, 128, 32, 2, 8)])
def test_prefill_wait_that_gives_up_is_reported_and_recovers(fmt, cfg, D, P, H, Hq):
    w = workload(cfg, D, P, [600, 200], H, Hq)
    c = gpu_cache(w, fmt)
    oc = oracle_cache(w, fmt)
    append_all(c, oc, w)
    q, cu = I.prefill_queries(w, [300, 200])
    run = lambda: c.prefill_attention(0, bf16_dev(q), dev(cu), dev(w.block_table), dev(w.seq_lens), 300)
    good = run().cpu().numpy()
    assert c.read_device_status() == 0
    with zero_wait_limit():
        run()
        torch.cuda.synchronize()
    assert c.read_device_status(clear=True) & K.STATUS_WAIT_TIMEOUT
    again = run().cpu().numpy()
    assert np.array_equal(again, good)
    assert c.read_device_status() == 0
    # and the recovered result is the right one
    want = oc.prefill(q, cu, w.block_table, w.seq_lens)
    vm = np.abs(I.bf16_to_f32(w.v)).max()
    assert np.abs(again.astype(np.float64) - want).max() <= 2e-3 * vm
