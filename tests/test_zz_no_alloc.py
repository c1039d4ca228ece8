"""The allocation-free decode entry point (kvq_decode_attention_noalloc).

Callers such as an engine plugin that is handed only its input and output
buffers, or a process whose device-memory budget is fixed at start-up, cannot
call cudaMalloc to provide a workspace.  This entry point keeps its scratch in
a fixed array inside the library instead.  The test calls it through the C ABI
twice in a row and checks both results against the workspace-taking
kvq_decode_attention on the same inputs, within the attention tolerance used
by the other decode tests -- and, since it is the same kernel on the same
inputs, bit for bit.  This file is named to be collected last."""
import ctypes

import numpy as np
import pytest
import torch

import quantized_paged_kv_03_b200 as K
from quantized_paged_kv_03_b200 import inputs as I
from kvq_testutil import ATTN_TOL, append_all, bf16_dev, dev, gpu_cache, vmax_per_head


def workload(lengths, H=2, Hq=8, seed=23):
    base = I.CONFIGS[1]
    spec = I.ConfigSpec("t", base.formats, B=len(lengths), n_kv_heads=H, n_q_heads=Hq,
                        head_dim=256, page_size=64, lengths=("fixed", 1),
                        outlier_frac=base.outlier_frac, outlier_gain=base.outlier_gain)
    return I.make_workload(spec, fmt="x", seed=seed, seq_lens=np.array(lengths))


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_decode_twice():
    w = workload([3000, 700, 1, 1500])          # segments split across many CTAs
    c = gpu_cache(w, "int8_g64")
    append_all(c, None, w)
    q, bt, sl = bf16_dev(w.q), dev(w.block_table), dev(w.seq_lens)
    ref = c.decode_attention(0, q, bt, sl, w.max_seq_len)
    L = K.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    vm = np.repeat(vmax_per_head(w), w.Hq // w.H, axis=1)[:, :, None]
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        st = L.kvq_decode_attention_noalloc(c.handle, 0, q.data_ptr(), w.Hq, bt.data_ptr(),
                                            bt.shape[1], sl.data_ptr(), w.B, w.max_seq_len,
                                            out.data_ptr(), 1, ctypes.c_float(0.0), stream)
        assert st == 0, L.kvq_status_string(st)
        torch.cuda.synchronize()
        got, want = out.cpu().numpy().astype(np.float64), ref.cpu().numpy().astype(np.float64)
        assert (np.abs(got - want) <= ATTN_TOL * vm).all()
        assert np.array_equal(got, want)
    assert c.read_device_status() == 0


@pytest.mark.gpu
def test_noalloc_scratch_covers_the_largest_plannable_decode():
    """The scratch limit is checked before any launch; on this device the
    largest decode the library can plan (head_dim 256, a full persistent grid)
    fits in it, and bad shapes are still rejected with a status code."""
    c = K.KVCache("int8_g64", 256, 8, 64, 1)
    L = K.lib()
    need = L.kvq_decode_workspace_bytes(c.handle, 4096, 8 * 8, 1 << 24)
    assert 0 < need <= K.NOALLOC_SCRATCH_BYTES
    p = ctypes.c_void_p(16)                      # never dereferenced: rejected before any launch
    st = L.kvq_decode_attention_noalloc(c.handle, 0, p, 8 * 8 + 1, p, 1 << 18, p, 4096, 1 << 24, p,
                                        1, ctypes.c_float(0.0), None)
    assert st == 3                               # n_q_heads not a multiple of n_kv_heads
