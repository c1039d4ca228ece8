"""The append kernel's element encoders (PTX cvt with satfinite, fp16 with
saturation, int8 nearest-even) against the oracle's encoders written from the
format definitions, over every finite fp32 bit pattern."""
import numpy as np
import pytest
import torch

import oracle as O
import quantized_paged_kv_03_b200 as K
from kvq_testutil import ensure_built

CHUNK = 1 << 28
CODES = [("e4m3", O.CODE_E4M3), ("e2m1", O.CODE_E2M1), ("ue4m3", O.CODE_UE4M3),
         ("int8", O.CODE_INT8), ("fp16", O.CODE_FP16)]


def not_nan_mask(start: int, n: int) -> np.ndarray:
    bits = (np.arange(start, start + n, dtype=np.uint64) & 0xFFFFFFFF).astype(np.uint32)
    return ~(((bits & 0x7F800000) == 0x7F800000) & ((bits & 0x007FFFFF) != 0))


@pytest.mark.gpu
@pytest.mark.parametrize("name,code", CODES)
def test_encoder_matches_oracle_on_every_fp32(name, code):
    ensure_built()
    threads = min(32, max(1, __import__("os").cpu_count() or 1))
    w = O.code_width(code)
    ones = 0
    if name == "ue4m3":
        # a scale encoder only sees non-negative values: the positive half
        ranges = [(0, 1 << 31)]
    else:
        ranges = [(0, 1 << 32)]
    for lo, hi in ranges:
        for start in range(lo, hi, CHUNK):
            n = min(CHUNK, hi - start)
            x = torch.arange(start, start + n, dtype=torch.int64, device="cuda").to(torch.int32)
            got = K.encode(name, x.view(torch.float32)).cpu().numpy()
            want = O.encode_bits(code, start, n, threads=threads)
            keep = not_nan_mask(start, n)
            if w == 2:
                keep = np.repeat(keep, 2)
            bad = np.nonzero((got != want) & keep)[0]
            assert bad.size == 0, (name, hex(start + int(bad[0]) // w), got[bad[:4]], want[bad[:4]])
            ones += 1
    assert ones >= 8
