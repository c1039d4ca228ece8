"""bench.py's accounting on CPU: the chunked-prefill FLOP count against the
visible (query, key) pairs of torch's lower-right causal mask, and the source
digest that guards a recorded ncu capture (comments may change, code may not)."""
import os
import shutil
import sys

import torch
from torch.nn.attention.bias import causal_lower_right

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_prefill_flops_count_the_causal_pairs():
    # chunks shorter than, equal to and longer than the cached sequence
    cases = [(8192, 512), (70, 70), (300, 1), (5, 8), (0, 0)]
    Hq, D = 6, 128
    for L, n in cases:
        if n == 0:
            pairs = 0
        elif n <= L:
            pairs = int(causal_lower_right(n, L)._materialize().sum())
        else:   # the first n - L rows see no key; the rest form the n = L case
            pairs = int(torch.tril(torch.ones(L, L, dtype=torch.bool)).sum())
        assert bench.prefill_flops([L], [n], Hq, D) == 4 * D * Hq * pairs, (L, n)
    both = bench.prefill_flops([8192, 300], [512, 1], Hq, D)
    assert both == bench.prefill_flops([8192], [512], Hq, D) + bench.prefill_flops([300], [1], Hq, D)


def test_kernel_digest_ignores_comments_only(tmp_path, monkeypatch):
    csrc = tmp_path / "quantized_paged_kv_03_b200" / "csrc"
    shutil.copytree(os.path.join(ROOT, "quantized_paged_kv_03_b200", "csrc"), csrc)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    files = bench.PREFILL_SOURCES
    base = bench.kernel_digest(files)
    f = csrc / "kvq_prefill.cu"
    src = f.read_text()
    f.write_text("// a new comment line\n" + src.replace("\n", "\n  ", 3) + "\n/* and a block */\n")
    assert bench.kernel_digest(files) == base
    f.write_text(src.replace("kPrefillWaitPolls = 1l << 22", "kPrefillWaitPolls = 1l << 21"))
    assert bench.kernel_digest(files) != base


def test_recorded_traffic_is_reported_only_for_its_workload():
    # a capture describes one workload: a reduced batch or another config gets none
    assert bench.headline_traffic(bench.HEADLINE_CONFIG, 4) is None
    assert bench.headline_traffic(bench.HEADLINE_CONFIG + 1, None) is None
