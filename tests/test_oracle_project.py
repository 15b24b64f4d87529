"""Pins of the projection oracle (CPU): its bf16 rounding against PyTorch's
fp32 -> bf16 conversion (round to nearest even) on random values, ties and
special values; its product against a plain Python triple loop on a small
case."""
import numpy as np
import torch

from oracle.project import bf16_rne, kv_project


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    a = (rng.standard_normal(100000) * np.exp2(rng.integers(-30, 30, 100000))).astype(np.float32)
    # exact ties between two bf16 values, both parities of the kept bit
    base = rng.integers(0, 1 << 16, 2000).astype(np.uint32) << 16
    ties = (base | 0x8000).view(np.float32)
    special = np.array([0.0, -0.0, np.inf, -np.inf, 3.3895314e38, 1e-40, -1e-45], np.float32)
    for v in (a, ties[np.isfinite(ties)], special):
        want = torch.from_numpy(v).to(torch.bfloat16).float().numpy()
        np.testing.assert_array_equal(bf16_rne(v).view(np.uint32), want.view(np.uint32))


def test_product_against_loops():
    rng = np.random.default_rng(1)
    x = bf16_rne(rng.standard_normal((5, 64)))
    w = bf16_rne(rng.standard_normal((7, 64)) / 8)
    got = kv_project(x, w)
    for i in range(5):
        for j in range(7):
            s = 0.0
            for k in range(64):
                s += float(x[i, k]) * float(w[j, k])
            want = torch.tensor(s, dtype=torch.float32).to(torch.bfloat16).float().item()
            assert got[i, j] == np.float32(want), (i, j)
