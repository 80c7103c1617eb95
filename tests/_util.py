"""Shared helpers of the test-suite (input sampling, tolerances)."""
import numpy as np
import torch

# Max-abs-error bounds against the float64 oracle, per compute dtype.
TOL = {torch.float32: 1e-4, torch.float16: 1e-2, torch.bfloat16: 2e-2}


def sample_rows(B, H, L, g_list, pad_list, n_random=400, seed=0):
    """(b, h, i) rows covering every global row of two heads, tile edges
    (i % 128 in {0, 127}), the padding boundary, the sequence end and random
    rows."""
    rng = np.random.default_rng(seed)
    rows = set()
    for b in range(B):
        g, pad = g_list[b], pad_list[b]
        for h in {0, H - 1}:
            rows.update((b, h, i) for i in range(g))
        for h in range(H):
            for i in list(range(0, L, 128)) + list(range(127, L, 128)):
                if rng.random() < 0.25:
                    rows.add((b, h, i))
        edge = [L - pad - 1, L - pad, L - 1, g, g - 1 if g > 0 else 0]
        rows.update((b, int(rng.integers(H)), i) for i in edge if 0 <= i < L)
    for _ in range(n_random):
        rows.add((int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(L))))
    return np.array(sorted(rows), dtype=np.int32)
