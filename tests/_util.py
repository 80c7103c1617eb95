"""Shared helpers of the test-suite (tolerances)."""
import torch

# Max-abs-error bounds against the float64 oracle, per compute dtype.
TOL = {torch.float32: 1e-4, torch.float16: 1e-2, torch.bfloat16: 2e-2}

