"""Helpers of the GPU parity tests: seeded inputs on both sides, layout conversion, tolerances."""
import numpy as np
import pytest
import torch

import oracle
import synth

# Attention tolerance (bf16 inputs, fp32 accumulation and softmax, bf16 output) against the
# float64 oracle: max abs error <= 2e-2 and mean abs error <= 2e-3 per call.
ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 2e-3
# LSE (float32 from the kernel; scores see the bf16 rounding of the rotated q and k)
LSE_MAX_ABS = 2e-2


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def attention_inputs(cfg: dict, seed: int):
    """q [L_blk][H][d], k, v [H][T][d]: bf16 CPU tensors drawn by ``synth``."""
    s = oracle.layout_sizes(cfg)
    H, d = cfg["n_heads"], cfg["head_dim"]
    q = synth.normal_bf16((s["L_blk"], H, d), seed, 0)
    k = synth.normal_bf16((H, s["T"], d), seed, 1)
    v = synth.normal_bf16((H, s["T"], d), seed, 2)
    return q, k, v


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def check_attention(got: np.ndarray, ref: np.ndarray, what: str = ""):
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert err.max() <= ATTN_MAX_ABS, f"{what}: max abs error {err.max():.3e}"
    assert err.mean() <= ATTN_MEAN_ABS, f"{what}: mean abs error {err.mean():.3e}"
    return float(err.max()), float(err.mean())
