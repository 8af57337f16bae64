"""Seeded synthetic inputs for the PR-Sink hot path.

This module is shared by the CPU oracle tests, the GPU parity tests and ``bench.py``.  It holds
random draws, the workload presets and a bf16 rounding of the drawn values, and nothing of the
method's arithmetic: no slot layout, no RoPE, no attention, no fingerprint, no similarity.
Every size it needs is passed in by the caller.

The pages fix no dataset that could be used here (the 3-minute pose benchmark and the 14B
weights are not available), so every input is synthetic with the shapes the pages and the
workload list give:

* attention: Q, K, V ~ N(0, 1), rounded to bf16 (round to nearest even), laid out as a QKV
  projection emits them (token-major ``[L][H][d]``) or as the head-major cache holds them
  (``[H][T][d]``);
* poses: whole-body keypoints (133 per frame, x and y normalised to [0, 1], a confidence in
  [0, 1]), a block being 3 latent frames; a share of frames is marked as a failed detection;
* the long stream: poses drawn around 12 recurring cluster centres (sigma 0.03 on x and y) whose
  order is a seeded random walk that revisits clusters.
"""
from __future__ import annotations

import numpy as np
import torch

__all__ = [
    "PRESETS",
    "preset",
    "normal_bf16",
    "keypoints",
    "pose_stream",
    "uniform_unit_rows",
]

# Workload presets.  The attention sizes follow the pages' resolution buckets (480x480, 384x672,
# 672x384 with a 16x spatial VAE factor and 2x2 patches, i.e. one latent token per 16x16 pixels)
# and a block of 3 latent frames; 40 heads of 128 are the attention shape of the 14B DiT.
PRESETS = {
    "tiny": dict(n_heads=1, head_dim=64, grid_h=4, grid_w=4, frames_per_block=3,
                 ref_frames=1, ring_slots=3, rope_mode=1, rope_split=(64, 0, 0),
                 rope_base=10000.0),
    "480x480": dict(n_heads=40, head_dim=128, grid_h=30, grid_w=30, frames_per_block=3,
                    ref_frames=1, ring_slots=3, rope_mode=3, rope_split=(44, 42, 42),
                    rope_base=10000.0),
    "384x672": dict(n_heads=40, head_dim=128, grid_h=24, grid_w=42, frames_per_block=3,
                    ref_frames=1, ring_slots=3, rope_mode=3, rope_split=(44, 42, 42),
                    rope_base=10000.0),
    "672x384": dict(n_heads=40, head_dim=128, grid_h=42, grid_w=24, frames_per_block=3,
                    ref_frames=1, ring_slots=3, rope_mode=3, rope_split=(44, 42, 42),
                    rope_base=10000.0),
    # the literal "1008 + 3x3024 + 3x3024 = 19152 keys" reading: four ring slots
    "384x672_r4": dict(n_heads=40, head_dim=128, grid_h=24, grid_w=42, frames_per_block=3,
                       ref_frames=1, ring_slots=4, rope_mode=3, rope_split=(44, 42, 42),
                       rope_base=10000.0),
}


def preset(name: str, **overrides) -> dict:
    """A copy of a preset with fields overridden (e.g. ``block_index``, ``valid_mask``)."""
    cfg = dict(PRESETS[name])
    cfg.update(overrides)
    return cfg


def _rng(seed: int, stream: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), int(stream)]))


def normal_bf16(shape, seed: int, stream: int = 0) -> torch.Tensor:
    """N(0, 1) draws of ``shape``, rounded to bf16 (RNE).  Returns a CPU bf16 tensor.

    Both sides consume exactly these bf16 values: the GPU path takes the bits, the oracle takes
    them widened to float64.
    """
    x = _rng(seed, stream).standard_normal(size=tuple(shape), dtype=np.float32)
    return torch.from_numpy(x).to(torch.bfloat16)


def uniform_unit_rows(n: int, dim: int, seed: int, stream: int = 0) -> np.ndarray:
    """``n`` rows of ``dim`` U[0, 1) float32 values (raw material for fingerprint tests)."""
    return _rng(seed, stream).random(size=(n, dim), dtype=np.float32)


def keypoints(seed: int, n_frames: int = 3, n_kp: int = 133, fail_frac: float = 0.05,
              stream: int = 0):
    """One block of whole-body keypoints.

    Returns ``(kp, ok)``: ``kp`` float32 ``[n_frames][n_kp][3]`` with x, y ~ U[0, 1] and
    conf ~ U[0, 1]; ``ok`` uint8 ``[n_frames]``, 0 for a frame whose detection failed (each
    frame fails with probability ``fail_frac``).  A failed frame's keypoints are still drawn;
    the method decides what to do with them.
    """
    g = _rng(seed, stream)
    kp = g.random(size=(n_frames, n_kp, 3), dtype=np.float32)
    ok = (g.random(size=n_frames) >= fail_frac).astype(np.uint8)
    return kp, ok


def pose_stream(seed: int, n_blocks: int, n_frames: int = 3, n_kp: int = 133,
                n_clusters: int = 12, sigma: float = 0.03, fail_frac: float = 0.05,
                stay_prob: float = 0.5, attempt=None):
    """Keypoints for a long stream whose poses recur.

    ``n_clusters`` centre poses are drawn (x, y ~ U[0.1, 0.9], conf ~ U[0.6, 1]).  The cluster
    of each block follows a seeded random walk: with probability ``stay_prob`` the block keeps
    the previous cluster, else it jumps to a uniformly drawn one, so clusters are revisited.
    Each frame is its cluster centre plus N(0, sigma^2) noise on x and y (conf unchanged), and
    fails with probability ``fail_frac``.

    ``attempt`` (optional int array ``[n_blocks]``) re-draws the noise of single blocks: block
    ``b`` uses noise stream ``attempt[b]``, so a caller can re-sample one block without moving
    any other.  Returns ``(kp [n_blocks][n_frames][n_kp][3] float32, ok [n_blocks][n_frames]
    uint8, cluster [n_blocks] int)``.
    """
    g = _rng(seed, 0)
    centres = np.empty((n_clusters, n_kp, 3), dtype=np.float64)
    centres[:, :, 0:2] = g.uniform(0.1, 0.9, size=(n_clusters, n_kp, 2))
    centres[:, :, 2] = g.uniform(0.6, 1.0, size=(n_clusters, n_kp))
    cluster = np.empty(n_blocks, dtype=np.int64)
    c = int(g.integers(n_clusters))
    for b in range(n_blocks):
        if b > 0 and g.random() >= stay_prob:
            c = int(g.integers(n_clusters))
        cluster[b] = c
    if attempt is None:
        attempt = np.zeros(n_blocks, dtype=np.int64)
    kp = np.empty((n_blocks, n_frames, n_kp, 3), dtype=np.float32)
    ok = np.empty((n_blocks, n_frames), dtype=np.uint8)
    for b in range(n_blocks):
        gb = _rng(seed, 1_000_000 + 1000 * b + int(attempt[b]))
        noise = gb.normal(0.0, sigma, size=(n_frames, n_kp, 2))
        frame = np.repeat(centres[cluster[b]][None], n_frames, axis=0)
        frame[:, :, 0:2] += noise
        kp[b] = frame.astype(np.float32)
        ok[b] = (gb.random(size=n_frames) >= fail_frac).astype(np.uint8)
    return kp, ok, cluster
