"""Adversarial inputs that make any key rotated at a wrong position dominate the attention.

Every raw key is the inverse rotation (at the key's own logical position) of the same vector
-a*u, every raw query the inverse rotation of +b*u.  Rotated correctly, all keys become -a*u and
every score equals -a*b/sqrt(d) = -S: the softmax is (nearly) uniform.  A key rotated at any
other position is no longer anti-parallel to u, so its score rises by a sizeable fraction of S
and its weight grows by orders of magnitude: the output then follows that key's value.  The
inputs are built with the oracle's positions and rotation (test infrastructure) and rounded to
bf16 like every other input.
"""
import math

import numpy as np
import torch

import oracle


def probe_inputs(cfg: dict, S: float, seed: int = 0, sign: float = -1.0):
    """(q [L_blk][H][d], k [H][T][d], v [H][T][d]) as bf16 CPU tensors.  With sign = +1 the
    keys are parallel to the queries instead: every score is about +S."""
    s = oracle.layout_sizes(cfg)
    d, H = cfg["head_dim"], cfg["n_heads"]
    g = np.random.default_rng(seed)
    u = g.standard_normal(d)
    u /= np.linalg.norm(u)
    a = b = math.sqrt(S * math.sqrt(d))
    kpos, _ = oracle.key_positions(cfg)
    qpos = oracle.query_positions(cfg)
    k1 = oracle.rope_rotate(cfg, np.broadcast_to(sign * a * u, (s["T"], d)), -kpos)
    q1 = oracle.rope_rotate(cfg, np.broadcast_to(b * u, (s["L_blk"], d)), -qpos)
    k = np.broadcast_to(k1[None], (H, s["T"], d))
    q = np.broadcast_to(q1[:, None], (s["L_blk"], H, d))
    v = g.standard_normal((H, s["T"], d))
    bf = lambda x: torch.from_numpy(np.ascontiguousarray(x)).float().to(torch.bfloat16)  # noqa
    return bf(q), bf(k), bf(v)
