"""A model of the attention kernel's roundings, for sizing test tolerances (CPU, numpy).

The kernel rotates q and k in float32 and keeps the rotated vectors as bf16 (the tensor-core
operands), accumulates q.k in float32, writes the softmax weights P as bf16 (the A operand of
the P.V product) while summing them unrounded, and rounds the normalised output to bf16.  This
module applies exactly those roundings to the float64 definition the oracle states, so that a
test can set a tolerance from what the roundings alone produce on its inputs.

The roundings move a logit s by about 2^-9 |s| (bf16 keeps 8 significant bits), so on N(0,1)
inputs (|s| up to ~5) the error stays far inside the stated tolerance (max 2e-2, mean 2e-3),
while inputs built to have logits of 20 or more (keys scaled x5, the position probe at S = 900)
already exceed it through rounding alone.  Those tests take ``max(stated bound, k * model
error)``.  Test infrastructure only: it uses the oracle's positions and rotation, never the
library.
"""
import math

import numpy as np
import torch

import oracle


def bf16(x) -> np.ndarray:
    """Round to bf16 (nearest even) and widen back to float64."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.to(torch.float64).numpy()


def _exact(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def attention_bf16_model(cfg: dict, q, k_cache, v_cache, rows, heads=None, rnd=bf16):
    """Oracle attention with the kernel's roundings applied by ``rnd``: rotated q and k, the
    weights P (their sum stays unrounded) and the output.  ``rnd=None`` applies none (the model
    then restates the oracle).  Returns ``(out [len(rows)][len(heads)][d], lse [len(heads)]
    [len(rows)])``."""
    rnd = _exact if rnd is None else rnd
    d = cfg["head_dim"]
    rows = np.asarray(rows)
    heads = np.arange(cfg["n_heads"]) if heads is None else np.asarray(heads)
    kpos, valid = oracle.key_positions(cfg)
    qpos = oracle.query_positions(cfg)[rows]
    q = np.asarray(q, dtype=np.float64)
    k_cache = np.asarray(k_cache, dtype=np.float64)
    v_cache = np.asarray(v_cache, dtype=np.float64)
    out = np.zeros((len(rows), len(heads), d))
    lse = np.zeros((len(heads), len(rows)))
    for hi, h in enumerate(heads):
        qr = rnd(oracle.rope_rotate(cfg, q[rows, h], qpos))
        kr = rnd(oracle.rope_rotate(cfg, k_cache[h][valid], kpos[valid]))
        sc = qr @ kr.T / math.sqrt(d)
        m = sc.max(axis=1, keepdims=True)
        e = np.exp(sc - m)
        l = e.sum(axis=1, keepdims=True)
        out[:, hi] = rnd((rnd(e) @ v_cache[h][valid]) / l)
        lse[hi] = (m + np.log(l))[:, 0]
    return out, lse


def model_errors(cfg: dict, q, k_cache, v_cache, rows, ref, ref_lse):
    """Max and mean |model - oracle| of the output and max |model - oracle| of the LSE."""
    out, lse = attention_bf16_model(cfg, q, k_cache, v_cache, rows)
    e = np.abs(out - ref)
    return float(e.max()), float(e.mean()), float(np.abs(lse - ref_lse).max())


def rescaled_rows(cfg: dict, q, k_cache, rows, head: int) -> np.ndarray:
    """Rows whose running maximum, taken key tile by key tile (128 physical cache rows, the
    order the kernel walks) in log2 units, grows by more than 8 at some tile: the rows for
    which the kernel rescales its output accumulator."""
    kpos, valid = oracle.key_positions(cfg)
    qpos = oracle.query_positions(cfg)[rows]
    sc = (oracle.rope_rotate(cfg, np.asarray(q, dtype=np.float64)[rows, head], qpos)
          @ oracle.rope_rotate(cfg, np.asarray(k_cache, dtype=np.float64)[head], kpos).T)
    sc = sc * (math.log2(math.e) / math.sqrt(cfg["head_dim"]))
    sc[:, ~valid] = -np.inf
    tiles = [sc[:, t:t + 128].max(axis=1) for t in range(0, sc.shape[1], 128)]
    tiles = [t for t in tiles if np.isfinite(t).any()]
    m = tiles[0].copy()
    hit = np.zeros(len(rows), dtype=bool)
    for t in tiles[1:]:
        g = t > m + 8.0
        hit |= g
        m = np.where(g, t, m)
    return hit


def max_logit(cfg: dict, q, k_cache, rows) -> float:
    """Largest |q~ . k~| / sqrt(d) over the given rows, every head and every valid key."""
    kpos, valid = oracle.key_positions(cfg)
    qpos = oracle.query_positions(cfg)[rows]
    q = np.asarray(q, dtype=np.float64)
    k_cache = np.asarray(k_cache, dtype=np.float64)
    return max(float(np.abs(oracle.rope_rotate(cfg, q[rows, h], qpos)
                            @ oracle.rope_rotate(cfg, k_cache[h][valid], kpos[valid]).T).max())
               for h in range(cfg["n_heads"])) / math.sqrt(cfg["head_dim"])
