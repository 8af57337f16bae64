"""Attention inputs shared by the CPU tolerance tests and the GPU parity tests: inputs whose
logits reach far beyond those of N(0,1) draws, and inputs that make the kernel rescale its
output accumulator while every logit stays small."""
import numpy as np
import torch

import oracle
import synth
from tests._gpu import attention_inputs


def sample_rows(lblk: int, seed: int) -> np.ndarray:
    """Edge rows (first tile, tile boundary, the ragged last tile) plus 40 random rows."""
    g = np.random.default_rng(seed)
    edge = [0, 1, 127, 128, lblk - 13, lblk - 12, lblk - 1]
    return np.unique(np.concatenate([edge, g.choice(lblk, 40, replace=False)]))


def _cfg(name: str, heads: int):
    cfg = synth.preset(name, block_index=1000, valid_mask=0xFF)
    return cfg if name == "tiny" else dict(cfg, n_heads=heads)


def gain_case(name: str, slot: int, gain: float):
    """N(0,1) inputs with the keys of one slot scaled by ``gain`` (5-6: logits up to ~24).
    Slot 5 is the last physical slot (the row max jumps up late), slot 0 the first (later
    tiles sit far below the max).  Returns ``(cfg, q, k, v, rows)``."""
    cfg = _cfg(name, 4)
    q, k, v = attention_inputs(cfg, seed=13)
    a, e = oracle.slot_ranges(cfg)[slot]
    k = k.clone()
    k[:, a:e] = (k[:, a:e].float() * gain).to(torch.bfloat16)
    s = oracle.layout_sizes(cfg)
    rows = np.arange(s["L_blk"]) if name == "tiny" else sample_rows(s["L_blk"], 9)
    return cfg, q, k, v, rows


GAIN_CASES = [("tiny", 5, 6.0), ("480x480", 5, 5.0), ("480x480", 0, 5.0)]


def rescale_case(name: str, gain: float):
    """Keys of every slot but the last physical one set to zero (logits 0), keys of the last
    slot scaled by ``gain``: the row max jumps by more than 2^8 (log2 units) at the first tile
    of the last slot for a good share of rows, while the largest logit stays below ~10.
    Returns ``(cfg, q, k, v, rows)``."""
    cfg = _cfg(name, 4)
    q, k, v = attention_inputs(cfg, seed=13)
    a, _ = oracle.slot_ranges(cfg)[oracle.SLOT_RING0 + cfg["ring_slots"] - 1]
    k = k.float()
    k[:, :a] = 0.0
    k[:, a:] *= gain
    s = oracle.layout_sizes(cfg)
    rows = np.arange(s["L_blk"]) if name == "tiny" else sample_rows(s["L_blk"], 9)
    return cfg, q, k.to(torch.bfloat16), v, rows


RESCALE_CASES = [("tiny", 2.0), ("480x480", 1.6)]
