"""Plain, slow, float64 oracle for LiveAnimate's PR-Sink per-block step.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the CPU-baseline leg of the
benchmark may import this module.  It shares no code with the CUDA library; both sides only
share the seeded input generators in ``synth``.

Sources (web pages about arXiv 2608.11745, "LiveAnimate: Stable Long-Form Streaming Human
Animation in Real-Time"); citations below use these tags:

  [digest]     paper.rainbus.top/paper/2608.11745, "LiveAnimate：实时稳定的长时间流式人体动画".
               Paragraphs: "pipeline" (完整流程…, with its training and inference clauses),
               "novelty" (技术新颖性…, points 2-4), "weaknesses" (弱点…), "reproducibility"
               (复现评估…).
  [explainer]  papers.ananclaw.com, "LiveAnimate：实时长流人体动画的 14B DiT 方案",
               section "Pose-Retrieval Sink Attention（PR-Sink）" (the KV-cache slot diagram).
  [abstract]   HF papers abstract, Chinese translation (bittide.aicompass.dev mirror).
  [news]       jiazhuangai.com, "LiveAnimate：让数字人实时跳舞…", section "三个关键突破", item 1.

What the oracle computes, function by function:

  layout_sizes / slot_ranges   slot structure [Ref; Static; Dynamic; Rolling x R]
  ring_rank                    age order of the rolling slots (oldest -> newest)
  key_positions                logical (t, h, w) / 1-D position of every cached key, validity
  query_positions              positions of the current block's queries
  rope_rotate                  rotary embedding of raw vectors at given positions
  attention                    softmax(q k^T / sqrt(d)) v over the valid cached keys
  kv_append                    write raw K/V of one block into a cache slot
  dyn_copy / bank_store        K/V row copies: bank -> dynamic sink, ring -> bank
  fingerprint                  558-d l2-normalised pose fingerprint with zero-filled failures
  retrieve                     r(b) = argmax phi_b . phi_i over the bank, excluding block b-1
  bank_objective / bank_update diversity-driven replacement (mean pairwise similarity)
  valid_mask                   which slots hold data at block b
  stream_decisions             the per-block decision sequence of a stream
  retrieve_fallback            retrieval that falls back to Static Sink + window when too few
                               frames were detected ([digest] weaknesses, point 5)
  bank_update_gated            bank refresh after the freeze, gated on fingerprint distance
  bank_update_decay /          decay-weighted continuous writes after the freeze (moving
    bank_blend_kv              average of the nearest entry's fingerprint and K/V)
                               ([digest] weaknesses, point 3)
  stream_decisions_policy      the decision sequence of a stream under one of these policies

Readings taken where the sources are silent (each is repeated at its function):

  * Logical order of the keys is [ref; static; dynamic; ring oldest..newest]; the sources give
    the slot order ([explainer] diagram; [digest] pipeline formula puts K_ref first) but not
    numeric positions.  Frames are numbered 0.. in that order; a 3-D token is (t, h, w) with t
    its logical frame and (h, w) its row-major grid cell; the 1-D position is the logical
    token index.  Positions of slots that hold no data are still reserved.
  * RoPE: RoFormer rotation of interleaved pairs (x[2j], x[2j+1]) per axis, theta_j =
    base^(-2j/d_axis); 3-D splits head_dim into (t, h, w) parts; queries and keys are rotated,
    values are not.
  * The current block sits in the newest ring slot and its queries take that slot's
    positions; within the valid slots there is no other mask (block-causal attention sees the
    whole current block).
  * Retrieval ties go to the lowest bank slot; an empty eligible set gives r = -1.
  * Bank objective: mean over unordered pairs i < j of phi_i . phi_j; options are "keep" and
    "replace slot j"; ties go to keep, then to the lowest j.
  * Fingerprint: a frame whose detection failed contributes zeros; an all-zero vector stays 0.
"""
from __future__ import annotations

import itertools
import math

import numpy as np

__all__ = [
    "SLOT_REF", "SLOT_STATIC", "SLOT_DYNAMIC", "SLOT_RING0",
    "FP_FRAMES", "FP_KEYPOINTS", "FP_CHANNELS", "FP_DIM",
    "layout_sizes", "slot_ranges", "ring_rank", "slot_frame_base", "key_positions",
    "query_positions", "rope_angles", "rope_rotate", "attention", "attention_probs",
    "kv_append", "dyn_copy", "bank_store", "fingerprint", "retrieve", "retrieval_margin",
    "bank_objective", "bank_update", "bank_margin", "valid_mask", "stream_decisions",
    "detected_frames", "retrieve_fallback", "fingerprint_distances", "bank_update_gated",
    "gate_margin", "nearest_entry", "nearest_margin", "blend_weights", "bank_update_decay",
    "bank_blend_kv", "stream_decisions_policy",
]

# Slot identifiers; bit i of a validity mask refers to slot i.
SLOT_REF = 0
SLOT_STATIC = 1
SLOT_DYNAMIC = 2
SLOT_RING0 = 3

# [digest] pipeline, inference clause: three frames x 62 keypoints x 3 values = 558.
FP_FRAMES = 3
FP_KEYPOINTS = 62
FP_CHANNELS = 3
FP_DIM = FP_FRAMES * FP_KEYPOINTS * FP_CHANNELS


# --------------------------------------------------------------------------------------------
# slot layout
# --------------------------------------------------------------------------------------------

def layout_sizes(cfg: dict) -> dict:
    """Token counts of the bounded cache.

    [explainer] PR-Sink section: the cache is [Static Sink][Dynamic Sink][Rolling t-2, t-1, t];
    [digest] pipeline formula prepends K_ref.  Static and dynamic sinks and each rolling slot
    hold one block (B_f latent frames, [digest] reproducibility: 3 latent frames per block);
    the ref sink holds ``ref_frames`` latent frames.
    """
    lf = cfg["grid_h"] * cfg["grid_w"]
    lblk = cfg["frames_per_block"] * lf
    lref = cfg["ref_frames"] * lf
    r = cfg["ring_slots"]
    return dict(L_f=lf, L_blk=lblk, L_ref=lref, R=r, T=lref + (2 + r) * lblk)


def slot_ranges(cfg: dict) -> list:
    """Physical [start, end) key rows of every slot id (ref, static, dynamic, ring 0..R-1)."""
    s = layout_sizes(cfg)
    out = [(0, s["L_ref"])]
    start = s["L_ref"]
    for _ in range(2 + s["R"]):
        out.append((start, start + s["L_blk"]))
        start += s["L_blk"]
    return out


def ring_rank(slot: int, b: int, R: int) -> int:
    """Age rank (0 = oldest, R-1 = newest) of physical ring slot ``slot`` while block b runs.

    [explainer] PR-Sink: the rolling window keeps the most recent blocks (t-2, t-1, t);
    [news] item 1: the current block and the two before it.  Block b' is written into ring
    slot b' mod R, so at block b slot s holds the b' in [b-R+1, b] with b' = s (mod R).
    """
    oldest = b - R + 1
    return (slot - oldest) % R


def slot_frame_base(cfg: dict, slot: int, b: int) -> int:
    """Logical frame index of the first frame of a slot (reading: frames numbered in the
    order ref, static, dynamic, ring oldest..newest)."""
    fref = cfg["ref_frames"]
    bf = cfg["frames_per_block"]
    if slot == SLOT_REF:
        return 0
    if slot == SLOT_STATIC:
        return fref
    if slot == SLOT_DYNAMIC:
        return fref + bf
    k = ring_rank(slot - SLOT_RING0, b, cfg["ring_slots"])
    return fref + (2 + k) * bf


def _frame_token_positions(cfg: dict, frame: np.ndarray, tok: np.ndarray) -> np.ndarray:
    gw = cfg["grid_w"]
    if cfg["rope_mode"] == 3:
        return np.stack([frame, tok // gw, tok % gw], axis=-1)
    lf = cfg["grid_h"] * gw
    return frame * lf + tok


def key_positions(cfg: dict):
    """Positions and validity of every physical key row of the cache at block ``block_index``.

    [digest] pipeline, inference clause (RoPE follow): keys are cached raw, before rotation,
    and are rotated at their *current* cache position at attention time.  [digest] novelty,
    point 4: a reused bank entry is thereby decoupled from its original time stamp.

    Returns ``(pos, valid)``: ``pos`` int64 ``[T, 3]`` (3-D) or ``[T]`` (1-D), ``valid`` bool
    ``[T]`` from bit ``slot`` of ``cfg['valid_mask']``.
    """
    s = layout_sizes(cfg)
    b = cfg["block_index"]
    lf = s["L_f"]
    frames = np.empty(s["T"], dtype=np.int64)
    toks = np.empty(s["T"], dtype=np.int64)
    valid = np.empty(s["T"], dtype=bool)
    mask = int(cfg["valid_mask"])
    for slot, (a, e) in enumerate(slot_ranges(cfg)):
        u = np.arange(e - a, dtype=np.int64)
        frames[a:e] = slot_frame_base(cfg, slot, b) + u // lf
        toks[a:e] = u % lf
        valid[a:e] = bool((mask >> slot) & 1)
    return _frame_token_positions(cfg, frames, toks), valid


def query_positions(cfg: dict) -> np.ndarray:
    """Positions of the current block's L_blk queries: the newest ring slot's positions
    (reading: the current block is rank R-1 of the rolling window, [explainer] "t")."""
    s = layout_sizes(cfg)
    base = cfg["ref_frames"] + (2 + s["R"] - 1) * cfg["frames_per_block"]
    u = np.arange(s["L_blk"], dtype=np.int64)
    return _frame_token_positions(cfg, base + u // s["L_f"], u % s["L_f"])


# --------------------------------------------------------------------------------------------
# RoPE
# --------------------------------------------------------------------------------------------

def _rope_axes(cfg: dict):
    d = cfg["head_dim"]
    if cfg["rope_mode"] == 3:
        split = [int(v) for v in cfg["rope_split"]]
        assert sum(split) == d and all(v % 2 == 0 for v in split)
        offs = [0, split[0], split[0] + split[1]]
        return list(zip(offs, split))
    return [(0, d)]


def rope_angles(cfg: dict, pos: np.ndarray) -> np.ndarray:
    """Rotation angle of every pair: ``[..., head_dim // 2]`` float64.

    Pair j of an axis with d_a dims turns by pos_axis * base^(-2j/d_a) (RoFormer frequencies).
    """
    base = float(cfg["rope_base"])
    pos = np.asarray(pos)
    parts = []
    for ax, (_, da) in enumerate(_rope_axes(cfg)):
        j = np.arange(da // 2, dtype=np.float64)
        theta = base ** (-2.0 * j / da)
        p = pos[..., ax] if cfg["rope_mode"] == 3 else pos
        parts.append(p.astype(np.float64)[..., None] * theta)
    return np.concatenate(parts, axis=-1)


def rope_rotate(cfg: dict, x: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """Rotate raw vectors ``x[..., head_dim]`` at positions ``pos``.

    Each interleaved pair (x[2i], x[2i+1]) (within its axis' dims) becomes
    (x0 cos a - x1 sin a, x0 sin a + x1 cos a), a the pair's angle.
    """
    x = np.asarray(x, dtype=np.float64)
    ang = rope_angles(cfg, pos)
    c, s = np.cos(ang), np.sin(ang)
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


# --------------------------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------------------------

def attention_probs(cfg: dict, q: np.ndarray, k_cache: np.ndarray, head: int, rows=None):
    """Softmax weights of one head: ``(P [nrows, T], valid [T])`` with zeros at invalid keys."""
    s = layout_sizes(cfg)
    d = cfg["head_dim"]
    kpos, valid = key_positions(cfg)
    qpos = query_positions(cfg)
    if rows is None:
        rows = np.arange(s["L_blk"])
    qr = rope_rotate(cfg, q[rows, head, :], qpos[rows])
    kr = rope_rotate(cfg, k_cache[head][valid], kpos[valid])
    sc = qr @ kr.T / math.sqrt(d)
    p = np.zeros((len(rows), s["T"]), dtype=np.float64)
    if sc.shape[1]:
        e = np.exp(sc - sc.max(axis=1, keepdims=True))
        p[:, valid] = e / e.sum(axis=1, keepdims=True)
    return p, valid


def attention(cfg: dict, q, k_cache, v_cache, rows=None, heads=None):
    """PR-Sink attention of the current block, float64.

    [digest] pipeline formula: Attn(Q_b, K, V) = softmax(Q_b [K_ref; K_<b]^T / sqrt(d))
    [V_ref; V_<b]; with PR-Sink ([explainer], [abstract]) the keys are those held by the
    bounded cache: ref, static, dynamic and the rolling window (which holds the current block).
    Queries and keys are rotated at their current positions (RoPE follow); the scale uses
    d = head_dim.

    ``q``: ``[L_blk][H][d]`` raw queries; ``k_cache``, ``v_cache``: ``[H][T][d]`` raw,
    slot-indexed.  ``rows`` / ``heads`` restrict the output to some queries / heads.
    Returns ``(out [nrows][nheads][d], lse [nheads][nrows])`` with lse the natural-log
    log-sum-exp of the scaled scores.  With no valid key: out = 0, lse = -inf.
    """
    s = layout_sizes(cfg)
    d = cfg["head_dim"]
    q = np.asarray(q, dtype=np.float64)
    k_cache = np.asarray(k_cache, dtype=np.float64)
    v_cache = np.asarray(v_cache, dtype=np.float64)
    if rows is None:
        rows = np.arange(s["L_blk"])
    rows = np.asarray(rows)
    if heads is None:
        heads = np.arange(cfg["n_heads"])
    kpos, valid = key_positions(cfg)
    qpos = query_positions(cfg)[rows]
    out = np.zeros((len(rows), len(heads), d), dtype=np.float64)
    lse = np.full((len(heads), len(rows)), -np.inf, dtype=np.float64)
    if not valid.any():
        return out, lse
    kp = kpos[valid]
    for hi, h in enumerate(heads):
        qr = rope_rotate(cfg, q[rows, h, :], qpos)
        kr = rope_rotate(cfg, k_cache[h][valid], kp)
        sc = qr @ kr.T / math.sqrt(d)
        m = sc.max(axis=1, keepdims=True)
        e = np.exp(sc - m)
        l = e.sum(axis=1, keepdims=True)
        out[:, hi, :] = (e @ v_cache[h][valid]) / l
        lse[hi] = (m + np.log(l))[:, 0]
    return out, lse


# --------------------------------------------------------------------------------------------
# cache writes
# --------------------------------------------------------------------------------------------

def kv_append(cfg: dict, k_new, v_new, k_cache, v_cache, slot: int):
    """Write a block's raw K/V (token-major ``[n][H][d]``, as a QKV projection emits them) into
    a slot of the head-major caches ``[H][T][d]``; returns the new caches (inputs untouched).

    [digest] pipeline, inference clause: Clean KV Update KV_cache <- KV_cache U Forward(z^0_b,
    t=0, C) is written into the rolling window; keys are cached raw (before RoPE).  The
    rolling slot of block b is b mod R; block 0's clean K/V also fills the static sink
    ([abstract]: the static sink permanently anchors the first generated block).
    """
    a, e = slot_ranges(cfg)[slot]
    k2 = np.array(k_cache, copy=True)
    v2 = np.array(v_cache, copy=True)
    k_new = np.asarray(k_new)
    v_new = np.asarray(v_new)
    assert k_new.shape[0] == e - a and v_new.shape[0] == e - a
    for h in range(cfg["n_heads"]):
        k2[h, a:e, :] = k_new[:, h, :]
        v2[h, a:e, :] = v_new[:, h, :]
    return k2, v2


def dyn_copy(cfg: dict, bank_kv, cache_kv, r: int):
    """Copy bank entry r's K/V into the dynamic-sink slot of every layer.

    [digest] pipeline, inference clause: the retrieved entry's KV is copied into the Dynamic
    Sink.  ``bank_kv``: ``[layers][M][2][H][L_blk][d]``; ``cache_kv``: ``[layers][2][H][T][d]``.
    Returns the new caches.
    """
    a, e = slot_ranges(cfg)[SLOT_DYNAMIC]
    out = np.array(cache_kv, copy=True)
    out[:, :, :, a:e, :] = np.asarray(bank_kv)[:, r]
    return out


def bank_store(cfg: dict, cache_kv, bank_kv, ring_slot: int, bank_slot: int):
    """Store the clean K/V held by ring slot ``ring_slot`` of every layer into bank entry
    ``bank_slot``; returns the new bank.  ([digest] weaknesses, point 3: the bank of M=5 is
    written during the first 20 blocks.)"""
    a, e = slot_ranges(cfg)[SLOT_RING0 + ring_slot]
    out = np.array(bank_kv, copy=True)
    out[:, bank_slot] = np.asarray(cache_kv)[:, :, :, a:e, :]
    return out


# --------------------------------------------------------------------------------------------
# fingerprint, retrieval, bank
# --------------------------------------------------------------------------------------------

def fingerprint(kp, ok) -> np.ndarray:
    """558-d pose fingerprint.

    [digest] pipeline, inference clause: 62 keypoints x 3 frames x 3 values concatenated into a
    558-d l2-normalised vector; [digest] novelty, point 2: confidence channel included, frames
    whose detection failed are zero-filled.  ``kp``: ``[3][62][3]`` (x, y, conf) per frame, in
    that flattening order; ``ok``: ``[3]`` nonzero where detection succeeded.  An all-zero
    vector is returned unchanged (reading).
    """
    kp = np.asarray(kp, dtype=np.float64)
    assert kp.shape == (FP_FRAMES, FP_KEYPOINTS, FP_CHANNELS)
    v = np.zeros(FP_DIM, dtype=np.float64)
    per = FP_KEYPOINTS * FP_CHANNELS
    for f in range(FP_FRAMES):
        if ok[f]:
            v[f * per:(f + 1) * per] = kp[f].reshape(-1)
    n = math.sqrt(float(np.dot(v, v)))
    return v / n if n > 0 else v


def _eligible(bank_src, count, exclude):
    return [i for i in range(int(count)) if int(bank_src[i]) != int(exclude)]


def retrieve(phi_b, bank_phi, bank_src, count: int, exclude: int):
    """r(b) = argmax_i phi_b . phi_i over bank entries whose source block is not ``exclude``.

    [digest] pipeline, inference clause: before generating block b, retrieve the most similar
    bank entry excluding b-1 (already in the window); [digest] novelty, point 2: with
    l2-normalised fingerprints the retrieval is one cosine-maximising dot product.
    Returns ``(r, score)``; ties go to the lowest slot (reading); no eligible entry gives
    ``(-1, -inf)``.
    """
    phi_b = np.asarray(phi_b, dtype=np.float64)
    best, best_s = -1, -np.inf
    for i in _eligible(bank_src, count, exclude):
        sc = float(np.dot(np.asarray(bank_phi[i], dtype=np.float64), phi_b))
        if best < 0 or sc > best_s:
            best, best_s = i, sc
    return best, best_s


def retrieval_margin(phi_b, bank_phi, bank_src, count: int, exclude: int) -> float:
    """Gap between the best and the second-best eligible score (inf with < 2 candidates)."""
    phi_b = np.asarray(phi_b, dtype=np.float64)
    sc = sorted((float(np.dot(np.asarray(bank_phi[i], dtype=np.float64), phi_b))
                 for i in _eligible(bank_src, count, exclude)), reverse=True)
    return sc[0] - sc[1] if len(sc) >= 2 else math.inf


def bank_objective(phis) -> float:
    """Mean similarity inside a bank: mean over unordered pairs i < j of phi_i . phi_j.

    [digest] novelty, point 3: the bank is updated to minimise the mean intra-bank
    similarity (reading: off-diagonal pairs only).
    """
    phis = [np.asarray(p, dtype=np.float64) for p in phis]
    pairs = list(itertools.combinations(range(len(phis)), 2))
    if not pairs:
        return 0.0
    return sum(float(np.dot(phis[i], phis[j])) for i, j in pairs) / len(pairs)


def _bank_options(bank_phi, M, phi_b):
    """Objective of every option: index 0 = keep, index 1 + j = replace slot j."""
    cur = [np.asarray(bank_phi[i], dtype=np.float64) for i in range(M)]
    objs = [bank_objective(cur)]
    for j in range(M):
        cand = list(cur)
        cand[j] = np.asarray(phi_b, dtype=np.float64)
        objs.append(bank_objective(cand))
    return objs


def bank_update(bank_phi, bank_src, count: int, M: int, phi_b, b: int, write_blocks: int):
    """Diversity-driven bank update after block b's Clean KV Update.

    [digest] novelty, point 3: not "replace the oldest" but an exhaustive search over
    replacements minimising the mean intra-bank similarity; [digest] weaknesses, point 3 and
    reproducibility: M = 5, written during the first 20 blocks, then frozen.
    While the bank has a free slot the block is inserted; once full, the options are "keep"
    and "replace slot j" (j < M), the smallest objective wins, ties go to keep and then to the
    lowest j (reading).

    Returns ``(action, bank_phi', bank_src', count')`` with ``action`` the slot written or -1.
    """
    bank_phi = np.array(bank_phi, dtype=np.float64, copy=True)
    bank_src = np.array(bank_src, copy=True)
    if b >= write_blocks:
        return -1, bank_phi, bank_src, count
    if count < M:
        action = count
        count = count + 1
    else:
        objs = _bank_options(bank_phi, M, phi_b)
        best = 0
        for o in range(1, M + 1):
            if objs[o] < objs[best]:
                best = o
        action = best - 1
    if action >= 0:
        bank_phi[action] = np.asarray(phi_b, dtype=np.float64)
        bank_src[action] = b
    return action, bank_phi, bank_src, count


def bank_margin(bank_phi, count: int, M: int, phi_b, b: int, write_blocks: int) -> float:
    """Gap between the best and the second-best option objective (inf when nothing is decided)."""
    if b >= write_blocks or count < M:
        return math.inf
    objs = sorted(_bank_options(bank_phi, M, phi_b))
    return objs[1] - objs[0]


# --------------------------------------------------------------------------------------------
# stream bookkeeping
# --------------------------------------------------------------------------------------------

def valid_mask(cfg: dict, b: int, dyn_valid: bool) -> int:
    """Slots holding data while block b is generated (reading of the pages' per-block flow):
    the ref sink always; the static sink once block 0's clean pass has filled it (b >= 1);
    the dynamic sink when retrieval found an entry; ring slot s when it holds a block >= 0
    (the current block's slot is written before its first attention)."""
    R = cfg["ring_slots"]
    m = 1 << SLOT_REF
    if b >= 1:
        m |= 1 << SLOT_STATIC
    if dyn_valid:
        m |= 1 << SLOT_DYNAMIC
    for s in range(R):
        held = b - R + 1 + ring_rank(s, b, R)
        if held >= 0:
            m |= 1 << (SLOT_RING0 + s)
    return m


def stream_decisions(phis, M: int = 5, write_blocks: int = 20):
    """Decisions of a stream given the per-block fingerprints ``phis[b]``.

    Per block b, in the pages' order ([digest] pipeline, inference clause): retrieve against
    the bank (excluding b-1) and copy the entry into the dynamic sink if it is not already
    there; generate; after the Clean KV Update, update the bank (b < write_blocks).

    Returns a list of dicts with keys r, score, src (source block of the retrieved entry or
    -1), copy (bool), dyn_src, action, count, bank_src, retrieval_margin, bank_margin.
    """
    dim = len(phis[0])
    bank_phi = np.zeros((M, dim), dtype=np.float64)
    bank_src = np.full(M, -1, dtype=np.int64)
    count = 0
    dyn_src = -1
    out = []
    for b, phi in enumerate(phis):
        rm = retrieval_margin(phi, bank_phi, bank_src, count, b - 1)
        r, sc = retrieve(phi, bank_phi, bank_src, count, b - 1)
        src = int(bank_src[r]) if r >= 0 else -1
        copy = r >= 0 and src != dyn_src
        dyn_src = src
        bm = bank_margin(bank_phi, count, M, phi, b, write_blocks)
        action, bank_phi, bank_src, count = bank_update(bank_phi, bank_src, count, M, phi, b,
                                                        write_blocks)
        out.append(dict(r=r, score=sc, src=src, copy=copy, dyn_src=dyn_src, action=action,
                        count=count, bank_src=bank_src.copy(), retrieval_margin=rm,
                        bank_margin=bm))
    return out


# --------------------------------------------------------------------------------------------
# bank policy variants ([digest] weaknesses, points 3 and 5: fixes the digest proposes for a
# frozen bank and for failed pose detection)
# --------------------------------------------------------------------------------------------

def detected_frames(ok) -> int:
    """Number of frames of a block whose pose detection succeeded."""
    return int(sum(1 for x in ok if x))


def retrieve_fallback(phi_b, ok, min_detected: int, bank_phi, bank_src, count: int,
                      exclude: int):
    """Retrieval with the fallback to the Static Sink + window cache.

    [digest] weaknesses, point 5: the fingerprint depends on detection quality and failed frames
    are zero-filled, so retrieval degrades under occlusion; one proposed fix is to fall back to
    the conservative cache of Static Sink + window when detection is missing.  Reading: when
    fewer than ``min_detected`` of the block's frames were detected, no entry is retrieved
    (r = -1, the dynamic sink is empty for the block); otherwise this is ``retrieve``.
    ``min_detected = 0`` never falls back.
    """
    if detected_frames(ok) < min_detected:
        return -1, -np.inf
    return retrieve(phi_b, bank_phi, bank_src, count, exclude)


def fingerprint_distances(phi_b, bank_phi, count: int) -> np.ndarray:
    """Euclidean distance ||phi_b - phi_i|| to every entry in use (float64)."""
    phi_b = np.asarray(phi_b, dtype=np.float64)
    return np.array([math.sqrt(float(np.sum((np.asarray(bank_phi[i], dtype=np.float64)
                                             - phi_b) ** 2))) for i in range(int(count))])


def bank_update_gated(bank_phi, bank_src, count: int, M: int, phi_b, b: int,
                      write_blocks: int, gate: float):
    """Diversity update with a refresh gated on fingerprint distance.

    [digest] weaknesses, point 3: a bank frozen after the first 20 blocks misses states that
    appear later; one proposed fix is to trigger a bank refresh gated on fingerprint distance.
    Reading: for b < write_blocks this is ``bank_update``; afterwards the bank stays frozen
    unless the block is farther than ``gate`` from every entry (min_i ||phi_b - phi_i|| >
    gate), in which case the diversity rule of ``bank_update`` runs for it (insert while the
    bank has room, else keep / replace j, whichever gives the least mean similarity).
    Returns ``(action, bank_phi', bank_src', count')``.
    """
    if b < write_blocks:
        return bank_update(bank_phi, bank_src, count, M, phi_b, b, write_blocks)
    dist = fingerprint_distances(phi_b, bank_phi, count)
    if count > 0 and not float(dist.min()) > gate:
        return -1, np.array(bank_phi, dtype=np.float64, copy=True), np.array(bank_src, copy=True), count
    return bank_update(bank_phi, bank_src, count, M, phi_b, b, b + 1)


def gate_margin(phi_b, bank_phi, count: int, b: int, write_blocks: int, gate: float) -> float:
    """|min distance - gate| (inf when the gate is not consulted)."""
    if b < write_blocks or count == 0:
        return math.inf
    return abs(float(fingerprint_distances(phi_b, bank_phi, count).min()) - gate)


def nearest_entry(phi_b, bank_phi, count: int):
    """argmax_i phi_b . phi_i over the entries in use (ties to the lowest slot): ``(j, score)``,
    ``(-1, -inf)`` for an empty bank."""
    return retrieve(phi_b, bank_phi, np.full(max(int(count), 1), -1, dtype=np.int64), count,
                    exclude=-2)


def nearest_margin(phi_b, bank_phi, count: int) -> float:
    return retrieval_margin(phi_b, bank_phi, np.full(max(int(count), 1), -1, dtype=np.int64),
                            count, exclude=-2)


def blend_weights(alpha: float):
    """The float32 weights of a decayed write: (1 - alpha) for the entry, alpha for the block."""
    a = np.float32(alpha)
    return np.float32(np.float32(1.0) - a), a


def bank_update_decay(bank_phi, bank_src, count: int, M: int, phi_b, b: int,
                      write_blocks: int, alpha: float):
    """Diversity update followed by decay-weighted continuous writes.

    [digest] weaknesses, point 3: instead of freezing the bank after 20 blocks, allow
    continuous writes with decaying weights.  Reading: for b < write_blocks this is
    ``bank_update``; afterwards (alpha > 0) every block is written into the entry nearest to
    it, j = argmax_i phi_b . phi_i, as an exponential moving average: the entry's fingerprint
    becomes the l2-normalised (1 - alpha) phi_j + alpha phi_b and its K/V (1 - alpha) KV_j +
    alpha KV_b (``bank_blend_kv``), so the weight of a write decays by (1 - alpha) with every
    later write; src_j becomes b.  alpha = 0 keeps the bank frozen.
    Returns ``(action, mode, bank_phi', bank_src', count')`` with mode "store" (a block's K/V
    replaces an entry), "blend" or None.
    """
    if b < write_blocks:
        action, bp, bs, c = bank_update(bank_phi, bank_src, count, M, phi_b, b, write_blocks)
        return action, ("store" if action >= 0 else None), bp, bs, c
    bank_phi = np.array(bank_phi, dtype=np.float64, copy=True)
    bank_src = np.array(bank_src, copy=True)
    if not alpha > 0.0 or count == 0:
        return -1, None, bank_phi, bank_src, count
    j, _ = nearest_entry(phi_b, bank_phi, count)
    w_old, w_new = blend_weights(alpha)
    t = float(w_old) * bank_phi[j] + float(w_new) * np.asarray(phi_b, dtype=np.float64)
    n = math.sqrt(float(np.dot(t, t)))
    bank_phi[j] = t / n if n > 0 else t
    bank_src[j] = b
    return j, "blend", bank_phi, bank_src, count


def bank_blend_kv(cfg: dict, cache_kv, bank_kv, ring_slot: int, bank_slot: int, alpha: float):
    """K/V of a decayed write: every element of bank entry ``bank_slot`` (all layers) becomes
    bf16(fl32(fl32(w_old * x) + fl32(w_new * z))) with x the entry's value, z the block's clean
    value in ring slot ``ring_slot`` and (w_old, w_new) = ``blend_weights(alpha)``: each product
    and the sum rounded to float32 (no fused multiply-add), the result rounded to bf16 (nearest
    even).  Returns the new bank as float64 holding bf16 values."""
    import torch
    a, e = slot_ranges(cfg)[SLOT_RING0 + ring_slot]
    w_old, w_new = blend_weights(alpha)
    x = np.asarray(bank_kv)[:, bank_slot].astype(np.float32)
    z = np.asarray(cache_kv)[:, :, :, a:e, :].astype(np.float32)
    y = (x * w_old).astype(np.float32) + (z * w_new).astype(np.float32)
    y16 = torch.from_numpy(np.ascontiguousarray(y.astype(np.float32))).to(torch.bfloat16)
    out = np.array(bank_kv, dtype=np.float64, copy=True)
    out[:, bank_slot] = y16.to(torch.float64).numpy()
    return out


def stream_decisions_policy(phis, oks, M: int = 5, write_blocks: int = 20, policy: str = "frozen",
                            alpha: float = 0.0, gate: float = 0.0, min_detected: int = 0):
    """Decisions of a stream under a bank policy: "frozen" (the pages' rule, as
    ``stream_decisions``), "decay" (``bank_update_decay`` with ``alpha``) or "gated"
    (``bank_update_gated`` with ``gate``); retrieval falls back to Static Sink + window for
    blocks with fewer than ``min_detected`` detected frames (``retrieve_fallback``).

    Returns a list of dicts with keys r, score, src, copy, dyn_src, action, mode, count,
    bank_src, bank_phi and the margins of the decisions taken (retrieval, bank, gate, nearest).
    """
    dim = len(phis[0])
    bank_phi = np.zeros((M, dim), dtype=np.float64)
    bank_src = np.full(M, -1, dtype=np.int64)
    count = 0
    dyn_src = -1
    out = []
    for b, (phi, ok) in enumerate(zip(phis, oks)):
        fallback = detected_frames(ok) < min_detected
        rm = math.inf if fallback else retrieval_margin(phi, bank_phi, bank_src, count, b - 1)
        r, sc = retrieve_fallback(phi, ok, min_detected, bank_phi, bank_src, count, b - 1)
        src = int(bank_src[r]) if r >= 0 else -1
        copy = r >= 0 and src != dyn_src
        dyn_src = src
        bm = bank_margin(bank_phi, count, M, phi, b, write_blocks)
        gm = nm = math.inf
        if policy == "frozen":
            action, bank_phi, bank_src, count = bank_update(bank_phi, bank_src, count, M, phi, b,
                                                            write_blocks)
            mode = "store" if action >= 0 else None
        elif policy == "gated":
            gm = gate_margin(phi, bank_phi, count, b, write_blocks, gate)
            if b >= write_blocks:
                opened = count == 0 or float(fingerprint_distances(phi, bank_phi, count).min()) > gate
                bm = bank_margin(bank_phi, count, M, phi, 0, 1) if opened else math.inf
            action, bank_phi, bank_src, count = bank_update_gated(bank_phi, bank_src, count, M,
                                                                  phi, b, write_blocks, gate)
            mode = "store" if action >= 0 else None
        elif policy == "decay":
            if b >= write_blocks and alpha > 0 and count > 0:
                nm = nearest_margin(phi, bank_phi, count)
            action, mode, bank_phi, bank_src, count = bank_update_decay(
                bank_phi, bank_src, count, M, phi, b, write_blocks, alpha)
        else:
            raise ValueError(policy)
        out.append(dict(r=r, score=sc, src=src, copy=copy, dyn_src=dyn_src, action=action,
                        mode=mode, count=count, bank_src=bank_src.copy(),
                        bank_phi=bank_phi.copy(), retrieval_margin=rm, bank_margin=bm,
                        gate_margin=gm, nearest_margin=nm))
    return out
