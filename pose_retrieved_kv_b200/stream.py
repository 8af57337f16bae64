"""Host-side bookkeeping of a PR-Sink stream on one GPU.

Per block b, in the order the pages give (LiveAnimate digest, pipeline paragraph, inference
clause): fingerprint the incoming poses and retrieve the most similar bank entry (excluding
block b-1) into the dynamic sink; run the denoising passes and the Clean KV Update pass, each
appending the block's raw K/V into ring slot b mod R and attending over the bounded cache;
then (first ``write_blocks`` blocks) update the memory bank with the clean K/V.

Decisions stay on the device: the retrieved slot, whether the dynamic sink was refilled and
the bank action are device scalars read by the copy kernels, and the attention kernel reads
the dynamic sink's source block to know whether that slot holds data.  Nothing here
synchronises with the host.
"""
from __future__ import annotations

import torch

from . import _lib as L


def stream_valid_mask(ring_slots: int, b: int) -> int:
    """Slots that hold data while block b is generated (the dynamic bit is refined on the
    device from the dynamic sink's source block): the ref sink; the static sink from block 1
    on (block 0's clean pass fills it); ring slot s once the block it holds, b-R+1+age(s),
    is >= 0."""
    R = ring_slots
    m = (1 << L.SLOT_REF) | (1 << L.SLOT_DYNAMIC)
    if b >= 1:
        m |= 1 << L.SLOT_STATIC
    oldest = b - R + 1
    for s in range(R):
        if oldest + (s - oldest) % R >= 0:
            m |= 1 << (L.SLOT_RING0 + s)
    return m


class PRSinkStream:
    """Caches, bank and decisions of one stream for ``n_layers`` attention layers.

    Nothing here synchronises, so a bounded device wait that ran out (the attention kernel
    then writes zeros for the affected rows and records a timeout in the device status word)
    is not noticed by these calls: check once per block, with ``end_block(check=True)`` or
    ``check_status()``, which synchronise the stream and raise ``PRSinkError`` on a timeout.
    """

    def __init__(self, cfg: dict, n_layers: int, M: int = 5, write_blocks: int = 20,
                 device="cuda", policy: str = "frozen", alpha: float = 0.0, gate: float = 0.0,
                 min_detected: int = 0, fused: bool = False):
        """``policy``, ``alpha``, ``gate``: the bank policy (the pages' frozen bank, or one of
        the variants of ``prsink_bank_update_policy``); ``min_detected`` > 0 makes retrieval
        fall back to Static Sink + window for blocks with fewer detected frames.  ``fused``:
        each layer keeps a rotated copy of its sink keys, refreshed once per block by
        ``prsink_rotate_sinks``, and every pass is one ``prsink_attention_fused`` launch (the
        append folded in) instead of an append and a ``prsink_attention`` launch."""
        self.cfg = dict(cfg)
        self.n_layers, self.M, self.write_blocks = int(n_layers), int(M), int(write_blocks)
        self.policy = L.make_policy(policy, write_blocks, alpha, gate)
        self.min_detected = int(min_detected)
        self.R = int(cfg["ring_slots"])
        lay = L.make_layout(**{**self.cfg, "block_index": 0, "valid_mask": 0})
        self.L_f, self.L_blk, self.L_ref, self.T = L.prsink_layout_tokens(lay)
        H, d = int(cfg["n_heads"]), int(cfg["head_dim"])
        dev = torch.device(device)
        bf = torch.bfloat16
        self.cache_kv = torch.zeros((n_layers, 2, H, self.T, d), dtype=bf, device=dev)
        self.bank_kv = torch.zeros((n_layers, M, 2, H, self.L_blk, d), dtype=bf, device=dev)
        self.bank_phi = torch.zeros((M, L.FP_DIM), dtype=torch.float32, device=dev)
        self.bank_src = torch.full((M,), -1, dtype=torch.int64, device=dev)
        self.bank_count = torch.zeros(1, dtype=torch.int32, device=dev)
        self.dyn_src = torch.full((1,), -1, dtype=torch.int64, device=dev)
        self.phi = torch.zeros(L.FP_DIM, dtype=torch.float32, device=dev)
        self.r = torch.zeros(1, dtype=torch.int32, device=dev)
        self.score = torch.zeros(1, dtype=torch.float32, device=dev)
        self.copied = torch.zeros(1, dtype=torch.int32, device=dev)
        self.action = torch.zeros(1, dtype=torch.int32, device=dev)
        self.mode = torch.zeros(1, dtype=torch.int32, device=dev)
        self.frame_ok = torch.ones(3, dtype=torch.uint8, device=dev)
        # the last wave split over the key range when the device's SMs leave it nearly empty
        # (few heads per GPU, the 3024-query layouts); scratch for the split partials
        n = L.prsink_attention_scratch_bytes(lay)
        self.scratch = torch.empty(n, dtype=torch.uint8, device=dev) if n > 0 else None
        self.fused = bool(fused)
        self.k_rot = (torch.zeros((n_layers, H, self.T, d), dtype=bf, device=dev)
                      if self.fused else None)
        self._rot_pending = [0] * self.n_layers     # ref / static slots written since rotated
        self._rot_block = [-1] * self.n_layers      # block of each layer's last rotation pass
        self.b = 0

    def reset(self):
        """Start a new stream at block 0 on the same buffers: empty bank, empty dynamic sink.
        The ref sink keeps its K/V; other slots are marked empty until written (their stale
        bytes are never read)."""
        self.bank_phi.zero_()
        self.bank_src.fill_(-1)
        self.bank_count.zero_()
        self.dyn_src.fill_(-1)
        self._rot_block = [-1] * self.n_layers
        self.b = 0

    def layout(self, b: int = None) -> L.Layout:
        b = self.b if b is None else b
        return L.make_layout(**{**self.cfg, "block_index": b,
                                "valid_mask": stream_valid_mask(self.R, b)})

    def kv(self, layer: int):
        return self.cache_kv[layer, 0], self.cache_kv[layer, 1]

    def set_ref(self, layer: int, k_ref, v_ref, stream=None):
        k, v = self.kv(layer)
        L.prsink_kv_append(self.layout(), k_ref, v_ref, k, v, L.SLOT_REF, stream)
        self.mark_written(layer, L.SLOT_REF)

    def begin_block(self, kp, frame_ok, stream=None):
        """Fingerprint (kp f32 [3][62][3], frame_ok u8 [3], on the device) and retrieval."""
        L.prsink_fingerprint(kp, frame_ok, self.phi, stream)
        if self.min_detected > 0:
            L.prsink_retrieve_fallback(self.layout(), self.phi, frame_ok, self.min_detected,
                                       self.bank_phi, self.bank_src, self.bank_count, self.M,
                                       self.b - 1, self.r, self.score, self.copied,
                                       self.dyn_src, self.bank_kv, self.cache_kv,
                                       self.n_layers, stream)
            return
        L.prsink_retrieve(self.layout(), self.phi, self.bank_phi, self.bank_src,
                          self.bank_count, self.M, self.b - 1, self.r, self.score, self.copied,
                          self.dyn_src, self.bank_kv, self.cache_kv, self.n_layers, stream)

    def mark_written(self, layer: int, slot: int):
        """Fused mode: a fixed-position slot (ref, static) of ``layer`` was written outside
        ``layer_pass``; its rotated copy is refreshed by the next ``prepare_layer``."""
        self._rot_pending[layer] |= 1 << int(slot)

    def prepare_layer(self, layer: int, stream=None):
        """Fused mode: refresh the layer's rotated sink keys once per block (ring slots move one
        rank per block; the dynamic slot when retrieval refilled it; ref and static once after
        they were written).  Called by ``layer_pass``; a no-op when unfused or already done."""
        if not self.fused or self._rot_block[layer] == self.b:
            return
        k, _ = self.kv(layer)
        ring = ((1 << self.R) - 1) << L.SLOT_RING0
        mask = ring | (1 << L.SLOT_DYNAMIC) | self._rot_pending[layer]
        L.prsink_rotate_sinks(self.layout(), k, self.k_rot[layer], mask, self.copied,
                              self.dyn_src, stream)
        self._rot_pending[layer] = 0
        self._rot_block[layer] = self.b

    def layer_pass(self, layer: int, q, k_new, v_new, out, lse=None, clean: bool = False,
                   stream=None):
        """Append this pass's raw K/V into ring slot b mod R (and, on block 0's clean pass,
        into the static sink), then attend."""
        lay = self.layout()
        k, v = self.kv(layer)
        if self.fused:
            self.prepare_layer(layer, stream)
            L.prsink_attention_fused(lay, q, k_new, v_new, self.k_rot[layer], k, v, out, lse,
                                     self.dyn_src, stream, scratch=self.scratch)
            if clean and self.b == 0:
                L.prsink_kv_append(lay, k_new, v_new, k, v, L.SLOT_STATIC, stream)
                self.mark_written(layer, L.SLOT_STATIC)
            return
        L.prsink_kv_append(lay, k_new, v_new, k, v, L.SLOT_RING0 + self.b % self.R, stream)
        if clean and self.b == 0:
            L.prsink_kv_append(lay, k_new, v_new, k, v, L.SLOT_STATIC, stream)
        if self.scratch is not None:
            L.prsink_attention_split(lay, q, k, v, out, self.scratch, lse, self.dyn_src, stream)
        else:
            L.prsink_attention(lay, q, k, v, out, lse, self.dyn_src, stream)

    def end_block(self, stream=None, check: bool = False):
        """Bank update with the clean K/V of block b, then advance to block b+1.  With
        ``check`` the stream is synchronised and a device timeout raises."""
        if self.policy.kind == L.BANK_FROZEN:
            L.prsink_bank_update(self.layout(), self.bank_phi, self.bank_src, self.bank_count,
                                 self.M, self.phi, self.b, self.write_blocks, self.action,
                                 self.cache_kv, self.bank_kv, self.n_layers, stream)
        else:
            L.prsink_bank_update_policy(self.layout(), self.policy, self.bank_phi,
                                        self.bank_src, self.bank_count, self.M, self.phi,
                                        self.b, self.action, self.mode, self.cache_kv,
                                        self.bank_kv, self.n_layers, stream)
        self.b += 1
        if check:
            self.check_status(stream)

    @staticmethod
    def check_status(stream=None):
        """Synchronise ``stream`` and raise ``PRSinkError`` if a bounded device wait ran out
        (on any stream of this device) since the status word was last read."""
        rc = L.prsink_sync_status(stream)
        if rc != L.PRSINK_OK:
            raise L.PRSinkError(rc, "PRSinkStream", L.prsink_last_error())
