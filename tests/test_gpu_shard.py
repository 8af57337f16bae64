"""The head partition on one GPU: calls on head shards (``pose_retrieved_kv_b200/shard.py``)
must reproduce the corresponding heads of the full call bit for bit, for one attention call at
the full workload size and for a whole stream (append, attention, retrieval with the dynamic
fill, bank update and store), with every shard taking the same pose decisions."""
import numpy as np
import pytest
import torch

import oracle
import pose_retrieved_kv_b200 as P
import synth
from pose_retrieved_kv_b200 import shard
from tests._gpu import need_gpu

pytestmark = pytest.mark.gpu


def _attn(cfg, q, k, v):
    s = oracle.layout_sizes(cfg)
    out = torch.empty((s["L_blk"], cfg["n_heads"], cfg["head_dim"]), dtype=torch.bfloat16,
                      device="cuda")
    lse = torch.empty((cfg["n_heads"], s["L_blk"]), dtype=torch.float32, device="cuda")
    P.prsink_attention(P.make_layout(**cfg), q, k, v, out, lse)
    return out, lse


@pytest.mark.parametrize("world", [2, 3, 4])
def test_attention_head_shards_are_bit_identical(world):
    need_gpu()
    cfg = synth.preset("480x480", block_index=1000, valid_mask=0xFF)
    s = oracle.layout_sizes(cfg)
    q = synth.normal_bf16((s["L_blk"], 40, 128), 2, 0).cuda()
    k = synth.normal_bf16((40, s["T"], 128), 2, 1).cuda()
    v = synth.normal_bf16((40, s["T"], 128), 2, 2).cuda()
    out, lse = _attn(cfg, q, k, v)
    outs, lses = [], []
    for r in range(world):
        o, l = _attn(shard.shard_config(cfg, world, r), shard.shard_tokens(q, world, r),
                     shard.shard_heads(k, world, r, 0), shard.shard_heads(v, world, r, 0))
        outs.append(o)
        lses.append(l)
    assert P.prsink_sync_status() == P.PRSINK_OK
    assert torch.equal(shard.gather_heads(outs, 1), out)
    assert torch.equal(shard.gather_heads(lses, 0), lse)


def test_stream_head_shards_reproduce_the_full_stream():
    need_gpu()
    cfg = dict(n_heads=4, head_dim=128, grid_h=5, grid_w=7, frames_per_block=3, ref_frames=1,
               ring_slots=3, rope_mode=3, rope_split=(44, 42, 42), rope_base=10000.0)
    n_layers, n_blocks, world = 2, 25, 2
    full = P.PRSinkStream(cfg, n_layers=n_layers, M=5, write_blocks=20)
    parts = [P.PRSinkStream(shard.shard_config(cfg, world, r), n_layers=n_layers, M=5,
                            write_blocks=20) for r in range(world)]
    s = oracle.layout_sizes(cfg)
    for layer in range(n_layers):
        kr = synth.normal_bf16((s["L_ref"], 4, 128), 50 + layer, 1).cuda()
        full.set_ref(layer, kr, kr)
        for r, st in enumerate(parts):
            st.set_ref(layer, shard.shard_tokens(kr, world, r), shard.shard_tokens(kr, world, r))
    kp, ok, _ = synth.pose_stream(9, n_blocks)
    out = torch.empty((s["L_blk"], 4, 128), dtype=torch.bfloat16, device="cuda")
    outs = [torch.empty((s["L_blk"], 2, 128), dtype=torch.bfloat16, device="cuda")
            for _ in range(world)]
    decided = []
    for b in range(n_blocks):
        kpd = torch.from_numpy(np.ascontiguousarray(kp[b][:, :62])).cuda()
        okd = torch.from_numpy(ok[b]).cuda()
        for st in [full] + parts:
            st.begin_block(kpd, okd)
        for layer in range(n_layers):
            for p in range(4):
                q, kn, vn = (synth.normal_bf16((s["L_blk"], 4, 128), 1000 + 10 * b + p, j).cuda()
                             for j in range(3))
                full.layer_pass(layer, q, kn, vn, out, clean=p == 3)
                for r, st in enumerate(parts):
                    st.layer_pass(layer, shard.shard_tokens(q, world, r),
                                  shard.shard_tokens(kn, world, r),
                                  shard.shard_tokens(vn, world, r), outs[r], clean=p == 3)
                assert torch.equal(shard.gather_heads(outs, 1), out), (b, layer, p)
        for st in [full] + parts:
            st.end_block()
        dec = [(int(st.r.item()), int(st.copied.item()), int(st.dyn_src.item()),
                int(st.action.item()), int(st.bank_count.item())) for st in [full] + parts]
        assert dec[0] == dec[1] == dec[2], (b, dec)
        decided.append(dec[0])
    assert P.prsink_sync_status() == P.PRSINK_OK
    assert torch.equal(shard.gather_heads([st.cache_kv for st in parts], 2), full.cache_kv)
    assert torch.equal(shard.gather_heads([st.bank_kv for st in parts], 3), full.bank_kv)
    assert any(d[0] >= 0 for d in decided) and any(d[3] >= 0 for d in decided)
