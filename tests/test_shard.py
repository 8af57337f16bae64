"""Head partition of the path over ranks (``pose_retrieved_kv_b200/shard.py``), on the CPU.

Two gloo ranks (one process each, as torchrun would start them) each take their heads of the
same seeded 40-head inputs through the package's partition helpers and run the oracle on their
shard with a layout of h1 - h0 heads; rank 0 gathers the shards and the concatenation must
equal the oracle's 40-head result exactly (heads are independent in every step).  Both ranks
also compute the pose decisions of a stream (retrieval, dynamic fill, bank action) from the
same inputs: the replicated decisions must be identical."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# 40 heads of 64 over a small 4x5 grid: the pages' head count at a size the oracle runs fast
CFG40 = dict(n_heads=40, head_dim=64, grid_h=4, grid_w=5, frames_per_block=3, ref_frames=1,
             ring_slots=3, rope_mode=3, rope_split=(24, 20, 20), rope_base=10000.0,
             block_index=11, valid_mask=0b111011)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _full_inputs():
    import oracle
    import synth
    s = oracle.layout_sizes(CFG40)
    q = synth.normal_bf16((s["L_blk"], 40, 64), 31, 0)
    k = synth.normal_bf16((40, s["T"], 64), 31, 1)
    v = synth.normal_bf16((40, s["T"], 64), 31, 2)
    kn = synth.normal_bf16((s["L_blk"], 40, 64), 31, 3)
    vn = synth.normal_bf16((s["L_blk"], 40, 64), 31, 4)
    return q, k, v, kn, vn


def _decisions(n_blocks=26):
    import oracle
    import synth
    kp, ok, _ = synth.pose_stream(5, n_blocks)
    phis = [oracle.fingerprint(kp[b][:, :62], ok[b]).astype(np.float32) for b in range(n_blocks)]
    return [(d["r"], d["copy"], d["dyn_src"], d["action"], d["count"])
            for d in oracle.stream_decisions(phis, M=5, write_blocks=20)]


def _worker(rank: int, world: int, port: int, results):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        import oracle
        from pose_retrieved_kv_b200 import shard
        q, k, v, kn, vn = _full_inputs()
        cfg = shard.shard_config(CFG40, world, rank)
        f64 = lambda t: t.to(torch.float64).numpy()       # noqa: E731
        # this rank's heads: the Clean KV Update append, then attention over the shard
        ring = oracle.SLOT_RING0 + CFG40["block_index"] % CFG40["ring_slots"]
        ks, vs = oracle.kv_append(cfg, f64(shard.shard_tokens(kn, world, rank)),
                                  f64(shard.shard_tokens(vn, world, rank)),
                                  f64(shard.shard_heads(k, world, rank, 0)),
                                  f64(shard.shard_heads(v, world, rank, 0)), ring)
        out, lse = oracle.attention(cfg, f64(shard.shard_tokens(q, world, rank)), ks, vs)
        parts = {"out": torch.from_numpy(np.ascontiguousarray(out)),
                 "lse": torch.from_numpy(np.ascontiguousarray(lse)),
                 "k": torch.from_numpy(ks), "v": torch.from_numpy(vs)}
        gathered = {}
        for name, t in parts.items():
            objs = [None] * world
            dist.all_gather_object(objs, t)
            gathered[name] = objs
        dec = [None] * world
        dist.all_gather_object(dec, _decisions())
        if rank == 0:
            results["out"] = shard.gather_heads(gathered["out"], 1).numpy()
            results["lse"] = shard.gather_heads(gathered["lse"], 0).numpy()
            results["k"] = shard.gather_heads(gathered["k"], 0).numpy()
            results["v"] = shard.gather_heads(gathered["v"], 0).numpy()
            results["dec"] = dec
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_head_shards_equal_the_full_oracle():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, results))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(300)
            assert p.exitcode == 0
        res = dict(results)
    sys.path.insert(0, ROOT)
    import oracle
    q, k, v, kn, vn = _full_inputs()
    f64 = lambda t: t.to(torch.float64).numpy()            # noqa: E731
    ring = oracle.SLOT_RING0 + CFG40["block_index"] % CFG40["ring_slots"]
    kf, vf = oracle.kv_append(CFG40, f64(kn), f64(vn), f64(k), f64(v), ring)
    out, lse = oracle.attention(CFG40, f64(q), kf, vf)
    assert np.array_equal(res["k"], kf) and np.array_equal(res["v"], vf)
    assert np.array_equal(res["out"], out) and np.array_equal(res["lse"], lse)
    d0, d1 = res["dec"]
    assert d0 == d1 == _decisions()
    assert any(x[0] >= 0 for x in d0) and any(x[3] >= 0 for x in d0)


@pytest.mark.parametrize("H,world", [(40, 1), (40, 2), (40, 3), (40, 8), (7, 3), (5, 5)])
def test_head_ranges_tile_the_heads(H, world):
    from pose_retrieved_kv_b200 import shard
    ranges = [shard.head_range(H, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == H
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    sizes = [h1 - h0 for h0, h1 in ranges]
    assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1


def test_head_range_rejects_bad_splits():
    from pose_retrieved_kv_b200 import shard
    with pytest.raises(ValueError):
        shard.head_range(4, 8, 0)
    with pytest.raises(ValueError):
        shard.head_range(40, 2, 2)


def test_shard_and_gather_round_trip():
    from pose_retrieved_kv_b200 import shard
    x = torch.arange(5 * 40 * 3).reshape(5, 40, 3)
    assert torch.equal(shard.gather_heads([shard.shard_tokens(x, 3, r) for r in range(3)], 1), x)
    c = torch.arange(2 * 40 * 6 * 3).reshape(2, 40, 6, 3)
    assert torch.equal(shard.gather_heads([shard.shard_heads(c, 4, r, 1) for r in range(4)], 1), c)
