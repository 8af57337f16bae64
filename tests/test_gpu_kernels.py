"""GPU parity of the KV append, fingerprint, retrieval (+ dynamic-sink fill) and bank update
(+ bank store) against the oracle, through the C ABI.  Cache and bank bytes, slot indices and
bank decisions must match bit for bit; fingerprints and similarity scores within float32
rounding."""
import numpy as np
import pytest
import torch

import oracle
import pose_retrieved_kv_b200 as P
import synth
from tests._gpu import f64, need_gpu

pytestmark = pytest.mark.gpu


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy()


# head_dim 32 (4 chunks per row) takes the generic chunk-indexed kernel, 64 and 128 the
# row-tiled one; the odd grids leave ragged last token blocks
APPEND_EXTRA = {
    "d32_5x7": dict(n_heads=3, head_dim=32, grid_h=5, grid_w=7, frames_per_block=3, ref_frames=1,
                    ring_slots=3, rope_mode=3, rope_split=(12, 10, 10), rope_base=10000.0),
    "d64_9x5": dict(n_heads=2, head_dim=64, grid_h=9, grid_w=5, frames_per_block=2, ref_frames=1,
                    ring_slots=2, rope_mode=3, rope_split=(24, 20, 20), rope_base=10000.0),
}


@pytest.mark.parametrize("name", ["tiny", "480x480", "384x672_r4", "d32_5x7", "d64_9x5"])
def test_kv_append_bit_exact_all_slots(name):
    need_gpu()
    if name in APPEND_EXTRA:
        cfg = dict(APPEND_EXTRA[name], block_index=5, valid_mask=0xFF)
    else:
        cfg = synth.preset(name, block_index=5, valid_mask=0xFF)
    s = oracle.layout_sizes(cfg)
    H, d, T = cfg["n_heads"], cfg["head_dim"], s["T"]
    lay = P.make_layout(**cfg)
    k = synth.normal_bf16((H, T, d), 1, 1)
    v = synth.normal_bf16((H, T, d), 1, 2)
    kd, vd = k.cuda(), v.cuda()
    # guard bands around the caches must stay untouched
    guard = 4096
    kbuf = torch.full((H * T * d + 2 * guard,), 7.0, dtype=torch.bfloat16, device="cuda")
    kbuf[guard:guard + H * T * d] = kd.reshape(-1)
    kview = kbuf[guard:guard + H * T * d].view(H, T, d)
    kr, vr = f64(k), f64(v)
    for slot in range(3 + cfg["ring_slots"]):
        n = s["L_ref"] if slot == 0 else s["L_blk"]
        kn = synth.normal_bf16((n, H, d), 2, 10 + slot)
        vn = synth.normal_bf16((n, H, d), 2, 20 + slot)
        P.prsink_kv_append(lay, kn.cuda(), vn.cuda(), kview, vd, slot)
        kr, vr = oracle.kv_append(cfg, f64(kn), f64(vn), kr, vr, slot)
    torch.cuda.synchronize()
    assert np.array_equal(f64(kview), kr) and np.array_equal(f64(vd), vr)
    assert torch.all(kbuf[:guard] == 7.0) and torch.all(kbuf[-guard:] == 7.0)


def test_fingerprint_matches_oracle():
    need_gpu()
    for seed in range(6):
        kp, ok = synth.keypoints(seed, n_kp=62)
        if seed == 4:
            ok[:] = 0                                  # every detection failed
        if seed == 5:
            ok[:] = [0, 1, 0]
        phi = torch.empty(558, dtype=torch.float32, device="cuda")
        P.prsink_fingerprint(torch.from_numpy(kp).cuda(), torch.from_numpy(ok).cuda(), phi)
        ref = oracle.fingerprint(kp, ok)
        got = f64(phi)
        assert np.max(np.abs(got - ref)) <= 1e-7
        if not ok.any():
            assert np.all(got == 0)


def _bank(seed, M, n_valid, sim=0.0):
    g = np.random.default_rng(seed)
    base = g.standard_normal(558)
    x = g.standard_normal((M, 558)) + sim * base
    x /= np.linalg.norm(x, axis=1, keepdims=True)
    x[n_valid:] = 0
    return x.astype(np.float32)


@pytest.mark.parametrize("seed", range(12))
def test_retrieve_decision_and_dynamic_fill(seed):
    need_gpu()
    g = np.random.default_rng(seed)
    M = [5, 5, 5, 3, 8, 32][seed % 6]
    count = int(g.integers(0, M + 1)) if seed % 4 else M
    src = g.permutation(1000)[:M].astype(np.int64)
    exclude = int(src[g.integers(0, M)]) if seed % 3 else -7
    for attempt in range(50):     # oracle on the very same float32 values; a decided case
        bank = _bank(1000 * seed + attempt, M, count, sim=2.0)
        phi = _bank(100 + 1000 * seed + attempt, 1, 1)[0] * 0.5 + bank[max(count, 1) - 1]
        phi = (phi / np.linalg.norm(phi)).astype(np.float32)
        margin = oracle.retrieval_margin(phi, bank, src, count, exclude)
        if margin >= 1e-4:
            break
    assert margin >= 1e-4
    r_ref, sc_ref = oracle.retrieve(phi, bank, src, count, exclude)
    cfg = synth.preset("tiny", block_index=9, valid_mask=0xFF)
    s = oracle.layout_sizes(cfg)
    n_layers = 3
    cache = synth.normal_bf16((n_layers, 2, 1, s["T"], 64), seed, 1).cuda()
    bank_kv = synth.normal_bf16((n_layers, M, 2, 1, s["L_blk"], 64), seed, 2).cuda()
    cache0 = f64(cache)
    old_src = int(src[r_ref]) if (r_ref >= 0 and seed % 2) else 123456
    dev = dict(r=torch.zeros(1, dtype=torch.int32, device="cuda"),
               sc=torch.zeros(1, dtype=torch.float32, device="cuda"),
               cp=torch.zeros(1, dtype=torch.int32, device="cuda"),
               dyn=torch.tensor([old_src], dtype=torch.int64, device="cuda"))
    P.prsink_retrieve(P.make_layout(**cfg), torch.from_numpy(phi).cuda(),
                      torch.from_numpy(bank).cuda(), torch.from_numpy(src).cuda(),
                      torch.tensor([count], dtype=torch.int32, device="cuda"), M, exclude,
                      dev["r"], dev["sc"], dev["cp"], dev["dyn"], bank_kv, cache, n_layers)
    torch.cuda.synchronize()
    r = int(dev["r"].item())
    assert r == r_ref
    expect_copy = r_ref >= 0 and int(src[r_ref]) != old_src
    assert bool(dev["cp"].item()) == expect_copy
    assert int(dev["dyn"].item()) == (int(src[r_ref]) if r_ref >= 0 else -1)
    if r_ref >= 0:
        assert abs(float(dev["sc"].item()) - sc_ref) <= 1e-6
    else:
        assert float(dev["sc"].item()) == -np.inf
    want = oracle.dyn_copy(cfg, f64(bank_kv), cache0, r_ref) if expect_copy else cache0
    assert np.array_equal(f64(cache), want)


@pytest.mark.parametrize("seed", range(16))
def test_bank_update_decision_and_store(seed):
    need_gpu()
    g = np.random.default_rng(seed)
    M = [5, 5, 5, 4, 7, 32][seed % 6]
    count = M if seed % 4 else int(g.integers(0, M))
    b = int(g.integers(0, 25))
    write_blocks = 20
    for attempt in range(50):
        bank = _bank(1000 * seed + attempt, M, count, sim=1.5)
        cand = _bank(5000 + 1000 * seed + attempt, 1, 1, sim=1.5)[0]
        if oracle.bank_margin(bank, count, M, cand, b, write_blocks) >= 1e-4:
            break
    src = np.where(np.arange(M) < count, g.permutation(100)[:M], -1).astype(np.int64)
    act_ref, bphi_ref, bsrc_ref, cnt_ref = oracle.bank_update(bank, src, count, M, cand, b,
                                                              write_blocks)
    cfg = synth.preset("tiny", block_index=b, valid_mask=0xFF)
    s = oracle.layout_sizes(cfg)
    n_layers = 2
    cache = synth.normal_bf16((n_layers, 2, 1, s["T"], 64), seed, 3).cuda()
    bank_kv = synth.normal_bf16((n_layers, M, 2, 1, s["L_blk"], 64), seed, 4).cuda()
    bank0 = f64(bank_kv)
    d_phi = torch.from_numpy(bank).cuda()
    d_src = torch.from_numpy(src).cuda()
    d_cnt = torch.tensor([count], dtype=torch.int32, device="cuda")
    d_act = torch.zeros(1, dtype=torch.int32, device="cuda")
    P.prsink_bank_update(P.make_layout(**cfg), d_phi, d_src, d_cnt, M,
                         torch.from_numpy(cand).cuda(), b, write_blocks, d_act, cache, bank_kv,
                         n_layers)
    torch.cuda.synchronize()
    assert int(d_act.item()) == act_ref
    assert int(d_cnt.item()) == cnt_ref
    assert np.array_equal(d_src.cpu().numpy(), bsrc_ref)
    assert np.array_equal(f64(d_phi), bphi_ref.astype(np.float32).astype(np.float64))
    want = (oracle.bank_store(cfg, f64(cache), bank0, b % cfg["ring_slots"], act_ref)
            if act_ref >= 0 else bank0)
    assert np.array_equal(f64(bank_kv), want)


def test_bounded_wait_reports_timeout_and_recovers():
    """A wait on a barrier nothing signals gives up after its limit; the status word reports
    it once, and the context keeps working."""
    need_gpu()
    P.prsink_debug_wait_timeout(2_000_000)             # 2 ms
    assert P.prsink_sync_status() == P.PRSINK_ERR_TIMEOUT
    assert P.prsink_sync_status() == P.PRSINK_OK       # cleared
    cfg = synth.preset("tiny", block_index=7, valid_mask=0xFF)
    q = torch.zeros((48, 1, 64), dtype=torch.bfloat16, device="cuda")
    k = torch.ones((1, 256, 64), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    P.prsink_attention(P.make_layout(**cfg), q, k, k, out)
    assert P.prsink_sync_status() == P.PRSINK_OK
    assert torch.all(out == 1)


def test_launch_counter_counts_kernels():
    need_gpu()
    cfg = synth.preset("tiny", block_index=7, valid_mask=0xFF)
    q = torch.zeros((48, 1, 64), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 256, 64), dtype=torch.bfloat16, device="cuda")
    n0 = P.prsink_launch_count()
    P.prsink_attention(P.make_layout(**cfg), q, k, k, torch.empty_like(q))
    P.prsink_kv_append(P.make_layout(**cfg), q, q, k, k, 3)
    torch.cuda.synchronize()
    assert P.prsink_launch_count() == n0 + 2


def test_attention_abort_path_reports_timeout_and_recovers():
    """The attention kernel's own abort path: a one-shot self-test makes the MMA issuer withhold
    one commit, so the softmax wait runs out after 2 ms.  The kernel must record the timeout,
    drain its copies and MMAs, free its tensor memory and write out = 0, lse = -inf; the next
    normal call must match the oracle."""
    need_gpu()
    from tests._gpu import attention_inputs, check_attention
    cfg = synth.preset("tiny", block_index=7, valid_mask=0xFF)
    q, k, v = attention_inputs(cfg, seed=31)
    lay = P.make_layout(**cfg)
    out = torch.full((48, 1, 64), 5.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 48), dtype=torch.float32, device="cuda")
    assert P.prsink_sync_status() == P.PRSINK_OK
    P.prsink_debug_attention_stall(2_000_000)
    P.prsink_attention(lay, q.cuda(), k.cuda(), v.cuda(), out, lse)
    assert P.prsink_sync_status() == P.PRSINK_ERR_TIMEOUT
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
    P.prsink_attention(lay, q.cuda(), k.cuda(), v.cuda(), out, lse)
    assert P.prsink_sync_status() == P.PRSINK_OK
    ref, _ = oracle.attention(cfg, f64(q), f64(k), f64(v))
    check_attention(f64(out), ref, "after the abort")
