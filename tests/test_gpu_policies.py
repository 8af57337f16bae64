"""GPU parity of the bank policy variants against the oracle (through the C ABI): the
retrieval fallback to Static Sink + window, the distance-gated refresh and the decay-weighted
continuous writes.  Decisions, slot indices and K/V bytes bit for bit (the decayed K/V write
is specified to the float32 rounding of each step); blended fingerprints within float32
rounding; every decision drawn with a margin."""
import itertools

import numpy as np
import pytest
import torch

import oracle
import pose_retrieved_kv_b200 as P
import synth
from tests._gpu import check_attention, f64, need_gpu

pytestmark = pytest.mark.gpu

MARGIN = 1e-4


def _unit_rows(g, n):
    x = g.standard_normal((n, 558))
    return (x / np.linalg.norm(x, axis=1, keepdims=True)).astype(np.float32)


def _dev(**kw):
    out = {}
    for k, (dt, v) in kw.items():
        out[k] = torch.tensor(v, dtype=dt, device="cuda")
    return out


@pytest.mark.parametrize("min_detected", range(4))
def test_retrieve_fallback_every_detection_pattern(min_detected):
    need_gpu()
    g = np.random.default_rng(40 + min_detected)
    cfg = synth.preset("tiny", block_index=9, valid_mask=0xFF)
    s = oracle.layout_sizes(cfg)
    n_layers, M = 2, 5
    for ok in itertools.product([0, 1], repeat=3):
        for attempt in range(50):
            bank = _unit_rows(g, M)
            phi = _unit_rows(g, 1)[0]
            src = np.arange(10, 10 + M, dtype=np.int64)
            if oracle.retrieval_margin(phi, bank, src, M, -1) >= MARGIN:
                break
        r_ref, _ = oracle.retrieve_fallback(phi, ok, min_detected, bank, src, M, -1)
        cache = synth.normal_bf16((n_layers, 2, 1, s["T"], 64), 7, 1).cuda()
        bank_kv = synth.normal_bf16((n_layers, M, 2, 1, s["L_blk"], 64), 7, 2).cuda()
        cache0 = f64(cache)
        d = _dev(r=(torch.int32, [0]), sc=(torch.float32, [0.0]), cp=(torch.int32, [0]),
                 dyn=(torch.int64, [99]))
        P.prsink_retrieve_fallback(P.make_layout(**cfg), torch.from_numpy(phi).cuda(),
                                   torch.tensor(ok, dtype=torch.uint8, device="cuda"),
                                   min_detected, torch.from_numpy(bank).cuda(),
                                   torch.from_numpy(src).cuda(),
                                   torch.tensor([M], dtype=torch.int32, device="cuda"), M, -1,
                                   d["r"], d["sc"], d["cp"], d["dyn"], bank_kv, cache, n_layers)
        torch.cuda.synchronize()
        assert int(d["r"].item()) == r_ref, (ok, min_detected)
        if r_ref < 0:
            assert int(d["cp"].item()) == 0 and int(d["dyn"].item()) == -1
            assert np.array_equal(f64(cache), cache0)
        else:
            assert int(d["cp"].item()) == 1 and int(d["dyn"].item()) == int(src[r_ref])
            assert np.array_equal(f64(cache), oracle.dyn_copy(cfg, f64(bank_kv), cache0, r_ref))


def _policy_call(cfg, pol, bank, src, count, M, phi, b, cache, bank_kv, n_layers):
    d = _dev(act=(torch.int32, [7]), mode=(torch.int32, [7]))
    d_phi = torch.from_numpy(bank).cuda()
    d_src = torch.from_numpy(src).cuda()
    d_cnt = torch.tensor([count], dtype=torch.int32, device="cuda")
    P.prsink_bank_update_policy(P.make_layout(**cfg), pol, d_phi, d_src, d_cnt, M,
                                torch.from_numpy(phi).cuda(), b, d["act"], d["mode"], cache,
                                bank_kv, n_layers)
    torch.cuda.synchronize()
    return (int(d["act"].item()), int(d["mode"].item()), f64(d_phi), d_src.cpu().numpy(),
            int(d_cnt.item()))


@pytest.mark.parametrize("seed", range(8))
def test_gated_refresh_decision_and_store(seed):
    need_gpu()
    g = np.random.default_rng(seed)
    M, n_layers, write_blocks = 5, 2, 20
    gate = 1.3
    b = 20 + int(g.integers(0, 10)) if seed % 4 else int(g.integers(0, 20))
    for attempt in range(100):
        base = _unit_rows(g, 1)[0].astype(np.float64)
        bank = base + [0.3, 0.6, 0.9][attempt % 3] * g.standard_normal((M, 558)) / np.sqrt(558)
        bank = (bank / np.linalg.norm(bank, axis=1, keepdims=True)).astype(np.float32)
        cand = _unit_rows(g, 1)[0] if seed % 2 else (bank[0] + 0.5 * _unit_rows(g, 1)[0])
        cand = (cand / np.linalg.norm(cand)).astype(np.float32)
        if (oracle.gate_margin(cand, bank, M, b, write_blocks, gate) >= MARGIN
                and oracle.bank_margin(bank, M, M, cand, 0, 1) >= MARGIN):
            break
    src = np.arange(M, dtype=np.int64)
    act_ref, phi_ref, src_ref, cnt_ref = oracle.bank_update_gated(bank, src, M, M, cand, b,
                                                                  write_blocks, gate)
    cfg = synth.preset("tiny", block_index=b, valid_mask=0xFF)
    s = oracle.layout_sizes(cfg)
    cache = synth.normal_bf16((n_layers, 2, 1, s["T"], 64), seed, 3).cuda()
    bank_kv = synth.normal_bf16((n_layers, M, 2, 1, s["L_blk"], 64), seed, 4).cuda()
    bank0 = f64(bank_kv)
    pol = P.make_policy("gated", write_blocks, gate=gate)
    act, mode, phi_g, src_g, cnt = _policy_call(cfg, pol, bank, src, M, M, cand, b, cache,
                                                bank_kv, n_layers)
    assert act == act_ref and cnt == cnt_ref
    assert mode == (P.BANK_MODE_STORE if act_ref >= 0 else P.BANK_MODE_NONE)
    assert np.array_equal(src_g, src_ref)
    assert np.array_equal(phi_g, phi_ref.astype(np.float32).astype(np.float64))
    want = (oracle.bank_store(cfg, f64(cache), bank0, b % 3, act_ref) if act_ref >= 0 else bank0)
    assert np.array_equal(f64(bank_kv), want)


@pytest.mark.parametrize("seed,alpha", [(0, 0.25), (1, 0.5), (2, 1.0), (3, 0.1), (4, 0.0),
                                        (5, 0.25)])
def test_decayed_write_decision_and_blend(seed, alpha):
    need_gpu()
    g = np.random.default_rng(100 + seed)
    M, n_layers, write_blocks = 5, 2, 20
    b = 20 + seed if seed != 5 else 7                       # seed 5: before the freeze
    for attempt in range(100):
        bank = _unit_rows(g, M)
        cand = (bank[seed % M] + 0.7 * _unit_rows(g, 1)[0])
        cand = (cand / np.linalg.norm(cand)).astype(np.float32)
        if (oracle.nearest_margin(cand, bank, M) >= MARGIN
                and oracle.bank_margin(bank, M, M, cand, b, write_blocks) >= MARGIN):
            break
    src = np.arange(M, dtype=np.int64)
    act_ref, mode_ref, phi_ref, src_ref, cnt_ref = oracle.bank_update_decay(
        bank, src, M, M, cand, b, write_blocks, alpha)
    cfg = synth.preset("tiny", block_index=b, valid_mask=0xFF)
    s = oracle.layout_sizes(cfg)
    cache = synth.normal_bf16((n_layers, 2, 1, s["T"], 64), seed, 5).cuda()
    bank_kv = synth.normal_bf16((n_layers, M, 2, 1, s["L_blk"], 64), seed, 6).cuda()
    bank0 = f64(bank_kv)
    pol = P.make_policy("decay", write_blocks, alpha=alpha)
    act, mode, phi_g, src_g, cnt = _policy_call(cfg, pol, bank, src, M, M, cand, b, cache,
                                                bank_kv, n_layers)
    modes = {None: P.BANK_MODE_NONE, "store": P.BANK_MODE_STORE, "blend": P.BANK_MODE_BLEND}
    assert (act, mode, cnt) == (act_ref, modes[mode_ref], cnt_ref)
    assert np.array_equal(src_g, src_ref)
    assert np.abs(phi_g - phi_ref).max() <= 1e-7
    if mode_ref == "blend":
        want = oracle.bank_blend_kv(cfg, f64(cache), bank0, b % 3, act_ref, alpha)
    elif mode_ref == "store":
        want = oracle.bank_store(cfg, f64(cache), bank0, b % 3, act_ref)
    else:
        want = bank0
    assert np.array_equal(f64(bank_kv), want)


# ------------------------------------------------------------------ whole streams

N_BLOCKS, N_LAYERS, PASSES, M, WRITE = 36, 2, 4, 5, 8


def _decided_stream(seed, **pol):
    attempt = np.zeros(N_BLOCKS, dtype=np.int64)
    for _ in range(800):
        kp, ok, _ = synth.pose_stream(seed, N_BLOCKS, attempt=attempt, fail_frac=0.15)
        kp = kp[:, :, :62, :]
        phis = [oracle.fingerprint(kp[b], ok[b]).astype(np.float32) for b in range(N_BLOCKS)]
        dec = oracle.stream_decisions_policy(phis, [list(o) for o in ok], M=M, write_blocks=WRITE,
                                             **pol)
        bad = [b for b, d in enumerate(dec)
               if min(d["retrieval_margin"], d["gate_margin"], d["nearest_margin"]) < MARGIN
               or d["bank_margin"] < 1e-6]
        if not bad:
            return kp, ok, dec
        attempt[bad[0]] += 1
    raise AssertionError("could not draw a stream with decided margins")


@pytest.mark.parametrize("pol", [dict(policy="decay", alpha=0.3),
                                 dict(policy="gated", gate=0.35),
                                 dict(policy="frozen", min_detected=3),
                                 dict(policy="decay", alpha=0.5, min_detected=2)])
def test_policy_stream_matches_oracle_replay(pol):
    need_gpu()
    cfg = synth.preset("tiny")
    kp, ok, dec = _decided_stream(31, **pol)
    s = oracle.layout_sizes(cfg)
    H, d, R = cfg["n_heads"], cfg["head_dim"], cfg["ring_slots"]
    st = P.PRSinkStream(cfg, n_layers=N_LAYERS, M=M, write_blocks=WRITE,
                        policy=pol.get("policy", "frozen"), alpha=pol.get("alpha", 0.0),
                        gate=pol.get("gate", 0.0), min_detected=pol.get("min_detected", 0))
    cache = np.zeros((N_LAYERS, 2, H, s["T"], d))
    bank = np.zeros((N_LAYERS, M, 2, H, s["L_blk"], d))
    for layer in range(N_LAYERS):
        kr = synth.normal_bf16((s["L_ref"], H, d), 1000 + layer, 1)
        st.set_ref(layer, kr.cuda(), kr.cuda())
        cache[layer, 0], cache[layer, 1] = oracle.kv_append(
            dict(cfg, block_index=0), f64(kr), f64(kr), cache[layer, 0], cache[layer, 1],
            oracle.SLOT_REF)
    out = torch.empty((s["L_blk"], H, d), dtype=torch.bfloat16, device="cuda")
    for b in range(N_BLOCKS):
        st.begin_block(torch.from_numpy(np.ascontiguousarray(kp[b])).cuda(),
                       torch.from_numpy(ok[b]).cuda())
        dref = dec[b]
        if dref["copy"]:
            cache = oracle.dyn_copy(cfg, bank, cache, dref["r"])
        cfg_b = dict(cfg, block_index=b, valid_mask=oracle.valid_mask(cfg, b, dref["r"] >= 0))
        for layer in range(N_LAYERS):
            for p in range(PASSES):
                sd = 20_000 + 100 * b + 10 * layer + p
                q, kn, vn = (synth.normal_bf16((s["L_blk"], H, d), sd, j) for j in range(3))
                st.layer_pass(layer, q.cuda(), kn.cuda(), vn.cuda(), out, clean=p == PASSES - 1)
                k2, v2 = oracle.kv_append(cfg_b, f64(kn), f64(vn), cache[layer, 0],
                                          cache[layer, 1], oracle.SLOT_RING0 + b % R)
                if p == PASSES - 1 and b == 0:
                    k2, v2 = oracle.kv_append(cfg_b, f64(kn), f64(vn), k2, v2, oracle.SLOT_STATIC)
                cache[layer, 0], cache[layer, 1] = k2, v2
                if p == PASSES - 1 and layer == 0:
                    ref, _ = oracle.attention(cfg_b, f64(q), k2, v2)
                    check_attention(f64(out), ref, f"b={b}")
        st.end_block()
        if dref["mode"] == "store":
            bank = oracle.bank_store(cfg, cache, bank, b % R, dref["action"])
        elif dref["mode"] == "blend":
            bank = oracle.bank_blend_kv(cfg, cache, bank, b % R, dref["action"], pol["alpha"])
        torch.cuda.synchronize()
        assert int(st.r.item()) == dref["r"], f"block {b}: retrieval"
        assert bool(st.copied.item()) == dref["copy"], f"block {b}: dynamic fill"
        assert int(st.dyn_src.item()) == dref["dyn_src"], f"block {b}"
        assert int(st.action.item()) == dref["action"], f"block {b}: bank action"
        assert int(st.bank_count.item()) == dref["count"]
        assert np.array_equal(st.bank_src.cpu().numpy(), dref["bank_src"]), f"block {b}"
        assert np.abs(f64(st.bank_phi) - dref["bank_phi"]).max() <= 1e-6
    assert P.prsink_sync_status() == P.PRSINK_OK
    assert np.array_equal(f64(st.cache_kv), cache)
    assert np.array_equal(f64(st.bank_kv), bank)
    # the policy acted after the freeze
    if pol["policy"] != "frozen":
        assert any(d["action"] >= 0 for d in dec[WRITE:])
    if pol.get("min_detected"):
        assert any(d["r"] == -1 for d in dec[WRITE:])
