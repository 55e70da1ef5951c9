"""Pins of the oracle's hybrid-mask attention.

* dense materialised mask == index predicate (bitwise);
* pure-causal mode == torch's scaled_dot_product_attention (fp64, library);
* hybrid mode == scaled_dot_product_attention given the hand-drawn masks;
* closed form with all keys equal: O = mean of the visible V rows and
  LSE = s + ln(#visible);
* group j does not depend on drafts beyond j, drafts do not depend on
  pre-draft tokens (bitwise), and group j does depend on d_j.

Source: "TiDAR: Think in Diffusion, Talk in Autoregression" (MLSys 2026),
awesome-system-papers summary, "并行 self-speculative 生成 (§3.2)" and Table 3
discussion (pure causal mask = AR mode).
"""
import numpy as np
import pytest
import torch

import oracle
from ar_lm_decoding_b200 import synth
from conftest import read_golden

TINY = synth.CONFIGS["tiny"]


def _f(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def _keys_values(inp, b, kv, P):
    kc = _f(inp["k_cache"][b, kv, :P])
    vc = _f(inp["v_cache"][b, kv, :P])
    kn = _f(inp["k_new"][b, :, kv])
    vn = _f(inp["v_new"][b, :, kv])
    return np.concatenate([kc, kn]), np.concatenate([vc, vn])


def _sdpa_reference(inp, cfg, mask):
    """O and LSE per (b, r, h) with torch's SDPA and logsumexp, mask [R, P+R] bool."""
    B, R, Hq, D, G = cfg.B, cfg.R, cfg.Hq, cfg.D, cfg.G
    o = np.zeros((B, R, Hq, D))
    lse = np.zeros((B, R, Hq))
    scale = 1.0 / np.sqrt(D)
    for b in range(B):
        P = int(inp["prefix_len"][b])
        mk = torch.from_numpy(mask(P))
        for h in range(Hq):
            K, Vv = _keys_values(inp, b, h // G, P)
            q = torch.from_numpy(_f(inp["q"][b, :, h]))
            Kt, Vt = torch.from_numpy(K), torch.from_numpy(Vv)
            o[b, :, h] = torch.nn.functional.scaled_dot_product_attention(
                q[None], Kt[None], Vt[None], attn_mask=mk[None], scale=scale)[0].numpy()
            s = torch.where(mk, (q @ Kt.T) * scale, torch.tensor(-torch.inf, dtype=torch.float64))
            lse[b, :, h] = torch.logsumexp(s, dim=-1).numpy()
    return o, lse


def test_dense_mask_equals_predicate_bitwise():
    cfg = TINY.with_(B=3, ragged=(0, 40))
    inp = synth.make_attn_inputs(cfg, seed=1)
    for mode in (oracle.MASK_HYBRID, oracle.MASK_CAUSAL):
        a = oracle.attn(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, mode=mode, dense=True)
        b = oracle.attn(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, mode=mode, dense=False)
        for x, y in zip(a, b):
            assert np.array_equal(x, y)


@pytest.mark.parametrize("B,Hq,Hkv,k,P", [(1, 2, 1, 4, 128), (2, 4, 2, 2, 17), (1, 3, 1, 1, 0)])
def test_causal_mode_matches_sdpa(B, Hq, Hkv, k, P):
    cfg = TINY.with_(B=B, Hq=Hq, Hkv=Hkv, k=k, P=P, D=32)
    inp = synth.make_attn_inputs(cfg, seed=2)
    o, lse, _ = oracle.attn(inp, Hq, Hkv, cfg.D, k, mode=oracle.MASK_CAUSAL)
    R = cfg.R
    # bottom-right aligned causal mask from torch's own tril
    ro, rl = _sdpa_reference(inp, cfg, lambda P_: torch.ones(R, P_ + R, dtype=torch.bool).tril(diagonal=P_).numpy())
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


@pytest.mark.parametrize("name,k,P", [("hybrid_mask_k2_P2.txt", 2, 2), ("hybrid_mask_k3_P0.txt", 3, 0),
                                      ("hybrid_mask_k1_P1.txt", 1, 1)])
def test_hybrid_matches_sdpa_with_hand_drawn_mask(name, k, P):
    rows = read_golden(name)
    mask = np.array([[int(c) for c in r[1:]] for r in rows], dtype=bool)
    cfg = TINY.with_(Hq=4, Hkv=2, D=16, k=k, P=P)
    inp = synth.make_attn_inputs(cfg, seed=3)
    o, lse, _ = oracle.attn(inp, cfg.Hq, cfg.Hkv, cfg.D, k)
    ro, rl = _sdpa_reference(inp, cfg, lambda P_: mask)
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


@pytest.mark.parametrize("k,P", [(1, 3), (4, 128), (3, 0)])
def test_all_keys_equal_closed_form(k, P):
    cfg = TINY.with_(k=k, P=P, D=8)
    inp = synth.make_attn_inputs(cfg, seed=4)
    R, D = cfg.R, cfg.D
    key = inp["k_new"][0, 0, 0].copy()
    inp["k_cache"][:, :, :P] = key
    inp["k_new"][:] = key
    o, lse, _ = oracle.attn(inp, cfg.Hq, cfg.Hkv, D, k)
    Vall = [_keys_values(inp, 0, kv, P)[1] for kv in range(cfg.Hkv)]
    for h in range(cfg.Hq):
        Vv = Vall[h // cfg.G]
        s = float(_f(inp["q"][0, 0, h]) @ _f(key)) / np.sqrt(D)
        for r in range(R):
            s = float(_f(inp["q"][0, r, h]) @ _f(key)) / np.sqrt(D)
            if r < k:  # draft d_{r+1}: the prefix and d_1..d_{r+1}
                vis = list(range(P)) + [P + i for i in range(r + 1)]
            else:  # slot of group j: the prefix, d_1..d_j and the group's own k slots
                j = (r - k) // k
                vis = list(range(P)) + [P + i for i in range(j)] + [P + k + j * k + s_ for s_ in range(k)]
            np.testing.assert_allclose(o[0, r, h], Vv[vis].mean(axis=0), rtol=0, atol=1e-12)
            assert abs(lse[0, r, h] - (s + np.log(len(vis)))) < 1e-12


def test_group_j_ignores_later_drafts_and_drafts_ignore_groups():
    cfg = TINY.with_(k=4, P=16)
    k, R = cfg.k, cfg.R
    base = synth.make_attn_inputs(cfg, seed=5)
    o0, l0, _ = oracle.attn(base, cfg.Hq, cfg.Hkv, cfg.D, k)
    rng = np.random.default_rng(0)
    for j in range(k + 1):
        pert = {n: v.copy() for n, v in base.items()}
        # change K/V of drafts d_{j+1}..d_k
        for n in ("k_new", "v_new"):
            pert[n][:, j:k] = synth.f32_to_bf16_bits(rng.standard_normal(pert[n][:, j:k].shape).astype(np.float32))
        o1, l1, _ = oracle.attn(pert, cfg.Hq, cfg.Hkv, cfg.D, k)
        rows = slice(k + j * k, k + (j + 1) * k)
        assert np.array_equal(o0[:, rows], o1[:, rows]) and np.array_equal(l0[:, rows], l1[:, rows])
        if j < k:  # ...but group j+1 sees d_{j+1}
            rows2 = slice(k + (j + 1) * k, k + (j + 2) * k)
            assert not np.array_equal(o0[:, rows2], o1[:, rows2])
    pert = {n: v.copy() for n, v in base.items()}
    for n in ("k_new", "v_new"):
        pert[n][:, k:] = synth.f32_to_bf16_bits(rng.standard_normal(pert[n][:, k:].shape).astype(np.float32))
    o1, l1, _ = oracle.attn(pert, cfg.Hq, cfg.Hkv, cfg.D, k)
    assert np.array_equal(o0[:, :k], o1[:, :k]) and np.array_equal(l0[:, :k], l1[:, :k])
    assert not np.array_equal(o0[:, k:], o1[:, k:])
    assert R == o0.shape[1]


def test_rows_subset_equals_full():
    cfg = TINY.with_(B=2, ragged=(30, 90), Hq=4, Hkv=2)
    inp = synth.make_attn_inputs(cfg, seed=6)
    o, lse, _ = oracle.attn(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k)
    rng = np.random.default_rng(1)
    sb = rng.integers(0, cfg.B, 20)
    sh = rng.integers(0, cfg.Hq, 20)
    sr = rng.integers(0, cfg.R, 20)
    so, sl = oracle.attn_rows(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, sb, sh, sr)
    assert np.array_equal(so, o[sb, sr, sh]) and np.array_equal(sl, lse[sb, sr, sh])


def test_bf16_output_rounding_is_nearest_even():
    cfg = TINY.with_(P=8)
    inp = synth.make_attn_inputs(cfg, seed=7)
    o, _, ob = oracle.attn(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k)
    # torch's own conversion rounds to nearest even (through fp32: skip the values
    # where that intermediate lands exactly on a bf16 halfway point)
    want = torch.from_numpy(o).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    f32 = o.astype(np.float32).view(np.uint32)
    ok = (f32 & 0xFFFF) != 0x8000
    assert ok.mean() > 0.99
    assert np.array_equal(ob[ok], want[ok])


def test_poisoned_rows_beyond_prefix_are_never_used():
    cfg = TINY.with_(B=2, ragged=(5, 40))
    inp = synth.make_attn_inputs(cfg, seed=8, poison=True)
    o, lse, _ = oracle.attn(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
