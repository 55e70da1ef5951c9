"""Pins of the oracle's AR rejection-sampling verify and of its commit/draft selection.

* a hand-worked 3-token example (tests/golden/verify_v3_hand.txt);
* special cases: p == q always accepts; disjoint supports always reject and
  resample from p; a pre-accepted slot 1 is accepted whatever u is;
* Monte-Carlo: with d ~ q the first emitted token is distributed as p, and the
  token emitted at slot 2 given slot 1 was accepted is distributed as p_2
  (speculative sampling is lossless); P(accept) = sum_v min(p(v), q(v));
* commit: exact copy of the accepted rows, nothing else touched, the prefix
  grows by the accept length; next drafts come from group j*, slot 0 is the
  resampled token after a rejection; draft sampling follows the group's
  softmax (Monte-Carlo) and the hand-worked inverse-CDF example.

Source: "TiDAR: Think in Diffusion, Talk in Autoregression" (MLSys 2026),
awesome-system-papers summary, "并行 self-speculative 生成 (§3.2)"; the
bxzpzcl.cn walkthrough, §1.3 (KV keep/evict rules).
"""
import numpy as np
import pytest
from scipy import stats

import oracle
from ar_lm_decoding_b200 import synth
from conftest import read_golden


def _verify_inputs(zp, zq, drafts, u_acc, u_res, pre=None):
    B, k, V = zp.shape
    return dict(p_logits=np.asarray(zp, np.float32), q_logits=np.asarray(zq, np.float32),
                drafts=np.asarray(drafts, np.int32).reshape(B, k),
                preaccepted=np.zeros(B, np.uint8) if pre is None else np.asarray(pre, np.uint8),
                u_acc=np.asarray(u_acc, np.float32).reshape(B, k), u_res=np.asarray(u_res, np.float32).reshape(B))


def test_hand_worked_three_token_example():
    p = np.log(np.array([0.5, 0.3, 0.2]))
    q = np.log(np.array([0.2, 0.3, 0.5]))
    for d, ua, ur, acc, res, ratio in read_golden("verify_v3_hand.txt"):
        inp = _verify_inputs(p[None, None], q[None, None], [[int(d)]], [[float(ua)]], [float(ur)])
        out = oracle.verify(inp)
        assert out["accept_len"][0] == int(acc)
        assert out["resampled"][0] == int(res)
        assert abs(out["ratio"][0, 0] - float(ratio)) < 1e-6
        if int(acc):
            assert out["n_emitted"][0] == 1 and out["tokens"][0, 0] == int(d)
        else:
            assert out["n_emitted"][0] == 1 and out["tokens"][0, 0] == int(res)


def test_p_equals_q_always_accepts():
    rng = np.random.default_rng(0)
    B, k, V = 64, 5, 50
    z = rng.standard_normal((B, k, V)).astype(np.float32) * 2
    inp = _verify_inputs(z, z, rng.integers(0, V, (B, k)), rng.random((B, k)) * 0.999999, rng.random(B))
    out = oracle.verify(inp)
    assert (out["accept_len"] == k).all() and (out["resampled"] == -1).all()
    assert (out["n_emitted"] == k).all()
    assert np.array_equal(out["tokens"], inp["drafts"])


def test_disjoint_supports_always_reject_and_resample_from_p():
    V = 6
    p = np.full(V, -1e4, np.float32)
    q = np.full(V, -1e4, np.float32)
    p[:3] = np.log([0.2, 0.3, 0.5])
    q[3:] = 0.0
    B = 20000
    rng = np.random.default_rng(1)
    zp = np.broadcast_to(p, (B, 1, V)).copy()
    zq = np.broadcast_to(q, (B, 1, V)).copy()
    inp = _verify_inputs(zp, zq, rng.integers(3, 6, (B, 1)), rng.random((B, 1)), rng.random(B))
    out = oracle.verify(inp)
    assert (out["accept_len"] == 0).all()
    counts = np.bincount(out["resampled"], minlength=V)
    assert counts[3:].sum() == 0
    assert stats.chisquare(counts[:3], B * np.array([0.2, 0.3, 0.5])).pvalue > 1e-3


def test_preaccepted_slot_one_is_accepted_regardless():
    V = 4
    p = np.log(np.array([0.97, 0.01, 0.01, 0.01]))
    q = np.log(np.array([0.01, 0.97, 0.01, 0.01]))
    zp = np.stack([p, p])[None]
    zq = np.stack([q, q])[None]
    # d_1 = 1 would be rejected (ratio ~0.01) unless pre-accepted; d_2 = 1 is rejected
    inp = _verify_inputs(zp, zq, [[1, 1]], [[0.9, 0.9]], [0.5], pre=[1])
    out = oracle.verify(inp)
    assert out["accept_len"][0] == 1
    assert out["n_emitted"][0] == 1 and out["tokens"][0, 0] == out["resampled"][0] == 0
    inp["preaccepted"][:] = 0
    out = oracle.verify(inp)
    assert out["accept_len"][0] == 0


def _mc_setup(V, seed, k=2):
    rng = np.random.default_rng(seed)
    P_ = rng.dirichlet(np.ones(V) * 0.7, size=k)
    Q_ = rng.dirichlet(np.ones(V) * 0.7, size=k)
    return rng, P_, Q_


@pytest.mark.parametrize("V,trials", [(8, 400000), (1000, 40000)])
def test_first_emitted_token_is_distributed_as_p(V, trials):
    rng, P_, Q_ = _mc_setup(V, seed=V)
    k = 2
    counts1 = np.zeros(V)
    counts2 = np.zeros(V)
    acc1 = 0
    chunk = 20000
    for start in range(0, trials, chunk):
        B = min(chunk, trials - start)
        drafts = np.stack([rng.choice(V, size=B, p=Q_[i]) for i in range(k)], axis=1)
        zp = np.broadcast_to(np.log(P_), (B, k, V)).astype(np.float32)
        zq = np.broadcast_to(np.log(Q_), (B, k, V)).astype(np.float32)
        inp = _verify_inputs(zp, zq, drafts, rng.random((B, k)), rng.random(B))
        out = oracle.verify(inp)
        counts1 += np.bincount(out["tokens"][:, 0], minlength=V)
        a1 = out["accept_len"] >= 1
        acc1 += a1.sum()
        counts2 += np.bincount(out["tokens"][a1, 1], minlength=V)
    # probabilities in float32 logits: use the rows the oracle actually saw
    p1 = np.exp(np.log(P_[0]).astype(np.float32).astype(np.float64))
    p1 /= p1.sum()
    p2 = np.exp(np.log(P_[1]).astype(np.float32).astype(np.float64))
    p2 /= p2.sum()
    q1 = np.exp(np.log(Q_[0]).astype(np.float32).astype(np.float64))
    q1 /= q1.sum()
    keep = p1 * trials > 5
    assert stats.chisquare(counts1[keep], counts1[keep].sum() * p1[keep] / p1[keep].sum()).pvalue > 1e-3
    keep2 = p2 * acc1 > 5
    assert stats.chisquare(counts2[keep2], counts2[keep2].sum() * p2[keep2] / p2[keep2].sum()).pvalue > 1e-3
    # acceptance probability of slot 1: sum_v min(p, q)
    pa = np.minimum(p1, q1).sum()
    se = np.sqrt(pa * (1 - pa) / trials)
    assert abs(acc1 / trials - pa) < 5 * se


# ---- commit --------------------------------------------------------------


def _commit_case(seed=0, L=2, B=3, Hkv=2, D=8, k=4, P=10, V=50):
    rng = np.random.default_rng(seed)
    R = k * (k + 2)
    P_max = P + k + 3
    kc = rng.integers(0, 2**16, (L, B, Hkv, P_max, D)).astype(np.uint16)
    vc = rng.integers(0, 2**16, (L, B, Hkv, P_max, D)).astype(np.uint16)
    kn = rng.integers(0, 2**16, (L, B, R, Hkv, D)).astype(np.uint16)
    vn = rng.integers(0, 2**16, (L, B, R, Hkv, D)).astype(np.uint16)
    pl = rng.integers(P - 3, P + 1, B).astype(np.int32)
    return rng, kc, vc, kn, vn, pl


def test_commit_copies_accepted_rows_exactly():
    rng, kc, vc, kn, vn, pl = _commit_case()
    L, B, Hkv, P_max, D = kc.shape
    k, V = 4, 50
    al = np.array([0, 2, 4], np.int32)
    rs = np.array([7, 9, -1], np.int32)
    g = rng.standard_normal((B, k + 1, k, V)).astype(np.float32)
    ud = rng.random((B, k)).astype(np.float32)
    out = oracle.kv_commit(kc, vc, kn, vn, pl, al, rs, g, ud)
    for b in range(B):
        P, j = pl[b], al[b]
        for cache, new, got in ((kc, kn, out["k_caches"]), (vc, vn, out["v_caches"])):
            assert np.array_equal(got[:, b, :, :P], cache[:, b, :, :P])
            assert np.array_equal(got[:, b, :, P + j:], cache[:, b, :, P + j:])
            for i in range(j):
                assert np.array_equal(got[:, b, :, P + i], new[:, b, i, :])
    assert np.array_equal(out["prefix_len"], pl + al)
    assert np.array_equal(out["next_q_group"], al)
    assert list(out["next_preaccepted"]) == [1, 1, 0]
    assert out["next_drafts"][0, 0] == 7 and out["next_drafts"][1, 0] == 9


def test_commit_accept_zero_writes_nothing():
    rng, kc, vc, kn, vn, pl = _commit_case(seed=1)
    B = kc.shape[1]
    g = rng.standard_normal((B, 5, 4, 50)).astype(np.float32)
    out = oracle.kv_commit(kc, vc, kn, vn, pl, np.zeros(B, np.int32), np.full(B, 3, np.int32), g,
                           rng.random((B, 4)).astype(np.float32))
    assert np.array_equal(out["k_caches"], kc) and np.array_equal(out["v_caches"], vc)
    assert np.array_equal(out["prefix_len"], pl)


def test_draft_sampling_hand_worked_inverse_cdf():
    # the token and its interval of the normalised CDF: the interval decides which GPU/oracle differences are
    # exempt, so it is pinned to the hand-worked values as well
    z = np.log(np.array([0.25, 0.25, 0.5], np.float64)).astype(np.float32)
    rows = read_golden("inverse_cdf_hand.txt")
    k = 1
    for u, tok, lo, hi in rows:
        g = np.broadcast_to(z, (1, k + 1, k, 3)).copy()
        _, kc, vc, kn, vn, pl = _commit_case(L=1, B=1, Hkv=1, D=2, k=k, P=4)
        out = oracle.kv_commit(kc, vc, kn, vn, pl, np.array([1], np.int32), np.array([-1], np.int32), g,
                               np.array([[float(u)]], np.float32))
        assert out["next_drafts"][0, 0] == int(tok), (u, tok)
        assert abs(out["draft_lo"][0, 0] - float(lo)) < 1e-6 and abs(out["draft_hi"][0, 0] - float(hi)) < 1e-6


def test_draft_interval_is_undefined_for_the_resampled_slot():
    # after a rejection slot 0 is the resampled token, not a draw: no interval, so no exemption can apply
    z = np.log(np.array([0.25, 0.25, 0.5], np.float64)).astype(np.float32)
    k = 2
    g = np.broadcast_to(z, (1, k + 1, k, 3)).copy()
    _, kc, vc, kn, vn, pl = _commit_case(L=1, B=1, Hkv=1, D=2, k=k, P=4)
    out = oracle.kv_commit(kc, vc, kn, vn, pl, np.array([1], np.int32), np.array([2], np.int32), g,
                           np.array([[0.3, 0.3]], np.float32))
    assert out["next_drafts"][0, 0] == 2 and np.isnan(out["draft_lo"][0, 0]) and np.isnan(out["draft_hi"][0, 0])
    assert out["next_drafts"][0, 1] == 1 and abs(out["draft_lo"][0, 1] - 0.25) < 1e-6


def test_residual_resample_hand_worked_interval():
    p = np.log(np.array([0.4, 0.1, 0.3, 0.2]))
    q = np.log(np.array([0.1, 0.3, 0.2, 0.4]))
    for u, tok, lo, hi in read_golden("residual_cdf_hand.txt"):
        inp = _verify_inputs(p[None, None], q[None, None], [[1]], [[0.5]], [float(u)])
        out = oracle.verify(inp)
        assert out["accept_len"][0] == 0 and abs(out["ratio"][0, 0] - 1 / 3) < 1e-6
        assert out["resampled"][0] == int(tok), (u, tok)
        assert abs(out["res_lo"][0] - float(lo)) < 1e-6 and abs(out["res_hi"][0] - float(hi)) < 1e-6
    # every draft accepted: no resample, no interval
    inp = _verify_inputs(p[None, None], q[None, None], [[0]], [[0.5]], [0.5])
    out = oracle.verify(inp)
    assert out["accept_len"][0] == 1 and out["resampled"][0] == -1
    assert np.isnan(out["res_lo"][0]) and np.isnan(out["res_hi"][0])


def test_residual_interval_when_p_equals_q_falls_back_to_p():
    # p == q leaves no residual mass (unreachable in exact arithmetic after a rejection, but forced here):
    # the draw falls back to p itself, and the interval is p's CDF interval
    p = np.log(np.array([0.5, 0.25, 0.25]))
    inp = _verify_inputs(p[None, None], p[None, None], [[2]], [[0.5]], [0.6])
    out = oracle.verify(inp, forced_accept_len=np.array([0], np.int32))
    assert out["resampled"][0] == 1
    assert abs(out["res_lo"][0] - 0.5) < 1e-6 and abs(out["res_hi"][0] - 0.75) < 1e-6


def test_draft_sampling_follows_group_softmax():
    rng = np.random.default_rng(3)
    V, k, B = 12, 2, 30000
    probs = rng.dirichlet(np.ones(V), size=(k + 1, k))
    z = np.log(probs).astype(np.float32)
    g = np.broadcast_to(z, (B, k + 1, k, V)).copy()
    kc = np.zeros((1, B, 1, 8, 2), np.uint16)
    kn = np.zeros((1, B, k * (k + 2), 1, 2), np.uint16)
    al = rng.integers(0, k + 1, B).astype(np.int32)
    rs = np.zeros(B, np.int32)
    out = oracle.kv_commit(kc, kc, kn, kn, np.zeros(B, np.int32), al, rs, g, rng.random((B, k)).astype(np.float32))
    for j in range(k + 1):
        sel = al == j
        for s in range(k):
            if j < k and s == 0:
                assert (out["next_drafts"][sel, 0] == 0).all()
                continue
            want = np.exp(z[j, s].astype(np.float64))
            want /= want.sum()
            cnt = np.bincount(out["next_drafts"][sel, s], minlength=V)
            assert stats.chisquare(cnt, cnt.sum() * want).pvalue > 1e-3


def test_synth_peaks_drive_accept_length():
    cfg = synth.CONFIGS["qwen2.5-1.5b_k4"].with_(B=6, V=4096)
    inp = synth.make_verify_inputs(cfg, seed=0)
    out = oracle.verify(inp)
    # with planted shared peaks the accept length follows the number of shared peaks
    m = inp["m_shared"]
    pre = inp["preaccepted"].astype(np.int32)
    assert np.abs(out["accept_len"] - np.maximum(m, pre)).max() <= 1


# ---- trust-mix verify (lambda mixes the AR and diffusion logits of the target) ----


def test_trust_mix_hand_worked_example():
    p = np.log(np.array([0.5, 0.3, 0.2]))
    q = np.log(np.array([0.2, 0.3, 0.5]))
    for d, ua, ur, acc, res, ratio, lo, hi in read_golden("verify_trust_mix_hand.txt"):
        inp = _verify_inputs(p[None, None], q[None, None], [[int(d)]], [[float(ua)]], [float(ur)])
        out = oracle.verify(inp, trust_ar=0.5)
        assert out["accept_len"][0] == int(acc) and out["resampled"][0] == int(res), (d, ua, ur)
        assert abs(out["ratio"][0, 0] - float(ratio)) < 2e-6
        if lo == "nan":
            assert np.isnan(out["res_lo"][0])
        else:
            assert abs(out["res_lo"][0] - float(lo)) < 2e-6 and abs(out["res_hi"][0] - float(hi)) < 2e-6


def test_trust_mix_endpoints():
    rng = np.random.default_rng(4)
    B, k, V = 40, 4, 30
    zp = (rng.standard_normal((B, k, V)) * 2).astype(np.float32)
    zq = (rng.standard_normal((B, k, V)) * 2).astype(np.float32)
    inp = _verify_inputs(zp, zq, rng.integers(0, V, (B, k)), rng.random((B, k)), rng.random(B))
    # lambda = 1: the plain AR verify
    a, b = oracle.verify(inp), oracle.verify(inp, trust_ar=1.0)
    for n in ("accept_len", "resampled", "tokens", "n_emitted"):
        assert np.array_equal(a[n], b[n])
    # lambda = 0: the target is q itself, every draft has ratio 1 and is accepted
    z = oracle.verify(inp, trust_ar=0.0)
    assert (z["accept_len"] == k).all() and (z["resampled"] == -1).all()
    assert np.allclose(z["logp_d"], z["logq_d"])
    with pytest.raises(ValueError):
        oracle.verify(inp, trust_ar=1.5)


def test_trust_mix_is_lossless_for_its_target():
    """With d ~ q, the first emitted token is distributed as p_lambda = softmax(lambda z_p + (1 - lambda) z_q)
    (speculative sampling is exact for whatever target it verifies against)."""
    lam, V, trials = 0.3, 8, 200000
    rng, P_, Q_ = _mc_setup(V, seed=77, k=1)
    zp, zq = np.log(P_[0]).astype(np.float32), np.log(Q_[0]).astype(np.float32)
    counts = np.zeros(V)
    for start in range(0, trials, 20000):
        B = 20000
        drafts = rng.choice(V, size=(B, 1), p=np.exp(zq.astype(np.float64)) / np.exp(zq.astype(np.float64)).sum())
        inp = _verify_inputs(np.broadcast_to(zp, (B, 1, V)).copy(), np.broadcast_to(zq, (B, 1, V)).copy(), drafts,
                             rng.random((B, 1)), rng.random(B))
        out = oracle.verify(inp, trust_ar=lam)
        counts += np.bincount(out["tokens"][:, 0], minlength=V)
    target = np.exp(lam * zp.astype(np.float64) + (1 - lam) * zq.astype(np.float64))
    target /= target.sum()
    assert stats.chisquare(counts, counts.sum() * target).pvalue > 1e-3
    # and it is not the AR distribution itself
    pa = np.exp(zp.astype(np.float64)) / np.exp(zp.astype(np.float64)).sum()
    assert stats.chisquare(counts, counts.sum() * pa).pvalue < 1e-6
