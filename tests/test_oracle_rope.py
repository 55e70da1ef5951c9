"""Pins of the oracle's rotary embedding of the step's rows (the input side of the attention: post-RoPE Q and
K_new, θ = 1e6 as in the Qwen backbones the TiDAR pages start from; summary, 核心方法 / initialisation).

* row positions: hand-worked table (tests/golden/row_positions_hand.txt);
* position 0 is the identity (cos 0 = 1, sin 0 = 0): output bits equal input bits;
* a hand-worked head of size 4 at position 1 (angles 1 and 1e6^-1/2 = 1e-3);
* every rotated pair keeps its length (a rotation), up to bf16 rounding;
* the attention score depends only on the position difference: q at m and k at n give the same dot product as q
  at m + c and k at n + c (the property RoPE is built for), up to bf16 rounding;
* V is copied unchanged.
"""
import numpy as np

import oracle
from ar_lm_decoding_b200 import synth
from conftest import read_golden


def test_row_positions_hand_worked():
    for row in read_golden("row_positions_hand.txt"):
        k, P, pos = int(row[0]), int(row[1]), [int(x) for x in row[2:]]
        assert len(pos) == k * (k + 2)
        assert oracle.row_positions(k, P).tolist() == pos


def _qkv(rng, B, R, H, D):
    return synth.f32_to_bf16_bits(rng.standard_normal((B, R, H, D), dtype=np.float32))


def test_position_zero_is_identity_and_v_is_copied():
    rng = np.random.default_rng(0)
    k, Hq, Hkv, D = 1, 2, 1, 8
    x = _qkv(rng, 1, 3, Hq + 2 * Hkv, D)
    q, kn, vn = oracle.rope_qkv(x, np.array([0], np.int32), Hq, Hkv, k)
    # row 0 (the draft) and row 1 (group 0, slot 0) sit at position 0
    assert np.array_equal(q[0, :2], x[0, :2, :Hq]) and np.array_equal(kn[0, :2], x[0, :2, Hq:Hq + Hkv])
    assert not np.array_equal(q[0, 2], x[0, 2, :Hq])  # row 2 sits at position 1
    assert np.array_equal(vn, x[:, :, Hq + Hkv:])


def test_hand_worked_head_of_four():
    # D = 4: pairs (x0, x2) turn by 1 * 1e6^0 = 1 radian, (x1, x3) by 1e6^(-2/4) = 1e-3 radian
    x = np.zeros((1, 3, 3, 4), np.float32)  # k = 1: rows at positions P, P, P + 1 with P = 0 -> 0, 0, 1
    x[0, 2, 0] = [1.0, 0.0, 0.0, 0.0]
    x[0, 2, 1] = [0.0, 2.0, 0.0, 0.0]
    q, kn, _ = oracle.rope_qkv(synth.f32_to_bf16_bits(x), np.array([0], np.int32), 1, 1, 1)
    got_q = synth.bf16_bits_to_f32(q[0, 2, 0])
    got_k = synth.bf16_bits_to_f32(kn[0, 2, 0])
    want_q = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(np.array([np.cos(1.0), 0, np.sin(1.0), 0], np.float32)))
    want_k = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(np.array([0, 2 * np.cos(1e-3), 0, 2 * np.sin(1e-3)],
                                                                     np.float32)))
    assert np.array_equal(got_q, want_q) and np.array_equal(got_k, want_k)


def test_rotation_keeps_pair_lengths():
    rng = np.random.default_rng(1)
    k, Hq, Hkv, D = 4, 4, 2, 128
    x = _qkv(rng, 2, k * (k + 2), Hq + 2 * Hkv, D)
    q, kn, _ = oracle.rope_qkv(x, np.array([100, 5000], np.int32), Hq, Hkv, k)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    for got, src in ((q, xf[:, :, :Hq]), (kn, xf[:, :, Hq:Hq + Hkv])):
        g = synth.bf16_bits_to_f32(got).astype(np.float64)
        n_in = np.hypot(src[..., :D // 2], src[..., D // 2:])
        n_out = np.hypot(g[..., :D // 2], g[..., D // 2:])
        assert np.abs(n_out - n_in).max() <= 2 ** -7 * n_in.max()


def test_scores_depend_on_the_position_difference_only():
    rng = np.random.default_rng(2)
    D = 128
    k = 1  # rows at P, P, P + 1
    base = _qkv(rng, 1, 3, 3, D)
    dots = []
    for shift in (0, 37, 4000):
        q, kn, _ = oracle.rope_qkv(base, np.array([shift], np.int32), 1, 1, k)
        qf = synth.bf16_bits_to_f32(q).astype(np.float64)
        kf = synth.bf16_bits_to_f32(kn).astype(np.float64)
        dots.append(float(qf[0, 2, 0] @ kf[0, 0, 0]))  # query at shift + 1, key at shift: difference 1
    assert max(dots) - min(dots) <= 0.05 * np.sqrt(D)
    q0, kn0, _ = oracle.rope_qkv(base, np.array([0], np.int32), 1, 1, k)
    far = float(synth.bf16_bits_to_f32(q0)[0, 2, 0].astype(np.float64) @
                synth.bf16_bits_to_f32(oracle.rope_qkv(base, np.array([50], np.int32), 1, 1, k)[1])[0, 0, 0])
    assert abs(far - dots[0]) > 0.05 * np.sqrt(D)  # another difference gives another score
