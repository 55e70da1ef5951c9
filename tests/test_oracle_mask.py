"""Pins of the oracle's hybrid mask against hand-drawn masks and closed-form counts.

Source: "TiDAR: Think in Diffusion, Talk in Autoregression" (MLSys 2026),
awesome-system-papers summary, "并行 self-speculative 生成 (§3.2)".
"""
import numpy as np
import pytest

import oracle
from conftest import read_golden


def _golden_mask(name):
    rows = read_golden(name)
    return np.array([[int(c) for c in r[1:]] for r in rows], dtype=bool), [r[0] for r in rows]


@pytest.mark.parametrize("name,k,P", [("hybrid_mask_k1_P1.txt", 1, 1), ("hybrid_mask_k2_P2.txt", 2, 2),
                                      ("hybrid_mask_k3_P0.txt", 3, 0)])
def test_mask_matches_hand_drawn(name, k, P):
    want, labels = _golden_mask(name)
    assert want.shape == (k * (k + 2), P + k * (k + 2))
    got = oracle.hybrid_mask(k, P)
    assert np.array_equal(got, want), f"{name}\n{got.astype(int)}"


@pytest.mark.parametrize("k", [1, 2, 3, 4, 7, 8, 16])
@pytest.mark.parametrize("P", [0, 1, 5, 64])
def test_mask_visible_key_counts(k, P):
    """Draft d_i sees the prefix and d_1..d_i (P + i keys); every slot of group j sees
    the prefix, d_1..d_j and its own k slots (P + j + k keys)."""
    m = oracle.hybrid_mask(k, P)
    counts = m.sum(axis=1)
    for i in range(1, k + 1):
        assert counts[i - 1] == P + i
    for j in range(k + 1):
        for s in range(k):
            assert counts[k + j * k + s] == P + j + k


@pytest.mark.parametrize("k", [1, 3, 8])
def test_mask_partition_structure(k):
    P = 3
    R = k * (k + 2)
    m = oracle.hybrid_mask(k, P)
    new = m[:, P:]
    assert m[:, :P].all(), "every row sees the whole cached prefix"
    assert not new[:k, k:].any(), "draft rows never see pre-draft tokens"
    for j in range(k + 1):
        rows = slice(k + j * k, k + (j + 1) * k)
        blk = new[rows, k:]
        own = np.zeros_like(blk)
        own[:, j * k:(j + 1) * k] = True
        assert np.array_equal(blk, own), "a group sees exactly itself among the pre-draft tokens"
    # the draft block is lower-triangular: causal among drafts
    assert np.array_equal(new[:k, :k], np.tril(np.ones((k, k), dtype=bool)))
    assert R == new.shape[0]


@pytest.mark.parametrize("k,P", [(1, 0), (2, 5), (4, 128)])
def test_causal_mode_is_bottom_right_tril(k, P):
    R = k * (k + 2)
    want = np.tril(np.ones((R, P + R), dtype=bool), k=P)
    assert np.array_equal(oracle.hybrid_mask(k, P, oracle.MASK_CAUSAL), want)
