"""The draft-length policy (host functions of the library) against the enumeration oracle, and the oracle
against closed forms and a Monte-Carlo run of the oracle's own verify."""
import math

import numpy as np
import pytest

from oracle import draft_length as odl


def _lib():
    from ar_lm_decoding_b200 import build
    build.build()
    from ar_lm_decoding_b200 import abi
    return abi


def test_oracle_closed_form_endpoints():
    # alpha = 1: nothing is ever rejected, k tokens per step
    for k in (1, 3, 8):
        assert odl.expected_tokens_per_step(k, 1.0) == pytest.approx(k)
    # alpha = 0, k >= 2: every step emits exactly the resampled token (slot 1 pre-accepted, slot 2 rejected)
    for k in (2, 5):
        assert odl.expected_tokens_per_step(k, 0.0) == pytest.approx(1.0)
    # alpha = 0, k = 1: a rejection (1 token), then a step that only re-verifies the resampled token (0 tokens)
    assert odl.expected_tokens_per_step(1, 0.0) == pytest.approx(0.5)


def test_oracle_matches_a_decode_chain_of_the_oracle_verify():
    """Run the oracle's verify as a decode loop on two-token distributions built so that each draft is accepted
    with probability alpha (p(d) / q(d) = alpha for the drafted token), carrying the pre-accepted flag from step
    to step: the mean number of new tokens per step converges to the enumeration's expectation."""
    import oracle
    rng = np.random.default_rng(0)
    for k, alpha in ((3, 0.6), (5, 0.85)):
        # q = (1, 0) always drafts token 0; p = (alpha, 1 - alpha): ratio alpha, residual all on token 1
        V, B, steps = 2, 4000, 12
        zq = np.log(np.array([1.0 - 1e-30, 1e-30]))
        zp = np.log(np.array([alpha, 1.0 - alpha]))
        inp = dict(p_logits=np.broadcast_to(zp, (B, k, V)).astype(np.float32).copy(),
                   q_logits=np.broadcast_to(zq, (B, k, V)).astype(np.float32).copy(),
                   drafts=np.zeros((B, k), np.int32), preaccepted=np.zeros(B, np.uint8))
        total = 0.0
        for s in range(steps):
            inp["u_acc"] = rng.random((B, k)).astype(np.float32)
            inp["u_res"] = rng.random(B).astype(np.float32)
            out = oracle.verify(inp)
            if s >= 4:  # past the start-up of the chain
                total += out["n_emitted"].sum()
            inp["preaccepted"] = (out["accept_len"] < k).astype(np.uint8)
        mean = total / (B * (steps - 4))
        e = odl.expected_tokens_per_step(k, alpha)
        assert abs(mean - e) < 0.03 * e, (k, alpha, mean, e)


@pytest.mark.parametrize("k", [1, 2, 3, 4, 6, 8, 11])
def test_library_expected_tokens_matches_enumeration(k):
    abi = _lib()
    for alpha in (0.0, 0.05, 0.3, 0.5, 0.77, 0.95, 1.0):
        assert abi.tidar_expected_tokens_per_step(k, alpha) == pytest.approx(odl.expected_tokens_per_step(k, alpha),
                                                                               rel=1e-9, abs=1e-12)


def test_library_pick_matches_brute_force():
    abi = _lib()
    rng = np.random.default_rng(1)
    for _ in range(30):
        n = int(rng.integers(1, 13))
        # latencies that grow with the query rows R = k(k+2), as an attention past its ridge does
        base = rng.uniform(50, 500)
        t = [base * (1 + rng.uniform(0, 0.05) * kk * (kk + 2)) for kk in range(1, n + 1)]
        if rng.random() < 0.3:
            t[int(rng.integers(0, n))] = 0.0  # an unmeasured entry
        alpha = float(rng.uniform(0, 1))
        k, rate = abi.tidar_pick_draft_length(t, alpha)
        ko, ro = odl.pick_draft_length(t, alpha)
        assert k == ko and math.isclose(rate, ro, rel_tol=1e-9)


def test_library_rejects_bad_arguments():
    abi = _lib()
    assert abi.tidar_expected_tokens_per_step(0, 0.5) == -1.0
    assert abi.tidar_expected_tokens_per_step(17, 0.5) == -1.0
    assert abi.tidar_expected_tokens_per_step(4, 1.5) == -1.0
    assert abi.tidar_pick_draft_length([], 0.5)[0] == 0
    assert abi.tidar_pick_draft_length([0.0, -1.0], 0.5)[0] == 0
    assert abi.tidar_pick_draft_length([10.0], float("nan"))[0] == 0
