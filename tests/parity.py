"""Comparison rules shared by the GPU parity tests (verify and commit against the oracle).

Accept lengths, emitted tokens, resampled tokens and next drafts must be
bit-exact given the same uniforms.  The only exemption: a decision whose
uniform lies within 1e-5 of the oracle's threshold (|u - p/q| for an accept
test; an edge of the chosen token's interval of the oracle's normalised CDF for
a draw).  After an exempt accept decision the oracle is re-run with the GPU's
accept length forced, so the later outputs are still compared.  Every
exemption is appended to `report`.
"""
import numpy as np

import oracle

EXEMPT = 1e-5


def compare_verify(inp, got, report, trust_ar=1.0):
    """Checks the GPU verify outputs `got` against the oracle on `inp`; returns the oracle's outputs (with
    exempt decisions replaced by the GPU's)."""
    ref = oracle.verify(inp, trust_ar=trust_ar)
    B, k = inp["drafts"].shape
    forced = np.full(B, -1, np.int32)
    for b in range(B):
        if got["accept_len"][b] != ref["accept_len"][b]:
            i = min(got["accept_len"][b], ref["accept_len"][b])  # first slot decided differently
            margin = abs(float(inp["u_acc"][b, i]) - ref["ratio"][b, i])
            assert margin < EXEMPT, (b, got["accept_len"][b], ref["accept_len"][b], margin)
            report.append(("accept", b, margin))
            forced[b] = got["accept_len"][b]
    if (forced >= 0).any():
        ref = oracle.verify(inp, forced_accept_len=forced, trust_ar=trust_ar)
    assert np.array_equal(got["accept_len"], ref["accept_len"])
    for b in range(B):
        if got["resampled"][b] != ref["resampled"][b]:
            u = float(inp["u_res"][b])
            margin = min(abs(u - ref["res_lo"][b]), abs(u - ref["res_hi"][b]))
            assert margin < EXEMPT, (b, got["resampled"][b], ref["resampled"][b], margin)
            report.append(("resample", b, margin))
            ref["resampled"][b] = got["resampled"][b]
            ref["tokens"][b, ref["n_emitted"][b] - 1] = got["resampled"][b]
    assert np.array_equal(got["resampled"], ref["resampled"])
    assert np.array_equal(got["n_emitted"], ref["n_emitted"])
    assert np.array_equal(got["tokens"], ref["tokens"])
    np.testing.assert_allclose(got["logp_d"], ref["logp_d"], rtol=0, atol=1e-4)
    np.testing.assert_allclose(got["logq_d"], ref["logq_d"], rtol=0, atol=1e-4)
    return ref


def compare_next_drafts(got, ref, u_draft, report):
    """Next drafts bit-exact except exempt draws; returns the oracle's drafts with those replaced."""
    nd = ref["next_drafts"].copy()
    for b, s in zip(*np.nonzero(got["next_drafts"] != ref["next_drafts"])):
        u = float(u_draft[b, s])
        margin = min(abs(u - ref["draft_lo"][b, s]), abs(u - ref["draft_hi"][b, s]))
        assert margin < EXEMPT, (b, s, got["next_drafts"][b, s], ref["next_drafts"][b, s], margin)
        report.append(("draft", b, s, margin))
        nd[b, s] = got["next_drafts"][b, s]
    return nd
