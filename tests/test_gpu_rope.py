"""tidar_rope_qkv against the oracle: the rotary embedding of the step's rows (positions of the TiDAR step
layout, θ = 1e6), fused with the re-layout of the QKV projection output.  Both sides rotate in double
precision and round once to bf16, so they agree bit for bit except where the two sides' double-precision
sine / cosine put a value on the other side of a bf16 rounding boundary: those elements differ by exactly one
bf16 unit and must be rare."""
import numpy as np
import pytest
import torch

import oracle
from ar_lm_decoding_b200 import abi, synth

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to("cuda").view(torch.bfloat16)


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("B,Hq,Hkv,D,k,P", [(1, 32, 8, 128, 8, (4096,)), (3, 12, 2, 128, 4, (0, 77, 1023)),
                                            (2, 4, 4, 64, 16, (16384, 5))])
def test_rope_qkv_matches_oracle(B, Hq, Hkv, D, k, P):
    rng = np.random.default_rng(B * 100 + k)
    R = k * (k + 2)
    qkv = synth.f32_to_bf16_bits(rng.standard_normal((B, R, Hq + 2 * Hkv, D), dtype=np.float32) * 2)
    pl = np.array(P, np.int32)
    q = torch.empty((B, R, Hq, D), dtype=torch.bfloat16, device="cuda")
    kn = torch.empty((B, R, Hkv, D), dtype=torch.bfloat16, device="cuda")
    vn = torch.empty((B, R, Hkv, D), dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.tidar_rope_qkv(_dev(qkv), torch.from_numpy(pl).to("cuda"), B, Hq, Hkv, D, k, 1e6, q, kn, vn, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    rq, rk, rv = oracle.rope_qkv(qkv, pl, Hq, Hkv, k, theta=1e6)
    assert np.array_equal(_bits(vn), rv)
    for got, want in ((_bits(q), rq), (_bits(kn), rk)):
        diff = got != want
        # a differing element is one bf16 unit away (adjacent bit patterns of the same sign)
        assert (np.abs(got[diff].astype(np.int32) - want[diff].astype(np.int32)) == 1).all()
        assert diff.mean() < 1e-3, diff.mean()
