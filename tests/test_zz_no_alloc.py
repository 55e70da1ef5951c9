"""tidar_verify_noalloc against tidar_verify.

tidar_verify_noalloc serves callers that cannot allocate device memory (for
example a plug-in inside a runtime that owns the device memory, or a serving
loop that must not allocate once it runs): instead of a caller workspace it
uses a fixed 2 MiB scratch array inside the library.  This test calls both
entry points through the C ABI on the same inputs and requires the same
results, on two calls in a row with different sizes (the second call finds
the first call's leftovers in the shared array), and checks that a size whose
scratch would not fit is refused.  It lives in its own file so that it runs
after every other test, and it passes on its own in a fresh process as well.
"""
import numpy as np
import pytest
import torch

from ar_lm_decoding_b200 import abi, synth

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _inputs(cfg, seed):
    import tidar_gpu
    v = synth.make_verify_inputs(cfg, seed=seed)
    p, dt = tidar_gpu.logits_dev(v["p_logits"])
    q, _ = tidar_gpu.logits_dev(v["q_logits"])
    dev = dict(p=p, q=q, dt=dt, drafts=tidar_gpu.to_dev(v["drafts"].astype(np.int32)),
               pre=tidar_gpu.to_dev(v["preaccepted"].astype(np.uint8)),
               ua=tidar_gpu.to_dev(v["u_acc"].astype(np.float32)), ur=tidar_gpu.to_dev(v["u_res"].astype(np.float32)))
    return v["p_logits"].shape, dev


def _outputs(B, k):
    return dict(accept_len=torch.full((B,), -7, dtype=torch.int32, device=DEV),
                resampled=torch.full((B,), -7, dtype=torch.int32, device=DEV),
                tokens=torch.full((B, k), -7, dtype=torch.int32, device=DEV),
                n_emitted=torch.full((B,), -7, dtype=torch.int32, device=DEV),
                logp=torch.zeros((B, k), dtype=torch.float32, device=DEV),
                logq=torch.zeros((B, k), dtype=torch.float32, device=DEV),
                status=torch.zeros(1, dtype=torch.int32, device=DEV))


def _run(shape, d, noalloc):
    B, k, V = shape
    o = _outputs(B, k)
    if noalloc:
        abi.tidar_verify_noalloc(d["p"], d["q"], d["dt"], d["drafts"], d["pre"], d["ua"], d["ur"], B, k, V,
                                 o["accept_len"], o["resampled"], o["tokens"], o["n_emitted"], o["logp"], o["logq"],
                                 o["status"])
    else:
        ws = torch.empty(abi.tidar_verify_workspace_size(B, k, V), dtype=torch.uint8, device=DEV)
        abi.tidar_verify(d["p"], d["q"], d["dt"], d["drafts"], d["pre"], d["ua"], d["ur"], B, k, V,
                         o["accept_len"], o["resampled"], o["tokens"], o["n_emitted"], o["logp"], o["logq"], ws,
                         ws.numel(), o["status"])
    torch.cuda.synchronize()
    return {n: t.cpu().numpy() for n, t in o.items()}


def _same(a, b):
    for n in ("accept_len", "resampled", "tokens", "n_emitted", "status"):
        assert np.array_equal(a[n], b[n]), n
    np.testing.assert_allclose(a["logp"], b["logp"], rtol=0, atol=1e-4)
    np.testing.assert_allclose(a["logq"], b["logq"], rtol=0, atol=1e-4)


def test_noalloc_verify_matches_workspace_verify_on_two_calls_in_a_row():
    cases = [(synth.CONFIGS["qwen3-8b_k8"].with_(B=4), 11),
             (synth.CONFIGS["tiny"].with_(B=64, k=16, V=3000, cfg_id=77), 12)]
    for cfg, seed in cases:
        shape, d = _inputs(cfg, seed)
        want = _run(shape, d, noalloc=False)
        got = _run(shape, d, noalloc=True)
        _same(got, want)
        assert (got["accept_len"] >= 0).all()


def test_noalloc_verify_refuses_sizes_beyond_its_scratch():
    B, k, V = 256, 16, 151936  # needs more than the 2 MiB scratch
    assert abi.tidar_verify_workspace_size(B, k, V) > 2 << 20
    o = _outputs(1, 1)
    with pytest.raises(abi.TidarError) as e:
        abi.tidar_verify_noalloc(8192, 8192, abi.TIDAR_DT_BF16, 8192, 8192, 8192, 8192, B, k, V, o["accept_len"],
                                 o["resampled"], o["tokens"], o["n_emitted"], None, None, o["status"])
    assert e.value.status == abi.TIDAR_ERR_WORKSPACE
