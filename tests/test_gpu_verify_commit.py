"""GPU parity of tidar_verify, tidar_kv_commit and tidar_verify_commit against the CPU oracle.

Accept lengths, emitted tokens, resampled tokens, next drafts and committed KV
must be bit-exact given the same uniforms.  The only exemption: a decision
whose uniform lies within 1e-5 of the oracle's threshold (|u - p/q| for an
accept test; the chosen token's normalised CDF interval edge for a draw).
After an exempt accept decision the oracle is re-run with the GPU's accept
length forced, so the later outputs are still compared.  Exemptions are
counted and reported.
"""
import numpy as np
import pytest

import oracle
from ar_lm_decoding_b200 import synth
from parity import compare_next_drafts, compare_verify

pytestmark = pytest.mark.gpu



def _gpu():
    import tidar_gpu
    return tidar_gpu


@pytest.mark.parametrize("name", ["tiny", "qwen2.5-1.5b_k4", "qwen2.5-1.5b_k16", "qwen3-8b_k8", "qwen3-8b_k8_b8",
                                  "qwen3-32b_k16"])
def test_verify_parity(name):
    cfg = synth.CONFIGS[name]
    report = []
    for seed in range(3):
        inp = synth.make_verify_inputs(cfg, seed=seed)
        got = _gpu().verify(inp)
        compare_verify(inp, got, report)
    print(f"{name}: exemptions {report}")
    assert len(report) <= 1


def test_verify_many_small_cases():
    """Many sequences on a small vocabulary: every accept length and the resample path."""
    report = []
    rng = np.random.default_rng(0)
    for V, k, dtype in ((8, 4, "f32"), (1000, 16, "f32"), (9000, 3, "bf16"), (17, 1, "bf16")):
        B = 256
        cfg = synth.CONFIGS["tiny"].with_(B=B, V=V, k=k, logits_dtype=dtype, cfg_id=100 + V)
        inp = synth.make_verify_inputs(cfg, seed=int(rng.integers(1 << 30)))
        # make p and q close on part of the batch so that long accept runs occur
        zp = synth.bf16_bits_to_f32(inp["p_logits"]) if dtype == "bf16" else inp["p_logits"].copy()
        zq = synth.bf16_bits_to_f32(inp["q_logits"]) if dtype == "bf16" else inp["q_logits"].copy()
        zq[: B // 2] = zp[: B // 2] + 0.1 * rng.standard_normal(zp[: B // 2].shape).astype(np.float32)
        inp["q_logits"] = synth.f32_to_bf16_bits(zq) if dtype == "bf16" else zq
        got = _gpu().verify(inp)
        compare_verify(inp, got, report)
        assert len(set(got["accept_len"].tolist())) > 1
    print(f"exemptions {report}")
    assert len(report) <= 2


@pytest.mark.parametrize("trust_ar", [0.0, 0.37, 0.8, 1.0])
@pytest.mark.parametrize("name", ["tiny", "qwen2.5-1.5b_k16", "qwen3-8b_k8_b8"])
def test_verify_trust_mix_parity(name, trust_ar):
    """tidar_verify_trust_mix against the oracle's mixed target softmax(lambda z_AR + (1 - lambda) z_diff)."""
    cfg = synth.CONFIGS[name]
    report = []
    for seed in range(2):
        inp = synth.make_verify_inputs(cfg, seed=seed)
        got = _gpu().verify(inp, trust_ar=trust_ar)
        compare_verify(inp, got, report, trust_ar=trust_ar)
        if trust_ar == 0.0:
            assert (got["accept_len"] == cfg.k).all()
    print(f"{name} lambda={trust_ar}: exemptions {report}")
    assert len(report) <= 1


def test_verify_trust_mix_many_small_cases():
    """Small vocabularies, many sequences: the mixed target moves accept lengths across 0..k."""
    report = []
    rng = np.random.default_rng(5)
    for V, k, dtype, lam in ((8, 4, "f32", 0.5), (1000, 16, "f32", 0.25), (9000, 3, "bf16", 0.75)):
        cfg = synth.CONFIGS["tiny"].with_(B=256, V=V, k=k, logits_dtype=dtype, cfg_id=200 + V)
        inp = synth.make_verify_inputs(cfg, seed=int(rng.integers(1 << 30)))
        got = _gpu().verify(inp, trust_ar=lam)
        compare_verify(inp, got, report, trust_ar=lam)
        assert len(set(got["accept_len"].tolist())) > 1
    print(f"exemptions {report}")
    assert len(report) <= 2


def test_verify_bad_draft_sets_status():
    cfg = synth.CONFIGS["tiny"].with_(B=2)
    inp = synth.make_verify_inputs(cfg, seed=1)
    inp["drafts"][1, 2] = cfg.V
    got = _gpu().verify(inp, want_status=True)
    assert got["status"] & 2
    ref = oracle.verify({n: (v[:1] if hasattr(v, "shape") and v.shape[:1] == (2,) else v) for n, v in inp.items()})
    assert got["accept_len"][0] == ref["accept_len"][0]


def _commit_inputs(cfg, seed, L=3):
    rng = np.random.default_rng(seed)
    B, k, R, Hkv, D = cfg.B, cfg.k, cfg.R, cfg.Hkv, cfg.D
    P_max = cfg.P_max
    kc = rng.integers(0, 2**16, (L, B, Hkv, P_max, D)).astype(np.uint16)
    vc = rng.integers(0, 2**16, (L, B, Hkv, P_max, D)).astype(np.uint16)
    kn = rng.integers(0, 2**16, (L, B, R, Hkv, D)).astype(np.uint16)
    vn = rng.integers(0, 2**16, (L, B, R, Hkv, D)).astype(np.uint16)
    pl = synth.prefix_lengths(cfg, seed)
    al = rng.integers(0, k + 1, B).astype(np.int32)
    rs = np.where(al < k, rng.integers(0, cfg.V, B), -1).astype(np.int32)
    v = synth.make_verify_inputs(cfg, seed=seed)
    return kc, vc, kn, vn, pl, al, rs, v["group_logits"], v["u_draft"]


@pytest.mark.parametrize("name", ["tiny", "qwen2.5-1.5b_k4", "qwen2.5-1.5b_k16", "qwen3-8b_k8", "qwen3-8b_k8_b8",
                                  "qwen3-32b_k16"])
def test_commit_parity(name):
    cfg = synth.CONFIGS[name]
    report = []
    for seed in range(2):
        kc, vc, kn, vn, pl, al, rs, g, ud = _commit_inputs(cfg, seed)
        got = _gpu().kv_commit(kc, vc, kn, vn, pl, al, rs, g, ud)
        ref = oracle.kv_commit(kc, vc, kn, vn, pl, al, rs, g, ud)
        assert np.array_equal(got["k_caches"], ref["k_caches"])
        assert np.array_equal(got["v_caches"], ref["v_caches"])
        assert np.array_equal(got["prefix_len"], ref["prefix_len"])
        assert np.array_equal(got["next_q_group"], ref["next_q_group"])
        assert np.array_equal(got["next_preaccepted"], ref["next_preaccepted"])
        compare_next_drafts(got, ref, ud, report)
    print(f"{name}: exemptions {report}")
    assert len(report) <= 1


def test_commit_bad_inputs_set_status_and_leave_sequence():
    cfg = synth.CONFIGS["tiny"].with_(B=3)
    kc, vc, kn, vn, pl, al, rs, g, ud = _commit_inputs(cfg, 5, L=2)
    al = np.array([2, cfg.k + 1, 2], np.int32)           # b=1: accept length out of range
    pl = np.array([cfg.P, cfg.P, cfg.P_max - 1], np.int32)  # b=2: P + j* beyond capacity
    rs = np.array([3, 3, 3], np.int32)
    got = _gpu().kv_commit(kc, vc, kn, vn, pl, al, rs, g, ud, want_status=True)
    assert got["status"] & 4 and got["status"] & 1
    assert np.array_equal(got["k_caches"][:, 1:], kc[:, 1:])
    assert list(got["prefix_len"]) == [cfg.P + 2, cfg.P, cfg.P_max - 1]
    ref = oracle.kv_commit(kc[:, :1], vc[:, :1], kn[:, :1], vn[:, :1], pl[:1], al[:1], rs[:1], g[:1], ud[:1])
    assert np.array_equal(got["k_caches"][:, :1], ref["k_caches"])


def test_step_chain_state_machine():
    """verify -> commit on the GPU, state handed over as the pages' decode loop does."""
    cfg = synth.CONFIGS["qwen2.5-1.5b_k4"].with_(B=4, V=30000, ragged=(100, 400))
    inp = synth.make_verify_inputs(cfg, seed=9)
    got = _gpu().verify(inp)
    ref = compare_verify(inp, got, [])
    kc, vc, kn, vn, pl, _, _, g, ud = _commit_inputs(cfg, 9, L=2)
    cg = _gpu().kv_commit(kc, vc, kn, vn, pl, got["accept_len"], got["resampled"], inp["group_logits"],
                          inp["u_draft"])
    co = oracle.kv_commit(kc, vc, kn, vn, pl, ref["accept_len"], ref["resampled"], inp["group_logits"],
                          inp["u_draft"])
    assert np.array_equal(cg["prefix_len"], pl + got["accept_len"])
    assert np.array_equal(cg["k_caches"], co["k_caches"])
    for b in range(cfg.B):
        if got["accept_len"][b] < cfg.k:
            assert cg["next_drafts"][b, 0] == got["resampled"][b] and cg["next_preaccepted"][b] == 1


def _check_fused(inp, got, kc, vc, kn, vn, pl, report, trust_ar=1.0):
    """The fused call's outputs against the oracle's verify, then its commit on the verify's outcome."""
    ref = compare_verify(inp, got, report, trust_ar=trust_ar)
    c = oracle.kv_commit(kc, vc, kn, vn, pl, ref["accept_len"], ref["resampled"], inp["group_logits"], inp["u_draft"])
    assert np.array_equal(got["k_caches"], c["k_caches"])
    assert np.array_equal(got["v_caches"], c["v_caches"])
    assert np.array_equal(got["prefix_len"], c["prefix_len"])
    assert np.array_equal(got["next_q_group"], c["next_q_group"])
    assert np.array_equal(got["next_preaccepted"], c["next_preaccepted"])
    compare_next_drafts(got, c, inp["u_draft"], report)


@pytest.mark.parametrize("name", ["tiny", "qwen2.5-1.5b_k4", "qwen2.5-1.5b_k16", "qwen3-8b_k8", "qwen3-8b_k8_b8",
                                  "qwen3-8b_k8_peaks", "qwen3-32b_k16"])
def test_verify_commit_parity(name):
    """One launch = tidar_verify then tidar_kv_commit: every output against the oracle's two steps."""
    cfg = synth.CONFIGS[name]
    report, seen = [], []
    for seed in range(2):
        inp = synth.make_verify_inputs(cfg, seed=seed)
        kc, vc, kn, vn, pl, _, _, _, _ = _commit_inputs(cfg, seed, L=2)
        got = _gpu().verify_commit(inp, kc, vc, kn, vn, pl)
        _check_fused(inp, got, kc, vc, kn, vn, pl, report)
        seen += got["accept_len"].tolist()
    print(f"{name}: accept lengths {seen}, exemptions {report}")
    assert len(report) <= 1


@pytest.mark.parametrize("trust_ar", [0.0, 0.37])
def test_verify_commit_trust_mix(trust_ar):
    cfg = synth.CONFIGS["qwen2.5-1.5b_k4"].with_(B=4, V=30000, ragged=(100, 400))
    report = []
    for seed in range(2):
        inp = synth.make_verify_inputs(cfg, seed=seed)
        kc, vc, kn, vn, pl, _, _, _, _ = _commit_inputs(cfg, seed, L=2)
        got = _gpu().verify_commit(inp, kc, vc, kn, vn, pl, trust_ar=trust_ar)
        _check_fused(inp, got, kc, vc, kn, vn, pl, report, trust_ar=trust_ar)
        if trust_ar == 0.0:
            assert (got["accept_len"] == cfg.k).all()
    assert len(report) <= 1


def test_verify_commit_many_sequences():
    """256 sequences on small vocabularies (several items per CTA in every phase), bf16 and f32."""
    report = []
    for V, k, dtype in ((8, 4, "f32"), (9000, 3, "bf16"), (17, 1, "bf16")):
        cfg = synth.CONFIGS["tiny"].with_(B=256, V=V, k=k, logits_dtype=dtype, cfg_id=200 + V)
        inp = synth.make_verify_inputs(cfg, seed=V)
        kc, vc, kn, vn, pl, _, _, _, _ = _commit_inputs(cfg, V, L=1)
        got = _gpu().verify_commit(inp, kc, vc, kn, vn, pl)
        _check_fused(inp, got, kc, vc, kn, vn, pl, report)
    assert len(report) <= 2


@pytest.mark.parametrize("seed", range(12))
def test_verify_commit_random_shapes(seed):
    """Seeded random shapes through the fused call: batch 1-5 with ragged prefixes, k 1-16, an odd vocabulary size
    (a last chunk of any length), bf16 or f32 logits, planted peaks or not, the trust mix on some seeds, 1-4 KV
    heads, D 64 or 128, 1-2 layers; every output against the oracle's verify and commit."""
    rng = np.random.default_rng(2000 + seed)
    k = int(rng.integers(1, 17))
    B = int(rng.integers(1, 6))
    V = int(rng.integers(2, 60001 if k <= 8 else 20001))
    cfg = synth.CONFIGS["tiny"].with_(B=B, k=k, V=V, Hq=4, Hkv=int(rng.choice([1, 2, 4])),
                                      D=int(rng.choice([64, 128])), logits_dtype=str(rng.choice(["bf16", "f32"])),
                                      peaks=bool(rng.integers(0, 2)), P=300, ragged=(0, 300), cfg_id=300 + seed)
    trust_ar = 1.0 if seed % 3 else float(rng.choice([0.3, 0.6]))
    inp = synth.make_verify_inputs(cfg, seed=seed)
    kc, vc, kn, vn, pl, _, _, _, _ = _commit_inputs(cfg, seed, L=int(rng.integers(1, 3)))
    got = _gpu().verify_commit(inp, kc, vc, kn, vn, pl, trust_ar=trust_ar)
    report = []
    _check_fused(inp, got, kc, vc, kn, vn, pl, report, trust_ar=trust_ar)
    print(f"seed {seed}: B {B} k {k} V {V} {cfg.logits_dtype} peaks {cfg.peaks} lambda {trust_ar}: "
          f"accept {got['accept_len'].tolist()}, exemptions {report}")
    assert len(report) <= 1


def test_verify_commit_bad_inputs():
    """A draft outside the vocabulary leaves its sequence untouched (no accept length); a prefix too close to
    the capacity keeps the verify outputs but skips that sequence's commit; the others are committed."""
    cfg = synth.CONFIGS["tiny"].with_(B=3)
    inp = synth.make_verify_inputs(cfg, seed=11)
    inp["drafts"] = inp["drafts"].copy()
    inp["drafts"][1, 2] = cfg.V                             # b=1: a draft outside [0, V)
    inp["preaccepted"] = np.zeros(3, inp["preaccepted"].dtype)
    inp["u_acc"] = np.zeros_like(inp["u_acc"])              # every valid draft accepted: j* = k
    kc, vc, kn, vn, _, _, _, _, _ = _commit_inputs(cfg, 11, L=2)
    pl = np.array([cfg.P, cfg.P, cfg.P_max - 1], np.int32)  # b=2: P + j* beyond capacity
    got = _gpu().verify_commit(inp, kc, vc, kn, vn, pl, want_status=True)
    assert got["status"] & 2 and got["status"] & 1
    assert list(got["prefix_len"]) == [cfg.P + cfg.k, cfg.P, cfg.P_max - 1]
    assert np.array_equal(got["k_caches"][:, 1:], kc[:, 1:]) and np.array_equal(got["v_caches"][:, 1:], vc[:, 1:])
    assert got["accept_len"][1] == -7 and got["next_q_group"][1] == -7 and got["next_q_group"][2] == -7
    sub = {n: (v[[0, 2]] if hasattr(v, "shape") and v.shape[:1] == (3,) else v) for n, v in inp.items()}
    ref = oracle.verify(sub)
    assert list(got["accept_len"][[0, 2]]) == list(ref["accept_len"]) == [cfg.k, cfg.k]
    assert np.array_equal(got["tokens"][[0, 2]], ref["tokens"])
    c = oracle.kv_commit(kc[:, :1], vc[:, :1], kn[:, :1], vn[:, :1], pl[:1], ref["accept_len"][:1],
                         ref["resampled"][:1], inp["group_logits"][:1], inp["u_draft"][:1])
    assert np.array_equal(got["k_caches"][:, :1], c["k_caches"])
    assert got["next_q_group"][0] == cfg.k and got["next_preaccepted"][0] == 0
