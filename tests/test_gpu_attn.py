"""GPU parity of tidar_attn_step against the CPU oracle (through the C ABI).

Tolerances: output max-abs 2e-2 (bf16), LSE max-abs 1e-4 (fp32 statistics).
Inputs carry NaN in every cache row at or beyond the prefix length and the
workspace starts as NaN, so a read outside the visible keys or of an
unwritten partial shows up as a mismatch.
"""
import numpy as np
import pytest

import oracle
from ar_lm_decoding_b200 import synth

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 2e-2, 1e-4
TINY = synth.CONFIGS["tiny"]


def _gpu():
    import tidar_gpu
    return tidar_gpu


def _check_full(cfg, seed=0, mode=oracle.MASK_HYBRID, inp=None):
    inp = synth.make_attn_inputs(cfg, seed=seed) if inp is None else inp
    o_ref, lse_ref, _ = oracle.attn(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, mode=mode, dense=False)
    o, lse = _gpu().attn(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, mode=mode)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    eo = np.abs(o - o_ref).max()
    el = np.abs(lse - lse_ref).max()
    assert eo <= O_TOL and el <= LSE_TOL, (cfg.name, eo, el)
    return o, lse


def test_tiny_config():
    _check_full(TINY)


@pytest.mark.parametrize("mode", [oracle.MASK_HYBRID, oracle.MASK_CAUSAL])
@pytest.mark.parametrize("D", [64, 128])
def test_modes_and_head_dims(mode, D):
    _check_full(TINY.with_(D=D, Hq=4, Hkv=2, P=200), seed=1, mode=mode)


@pytest.mark.parametrize("k", [1, 2, 3, 5, 8, 16])
def test_draft_lengths(k):
    _check_full(TINY.with_(k=k, P=77, Hq=8, Hkv=2, D=128), seed=k)


@pytest.mark.parametrize("P", [0, 1, 63, 64, 65, 300])
def test_prefix_edges(P):
    _check_full(TINY.with_(P=P, Hq=4, Hkv=1, D=128), seed=P + 10)


def test_ragged_batch():
    _check_full(TINY.with_(B=5, ragged=(0, 700), Hq=6, Hkv=2, D=128, k=3), seed=3)


def test_gqa_groups():
    for Hq, Hkv in ((8, 1), (12, 2), (32, 8), (5, 5)):
        _check_full(TINY.with_(Hq=Hq, Hkv=Hkv, P=130, D=128), seed=Hq)


@pytest.mark.parametrize("name", ["qwen2.5-1.5b_k4", "qwen2.5-1.5b_k16", "qwen3-8b_k8", "qwen3-8b_k8_b8",
                                  "qwen3-32b_k4", "qwen3-32b_k8", "qwen3-32b_k16"])
def test_full_size_every_row(name):
    """One layer at the full size of each workload, in the launch configuration the benchmark times (same
    shapes, so the same split count and cluster size): every (sequence, row, head) output row and LSE against
    the oracle, element by element."""
    cfg = synth.CONFIGS[name]
    inp = synth.make_attn_inputs(cfg, seed=0)
    o, lse = _gpu().attn(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    o_ref, lse_ref, _ = oracle.attn(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, dense=False)
    eo = np.abs(o - o_ref).max()
    el = np.abs(lse - lse_ref).max()
    assert eo <= O_TOL and el <= LSE_TOL, (name, eo, el)


def test_split_choice():
    """The cluster size each workload launches with: a supported size (2-8, or the non-portable 9, 10, 12, 15 the
    device grants), never more splits than key tiles, and the whole grid in one wave unless it is a single split.
    (test_full_size_every_row runs these same launch configurations against the oracle.)"""
    from ar_lm_decoding_b200 import abi
    for name, cfg in synth.CONFIGS.items():
        S = abi.tidar_testing_attn_splits(cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, cfg.P_max)
        tiles = -(-cfg.P_max // 128) + -(-cfg.R // 128)
        row_tiles = cfg.B * cfg.Hkv * -(-cfg.R * (cfg.Hq // cfg.Hkv) // 128)
        assert S in (1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 12, 15) and S <= max(1, tiles), (name, S)
        assert S == 1 or S * row_tiles <= 148, (name, S, row_tiles)
    assert abi.tidar_testing_attn_splits(1, 4, 3, 128, 4, 100) == 0  # Hq not a multiple of Hkv: rejected


def _plant_growing_spikes(cfg, inp, step_nat):
    """For every 128-key tile t of the cache and every KV head, overwrite one key so that it scores
    (4 + step_nat * t) natural-log units against one query row of that head's group (a different row each
    tile, the key in column 37 t mod 128 so both column halves get spikes).  The running max of those rows
    grows by ~step_nat / ln 2 log2-units on every tile -- more than the 2^8 stale-max allowance -- while the
    other rows of the same warps do not grow."""
    q = synth.bf16_bits_to_f32(inp["q"]).astype(np.float64)
    kc = synth.bf16_bits_to_f32(inp["k_cache"]).copy()
    G = cfg.Hq // cfg.Hkv
    scale = 1.0 / np.sqrt(cfg.D)
    for b in range(cfg.B):
        P = int(inp["prefix_len"][b])
        for h in range(cfg.Hkv):
            for t in range((P + 127) // 128):
                n = t * 128 + (37 * t) % 128
                if n >= P:
                    continue
                r, g = t % cfg.R, h * G + (t % G)
                qv = q[b, r, g]
                target = 4.0 + step_nat * t
                kc[b, h, n] = (qv * (target / (scale * float(qv @ qv)))).astype(np.float32)
    out = dict(inp)
    out["k_cache"] = synth.f32_to_bf16_bits(kc)
    return out


@pytest.mark.parametrize("B,Hq,Hkv,P", [(1, 8, 2, 2000), (2, 4, 1, 1200)])
def test_running_max_growth_rescales(B, Hq, Hkv, P):
    # every tile raises some rows' maxima by ~10 log2-units: the rescale of O and the redone exponentials
    cfg = TINY.with_(B=B, Hq=Hq, Hkv=Hkv, D=128, k=3, P=P)
    inp = _plant_growing_spikes(cfg, synth.make_attn_inputs(cfg, seed=7), step_nat=7.0)
    _check_full(cfg, inp=inp)


def _plant_deep_first_tiles(cfg, inp, depth_nat=100.0):
    """For every KV head and every even 128-key tile t of the cache (with a tile after it), pull all keys of
    tile t, and the keys in columns 64..127 of tile t+1, away from one query row of that head's group, so that
    the row scores about -depth_nat natural-log units there.  A CTA that meets tile t first sets that row's
    running max ~depth_nat / ln 2 log2-units below the scores of tile t+1's first half: exponentials against
    the stale max overflow there (in one column half only) before the row's max is renewed."""
    q = synth.bf16_bits_to_f32(inp["q"]).astype(np.float64)
    kc = synth.bf16_bits_to_f32(inp["k_cache"]).astype(np.float64)
    G = cfg.Hq // cfg.Hkv
    scale = 1.0 / np.sqrt(cfg.D)
    for b in range(cfg.B):
        P = int(inp["prefix_len"][b])
        nt = (P + 127) // 128
        for h in range(cfg.Hkv):
            for t in range(0, nt - 1, 2):
                r, g = t % cfg.R, h * G + (t // 2) % G
                qv = q[b, r, g]
                alpha = depth_nat / (scale * float(qv @ qv))
                for n in list(range(t * 128, t * 128 + 128)) + list(range(t * 128 + 192, t * 128 + 256)):
                    if n < P:
                        kc[b, h, n] = kc[b, h, n] - alpha * qv
    out = dict(inp)
    out["k_cache"] = synth.f32_to_bf16_bits(kc.astype(np.float32))
    return out


@pytest.mark.parametrize("B,Hq,Hkv,P", [(1, 8, 2, 2000), (2, 4, 1, 1200)])
def test_running_max_jump_beyond_float_range(B, Hq, Hkv, P):
    # a row's max jumps by ~144 log2-units from one tile to the next (2^144 overflows fp32 and bf16)
    cfg = TINY.with_(B=B, Hq=Hq, Hkv=Hkv, D=128, k=3, P=P)
    inp = _plant_deep_first_tiles(cfg, synth.make_attn_inputs(cfg, seed=11))
    _check_full(cfg, inp=inp)


@pytest.mark.parametrize("seed", range(16))
def test_random_shapes(seed):
    """Seeded random shapes, every row against the oracle: batch 1..4 with ragged prefix lengths (short sequences
    beside long ones in one launch, so splits whose first key tile lies past a short prefix sit next to splits
    that keep it), 1..4 KV heads, group sizes 1..8, D 64 or 128, draft length 1..10, both mask modes."""
    rng = np.random.default_rng(1000 + seed)
    Hkv = int(rng.choice([1, 2, 4]))
    G = int(rng.choice([1, 2, 3, 4, 8]))
    hi = int(rng.integers(1, 2500))
    cfg = TINY.with_(B=int(rng.integers(1, 5)), Hq=Hkv * G, Hkv=Hkv, D=int(rng.choice([64, 128])),
                     k=int(rng.integers(1, 11)), P=hi, ragged=(0, hi))
    mode = oracle.MASK_HYBRID if seed % 3 else oracle.MASK_CAUSAL
    _check_full(cfg, seed=seed, mode=mode)


def test_group_rows_ignore_later_drafts_bitwise():
    cfg = TINY.with_(k=4, P=190, Hq=4, Hkv=2)
    k = cfg.k
    base = synth.make_attn_inputs(cfg, seed=5)
    o0, l0 = _gpu().attn(base, cfg.Hq, cfg.Hkv, cfg.D, k)
    rng = np.random.default_rng(0)
    for j in range(k + 1):
        pert = {n: v.copy() for n, v in base.items()}
        for n in ("k_new", "v_new"):
            pert[n][:, j:k] = synth.f32_to_bf16_bits(rng.standard_normal(pert[n][:, j:k].shape).astype(np.float32))
        o1, l1 = _gpu().attn(pert, cfg.Hq, cfg.Hkv, cfg.D, k)
        rows = slice(k + j * k, k + (j + 1) * k)
        assert np.array_equal(o0[:, rows], o1[:, rows]) and np.array_equal(l0[:, rows], l1[:, rows])
    pert = {n: v.copy() for n, v in base.items()}
    for n in ("k_new", "v_new"):
        pert[n][:, k:] = synth.f32_to_bf16_bits(rng.standard_normal(pert[n][:, k:].shape).astype(np.float32))
    o1, l1 = _gpu().attn(pert, cfg.Hq, cfg.Hkv, cfg.D, k)
    assert np.array_equal(o0[:, :k], o1[:, :k]) and np.array_equal(l0[:, :k], l1[:, :k])


def test_deterministic():
    cfg = synth.CONFIGS["qwen3-8b_k8"].with_(P=1000)
    inp = synth.make_attn_inputs(cfg, seed=2)
    a = _gpu().attn(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k)
    b = _gpu().attn(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_bad_prefix_sets_status_and_skips():
    cfg = TINY.with_(B=2)
    inp = synth.make_attn_inputs(cfg, seed=4)
    inp["prefix_len"] = np.array([cfg.P, cfg.P_max + 1], np.int32)
    o, lse, st = _gpu().attn(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, want_status=True)
    assert st & 1
    assert np.isnan(lse[1]).all()  # the bad sequence is left untouched
    inp2 = {n: v[:1] if n != "prefix_len" else v[:1] for n, v in inp.items()}
    o_ref, lse_ref, _ = oracle.attn(inp2, cfg.Hq, cfg.Hkv, cfg.D, cfg.k)
    assert np.abs(o[0] - o_ref[0]).max() <= O_TOL and np.abs(lse[0] - lse_ref[0]).max() <= LSE_TOL


@pytest.mark.parametrize("name", ["tiny", "qwen3-8b_k8"])
def test_wait_that_runs_out_sets_timeout_and_the_context_stays_usable(name):
    """The attention's on-chip waits are bounded.  The test hook makes one of them wait on a barrier nothing
    arrives on, with a bound of ~2e6 cycles (about 1 ms): the launch must return with TIDAR_DEV_TIMEOUT set,
    after draining its copies and MMAs and freeing its tensor memory, so that the next normal launch on the same
    context (every SM reallocates tensor memory) still matches the oracle.  On the Qwen3-8B shape every row tile
    is split over a cluster, so the aborted CTAs also pass the cluster exchange."""
    import torch

    from ar_lm_decoding_b200 import abi
    cfg = TINY.with_(P=1000, Hq=8, Hkv=2, D=128) if name == "tiny" else synth.CONFIGS[name]
    inp = synth.make_attn_inputs(cfg, seed=21)
    g = _gpu()
    q, kn, vn = g.dev_u16_as_bf16(inp["q"]), g.dev_u16_as_bf16(inp["k_new"]), g.dev_u16_as_bf16(inp["v_new"])
    kc, vc = g.dev_u16_as_bf16(inp["k_cache"]), g.dev_u16_as_bf16(inp["v_cache"])
    pl = g.to_dev(inp["prefix_len"].astype(np.int32))
    out = torch.zeros((cfg.B, cfg.R, cfg.Hq, cfg.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((cfg.B, cfg.R, cfg.Hq), dtype=torch.float32, device="cuda")
    for _ in range(2):  # twice in a row: the first launch left the SMs' tensor memory free
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        abi.tidar_testing_attn_step_stalled(q, kn, vn, kc, vc, pl, cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, cfg.P_max,
                                            1.0 / np.sqrt(cfg.D), abi.TIDAR_MASK_HYBRID, out, lse, st, 2_000_000)
        torch.cuda.synchronize()
        assert st.item() & abi.TIDAR_DEV_TIMEOUT, st.item()
    _check_full(cfg, seed=21, inp=inp) if name == "tiny" else None
    if name != "tiny":
        o, l_ = g.attn(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k)
        rows = np.random.default_rng(0).integers(0, cfg.R, 16)
        sb, sh = np.zeros(16, int), np.random.default_rng(1).integers(0, cfg.Hq, 16)
        o_ref, lse_ref = oracle.attn_rows(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, sb, sh, rows)
        assert np.abs(o[sb, rows, sh] - o_ref).max() <= O_TOL and np.abs(l_[sb, rows, sh] - lse_ref).max() <= LSE_TOL
