"""Several consecutive TiDAR decode steps on the GPU through the C ABI, against the same loop in the oracle.

One step is the pages' decode step ("TiDAR: Think in Diffusion, Talk in Autoregression", awesome-system-papers
summary, "并行 self-speculative 生成 (§3.2)"; notes.yuuk.io talk notes, §推論パイプライン): the forward over
[cached prefix | k drafts | k+1 pre-draft groups] (here: L tidar_attn_step calls), the AR rejection-sampling
verify of the drafts (tidar_verify), then the exact-KV commit and the choice of the next draft block from group
j* (tidar_kv_commit) -- or those two as one tidar_verify_commit call.  The state a step hands to the next stays
where a caller keeps it:

* on the GPU side, on the device: the per-layer KV caches and prefix_len (updated in place by the commit and
  read by the next step's attention), next_drafts and next_preaccepted (the next step's drafts and pre-accepted
  flags), and the next q logits, rows group_logits[b, next_q_group[b]] of this step's group logits;
* on the oracle side, in its own numpy copies, updated by the oracle's commit.

Every step compares every layer's output and LSE (2e-2 / 1e-4), the accept lengths, emitted and resampled
tokens, next drafts, next pre-accepted flags, next q group, prefix lengths and the full caches (bit-exact; the
1e-5 exemptions of tests/parity.py are reported and the oracle follows the GPU's decision).  The model's fresh
inputs of each step (Q / K_new / V_new per layer, the AR logits p, the group logits, the uniforms) are drawn
on the host; p carries a planted peak at the previous step's draft for a random number of leading slots and
every group row a planted peak, so that the accept length varies over 0..k across sequences and steps.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from ar_lm_decoding_b200 import abi, synth
from parity import compare_next_drafts, compare_verify

pytestmark = pytest.mark.gpu

DEV = "cuda"
O_TOL, LSE_TOL = 2e-2, 1e-4


def _bf16_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(DEV).view(torch.bfloat16)


def _logits_dev(a):
    if a.dtype == np.uint16:
        return _bf16_dev(a)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)


def _u16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


class Draws:
    """Seeded fresh inputs of each step (what the model forward would produce)."""

    def __init__(self, cfg, seed):
        self.cfg = cfg
        self.rng = np.random.default_rng(seed)

    def bf16(self, shape, sigma=1.0):
        return synth.f32_to_bf16_bits(self.rng.standard_normal(shape, dtype=np.float32) * np.float32(sigma))

    def logits(self, shape):
        return self.rng.standard_normal(shape, dtype=np.float32) * np.float32(self.cfg.sigma)

    def encode(self, z):
        return synth.f32_to_bf16_bits(z) if self.cfg.logits_dtype == "bf16" else np.ascontiguousarray(z)

    def uniforms(self, shape):
        bits = self.rng.integers(0, 2**32, size=shape, dtype=np.uint64).astype(np.uint32)
        return ((bits >> 8).astype(np.float32) * np.float32(2.0**-24)).astype(np.float32)

    def p_logits(self, drafts):
        """AR logits of the k slots: a planted peak at the draft on the first m slots (m ~ U{0..k} per
        sequence), at another token on the others."""
        B, k = drafts.shape
        z = self.logits((B, k, self.cfg.V))
        m = self.rng.integers(0, k + 1, size=B)
        for b in range(B):
            for i in range(k):
                t = int(drafts[b, i]) if i < m[b] else int((drafts[b, i] + 1 + self.rng.integers(0, self.cfg.V - 1))
                                                           % self.cfg.V)
                z[b, i, t] = z[b, i].max() + np.float32(2 * self.cfg.sigma)
        return self.encode(z)

    def group_logits(self):
        B, k, V = self.cfg.B, self.cfg.k, self.cfg.V
        z = self.logits((B, k + 1, k, V))
        peaks = self.rng.integers(0, V, size=(B, k + 1, k))
        for idx in np.ndindex(B, k + 1, k):
            z[idx][peaks[idx]] = z[idx].max() + np.float32(2 * self.cfg.sigma)
        return self.encode(z)


CASES = {
    "qwen-shaped k4 bf16": synth.CONFIGS["qwen2.5-1.5b_k4"].with_(L=3, Hq=4, Hkv=2, B=2, V=20000, ragged=(250, 400)),
    "k3 f32 D64 G4": synth.CONFIGS["tiny"].with_(L=2, Hq=8, Hkv=2, D=64, B=3, k=3, V=9000, sigma=3.0, peaks=True,
                                                 ragged=(100, 700)),
}


@pytest.mark.parametrize("fused", [False, True], ids=["verify+commit", "verify_commit"])
@pytest.mark.parametrize("name", list(CASES))
def test_decode_loop_matches_oracle(name, fused):
    """fused: the verify and the commit as one tidar_verify_commit call."""
    steps = 5
    cfg0 = CASES[name]
    # capacity for every step accepting the whole block
    cfg = cfg0.with_(P=cfg0.ragged[1] + steps * cfg0.k)
    B, L, R, Hq, Hkv, D, k, V = cfg.B, cfg.L, cfg.R, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, cfg.V
    P_max = cfg0.ragged[1] + (steps + 1) * k
    draws = Draws(cfg, seed=101 + list(CASES).index(name))
    pl0 = synth.prefix_lengths(cfg0, seed=1)
    # caches: rows at or beyond each prefix length are NaN (never valid until committed)
    kc = np.stack([draws.bf16((B, Hkv, P_max, D)) for _ in range(L)])
    vc = np.stack([draws.bf16((B, Hkv, P_max, D)) for _ in range(L)])
    for b in range(B):
        kc[:, b, :, pl0[b]:] = synth.BF16_NAN
        vc[:, b, :, pl0[b]:] = synth.BF16_NAN
    vin = synth.make_verify_inputs(cfg0.with_(peaks=True), seed=3)
    # ---- the oracle's state
    o_kc, o_vc, o_pl = kc.copy(), vc.copy(), pl0.copy()
    o_drafts, o_q, o_pre = vin["drafts"].copy(), vin["q_logits"].copy(), vin["preaccepted"].copy()
    # ---- the GPU's state (device)
    g_kc = [_bf16_dev(kc[l]) for l in range(L)]
    g_vc = [_bf16_dev(vc[l]) for l in range(L)]
    g_pl = torch.from_numpy(pl0.astype(np.int32)).to(DEV)
    g_drafts = torch.from_numpy(vin["drafts"].astype(np.int32)).to(DEV)
    g_pre = torch.from_numpy(vin["preaccepted"].astype(np.uint8)).to(DEV)
    g_q = _logits_dev(vin["q_logits"])
    dt = abi.TIDAR_DT_BF16 if cfg.logits_dtype == "bf16" else abi.TIDAR_DT_F32
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    ws = torch.empty(max(abi.tidar_verify_workspace_size(B, k, V), abi.tidar_kv_commit_workspace_size(B, k, V),
                         abi.tidar_verify_commit_workspace_size(B, k, V)), dtype=torch.uint8, device=DEV)
    report, accept_seen = [], []
    for step in range(steps):
        # fresh model outputs of this step
        q = [draws.bf16((B, R, Hq, D)) for _ in range(L)]
        kn = np.stack([draws.bf16((B, R, Hkv, D)) for _ in range(L)])
        vn = np.stack([draws.bf16((B, R, Hkv, D)) for _ in range(L)])
        p_logits = draws.p_logits(o_drafts)
        g_logits = draws.group_logits()
        u_acc, u_res, u_draft = draws.uniforms((B, k)), draws.uniforms((B,)), draws.uniforms((B, k))

        # ---- GPU: L attention layers, verify, commit (state read from and written to the device)
        g_kn = [_bf16_dev(kn[l]) for l in range(L)]
        g_vn = [_bf16_dev(vn[l]) for l in range(L)]
        outs, lses = [], []
        for l in range(L):
            o = torch.full((B, R, Hq, D), float("nan"), dtype=torch.bfloat16, device=DEV)
            lse = torch.full((B, R, Hq), float("nan"), dtype=torch.float32, device=DEV)
            abi.tidar_attn_step(_bf16_dev(q[l]), g_kn[l], g_vn[l], g_kc[l], g_vc[l], g_pl, B, Hq, Hkv, D, k, P_max,
                                1.0 / math.sqrt(D), abi.TIDAR_MASK_HYBRID, o, lse, None, 0, status)
            outs.append(o)
            lses.append(lse)
        g_p, g_g = _logits_dev(p_logits), _logits_dev(g_logits)
        acc = torch.full((B,), -7, dtype=torch.int32, device=DEV)
        res = torch.full((B,), -7, dtype=torch.int32, device=DEV)
        tok = torch.full((B, k), -7, dtype=torch.int32, device=DEV)
        nem = torch.full((B,), -7, dtype=torch.int32, device=DEV)
        lp = torch.zeros((B, k), dtype=torch.float32, device=DEV)
        lq = torch.zeros((B, k), dtype=torch.float32, device=DEV)
        nd = torch.full((B, k), -7, dtype=torch.int32, device=DEV)
        npre = torch.full((B,), 7, dtype=torch.uint8, device=DEV)
        nqg = torch.full((B,), -7, dtype=torch.int32, device=DEV)
        if fused:
            abi.tidar_verify_commit(g_p, g_q, dt, g_drafts, g_pre, torch.from_numpy(u_acc).to(DEV),
                                    torch.from_numpy(u_res).to(DEV), 1.0, abi.pointer_array(g_kc, DEV),
                                    abi.pointer_array(g_vc, DEV), abi.pointer_array(g_kn, DEV),
                                    abi.pointer_array(g_vn, DEV), None, 0, 0, L, B, Hkv, D, k, P_max, V, g_pl, g_g,
                                    torch.from_numpy(u_draft).to(DEV), acc, res, tok, nem, lp, lq, nd, npre, nqg, ws,
                                    ws.numel(), status)
        else:
            abi.tidar_verify(g_p, g_q, dt, g_drafts, g_pre, torch.from_numpy(u_acc).to(DEV),
                             torch.from_numpy(u_res).to(DEV), B, k, V, acc, res, tok, nem, lp, lq, ws, ws.numel(),
                             status)
            abi.tidar_kv_commit(abi.pointer_array(g_kc, DEV), abi.pointer_array(g_vc, DEV),
                                abi.pointer_array(g_kn, DEV), abi.pointer_array(g_vn, DEV), L, B, Hkv, D, k, P_max,
                                g_pl, acc, res, g_g, dt, V, torch.from_numpy(u_draft).to(DEV), nd, npre, nqg, ws,
                                ws.numel(), status)
        torch.cuda.synchronize()
        assert status.item() == 0, (step, status.item())

        # ---- oracle: the same step on its own state
        o_inp = dict(q=None, k_new=None, v_new=None, k_cache=None, v_cache=None, prefix_len=o_pl)
        for l in range(L):
            o_inp.update(q=q[l], k_new=kn[l], v_new=vn[l], k_cache=o_kc[l], v_cache=o_vc[l])
            o_ref, lse_ref, _ = oracle.attn(o_inp, Hq, Hkv, D, k, dense=False)
            eo = np.abs(outs[l].float().cpu().numpy() - o_ref).max()
            el = np.abs(lses[l].cpu().numpy() - lse_ref).max()
            assert eo <= O_TOL and el <= LSE_TOL, (step, l, eo, el)
        v_inp = dict(p_logits=p_logits, q_logits=o_q, drafts=o_drafts, preaccepted=o_pre, u_acc=u_acc, u_res=u_res)
        got_v = dict(accept_len=acc.cpu().numpy(), resampled=res.cpu().numpy(), tokens=tok.cpu().numpy(),
                     n_emitted=nem.cpu().numpy(), logp_d=lp.cpu().numpy(), logq_d=lq.cpu().numpy())
        ref_v = compare_verify(v_inp, got_v, report)
        c = oracle.kv_commit(o_kc, o_vc, kn, vn, o_pl, ref_v["accept_len"], ref_v["resampled"], g_logits, u_draft)
        got_c = dict(next_drafts=nd.cpu().numpy(), next_preaccepted=npre.cpu().numpy(),
                     next_q_group=nqg.cpu().numpy(), prefix_len=g_pl.cpu().numpy())
        o_next = compare_next_drafts(got_c, c, u_draft, report)
        assert np.array_equal(got_c["prefix_len"], c["prefix_len"]), step
        assert np.array_equal(got_c["next_q_group"], c["next_q_group"]), step
        assert np.array_equal(got_c["next_preaccepted"], c["next_preaccepted"]), step
        for l in range(L):
            assert np.array_equal(_u16(g_kc[l]), c["k_caches"][l]), (step, l)
            assert np.array_equal(_u16(g_vc[l]), c["v_caches"][l]), (step, l)
        accept_seen += got_v["accept_len"].tolist()

        # ---- hand the state to the next step, each side from its own outputs
        o_kc, o_vc, o_pl = c["k_caches"], c["v_caches"], c["prefix_len"]
        o_drafts, o_pre = o_next, c["next_preaccepted"]
        o_q = np.ascontiguousarray(g_logits[np.arange(B), c["next_q_group"]])
        g_drafts, g_pre = nd, npre
        g_q = g_g[torch.arange(B, device=DEV), nqg.long()].contiguous()  # rows group_logits[b, j*]
    print(f"{name}: accept lengths {accept_seen}, exemptions {report}")
    assert len(set(accept_seen)) >= 3  # the planted peaks drive several accept lengths
    assert len(report) <= 2
