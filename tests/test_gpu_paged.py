"""Paged KV cache (tidar_attn_step_paged, tidar_kv_commit_paged, tidar_verify_commit with a block table) on the GPU.

A paged cache is a storage layout: cache row n of sequence b is row n % 64 of page block_table[b][n / 64] of a
pool shared by all sequences.  The tests scatter the rows of contiguous caches over randomly permuted pages of a
pool whose other pages hold NaN, so a read of a wrong page shows, and require:
  * attention: the same bits as tidar_attn_step on the contiguous caches, and the oracle's results (2e-2 / 1e-4);
  * commit: the oracle's commit applied to the contiguous caches, read back through the block table (bit-exact),
    and nothing outside the accepted rows written;
  * a continuous-batching loop: sequences at different prefix lengths decode step after step, finished sequences
    give their pages back and new ones join with pages from the free list, each step checked against the oracle.
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
PAGE = 64
O_TOL, LSE_TOL = 2e-2, 1e-4


def _bf16_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(DEV).view(torch.bfloat16)


def _u16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


class Pool:
    """Host model of paged caches: per layer a pool (uint16 bf16 bits [num_pages, Hkv, 64, D]) of K and of V,
    one block table [B, max_pages] and one free list shared by the layers (a page id names the same page in
    every layer's pool)."""

    def __init__(self, L, num_pages, Hkv, D, B, max_pages, rng):
        self.k = [np.full((num_pages, Hkv, PAGE, D), synth.BF16_NAN, np.uint16) for _ in range(L)]
        self.v = [a.copy() for a in self.k]
        self.table = np.full((B, max_pages), -1, np.int32)
        self.free = [int(x) for x in rng.permutation(num_pages)]
        self.max_pages = max_pages

    def ensure(self, b, rows):
        """Pages for rows [0, rows) of sequence b (taken from the free list)."""
        for i in range((rows + PAGE - 1) // PAGE):
            if self.table[b, i] < 0:
                self.table[b, i] = self.free.pop()

    def release(self, b):
        for i in range(self.max_pages):
            pg = self.table[b, i]
            if pg >= 0:
                for a in self.k + self.v:
                    a[pg] = synth.BF16_NAN
                self.free.append(int(pg))
                self.table[b, i] = -1

    def write_rows(self, l, b, kc, vc, rows):
        """Scatter contiguous rows [0, rows) ([Hkv, rows, D]) of sequence b of layer l into its pages."""
        self.ensure(b, rows)
        for n in range(rows):
            pg = self.table[b, n // PAGE]
            self.k[l][pg, :, n % PAGE] = kc[:, n]
            self.v[l][pg, :, n % PAGE] = vc[:, n]

    def gather(self, l, b, P_max):
        """Contiguous [Hkv, P_max, D] view of sequence b of layer l (rows without a page: NaN)."""
        Hkv, D = self.k[l].shape[1], self.k[l].shape[3]
        kc = np.full((Hkv, P_max, D), synth.BF16_NAN, np.uint16)
        vc = kc.copy()
        for i in range(P_max // PAGE):
            pg = self.table[b, i]
            if pg >= 0:
                kc[:, i * PAGE:(i + 1) * PAGE] = self.k[l][pg]
                vc[:, i * PAGE:(i + 1) * PAGE] = self.v[l][pg]
        return kc, vc


def _paged_attn(pool_k, pool_v, table, inp, cfg, num_pages):
    B, R, Hq, Hkv, D, k = cfg.B, cfg.R, cfg.Hq, cfg.Hkv, cfg.D, cfg.k
    out = torch.full((B, R, Hq, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, R, Hq), float("nan"), dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    abi.tidar_attn_step_paged(_bf16_dev(inp["q"]), _bf16_dev(inp["k_new"]), _bf16_dev(inp["v_new"]), pool_k, pool_v,
                              torch.from_numpy(table).to(DEV), table.shape[1], num_pages,
                              torch.from_numpy(inp["prefix_len"].astype(np.int32)).to(DEV), B, Hq, Hkv, D, k,
                              1.0 / math.sqrt(D), abi.TIDAR_MASK_HYBRID, out, lse, st)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64), int(st.item())


@pytest.mark.parametrize("case", ["qwen3-8b b8 ragged", "small G3 D64 k3"])
def test_paged_attention_equals_contiguous_and_oracle(case):
    if case == "qwen3-8b b8 ragged":
        cfg = synth.CONFIGS["qwen3-8b_k8_b8"].with_(ragged=(1, 2500))
    else:
        cfg = synth.CONFIGS["tiny"].with_(B=3, Hq=6, Hkv=2, D=64, k=3, ragged=(0, 700))
    rng = np.random.default_rng(8)
    inp = synth.make_attn_inputs(cfg, seed=5)
    max_pages = cfg.P_max // PAGE
    num_pages = cfg.B * max_pages + 7
    pool = Pool(1, num_pages, cfg.Hkv, cfg.D, cfg.B, max_pages, rng)
    for b in range(cfg.B):
        pool.write_rows(0, b, inp["k_cache"][b], inp["v_cache"][b], int(inp["prefix_len"][b]))
    o, lse, st = _paged_attn(_bf16_dev(pool.k[0]), _bf16_dev(pool.v[0]), pool.table, inp, cfg, num_pages)
    assert st == 0
    import tidar_gpu
    oc, lc = tidar_gpu.attn(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k)
    assert np.array_equal(o, oc) and np.array_equal(lse, lc)  # same arithmetic, another layout
    o_ref, lse_ref, _ = oracle.attn(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, dense=False)
    assert np.abs(o - o_ref).max() <= O_TOL and np.abs(lse - lse_ref).max() <= LSE_TOL


@pytest.mark.parametrize("seed", range(8))
def test_paged_attention_random_shapes(seed):
    """Seeded random shapes over randomly permuted pages: batch 1-4 with ragged prefixes (0 included), 1-4 KV heads,
    group sizes 1-4, D 64 or 128, k 1-10; the same bits as the contiguous call and the oracle's results."""
    rng = np.random.default_rng(3000 + seed)
    Hkv = int(rng.choice([1, 2, 4]))
    cfg = synth.CONFIGS["tiny"].with_(B=int(rng.integers(1, 5)), Hq=Hkv * int(rng.integers(1, 5)), Hkv=Hkv,
                                      D=int(rng.choice([64, 128])), k=int(rng.integers(1, 11)),
                                      ragged=(0, int(rng.integers(1, 1500))))
    inp = synth.make_attn_inputs(cfg, seed=seed)
    max_pages = cfg.P_max // PAGE
    num_pages = cfg.B * max_pages + int(rng.integers(0, 9))
    pool = Pool(1, num_pages, cfg.Hkv, cfg.D, cfg.B, max_pages, rng)
    for b in range(cfg.B):
        pool.write_rows(0, b, inp["k_cache"][b], inp["v_cache"][b], int(inp["prefix_len"][b]))
    o, lse, st = _paged_attn(_bf16_dev(pool.k[0]), _bf16_dev(pool.v[0]), pool.table, inp, cfg, num_pages)
    assert st == 0
    import tidar_gpu
    oc, lc = tidar_gpu.attn(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k)
    assert np.array_equal(o, oc) and np.array_equal(lse, lc)
    o_ref, lse_ref, _ = oracle.attn(inp, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, dense=False)
    assert np.abs(o - o_ref).max() <= O_TOL and np.abs(lse - lse_ref).max() <= LSE_TOL


def test_paged_attention_bad_page_sets_status_and_skips():
    cfg = synth.CONFIGS["tiny"].with_(B=2, P=300)
    rng = np.random.default_rng(9)
    inp = synth.make_attn_inputs(cfg, seed=6)
    max_pages = cfg.P_max // PAGE
    pool = Pool(1, 2 * max_pages, cfg.Hkv, cfg.D, cfg.B, max_pages, rng)
    for b in range(cfg.B):
        pool.write_rows(0, b, inp["k_cache"][b], inp["v_cache"][b], cfg.P)
    table = pool.table.copy()
    table[1, 2] = 2 * max_pages  # outside the pool
    o, lse, st = _paged_attn(_bf16_dev(pool.k[0]), _bf16_dev(pool.v[0]), table, inp, cfg, 2 * max_pages)
    assert st & abi.TIDAR_DEV_BAD_PAGE
    assert np.isnan(lse[1]).all()  # that sequence is left untouched
    o_ref, lse_ref, _ = oracle.attn({n: v[:1] for n, v in inp.items()}, cfg.Hq, cfg.Hkv, cfg.D, cfg.k)
    assert np.abs(o[0] - o_ref[0]).max() <= O_TOL and np.abs(lse[0] - lse_ref[0]).max() <= LSE_TOL


@pytest.mark.parametrize("fused", [False, True], ids=["verify+commit", "verify_commit"])
def test_paged_continuous_batching_loop(fused):
    """Four sequence slots decode for six steps; when a slot's sequence reaches its length it is replaced by a
    new sequence (fresh prefix in fresh pages).  Attention (2 layers), verify and the paged commit run on the
    GPU with the block table and pools on the device; the oracle runs the same steps on gathered contiguous
    caches, and the pools read back through the block table must equal its caches."""
    cfg = synth.CONFIGS["qwen2.5-1.5b_k4"].with_(L=2, Hq=4, Hkv=2, B=4, V=12000, ragged=(1, 330))
    B, L, R, Hq, Hkv, D, k, V = cfg.B, cfg.L, cfg.R, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, cfg.V
    rng = np.random.default_rng(12)
    max_pages = 8
    P_max = max_pages * PAGE
    num_pages = B * max_pages + 4
    pool = Pool(L, num_pages, Hkv, D, B, max_pages, rng)
    prefix = np.zeros(B, np.int32)
    limit = np.zeros(B, np.int32)

    def start(b):
        P = int(rng.integers(1, 330))
        pool.release(b)
        for l in range(L):
            kc = synth.f32_to_bf16_bits(rng.standard_normal((Hkv, P, D), dtype=np.float32))
            vc = synth.f32_to_bf16_bits(rng.standard_normal((Hkv, P, D), dtype=np.float32))
            pool.write_rows(l, b, kc, vc, P)
        pool.ensure(b, P + k)
        prefix[b] = P
        limit[b] = min(P + 3 * k, P_max - k)

    for b in range(B):
        start(b)
    vin = synth.make_verify_inputs(cfg.with_(peaks=True), seed=4)
    drafts, q_log, pre = vin["drafts"].copy(), vin["q_logits"].copy(), vin["preaccepted"].copy()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    ws = torch.empty(max(abi.tidar_verify_workspace_size(B, k, V), abi.tidar_kv_commit_workspace_size(B, k, V),
                         abi.tidar_verify_commit_workspace_size(B, k, V)), dtype=torch.uint8, device=DEV)
    report, turnovers = [], 0
    for step in range(6):
        table_d = torch.from_numpy(pool.table).to(DEV)
        g_kp = [_bf16_dev(pool.k[l]) for l in range(L)]
        g_vp = [_bf16_dev(pool.v[l]) for l in range(L)]
        g_pl = torch.from_numpy(prefix.copy()).to(DEV)
        q = [synth.f32_to_bf16_bits(rng.standard_normal((B, R, Hq, D), dtype=np.float32)) for _ in range(L)]
        kn = np.stack([synth.f32_to_bf16_bits(rng.standard_normal((B, R, Hkv, D), dtype=np.float32)) for _ in range(L)])
        vn = np.stack([synth.f32_to_bf16_bits(rng.standard_normal((B, R, Hkv, D), dtype=np.float32)) for _ in range(L)])
        # oracle view: contiguous caches gathered through the block table
        o_kc = np.stack([np.stack([pool.gather(l, b, P_max)[0] for b in range(B)]) for l in range(L)])
        o_vc = np.stack([np.stack([pool.gather(l, b, P_max)[1] for b in range(B)]) for l in range(L)])
        for l in range(L):
            inp = dict(q=q[l], k_new=kn[l], v_new=vn[l], k_cache=o_kc[l], v_cache=o_vc[l], prefix_len=prefix.copy())
            o, lse, st = _paged_attn(g_kp[l], g_vp[l], pool.table, inp, cfg, num_pages)
            assert st == 0
            o_ref, lse_ref, _ = oracle.attn(inp, Hq, Hkv, D, k, dense=False)
            assert np.abs(o - o_ref).max() <= O_TOL and np.abs(lse - lse_ref).max() <= LSE_TOL, (step, l)
        # verify (planted peaks at the drafts on a random number of leading slots)
        zp = rng.standard_normal((B, k, V), dtype=np.float32) * np.float32(3)
        m = rng.integers(0, k + 1, B)
        for b in range(B):
            for i in range(k):
                t = int(drafts[b, i]) if i < m[b] else int((drafts[b, i] + 1) % V)
                zp[b, i, t] = zp[b, i].max() + np.float32(6)
        g_logits = synth.f32_to_bf16_bits(rng.standard_normal((B, k + 1, k, V), dtype=np.float32) * np.float32(3))
        v_inp = dict(p_logits=synth.f32_to_bf16_bits(zp), q_logits=q_log, drafts=drafts, preaccepted=pre,
                     u_acc=rng.random((B, k)).astype(np.float32), u_res=rng.random(B).astype(np.float32))
        import tidar_gpu
        u_draft = rng.random((B, k)).astype(np.float32)
        g_kn = [_bf16_dev(kn[l]) for l in range(L)]
        g_vn = [_bf16_dev(vn[l]) for l in range(L)]
        nd = torch.full((B, k), -7, dtype=torch.int32, device=DEV)
        npre = torch.full((B,), 7, dtype=torch.uint8, device=DEV)
        nqg = torch.full((B,), -7, dtype=torch.int32, device=DEV)
        if fused:  # verify and paged commit in one launch
            outs = [torch.full((B,), -7, dtype=torch.int32, device=DEV) for _ in range(3)]
            tok = torch.full((B, k), -7, dtype=torch.int32, device=DEV)
            lp = torch.zeros((B, k), dtype=torch.float32, device=DEV)
            lq = torch.zeros((B, k), dtype=torch.float32, device=DEV)
            abi.tidar_verify_commit(_bf16_dev(v_inp["p_logits"]), _bf16_dev(q_log), abi.TIDAR_DT_BF16,
                                    torch.from_numpy(drafts.astype(np.int32)).to(DEV),
                                    torch.from_numpy(pre.astype(np.uint8)).to(DEV),
                                    torch.from_numpy(v_inp["u_acc"]).to(DEV), torch.from_numpy(v_inp["u_res"]).to(DEV),
                                    1.0, abi.pointer_array(g_kp, DEV), abi.pointer_array(g_vp, DEV),
                                    abi.pointer_array(g_kn, DEV), abi.pointer_array(g_vn, DEV), table_d, max_pages,
                                    num_pages, L, B, Hkv, D, k, 0, V, g_pl, _bf16_dev(g_logits),
                                    torch.from_numpy(u_draft).to(DEV), outs[0], outs[1], tok, outs[2], lp, lq, nd,
                                    npre, nqg, ws, ws.numel(), status)
            torch.cuda.synchronize()
            got_v = dict(accept_len=outs[0].cpu().numpy(), resampled=outs[1].cpu().numpy(),
                         tokens=tok.cpu().numpy(), n_emitted=outs[2].cpu().numpy(), logp_d=lp.cpu().numpy(),
                         logq_d=lq.cpu().numpy())
            ref_v = compare_verify(v_inp, got_v, report)
        else:
            got_v = tidar_gpu.verify(v_inp)
            ref_v = compare_verify(v_inp, got_v, report)
            # paged commit on the GPU
            abi.tidar_kv_commit_paged(abi.pointer_array(g_kp, DEV), abi.pointer_array(g_vp, DEV),
                                      abi.pointer_array(g_kn, DEV), abi.pointer_array(g_vn, DEV), table_d, max_pages,
                                      num_pages, L, B, Hkv, D, k, g_pl,
                                      torch.from_numpy(got_v["accept_len"]).to(DEV),
                                      torch.from_numpy(got_v["resampled"]).to(DEV), _bf16_dev(g_logits),
                                      abi.TIDAR_DT_BF16, V, torch.from_numpy(u_draft).to(DEV), nd, npre, nqg, ws,
                                      ws.numel(), status)
        torch.cuda.synchronize()
        assert status.item() == 0
        c = oracle.kv_commit(o_kc, o_vc, kn, vn, prefix, ref_v["accept_len"], ref_v["resampled"], g_logits, u_draft)
        got_c = dict(next_drafts=nd.cpu().numpy(), next_preaccepted=npre.cpu().numpy(),
                     next_q_group=nqg.cpu().numpy(), prefix_len=g_pl.cpu().numpy())
        nxt = compare_next_drafts(got_c, c, u_draft, report)
        assert np.array_equal(got_c["prefix_len"], c["prefix_len"])
        for l in range(L):  # the pools, read back through the block table, equal the oracle's caches
            pool.k[l] = _u16(g_kp[l])
            pool.v[l] = _u16(g_vp[l])
            for b in range(B):
                gk, gv = pool.gather(l, b, P_max)
                assert np.array_equal(gk, c["k_caches"][l, b]) and np.array_equal(gv, c["v_caches"][l, b]), (step, l, b)
        prefix = c["prefix_len"].astype(np.int32)
        drafts, pre = nxt, c["next_preaccepted"]
        q_log = np.ascontiguousarray(g_logits[np.arange(B), c["next_q_group"]])
        for b in range(B):  # finished sequences leave, new ones join in fresh pages
            if prefix[b] >= limit[b]:
                start(b)
                pre[b] = 0
                turnovers += 1
            else:
                pool.ensure(b, int(prefix[b]) + k)
    print(f"turnovers {turnovers}, exemptions {report}")
    assert turnovers >= 1
    assert len(report) <= 2
