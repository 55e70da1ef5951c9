"""Run the CUDA library (through its C ABI) on the numpy inputs of ar_lm_decoding_b200.synth."""
from __future__ import annotations

import math

import numpy as np
import torch

from ar_lm_decoding_b200 import abi

DEV = "cuda"


def dev_u16_as_bf16(a: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(DEV)
    return t.view(torch.bfloat16)


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def logits_dev(a: np.ndarray):
    if a.dtype == np.uint16:
        return dev_u16_as_bf16(a), abi.TIDAR_DT_BF16
    return to_dev(a.astype(np.float32)), abi.TIDAR_DT_F32


def workspace(nbytes: int) -> torch.Tensor:
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=DEV)


def attn(inp: dict, Hq: int, Hkv: int, D: int, k: int, mode: int = abi.TIDAR_MASK_HYBRID, scale=None,
         want_status=False, fill_ws_nan=True):
    q = dev_u16_as_bf16(inp["q"])
    B, R = q.shape[0], q.shape[1]
    P_max = inp["k_cache"].shape[2]
    kn, vn = dev_u16_as_bf16(inp["k_new"]), dev_u16_as_bf16(inp["v_new"])
    kc, vc = dev_u16_as_bf16(inp["k_cache"]), dev_u16_as_bf16(inp["v_cache"])
    pl = to_dev(inp["prefix_len"].astype(np.int32))
    out = torch.full((B, R, Hq, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, R, Hq), float("nan"), dtype=torch.float32, device=DEV)
    nbytes = abi.tidar_attn_workspace_size(B, Hq, Hkv, D, k, P_max)
    ws = workspace(nbytes)
    if fill_ws_nan:
        ws.view(torch.uint8).fill_(0xFF)  # NaN canaries: a workspace read before its write shows up
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    abi.tidar_attn_step(q, kn, vn, kc, vc, pl, B, Hq, Hkv, D, k, P_max,
                        1.0 / math.sqrt(D) if scale is None else scale, mode, out, lse, ws, ws.numel(), st)
    torch.cuda.synchronize()
    res = (out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64))
    if want_status:
        return res + (int(st.item()),)
    assert st.item() == 0, f"device status {st.item()}"
    return res


def verify(inp: dict, want_status=False, trust_ar=None):
    """tidar_verify on the numpy inputs (tidar_verify_trust_mix when trust_ar is given)."""
    p, dt = logits_dev(inp["p_logits"])
    q, _ = logits_dev(inp["q_logits"])
    B, k, V = inp["p_logits"].shape
    outs = dict(accept_len=torch.full((B,), -7, dtype=torch.int32, device=DEV),
                resampled=torch.full((B,), -7, dtype=torch.int32, device=DEV),
                tokens=torch.full((B, k), -7, dtype=torch.int32, device=DEV),
                n_emitted=torch.full((B,), -7, dtype=torch.int32, device=DEV),
                logp_d=torch.zeros((B, k), dtype=torch.float32, device=DEV),
                logq_d=torch.zeros((B, k), dtype=torch.float32, device=DEV))
    ws = workspace(abi.tidar_verify_workspace_size(B, k, V))
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    args = (p, q, dt, to_dev(inp["drafts"].astype(np.int32)), to_dev(inp["preaccepted"].astype(np.uint8)),
            to_dev(inp["u_acc"].astype(np.float32)), to_dev(inp["u_res"].astype(np.float32)), B, k, V)
    rest = (outs["accept_len"], outs["resampled"], outs["tokens"], outs["n_emitted"], outs["logp_d"],
            outs["logq_d"], ws, ws.numel(), st)
    if trust_ar is None:
        abi.tidar_verify(*args, *rest)
    else:
        abi.tidar_verify_trust_mix(*args, trust_ar, *rest)
    torch.cuda.synchronize()
    res = {n: t.cpu().numpy() for n, t in outs.items()}
    if want_status:
        res["status"] = int(st.item())
    else:
        assert st.item() == 0, f"device status {st.item()}"
    return res


def kv_commit(k_caches, v_caches, k_news, v_news, prefix_len, accept_len, resampled, group_logits, u_draft,
              want_status=False):
    """Caches [L,B,Hkv,P_max,D], new K/V [L,B,R,Hkv,D] (uint16 bf16 bits); returns host copies."""
    L, B, Hkv, P_max, D = k_caches.shape
    kc = [dev_u16_as_bf16(k_caches[l]) for l in range(L)]
    vc = [dev_u16_as_bf16(v_caches[l]) for l in range(L)]
    kn = [dev_u16_as_bf16(k_news[l]) for l in range(L)]
    vn = [dev_u16_as_bf16(v_news[l]) for l in range(L)]
    g, dt = logits_dev(group_logits)
    k = group_logits.shape[2]
    V = group_logits.shape[3]
    pl = to_dev(np.asarray(prefix_len, np.int32))
    nd = torch.full((B, k), -7, dtype=torch.int32, device=DEV)
    npre = torch.full((B,), 7, dtype=torch.uint8, device=DEV)
    nqg = torch.full((B,), -7, dtype=torch.int32, device=DEV)
    ws = workspace(abi.tidar_kv_commit_workspace_size(B, k, V))
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    abi.tidar_kv_commit(abi.pointer_array(kc, DEV), abi.pointer_array(vc, DEV), abi.pointer_array(kn, DEV),
                        abi.pointer_array(vn, DEV), L, B, Hkv, D, k, P_max, pl,
                        to_dev(np.asarray(accept_len, np.int32)), to_dev(np.asarray(resampled, np.int32)), g, dt, V,
                        to_dev(np.asarray(u_draft, np.float32)), nd, npre, nqg, ws, ws.numel(), st)
    torch.cuda.synchronize()

    def back(ts):
        return np.stack([t.view(torch.int16).cpu().numpy().view(np.uint16) for t in ts])

    res = dict(k_caches=back(kc), v_caches=back(vc), prefix_len=pl.cpu().numpy(), next_drafts=nd.cpu().numpy(),
               next_preaccepted=npre.cpu().numpy(), next_q_group=nqg.cpu().numpy(), status=int(st.item()))
    if not want_status:
        assert res["status"] == 0, f"device status {res['status']}"
    return res


def verify_commit(inp: dict, k_caches, v_caches, k_news, v_news, prefix_len, trust_ar=1.0, want_status=False):
    """tidar_verify_commit on the numpy verify inputs (with group_logits and u_draft) and contiguous caches
    [L,B,Hkv,P_max,D] / new K/V [L,B,R,Hkv,D] (uint16 bf16 bits); returns host copies of every output."""
    L, B, Hkv, P_max, D = k_caches.shape
    p, dt = logits_dev(inp["p_logits"])
    q, _ = logits_dev(inp["q_logits"])
    g, _ = logits_dev(inp["group_logits"])
    _, k, V = inp["p_logits"].shape
    kc = [dev_u16_as_bf16(k_caches[l]) for l in range(L)]
    vc = [dev_u16_as_bf16(v_caches[l]) for l in range(L)]
    kn = [dev_u16_as_bf16(k_news[l]) for l in range(L)]
    vn = [dev_u16_as_bf16(v_news[l]) for l in range(L)]
    pl = to_dev(np.asarray(prefix_len, np.int32))
    i32 = dict(dtype=torch.int32, device=DEV)
    outs = dict(accept_len=torch.full((B,), -7, **i32), resampled=torch.full((B,), -7, **i32),
                tokens=torch.full((B, k), -7, **i32), n_emitted=torch.full((B,), -7, **i32),
                logp_d=torch.zeros((B, k), dtype=torch.float32, device=DEV),
                logq_d=torch.zeros((B, k), dtype=torch.float32, device=DEV),
                next_drafts=torch.full((B, k), -7, **i32),
                next_preaccepted=torch.full((B,), 7, dtype=torch.uint8, device=DEV),
                next_q_group=torch.full((B,), -7, **i32))
    ws = workspace(abi.tidar_verify_commit_workspace_size(B, k, V))
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = outs
    abi.tidar_verify_commit(p, q, dt, to_dev(inp["drafts"].astype(np.int32)),
                            to_dev(inp["preaccepted"].astype(np.uint8)), to_dev(inp["u_acc"].astype(np.float32)),
                            to_dev(inp["u_res"].astype(np.float32)), trust_ar, abi.pointer_array(kc, DEV),
                            abi.pointer_array(vc, DEV), abi.pointer_array(kn, DEV), abi.pointer_array(vn, DEV), None, 0,
                            0, L, B, Hkv, D, k, P_max, V, pl, g, to_dev(inp["u_draft"].astype(np.float32)),
                            o["accept_len"], o["resampled"], o["tokens"], o["n_emitted"], o["logp_d"], o["logq_d"],
                            o["next_drafts"], o["next_preaccepted"], o["next_q_group"], ws, ws.numel(), st)
    torch.cuda.synchronize()

    def back(ts):
        return np.stack([t.view(torch.int16).cpu().numpy().view(np.uint16) for t in ts])

    res = {n: t.cpu().numpy() for n, t in outs.items()}
    res.update(k_caches=back(kc), v_caches=back(vc), prefix_len=pl.cpu().numpy(), status=int(st.item()))
    if not want_status:
        assert res["status"] == 0, f"device status {res['status']}"
    return res
