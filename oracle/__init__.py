"""ctypes front end of the CPU oracle (oracle.c).

TEST INFRASTRUCTURE: only the tests, the smoke check and the benchmark's CPU
baseline use this package.  The product library never imports it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None

MASK_HYBRID, MASK_CAUSAL = 0, 1
LOGITS_BF16, LOGITS_F32 = 0, 1


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "oracle.c")
    hdr = os.path.join(_HERE, "oracle.h")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < max(os.path.getmtime(src), os.path.getmtime(hdr)):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", tmp, src, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def default_threads() -> int:
    return len(os.sched_getaffinity(0))


def hybrid_mask(k: int, P: int, mode: int = MASK_HYBRID) -> np.ndarray:
    R = k * (k + 2)
    m = np.zeros((R, P + R), dtype=np.uint8)
    rc = lib().oracle_hybrid_mask(ctypes.c_int(k), ctypes.c_int(P), ctypes.c_int(mode), _p(m))
    if rc:
        raise ValueError("oracle_hybrid_mask: invalid arguments")
    return m.astype(bool)


def attn(inp: dict, Hq: int, Hkv: int, D: int, k: int, scale: float | None = None, mode: int = MASK_HYBRID,
         dense: bool = True, nthreads: int = 0):
    """One layer of hybrid-mask attention; returns (o float64 [B,R,Hq,D], lse float64 [B,R,Hq], o_bf16 uint16)."""
    q = _c(inp["q"], np.uint16)
    B, R = q.shape[0], q.shape[1]
    P_max = inp["k_cache"].shape[2]
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    o = np.zeros((B, R, Hq, D), dtype=np.float64)
    lse = np.zeros((B, R, Hq), dtype=np.float64)
    ob = np.zeros((B, R, Hq, D), dtype=np.uint16)
    args = [_c(inp[n], np.uint16) for n in ("k_new", "v_new", "k_cache", "v_cache")]
    pl = _c(inp["prefix_len"], np.int32)
    rc = lib().oracle_attn(_p(q), *[_p(a) for a in args], _p(pl),
                           ctypes.c_int(B), ctypes.c_int(Hq), ctypes.c_int(Hkv), ctypes.c_int(D), ctypes.c_int(k),
                           ctypes.c_int(P_max), ctypes.c_double(scale), ctypes.c_int(mode), ctypes.c_int(int(dense)),
                           ctypes.c_int(nthreads or default_threads()), _p(o), _p(lse), _p(ob))
    if rc:
        raise ValueError("oracle_attn: invalid arguments")
    return o, lse, ob


def attn_rows(inp: dict, Hq: int, Hkv: int, D: int, k: int, sel_b, sel_h, sel_r, scale: float | None = None,
              mode: int = MASK_HYBRID, nthreads: int = 0):
    """Attention for selected (b, h, r) rows only; returns (o [n,D], lse [n])."""
    q = _c(inp["q"], np.uint16)
    B = q.shape[0]
    P_max = inp["k_cache"].shape[2]
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    sb, sh, sr = (_c(x, np.int32) for x in (sel_b, sel_h, sel_r))
    n = len(sb)
    o = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    args = [_c(inp[nm], np.uint16) for nm in ("k_new", "v_new", "k_cache", "v_cache")]
    pl = _c(inp["prefix_len"], np.int32)
    rc = lib().oracle_attn_rows(_p(q), *[_p(a) for a in args], _p(pl),
                                ctypes.c_int(B), ctypes.c_int(Hq), ctypes.c_int(Hkv), ctypes.c_int(D), ctypes.c_int(k),
                                ctypes.c_int(P_max), ctypes.c_double(scale), ctypes.c_int(mode), ctypes.c_int(n),
                                _p(sb), _p(sh), _p(sr), ctypes.c_int(nthreads or default_threads()), _p(o), _p(lse))
    if rc:
        raise ValueError("oracle_attn_rows: invalid arguments")
    return o, lse


def _logits_arg(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return a, LOGITS_BF16
    return np.ascontiguousarray(a, dtype=np.float32), LOGITS_F32


def verify(inp: dict, forced_accept_len=None, nthreads: int = 0, trust_ar: float = 1.0) -> dict:
    """AR rejection-sampling verify; trust_ar = lambda mixes the target logits as
    lambda * p_logits + (1 - lambda) * q_logits (1: the AR logits alone)."""
    p, dt = _logits_arg(inp["p_logits"])
    q, dt2 = _logits_arg(inp["q_logits"])
    assert dt == dt2
    B, k, V = p.shape
    drafts = _c(inp["drafts"], np.int32)
    pre = _c(inp["preaccepted"], np.uint8)
    ua = _c(inp["u_acc"], np.float32)
    ur = _c(inp["u_res"], np.float32)
    forced = None if forced_accept_len is None else _c(forced_accept_len, np.int32)
    out = dict(
        accept_len=np.zeros(B, np.int32), resampled=np.zeros(B, np.int32), tokens=np.zeros((B, k), np.int32),
        n_emitted=np.zeros(B, np.int32), logp_d=np.zeros((B, k)), logq_d=np.zeros((B, k)), ratio=np.zeros((B, k)),
        res_lo=np.zeros(B), res_hi=np.zeros(B))
    rc = lib().oracle_verify(_p(p), _p(q), ctypes.c_int(dt), _p(drafts), _p(pre), _p(ua), _p(ur),
                             ctypes.c_int(B), ctypes.c_int(k), ctypes.c_int(V), ctypes.c_double(trust_ar), _p(forced),
                             ctypes.c_int(nthreads or default_threads()),
                             *[_p(out[n]) for n in ("accept_len", "resampled", "tokens", "n_emitted", "logp_d",
                                                    "logq_d", "ratio", "res_lo", "res_hi")])
    if rc:
        raise ValueError("oracle_verify: invalid arguments")
    return out


def kv_commit(k_caches, v_caches, k_news, v_news, prefix_len, accept_len, resampled, group_logits, u_draft,
              nthreads: int = 0) -> dict:
    """Caches [L,B,Hkv,P_max,D] and new K/V [L,B,R,Hkv,D] (uint16, updated in place copies returned)."""
    kc = np.array(k_caches, dtype=np.uint16, order="C", copy=True)
    vc = np.array(v_caches, dtype=np.uint16, order="C", copy=True)
    kn = _c(k_news, np.uint16)
    vn = _c(v_news, np.uint16)
    L, B, Hkv, P_max, D = kc.shape
    g, dt = _logits_arg(group_logits)
    k = g.shape[2]
    V = g.shape[3]
    pl = np.array(prefix_len, dtype=np.int32, copy=True)
    al = _c(accept_len, np.int32)
    rs = _c(resampled, np.int32)
    ud = _c(u_draft, np.float32)
    out = dict(next_drafts=np.zeros((B, k), np.int32), next_preaccepted=np.zeros(B, np.uint8),
               next_q_group=np.zeros(B, np.int32), draft_lo=np.zeros((B, k)), draft_hi=np.zeros((B, k)))
    rc = lib().oracle_kv_commit(_p(kc), _p(vc), _p(kn), _p(vn), ctypes.c_int(L), ctypes.c_int(B), ctypes.c_int(Hkv),
                                ctypes.c_int(D), ctypes.c_int(k), ctypes.c_int(P_max), _p(pl), _p(al), _p(rs), _p(g),
                                ctypes.c_int(dt), ctypes.c_int(V), _p(ud), ctypes.c_int(nthreads or default_threads()),
                                *[_p(out[n]) for n in ("next_drafts", "next_preaccepted", "next_q_group", "draft_lo",
                                                       "draft_hi")])
    if rc:
        raise ValueError("oracle_kv_commit: invalid arguments")
    out.update(k_caches=kc, v_caches=vc, prefix_len=pl)
    return out


def row_positions(k: int, P: int) -> np.ndarray:
    """Positions of the R = k(k+2) rows of a step with cached prefix P."""
    R = k * (k + 2)
    return np.array([lib().oracle_row_position(ctypes.c_int(k), ctypes.c_int(P), ctypes.c_int(r)) for r in range(R)],
                    dtype=np.int64)


def rope_qkv(qkv, prefix_len, Hq: int, Hkv: int, k: int, theta: float = 1e6):
    """Rotary embedding of qkv [B,R,Hq+2Hkv,D] (bf16 bits) -> (q, k_new, v_new) bf16 bits."""
    x = _c(qkv, np.uint16)
    B, R, H, D = x.shape
    q = np.zeros((B, R, Hq, D), np.uint16)
    kn = np.zeros((B, R, Hkv, D), np.uint16)
    vn = np.zeros((B, R, Hkv, D), np.uint16)
    pl = _c(prefix_len, np.int32)
    rc = lib().oracle_rope_qkv(_p(x), _p(pl), ctypes.c_int(B), ctypes.c_int(Hq), ctypes.c_int(Hkv), ctypes.c_int(D),
                               ctypes.c_int(k), ctypes.c_double(theta), _p(q), _p(kn), _p(vn))
    if rc:
        raise ValueError("oracle_rope_qkv: invalid arguments")
    return q, kn, vn
