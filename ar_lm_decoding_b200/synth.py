"""Seeded synthetic inputs for one TiDAR decode step.

This module only draws random data.  It computes nothing the decode step
computes: no softmax, no mask, no sampling.  Both the CPU oracle (through the
tests) and the CUDA library consume exactly the arrays returned here, so the
two sides see bit-identical inputs.

Workloads follow the shapes of the models the TiDAR pages evaluate
(Qwen2.5-1.5B, Qwen3-8B, Qwen3-32B backbones; "TiDAR: Think in Diffusion, Talk
in Autoregression", awesome-system-papers summary, section "核心方法" /
initialisation) with the draft block layout of the same summary, section
"并行 self-speculative 生成 (§3.2)": k previous drafts plus k+1 pre-draft
groups of k mask tokens, so R = k(k+2) query rows per sequence.

Recipe (all streams are numpy PCG64 seeded by SeedSequence([seed, cfg_id,
tensor_id])):

* Q, K_new, V_new, K/V cache: fp32 N(0,1), rounded once to bf16 (RNE).
* logits: N(0, sigma) (sigma = 2 for the tiny case, 3 otherwise), fp32 or
  rounded to bf16.
* planted peaks (``peaks=True``): per sequence m ~ U{0..k}; for slot i the
  q row gets a peak at a uniform token t_i, z_q[t_i] := max(z_q) + 2 sigma; the
  p row gets its peak at the same token when i <= m and at another uniform
  token otherwise.  The draft d_i is t_i.  The accept length therefore tracks m.
* ``q_temp``: stored q logits are z_q / q_temp (sharpened drafts).
* uniforms: 24-bit fractions (bits >> 8) * 2**-24 in [0, 1).
"""
from __future__ import annotations

import dataclasses
import numpy as np

BF16_NAN = np.uint16(0x7FC0)

# tensor ids for the per-tensor streams
_T_Q, _T_KN, _T_VN, _T_KC, _T_VC, _T_P, _T_Q_LOG, _T_G, _T_DR, _T_PRE, _T_UA, _T_UR, _T_UD, _T_PL, _T_PK = range(15)


@dataclasses.dataclass(frozen=True)
class StepConfig:
    name: str
    L: int
    Hq: int
    Hkv: int
    D: int
    P: int
    k: int
    V: int
    B: int = 1
    logits_dtype: str = "bf16"  # "bf16" or "f32"
    sigma: float = 3.0
    peaks: bool = False
    q_temp: float = 1.0
    ragged: tuple | None = None  # (lo, hi) inclusive prefix-length range per sequence
    cfg_id: int = 0

    @property
    def R(self) -> int:
        return self.k * (self.k + 2)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def P_max(self) -> int:
        # capacity: the longest prefix plus one full accepted block, rounded to 64 rows
        pmax = (self.ragged[1] if self.ragged else self.P) + self.k
        return (pmax + 63) // 64 * 64

    def with_(self, **kw) -> "StepConfig":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": StepConfig("tiny", L=1, Hq=2, Hkv=1, D=64, P=128, k=4, V=1000, logits_dtype="f32", sigma=2.0, cfg_id=0),
    "qwen2.5-1.5b_k4": StepConfig("qwen2.5-1.5b_k4", L=28, Hq=12, Hkv=2, D=128, P=1024, k=4, V=151936, peaks=True, cfg_id=1),
    "qwen2.5-1.5b_k16": StepConfig("qwen2.5-1.5b_k16", L=28, Hq=12, Hkv=2, D=128, P=4096, k=16, V=151936, peaks=True, q_temp=0.5, cfg_id=2),
    "qwen3-8b_k8": StepConfig("qwen3-8b_k8", L=36, Hq=32, Hkv=8, D=128, P=4096, k=8, V=151936, cfg_id=3),
    "qwen3-8b_k8_b8": StepConfig("qwen3-8b_k8_b8", L=36, Hq=32, Hkv=8, D=128, P=4096, k=8, V=151936, B=8, ragged=(512, 4096), cfg_id=4),
    "qwen3-32b_k4": StepConfig("qwen3-32b_k4", L=64, Hq=64, Hkv=8, D=128, P=16384, k=4, V=151936, cfg_id=5),
    "qwen3-32b_k8": StepConfig("qwen3-32b_k8", L=64, Hq=64, Hkv=8, D=128, P=16384, k=8, V=151936, cfg_id=6),
    "qwen3-32b_k16": StepConfig("qwen3-32b_k16", L=64, Hq=64, Hkv=8, D=128, P=16384, k=16, V=151936, cfg_id=7),
    # the Qwen3-8B step once more with the planted-peak logits of the Qwen2.5 workloads, so that accept lengths
    # vary and the commit copies rows
    "qwen3-8b_k8_peaks": StepConfig("qwen3-8b_k8_peaks", L=36, Hq=32, Hkv=8, D=128, P=4096, k=8, V=151936, peaks=True,
                                    cfg_id=8),
}


def _rng(seed: int, cfg: StepConfig, tid: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, cfg.cfg_id, tid])))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        rounded[nan] = BF16_NAN
    return rounded


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(rng: np.random.Generator, shape, sigma: float = 1.0) -> np.ndarray:
    return f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(sigma))


def uniforms(rng: np.random.Generator, shape) -> np.ndarray:
    bits = rng.integers(0, 2**32, size=shape, dtype=np.uint64).astype(np.uint32)
    return ((bits >> 8).astype(np.float32) * np.float32(2.0**-24)).astype(np.float32)


def prefix_lengths(cfg: StepConfig, seed: int) -> np.ndarray:
    if cfg.ragged is None:
        return np.full(cfg.B, cfg.P, dtype=np.int32)
    lo, hi = cfg.ragged
    return _rng(seed, cfg, _T_PL).integers(lo, hi + 1, size=cfg.B).astype(np.int32)


def make_attn_inputs(cfg: StepConfig, seed: int = 0, poison: bool = True, prefix_len=None) -> dict:
    """One layer's attention inputs (bf16 bits as uint16)."""
    B, R, Hq, Hkv, D, Pm = cfg.B, cfg.R, cfg.Hq, cfg.Hkv, cfg.D, cfg.P_max
    pl = prefix_lengths(cfg, seed) if prefix_len is None else np.asarray(prefix_len, dtype=np.int32)
    q = normal_bf16(_rng(seed, cfg, _T_Q), (B, R, Hq, D))
    kn = normal_bf16(_rng(seed, cfg, _T_KN), (B, R, Hkv, D))
    vn = normal_bf16(_rng(seed, cfg, _T_VN), (B, R, Hkv, D))
    kc = normal_bf16(_rng(seed, cfg, _T_KC), (B, Hkv, Pm, D))
    vc = normal_bf16(_rng(seed, cfg, _T_VC), (B, Hkv, Pm, D))
    if poison:
        # rows at or beyond each prefix length are not part of the cache: NaN so any use shows
        for b in range(B):
            kc[b, :, pl[b]:, :] = BF16_NAN
            vc[b, :, pl[b]:, :] = BF16_NAN
    return dict(q=q, k_new=kn, v_new=vn, k_cache=kc, v_cache=vc, prefix_len=pl)


def _logits(rng, shape, cfg: StepConfig) -> np.ndarray:
    return rng.standard_normal(shape, dtype=np.float32) * np.float32(cfg.sigma)


def _plant(z: np.ndarray, tok: int, sigma: float) -> None:
    z[tok] = z.max() + np.float32(2.0 * sigma)


def _encode_logits(z: np.ndarray, cfg: StepConfig) -> np.ndarray:
    return f32_to_bf16_bits(z) if cfg.logits_dtype == "bf16" else np.ascontiguousarray(z, dtype=np.float32)


def make_verify_inputs(cfg: StepConfig, seed: int = 0) -> dict:
    """Logits, drafts and uniforms for the verify and the commit's draft selection."""
    B, k, V = cfg.B, cfg.k, cfg.V
    zp = _logits(_rng(seed, cfg, _T_P), (B, k, V), cfg)
    zq = _logits(_rng(seed, cfg, _T_Q_LOG), (B, k, V), cfg)
    zg = _logits(_rng(seed, cfg, _T_G), (B, k + 1, k, V), cfg)
    rd = _rng(seed, cfg, _T_DR)
    drafts = rd.integers(0, V, size=(B, k)).astype(np.int32)
    m_shared = np.full(B, -1, dtype=np.int32)
    if cfg.peaks:
        rk = _rng(seed, cfg, _T_PK)
        m_shared = rk.integers(0, k + 1, size=B).astype(np.int32)
        for b in range(B):
            for i in range(k):
                t = int(rk.integers(0, V))
                _plant(zq[b, i], t, cfg.sigma)
                tp = t if i < m_shared[b] else int((t + 1 + rk.integers(0, V - 1)) % V)
                _plant(zp[b, i], tp, cfg.sigma)
                drafts[b, i] = t
    if cfg.q_temp != 1.0:
        zq = zq / np.float32(cfg.q_temp)
    pre = (_rng(seed, cfg, _T_PRE).integers(0, 2, size=B)).astype(np.uint8)
    return dict(
        p_logits=_encode_logits(zp, cfg),
        q_logits=_encode_logits(zq, cfg),
        group_logits=_encode_logits(zg, cfg),
        drafts=drafts,
        preaccepted=pre,
        u_acc=uniforms(_rng(seed, cfg, _T_UA), (B, k)),
        u_res=uniforms(_rng(seed, cfg, _T_UR), (B,)),
        u_draft=uniforms(_rng(seed, cfg, _T_UD), (B, k)),
        m_shared=m_shared,
    )
