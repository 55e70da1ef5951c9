"""Python binding of libtidar (include/tidar.h): argument marshalling only.

Every function has the name and argument order of its C entry point.  Pointer
arguments accept a torch tensor (its data_ptr() is passed), a raw integer
address or None (NULL).  `stream` defaults to torch's current CUDA stream.
A non-OK status raises TidarError.  There is no fallback: if libtidar.so is
missing, importing this module fails.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtidar.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built: run `python -m ar_lm_decoding_b200.build` "
                      "(needs nvcc); there is no CPU fallback")

_lib = ctypes.CDLL(LIB_PATH)

TIDAR_OK, TIDAR_ERR_INVALID_ARG, TIDAR_ERR_UNSUPPORTED, TIDAR_ERR_WORKSPACE, TIDAR_ERR_CUDA = range(5)
TIDAR_DEV_BAD_PREFIX, TIDAR_DEV_BAD_TOKEN, TIDAR_DEV_BAD_ACCEPT, TIDAR_DEV_TIMEOUT, TIDAR_DEV_BAD_PAGE = 1, 2, 4, 8, 16
TIDAR_DT_BF16, TIDAR_DT_F32 = 0, 1
TIDAR_MASK_HYBRID, TIDAR_MASK_CAUSAL = 0, 1

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t

_SIGS = {
    "tidar_attn_workspace_size": (_sz, [_i] * 6),
    "tidar_attn_step": (_i, [_vp] * 6 + [_i] * 6 + [_f, _i] + [_vp, _vp, _vp, _sz, _vp, _vp]),
    "tidar_verify_workspace_size": (_sz, [_i] * 3),
    "tidar_verify": (_i, [_vp, _vp, _i] + [_vp] * 4 + [_i] * 3 + [_vp] * 7 + [_sz, _vp, _vp]),
    "tidar_verify_trust_mix": (_i, [_vp, _vp, _i] + [_vp] * 4 + [_i] * 3 + [_f] + [_vp] * 7 + [_sz, _vp, _vp]),
    "tidar_verify_noalloc": (_i, [_vp, _vp, _i] + [_vp] * 4 + [_i] * 3 + [_vp] * 7 + [_vp]),
    "tidar_kv_commit_workspace_size": (_sz, [_i] * 3),
    "tidar_kv_commit": (_i, [_vp] * 4 + [_i] * 6 + [_vp] * 4 + [_i, _i, _vp] + [_vp] * 4 + [_sz, _vp, _vp]),
    "tidar_status_string": (ctypes.c_char_p, [_i]),
    "tidar_expected_tokens_per_step": (ctypes.c_double, [_i, ctypes.c_double]),
    "tidar_pick_draft_length": (_i, [_vp, _i, ctypes.c_double, _vp]),
    "tidar_attn_step_paged": (_i, [_vp] * 6 + [_i, _i, _vp] + [_i] * 5 + [_f, _i] + [_vp, _vp, _vp, _vp]),
    "tidar_kv_commit_paged": (_i, [_vp] * 5 + [_i] * 7 + [_vp] * 4 + [_i, _i, _vp] + [_vp] * 4 + [_sz, _vp, _vp]),
    "tidar_rope_qkv": (_i, [_vp, _vp] + [_i] * 5 + [ctypes.c_double] + [_vp] * 5),
    "tidar_verify_commit_workspace_size": (_sz, [_i] * 3),
    "tidar_verify_commit": (_i, [_vp, _vp, _i] + [_vp] * 4 + [_f] + [_vp] * 5 + [_i] * 9 + [_vp] * 12
                            + [_vp, _sz, _vp, _vp]),
    "tidar_testing_attn_step_stalled": (_i, [_vp] * 6 + [_i] * 6 + [_f, _i] + [_vp, _vp, _vp, ctypes.c_longlong, _vp]),
    "tidar_testing_attn_splits": (_i, [_i] * 6),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class TidarError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {tidar_status_string(status)}")
        self.status = status


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, status: int) -> None:
    if status != TIDAR_OK:
        raise TidarError(fn, status)


def tidar_status_string(status: int) -> str:
    return _lib.tidar_status_string(status).decode()


def tidar_attn_workspace_size(B, Hq, Hkv, D, k, P_max) -> int:
    return _lib.tidar_attn_workspace_size(B, Hq, Hkv, D, k, P_max)


def tidar_attn_step(q, k_new, v_new, k_cache, v_cache, prefix_len, B, Hq, Hkv, D, k, P_max, softmax_scale,
                    mask_mode, out, lse, workspace, ws_bytes, dev_status, stream=None) -> None:
    _check("tidar_attn_step", _lib.tidar_attn_step(
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(prefix_len), B, Hq, Hkv, D, k, P_max,
        softmax_scale, mask_mode, _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream)))


def tidar_attn_step_paged(q, k_new, v_new, k_pool, v_pool, block_table, max_pages, num_pages, prefix_len, B, Hq,
                          Hkv, D, k, softmax_scale, mask_mode, out, lse, dev_status, stream=None) -> None:
    _check("tidar_attn_step_paged", _lib.tidar_attn_step_paged(
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool), _ptr(block_table), max_pages, num_pages,
        _ptr(prefix_len), B, Hq, Hkv, D, k, softmax_scale, mask_mode, _ptr(out), _ptr(lse), _ptr(dev_status),
        _stream(stream)))


def tidar_kv_commit_paged(k_pools, v_pools, k_news, v_news, block_table, max_pages, num_pages, L, B, Hkv, D, k,
                          prefix_len, accept_len, resampled, group_logits, logits_dtype, V, u_draft, next_drafts,
                          next_preaccepted, next_q_group, workspace, ws_bytes, dev_status, stream=None) -> None:
    _check("tidar_kv_commit_paged", _lib.tidar_kv_commit_paged(
        _ptr(k_pools), _ptr(v_pools), _ptr(k_news), _ptr(v_news), _ptr(block_table), max_pages, num_pages, L, B, Hkv,
        D, k, _ptr(prefix_len), _ptr(accept_len), _ptr(resampled), _ptr(group_logits), logits_dtype, V,
        _ptr(u_draft), _ptr(next_drafts), _ptr(next_preaccepted), _ptr(next_q_group), _ptr(workspace), ws_bytes,
        _ptr(dev_status), _stream(stream)))


def tidar_rope_qkv(qkv, prefix_len, B, Hq, Hkv, D, k, theta, q, k_new, v_new, dev_status, stream=None) -> None:
    _check("tidar_rope_qkv", _lib.tidar_rope_qkv(
        _ptr(qkv), _ptr(prefix_len), B, Hq, Hkv, D, k, theta, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(dev_status),
        _stream(stream)))


def tidar_testing_attn_step_stalled(q, k_new, v_new, k_cache, v_cache, prefix_len, B, Hq, Hkv, D, k, P_max,
                                    softmax_scale, mask_mode, out, lse, dev_status, wait_cycles,
                                    stream=None) -> None:
    """Test hook (include/tidar_testing.h): the attention launch with a wait that runs out on purpose."""
    _check("tidar_testing_attn_step_stalled", _lib.tidar_testing_attn_step_stalled(
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(prefix_len), B, Hq, Hkv, D, k, P_max,
        softmax_scale, mask_mode, _ptr(out), _ptr(lse), _ptr(dev_status), wait_cycles, _stream(stream)))


def tidar_testing_attn_splits(B, Hq, Hkv, D, k, P_max) -> int:
    """Test hook (include/tidar_testing.h): the cluster size the attention launch would use (0: rejected sizes)."""
    return _lib.tidar_testing_attn_splits(B, Hq, Hkv, D, k, P_max)


def tidar_verify_workspace_size(B, k, V) -> int:
    return _lib.tidar_verify_workspace_size(B, k, V)


def tidar_verify(p_logits, q_logits, logits_dtype, drafts, preaccepted, u_acc, u_res, B, k, V, accept_len, resampled,
                 tokens, n_emitted, logp_d, logq_d, workspace, ws_bytes, dev_status, stream=None) -> None:
    _check("tidar_verify", _lib.tidar_verify(
        _ptr(p_logits), _ptr(q_logits), logits_dtype, _ptr(drafts), _ptr(preaccepted), _ptr(u_acc), _ptr(u_res),
        B, k, V, _ptr(accept_len), _ptr(resampled), _ptr(tokens), _ptr(n_emitted), _ptr(logp_d), _ptr(logq_d),
        _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream)))


def tidar_verify_trust_mix(p_logits, q_logits, logits_dtype, drafts, preaccepted, u_acc, u_res, B, k, V, trust_ar,
                           accept_len, resampled, tokens, n_emitted, logp_d, logq_d, workspace, ws_bytes, dev_status,
                           stream=None) -> None:
    _check("tidar_verify_trust_mix", _lib.tidar_verify_trust_mix(
        _ptr(p_logits), _ptr(q_logits), logits_dtype, _ptr(drafts), _ptr(preaccepted), _ptr(u_acc), _ptr(u_res),
        B, k, V, trust_ar, _ptr(accept_len), _ptr(resampled), _ptr(tokens), _ptr(n_emitted), _ptr(logp_d),
        _ptr(logq_d), _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream)))


def tidar_verify_noalloc(p_logits, q_logits, logits_dtype, drafts, preaccepted, u_acc, u_res, B, k, V, accept_len,
                         resampled, tokens, n_emitted, logp_d, logq_d, dev_status, stream=None) -> None:
    """tidar_verify for callers that cannot allocate device memory: the scratch is a fixed 2 MiB array
    inside the library, shared by every call on the device (overlapping calls race)."""
    _check("tidar_verify_noalloc", _lib.tidar_verify_noalloc(
        _ptr(p_logits), _ptr(q_logits), logits_dtype, _ptr(drafts), _ptr(preaccepted), _ptr(u_acc), _ptr(u_res),
        B, k, V, _ptr(accept_len), _ptr(resampled), _ptr(tokens), _ptr(n_emitted), _ptr(logp_d), _ptr(logq_d),
        _ptr(dev_status), _stream(stream)))


def tidar_kv_commit_workspace_size(B, k, V) -> int:
    return _lib.tidar_kv_commit_workspace_size(B, k, V)


def tidar_kv_commit(k_caches, v_caches, k_news, v_news, L, B, Hkv, D, k, P_max, prefix_len, accept_len, resampled,
                    group_logits, logits_dtype, V, u_draft, next_drafts, next_preaccepted, next_q_group, workspace,
                    ws_bytes, dev_status, stream=None) -> None:
    _check("tidar_kv_commit", _lib.tidar_kv_commit(
        _ptr(k_caches), _ptr(v_caches), _ptr(k_news), _ptr(v_news), L, B, Hkv, D, k, P_max, _ptr(prefix_len),
        _ptr(accept_len), _ptr(resampled), _ptr(group_logits), logits_dtype, V, _ptr(u_draft), _ptr(next_drafts),
        _ptr(next_preaccepted), _ptr(next_q_group), _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream)))


def tidar_verify_commit_workspace_size(B, k, V) -> int:
    return _lib.tidar_verify_commit_workspace_size(B, k, V)


def tidar_verify_commit(p_logits, q_logits, logits_dtype, drafts, preaccepted, u_acc, u_res, trust_ar, k_caches,
                        v_caches, k_news, v_news, block_table, max_pages, num_pages, L, B, Hkv, D, k, P_max, V,
                        prefix_len, group_logits, u_draft, accept_len, resampled, tokens, n_emitted, logp_d, logq_d,
                        next_drafts, next_preaccepted, next_q_group, workspace, ws_bytes, dev_status,
                        stream=None) -> None:
    """tidar_verify_trust_mix followed by tidar_kv_commit (or its paged form when block_table is given) in one
    launch."""
    _check("tidar_verify_commit", _lib.tidar_verify_commit(
        _ptr(p_logits), _ptr(q_logits), logits_dtype, _ptr(drafts), _ptr(preaccepted), _ptr(u_acc), _ptr(u_res),
        trust_ar, _ptr(k_caches), _ptr(v_caches), _ptr(k_news), _ptr(v_news), _ptr(block_table), max_pages,
        num_pages, L, B, Hkv, D, k, P_max, V, _ptr(prefix_len), _ptr(group_logits), _ptr(u_draft),
        _ptr(accept_len), _ptr(resampled), _ptr(tokens), _ptr(n_emitted), _ptr(logp_d), _ptr(logq_d),
        _ptr(next_drafts), _ptr(next_preaccepted), _ptr(next_q_group), _ptr(workspace), ws_bytes,
        _ptr(dev_status), _stream(stream)))


def tidar_expected_tokens_per_step(k, alpha) -> float:
    return _lib.tidar_expected_tokens_per_step(k, alpha)


def tidar_pick_draft_length(step_us, alpha):
    """(k, tokens per microsecond) for the step latencies step_us[k-1] (a sequence of floats, k = 1..n)."""
    n = len(step_us)
    arr = (ctypes.c_double * n)(*[float(x) for x in step_us])
    rate = ctypes.c_double(0.0)
    k = _lib.tidar_pick_draft_length(ctypes.cast(arr, ctypes.c_void_p), n, alpha, ctypes.byref(rate))
    return k, rate.value


def pointer_array(tensors, device):
    """Device int64 array holding the data pointers of `tensors` (for tidar_kv_commit)."""
    import torch
    return torch.tensor([t.data_ptr() for t in tensors], dtype=torch.int64, device=device)


def library_path() -> str:
    return LIB_PATH
