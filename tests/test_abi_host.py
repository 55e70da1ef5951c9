"""Host-only checks of the C ABI: the library loads without a GPU, exports every
function include/tidar.h declares, and rejects bad arguments before launching
anything.  No call here reaches a kernel."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER_DIR = os.path.join(ROOT, "include")


def _lib_path():
    from ar_lm_decoding_b200 import build
    return build.build()


def _declared_functions():
    names = []
    for h in sorted(os.listdir(HEADER_DIR)):
        if not h.endswith(".h"):
            continue
        src = open(os.path.join(HEADER_DIR, h)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b(tidar_\w+)\s*\(", src, flags=re.M):
            names.append(m.group(1))
    return sorted(set(names))


def test_header_declares_the_three_entry_points():
    names = _declared_functions()
    for n in ("tidar_attn_step", "tidar_verify", "tidar_kv_commit"):
        assert n in names


def test_every_declared_symbol_is_exported():
    lib = ctypes.CDLL(_lib_path())
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_names_match_the_header():
    _lib_path()
    from ar_lm_decoding_b200 import abi
    for n in _declared_functions():
        assert callable(getattr(abi, n)), n


def test_workspace_sizes_and_validation():
    _lib_path()
    from ar_lm_decoding_b200 import abi
    # attention needs no scratch: split-KV partials pass through the cluster's distributed shared memory
    assert abi.tidar_attn_workspace_size(1, 32, 8, 128, 8, 4160) == 0
    assert abi.tidar_attn_workspace_size(8, 64, 8, 128, 16, 4160) == 0
    assert abi.tidar_verify_workspace_size(1, 8, 151936) > 0
    assert abi.tidar_kv_commit_workspace_size(8, 8, 151936) > 0
    assert abi.tidar_verify_workspace_size(0, 8, 151936) == 0
    assert abi.tidar_status_string(abi.TIDAR_ERR_WORKSPACE) == "TIDAR_ERR_WORKSPACE"


def _attn_call(abi, **over):
    args = dict(q=8192, k_new=8192, v_new=8192, k_cache=8192, v_cache=8192, prefix_len=8192, B=1, Hq=2, Hkv=1, D=64,
                k=4, P_max=256, softmax_scale=0.125, mask_mode=0, out=8192, lse=None, workspace=1 << 20,
                ws_bytes=1 << 30, dev_status=8192, stream=0)
    args.update(over)
    abi.tidar_attn_step(**args)


@pytest.mark.parametrize("over,code", [
    (dict(D=96), 2), (dict(k=17), 2), (dict(Hq=3, Hkv=2), 2), (dict(k=0), 1), (dict(B=0), 1),
    (dict(q=None), 1), (dict(out=8200), 1), (dict(mask_mode=5), 1), (dict(softmax_scale=float("nan")), 1),
    (dict(dev_status=None), 1), (dict(k_cache=8200), 1), (dict(lse=8194), 1), (dict(softmax_scale=0.0), 1),
])
def test_attn_rejects_bad_arguments_without_launch(over, code):
    _lib_path()
    from ar_lm_decoding_b200 import abi
    with pytest.raises(abi.TidarError) as e:
        _attn_call(abi, **over)
    assert e.value.status == code


def test_verify_and_commit_reject_bad_arguments():
    _lib_path()
    from ar_lm_decoding_b200 import abi
    base = dict(p_logits=8192, q_logits=8192, logits_dtype=0, drafts=8192, preaccepted=8192, u_acc=8192,
                u_res=8192, B=1, k=4, V=1000, accept_len=8192, resampled=8192, tokens=8192, n_emitted=8192,
                logp_d=None, logq_d=None, workspace=1 << 20, ws_bytes=1 << 30, dev_status=8192, stream=0)
    for over, code in ((dict(k=17), 2), (dict(logits_dtype=3), 1), (dict(drafts=None), 1), (dict(ws_bytes=8), 3)):
        with pytest.raises(abi.TidarError) as e:
            abi.tidar_verify(**{**base, **over})
        assert e.value.status == code
    cbase = dict(k_caches=8192, v_caches=8192, k_news=8192, v_news=8192, L=2, B=1, Hkv=1, D=64, k=4, P_max=100,
                 prefix_len=8192, accept_len=8192, resampled=8192, group_logits=8192, logits_dtype=0, V=1000,
                 u_draft=8192, next_drafts=8192, next_preaccepted=8192, next_q_group=8192, workspace=1 << 20,
                 ws_bytes=1 << 30, dev_status=8192, stream=0)
    for over, code in ((dict(D=80), 2), (dict(L=0), 1), (dict(k_news=None), 1), (dict(ws_bytes=0), 3)):
        with pytest.raises(abi.TidarError) as e:
            abi.tidar_kv_commit(**{**cbase, **over})
        assert e.value.status == code
