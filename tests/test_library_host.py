"""Host-side checks of the C-ABI library (no GPU): it loads, exports every entry point that
include/iskv.h declares, validates configurations before touching CUDA, and its fold schedule is
the window rule of the iS-KV summary ("Architecture Overview": fold the oldest block once
window + block rows are exact)."""
import os
import re

import pytest

import rank_kv_cache_isvd_b200 as iskv
from oracle import n_compressed

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "iskv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(iskv_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 11
    for n in names:
        assert hasattr(iskv.lib, n), n
        assert hasattr(iskv, n), n           # the binding keeps the C names


def test_binding_requires_built_library():
    assert os.path.exists(iskv.LIB_PATH)
    assert iskv.LIB_PATH.endswith("libiskv.so")


@pytest.mark.parametrize("block,window", [(64, 256), (32, 64), (128, 256), (1, 0), (7, 3), (64, 128)])
def test_schedule_matches_window_rule(block, window):
    for t in list(range(0, 700, 13)) + [4095, 4096]:
        for m in (0, 1, 5, 64, 129, 1000):
            code, nc, folds = iskv.iskv_schedule(block, window, t, m)
            assert code == 0
            assert nc == n_compressed(t + m, block, window)
            assert folds * block == nc - n_compressed(t, block, window)


def test_schedule_rejects_bad_arguments():
    assert iskv.iskv_schedule(0, 4, 0, 1)[0] == iskv.ISKV_ERR_INVALID_ARG
    assert iskv.iskv_schedule(4, -1, 0, 1)[0] == iskv.ISKV_ERR_INVALID_ARG
    assert iskv.iskv_schedule(4, 4, -1, 1)[0] == iskv.ISKV_ERR_INVALID_ARG


def _cfg(**kw):
    base = dict(batch=1, n_layers=1, n_kv_heads=8, n_q_heads=32, head_dim=128, rank_k=32,
                rank_v=48, block=64, window=256, max_tokens=4096, kv_dtype=iskv.ISKV_BF16,
                rope=1, rope_theta=5e5, rotate_history=1)
    base.update(kw)
    return iskv.iskv_config(**base)


@pytest.mark.parametrize("bad", [
    dict(head_dim=64), dict(rank_k=0), dict(rank_v=129), dict(block=0), dict(window=-1),
    dict(n_q_heads=12), dict(n_q_heads=128), dict(batch=0), dict(max_tokens=0), dict(kv_dtype=7),
    dict(rope=1, rope_theta=0.0), dict(n_layers=0), dict(fixed_basis=1, rotate_history=0),
])
def test_create_rejects_invalid_config(bad):
    code, h = iskv.iskv_create(_cfg(**bad))
    assert code == iskv.ISKV_ERR_INVALID_ARG and h == 0


def test_create_reports_unsupported_block():
    code, h = iskv.iskv_create(_cfg(block=2048))
    assert code == iskv.ISKV_ERR_UNSUPPORTED and h == 0


@pytest.mark.parametrize("bad", [
    dict(joint_heads=1, rank_k=80, block=64),           # rank + block > 128
    dict(joint_heads=1, rank_v=72, block=64),
    dict(joint_heads=1, fixed_basis=1),
    dict(joint_heads=1, prot_cap=16),
])
def test_joint_factorisation_limits_are_refused_before_any_cuda_call(bad):
    code, h = iskv.iskv_create(_cfg(**bad))
    assert code == iskv.ISKV_ERR_UNSUPPORTED and h == 0


def test_null_handle_and_strerror():
    assert iskv.iskv_destroy(None) == 0
    assert iskv.iskv_append_block(None, 0, 1, 1, 1, 0) == iskv.ISKV_ERR_INVALID_ARG
    assert iskv.iskv_decode_attn(None, 0, 1, 1, 0) == iskv.ISKV_ERR_INVALID_ARG
    assert iskv.iskv_sync_status(None, 0) == iskv.ISKV_ERR_INVALID_ARG
    for code in range(-7, 1):
        assert iskv.iskv_strerror(code) != "unknown error"
    assert iskv.iskv_strerror(-99) == "unknown error"


def test_create_without_gpu_fails_cleanly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is visible")
    code, h = iskv.iskv_create(_cfg())
    assert code == iskv.ISKV_ERR_CUDA and h == 0


def _view(**kw):
    base = dict(n_c=0, t=8192, n_max=0, batch=8, n_kv_heads=8, n_q_heads=32, head_dim=128,
                rank_k=32, rank_v=48, k_k=0, k_v=0, ring_rows=8192, kv_dtype=iskv.ISKV_BF16)
    base.update(kw)
    return iskv.iskv_decode_view(**base)


def test_no_alloc_decode_refuses_oversize_requests_before_any_cuda_call():
    # 64 window splits x 64 kv-heads x GQA 4 x 130 floats > the fixed scratch: refused on the host
    # (the pointers are never read: the size check comes first)
    need = 8 * 8 * (8192 // 128) * 4 * 130
    assert need > iskv.ISKV_NOALLOC_SCRATCH_FLOATS
    v = _view(ring_k=256, ring_v=256)
    assert iskv.iskv_decode_attn_noalloc(v, 256, 256) == iskv.ISKV_ERR_CAPACITY
    assert iskv.iskv_decode_attn_noalloc(None, 256, 256) == iskv.ISKV_ERR_INVALID_ARG
    assert iskv.iskv_decode_attn_noalloc(_view(), 256, 256) == iskv.ISKV_ERR_INVALID_ARG  # no ring
    assert iskv.iskv_decode_attn_noalloc(_view(head_dim=64, ring_k=256, ring_v=256), 256,
                                         256) == iskv.ISKV_ERR_INVALID_ARG
    assert iskv.iskv_decode_attn_noalloc(_view(n_c=128, t=200, n_max=128, ring_rows=72,
                                               ring_k=256, ring_v=256), 256,
                                         256) == iskv.ISKV_ERR_INVALID_ARG  # n_c > 0, no factors
