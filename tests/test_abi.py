"""C-ABI checks that need no GPU: libsfa.so loads, exports every function that
include/sfa.h declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def sfa():
    import frame_sparse_attention_b200 as sfa
    from frame_sparse_attention_b200 import build
    if not os.path.exists(build.LIB):
        build.build()
    sfa.load()
    return sfa


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w+\s*\**\s*(sfa_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(sfa):
    declared = _declared_functions()
    assert {"sfa_build_sets", "sfa_forward", "sfa_lse_merge", "sfa_error_string"} <= set(declared)
    lib = ctypes.CDLL(sfa._lib.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert set(sfa._lib.EXPORTS) == set(declared)


def test_error_strings_and_version(sfa):
    for code in range(6):
        assert sfa.error_string(code).startswith("SFA_")
    assert "unknown" in sfa.error_string(99)
    assert sfa.version() >= 100


def test_set_max_count(sfa):
    P = sfa.set_params
    assert sfa.set_max_count(P(T_kv=41, Tq=41, C=21, W=9, T_per=4, step=0), ["lvsa"] * 12) == 21
    assert sfa.set_max_count(P(T_kv=121, Tq=121, C=21, W=13, T_per=6), ["lvsa"] * 12) == 34
    stream = P(T_kv=24, Tq=3, q_off=21, n_sink=1, n_prev=3, chunk_len=3)
    kinds = ["local"] * 4 + ["anchor"] * 4 + ["memory"] * 4
    assert sfa.set_max_count(stream, kinds, n_extra=6) == 13
    assert sfa.set_max_count(P(T_kv=4, Tq=4, n_sink=1, n_prev=1, chunk_len=1), ["anchor"] * 2) == 3
    assert sfa.set_max_count(P(T_kv=14, Tq=1, q_off=13), ["dense"]) == 14
    assert sfa.set_max_count(P(T_kv=14, Tq=1, q_off=13), ["explicit"], n_extra=20) == 14


@pytest.mark.parametrize("kw,kinds", [
    (dict(T_kv=0, Tq=1), ["dense"]),
    (dict(T_kv=4, Tq=3, q_off=2), ["dense"]),
    (dict(T_kv=4, Tq=4, C=0, W=1, T_per=1), ["lvsa"]),
    (dict(T_kv=4, Tq=4, C=2, W=1, T_per=0), ["lvsa"]),
    (dict(T_kv=4, Tq=4, chunk_len=0), ["local"]),
    (dict(T_kv=4, Tq=4), [7]),
])
def test_set_params_rejected(sfa, kw, kinds):
    with pytest.raises(sfa.SfaError) as e:
        sfa.set_max_count(sfa.set_params(**kw), kinds)
    assert e.value.status == sfa.SFA_ERR_INVALID_ARG


def test_build_sets_rejects_small_amax_without_launch(sfa):
    lib = sfa.load()
    p = sfa.set_params(T_kv=41, Tq=41, C=21, W=9, T_per=4)
    kinds = (ctypes.c_int32 * 1)(1)
    # Amax below the bound: refused on the host, the (bogus) device pointers are never used
    assert lib.sfa_build_sets(ctypes.byref(p), 1, kinds, None, 0, 16, 16, 20, None) == sfa.SFA_ERR_INVALID_ARG
    assert lib.sfa_build_sets(ctypes.byref(p), 1, kinds, None, 0, None, 16, 21, None) == sfa.SFA_ERR_INVALID_ARG
    assert lib.sfa_build_sets(ctypes.byref(p), 0, kinds, None, 0, 16, 16, 21, None) == sfa.SFA_ERR_INVALID_ARG


def _desc(sfa, **over):
    d = sfa.AttnDesc()
    d.B, d.H, d.Tq, d.T_kv, d.P, d.d, d.scale, d.Amax = 1, 2, 4, 4, 64, 64, 0.125, 4
    for f in ("q_stride", "k_stride", "v_stride", "o_stride"):
        arr = getattr(d, f)
        arr[0], arr[1], arr[2] = 2 * 256 * 64, 256 * 64, 64
    for k, v in over.items():
        setattr(d, k, v)
    return d


@pytest.mark.parametrize("over,code", [
    (dict(d=96), 2), (dict(d=32), 2), (dict(H=0), 1), (dict(P=0), 1), (dict(Amax=0), 1),
    (dict(scale=0.0), 1), (dict(scale=float("nan")), 1), (dict(B=-1), 1),
])
def test_forward_rejects_bad_desc(sfa, over, code):
    lib = sfa.load()
    d = _desc(sfa, **over)
    good = 1 << 20
    assert lib.sfa_forward(ctypes.byref(d), good, good, good, good, good, good, good, None, None) == code


def test_forward_rejects_bad_pointers_and_strides(sfa):
    lib = sfa.load()
    good = 1 << 20
    d = _desc(sfa)
    assert lib.sfa_forward(None, good, good, good, good, good, good, good, None, None) == 1
    assert lib.sfa_forward(ctypes.byref(d), good + 2, good, good, good, good, good, good, None, None) == 1
    assert lib.sfa_forward(ctypes.byref(d), good, good, good, None, good, good, good, None, None) == 1
    d.k_stride[2] = 36  # token stride not a multiple of 8 elements (16 bytes)
    assert lib.sfa_forward(ctypes.byref(d), good, good, good, good, good, good, good, None, None) == 1
    d = _desc(sfa)
    d.B = 0  # nothing to do
    assert lib.sfa_forward(ctypes.byref(d), good, good, good, good, good, good, good, None, None) == 0


def test_merge_rejects_bad_args(sfa):
    lib = sfa.load()
    good = 1 << 20
    assert lib.sfa_lse_merge(-1, 128, good, good, good, good, good, good, None) == 1
    assert lib.sfa_lse_merge(10, 96, good, good, good, good, good, good, None) == 2
    assert lib.sfa_lse_merge(0, 128, None, None, None, None, None, None, None) == 0
    assert lib.sfa_lse_merge(10, 128, good + 8, good, good, good, good, good, None) == 1


def test_no_oracle_in_product_path():
    # the product package and its C sources never reach for the oracle
    pkg = os.path.join(ROOT, "frame_sparse_attention_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert "oracle" not in text.lower(), f"{fn} mentions the oracle"


def _round256(n):
    return (n + 255) // 256 * 256


def test_split_workspace_and_arguments(sfa):
    lib = sfa.load()
    d = _desc(sfa)  # B=1, H=2, Tq=4, P=64, d=64: 512 query rows
    out = ctypes.c_size_t(0)
    assert lib.sfa_forward_split_workspace(ctypes.byref(d), 1, ctypes.byref(out)) == 0 and out.value == 0
    assert lib.sfa_forward_split_workspace(ctypes.byref(d), 2, ctypes.byref(out)) == 0
    assert out.value == 2 * 512 * 64 * 2 + 2 * 512 * 4
    assert lib.sfa_forward_split_workspace(ctypes.byref(d), 9, ctypes.byref(out)) == 1   # > d/8
    assert lib.sfa_forward_split_workspace(ctypes.byref(d), -1, ctypes.byref(out)) == 1
    # n_split = 0: a scheduled launch; its workspace holds the partials (more than one
    # range) and one 8-byte work item per CTA, each part rounded up to 256 bytes
    k0, _ = sfa.split_plan(d)
    assert 1 <= k0 <= 8
    part = 0 if k0 == 1 else _round256(k0 * 512 * 64 * 2) + _round256(k0 * 512 * 4)
    assert lib.sfa_forward_split_workspace(ctypes.byref(d), 0, ctypes.byref(out)) == 0
    assert out.value == part + _round256(8 * k0 * 1 * 2 * 4 * 1)
    good = 1 << 20
    # workspace missing, too small or misaligned: refused before any launch
    assert lib.sfa_forward_split(ctypes.byref(d), good, good, good, good, good, good, good, 2, None, 0,
                                 None, None) == 1
    assert lib.sfa_forward_split(ctypes.byref(d), good, good, good, good, good, good, good, 2, good, 1024,
                                 None, None) == 1
    assert lib.sfa_forward_split(ctypes.byref(d), good, good, good, good, good, good, good, 2, good + 128,
                                 out.value, None, None) == 1


def test_hsa_host_checks(sfa):
    lib = sfa.load()
    P = sfa.set_params
    # (n_sink + n_prev + chunk_len) * nblk + min(k_blocks, k_frames * nblk); P = 1560 -> 13 blocks
    p = P(T_kv=24, Tq=3, q_off=21, n_sink=1, n_prev=3, chunk_len=3)
    assert sfa.hsa_max_count(p, 1560, 4, 24) == 7 * 13 + 24
    assert sfa.hsa_max_count(p, 1560, 1, 24) == 7 * 13 + 13
    assert sfa.hsa_max_count(p, 200, 0, 5) == 7 * 2
    with pytest.raises(sfa.SfaError):
        sfa.hsa_max_count(p, 1560, -1, 3)
    d = _desc(sfa, Tq=3, T_kv=24, P=1560, Amax=7 * 13 + 24 - 1)
    good = 1 << 20
    ws = ctypes.c_size_t(0)
    assert lib.sfa_hsa_workspace(ctypes.byref(d), ctypes.byref(ws)) == 0 and ws.value > 0
    # Amax below the bound, Tq mismatch, misaligned workspace: refused before any launch
    assert lib.sfa_hsa_select(ctypes.byref(d), ctypes.byref(p), 4, 24, good, good, good, ws.value, good, good,
                              None) == sfa.SFA_ERR_INVALID_ARG
    d.Amax = 7 * 13 + 24
    p2 = P(T_kv=24, Tq=2, q_off=21, n_sink=1, n_prev=3, chunk_len=3)
    assert lib.sfa_hsa_select(ctypes.byref(d), ctypes.byref(p2), 4, 24, good, good, good, ws.value, good, good,
                              None) == sfa.SFA_ERR_INVALID_ARG
    assert lib.sfa_hsa_select(ctypes.byref(d), ctypes.byref(p), 4, 24, good, good, good + 16, ws.value, good,
                              good, None) == sfa.SFA_ERR_INVALID_ARG
    assert lib.sfa_hsa_select(ctypes.byref(d), ctypes.byref(p), 4, 24, good, good, good, ws.value - 1, good,
                              good, None) == sfa.SFA_ERR_INVALID_ARG
    d.B = 0  # nothing to do
    assert lib.sfa_hsa_select(ctypes.byref(d), ctypes.byref(p), 4, 24, good, good, good, ws.value, good, good,
                              None) == 0
    d = _desc(sfa, d=96)
    assert lib.sfa_forward_blocks(ctypes.byref(d), good, good, good, good, good, good, good, None, None) == 2
    d = _desc(sfa)
    assert lib.sfa_forward_blocks(ctypes.byref(d), good, good, good, None, good, good, good, None, None) == 1


def test_dual_host_checks(sfa):
    lib = sfa.load()
    d = _desc(sfa)  # d = 64: 2 * n_split <= 8
    out = ctypes.c_size_t(0)
    assert lib.sfa_forward_dual_workspace(ctypes.byref(d), 2, ctypes.byref(out)) == 0
    assert out.value == 4 * 512 * 64 * 2 + 4 * 512 * 4
    assert lib.sfa_forward_dual_workspace(ctypes.byref(d), 5, ctypes.byref(out)) == 1
    good = 1 << 20
    # history lists missing, workspace too small: refused before any launch
    assert lib.sfa_forward_dual(ctypes.byref(d), good, good, good, good, good, None, good, good, good, good, good,
                                1, good, 1 << 20, None, None) == 1
    assert lib.sfa_forward_dual(ctypes.byref(d), good, good, good, good, good, good, good, good, good, good, good,
                                1, good, 1024, None, None) == 1


def test_binding_rejects_host_tensors(sfa):
    # the binding's own argument checks run before any CUDA call: host tensors are refused
    import torch
    o = torch.zeros(4, 128, dtype=torch.bfloat16)
    lse = torch.zeros(4, dtype=torch.float32)
    with pytest.raises(ValueError):
        sfa.lse_merge(o, lse, o, lse)
    q = torch.zeros(1, 1, 128, 128, dtype=torch.bfloat16)
    a = torch.zeros(1, 1, 1, dtype=torch.float32)
    b = torch.zeros(1, 1, 128, dtype=torch.float32)
    with pytest.raises(ValueError):
        sfa.gdn_forward(q, q, q, a, b, 128)
    frames = torch.zeros(1, 1, 1, dtype=torch.int32)
    counts = torch.ones(1, 1, dtype=torch.int32)
    with pytest.raises(ValueError):
        sfa.forward(q, q, q, frames, counts, 128)


def test_gdn_host_checks(sfa):
    lib = sfa.load()
    d = sfa.GdnDesc()
    d.B, d.H, d.T, d.P, d.d = 1, 12, 24, 1560, 128
    for f in ("q_stride", "k_stride", "v_stride", "o_stride"):
        arr = getattr(d, f)
        arr[0], arr[1], arr[2] = 12 * 24 * 1560 * 128, 24 * 1560 * 128, 128
    ws = ctypes.c_size_t(0)
    assert lib.sfa_gdn_workspace(ctypes.byref(d), ctypes.byref(ws)) == 0
    assert ws.value == 12 * 24 * 128 * 128 * (2 + 4)  # M_N bf16 and B_N fp32 per frame and head
    good = 1 << 20

    def call(w, nbytes, update=1):
        return lib.sfa_gdn_forward(ctypes.byref(d), good, good, good, good, good, None, good, good, update, w,
                                   nbytes, None, None)

    # an updating step without, with too small or with a misaligned workspace: refused before any launch
    assert call(None, 0) == sfa.SFA_ERR_INVALID_ARG
    assert call(good, ws.value - 1) == sfa.SFA_ERR_INVALID_ARG
    assert call(good + 16, ws.value) == sfa.SFA_ERR_INVALID_ARG
    d.q_stride[2] = 100  # token stride below d
    assert call(good, ws.value) == sfa.SFA_ERR_INVALID_ARG
    d.q_stride[2] = 128
    d.d = 64
    assert lib.sfa_gdn_workspace(ctypes.byref(d), ctypes.byref(ws)) == sfa.SFA_ERR_UNSUPPORTED
    assert call(good, 1 << 30) == sfa.SFA_ERR_UNSUPPORTED
    d.d, d.B = 128, 0  # nothing to do
    assert call(None, 0) == sfa.SFA_OK


def test_scheduled_split_plan(sfa):
    # the choice of key-tile ranges of a scheduled launch (n_split = 0), on the host; with
    # no GPU visible the SM count defaults to the B200's 148
    lib = sfa.load()
    # a launch of many full waves (the 41-frame LVSA shape: 3444 units) keeps one range
    d = _desc(sfa, B=1, H=12, Tq=41, T_kv=41, P=1560, d=128, Amax=21)
    assert sfa.split_plan(d) == (1, 0)
    out = ctypes.c_size_t(0)
    assert lib.sfa_forward_split_workspace(ctypes.byref(d), 0, ctypes.byref(out)) == 0
    assert out.value == _round256(8 * 12 * 41 * 7)          # the work items only
    # one query frame over 12 history frames (84 units of up to 156 key tiles): split
    d = _desc(sfa, B=1, H=12, Tq=1, T_kv=14, P=1560, d=128, Amax=12)
    k0, _ = sfa.split_plan(d)
    assert 2 <= k0 <= 16
    # two branches: the local lists keep one range, the history lists are split; on this
    # shape (the ISPA step: lists of 2 and 12 frames) into 4 ranges, the fastest of a
    # measured sweep of 4 to 10 ranges
    k_local, k_hist = sfa.split_plan(d, n_lists=2)
    assert k_local == 1 and k_hist == 4
    assert lib.sfa_forward_dual_workspace(ctypes.byref(d), 0, ctypes.byref(out)) == 0
    rows = 12 * 1560
    slices = k_local + k_hist
    assert out.value == _round256(slices * rows * 128 * 2) + _round256(slices * rows * 4) + _round256(8 * 84 * slices)
    k_blocks, _ = sfa.split_plan(d, key_blocks=True)
    assert 1 <= k_blocks <= 16
    with pytest.raises(sfa.SfaError):
        sfa.split_plan(d, n_lists=3)
    # the plans the measurements were taken with: one history call of the ISPA step in 7
    # ranges, the streaming chunk (3 query frames, lists of up to 13 frames) in 4, the
    # hsa block lists (3 query frames, up to 115 key blocks) whole
    assert sfa.split_plan(d) == (7, 0)
    assert sfa.split_plan(_desc(sfa, B=1, H=12, Tq=3, T_kv=24, P=1560, d=128, Amax=13)) == (4, 0)
    assert sfa.split_plan(_desc(sfa, B=1, H=12, Tq=3, T_kv=24, P=1560, d=128, Amax=115), key_blocks=True) == (1, 0)


def test_forward_host_host_checks(sfa):
    # sfa_forward_host: workspace size (device copies of Q, K, V, O, LSE, each rounded up to
    # 256 bytes) and refusals before anything is queued
    lib = sfa.load()
    d = _desc(sfa)  # B=1, H=2, Tq=4, T_kv=4, P=64, d=64
    out = ctypes.c_size_t(0)
    assert lib.sfa_forward_host_workspace(ctypes.byref(d), ctypes.byref(out)) == 0
    q = _round256(2 * 256 * 64 * 2)
    assert out.value == 4 * q + _round256(2 * 256 * 4)
    good = 1 << 20
    args = [good] * 7
    # n_chunks < 1
    assert lib.sfa_forward_host(ctypes.byref(d), *args, 0, good, out.value, None, None) == 1
    # no workspace, a short one, a misaligned one
    assert lib.sfa_forward_host(ctypes.byref(d), *args, 4, None, out.value, None, None) == 1
    assert lib.sfa_forward_host(ctypes.byref(d), *args, 4, good, out.value - 1, None, None) == 1
    assert lib.sfa_forward_host(ctypes.byref(d), *args, 4, good + 16, out.value, None, None) == 1
    # a missing host pointer
    assert lib.sfa_forward_host(ctypes.byref(d), None, *args[1:], 4, good, out.value, None, None) == 1
    # B = 0 is a no-op
    d0 = _desc(sfa, B=0)
    assert lib.sfa_forward_host(ctypes.byref(d0), *args, 4, None, 0, None, None) == 0


def test_hsa_pooled_host_checks(sfa):
    lib = sfa.load()
    d = _desc(sfa, Tq=3, T_kv=24, P=1560, d=128, Amax=7 * 13 + 24)
    need = ctypes.c_size_t(0)
    assert lib.sfa_hsa_workspace(ctypes.byref(d), ctypes.byref(need)) == 0
    good = 1 << 20
    assert lib.sfa_hsa_pool_keys(ctypes.byref(d), None, good, need.value, None) == 1          # no keys
    assert lib.sfa_hsa_pool_keys(ctypes.byref(d), good, good + 16, need.value, None) == 1     # misaligned
    assert lib.sfa_hsa_pool_keys(ctypes.byref(d), good, good, need.value - 1, None) == 1      # short
    p = sfa.set_params(T_kv=24, Tq=3, q_off=21, n_sink=1, n_prev=3, chunk_len=3)
    assert lib.sfa_hsa_select_pooled(ctypes.byref(d), ctypes.byref(p), 4, 24, good, good, need.value - 256,
                                     good, good, None) == 1
    assert lib.sfa_hsa_select_pooled(ctypes.byref(d), ctypes.byref(p), 4, 24, None, good, need.value,
                                     good, good, None) == 1
