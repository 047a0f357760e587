"""GPU frame-sparse attention vs the float64 oracle on the same seeded bf16 inputs.

Bar: O max-abs error <= 1e-2, LSE max-abs error <= 1e-3; frame lists bit-exact.
Small shapes are checked on every row; the full-size workloads on seeded samples of
rows (the oracle computes them one by one), in the launch configuration the bench uses.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import sets as S
from sfa_workloads import SetSpec, WORKLOADS, Workload, qkv, sample_rows, workload_qkv

from gpu_helpers import compare, gpu_sets, run_and_check, sfa

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ every row, small shapes
@pytest.mark.parametrize("name", ["tiny_dense", "tiny_sinkwin"])
def test_tiny_full(name):
    w = WORKLOADS[name]
    q, k, v = workload_qkv(w, seed=0)
    run_and_check(w, q, k, v)


SMALL = {
    # several full 128-key tiles per frame plus a ragged 72-row tail, LVSA sets
    "lvsa_p200": Workload("lvsa_p200", B=1, H=3, Tq=12, Tkv=12, q_off=0, P=200, d=128,
                          C=6, W=3, T_per=4, heads=(SetSpec("lvsa"),) * 3),
    # d = 64, P = 136 (one tile + 8 rows)
    "lvsa_d64": Workload("lvsa_d64", B=2, H=2, Tq=10, Tkv=10, q_off=0, P=136, d=64,
                         C=5, W=3, T_per=3, heads=(SetSpec("lvsa"),) * 2),
    # per-head cache kinds on a short stream, P = 160
    "stream_small": Workload("stream_small", B=1, H=5, Tq=2, Tkv=9, q_off=7, P=160, d=128,
                             n_sink=1, n_prev=2, chunk_len=2,
                             heads=(SetSpec("local"), SetSpec("anchor"), SetSpec("memory", (2, 4)),
                                    SetSpec("explicit", (0, 3, 5)), SetSpec("dense"))),
    # P = 8: one 128-key tile spans 16 consecutive frames
    "dense_p8": Workload("dense_p8", B=1, H=2, Tq=40, Tkv=40, q_off=0, P=8, d=128,
                         heads=(SetSpec("dense"), SetSpec("lvsa")), C=9, W=3, T_per=5),
    # P = 1: every token is its own frame
    "lvsa_p1": Workload("lvsa_p1", B=1, H=1, Tq=300, Tkv=300, q_off=0, P=1, d=64,
                        C=150, W=31, T_per=7, heads=(SetSpec("lvsa"),)),
    # P = 128 exactly: no ragged tiles at all
    "lvsa_p128": Workload("lvsa_p128", B=1, H=2, Tq=9, Tkv=9, q_off=0, P=128, d=128,
                          C=5, W=3, T_per=3, heads=(SetSpec("lvsa"),) * 2),
}


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("step", [0, 1])
def test_small_full(name, step):
    w = SMALL[name]
    q, k, v = workload_qkv(w, seed=step + 1)
    run_and_check(w, q, k, v, step=step)


def test_blhd_layout_and_batch():
    w = SMALL["lvsa_d64"]
    q, k, v = workload_qkv(w, seed=5)
    run_and_check(w, q, k, v, step=2, layout="blhd")


def test_custom_scale():
    # A sharp softmax (scale 0.3 instead of 1/sqrt(128) = 0.088) concentrates the weight on
    # few keys, so the bf16 rounding of P before P V no longer averages out: with
    # p^ = p (1 + e), |e| <= 2^-8, and O rounded to bf16 once more, |dO| <= 2^-7 max|v|.
    w = SMALL["lvsa_p200"]
    q, k, v = workload_qkv(w, seed=9)
    bound = 2.0 ** -7 * float(v.float().abs().max()) + 1e-5
    for scale in (0.3, 0.15, 0.05):
        o_err, l_err = run_and_check(w, q, k, v, scale=scale, o_tol=bound)
        print(f"scale {scale}: O max-abs error {o_err:.2e} (bound {bound:.2e}), LSE {l_err:.2e}")


def test_empty_sets_give_zero_and_neg_inf():
    w = Workload("empty", B=1, H=3, Tq=3, Tkv=5, q_off=0, P=40, d=128,
                 heads=(SetSpec("explicit", (-1,)), SetSpec("explicit", (4,)), SetSpec("explicit", (9, 9))))
    q, k, v = workload_qkv(w, seed=3)
    run_and_check(w, q, k, v)
    fr, cn = gpu_sets(w)
    o, lse = sfa().forward(q.cuda(), k.cuda(), v.cuda(), fr, cn, w.P)
    torch.cuda.synchronize()
    assert (o[0, 0] == 0).all() and torch.isneginf(lse[0, 0]).all()
    assert (o[0, 2] == 0).all() and torch.isneginf(lse[0, 2]).all()


def test_caller_built_sets():
    # frame lists need not come from sfa_build_sets: any strictly increasing list works
    B, H, Tq, Tkv, P, d = 1, 2, 3, 7, 96, 128
    q, k, v = qkv(B, H, Tq * P, Tkv * P, d, seed=4)
    lists = [[[0, 1, 2, 3, 4, 5, 6], [1, 3, 5], [6]], [[2], [0, 6], [0, 1, 5, 6]]]
    frames = np.full((H, Tq, 7), -1, np.int32)
    counts = np.zeros((H, Tq), np.int32)
    for h in range(H):
        for t in range(Tq):
            frames[h, t, :len(lists[h][t])] = lists[h][t]
            counts[h, t] = len(lists[h][t])
    o, lse = sfa().forward(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(frames).cuda(),
                           torch.from_numpy(counts).cuda(), P)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(q, k, v, frames, counts, P, 1 / math.sqrt(d))
    compare(o.float().cpu().reshape(-1, d).numpy(), lse.cpu().reshape(-1).numpy(), o_ref, l_ref)


@pytest.mark.parametrize("name", ["lvsa_p200", "lvsa_d64"])
def test_repeat_runs_identical_and_correct(name):
    # repeated launches must agree bit for bit (no read of O before its last P V lands)
    w = SMALL[name]
    q, k, v = workload_qkv(w, seed=2)
    run_and_check(w, q, k, v)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    fr, cn = gpu_sets(w)
    o1, l1 = sfa().forward(qc, kc, vc, fr, cn, w.P)
    for _ in range(12):
        o2, l2 = sfa().forward(qc, kc, vc, fr, cn, w.P)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("d,P", [(64, 192), (128, 192), (128, 320)])
def test_running_max_rescale_path(d, P):
    # Keys of frame f are scaled by 2^(f // 2) (exact in bf16), so a row's running max grows
    # by far more than 2^8 from tile to tile and O is rescaled in flight many times.  The
    # softmax ends up sharp, so the bound is the bf16-P one: |dO| <= 2^-7 max|v|.  P = 320
    # gives every frame a CTA with one query tile (S two key tiles ahead of its softmax),
    # whose rescales first wait for the previous tile's P V.
    T, H = 8, 2
    w = Workload("rescale", B=1, H=H, Tq=T, Tkv=T, q_off=0, P=P, d=d, heads=(SetSpec("dense"),) * H)
    q, k, v = workload_qkv(w, seed=6)
    factor = (2.0 ** (torch.arange(T * P) // P // 2)).to(torch.float32)
    k = (k.float() * factor[None, None, :, None]).to(torch.bfloat16)
    assert torch.isfinite(k.float()).all()
    bound = 2.0 ** -7 * float(v.float().abs().max()) + 1e-5
    o_err, l_err = run_and_check(w, q, k, v, o_tol=bound)
    print(f"rescale path, d = {d}, P = {P}: O max-abs error {o_err:.2e} (bound {bound:.2e}), LSE {l_err:.2e}")


@pytest.mark.parametrize("d,P", [(64, 192), (128, 192), (128, 320)])
def test_moderate_max_growth_path(d, P):
    # One query row repeated; every key of frame f is that row scaled so that it scores
    # 1.5 f in log2 units after the softmax scale.  The first key tile of each new frame
    # lifts the row max by 1.5, far below 2^8, but its row sum against the stale max
    # (128 x 2^1.5) exceeds the limit of 256, so that tile takes the exact pass and adopts
    # the larger max; the frame's second tile (64 keys at P = 192) stays on the streaming
    # pass.  Bound as in the rescale test: bf16 P, |dO| <= 2^-7 max|v|.
    T, H = 8, 2
    w = Workload("growth", B=1, H=H, Tq=T, Tkv=T, q_off=0, P=P, d=d, heads=(SetSpec("dense"),) * H)
    q, _, v = workload_qkv(w, seed=7)
    q0 = q[:, :, :1, :].float()                              # [B, H, 1, d]
    q = q0.expand(-1, -1, T * P, -1).to(torch.bfloat16).contiguous()
    sl2 = (1.0 / math.sqrt(d)) / math.log(2.0)               # softmax scale in log2 units
    beta = 1.5 * (torch.arange(T * P) // P).to(torch.float32) / sl2
    k = (beta[None, None, :, None] * q0 / (q0 * q0).sum(-1, keepdim=True)).to(torch.bfloat16)
    assert torch.isfinite(k.float()).all()
    bound = 2.0 ** -7 * float(v.float().abs().max()) + 1e-5
    o_err, l_err = run_and_check(w, q, k, v, o_tol=bound)
    print(f"moderate growth, d = {d}, P = {P}: O max-abs error {o_err:.2e} (bound {bound:.2e}), LSE {l_err:.2e}")


# ------------------------------------------------------------------ full-size workloads, sampled rows
@pytest.fixture(scope="module")
def lvsa41_inputs():
    return workload_qkv(WORKLOADS["lvsa41"], seed=0)


def test_lvsa41_step0_sampled(lvsa41_inputs):
    w = WORKLOADS["lvsa41"]
    rng = np.random.default_rng(0)
    rows = [sample_rows(w, 256, seed=0)]
    for h in range(w.H):  # boundary frames 0 and 40: 128 rows each per head
        base = h * w.Lq
        for t in (0, 40):
            rows.append(base + t * w.P + rng.integers(0, w.P, 128))
    for h in (0, 11):     # every row of the middle frame for two heads
        rows.append(h * w.Lq + 20 * w.P + np.arange(w.P))
    rows = np.unique(np.concatenate(rows)).astype(np.int64)
    run_and_check(w, *lvsa41_inputs, step=0, rows=rows)


@pytest.mark.parametrize("step", [1, 2, 3])
def test_lvsa41_other_steps_sampled(lvsa41_inputs, step):
    w = WORKLOADS["lvsa41"]
    run_and_check(w, *lvsa41_inputs, step=step, rows=sample_rows(w, 48, seed=step))


def test_long121_sampled():
    w = WORKLOADS["long121"]
    q, k, v = workload_qkv(w, seed=0)
    run_and_check(w, q, k, v, step=0, rows=sample_rows(w, 256, seed=0))


def test_stream_sampled():
    w = WORKLOADS["stream"]
    q, k, v = workload_qkv(w, seed=0)
    rows = [sample_rows(w, 384, seed=0)]
    for h in (0, 4, 8):   # all rows of query frame 1 for one head of each kind
        rows.append(h * w.Lq + 1 * w.P + np.arange(w.P))
    rows = np.unique(np.concatenate(rows)).astype(np.int64)
    run_and_check(w, q, k, v, rows=rows)


def test_forward_host_pipeline_equals_device_forward():
    # the host-to-host call (copies pipelined with the attention over head groups) gives
    # exactly the device call's result
    w = Workload("host", B=2, H=5, Tq=3, Tkv=5, q_off=2, P=200, d=128, n_sink=1, n_prev=1, chunk_len=1,
                 heads=(SetSpec("anchor"),) * 5)
    q, k, v = workload_qkv(w, seed=12)
    fr, cn = gpu_sets(w)
    o_ref, l_ref = sfa().forward(q.cuda(), k.cuda(), v.cuda(), fr, cn, w.P)
    qp, kp, vp = (x.pin_memory() for x in (q, k, v))
    for n_chunks in (1, 3, 7, 100):
        o, l = sfa().forward_host(qp, kp, vp, fr, cn, w.P, n_chunks=n_chunks)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref.cpu()) and torch.equal(l, l_ref.cpu())


def test_forward_host_d64_and_pageable_memory():
    # sfa_forward_host at d = 64 with a ragged frame (P = 136), from pageable host memory
    # (the copies then run synchronously): the device call's result exactly
    w = Workload("host64", B=1, H=3, Tq=4, Tkv=4, q_off=0, P=136, d=64, C=3, W=3, T_per=2,
                 heads=(SetSpec("lvsa"),) * 3)
    q, k, v = workload_qkv(w, seed=13)
    fr, cn = gpu_sets(w)
    o_ref, l_ref = sfa().forward(q.cuda(), k.cuda(), v.cuda(), fr, cn, w.P)
    o, l = sfa().forward_host(q, k, v, fr, cn, w.P, out_host=torch.empty(q.shape, dtype=torch.bfloat16),
                              lse_host=torch.empty(w.B, w.H, w.Lq), n_chunks=2)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref.cpu()) and torch.equal(l, l_ref.cpu())
