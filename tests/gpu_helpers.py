"""Shared plumbing for the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, and compare."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from oracle import sets as S

O_TOL = 1e-2     # max-abs error allowed on O (bf16 output)
LSE_TOL = 1e-3   # max-abs error allowed on LSE (fp32)


def sfa():
    import frame_sparse_attention_b200 as m
    m.load()
    return m


def set_params(w, step=0):
    return sfa().set_params(T_kv=w.Tkv, Tq=w.Tq, q_off=w.q_off, C=max(w.C, 1), W=max(w.W, 1),
                            T_per=w.T_per, step=step, n_sink=w.n_sink, n_prev=w.n_prev,
                            chunk_len=w.chunk_len)


def extra_tensor(w):
    n_extra = max((len(hs.extra) for hs in w.heads), default=0)
    if n_extra == 0:
        return None
    ex = torch.full((w.H, n_extra), -1, dtype=torch.int32)
    for h, hs in enumerate(w.heads):
        ex[h, :len(hs.extra)] = torch.tensor(hs.extra, dtype=torch.int32)
    return ex.cuda()


def gpu_sets(w, step=0, Amax=None):
    m = sfa()
    kinds = [hs.kind for hs in w.heads]
    return m.build_sets(set_params(w, step), kinds, extra_tensor(w), Amax)


def oracle_sets(w, step, Amax):
    return S.workload_sets(w, step=step, Amax=Amax)


def check_sets_equal(w, step=0):
    fr, cn = gpu_sets(w, step)
    Amax = fr.shape[2]
    ofr, ocn = oracle_sets(w, step, Amax)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cn.cpu().numpy(), ocn)
    np.testing.assert_array_equal(fr.cpu().numpy(), ofr)
    return fr, cn, ofr, ocn


def compare(o_gpu, lse_gpu, o_ref, lse_ref, o_tol=O_TOL, lse_tol=LSE_TOL):
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    assert o_gpu.shape == o_ref.shape
    assert np.isfinite(o_gpu).all(), "non-finite O"
    o_err = np.abs(o_gpu - o_ref).max() if o_ref.size else 0.0
    ninf_ref = np.isneginf(lse_ref)
    np.testing.assert_array_equal(np.isneginf(lse_gpu), ninf_ref)
    fin = ~ninf_ref
    lse_err = np.abs(lse_gpu[fin] - lse_ref[fin]).max() if fin.any() else 0.0
    assert o_err <= o_tol, f"O max-abs error {o_err:.3e} > {o_tol}"
    assert lse_err <= lse_tol, f"LSE max-abs error {lse_err:.3e} > {lse_tol}"
    return o_err, lse_err


def run_and_check(w, q, k, v, step=0, rows=None, scale=None, layout="bhld", o_tol=O_TOL):
    """GPU forward (sets built on the GPU) vs oracle (sets from the oracle) on `rows`."""
    m = sfa()
    scale = 1.0 / math.sqrt(w.d) if scale is None else scale
    fr, cn, ofr, ocn = check_sets_equal(w, step)
    if layout == "blhd":
        qc = q.transpose(1, 2).contiguous().cuda().transpose(1, 2)
        kc = k.transpose(1, 2).contiguous().cuda().transpose(1, 2)
        vc = v.transpose(1, 2).contiguous().cuda().transpose(1, 2)
        out = torch.empty(w.B, w.Lq, w.H, w.d, dtype=torch.bfloat16, device="cuda").transpose(1, 2)
    else:
        qc, kc, vc, out = q.cuda(), k.cuda(), v.cuda(), None
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = m.forward(qc, kc, vc, fr, cn, w.P, scale=scale, out=out, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, m.error_string(status.item())
    o_flat = o.float().cpu().reshape(-1, w.d).numpy() if layout == "bhld" else \
        o.float().cpu().contiguous().reshape(-1, w.d).numpy()
    lse_flat = lse.cpu().reshape(-1).numpy()
    o_ref, lse_ref = oracle.attention(q, k, v, ofr, ocn, w.P, scale, rows=rows)
    if rows is not None:
        o_flat, lse_flat = o_flat[rows], lse_flat[rows]
    return compare(o_flat, lse_flat, o_ref, lse_ref, o_tol=o_tol)
