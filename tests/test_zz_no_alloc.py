"""sfa_forward_split_noalloc: the split-KV forward for callers that cannot allocate.

Callers whose device memory belongs to an allocator they may not call into, or that
must not call cudaMalloc / cudaFree (both synchronise the device), get the split-KV
scratch from a fixed array inside the library instead of a workspace argument.  This
test calls that entry point through the C ABI twice in a row, on different shapes.  It
launches the same kernels as sfa_forward_split given a PyTorch-allocated workspace, so
each result must equal that one bit for bit; each is also checked against the float64
oracle with the tolerance the parity tests use.  It also checks that a request larger
than the array is refused before anything runs.
"""
import ctypes
import math

import pytest
import torch

from sfa_workloads import SetSpec, Workload, workload_qkv

import oracle

from gpu_helpers import compare, gpu_sets, oracle_sets, sfa

pytestmark = pytest.mark.gpu

CASES = [
    # per-head cache kinds, d = 128, 4 key ranges per unit
    (Workload("noalloc_stream", B=1, H=5, Tq=2, Tkv=9, q_off=7, P=160, d=128, n_sink=1, n_prev=2,
              chunk_len=2, heads=(SetSpec("local"), SetSpec("anchor"), SetSpec("memory", (2, 4)),
                                  SetSpec("explicit", (0, 3, 5)), SetSpec("dense"))), 4, 1),
    # LVSA sets, d = 64, two batch entries, 2 key ranges per unit
    (Workload("noalloc_lvsa", B=2, H=2, Tq=10, Tkv=10, q_off=0, P=136, d=64, C=5, W=3, T_per=3,
              heads=(SetSpec("lvsa"),) * 2), 2, 2),
]


def _noalloc(q, k, v, frames, counts, P, n_split, status):
    m = sfa()
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    desc = m.attn_desc(q, k, v, out, P, frames.shape[2])
    rc = m.load().sfa_forward_split_noalloc(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                            frames.data_ptr(), counts.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                            n_split, status.data_ptr(),
                                            torch.cuda.current_stream().cuda_stream)
    assert rc == m.SFA_OK, m.error_string(rc)
    return out, lse


def test_noalloc_matches_split_forward_on_two_calls_in_a_row():
    m = sfa()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for w, n_split, seed in CASES:
        q, k, v = (x.cuda() for x in workload_qkv(w, seed=seed))
        fr, cn = gpu_sets(w)
        o_ref, l_ref = m.forward_split(q, k, v, fr, cn, w.P, n_split)
        o, lse = _noalloc(q, k, v, fr, cn, w.P, n_split, status)
        torch.cuda.synchronize()
        assert status.item() == 0
        # the same kernels on the same inputs: identical results
        assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
        ofr, ocn = oracle_sets(w, 0, fr.shape[2])
        o_or, l_or = oracle.attention(q.cpu(), k.cpu(), v.cpu(), ofr, ocn, w.P, 1 / math.sqrt(w.d))
        compare(o.float().cpu().reshape(-1, w.d).numpy(), lse.cpu().reshape(-1).numpy(), o_or, l_or)


def test_noalloc_refuses_more_than_its_scratch():
    m = sfa()
    lib = m.load()
    d = m.AttnDesc()
    # 41 frames of 1560 tokens, 12 heads, d = 128, 2 ranges: ~400 MB of workspace
    d.B, d.H, d.Tq, d.T_kv, d.P, d.d, d.scale, d.Amax = 1, 12, 41, 41, 1560, 128, 0.088, 21
    for f in ("q_stride", "k_stride", "v_stride", "o_stride"):
        arr = getattr(d, f)
        arr[0], arr[1], arr[2] = 12 * 63960 * 128, 63960 * 128, 128
    need = ctypes.c_size_t(0)
    assert lib.sfa_forward_split_workspace(ctypes.byref(d), 2, ctypes.byref(need)) == 0
    assert need.value > 32 * 1024 * 1024
    good = 1 << 20  # never dereferenced: the size check comes first
    assert lib.sfa_forward_split_noalloc(ctypes.byref(d), good, good, good, good, good, good, good, 2,
                                         None, None) == m.SFA_ERR_INVALID_ARG
