"""Device-side error reporting without faulting the GPU.

* a malformed frame list is caught on the device and reported as SFA_ERR_BAD_SET;
* a pipeline wait that nothing satisfies (the softmax warps withhold their first
  probability tile, a test hook) runs into its iteration limit: the kernel reports
  SFA_ERR_TIMEOUT, drains its copies, frees tensor memory and returns, and the
  context stays usable for the next, normal call.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from sfa_workloads import qkv

from gpu_helpers import compare, sfa

pytestmark = pytest.mark.gpu

B, H, Tq, Tkv, P, d = 1, 2, 2, 4, 192, 128


def _inputs():
    q, k, v = qkv(B, H, Tq * P, Tkv * P, d, seed=8)
    return q, k, v, q.cuda(), k.cuda(), v.cuda()


def _sets(lists, Amax=4):
    frames = np.full((H, Tq, Amax), -1, np.int32)
    counts = np.zeros((H, Tq), np.int32)
    for h in range(H):
        for t in range(Tq):
            frames[h, t, :len(lists[h][t])] = lists[h][t]
            counts[h, t] = len(lists[h][t])
    return frames, counts


@pytest.mark.parametrize("bad", [[2, 1], [1, 1], [0, 4], [-1, 2]])
def test_bad_frame_list_reported(bad):
    q, k, v, qc, kc, vc = _inputs()
    frames, counts = _sets([[[0, 1], bad], [[3], [0, 2, 3]]])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = sfa().forward(qc, kc, vc, torch.from_numpy(frames).cuda(), torch.from_numpy(counts).cuda(), P,
                           dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == sfa().SFA_ERR_BAD_SET
    # the well-formed units are still right (oracle on the same lists minus the bad one)
    good_frames, good_counts = _sets([[[0, 1], []], [[3], [0, 2, 3]]])
    o_ref, l_ref = oracle.attention(q, k, v, good_frames, good_counts, P, 1 / math.sqrt(d))
    o_g = o.float().cpu().reshape(B, H, Tq, P, d).numpy()
    l_g = lse.cpu().reshape(B, H, Tq, P).numpy()
    o_r = o_ref.reshape(B, H, Tq, P, d)
    l_r = l_ref.reshape(B, H, Tq, P)
    for h, t in ((0, 0), (1, 0), (1, 1)):
        compare(o_g[0, h, t], l_g[0, h, t], o_r[0, h, t], l_r[0, h, t])
    assert np.isnan(l_g[0, 0, 1]).all()


def test_count_above_amax_reported():
    _, _, _, qc, kc, vc = _inputs()
    frames, counts = _sets([[[0], [1]], [[2], [3]]])
    counts[1, 1] = 9
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sfa().forward(qc, kc, vc, torch.from_numpy(frames).cuda(), torch.from_numpy(counts).cuda(), P,
                  dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == sfa().SFA_ERR_BAD_SET


def test_stalled_pipeline_times_out_and_context_survives():
    q, k, v, qc, kc, vc = _inputs()
    frames, counts = _sets([[[0, 1, 2, 3], [1, 2]], [[0, 3], [2]]])
    fr, cn = torch.from_numpy(frames).cuda(), torch.from_numpy(counts).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sfa().forward(qc, kc, vc, fr, cn, P, dev_status=status, timeout_us=20000,
                  debug_flags=sfa().SFA_DEBUG_STALL_SOFTMAX)
    torch.cuda.synchronize()
    assert status.item() == sfa().SFA_ERR_TIMEOUT
    # same context, normal call: correct results
    status.zero_()
    o, lse = sfa().forward(qc, kc, vc, fr, cn, P, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    o_ref, l_ref = oracle.attention(q, k, v, frames, counts, P, 1 / math.sqrt(d))
    compare(o.float().cpu().reshape(-1, d).numpy(), lse.cpu().reshape(-1).numpy(), o_ref, l_ref)
