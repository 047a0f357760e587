"""GPU set builder vs the set oracle: frame lists and counts must be bit-identical."""
import numpy as np
import pytest
import torch

from sfa_workloads import SetSpec, WORKLOADS, Workload

from gpu_helpers import check_sets_equal, oracle_sets, sfa

pytestmark = pytest.mark.gpu

CASES = [("lvsa41", s) for s in range(4)] + [("long121", s) for s in range(6)] + [
    ("stream", 0), ("tiny_dense", 0), ("tiny_sinkwin", 0), ("lsemerge_local", 0),
    ("lsemerge_hist", 0), ("lsemerge_full", 0)]


@pytest.mark.parametrize("name,step", CASES)
def test_workload_sets_bit_exact(name, step):
    check_sets_equal(WORKLOADS[name], step)


def test_random_parameter_sweep_bit_exact():
    rng = np.random.default_rng(1234)
    kinds_all = ["dense", "lvsa", "local", "anchor", "memory", "explicit"]
    for trial in range(60):
        T = int(rng.integers(1, 70))
        Tq = int(rng.integers(1, T + 1))
        q_off = int(rng.integers(0, T - Tq + 1))
        H = int(rng.integers(1, 7))
        n_extra = int(rng.integers(0, 6))
        heads = []
        for _ in range(H):
            k = kinds_all[int(rng.integers(0, 6))]
            ex = tuple(int(x) for x in rng.integers(-2, T + 3, size=n_extra)) if k in ("memory", "explicit") else ()
            heads.append(SetSpec(k, ex))
        if n_extra and not any(hs.extra for hs in heads):
            heads[0] = SetSpec("explicit", tuple(int(x) for x in rng.integers(-2, T + 3, size=n_extra)))
        w = Workload(f"sweep{trial}", B=1, H=H, Tq=Tq, Tkv=T, q_off=q_off, P=1,
                     d=64, C=int(rng.integers(1, T + 4)), W=int(rng.integers(1, T + 4)),
                     T_per=int(rng.integers(1, 9)), n_sink=int(rng.integers(0, 4)),
                     n_prev=int(rng.integers(0, 5)), chunk_len=int(rng.integers(1, 5)),
                     heads=tuple(heads))
        for step in (0, int(rng.integers(1, 20))):
            check_sets_equal(w, step)


def test_amax_padding_larger_than_bound():
    w = WORKLOADS["lvsa41"]
    fr, cn = __import__("gpu_helpers").gpu_sets(w, 0, Amax=30)
    ofr, ocn = oracle_sets(w, 0, 30)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(fr.cpu().numpy(), ofr)
    np.testing.assert_array_equal(cn.cpu().numpy(), ocn)
    assert (fr.cpu().numpy()[:, :, 21:] == -1).all()


def test_build_is_deterministic():
    m = sfa()
    w = WORKLOADS["long121"]
    a = __import__("gpu_helpers").gpu_sets(w, 3)
    b = __import__("gpu_helpers").gpu_sets(w, 3)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert m is not None
