"""CPU oracle for frame-sparse attention.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the bench's CPU-baseline /
reference leg may import this package.  The product path (the CUDA library and
its binding) never imports it, and it shares no code with that path.

* ``attention``  - float64 attention restricted to A(h, t) (C, ``sfa_oracle.c``)
* ``sets``       - attended-frame-set rules (Python, ``sets.py``)
* ``lse_merge``  - merge of two partial attentions by LSE (numpy, ``merge.py``)
* ``hsa``        - hierarchical frame/block selection and block-list attention
                   (numpy float64, ``hsa.py``)
* ``gdn``        - ARL2 inter-frame gated delta rule over frames (numpy float64,
                   ``gdn.py``)
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from . import sets  # noqa: F401
from .merge import lse_merge  # noqa: F401
from . import hsa  # noqa: F401
from . import gdn  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sfa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (plain C99, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=c99", "-O2", "-fPIC", "-shared", "-o", tmp, _SRC,
                               "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_attention.restype = ctypes.c_int
        lib.oracle_attention.argtypes = (
            [ctypes.c_int] * 6 + [ctypes.c_double] + [ctypes.c_void_p] * 5 + [ctypes.c_int]
            + [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int])
        _lib = lib
    return _lib


def _bf16_bits(x) -> np.ndarray:
    """bf16 tensor/array -> contiguous uint16 bit patterns."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            assert x.dtype == torch.bfloat16
            return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16
    return x


def attention(q, k, v, frames, counts, P: int, scale: float, rows=None, n_threads: int = 0):
    """Float64 attention of each query row over the tokens of its attended frames.

    q: bf16 [B, H, Tq*P, d]; k, v: bf16 [B, H, Tkv*P, d] (torch or uint16 bits).
    frames: int32 [H, Tq, Amax]; counts: int32 [H, Tq].
    rows: optional flat row ids ``(b*H + h)*Tq*P + i``; None means every row.
    Returns (O float64 [n_rows, d], LSE float64 [n_rows]).
    """
    qb, kb, vb = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    B, H, Lq, d = qb.shape
    Lkv = kb.shape[2]
    assert Lq % P == 0 and Lkv % P == 0
    Tq, Tkv = Lq // P, Lkv // P
    frames = np.ascontiguousarray(frames, dtype=np.int32)
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    assert frames.shape[:2] == (H, Tq) and counts.shape == (H, Tq)
    Amax = frames.shape[2]
    if rows is None:
        n_rows = B * H * Lq
        rows_ptr = None
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = rows.size
        rows_ptr = rows.ctypes.data
    o = np.zeros((n_rows, d), dtype=np.float64)
    lse = np.zeros(n_rows, dtype=np.float64)
    rc = _load().oracle_attention(B, H, Tq, Tkv, P, d, float(scale), qb.ctypes.data,
                                  kb.ctypes.data, vb.ctypes.data, frames.ctypes.data,
                                  counts.ctypes.data, Amax, rows_ptr, n_rows, o.ctypes.data,
                                  lse.ctypes.data, n_threads)
    if rc != 0:
        raise RuntimeError(f"oracle_attention failed with code {rc}")
    return o, lse
