"""ctypes binding of libsfa.so (the C ABI declared in include/sfa.h).

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  If the
shared library is missing this module raises; there is no fallback path.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsfa.so")

# sfa_status
SFA_OK = 0
SFA_ERR_INVALID_ARG = 1
SFA_ERR_UNSUPPORTED = 2
SFA_ERR_CUDA = 3
SFA_ERR_TIMEOUT = 4
SFA_ERR_BAD_SET = 5

# sfa_set_kind
SET_KINDS = {"dense": 0, "lvsa": 1, "local": 2, "anchor": 3, "memory": 4, "explicit": 5}
SFA_MAX_HEADS = 1024
SFA_DEBUG_STALL_SOFTMAX = 1
SFA_DEBUG_STALL_GDN_STATE = 2


class SfaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {error_string(status)} (status {status})")


class SetParams(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("T_kv", "Tq", "q_off", "C", "W", "T_per", "step", "n_sink", "n_prev", "chunk_len")]


class AttnDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("Tq", ctypes.c_int32),
                ("T_kv", ctypes.c_int32), ("P", ctypes.c_int32), ("d", ctypes.c_int32),
                ("scale", ctypes.c_float), ("Amax", ctypes.c_int32),
                ("q_stride", ctypes.c_int64 * 3), ("k_stride", ctypes.c_int64 * 3),
                ("v_stride", ctypes.c_int64 * 3), ("o_stride", ctypes.c_int64 * 3),
                ("timeout_us", ctypes.c_uint32), ("debug_flags", ctypes.c_uint32)]


class GdnDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("T", ctypes.c_int32), ("P", ctypes.c_int32),
                ("d", ctypes.c_int32), ("q_stride", ctypes.c_int64 * 3), ("k_stride", ctypes.c_int64 * 3),
                ("v_stride", ctypes.c_int64 * 3), ("o_stride", ctypes.c_int64 * 3), ("timeout_us", ctypes.c_uint32),
                ("debug_flags", ctypes.c_uint32)]


_lib = None

EXPORTS = ("sfa_error_string", "sfa_version", "sfa_set_max_count", "sfa_build_sets", "sfa_forward",
           "sfa_forward_split_workspace", "sfa_forward_split", "sfa_forward_split_noalloc", "sfa_forward_paged",
           "sfa_lse_merge", "sfa_hsa_max_count", "sfa_hsa_workspace", "sfa_hsa_select", "sfa_forward_blocks",
           "sfa_forward_blocks_split", "sfa_forward_blocks_split_workspace", "sfa_forward_split_plan",
           "sfa_forward_host_workspace", "sfa_forward_host", "sfa_hsa_pool_keys", "sfa_hsa_select_pooled",
           "sfa_forward_dual_workspace", "sfa_forward_dual", "sfa_gdn_workspace", "sfa_gdn_forward")


def load():
    """Load libsfa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m frame_sparse_attention_b200.build` (needs nvcc)")
    lib = ctypes.CDLL(LIB_PATH)
    i32, i64, vp, st = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
    lib.sfa_error_string.restype = ctypes.c_char_p
    lib.sfa_error_string.argtypes = [st]
    lib.sfa_version.restype = i32
    lib.sfa_version.argtypes = []
    lib.sfa_set_max_count.restype = st
    lib.sfa_set_max_count.argtypes = [ctypes.POINTER(SetParams), i32, ctypes.POINTER(i32), i32,
                                      ctypes.POINTER(i32)]
    lib.sfa_build_sets.restype = st
    lib.sfa_build_sets.argtypes = [ctypes.POINTER(SetParams), i32, ctypes.POINTER(i32), vp, i32, vp, vp,
                                   i32, vp]
    lib.sfa_forward.restype = st
    lib.sfa_forward.argtypes = [ctypes.POINTER(AttnDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.sfa_forward_split_workspace.restype = st
    lib.sfa_forward_split_workspace.argtypes = [ctypes.POINTER(AttnDesc), i32, ctypes.POINTER(ctypes.c_size_t)]
    lib.sfa_forward_split.restype = st
    lib.sfa_forward_split.argtypes = [ctypes.POINTER(AttnDesc), vp, vp, vp, vp, vp, vp, vp, i32, vp,
                                      ctypes.c_size_t, vp, vp]
    lib.sfa_forward_split_noalloc.restype = st
    lib.sfa_forward_split_noalloc.argtypes = [ctypes.POINTER(AttnDesc), vp, vp, vp, vp, vp, vp, vp, i32, vp, vp]
    lib.sfa_forward_paged.restype = st
    lib.sfa_forward_paged.argtypes = [ctypes.POINTER(AttnDesc), vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp]
    lib.sfa_lse_merge.restype = st
    lib.sfa_lse_merge.argtypes = [i64, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.sfa_hsa_max_count.restype = st
    lib.sfa_hsa_max_count.argtypes = [ctypes.POINTER(SetParams), i32, i32, i32, ctypes.POINTER(i32)]
    lib.sfa_hsa_workspace.restype = st
    lib.sfa_hsa_workspace.argtypes = [ctypes.POINTER(AttnDesc), ctypes.POINTER(ctypes.c_size_t)]
    lib.sfa_hsa_select.restype = st
    lib.sfa_hsa_select.argtypes = [ctypes.POINTER(AttnDesc), ctypes.POINTER(SetParams), i32, i32, vp, vp, vp,
                                   ctypes.c_size_t, vp, vp, vp]
    lib.sfa_hsa_pool_keys.restype = st
    lib.sfa_hsa_pool_keys.argtypes = [ctypes.POINTER(AttnDesc), vp, vp, ctypes.c_size_t, vp]
    lib.sfa_hsa_select_pooled.restype = st
    lib.sfa_hsa_select_pooled.argtypes = [ctypes.POINTER(AttnDesc), ctypes.POINTER(SetParams), i32, i32, vp, vp,
                                          ctypes.c_size_t, vp, vp, vp]
    lib.sfa_forward_dual_workspace.restype = st
    lib.sfa_forward_dual_workspace.argtypes = [ctypes.POINTER(AttnDesc), i32, ctypes.POINTER(ctypes.c_size_t)]
    lib.sfa_forward_dual.restype = st
    lib.sfa_forward_dual.argtypes = [ctypes.POINTER(AttnDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp,
                                     ctypes.c_size_t, vp, vp]
    lib.sfa_gdn_forward.restype = st
    lib.sfa_gdn_workspace.restype = st
    lib.sfa_gdn_workspace.argtypes = [ctypes.POINTER(GdnDesc), ctypes.POINTER(ctypes.c_size_t)]
    lib.sfa_gdn_forward.argtypes = [ctypes.POINTER(GdnDesc), vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, ctypes.c_size_t,
                                    vp, vp]
    lib.sfa_forward_blocks_split.restype = st
    lib.sfa_forward_blocks_split.argtypes = [ctypes.POINTER(AttnDesc), vp, vp, vp, vp, vp, vp, vp, i32, vp,
                                             ctypes.c_size_t, vp, vp]
    lib.sfa_forward_blocks_split_workspace.restype = st
    lib.sfa_forward_blocks_split_workspace.argtypes = [ctypes.POINTER(AttnDesc), i32, ctypes.POINTER(ctypes.c_size_t)]
    lib.sfa_forward_split_plan.restype = st
    lib.sfa_forward_split_plan.argtypes = [ctypes.POINTER(AttnDesc), i32, i32, ctypes.POINTER(i32), ctypes.POINTER(i32)]
    lib.sfa_forward_host_workspace.restype = st
    lib.sfa_forward_host_workspace.argtypes = [ctypes.POINTER(AttnDesc), ctypes.POINTER(ctypes.c_size_t)]
    lib.sfa_forward_host.restype = st
    lib.sfa_forward_host.argtypes = [ctypes.POINTER(AttnDesc), vp, vp, vp, vp, vp, vp, vp, i32, vp, ctypes.c_size_t,
                                     vp, vp]
    lib.sfa_forward_blocks.restype = st
    lib.sfa_forward_blocks.argtypes = [ctypes.POINTER(AttnDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp]
    _lib = lib
    return lib


def error_string(status: int) -> str:
    return load().sfa_error_string(status).decode()


def version() -> int:
    return load().sfa_version()


def _require(cond: bool, what: str):
    """Argument check of the binding (a ValueError, kept under ``python -O``)."""
    if not cond:
        raise ValueError(what)


def _check(status: int, what: str):
    if status != SFA_OK:
        raise SfaError(status, what)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _kinds(kinds):
    arr = (ctypes.c_int32 * len(kinds))()
    for i, k in enumerate(kinds):
        arr[i] = SET_KINDS[k] if isinstance(k, str) else int(k)
    return arr


def set_params(*, T_kv, Tq, q_off=0, C=1, W=1, T_per=1, step=0, n_sink=0, n_prev=0, chunk_len=1):
    return SetParams(T_kv, Tq, q_off, C, W, T_per, step, n_sink, n_prev, chunk_len)


def set_max_count(params: SetParams, kinds, n_extra: int = 0) -> int:
    out = ctypes.c_int32(0)
    _check(load().sfa_set_max_count(ctypes.byref(params), len(kinds), _kinds(kinds), n_extra,
                                    ctypes.byref(out)), "sfa_set_max_count")
    return out.value


def build_sets(params: SetParams, kinds, extra: torch.Tensor | None = None, Amax: int | None = None,
               frames: torch.Tensor | None = None, counts: torch.Tensor | None = None, stream=None):
    """Attended frame lists on the device: frames int32 [H, Tq, Amax], counts int32 [H, Tq]."""
    H = len(kinds)
    n_extra = 0 if extra is None else int(extra.shape[1])
    if Amax is None:
        Amax = max(1, set_max_count(params, kinds, n_extra))
    dev = torch.device("cuda", torch.cuda.current_device()) if extra is None else extra.device
    if frames is None:
        frames = torch.empty((H, params.Tq, Amax), dtype=torch.int32, device=dev)
    if counts is None:
        counts = torch.empty((H, params.Tq), dtype=torch.int32, device=dev)
    if extra is not None:
        _require(extra.dtype == torch.int32 and extra.is_cuda and extra.is_contiguous(),
                 "expected extra.dtype == torch.int32 and extra.is_cuda and extra.is_contiguous()")
        _require(extra.shape[0] == H, "expected extra.shape[0] == H")
    _require(frames.is_contiguous() and counts.is_contiguous(),
             "expected frames.is_contiguous() and counts.is_contiguous()")
    _check(load().sfa_build_sets(ctypes.byref(params), H, _kinds(kinds), _ptr(extra), n_extra,
                                 frames.data_ptr(), counts.data_ptr(), Amax, _stream(stream)),
           "sfa_build_sets")
    return frames, counts


def attn_desc(q, k, v, o, P: int, Amax: int, scale: float | None = None, timeout_us: int = 0,
              debug_flags: int = 0, on_host: bool = False) -> AttnDesc:
    B, H, Lq, d = q.shape
    Lkv = k.shape[2]
    if Lq % P or Lkv % P:
        raise ValueError(f"sequence lengths {Lq}, {Lkv} are not multiples of P = {P}")
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        if t.dtype != torch.bfloat16 or t.is_cuda == on_host:
            raise ValueError(f"{name} must be a bf16 {'CPU' if on_host else 'CUDA'} tensor")
        if t.dim() != 4 or t.stride(3) != 1:
            raise ValueError(f"{name} must be [B, H, L, d] with d contiguous")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    desc = AttnDesc()
    desc.B, desc.H, desc.Tq, desc.T_kv, desc.P, desc.d = B, H, Lq // P, Lkv // P, P, d
    desc.scale, desc.Amax = float(scale), int(Amax)
    for field, t in (("q_stride", q), ("k_stride", k), ("v_stride", v), ("o_stride", o)):
        arr = getattr(desc, field)
        arr[0], arr[1], arr[2] = t.stride(0), t.stride(1), t.stride(2)
    desc.timeout_us = timeout_us
    desc.debug_flags = debug_flags
    return desc


def forward(q, k, v, frames, counts, P: int, scale: float | None = None, out=None, lse=None,
            dev_status=None, stream=None, timeout_us: int = 0, debug_flags: int = 0):
    """Frame-sparse attention: (O bf16 like q, LSE fp32 [B, H, Tq*P])."""
    B, H, Lq, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
    _require(lse.is_contiguous() and lse.dtype == torch.float32,
             "expected lse.is_contiguous() and lse.dtype == torch.float32")
    _require(frames.dtype == torch.int32 and counts.dtype == torch.int32,
             "expected frames.dtype == torch.int32 and counts.dtype == torch.int32")
    _require(frames.is_contiguous() and counts.is_contiguous(),
             "expected frames.is_contiguous() and counts.is_contiguous()")
    desc = attn_desc(q, k, v, out, P, frames.shape[2], scale, timeout_us, debug_flags)
    _require(tuple(frames.shape[:2]) == (H, desc.Tq) and tuple(counts.shape) == (H, desc.Tq),
             "expected tuple(frames.shape[:2]) == (H, desc.Tq) and tuple(counts.shape) == (H, desc.Tq)")
    _check(load().sfa_forward(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                              frames.data_ptr(), counts.data_ptr(), out.data_ptr(), lse.data_ptr(),
                              _ptr(dev_status), _stream(stream)), "sfa_forward")
    return out, lse


def forward_paged(q, k_cache, v_cache, slots, frames, counts, P: int, T_kv: int, scale: float | None = None,
                  out=None, lse=None, dev_status=None, stream=None, timeout_us: int = 0):
    """Frame-sparse attention with K/V read through a per-head slot table [H, T_kv]
    (logical frame -> physical frame slot of k_cache / v_cache [B, H, n_slots*P, d])."""
    B, H, Lq, d = q.shape
    n_slots = k_cache.shape[2] // P
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
    _require(slots.dtype == torch.int32 and slots.is_contiguous() and tuple(slots.shape) == (H, T_kv),
             "expected slots.dtype == torch.int32 and slots.is_contiguous() and tuple(slots.shape) == (H, T_kv)")
    _require(frames.dtype == torch.int32 and counts.dtype == torch.int32,
             "expected frames.dtype == torch.int32 and counts.dtype == torch.int32")
    _require(frames.is_contiguous() and counts.is_contiguous() and lse.is_contiguous(),
             "expected frames.is_contiguous() and counts.is_contiguous() and lse.is_contiguous()")
    desc = attn_desc(q, k_cache, v_cache, out, P, frames.shape[2], scale, timeout_us)
    desc.T_kv = T_kv
    _check(load().sfa_forward_paged(ctypes.byref(desc), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                    slots.data_ptr(), n_slots, frames.data_ptr(), counts.data_ptr(),
                                    out.data_ptr(), lse.data_ptr(), _ptr(dev_status), _stream(stream)),
           "sfa_forward_paged")
    return out, lse


def split_workspace_bytes(desc: AttnDesc, n_split: int) -> int:
    out = ctypes.c_size_t(0)
    _check(load().sfa_forward_split_workspace(ctypes.byref(desc), n_split, ctypes.byref(out)),
           "sfa_forward_split_workspace")
    return out.value


def split_plan(desc: AttnDesc, n_lists: int = 1, key_blocks: bool = False) -> tuple:
    """Key-tile ranges per unit that a scheduled call (n_split = 0) uses: (k_first, k_second)."""
    k0, k1 = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(load().sfa_forward_split_plan(ctypes.byref(desc), n_lists, 1 if key_blocks else 0, ctypes.byref(k0),
                                         ctypes.byref(k1)), "sfa_forward_split_plan")
    return k0.value, k1.value


def forward_split(q, k, v, frames, counts, P: int, n_split: int, scale: float | None = None, out=None,
                  lse=None, workspace=None, dev_status=None, stream=None, timeout_us: int = 0):
    """Split-KV frame-sparse attention (same result as forward); workspace is allocated
    here with torch when not given.  n_split = 0: the library chooses the ranges and runs
    the CTAs longest range first (a scheduled launch)."""
    B, H, Lq, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
    _require(frames.dtype == torch.int32 and counts.dtype == torch.int32,
             "expected frames.dtype == torch.int32 and counts.dtype == torch.int32")
    _require(frames.is_contiguous() and counts.is_contiguous() and lse.is_contiguous(),
             "expected frames.is_contiguous() and counts.is_contiguous() and lse.is_contiguous()")
    desc = attn_desc(q, k, v, out, P, frames.shape[2], scale, timeout_us)
    need = split_workspace_bytes(desc, n_split)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().sfa_forward_split(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                    frames.data_ptr(), counts.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                    n_split, _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream)),
           "sfa_forward_split")
    return out, lse


def lse_merge(o1, lse1, o2, lse2, out=None, lse=None, stream=None):
    """Merge two partial attentions by LSE: returns (O bf16, LSE fp32) shaped like o1 / lse1."""
    d = o1.shape[-1]
    rows = lse1.numel()
    for t in (o1, o2, lse1, lse2):
        _require(t.is_cuda and t.is_contiguous(), "expected t.is_cuda and t.is_contiguous()")
    _require(o1.dtype == torch.bfloat16 and o2.dtype == torch.bfloat16,
             "expected o1.dtype == torch.bfloat16 and o2.dtype == torch.bfloat16")
    _require(lse1.dtype == torch.float32 and lse2.dtype == torch.float32,
             "expected lse1.dtype == torch.float32 and lse2.dtype == torch.float32")
    _require(o1.numel() == rows * d and o2.shape == o1.shape and lse2.shape == lse1.shape,
             "expected o1.numel() == rows * d and o2.shape == o1.shape and lse2.shape == lse1.shape")
    if out is None:
        out = torch.empty_like(o1)
    if lse is None:
        lse = torch.empty_like(lse1)
    _check(load().sfa_lse_merge(rows, d, o1.data_ptr(), lse1.data_ptr(), o2.data_ptr(), lse2.data_ptr(),
                                out.data_ptr(), lse.data_ptr(), _stream(stream)), "sfa_lse_merge")
    return out, lse


KEY_BLOCK = 128    # tokens per key block of the hierarchical selection
QUERY_BLOCK = 256  # query rows per query block


def hsa_max_count(params: SetParams, P: int, k_frames: int, k_blocks: int) -> int:
    """Length bound of a key-block list: the smallest Amax that hsa_select accepts."""
    out = ctypes.c_int32(0)
    _check(load().sfa_hsa_max_count(ctypes.byref(params), P, k_frames, k_blocks, ctypes.byref(out)),
           "sfa_hsa_max_count")
    return out.value


def hsa_select(q, k, params: SetParams, k_frames: int, k_blocks: int, Amax: int | None = None, workspace=None,
               stream=None):
    """Hierarchical selection (pooled keys, top frames, then top blocks): (blocks int32
    [B, H, Tq, nqb, Amax] sorted key-block ids with -1 padding, counts int32 [B, H, Tq, nqb])."""
    B, H, Lq, d = q.shape
    P = Lq // params.Tq
    if Amax is None:
        Amax = hsa_max_count(params, P, k_frames, k_blocks)
    nqb = (P + QUERY_BLOCK - 1) // QUERY_BLOCK
    desc = attn_desc(q, k, k, q, P, Amax)
    nbytes = ctypes.c_size_t(0)
    _check(load().sfa_hsa_workspace(ctypes.byref(desc), ctypes.byref(nbytes)), "sfa_hsa_workspace")
    if workspace is None:
        workspace = torch.empty(max(nbytes.value, 1), dtype=torch.uint8, device=q.device)
    blocks = torch.empty((B, H, params.Tq, nqb, Amax), dtype=torch.int32, device=q.device)
    counts = torch.empty((B, H, params.Tq, nqb), dtype=torch.int32, device=q.device)
    _check(load().sfa_hsa_select(ctypes.byref(desc), ctypes.byref(params), k_frames, k_blocks, q.data_ptr(),
                                 k.data_ptr(), workspace.data_ptr(), workspace.numel(), blocks.data_ptr(),
                                 counts.data_ptr(), _stream(stream)), "sfa_hsa_select")
    return blocks, counts


def hsa_pool_keys(k, q_like, P: int, workspace, Amax: int = 1, stream=None):
    """Pool the keys' frame and block means into ``workspace`` (a uint8 CUDA tensor of
    ``sfa_hsa_workspace`` bytes for the descriptor of (q_like, k)), for later
    ``hsa_select_pooled`` calls over the same keys."""
    desc = attn_desc(q_like, k, k, q_like, P, Amax)
    _check(load().sfa_hsa_pool_keys(ctypes.byref(desc), k.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                    _stream(stream)), "sfa_hsa_pool_keys")
    return workspace


def hsa_select_pooled(q, k_like, params: SetParams, k_frames: int, k_blocks: int, workspace, Amax: int | None = None,
                      stream=None):
    """hsa_select from the pooled keys already in ``workspace`` (``hsa_pool_keys``): pools
    the queries only.  ``k_like`` gives the key shape (its data is not read)."""
    B, H, Lq, d = q.shape
    P = Lq // params.Tq
    if Amax is None:
        Amax = hsa_max_count(params, P, k_frames, k_blocks)
    nqb = (P + QUERY_BLOCK - 1) // QUERY_BLOCK
    desc = attn_desc(q, k_like, k_like, q, P, Amax)
    blocks = torch.empty((B, H, params.Tq, nqb, Amax), dtype=torch.int32, device=q.device)
    counts = torch.empty((B, H, params.Tq, nqb), dtype=torch.int32, device=q.device)
    _check(load().sfa_hsa_select_pooled(ctypes.byref(desc), ctypes.byref(params), k_frames, k_blocks, q.data_ptr(),
                                        workspace.data_ptr(), workspace.numel(), blocks.data_ptr(), counts.data_ptr(),
                                        _stream(stream)), "sfa_hsa_select_pooled")
    return blocks, counts


def hsa_workspace_bytes(q, k, P: int, Amax: int = 1) -> int:
    desc = attn_desc(q, k, k, q, P, Amax)
    nbytes = ctypes.c_size_t(0)
    _check(load().sfa_hsa_workspace(ctypes.byref(desc), ctypes.byref(nbytes)), "sfa_hsa_workspace")
    return nbytes.value


def forward_blocks(q, k, v, blocks, counts, P: int, scale: float | None = None, out=None, lse=None,
                   dev_status=None, stream=None, timeout_us: int = 0, n_split: int = 1, workspace=None):
    """Attention of every query block over its key-block list: (O bf16 like q, LSE fp32).
    n_split > 1 cuts every unit's key tiles into ranges merged by LSE; 0 schedules the
    launch (the library's choice of ranges, longest first)."""
    B, H, Lq, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
    _require(lse.is_contiguous() and lse.dtype == torch.float32,
             "expected lse.is_contiguous() and lse.dtype == torch.float32")
    _require(blocks.dtype == torch.int32 and counts.dtype == torch.int32,
             "expected blocks.dtype == torch.int32 and counts.dtype == torch.int32")
    _require(blocks.is_contiguous() and counts.is_contiguous(),
             "expected blocks.is_contiguous() and counts.is_contiguous()")
    desc = attn_desc(q, k, v, out, P, blocks.shape[-1], scale, timeout_us)
    nqb = (P + QUERY_BLOCK - 1) // QUERY_BLOCK
    _require(tuple(blocks.shape[:4]) == (B, H, desc.Tq, nqb) and tuple(counts.shape) == (B, H, desc.Tq, nqb),
             "expected tuple(blocks.shape[:4]) == (B, H, desc.Tq, nqb) and tuple(counts.shape) == (B, H, desc.Tq, nqb)")
    if n_split == 1:
        _check(load().sfa_forward_blocks(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                         blocks.data_ptr(), counts.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                         _ptr(dev_status), _stream(stream)), "sfa_forward_blocks")
        return out, lse
    if workspace is None:
        nbytes = ctypes.c_size_t(0)
        _check(load().sfa_forward_blocks_split_workspace(ctypes.byref(desc), n_split, ctypes.byref(nbytes)),
               "sfa_forward_blocks_split_workspace")
        workspace = torch.empty(max(nbytes.value, 1), dtype=torch.uint8, device=q.device)
    _check(load().sfa_forward_blocks_split(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                           blocks.data_ptr(), counts.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                           n_split, workspace.data_ptr(), workspace.numel(), _ptr(dev_status),
                                           _stream(stream)), "sfa_forward_blocks_split")
    return out, lse


def forward_dual(q, k, v, frames_local, counts_local, frames_hist, counts_hist, P: int, n_split: int = 1,
                 scale: float | None = None, out_local=None, lse_local=None, out_full=None, lse_full=None,
                 workspace=None, dev_status=None, stream=None, timeout_us: int = 0):
    """Local and history branches in one launch: (O_local, LSE_local, O_full, LSE_full), the
    full result being the LSE merge of both branches."""
    B, H, Lq, d = q.shape
    out_local = torch.empty_like(q) if out_local is None else out_local
    out_full = torch.empty_like(q) if out_full is None else out_full
    if lse_local is None:
        lse_local = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
    if lse_full is None:
        lse_full = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
    for f, c in ((frames_local, counts_local), (frames_hist, counts_hist)):
        _require(f.dtype == torch.int32 and c.dtype == torch.int32 and f.is_contiguous() and c.is_contiguous(),
                 "expected f.dtype == torch.int32 and c.dtype == torch.int32 and f.is_contiguous() and c.is_contiguous()")
    _require(frames_local.shape == frames_hist.shape, "expected frames_local.shape == frames_hist.shape")
    _require(tuple(out_local.stride()) == tuple(out_full.stride()),
             "expected tuple(out_local.stride()) == tuple(out_full.stride())")
    desc = attn_desc(q, k, v, out_full, P, frames_local.shape[2], scale, timeout_us)
    nbytes = ctypes.c_size_t(0)
    _check(load().sfa_forward_dual_workspace(ctypes.byref(desc), n_split, ctypes.byref(nbytes)),
           "sfa_forward_dual_workspace")
    if workspace is None:
        workspace = torch.empty(max(nbytes.value, 1), dtype=torch.uint8, device=q.device)
    _check(load().sfa_forward_dual(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                   frames_local.data_ptr(), counts_local.data_ptr(), frames_hist.data_ptr(),
                                   counts_hist.data_ptr(), out_local.data_ptr(), lse_local.data_ptr(),
                                   out_full.data_ptr(), lse_full.data_ptr(), n_split, workspace.data_ptr(),
                                   workspace.numel(), _ptr(dev_status), _stream(stream)), "sfa_forward_dual")
    return out_local, lse_local, out_full, lse_full


def gdn_forward(q, k, v, alpha, beta, P: int, state_in=None, state_out=None, out=None, update: bool = True,
                workspace="auto", dev_status=None, stream=None, timeout_us: int = 0, debug_flags: int = 0):
    """ARL2 inter-frame branch over the T = L / P frames of q, k, v [B, H, L, d]: (O bf16
    like q, final state fp32 [B, H, d, d]).  alpha fp32 [B, H, T], beta fp32 [B, H, L]
    (>= 0); state_in fp32 [B, H, d, d] or None (zeros).  workspace: "auto" (allocated here),
    a uint8 CUDA tensor of at least ``sfa_gdn_workspace`` bytes, or None (only for
    update=False: the update needs it).  debug_flags: SFA_DEBUG_* test hooks, 0 in normal
    use."""
    B, H, L, d = q.shape
    if L % P:
        raise ValueError(f"sequence length {L} is not a multiple of P = {P}")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or t.stride(3) != 1:
            raise ValueError(f"{name} must be a bf16 CUDA tensor [B, H, L, d] with d contiguous")
    out = torch.empty_like(q) if out is None else out
    if state_out is None:
        state_out = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device)
    for name, t in (("alpha", alpha), ("beta", beta), ("state_out", state_out)):
        _require(t.dtype == torch.float32 and t.is_contiguous(), f"{name} must be fp32 and contiguous")
    _require(tuple(alpha.shape) == (B, H, L // P) and tuple(beta.shape) == (B, H, L),
             "expected tuple(alpha.shape) == (B, H, L // P) and tuple(beta.shape) == (B, H, L)")
    if state_in is not None:
        _require(state_in.dtype == torch.float32 and state_in.is_contiguous() and tuple(state_in.shape) == (B, H, d, d),
                 "expected state_in.dtype == torch.float32 and state_in.is_contiguous() and tuple(state_in.shape) == (B, H, d, d)")
    desc = GdnDesc()
    desc.B, desc.H, desc.T, desc.P, desc.d = B, H, L // P, P, d
    for field, t in (("q_stride", q), ("k_stride", k), ("v_stride", v), ("o_stride", out)):
        arr = getattr(desc, field)
        arr[0], arr[1], arr[2] = t.stride(0), t.stride(1), t.stride(2)
    desc.timeout_us = timeout_us
    desc.debug_flags = debug_flags
    if isinstance(workspace, str):
        workspace = None
        if update:
            nbytes = ctypes.c_size_t(0)
            _check(load().sfa_gdn_workspace(ctypes.byref(desc), ctypes.byref(nbytes)), "sfa_gdn_workspace")
            workspace = torch.empty(nbytes.value, dtype=torch.uint8, device=q.device)
    ws_ptr, ws_bytes = (workspace.data_ptr(), workspace.numel()) if workspace is not None else (None, 0)
    _check(load().sfa_gdn_forward(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(), alpha.data_ptr(),
                                  beta.data_ptr(), _ptr(state_in), state_out.data_ptr(), out.data_ptr(),
                                  1 if update else 0, ws_ptr, ws_bytes, _ptr(dev_status), _stream(stream)),
           "sfa_gdn_forward")
    return out, state_out


def host_workspace_bytes(q_host, k_host, P: int, Amax: int) -> int:
    """Device workspace bytes of forward_host for these shapes."""
    desc = attn_desc(q_host, k_host, k_host, q_host, P, Amax, on_host=True)
    out = ctypes.c_size_t(0)
    _check(load().sfa_forward_host_workspace(ctypes.byref(desc), ctypes.byref(out)), "sfa_forward_host_workspace")
    return out.value


def forward_host(q_host, k_host, v_host, frames, counts, P: int, out_host=None, lse_host=None, n_chunks: int = 12,
                 scale: float | None = None, workspace=None, dev_status=None, stream=None, timeout_us: int = 0):
    """Frame-sparse attention of host tensors (sfa_forward_host): (O, LSE) in pinned host
    memory.  q_host, k_host, v_host: pinned, contiguous bf16 CPU tensors [B, H, L, d];
    frames / counts as for ``forward`` (device).  The copies in, the attention and the
    copies out run inside the library as a pipeline over (batch, head-group) chunks.  The
    call is asynchronous on ``stream`` like a kernel: synchronise before reading the
    results.  ``workspace``: a uint8 CUDA tensor of at least ``host_workspace_bytes``
    (allocated here when not given)."""
    B, H, Lq, d = q_host.shape
    for name, t in (("q_host", q_host), ("k_host", k_host), ("v_host", v_host)):
        if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CPU tensor [B, H, L, d]")
    _require(frames.dtype == torch.int32 and counts.dtype == torch.int32 and frames.is_cuda,
             "expected frames.dtype == torch.int32 and counts.dtype == torch.int32 and frames.is_cuda")
    if out_host is None:
        out_host = torch.empty(q_host.shape, dtype=torch.bfloat16).pin_memory()
    if lse_host is None:
        lse_host = torch.empty((B, H, Lq), dtype=torch.float32).pin_memory()
    _require(out_host.is_contiguous() and lse_host.is_contiguous() and not out_host.is_cuda,
             "expected contiguous host out_host and lse_host")
    desc = attn_desc(q_host, k_host, v_host, out_host, P, frames.shape[2], scale, timeout_us, on_host=True)
    if workspace is None:
        nbytes = ctypes.c_size_t(0)
        _check(load().sfa_forward_host_workspace(ctypes.byref(desc), ctypes.byref(nbytes)),
               "sfa_forward_host_workspace")
        workspace = torch.empty(nbytes.value, dtype=torch.uint8, device=frames.device)
    _check(load().sfa_forward_host(ctypes.byref(desc), q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr(),
                                   frames.data_ptr(), counts.data_ptr(), out_host.data_ptr(), lse_host.data_ptr(),
                                   n_chunks, workspace.data_ptr(), workspace.numel(), _ptr(dev_status),
                                   _stream(stream)), "sfa_forward_host")
    return out_host, lse_host
