"""Frame-sparse attention for video diffusion transformers on B200 (sm_100a).

Python face of libsfa.so (C ABI in include/sfa.h):

* ``build_sets``  - attended frame sets A(h, t) (LVSA anchors + window, sink/local/memory
                    caches, explicit lists), built on the GPU
* ``forward``     - softmax attention over the tokens of A(h, t) only, O bf16 + LSE fp32
* ``forward_host`` - the same for pinned host tensors (sfa_forward_host: the copies and the
                    attention pipelined inside the library)
* ``forward_split`` - the same with each unit's key tiles split over several CTAs and the
                    partials merged by LSE (short or uneven grids); ``n_split=0`` lets the
                    library choose the split and run the CTAs longest first
* ``forward_paged`` - the same with K/V read through a per-head frame -> slot table
* ``forward_dual`` - local and history branches in one launch: the local result and their
                    LSE merge (the full attention)
* ``lse_merge``   - merge of two partial attentions (local + history branch) by LSE
* ``hsa_select``  - hierarchical selection (Light Forcing HSA): pooled keys, top history
                    frames, then top 128-token key blocks, per 256-row query block
* ``forward_blocks`` - attention of every query block over its key-block list
* ``gdn_forward`` - ARL2's inter-frame branch: gated delta rule over frames (fp32 state)

Tensors are PyTorch CUDA tensors; calls run on the current CUDA stream.
"""
from ._lib import (SET_KINDS, SFA_DEBUG_STALL_GDN_STATE, SFA_DEBUG_STALL_SOFTMAX, SFA_ERR_BAD_SET, SFA_ERR_CUDA,
                   SFA_ERR_INVALID_ARG, SFA_ERR_TIMEOUT, SFA_ERR_UNSUPPORTED, SFA_OK, AttnDesc,
                   SetParams, SfaError, attn_desc, build_sets, error_string, forward, forward_blocks, forward_dual,
                   forward_host, host_workspace_bytes,
                   forward_paged, forward_split, gdn_forward, GdnDesc, hsa_max_count, hsa_pool_keys, hsa_select, hsa_select_pooled,
                   hsa_workspace_bytes, load, lse_merge,
                   set_max_count,
                   set_params, split_plan, split_workspace_bytes, version)

__all__ = ["SET_KINDS", "SFA_DEBUG_STALL_GDN_STATE", "SFA_DEBUG_STALL_SOFTMAX", "SFA_ERR_BAD_SET", "SFA_ERR_CUDA",
           "SFA_ERR_INVALID_ARG", "SFA_ERR_TIMEOUT", "SFA_ERR_UNSUPPORTED", "SFA_OK", "AttnDesc",
           "SetParams", "SfaError", "attn_desc", "build_sets", "error_string", "forward", "forward_blocks",
           "forward_dual", "forward_host", "host_workspace_bytes",
           "forward_paged", "forward_split", "gdn_forward", "GdnDesc", "hsa_max_count", "hsa_pool_keys", "hsa_select",
           "hsa_select_pooled", "hsa_workspace_bytes",
           "load", "lse_merge", "set_max_count", "set_params", "split_plan", "split_workspace_bytes", "version"]
