"""Kimi Delta Attention (KDA) on NVIDIA B200 (sm_100a).

The gated delta-rule recurrence with one forgetting factor per key channel,
S_t = (I - b_t k_t k_t^T) Diag(exp g_t) S_{t-1} + b_t k_t v_t^T, o_t = S_t^T q_t
("Kimi K3" open-weights field notes, ailearn.mscapital.top/kimi-k3.html,
panel "KDA 单头递归"), as a C-ABI CUDA library:

* ``kda_fwd``          chunkwise prefill (fixed-length or packed varlen batches,
                       initial and final states);
* ``kda_fwd_segmented`` the same prefill with the state pass split in time
                       (per-segment affine maps combined in prefix order);
* ``kda_fwd_overlapped`` the same prefill (fixed-length) as one launch in which
                       the state pass consumes each chunk record once published;
* ``kda_fwd_checkpointed`` prefill that also stores the state every n tokens
                       (prefix caching);
* ``kda_fwd_context_parallel``  prefill split in time over the ranks of a process
                       group (local map, one all-gather, prefix combine, local pass);
* ``kda_bwd``          the backward pass: gradients of a loss with respect to
                       q, k, v, g, beta and h0 (``kda_bwd_segmented``: the same
                       with the schedule chosen: whole chains, or segments of a
                       chain run at once from the tensor-core forward's states);
* ``kda_decode_step``  one token per sequence, state updated in place;
* ``kda_decode_verify`` / ``kda_decode_commit``  speculative decoding: run K
                       drafted tokens without touching the state, then advance
                       the state over the accepted prefix only.

This package is the thin Python binding; ``include/kda.h`` is the interface.
"""
from ._lib import (KDAError, bwd_plan_segments, bwd_segmented_workspace_size,  # noqa: F401
                   bwd_workspace_size,
                   checkpoint_count, cp_workspace_size,
                   device_error, gather_segment_maps, kda_cp_finish, kda_cp_local_map,
                   kda_fwd_context_parallel,
                   kda_bwd, kda_bwd_segmented, kda_decode_commit, kda_decode_step,
                   kda_decode_verify,
                   kda_fwd, kda_fwd_checkpointed, kda_fwd_inter, kda_fwd_intra,
                   kda_fwd_noalloc, kda_fwd_overlapped, kda_fwd_segmented, load_library,
                   plan_overlap, plan_segments, segmented_workspace_size, workspace_size)

__all__ = ["kda_fwd", "kda_bwd", "bwd_workspace_size", "kda_bwd_segmented",
           "bwd_segmented_workspace_size", "bwd_plan_segments", "kda_fwd_context_parallel",
           "kda_cp_local_map", "kda_cp_finish", "gather_segment_maps", "cp_workspace_size",
           "kda_fwd_intra", "kda_fwd_inter", "kda_fwd_noalloc", "kda_fwd_segmented",
           "kda_fwd_overlapped", "plan_overlap",
           "kda_fwd_checkpointed", "checkpoint_count", "kda_decode_step",
           "kda_decode_verify", "kda_decode_commit", "workspace_size",
           "segmented_workspace_size", "plan_segments", "device_error", "load_library",
           "KDAError"]
