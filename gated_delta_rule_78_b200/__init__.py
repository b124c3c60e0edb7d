"""Gated DeltaNet-2 chunkwise gated delta-rule recurrence on one B200 (sm_100a).

The product is ``libgdn2.so`` (C ABI, declared in ``include/gdn2.h``); this
package is its thin Python binding.  Functions carry the C names:

* ``gdn2_chunk_fwd(q, k, v, log_alpha, b, w, S0) -> (o, S_T)``
* ``gdn2_decode_step(q, k, v, log_alpha, b, w, S) -> o``   (S updated in place)
* ``gdn2_chunk_bwd(q, k, v, log_alpha, b, w, S0, d_o, dS_T) -> grads``
* ``gdn2_chunk_fwd_host``: the forward on host tensors, copies pipelined with the kernels
* ``gdn2_chunk_fwd_save`` / ``gdn2_chunk_bwd_saved``: the training pair, whose forward records the
  chunk-boundary states into the backward's workspace
* ``gdn2_chunk_bwd_noalloc(..., out=grads)``: the backward with the library's
  static scratch array, for callers that cannot allocate device memory
* ``gdn2_chunk_fwd_varlen`` / ``gdn2_chunk_bwd_varlen``: the same over N sequences
  packed along the token axis (``cu_seqlens`` int32 [N+1] on the device)
* ``gdn2_chunk_fwd_gated`` / ``gdn2_chunk_bwd_gated`` / ``gdn2_decode_step_gated``: gates given
  per channel, as per-(token, head) scalars, or absent (``flags``: DECAY_SCALAR, ERASE_SCALAR,
  WRITE_SCALAR, DECAY_NONE, ERASE_NONE, WRITE_NONE), and the input prologue (QK_L2NORM: raw q, k
  normalised in the call; BW_LOGITS: b, w given as logits)
* ``gdn2_prologue``: the input prologue alone (normalised q, k; sigmoid gates)
* ``gdn2_workspace_size``, ``gdn2_sync_status``, ``gdn2_strerror``

The library is loaded lazily by ``load()``; a missing library raises.
"""
from ._lib import (EXPORTS, GDN2_BF16, GDN2_F32, GDN2_OK, LIB_PATH, NOALLOC_MAX_SCRATCH_BYTES,  # noqa: F401
                   STATUS_NAMES, Gdn2Error, gdn2_chunk_bwd, gdn2_chunk_bwd_noalloc, gdn2_chunk_bwd_varlen,
                   gdn2_chunk_fwd, gdn2_chunk_fwd_varlen, gdn2_chunk_fwd_gated, gdn2_chunk_bwd_gated,
                   gdn2_decode_step_gated, gdn2_workspace_size_gated, DECAY_SCALAR, ERASE_SCALAR, WRITE_SCALAR,
                   DECAY_NONE, ERASE_NONE, WRITE_NONE, QK_L2NORM, BW_LOGITS, gdn2_decode_step, gdn2_prologue, gdn2_chunk_fwd_save, gdn2_chunk_bwd_saved, gdn2_chunk_fwd_host, gdn2_strerror, gdn2_sync_status, gdn2_selftest_timeout,
                   gdn2_workspace_size, load, raw)
