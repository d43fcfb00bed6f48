"""Momentum DeltaNet (MDN) forward pass and decode step on B200 (sm_100a).

The compute lives in ``lib/libmdn.so`` (hand-written CUDA behind the C ABI of
``include/mdn.h``); this package only marshals torch tensors into it.  The
library is loaded on first use and there is no CPU fallback.
"""
from .api import (MDNError, chunk_bwd, chunk_fwd, chunk_fwd_preact, chunk_fwd_status,  # noqa: F401
                  chunk_fwd_varlen,
                  chunk_fwd_workspace_size,
                  chunk_gate_prep,
                  step, step_with_delta_norm, gate_params, status_string, library,
                  profile_enable, profile_read)
