"""B200-native Kimi Delta Attention (KDA): C-ABI CUDA library + thin Python binding.

    kda_chunk_fwd(q, k, v, g, beta, scale, initial_state) -> (o, final_state)
    kda_recurrent_step(q, k, v, g, beta, state, scale) -> o   (state updated in place)
    kda_backward(q, k, v, g, beta, grad_o, scale, initial_state, grad_final_state) -> gradients

The compiled library (libkda.so, built by ``build.build()``) does all the
work; the binding only marshals arguments.  It is loaded on first use.
"""
from .binding import (KDAError, kda_backward, kda_chunk_fwd, kda_chunk_fwd_check, kda_chunk_fwd_launch_count,
                      kda_chunk_fwd_workspace_size, kda_recurrent_step, load, status_string, version)

__all__ = ["KDAError", "kda_backward", "kda_chunk_fwd", "kda_chunk_fwd_check", "kda_chunk_fwd_launch_count",
           "kda_chunk_fwd_workspace_size", "kda_recurrent_step", "load", "status_string", "version"]
