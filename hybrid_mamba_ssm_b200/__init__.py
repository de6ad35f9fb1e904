"""B200-native Mamba-2 selective state-space scan.

Two entry points, both hand-written CUDA for sm_100a behind the C ABI declared
in ``include/ssm.h`` (library ``libssm.so``):

* ``ssd_chunk_scan``   -- chunked SSD prefill over packed sequences, returning
  y and the final fp32 state;
* ``ssm_state_update`` -- single-token decode update, in place on an fp32
  ``[batch, heads, head_dim, d_state]`` state;

and around them: slot-pool variants of both (fp32 or fp16 pools with
stochastic rounding, raw dt with bias/softplus/clamp), speculative
multi-token decode (``ssm_state_update_multi``, ``ssm_state_commit``), the
causal conv1d that feeds the scan (``causal_conv1d_fwd``,
``causal_conv1d_update``, ``causal_conv1d_update_multi``) and the gated group
RMSNorm after it (``ssm_gated_rmsnorm``).

The Python binding (``hybrid_mamba_ssm_b200.ssm``) only marshals torch tensors
into that ABI; importing it loads the CUDA library and raises if it is missing.
``hybrid_mamba_ssm_b200.inputs`` (seeded synthetic inputs) needs neither torch
nor the library.
"""

__all__ = ["ssd_chunk_scan", "ssm_state_update", "ssd_chunk_scan_workspace_size",
           "ssd_chunk_scan_slots", "ssm_state_update_slots", "ssm_state_update_multi",
           "ssm_state_commit", "causal_conv1d_fwd", "causal_conv1d_update",
           "causal_conv1d_update_multi", "ssm_gated_rmsnorm", "SSMError"]


def __getattr__(name):
    if name in __all__:
        from . import ssm
        return getattr(ssm, name)
    raise AttributeError(name)
