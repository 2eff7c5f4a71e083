"""fp64 CPU oracle for the causal sliding-window GQA attention block.

TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only the tests, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this package. The CUDA library never calls it and shares no code with it.

Every function is the plain definition of one step of the attention block, as
the nanochat and nanoGPT guides describe it, written out in float64 with numpy:
no tiling, no online softmax, no fused passes. See ``attention.py``.
"""
from .attention import (  # noqa: F401
    rms_norm,
    rope_frequencies,
    rope_angles,
    rope,
    rope_transpose,
    row_positions,
    prologue,
    prologue_bwd,
    round_bf16,
    round_e4m3,
    quantize_e4m3_tensorwise,
    E4M3_MAX,
    visible,
    attention_fwd,
    attention_bwd,
    attention_bwd_rows,
    attention_bwd_keys,
    decode,
    prefill,
    layer_windows,
    kv_replicate,
    useful_pairs,
)
