"""CPU oracle for the Ideogram 4 DiT block (TEST INFRASTRUCTURE ONLY).

A plain, slow, float64 numpy statement of what one Ideogram4TransformerBlock
forward and the 34-block stack compute (``ig4_oracle``), and of one sampler
step with asymmetric classifier-free guidance and its schedule
(``ig4_sampler``).  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may import it; the
product path (``stream_diffusion_transformer_fwd_b200``) never does, and this
package imports nothing from the product.  It shares no code, table or
constant generator with the CUDA library; the two meet only in the seeded
inputs of ``synth/``.

Parity status: every function is pinned by ``tests/test_oracle_*.py``
(closed forms, invariants, brute force on tiny inputs, the E4M3 decoder
against an independent library conversion).  No function is unpinned.
"""

from .ig4_oracle import (  # noqa: F401
    ADALN_CHUNKS,
    BLOCK_WEIGHT_NAMES,
    EPS,
    MROPE_SECTION,
    ROPE_THETA,
    ROTARY_DIM,
    adaln_modulation,
    apply_mrope,
    block_flops,
    block_forward,
    block_forward_rows,
    bf16_round,
    dequant_e4m3,
    dequant_nvfp4,
    e2m1_decode_table,
    e4m3_decode_table,
    e2m1_encode,
    e4m3_encode,
    final_layer,
    joint_attention,
    merge_heads,
    modulate,
    nvfp4_activation_values,
    quantize_nvfp4_activations,
    quantize_mx8_activations,
    mx8_values,
    MX8_BLOCK,
    mrope_angles,
    mrope_axis_of_pair,
    mrope_positions,
    rms_norm,
    rope_inv_freq,
    silu,
    softmax,
    split_heads,
    stack_forward,
    stack_input,
    swiglu,
    text_cond_projection,
    TEXT_RAW_LAYERS,
    TEXT_RAW_WIDTH,
)
