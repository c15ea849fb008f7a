"""Float64 CPU oracle of the Llama-style decode step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product path (``bandwidth_bound_b200``) never imports it and has no CPU
fallback; the two share no code beyond the seeded input generators in
``synth``.
"""
from .decode import (  # noqa: F401
    bf16_rne,
    to_f64,
    rmsnorm,
    rope_inv_freq,
    rope,
    kv_head_of,
    attention,
    attention_partial,
    combine_partials,
    silu,
    decode_step,
    decode_layer,
    layer_weights_f64,
    lm_head,
    model_bytes,
    argmax_lowest,
)
from .sampling import boundary_margin, sample_top_k, top_k_ranked  # noqa: F401,E402
