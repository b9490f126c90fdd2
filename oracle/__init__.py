"""CPU oracle for multi-head latent attention (MLA): test infrastructure only.

This package is the plain, slow, fp64 statement of what the CUDA path computes.
Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import it; the product path (the C-ABI library and its Python
binding) never does, and shares no code with it.

Pinned against what the pages and the mathematics fix (see ``tests/test_oracle_pins.py``):
the absorb/naive identity, closed forms (one cached row, zero query, two keys),
library special cases (``scaled_dot_product_attention`` in fp64), brute-force
top-k masking, the page's parameter counts and cache-size formulas, the RMSNorm and
rotation invariants of the cache append, the FP8 codes and block scales of the FP8 latent
cache (``tests/test_oracle_fp8kv.py``), and planted mistakes that must be caught.  Every function here has at least one such pin.
"""

from .mla_oracle import (  # noqa: F401
    absorb_q,
    absorbed_decode,
    cache_append,
    e4m3_value,
    fp8_block_scale_shape,
    index_mask,
    latent_attention,
    latent_cache_dequant,
    mha_cache_bytes,
    mla_cache_bytes,
    multi_token_decode,
    naive_decode,
    naive_prefill,
    out_up,
    rms_norm,
    rope_interleaved,
    softmax,
    softmax_scale,
    split_wkv_b,
    value_up_params,
    weight_dequant,
)
