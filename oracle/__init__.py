"""Plain, slow CPU oracle for absorbed MLA decode (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (``mla_latent_kv_35_b200``) never imports it, and this package
imports nothing from the product path.
"""

from .mla_oracle import (  # noqa: F401
    rope,
    project,
    attention_nonabsorbed,
    attention_absorbed,
    absorb_query,
    latent_attention,
    latent_attention_range,
    out_proj,
    decode_step,
    cache_append,
    combine_splits,
    dense_cache_bytes,
    mla_cache_bytes,
    cache_elems_per_token,
    gqa_equivalent_groups,
    quantize_latent_fp8,
    dequantize_fp8,
)
