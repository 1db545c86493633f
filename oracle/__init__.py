"""fp64 CPU oracle for MLA decode over a paged latent KV cache.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.  The
product path (``mla_latent_kv_19_b200`` and its CUDA library) never imports,
links or calls anything here, and this package imports nothing from it.

It is a plain, slow and obviously correct restatement of what the method
computes, written from the pages:

* "DeepSeek V2的MLA注意力机制" (snabindia.com), section 2.1 (low-rank joint
  KV compression), section 2.2 (decoupled RoPE, ``apply_rope``/``mla_rope``),
  section 2.3 (cache only KV_comp and k_R; absorb W_UK into the query side and
  W_UV into the output side), section 3.1 (configuration table);
* the CSDN practical guide, section 2.1 (scaled dot-product attention) and the
  ``RotaryEmbedding`` listing in section 4 (rotate-half pairing);
* the hotdry.top DeepSeek-V3 page (MLA module sketch; FP8 KV cache).

Every function is pinned by ``tests/test_oracle_*.py`` against something other
than itself (closed forms, a library routine, brute force, invariants, figures
printed on the pages).  See the module docstrings for which pin covers what.
"""
from .mla import (  # noqa: F401
    softmax_scale,
    rope_inv_freq,
    rope,
    down_project,
    cache_row,
    paged_slot,
    append_tokens,
    fp8_quantize_row,
    absorb_q,
    decode_unabsorbed,
    decode_absorbed,
    split_partials,
    combine,
    up_project_out,
    out_project,
    step_outputs,
    step_outputs_unabsorbed,
    round_bf16,
    cache_bytes_per_token,
)
from .e4m3 import e4m3_encode, e4m3_decode, E4M3_MAX  # noqa: F401
