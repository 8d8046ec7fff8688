"""Plain, slow, fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (the CUDA library and its Python binding) never
imports it and shares no code with it.

Sources are cited by page title and section:

* [Librarian]  "FlashAttention v1/v2/v3/v4: the librarian who never clears the
  desk -- IO-awareness, async and Blackwell's asymmetry" (blog.lo0.es).
* [Concept]    "FlashAttention" concept note (research-hub), sections
  "Definition" and "How it works".
* [Lineage]    "The FlashAttention lineage -- FA1 / FA2 / FA3 / FA4"
  (project-fortress), sections "FA1 (2022)" ... "FA4 (2026)".

Modules:

* ``attention_ref``  -- forward (O, L), backward (dQ, dK, dV), the online
  softmax recurrence, and grouped K/V heads (GQA / MQA).  Every function is pinned by ``tests/test_oracle_*.py``.
* ``fp8_ref``        -- Sylvester Hadamard rotation, per-128-row block scale,
  a table-driven E4M3 (OCP e4m3fn) encoder/decoder.  Pinned likewise.
"""
from .attention_ref import (  # noqa: F401
    attn_fwd_ref,
    attn_fwd_rows_ref,
    attn_bwd_ref,
    attn_fwd_gqa_ref,
    attn_bwd_gqa_ref,
    online_softmax_ref,
    attn_fwd_online_ref,
    softmax_ref,
)
from .fp8_ref import (  # noqa: F401
    E4M3_MAX,
    e4m3_decode_table,
    e4m3_encode_ref,
    e4m3_decode_ref,
    hadamard_ref,
    rotation_ref,
    quant_fp8_ref,
    dequant_fp8_ref,
    quant_fp8_per_tensor_ref,
    quant_fp8_per_tensor_codes_ref,
    MIN_SCALE,
)
