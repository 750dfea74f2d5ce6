"""fp64 CPU oracle for absorbed-MLA decode.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import anything from this package.
It shares no code with the CUDA library: it reads the same seeded inputs (bf16 bit
patterns from ``mla_synth``) and computes, slowly and plainly, what the decode path
is defined to compute.

Sources (page title, section, equation):

* "Multi-head Latent Attention" glossary entry (llm-glossary.tokens-kit.com), the
  teaching abstraction: latent ``c_t = x_t W^DKV``, per-head up-projections
  ``k^C = c W^UK``, ``v^C = c W^UV``, decoupled rope key ``k^R`` shared by all heads,
  and the two-part score ``s = q^C k^C^T + q^R k^R^T``;
  section "why absorb in decode": ``q^C (W^UK)^T c^T`` (key absorption) and
  ``sum_t p_t (c_t W^UV) = (sum_t p_t c_t) W^UV`` (value absorption);
  the runnable expanded-vs-absorbed check: softmax scale ``1/sqrt(d_k + d_r)``,
  fp64, both forms equal to 1e-10;
  section "capacity and cost": ``M_MLA ~ L B T (d_c + d_rope) s`` cache bytes, and the
  note that the latent cache can still be paged into blocks and that online softmax
  applies to the merged score.
* FlashMLA issue #16 "up matrix is not involved?": q absorb and o absorb sit outside
  the attention kernel; q goes from [bs, H, 128] to [bs, H, 512] concatenated with
  q_rope [bs, H, 64]; the kernel output is [bs, H, 512].

Parity pins (what fixes this oracle independently of itself) live in
``tests/test_oracle.py``.  No function here is "parity unpinned".
"""
from .mla_oracle import (  # noqa: F401
    bf16_to_f64,
    gather_rows,
    mla_decode_ref,
    mla_decode_multi_ref,
    mla_decode_probs_ref,
    mla_decode_expanded_ref,
    mla_absorb_q_ref,
    mla_absorb_o_ref,
    mla_layer_absorbed_ref,
    lse_merge_ref,
    cache_elements_per_token,
    latent_cache_bytes,
)
from .fp8_cache import e4m3_to_f64, dequant_rows, mla_decode_fp8_ref  # noqa: F401
