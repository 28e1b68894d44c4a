"""CPU oracle for the hybrid CSA/HCA attention layer.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, float64 NumPy
restatement of what the layer computes, written from the DeepSeek-V4 write-ups
(see the docstrings of ``oracle.hca`` for the passage each function follows).

Who may use it: ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
``cpu_baseline`` / ``--impl reference`` legs.  The product library
(``long_context_attention_compress_b200``) never imports, calls or links
anything here, and this package imports nothing from the product: the two
share no code.  Inputs come from the seeded generators in
``long_context_attention_compress_b200.workloads`` (which hold none of the
method's arithmetic) and are handed to both sides as arrays.
"""

from .hca import (  # noqa: F401
    round_bf16,
    softmax,
    csa_compress,
    hca_compress,
    compress_weights_csa,
    compress_weights_hca,
    n_visible,
    indexer_scores,
    topk_select,
    window_rows,
    mqa_attend,
    mqa_partial,
    combine_partials,
    csa_layer_prefill,
    hca_layer_prefill,
    csa_layer_decode,
    hca_layer_decode,
    QKNorm,
    rms_norm,
    rope_theta,
    rope,
    entry_position,
    norm_rope_rows,
    attend_norm_rope,
    cache_entries,
    E2M1_GRID,
    MX_BLOCK,
    e2m1_value,
    mxfp4_quantize,
    mxfp4_dequantize,
    mxfp4_pack,
    mxfp4_unpack,
    indexer_scores_fp4,
    topk_recall,
    classical_block_tokens,
    paged_rows,
    ring_window,
    csa_layer_decode_paged,
    hca_attend_decode_paged,
    round_e4m3,
    fp8_kv_quantize,
    fp8_kv_dequantize,
)
