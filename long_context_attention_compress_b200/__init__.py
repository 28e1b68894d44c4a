"""Hybrid CSA/HCA attention (DeepSeek-V4) on B200: Python binding of libhca.so.

The entry points carry the C ABI's names (include/hca.h):
``csa_compress``, ``hca_compress``, ``csa_indexer_topk``, ``sparse_mqa_attend``,
``rms_norm_rope``, ``mxfp4_quantize``, ``csa_indexer_topk_fp4``, ``kv_fp8_quantize``,
``hybrid_attn_decode``, ``hybrid_attn_prefill`` (+ workspace queries).  They
are loaded lazily from ``_lib`` so that ``workloads`` (seeded inputs) imports
without the built library; the first use of an entry point raises ImportError
if libhca.so is missing -- there is no fallback implementation.
"""

_EXPORTS = {
    "csa_compress", "hca_compress", "csa_indexer_topk", "sparse_mqa_attend", "rms_norm_rope", "mxfp4_quantize",
    "csa_indexer_topk_fp4", "kv_fp8_quantize", "make_kv_fp8", "KvFp8", "hybrid_attn_decode",
    "hybrid_attn_prefill", "hybrid_attn_decode_workspace", "hybrid_attn_prefill_workspace", "workspace_size",
    "make_cfg", "make_decode_args", "make_prefill_args", "HcaError", "version", "last_error", "LayerCfg",
    "DecodeArgs", "PrefillArgs", "HCA_MODE_PREFILL", "HCA_MODE_DECODE", "HCA_OP_INDEXER_TOPK", "HCA_OP_SPARSE_MQA",
    "lib", "LIB_PATH",
}


def __getattr__(name):
    if name in _EXPORTS:
        from . import _lib
        return getattr(_lib, name)
    raise AttributeError(name)
