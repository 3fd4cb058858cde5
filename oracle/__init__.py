"""Float64 CPU oracle for the TurboQuant hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py``
(its ``cpu_baseline`` and its reference arm, ``--impl reference``) may import
this package.  The product (the CUDA library and its
Python binding) never imports, links or calls anything here, and this package
imports nothing from the product.  The only code the two sides share is the
seeded input generator module ``synth``, which holds no quantizer arithmetic.

The oracle is plain numpy/scipy in float64: slow, unblocked, written step by
step in the order the pages describe the method, so that it can be read
against them.  Pages cited in this package:

* [ttakun]  "KV缓存52GB瞬间爆内存？TurboQuant随机旋转+标量量化如何把LLM长上下文推理成本
  砍到1/16且失真逼近理论极限" (ttakun.com/news/45354)
* [tmdm]    "谷歌悄悄扔下一颗“性能核弹”：KV缓存压缩6倍，推理提速8倍，还不用重训模型"
  (tmdm.cn/turboquant-kv-compression)
* [admirer] m.admirer.cn report on "TurboQuant: Online Vector Quantization with
  Near-optimal Distortion Rate" (arXiv 2504.19874)
* [tq.net]  turboquant.net/zh, "TurboQuant 最近的进展和外溢影响"

Parity status of each function is stated in its docstring ("pinned by ...").
"""
from .codebook import (coord_pdf, coord_cdf, bin_first_moment, lloyd_max, lloyd_max_quadrature,
                       distortion, b1_centroid)
from .turboquant import (haar_rotation, quantize_indices, nearest_centroid_bruteforce,
                         quant_mse, dequant_mse, quant_prod, prod_estimate, mse_estimate,
                         pack_codes, pack_codes_vec, unpack_codes, pack_signs, unpack_signs, code_words,
                         attention_decode, attention_prefill, attention_partial, merge_attention_partials, topk, channel_split,
                         near_threshold_mask)

__all__ = [
    "coord_pdf", "coord_cdf", "bin_first_moment", "lloyd_max", "lloyd_max_quadrature", "distortion",
    "b1_centroid", "haar_rotation", "quantize_indices", "nearest_centroid_bruteforce", "quant_mse",
    "dequant_mse", "quant_prod", "prod_estimate", "mse_estimate", "pack_codes", "pack_codes_vec", "unpack_codes",
    "pack_signs", "unpack_signs", "code_words", "attention_decode", "attention_prefill", "attention_partial",
    "merge_attention_partials", "topk", "channel_split",
    "near_threshold_mask",
]
