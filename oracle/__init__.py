"""CPU oracle for the bit-plane quantized linear layer — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package. The product path (``bit_weight_quantization_b200``)
never imports, links or calls it, and shares no code with it.

It is a plain, slow, numpy implementation in float64 / int64 of what the layer
computes, written from the five source pages (cited by page and section):

  [RaBiT]   "RaBiT框架：突破2比特量化性能瓶颈的LLM部署方案" (jsqmd.com/news/742913)
  [HGF]     "1.58位LLM混合门控流优化技术解析" (jsqmd.com/news/748691)
  [ABQ]     "ABQ-LLM：用于大語言模型的任意比特量化推理加速" (hk.pswp.cn/pingmian/90308.shtml)
  [BVSR]    "BVSR：面向分布感知的大语言模型权重量化的比特向量求和表示" (ebiotrade.com, Neurocomputing summary)
  [BitNet]  "1-bit LLM的端侧推理革命" (bjdmk.com.cn/news/6115140)

Modules:
  bq_oracle  quantizers (pack), activation quantizers and reference layers
  layout     independent readers of the library's packed-weight and
             activation byte formats (decode bytes back to codes and scales)

Parity status per function is stated in each docstring ("pinned by ..." or
"parity unpinned").
"""
