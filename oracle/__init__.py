"""CPU oracle for the bit-plane quantized linear layer — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package. The product path (``bit_weight_quantization_b200``)
never imports, links or calls it, and shares no code with it.

It holds two plain, slow implementations in float64 / int64 of what the layer
computes, written independently from the five source pages (cited by page and
section): the C++ reference (``bq_ref.cpp``: plain loops, OpenMP over rows, built
by ``build_ref`` into ``libbqref.so`` and called through ``cref``), which the GPU
parity tests, the smoke check and the bench's CPU legs use, and the numpy one
(``bq_oracle``). Both are held to the same pins, and to each other bit for bit.

  [RaBiT]   "RaBiT框架：突破2比特量化性能瓶颈的LLM部署方案" (jsqmd.com/news/742913)
  [HGF]     "1.58位LLM混合门控流优化技术解析" (jsqmd.com/news/748691)
  [ABQ]     "ABQ-LLM：用于大語言模型的任意比特量化推理加速" (hk.pswp.cn/pingmian/90308.shtml)
  [BVSR]    "BVSR：面向分布感知的大语言模型权重量化的比特向量求和表示" (ebiotrade.com, Neurocomputing summary)
  [BitNet]  "1-bit LLM的端侧推理革命" (bjdmk.com.cn/news/6115140)

Modules:
  bq_ref.cpp the C++ reference: quantizers, activation quantizers, reference layers
  build_ref  builds it with g++ -O2 -fopenmp -ffp-contract=off
  cref       the C++ reference behind the same Python API as bq_oracle
  bq_oracle  the numpy implementation of the same
  layout     independent readers of the library's packed-weight and
             activation byte formats (decode bytes back to codes and scales)

Parity status per function is stated in each docstring ("pinned by ..." or
"parity unpinned").
"""
