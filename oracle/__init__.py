"""CPU oracle for the MXFP4 MoE decode layer -- TEST INFRASTRUCTURE ONLY.

Plain, slow, float64 code that states what the layer computes, twice: numpy
(``formats.py``, ``moe.py``, ``lmhead.py``) and plain C++17 with OpenMP over
matrix rows (``moe_oracle.cpp``, loaded through ``cpp.py``; bit-equal to the
numpy layer on seeded inputs, and the one timed as the CPU baseline).  Only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import it; the product path (the CUDA library and its Python binding)
never does, and this package imports nothing from the product.

Sources cited in this package:

* [tanhow] "NVIDIA 在单台 DGX Spark 上叠加三项优化，Ling-3.0-flash 的 MoE 推理
  吞吐提升 42.5%" (tanhow.com), a retelling of NVIDIA's "3 Ways to Boost MoE
  Inference on NVIDIA DGX Spark".  Sections used: "为什么 DGX Spark 上的 MoE
  解码是内存受限的？" (decode is weight-read bound; the W4A8 recipe),
  "三项优化是什么？" item 1 (expert width 768), item 2 (LM head
  157,184 x 2,560, hence hidden 2560), item 3 (4 verified tokens touch up to
  32 experts), "Ling 3.0 是什么" sparse-MoE bullet (8 of 512 routed experts
  plus 1 shared expert per MoE layer).
* [devotd] the devotd.net retelling of the same post, section
  "2. 同时应用内核替换和 FP8 输出层" (MXFP4 is a blocked 4-bit float format;
  baseline recipe is 4-bit weights with 8-bit activations).
* [aivibenews] "Три приёма ускорить MoE-инференс на DGX Spark без потери
  GSM8K", opening paragraph (routing to eight of 512 experts).
* [OCP-MX] OCP Microscaling Formats (MX) Specification v1.0: the MXFP4
  block (32 FP4 E2M1 elements sharing one E8M0 scale), the E2M1 element
  encoding and the E8M0 scale encoding.
* [OCP-FP8] OCP 8-bit Floating Point Specification (OFP8): the E4M3
  encoding (bias 7, no infinities, S.1111.111 is NaN, largest finite 448).

The pages state the routing shape and the precision recipe but not the
routing function, the FFN form, the block size or the activation scale
granularity; those follow the layer's problem statement (softmax over fp32
router logits, top-8, renormalised; SwiGLU experts; 32-element blocks along
K; one FP8 scale per token, amax/448).  Where the text is silent the plain
reading is taken and named at the function that takes it.

Parity status of each function is listed in ``oracle/moe.py``'s header.
"""
