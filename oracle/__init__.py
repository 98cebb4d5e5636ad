"""Oracle: a plain, slow, obviously-correct CPU statement of what the hot path computes.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import, call or run
anything in this package. Only the test-suite, the smoke check in
``__graft_entry__.smoke`` and the CPU-baseline leg of ``bench.py`` use it. It shares
no code, header, table or helper with the CUDA library under
``group_wise_int4_b200``; the two meet only through the seeded inputs of ``synth``.

Sources (the web pages on FlexGen's group-wise int4 method):

* the walkthrough page «FlexGen 单 GPU 高吞吐大模型推理引擎：论文解读与源码实战指南», section 6.3 "4-bit group-wise quantisation of weights
  and KV cache": the compression configuration (num_bits 4, group_size 64,
  group_dim 0 for weights and 2 for the cache, asymmetric), the packed data shape
  ``shape[:group_dim] + (num_groups * (group_size // 2),) + shape[group_dim+1:]``
  with two 4-bit codes per uint8, and a per-group fp16 scale tensor.
* the source-notes page «FlexGen» (PtirisNote), "Pytorch Backend" and "Flex Opt": prefill attention
  is ``mha``, the decode step is ``mha_gen``; the generation loop runs load_cache,
  compute_layer and then store_cache, so a decode step attends to the cache of the
  earlier tokens plus its own fresh key and value, and its own key/value are
  quantised into the cache after the layer has run.

Modules:

* ``oracle.codec`` - group-wise min/max quantiser and dequantiser, IEEE fp32 (the
  precision in which the integer codes are decided on both sides).
* ``oracle.layer`` - the OPT decoder layer (pre-LayerNorm, fused QKV, causal softmax
  attention, output projection, ReLU FFN, residuals) in fp64 on dequantised weights.
* ``oracle.cpp`` - access to ``oracle/cpp/flexq_oracle.cpp``, a second, plain C++17
  statement of the quantiser and of the layer in IEEE fp32 (every operation rounded on
  its own, no fused multiply-add), written independently of the numpy modules. It is
  the program the benchmark times as the CPU baseline; its pins cross-check it against
  the numpy oracle and against closed forms.

Every function is pinned by the tests under ``tests/test_oracle_*.py`` against
closed forms, hand-worked examples, invariants and brute force; none is
"parity unpinned".
"""
from . import codec, layer  # noqa: F401   (oracle.cpp is imported on demand: it compiles C++)
