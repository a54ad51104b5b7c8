"""CPU oracle for the group-wise 4-bit OPT decode path.  TEST INFRASTRUCTURE.

A plain, slow restatement of what the hot path computes, written from the
FlexGen pages and nothing else:

* ``q64``  - FlexGen's group-wise asymmetric 4-bit format (groups of 64
  contiguous elements, fp16 min and scale per group), "FlexGen研究学术报告",
  section 三(C) "近似方法的应用" (group-wise quantization).  The quantizer
  decides integer codes, so it works in fp32 with round-to-nearest-even and
  no fused multiply-add, the precision the CUDA kernels decide them in.
* ``opt``  - the OPT-style decoder layer (prefill and decode), the KV cache
  update, the tied LM head and greedy generation, from the equations of
  "FlexGen: High-Throughput Generative Inference ..." (qingweiji.github.io),
  section "P/D阶段计算", and the multi-head form of eqs. (1)-(3) of the survey
  notes (gumorming.cn, "Transformer-Styles LLMs").  The layer math is float64.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  It shares no code with the CUDA library and
imports nothing from it; the only module both sides use is ``synth`` (seeded
input generation, no method arithmetic).
"""
from . import q64, opt  # noqa: F401
