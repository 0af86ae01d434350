"""CPU oracle for the quantized-KV decode path.

TEST INFRASTRUCTURE ONLY. This package is the slow, obviously-correct reference
that the CUDA library is checked against. Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it. The product path (the ``rq_*`` C-ABI
library and its Python binding) never imports, links or calls anything here,
and this package never imports the product.

Modules
-------
allocation  RateQuant per-head bit allocation: continuous reverse waterfilling
            on D(b) = alpha * beta**-b and integer allocation onto an allowed
            bit set (exact DP, the greedy max-heap of the paper, brute force).
quantize    InnerQ-style group-wise asymmetric quantizer (fp32 rule, fp16
            scale, bf16 zero) and the packed tile-record byte format.
cache       Cache assembly (sink / quantized tiles / recent ring) and the
            append-with-flush rule.
attention   fp64 decode attention over the dequantized cache (GQA).

Every floating-point step of the quantizer is written with numpy float32 /
float16 scalars so that its rounding is IEEE round-to-nearest-even, one
operation at a time, with no fused multiply-add.
"""
