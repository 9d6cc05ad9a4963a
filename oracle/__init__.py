"""CPU oracle for compressed decode attention — TEST INFRASTRUCTURE ONLY.

A plain, slow, float64 restatement of what the method computes, written from
the source pages and kept independent of the CUDA library (no shared code,
headers, tables or helpers). Only the test suite, the smoke check of
``__graft_entry__`` and the CPU-baseline legs of ``bench.py`` may import it;
the library's product path never does.

Sources, cited in each function by key and section:
  [TQAI]   "We Built a Python Library That Cuts LLM Memory Usage by 80%" (dev.to)
  [ADAPTQ] "AdapTQ — Adaptive Streaming Vector Quantization KV Cache for LLMs"
           (PyPI adaptq 0.2.3)
  [TQPLUS] "TurboQuant+: Compresión de Caché KV 6.4x para LLMs" (aibit.im)

Pinning (tests/test_oracle_*.py): every function here is checked against
values the pages print, closed forms, textbook tables or brute force, except
the sign-vector generator, whose bits are a definition of this library (the
pages name no generator); it is pinned to SplitMix64's published reference
output, not to the pages.

Modules:
  codebook   Lloyd-Max quantizer for N(0,1)
  rotation   SplitMix64 sign vector, Sylvester Hadamard matrix, rotation
  codec      norm / rotate / index / pack, unpack / dequantize
  attention  compressed-domain decode attention with the sparse-V gate, the
             per-slice log-sum-exp records of a split context and their
             combine
  qjl        stage-2 residual sketch of the keys and the unbiased score
             estimate
"""
from . import codebook, rotation, codec, attention, qjl  # noqa: F401
