"""Float64 CPU oracle for the packed low-bit KV cache and decode attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package: only
the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may use it.  It shares no code, table or constant generator
with the CUDA library; the only module both sides use is ``synth`` (seeded inputs,
which holds none of the method's arithmetic).

Every function is a plain, slow restatement of what the pages define, in numpy:
float64 wherever the pages leave the precision open, and explicit fp32 / fp16 steps
exactly where the quantizer's definition fixes them (see ``oracle.fp``).

Sources (web pages, cited by title and section):
  [AXES]  "KV quantization axes: why Key and Value need separate reasoning"
  [KVQ]   "KVQuant: Towards 10 Million Context Length LLM Inference with KV Cache
          Quantization"
  [MIX]   "MixKVQ: Query-Aware Mixed-Precision KV Cache Quantization for
          Long-Context Reasoning"
  [K4V2]  "Quantize What Counts: More for Keys, Less for Values"
  [TQ]    "Statistical Inference and Quality Measures of KV Cache Quantisations
          Inspired by TurboQuant"

Parity status of each module is stated in its docstring.  Parts with no pin to
anything outside the oracle are marked "parity unpinned".
"""
