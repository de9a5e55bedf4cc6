"""CPU oracle for quantized paged-KV attention (Q8_0 or Q4_0 keys, Q4_0 or Q8_0 values).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import anything
from this package.  The product path (the CUDA library and its Python binding)
never imports it and never falls back to it.

What it computes, plainly and slowly, in float64 unless a format fixes another
precision:

* ``quant``     Q8_0 / Q4_0 block quantisation and dequantisation (fp32 decisions,
                fp16 scales), the KV-cache formats named on the pages;
* ``layout``    the byte layout of one 128-token K or V page (a storage spec that
                this library defines; the pages fix only bits per element);
* ``attention`` masked softmax attention with log-sum-exp, and the log-sum-exp
                merge of partial results;
* ``select``    per-block mean keys, block scores and top-k block selection.

Sources (page title, section):

* Vulkan speculative-decoding report, 7900 XTX (lcz.me/topic/1398), section
  "model structure": 16 full-attention layers x 4 KV heads x 256 = 16,384 K (or V)
  elements per token; section "pitfalls" (KV quantisation): q4_0 K+V costs
  18 KiB per token (18 bytes per 32 elements), q8_0 is 8.5 bits per element, and
  the KV cache accepts only the legacy block formats.
* KVMem reproduction on one 7900 XTX (lcz.me/topic/1972), test command and
  recall sections: 128-token KV blocks, a 32,768-token GPU budget plus a
  16,384-token generation reserve, retrieval by a query.
* Adaptive KV Streaming + RDNA 4 announcement (wqu.guru), method list: paged decode
  attention extended to verify batches; chunked prefill across streamed pages
  merged by online log-sum-exp; layer L+1 transfers overlapped with layer L.

Parity pins: every function is pinned by tests under ``tests/test_oracle_*.py``
against closed forms, brute force on tiny inputs, invariants and the sizes the
pages print.  The pages print no worked numeric example of the attention itself,
so its values are pinned by definition (brute force) and invariants only.
"""
from . import attention, layout, quant, select  # noqa: F401
