"""CPU oracle for the NF4 + double-quantization + LoRA linear hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code,
table or constant generator with the CUDA library; both sides consume the same
seeded inputs from ``qlora_inputs`` (which holds none of the method's
arithmetic).

Sources (web pages, cited by title and section):
  [QLoRA-abs]  "QLoRA: efficient finetuning of quantized LLMs", Abstract.
  [Blog-mem]   "QLoRA: fine-tuning a 65B model on one GPU", section
               "Where the memory goes".
  [Blog-nf4]   same page, section "NormalFloat, double quantization, paged
               optimizers".
  [Cap-nf4]    "Qlora 4 Bit Quantization With Nf4 Fp4 Data Types And Lora
               Adapters", entry "4-bit quantization with nf4 data type for llm
               weight compression".
  [Cap-qlora]  same page, entry "qlora 4-bit quantization with nf4/fp4 data
               types and lora adapters".
  [LQ-abs]     "LQ-LoRA: Low-rank Plus Quantized Matrix Decomposition for
               Efficient Language Model Finetuning", abstract.

Module map:
  nf4.py     codebook, blockwise absmax, nearest-code encode, double
             quantization, packing, dequantization (fp32 step semantics).
  linear.py  fp64 LoRA linear forward / backward on the dequantized weight.
  layer.py   fp64 LLaMA-shaped decoder layer around seven such linears
             (torch CPU fp64 with autograd), for the decoder-layer tests.
  lq.py      low-rank plus quantized decomposition W ~ Q + L1 L2 ("LQ-LoRA",
             abstract): residuals, truncated and randomized SVD, the
             alternation.

Parity status: every function is pinned by ``tests/test_oracle_*.py`` except
the quantitative equal-usage property of the codebook levels,
which is reported only (parity unpinned for that claim; absmax normalisation
makes it approximate).
"""

from . import nf4, linear, lq  # noqa: F401
# layer.py imports torch; it is imported where used (from oracle import layer).
