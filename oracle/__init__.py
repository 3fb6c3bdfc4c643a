"""CPU oracle for the QLoRA NF4 frozen-base linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It is a plain, slow,
fp64 NumPy restatement of what the source pages define, written so that a
reader can check each step against the pages by eye.  It shares no code,
table or constant generator with the CUDA library under
``bit_nf4_quantized_pack_b200/csrc``.

Sources (cited by page title and section):
  [P1] "QLoRA：冻结的 4-bit 权重怎样参与一次微调" (charlestar.github.io)
  [P2] "SFT（四）：QLoRA的4-bit量化与LoRA微调原理" (lsworl.github.io)
  [P3] "精读笔记 · QLoRA: Efficient Finetuning of Quantized LLMs"
       (llm-papers-study.pages.dev)

Parity status of each function is stated in its module header.
"""
from .nf4 import (  # noqa: F401
    NF4, BLOCKSIZE, DQ_BLOCKSIZE, NonFiniteError, PaddingError,
    encode_block, block_scales, quantize_nf4, pack_codes, unpack_codes,
    dq_codebook, exact_mean_f32, double_quantize, decode_scales,
    round_to_bf16, dequantize, bit_budget,
)
from .linear import lora_forward, lora_backward  # noqa: F401
from .int4 import int4_quantize_block, int4_dequantize_block  # noqa: F401
