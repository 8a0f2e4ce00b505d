"""CPU oracle for the grouped NF4 expert block with per-expert LoRA.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, obviously correct
restatement of what the method computes, in float64 numpy (the only float32
steps are the ones that decide bits: the NF4 dequantisation product and its
bfloat16 rounding).  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
It shares no code, table or constant with the CUDA library and must never be
imported by the library or its Python binding.

Sources (page title, section):

* "How do I QLoRA-train the fused experts of a MoE (per-expert LoRA on 4-bit
  experts)?" -- §"The abstraction that fails, and what replaces it" (fused
  3-D stacks ``gate_up_proj [E,2I,H]``, ``down_proj [E,H,I]``; each routed
  expert adds its delta inside its activation; B starts at zero; the base is
  frozen), §"Why it happens" (the LoRA term is
  ``scaling * (x @ A[e].T) @ B[e].T``; the backward decodes the 4-bit base
  again; the method's plain forward visits the experts one at a time),
  §"Limitations" (the stock epilogue ``act(gate) * up``).
* experts4bit-qlora package METADATA -- §"The package family" (the experts
  are stored as packed 4-bit stacks, decoded in registers, with fp32 sums).
* The NF4 code book itself is not printed on those pages; it is the
  NormalFloat-4 data type of Dettmers et al., "QLoRA: Efficient Finetuning of
  Quantized LLMs" (2023), whose construction ``nf4_table`` restates.

Parity status of each function is listed in ``oracle/moe.py`` and
``oracle/nf4.py`` headers; every function here is pinned by a test under
``tests/test_oracle_*.py``.
"""

from .nf4 import (  # noqa: F401
    nf4_table,
    bf16_round_bits,
    bf16_bits_to_f32,
    dequantize_nf4,
    dequantize_nf4_matrix,
    quantize_nf4,
)
from .moe import (  # noqa: F401
    Experts,
    expert_forward,
    expert_backward,
    route_topk,
    group_by_expert,
    moe_forward,
    moe_backward,
    router_backward,
    topk_softmax_backward,
    expert_weights,
)
