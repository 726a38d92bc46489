"""fp64 CPU oracle for the MoE + multi-LoRA hot path.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.  The
product path (``moe_lora_b200``) never imports, calls or links anything here, and
this package imports nothing from the product path: the two share no code.

Sources (web pages; cited by page and section):
  [vLLM MoE-LoRA page]  "vllm-moe-lora-sagemaker-bedrock" (wp.cloudtroop.com.br),
                        sections "Entendendo os Modelos MoE", "O Papel da Multi-LoRA",
                        "Implementação Técnica no vLLM", "Otimizações em Nível de Kernel".
  [SageMaker MoE kernels page] "aws-sagemaker-moe-kernel-optimizations" (aib.vote),
                        first (operand swap, topk=8) and second (FP8 per-tensor MoE) items.
  [Punica review page]  "Punica: Multi-Tenant LoRA Serving" review (nubint.ai),
                        sections "ひとこと要約", "提案手法", "主な発見".

Modules:
  formats      stored-precision decoding (bf16 bit patterns, OCP e4m3) to fp64.
  moe_lora_ref vectorised reference: router logits, top-k + renormalised softmax,
               (expert, adapter) stable sort, LoRA expert FFN, weighted combine, SGMV.
  brute        pure-Python loops over tokens/features for tiny inputs; shares no
               helper with moe_lora_ref (its own decoding, its own sort).

Pins (tests/test_oracle_*.py, ``-m "not gpu"``): brute force on tiny inputs,
hand-derived golden cases (tests/golden/), library routines (torch casts, softmax),
closed forms and invariants (zero adapters, merged weights, linearity, top-k = E,
permutation invariance of SGMV).  Every public function here is checked by at least one
of them (helpers through the functions that call them).  The pages print no worked
numeric example, so no pin is a value printed by the pages; the golden cases are closed
forms derived by hand from the definitions.
"""
