"""fp64 CPU oracle for the nanochat GPT block stack — TEST INFRASTRUCTURE ONLY.

This package is the slow, obviously-correct definition that the CUDA library is
checked against.  Only the tests, the smoke check and the benchmark's CPU
baseline leg may import it; the library itself never does and has no CPU
fallback.  It shares no code with the CUDA path.

Everything is computed in float64 with numpy; library matmuls serve as steps,
with no blocking, fusion or reordering beyond the definitions.

Sources (page title and section; the pages print no equations, only short
Python snippets and a feature list, so the block is assembled from these):

  [AP-feat]  apidog.com/fr "Comment Entraîner Votre Propre ChatGPT Pour 50€ ?",
             § "Comment nanochat fonctionne" › 1. Le modèle GPT › feature list
             (RoPE, QK normalisation, untied weights, ReLU², GQA, sliding
             window, FlashAttention call).
  [AP-ve]    same page, § 1 › "Embeddings de valeur (ResFormer)" snippet.
  [AP-mix]   same page, § 1 › "Astuces d'efficacité" snippet 1 (per-layer
             residual lambdas).
  [AP-smear] same page, § 1 › "Astuces d'efficacité" snippet 2 (smear).
  [AP-back]  same page, § 1 › "Astuces d'efficacité" snippet 3 (backout).
  [AP-lin]   same page, § 3 "Gestion de la précision" (Linear casts the weight
             to the activation dtype; FP8 with per-tensor scaling).
  [AP-fa]    same page, § 5 "Unification de Flash Attention"
             (flash_attn_func(q, k, v, causal=True, window_size=...)).
  [JA-tok]   dev.to/aakira "ChatGPTを50ドルでトレーニングする方法",
             § "nanochatがカバーするもの" table (BPE vocabulary 32,768).

Readings where the pages are silent (each is also listed in the design notes):
pre-norm parameter-free RMSNorm (eps 1e-6) before attention, before the MLP and
before lm_head; QK-norm is the same RMSNorm over each head; RoPE rotates the
split halves (j, j+hd/2) by +t*base^(-2j/hd); softmax scale 1/sqrt(hd);
window W keeps keys t-W..t; kv head of q head h is h // (H/H_kv); the VE gate
reads the first 32 channels of the normed block input; smear adds the previous
token's embedding, gated from the current token's first 24 channels; backout
subtracts the residual entering layer L/2 after the last layer; the loss is the
mean next-token cross-entropy over all B*T positions; FP8 quantises each
operand of every product of the four block GEMMs (forward, input gradient,
weight gradient), taken as the bf16 tensor it is in the model, per tensor
with scale 448/amax, round-to-nearest-even, saturating.

Parity status: every function here is pinned by the "not gpu" tests in
tests/test_oracle_*.py (finite differences, closed forms, invariants, and
independent torch CPU library routines).
"""
from .model import (  # noqa: F401
    rmsnorm, rmsnorm_backward, rope_tables, rope, rope_backward,
    attention_forward, attention_backward, visible_mask,
    block_forward, block_backward, stack_forward, stack_backward,
    lm_head_xent, smear_forward, smear_backward,
)
from .fp8 import bf16_round, e4m3_round, quantize_e4m3, fp8_scale, fp8_matmul  # noqa: F401
