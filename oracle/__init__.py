"""CPU oracle for the MXFP8 grouped expert MLP -- TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 restatement of what the hot path computes, used to check the
CUDA library. Only the test-suite, ``__graft_entry__.smoke()`` and the benchmark's
``cpu_baseline`` / ``--impl reference`` legs may import it; the product package
never does, and the oracle never imports the product package. Both sides share only
the seeded input generators in ``moe_workloads``.

Sources (three short web pages on one NVIDIA tutorial; no code, no formulas):
  * "MoE-Training für biologische Grundmodelle optimieren" (hyper.ai, German)
  * "NVIDIA apresenta técnicas para tornar mais eficiente o treinamento de modelos
    biológicos baseados em arquitetura MoE" (conexaotc.com.br, Portuguese)
  * "NVIDIA optimise l'entraînement MoE des modèles biologiques" (hyper.ai, French)
They name the steps (grouping tokens by per-expert counts, MXFP8 with one scale per
32-value block, a fused gate-up + SwiGLU + routing-scale kernel, forward and backward)
but fix no element format, rounding or layout; every such choice below is a stated
reading, and each function's docstring says which.

Pins (tests marked ``not gpu``): exhaustive E4M3 round trip, hand-built
quantisation blocks, brute-force permutation, per-token loop == grouped forward,
dense-MLP reduction, SwiGLU closed forms, finite differences of the backward (quantisation
off); the quantised backward equals ``moe.mlp_bwd_per_expert``, an expert-by-expert
restatement that quantises each backward GEMM's operands along that GEMM's contraction
index in an explicit block loop (a planted swap of any operand's block direction fails
it); for the
router (``router``): softmax closed forms, brute-force top-k with ties, -inf experts,
finite differences of the top-k backward; for the per-tensor FP8 recipe
(``moe.mlp_fwd_fp8_tensor`` / ``mlp_bwd_fp8_tensor``): the fp32 multiplier against exact
rational arithmetic, the largest magnitude onto 448, the fp32 rounding of the product, the
2^-4 error bound, reduction to the unquantised layer under an identity quantiser, and a
token-by-token restatement (with and without saturation of the delayed Z / dGU scales).
Parity unpinned: the end-to-end numeric level against the pages (they print no
accuracy, loss or worked example).
"""
from . import mxfp8, moe, router  # noqa: F401
