"""CPU oracle for the SVDQuant W4A4 linear layer -- TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously-correct restatement of what the layer computes, in
numpy (fp64 unless a step fixes a narrower precision).  It shares no code with
the CUDA library: no kernels, headers, tables or helpers.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it; the product path never does.

Sources (page title, section):
  [Lite]    "Nunchaku Lite: the 50% VRAM reduction now integrated into
            Diffusers" (axbrief.com), section "The Mechanics of 4-Bit
            Efficiency and SVDQuant" -- outliers moved from activations to
            weights, weight split into a 16-bit low-rank branch plus a 4-bit
            residual, W4A4.
  [Apatero] "Problemas do Nunchaku Qwen e como corrigi-los em 2025"
            (apatero.com), section "O que e Nunchaku e como acelera modelos
            Qwen" -- outlier migration, SVD low-rank branch, the down
            projection fused with quantisation and the up projection fused
            with the 4-bit GEMM (the branches share the activations).
  [Note]    "Nunchaku 1.3.0 for Python3.14.x & alpha" (note.com), section
            "SVDQ-FP4 on Blackwell", part "1. INT4" -- INT4 is -8..+7 and
            W ~ int4 * scale; part "2. SVDQ-FP4" -- FP4 has a sign bit, a
            small exponent and the rest mantissa.

Readings where the pages are silent: alpha = 0.5
balanced migration; lambda calibrated on the runtime X; sqrt(Sigma) split of
the SVD factors; groups along K for both operands; scale = amax/7 (INT4, bf16)
and amax/6 (NVFP4, E4M3); round-half-to-even everywhere; X' rounded to bf16;
T = X'.L1 kept in fp32; tanh-form GELU.

Parity status per function is stated in each module's header.
"""
