"""CPU oracle for the SVDQuant W4A4 + low-rank linear layer.

TEST INFRASTRUCTURE ONLY. This package is a plain, slow, obviously correct
float64 restatement of what the layer computes. Only the test suite, the smoke
check in ``__graft_entry__`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it. The product path (the CUDA library and its
Python binding) never imports, links or executes anything in here, and this
package shares no code with it: the only module both sides use is the seeded
input generator in ``workloads``.

Sources (cited per function):

* "SVDQuant Low-Rank Residual Quantization Algorithm Terminology Entry"
  (msModelSlim knowledge base), section 2.3: the migration identity
  Y = XW + b = (X diag(s)^-1)(diag(s) W) + b (eq. 1), the smoothing factor
  s = A_scale^alpha / W_scale^(1-alpha), s >= s_min (eq. 2), the split
  W ~ (U S) V^T, R = W - (U S) V^T (eq. 3), the dual-path output
  Q(X diag(s)^-1) Q(R) + (X diag(s)^-1 V)(U S)^T (eq. 4), Eckart-Young (eq. 5)
  and the residual energy sum of the discarded sigma_i^2 (eq. 6); section 2.2
  (W = L + R, L = U_r Sigma_r V_r^T); section 2.6 (2-D weights, rank <= 128
  recommended).
* "SVDQuant: Absorbing Outliers by Low-Rank Components for 4-Bit Diffusion
  Models" (arXiv 2411.05007), abstract: 4-bit weights and activations, a
  high-precision low-rank branch, LoRA attached without re-quantization.
* The 4-bit formats are not defined on those pages. INT4 group 64 and NVFP4
  (E2M1 elements, group 16, E4M3 group scales, one fp32 tensor scale) follow
  the OCP Microscaling Formats (MX) v1.0 specification and the FP8 E4M3
  definition of "FP8 Formats for Deep Learning" (Micikevicius et al., 2022).

Every function here is pinned by a test in ``tests/test_oracle_*.py`` against
something other than itself (closed forms, brute force, library routines,
invariants). Nothing is marked "parity unpinned".
"""
from .formats import (  # noqa: F401
    E2M1_VALUES,
    E4M3_MAX,
    bf16_round,
    e2m1_decode,
    e2m1_encode,
    e4m3_decode,
    e4m3_encode,
    quantize_int4_g64,
    quantize_nvfp4_g16,
    dequantize,
)
from .svdquant import (  # noqa: F401
    Prepared,
    attach_lora,
    calibrate_absmax,
    forward,
    forward_unquantized,
    prepare,
    prepare_from_factors,
    smoothing_factors,
    svd_factors,
)
