"""CPU oracle for the SVDQuant-style W4A4 + low-rank linear layer.

TEST INFRASTRUCTURE ONLY. This package is a plain, slow, fp64 restatement of what the layer
computes; it exists to check the CUDA library against. Only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference arm may import it. The product path (the C-ABI library
and its Python binding) never imports, links or executes anything here, and this package imports
nothing from the product.

Modules:
  nvfp4     -- E2M1 / E4M3 codecs and the NVFP4 block quantizer.
  svdquant  -- smoothing factors, the low-rank/residual split, and the layer forward.
  fp8r      -- the row-wise FP8 (W8A8) variant of the same layer.

Pins (what each function is checked against, in ``tests/test_oracle_*.py``):
  codecs            -- the format's printed E2M1 grid and hand-derived tie cases; a closed-form
                       round-half-even formulation over every rounding boundary and over every
                       fp32 bit pattern of the window that holds all rounding decisions (the
                       zero and saturation tails sampled); torch's float8_e4m3fn conversion (a
                       library routine) over that window below its non-saturating range.
  bf16 rounding     -- hand-derived ties, and torch's fp32 -> bf16 cast on random values and ties.
  block quantizer   -- quantize/dequantize idempotence with scales held fixed, scale bounds,
                       the amax block landing on the largest E4M3 code, all-zero blocks.
  smoothing         -- the identity X.W = (X.diag(lambda)^-1)(diag(lambda).W) and lambda=1 cases.
  low-rank split    -- W_hat = L1.L2 + R to fp32 rounding, Eckart-Young (spectral norm of the
                       unrounded residual equals sigma_{r+1}), r=0 giving R = W_hat.
  layer forward     -- brute-force exact-rational triple loop on tiny shapes; r=0 reducing to plain
                       W4A4; SwiGLU closed form and special values.
  fp8r              -- row quantizer: idempotence with scales held fixed, the amax element landing
                       on +-448, zero rows, the E4M3 half-ulp error bound, scale invariance under
                       power-of-two row scaling; layer: exact-rational triple loop, r=0 reducing
                       to plain W8A8.
No function here is left without a pin.
"""
