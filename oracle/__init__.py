"""CPU oracle for the SVDQuant W4A4 linear layer and the AWQ W4A16 projection.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code,
table or constant generator with the CUDA library; the two meet only through
the seeded inputs of ``bit_w4a4_diffusion_smooth_b200.synthetic``.

Everything here is plain numpy: float64 for the exact arithmetic of the
method, float32 (IEEE round-to-nearest-even, one rounding per operation) for
the steps whose precision decides an integer code, and small pure-Python
loops only in the brute-force helpers used by the pins.

Sources (web pages on Nunchaku / SVDQuant 4-bit diffusion inference):
  [Remio]    "Nunchaku Diffusers 支持降低显存占用，但硬件仍决定适用范围" (remio.ai),
             section "SVDQuant 将棘手数值移出 4 位路径" (smoothing, low-rank
             16-bit branch, 4-bit residual, the two kernel fusions) and
             "Nunchaku Diffusers 支持改变了加载路径" (SVDQ W4A4 vs AWQ W4A16 layers).
  [Donmalab] "Diffusers × Nunchaku 4-bit" (donmalab.com), sections
             "量化的核心挑戰" (outliers; low-rank branch plus 4-bit rest, results
             added) and "Nunchaku Lite" (the two layer kinds).
The pages fix no numeric format beyond the names NVFP4 / INT4 / W4A16; the
NVFP4 element grid (e2m1), the 16-element block with an e4m3 block scale and
an fp32 tensor scale follow NVIDIA's published NVFP4 definition, and every
reading the pages leave open is listed in the repository's design notes.

Parity status per function (what pins it; see tests/test_oracle_*.py):
  formats.e2m1_encode / ue4m3_encode / bf16_round   brute force + torch e4m3/bf16
  nvfp4.quantize_blocks / dequantize                grid special cases, max-code
                                                     invariant, error bound
  svdquant.smooth                                   X^.W' == X.W invariant
  svdquant.low_rank                                 Eckart-Young, exact rank-r
  svdquant.quantize_act / w4a4_linear               r=0 reduction, brute-force
                                                     tiny GEMM, rank-r residual 0
  awq.*                                             brute-force group search,
                                                     error bound, grid cases
  svdquant.forward accuracy against X.W + b         parity unpinned (the pages
                                                     print no accuracy figure)
"""
