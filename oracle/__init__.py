"""Float64 CPU checker for the per-layer GPTQ path.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg are the only callers.  The CUDA library never imports or links
anything here, and nothing here imports the CUDA library.

Parity status per function (the pins live in tests/test_oracle_pins.py):
  hessian            pinned: brute-force triple loop, symmetry, PSD
  hessian_block      pinned: equals entries of hessian()
  damp               pinned: closed form on hand-written matrices
  act_order_perm     pinned: hand-checked orders, ties, invariance
  inverse_gauss_jordan  pinned: A A^-1 = I, LAPACK inverse
  obs_upper / prepare   pinned: LAPACK chol(inv(H_d)) and the reversal route
  quantize / gptq_rows  pinned: diagonal H -> RTN, W - Q = E U identity,
                        blocked == unblocked, d_in = 1 and 2 closed forms,
                        power-of-two invariances, brute-force lower bound,
                        GPTQ <= RTN on output error
  rtn                pinned: hand-computed quantizer fixtures (tests/golden)
  pack_int4 / g_idx  pinned: hand-computed nibble fixtures
  output_mse         pinned: equals ||(W - W^) X^T||^2 / (N d_out) directly
"""
from .gptq import *  # noqa: F401,F403
