"""CPU oracle for the verification step of masked-diffusion speculative / revocable decoding.

TEST INFRASTRUCTURE ONLY. This package is a plain, slow, fp64 restatement of
what the verification step computes, written from the three source pages:

  [COVER]  "Stop the Flip-Flop: Context-Preserving Verification for Fast
           Revocable Diffusion Decoding" (Methodology: COVER, sections 1-3)
  [DD]     "DualDiffusion: A Speculative Decoding Strategy for Masked Diffusion
           Models" (section 2, Methodology: Verification Algorithms)
  [SPOT]   "[Review] On the SPOT: Enhancing Speculative Decoding for Diffusion
           Language Models via Commit-Order Prediction" (section 1 Key Terms:
           Coupled-Noise Verification; section 3 Method)

Only the test suite, the smoke check and the benchmark's CPU-baseline arm may
import it. It shares no code with the CUDA library (no common kernels,
headers, helpers or tables) and imports nothing from it. Inputs are widened
to fp64 from the exact fp32/bf16 bits the CUDA path receives.

Modules:
  philox     Philox4x32-10 and the Gumbel noise drawn from it
  attention  dual-view (cache-override + leave-one-out) attention, d_in, d_out
  vocab      per-row verifier/drafter statistics and coupled Gumbel samples
  seeds      stability score and top-k seed selection
  decide     KEEP / REPLACE / REMASK policies

Parity status: every function is pinned by invariants, closed forms, brute
force or library routines (see tests/test_oracle_*.py); the pages print no
worked numeric example for any step, so no value-level golden from the pages
exists.
"""
from . import philox, attention, vocab, seeds, decide  # noqa: F401
