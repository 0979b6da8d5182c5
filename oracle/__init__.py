"""CPU oracle of the canvas-denoising hot path.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, fp64 (and, for the
random draws and every selection, integer-exact) restatement of what the
denoising method computes.  It exists to check the CUDA path.  Only the test
suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import it; the product path never does, and it imports nothing from the
product package.

Modules:
  philox   Philox4x32-10 from its published definition, plus the draw layout.
  model    the transformer forward (prefill, bidirectional canvas pass, block
           re-encode and KV append).
  sampler  temperature schedule, per-position statistics, Gumbel-max sample,
           top-k commit, threshold re-noise, adaptive stop.
  loop     the block-autoregressive loop composed from the two.
  fp8      e4m3 encoding from the format's definition, per-row / per-tensor
           scaling, and the FP8 unembedding's logits.

Parity status: every function is pinned by a test under tests/ against the
pages' fixed settings, closed forms, library routines or invariants, except
the exact bit layout of the Philox draws (counter/key assignment), which the
pages do not fix: "parity unpinned" for that layout beyond the generator's
published known-answer vectors.
"""
