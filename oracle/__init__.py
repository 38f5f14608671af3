"""Plain, slow, fp64 CPU oracle for rotation-based W4A4 quantization.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or call
anything in this package.  The product path (the CUDA library and its Python
binding) never imports it and never falls back to it.

The oracle shares no code with the CUDA path.  It follows the pages directly:

* "Rotations for 4-Bit Activations: QuaRot, SpinQuant, and Friends"
  (theservingstack.com/rotation-quantization), sections
  "A rotation changes nothing, and that is the point" (the invariance
  Y = X.W^T = (X.Q).(W.Q)^T, the 1/sqrt(n)-scaled Hadamard, the ratio and
  kurtosis measures), "What it buys in 4 bits, and what it doesn't" (INT4 with
  one scale per token / per output channel, NVFP4 with an FP8 scale per 16
  values, the relative product error), "The recipe" and "Gotchas" (128-wide
  Hadamard blocks, randomized Hadamard).
* "QuaRot (rotation-based outlier removal, W4A4KV4)", field "Activation scheme"
  (randomized Hadamard, applied to the KV cache too).
* "SpinQuant (learned rotations + W4A4KV4)", field "Activation scheme"
  (asymmetric INT4 for the KV cache).

Every function computes in float64 unless a format fixes the precision (fp32
scales, fp16 KV scale/zero, E4M3 / E2M1 codes).  Library primitives used as
steps: numpy matmul (dense Hadamard product, integer-valued GEMM), numpy
rounding (np.rint is round-half-to-even), numpy float16 conversion.

Parity pins: every function here is pinned by a ``-m "not gpu"`` test in
``tests/test_oracle_*.py`` against closed forms, brute force or library
routines.  The per-config percentages the pages print for real Qwen3-8B layers
(46%->11% etc.) are not reproducible on synthetic data: those qualitative
claims are checked as inequalities only ("parity unpinned" for the exact
figures, see ``metrics.py``).
"""

from . import formats, gemm, hadamard, metrics, quant  # noqa: F401
