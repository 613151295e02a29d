"""CPU oracle for random-rotation vector quantization — TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, fp64 (numpy) restatement of what the GPU library
computes.  It exists to check the CUDA path: only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it.  The product path (``random_rotation_kv_b200``)
never imports, links or executes anything here, and nothing here imports the
product: the two share no code.

Sources (web pages, cited by title and section):

* "Random-rotation quantization" (brain.bigb.es, Russian title
  "Квантование со случайным поворотом") — the method itself: the three-step
  scheme, "Why rotation works", "History" (DRIVE, EDEN, QJL, TurboQuant),
  "Three decoders, one rotation", "Bias vs unbiasedness".
* "Attn-rot (TurboQuant lite) in llama.cpp" (ai-manual.ru) — rotate K/V, then
  q4_0 blocks.
* "TurboQuant and per-layer outlier-aware K" (ai-manual.ru), section
  "TurboQuant 2026: smart rotation" — the rotation is a fast Walsh–Hadamard
  transform (FWHT).

Module map:

* ``rng``       — SplitMix64 counter generator, rotation sign vector, Gaussian
                  QJL matrix (Box–Muller), bf16 rounding.
* ``hadamard``  — dense Sylvester–Hadamard matrix and the rotation Π = H·D/√d.
* ``codebook``  — Lloyd–Max codebook for N(0,1) and its distortion.
* ``rrq``       — encode / decode / rotate / packed codes / attention scores.
* ``q4_0``      — rotate-then-q4_0 ("Attn-rot") encode and decode.
* ``qjl``       — 1-bit QJL sign sketch of the residual and its estimator.
* ``sphere``    — the sphere marginal (Beta density) and the DRIVE scales, used
                  only to pin the rotation against the page's statements.

Parity status of each function is stated in its module header.
"""

from . import rng, hadamard, codebook, rrq, q4_0, qjl, sphere  # noqa: F401
