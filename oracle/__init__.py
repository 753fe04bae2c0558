"""CPU oracle for the SVDQuant W4A4 linear and the AWQ W4A16 linear.

TEST INFRASTRUCTURE ONLY.  Plain, slow, obviously-correct numpy code
(fp64 for the contractions, per-operation IEEE fp32 where the method
rounds).  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
It shares no code, table or helper with the CUDA library
(``svdquant_w4a4_gemm_b200``) and imports nothing from it; the product path
never calls it.

What it follows (pages cited by title and section):

* "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers" and its
  re-tellings (ainews.surl.tw "Diffusers Natively Integrates Nunchaku Lite…",
  paragraph 2; blog.margrop.com "技术细节 §1", the four-step SVDQuant list;
  app.hamidun.com "Что такое Nunchaku и SVDQuant"): activation outliers are
  migrated into the weights (smoothing), the hardest part of each weight is
  a 16-bit low-rank branch, the residual is quantized to 4 bits, and both
  weights and activations are 4-bit (W4A4).
* The same pages' hardware table (blog.margrop.com "技术细节 §3"): the
  Blackwell precision is NVFP4.  The NVFP4 encoding (E2M1 element codes,
  one E4M3 scale per 16 elements, an fp32 tensor scale) and the 128x4
  swizzled scale layout are public format definitions (OCP MX / NVIDIA
  NVFP4 and cuBLAS block-scaling documentation); the pages name the format
  but do not define it.
* AWQ W4A16 for modulation layers (ainews.surl.tw paragraph 2;
  app.hamidun.com "Что такое Nunchaku и SVDQuant"; keryc.com "Nunchaku
  Lite: integración y modelo de ejecución").

Every function is pinned by ``tests/test_oracle_*.py`` to something other
than itself (closed forms, a library routine, brute force, printed format
tables under ``tests/golden/``).  No function here is "parity unpinned".
"""

from . import codecs, svdq, awq, prep  # noqa: F401
