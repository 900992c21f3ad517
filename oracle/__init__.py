"""CPU oracle for the asym_w4a8_int8 ConvRot linear layer.

TEST INFRASTRUCTURE ONLY.  This package is the slow, plain, fp64 statement of
what the layer computes.  It exists so that the CUDA library can be checked
against something written independently of it.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it.  The product path (the C-ABI library and
its Python binding) never imports, calls or links anything in here, and this
package imports nothing from the product.

Sources (page title and section):

* "Qwen3.8-27B-AEON-ULTIMATE-UNCENSORED-BF16 — W4A8 ConvRot for ComfyUI"
  model card (KENIC-1), sections "Why this exists", "Format", "Verification"
  and "Reproducing" -- called the *ConvRot card* below.
* "Qwen3.8-27B-W4A8" model card (CuTIsolation), sections "Model Overview" and
  "Accuracy" -- called the *W4A8 card* below.
* "Qwen3.8-27B-Uncensored-NVFP4: En runbook för servering på Blackwell-GPU:er",
  section "Vad NVFP4 är, och hur det skiljer sig från FP8 och från INT8/AWQ"
  -- the *NVFP4 runbook*: the format of the comparison foil in
  :mod:`oracle.nvfp4_ref` (imported explicitly, not re-exported here).

Every function in :mod:`oracle.w4a8_ref` names the passage it follows.  Where
the pages leave a step open, the reading taken is written beside the code.
"""

from .w4a8_ref import *  # noqa: F401,F403
