"""CPU oracle for the QK4V8 block-scaled attention path — TEST INFRASTRUCTURE ONLY.

A plain, slow, float64 restatement of what the CUDA library computes, written from the
method's description and checked against closed forms, brute force and invariants in
``tests/``. Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import it. It shares no code with the library and imports nothing from it.

Modules: ``formats`` (E2M1 / E4M3 / E8M0 tables and encoders), ``quant`` (NVFP4 for Q/K,
MXFP8 for V), ``attention`` (tiled online-softmax QK4V8 attention, FP16 tiles, split-K
decode), ``tilescore`` (exact tile scores and top-fraction selection), ``paged`` (the paged
KV-cache layout read back into dense form).
"""
from . import formats, quant, attention, tilescore, paged  # noqa: F401
