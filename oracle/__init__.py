"""CPU oracle for the Qwen3-VL text-decoder prefill (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package; the library never does.
"""
from . import q3vl_oracle  # noqa: F401
