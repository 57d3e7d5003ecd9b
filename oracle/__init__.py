"""Plain fp64 CPU oracle of one Flash-Cache step and of the model step around
it (``model_oracle``); test infrastructure only.

Only the tests, the package's ``__graft_entry__.smoke()`` check and the CPU
baseline leg of ``bench.py`` may import this package.  The CUDA library never
calls it and shares no code with it.
"""
from .flashcache_oracle import (  # noqa: F401
    bf16_round,
    round_for_cache,
    qkv_project,
    rope_angles,
    rope_rotate,
    write_cache,
    attend_sequence,
    step_sequence,
    flashcache_step,
    topk_tracked,
)
from . import model_oracle  # noqa: F401,E402
