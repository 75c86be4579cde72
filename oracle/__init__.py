"""fp64 CPU oracle for PBD window attention.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package. The CUDA library never calls it, and it shares no code with the CUDA
path: the only module both sides use is ``workloads`` (seeded random inputs,
no arithmetic of the method).
"""
from .pbd import (  # noqa: F401
    kv_append,
    visible_keys,
    pbd_window_mask,
    causal_window_mask,
    block_mask_bruteforce,
    pbd_block_ids,
    kv_head_of,
    window_attention,
    pbd_step,
    block_prefill_attention,
    block_prefill_row,
    kv_append_varwin,
    window_attention_varwin,
    pbd_step_varwin,
)
