"""fp64 CPU oracle for exact attention.  Test infrastructure only: imported by
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py``, never by the CUDA library or its Python binding."""
from .attention_ref import (  # noqa: F401
    attention_backward,
    attention_bruteforce,
    attention_delta,
    attention_forward,
    attention_forward_online,
    attention_probs,
    attention_sampled_rows,
    to_f64,
)
