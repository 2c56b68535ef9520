"""fp64 CPU oracle for sliding-window / global causal GQA attention with a
per-head attention-sink logit.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package. The product
library never imports it, and it imports nothing from the product package.

``oracle.fp8`` adds the E4M3 code table and encoder and the decode / commit
over a ring of E4M3 codes with per-kv-head scales (numpy, fp64).
``oracle.rope`` adds the rotary position embedding applied before the
attention (fp64 rotation, bf16 rounding) and the ring the prefill writes.
``oracle.backward`` adds the gradients of the prefill (dq, dk, dv and the
sink's), whole or at sampled rows and keys.
"""
from .oracle import (  # noqa: F401
    decode,
    kv_commit,
    prefill,
    prefill_rows,
    default_threads,
)
