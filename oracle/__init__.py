"""fp64 CPU oracle for the ByteCross decode step — TEST INFRASTRUCTURE ONLY.

This package is the checker, not the product.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import or run it.  It shares no code with the CUDA library
(``activation_kv_sparsity_b200``): neither imports the other, and the only
thing both sides consume is the seeded input module ``synth``.

Sources.  The method is the one of "Where Activation Sparsity and KV-Cache
Sparsity Cross in LLM Decoding" as described on the ByteCross README (the
GitHub page of js-lee-AI/ByteCross) and its arXiv abstract.  The pages do not
print Equations 1-5 nor any model code; ``byte_account`` restates the
equations in the form that reproduces every value the README prints, and
``decoder`` follows the Llama-style GQA decoder the pages time.

Pins (see tests/test_oracle_*.py): the byte account against the README's
printed values; the dense decoder against Hugging Face's Llama
implementation run in fp64; the activation-sparse and KV-selected modes
against the same implementation with masked projection inputs and per-head
attention masks; every selection routine against brute force on small inputs.
"""
from . import batch, byte_account, decoder  # noqa: F401
