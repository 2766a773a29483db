"""MSA on B200: two-stage block-sparse GQA attention (index select, then sparse attention).

The compute lives in ``libmsa.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/msa.h``).  This package is a thin ctypes binding over it:
argument marshalling only, torch tensors are used for device memory and
streams.  ``inputs`` draws seeded synthetic problems.
"""

from .inputs import WORKLOADS, Problem, make_inputs  # noqa: F401

__all__ = ["WORKLOADS", "Problem", "make_inputs"]
