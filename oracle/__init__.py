"""CPU oracle for content-adaptive block-sparse attention (test infrastructure).

THIS PACKAGE IS TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT. Only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it. The library's compute path never calls it, and it shares no code with the
CUDA path (no common helpers, tables or constants); the only module both sides
use is ``sa_workloads``, which draws seeded random inputs and holds none of the
method's arithmetic.

Everything here is plain, slow and meant to be read against the method's
published description:

* ``gzip_mask``  - compression-ratio literal flags, the three per-head block
  masks and their token-level form ("Gzip-guided sparse attention: Selecting
  long-range content by compressibility", Core equations).
* ``attention``  - masked softmax attention forward (O, LSE) and its gradients,
  in float64, with the mask materialised densely (row chunks for long inputs).
* ``gist``       - the UniGist sink + interleaved gist + local window layout,
  its visibility rule and the per-tile gist shift ("UniGist: Towards General
  and Hardware-aligned Sequence-level Long Context Compression", Approach).
* ``decode``     - gist-scored top-k chunk selection and selective unfolding at
  decode ("Simplified Sparse Attention via Gist Tokens", abstract; "Forget,
  Then Recall: ... Gist Sparse Attention", abstract).

Where the pages leave a step open, the reading taken is stated in the
function's docstring. Every function is pinned by tests against closed forms,
special cases that reduce to library routines, invariants or brute force.
"""
from . import attention, decode, gist, gzip_mask  # noqa: F401
