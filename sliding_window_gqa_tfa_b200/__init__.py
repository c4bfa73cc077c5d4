"""B200-native tiled GQA prefill attention.

The product is the C-ABI library ``libtfa.so`` (``include/tfa.h``); this
package holds its CUDA sources (``csrc/``), the thin ctypes binding with the
same entry-point names, and the seeded input generator shared with the tests.
"""
from .inputs import HEADLINE, WORKLOADS, Workload, make_inputs, shaped  # noqa: F401
