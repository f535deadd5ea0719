"""Float64 CPU oracle for CommVQ decode attention (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import this
package.  It shares no code with the CUDA library and the library never imports it.
"""
from . import brute, cvq_oracle, encode, pack  # noqa: F401
