"""CPU oracle for the IQ8R rotated W8A8 linear -- test infrastructure only.

Imported by the tests, the package's smoke check and the CPU-baseline leg of
the benchmark; never by the library.
"""

from .iq8r_oracle import *  # noqa: F401,F403
from .iq8r_oracle import __all__  # noqa: F401
