"""CPU oracle for CoSA block-sparse causal prefill attention (test infrastructure).

Only the tests, the smoke check and the benchmark's CPU-baseline leg import this
package.  The product path (the C-ABI library and its Python binding) never
imports, links or calls it.
"""
from .cosa_oracle import *  # noqa: F401,F403
from .cosa_oracle import __all__  # noqa: F401
