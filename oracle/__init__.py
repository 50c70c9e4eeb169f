"""fp64 CPU oracle of absorbed multi-head latent attention over a latent KV ring.

Test infrastructure only: the tests, the package smoke check and the benchmark's CPU
baseline leg may use it; the CUDA path never does.
"""

from .mla_oracle import *  # noqa: F401,F403
