"""B200-native (sm_100a) VanillaMarkov transition-bias head.

The compute lives in libdspark_markov.so (CUDA kernels behind the C ABI in
include/dspark_markov.h); this package is its thin Python face. Importing the
package does not load the library; the first head constructed does, and fails
loudly if it has not been built.
"""
from .head import (VanillaMarkov, build_markov_head, device_status, last_algo, last_variant, launch_count,  # noqa: F401
                   set_algo, set_debug)
from ._native import DSparkError  # noqa: F401

__all__ = ["VanillaMarkov", "build_markov_head", "device_status", "set_algo", "launch_count", "last_algo",
           "last_variant", "set_debug", "DSparkError"]
