"""B200-native (sm_100a) GSPN 4-direction line-scan propagation.

The propagation runs in the CUDA library built from ``csrc/`` (C ABI in
``include/gspn.h``); ``gspn`` is its thin Python binding and ``inputs`` the
seeded synthetic input generator.  Importing the package does not load the
library; the first call does, and fails loudly if it is missing.
"""
from .gspn import (GSPN_BF16, GSPN_F32, GSPNError, forward, forward_dir, forward_host,
                   last_launch_count, library_path, load_library, release, status_string,
                   version)
from .inputs import HEADLINE, WORKLOADS, Workload, make_inputs

__all__ = [
    "GSPN_BF16", "GSPN_F32", "GSPNError", "forward", "forward_dir", "forward_host",
    "last_launch_count", "library_path", "load_library", "release", "status_string", "version",
    "HEADLINE", "WORKLOADS", "Workload", "make_inputs",
]
