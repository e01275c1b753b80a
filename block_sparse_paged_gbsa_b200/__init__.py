"""Block-sparse paged GQA flash attention (forward, and its gradients) for NVIDIA
B200 (sm_100a).

The compute path is the C-ABI library ``libgbsa.so`` built from ``csrc/``; this
package only marshals arguments to it (``gbsa.py``).  Importing the package
does not load the library; the first call does, and fails loudly if the
library is missing.
"""
from .gbsa import (GbsaError, Problem, backward, forward, library_path, metadata,  # noqa: F401
                   metadata_size, workspace_size)

__all__ = ["GbsaError", "Problem", "backward", "forward", "metadata", "metadata_size", "workspace_size",
           "library_path"]
