"""B200-native (sm_100a) decode step of Step-3's MFA attention layer.

The compute path is the C-ABI library ``libmfa.so`` built from ``csrc/`` (hand-written CUDA
for sm_100a); ``mfa`` holds the thin Python binding (argument marshalling only).
``workloads`` draws the seeded synthetic inputs. Importing this package does not load the
library; the first call into ``mfa`` does, and fails loudly if it is missing.
"""

__all__ = ["mfa", "workloads"]
