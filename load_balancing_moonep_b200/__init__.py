"""MoonEP redundant-expert plan and fused permute/unpermute for B200 (sm_100a).

The CUDA library lives in ``csrc/`` behind the C ABI declared in
``include/moonep.h``; ``moonep`` is its thin ctypes binding.  Importing the
package itself loads nothing: ``from load_balancing_moonep_b200 import moonep``
loads the shared library and fails loudly if it has not been built.
"""
__all__ = ["moonep", "workloads"]
