"""2:4 fine-grained structured sparsity for linear and 1x1-conv layers on B200.

* :mod:`.sp24`     -- binding of the C ABI (include/sp24.h), libsp24.so
* :mod:`.pipeline` -- allocate-and-call helpers (torch for device memory)
* :mod:`.inputs`   -- seeded synthetic workloads
* :mod:`.build`    -- builds libsp24.so in-tree with nvcc (sm_100a)
"""
__all__ = ["sp24", "pipeline", "inputs", "build"]
