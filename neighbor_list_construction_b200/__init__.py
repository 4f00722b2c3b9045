"""B200-native periodic neighbor-list build.

The compute path is the CUDA library ``libnl.so`` (sources in ``csrc/``,
C ABI in ``include/nl.h``); :mod:`neighbor_list_construction_b200.nl` is its
thin Python binding.  :mod:`neighbor_list_construction_b200.workloads` draws
the seeded synthetic inputs.  Importing this package loads nothing; importing
``.nl`` loads the library and fails loudly if it is missing.
"""
__all__ = ["nl", "workloads"]
