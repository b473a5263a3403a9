"""B200 (sm_100a) block-sparse attention with cumulant-order block selection (COBS).

The compute lives in the CUDA library ``lib/libcobs.so`` (C ABI in ``include/cobs.h``);
``block_sparse_long_summary_b200.cobs`` is its thin Python binding (PyTorch supplies
device memory and streams). Build the library with
``python -m block_sparse_long_summary_b200.build``.
"""

__all__ = ["build", "cobs"]
