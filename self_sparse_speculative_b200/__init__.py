"""S3R decode step on B200: sparse draft attention, dense verify attention and
exact speculative sampling as sm_100a CUDA kernels behind a C ABI (libs3r.so).

``self_sparse_speculative_b200.s3r`` is the ctypes binding of that library;
``self_sparse_speculative_b200.workloads`` draws the seeded synthetic inputs.
Importing the package itself loads nothing.
"""
