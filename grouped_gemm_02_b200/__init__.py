"""B200 (sm_100a) fused Mixture-of-Experts layer forward.

``grouped_gemm_02_b200.moe`` is the Python binding of the C ABI in
``include/moe.h`` (libmoe_b200.so, built by ``grouped_gemm_02_b200/build.py``);
``grouped_gemm_02_b200.workload`` draws the seeded synthetic inputs.  Importing
the package loads nothing; the CUDA library is opened on first use and a
missing library raises instead of falling back to anything else.
"""

__all__ = ["moe", "workload", "stats", "build"]
