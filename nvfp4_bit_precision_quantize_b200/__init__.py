"""B200-native NVFP4 linear layer: quantiser + block-scaled GEMM behind a C ABI.

The CUDA library (libnvfp4.so, built in-tree for sm_100a) does all the work;
`binding` marshals torch tensors into its C calls.  `workloads` draws the
seeded synthetic inputs.  Importing the package loads nothing; the first call
into `binding` loads the library and raises if it is missing.
"""
