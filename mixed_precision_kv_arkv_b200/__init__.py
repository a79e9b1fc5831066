"""B200 (sm_100a) decode path of the ARKV tri-state KV cache.

`abi` binds the C ABI of libarkv (include/arkv.h); `cache` holds the device
buffers and issues the calls of one layer's decode step; `workloads` and
`inputs` describe and draw the synthetic workloads.  Importing the package does
not load the CUDA library; the first call through `abi` does, and fails loudly
if it has not been built.
"""
