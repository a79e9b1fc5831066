// arkv_copy_async: a byte copy done by a kernel (16-byte vectors, grid-stride), for
// moving the decode loop's inputs and outputs between page-locked host memory and the
// device inside a CUDA graph without a copy-engine node.
#include "arkv_internal.cuh"

namespace arkv {

namespace {

__global__ void __launch_bounds__(256) copy16_kernel(uint4* __restrict__ dst, const uint4* __restrict__ src,
                                                     size_t n16) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += stride) dst[i] = src[i];
}

}  // namespace

cudaError_t launch_copy16(void* dst, const void* src, size_t bytes, cudaStream_t s) {
    const size_t n16 = bytes / 16;
    size_t blocks = (n16 + 255) / 256;
    if (blocks > 1184) blocks = 1184;   // enough 16-byte loads in flight for the bus; the rest loop
    copy16_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<uint4*>(dst),
                                                   reinterpret_cast<const uint4*>(src), n16);
    return cudaGetLastError();
}

}  // namespace arkv
