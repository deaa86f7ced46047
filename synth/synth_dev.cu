// synth_dev.cu — device side of the seeded input generator (see philox.h). Generates the
// synthetic weights directly in HBM so that 100+ GB workloads never pass through the host.
#include <cuda_runtime.h>
#include <stdint.h>

#include "philox.h"

__global__ void syn_fill_normal_kernel(float* __restrict__ out, uint64_t n, uint64_t seed,
                                       uint64_t st, uint64_t offset, float c) {
    uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t j = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n; j += stride) {
        int32_t s = syn_ih_int(seed, st, offset + j);
        out[j] = __fmul_rn((float)s, c);  // int -> float is exact (|s| < 2^24)
    }
}

extern "C" int syn_fill_normal_dev(float* out, uint64_t n, uint64_t seed, uint64_t st,
                                   uint64_t offset, float c, void* stream) {
    if (n == 0) return 0;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    uint64_t blocks = (n + 255) / 256;
    uint64_t cap = (uint64_t)sms * 16;
    if (blocks > cap) blocks = cap;
    syn_fill_normal_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(out, n, seed, st,
                                                                              offset, c);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}
