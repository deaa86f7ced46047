// pack.cu — binary32 weights -> packed 4-bit / 2-bit group-affine matrix (layout in fmoe.h).
//
// The pages mention the offline weight-conversion scripts ("Qu'est-ce que Flash-MoE ?"
// (a2a-mcp.org, fr), "Conclusion") and the 4-/2-bit codes with a scale and bias per group
// (§2 "Noyaux de Déquantification Optimisés pour FMA"), not how scale and bias are chosen. The
// reading implemented here: per 64-weight group, s = bf16((max - min) / (2^bits - 1)),
// z = bf16(min), q = clamp(rint((w - z) / s), 0, 2^bits - 1) (q = 0 when s == 0), every
// operation an IEEE-rounded binary32 operation so the result is reproducible bit for bit.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fmoe {

template <int BITS>
__global__ void pack_kernel(const float* __restrict__ w, int rows, int cols,
                            uint8_t* __restrict__ dst) {
  constexpr int kPer = 32 / BITS;           // codes per word
  constexpr int kWords = 64 / kPer;         // words per group
  constexpr float kQmax = (float)((1 << BITS) - 1);
  const int groups = cols / 64;
  const long long ng = (long long)rows * groups;
  const size_t code_bytes = (size_t)rows * cols * BITS / 8;
  uint32_t* words = reinterpret_cast<uint32_t*>(dst);
  uint32_t* sb = reinterpret_cast<uint32_t*>(dst + code_bytes);
  for (long long gi = (long long)blockIdx.x * blockDim.x + threadIdx.x; gi < ng;
       gi += (long long)gridDim.x * blockDim.x) {
    const long long r = gi / groups;
    const int g = (int)(gi - r * groups);
    const float4* v4 = reinterpret_cast<const float4*>(w + r * cols + (size_t)g * 64);
    float v[64];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float4 a = __ldg(v4 + i);
      v[4 * i] = a.x;
      v[4 * i + 1] = a.y;
      v[4 * i + 2] = a.z;
      v[4 * i + 3] = a.w;
    }
    float mn = v[0], mx = v[0];
#pragma unroll
    for (int i = 1; i < 64; ++i) {
      mn = v[i] < mn ? v[i] : mn;
      mx = v[i] > mx ? v[i] : mx;
    }
    const float step = __fdiv_rn(__fsub_rn(mx, mn), kQmax);
    const __nv_bfloat16 sbf = __float2bfloat16_rn(step);
    const __nv_bfloat16 zbf = __float2bfloat16_rn(mn);
    const float s = __bfloat162float(sbf);
    const float z = __bfloat162float(zbf);
    const uint32_t s16 = __bfloat16_as_ushort(sbf), z16 = __bfloat16_as_ushort(zbf);
    sb[r * groups + g] = s16 | (z16 << 16);
    uint32_t out[kWords];
#pragma unroll
    for (int i = 0; i < kWords; ++i) out[i] = 0u;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      uint32_t q = 0;
      if (s != 0.0f) {
        float t = rintf(__fdiv_rn(__fsub_rn(v[i], z), s));
        t = fminf(fmaxf(t, 0.0f), kQmax);
        q = (uint32_t)t;
      }
      out[i / kPer] |= q << ((i % kPer) * BITS);
    }
    uint32_t* wd = words + (size_t)r * (cols / kPer) + (size_t)g * kWords;
#pragma unroll
    for (int i = 0; i < kWords; i += 4)
      *reinterpret_cast<uint4*>(wd + i) = make_uint4(out[i], out[i + 1], out[i + 2], out[i + 3]);
  }
}

}  // namespace fmoe

extern "C" cudaError_t fmoe_pack_launch(const float* w, int rows, int cols, int bits, void* dst,
                                        int sms, cudaStream_t stream) {
  const long long ng = (long long)rows * (cols / 64);
  long long blocks = (ng + 127) / 128;
  const long long cap = (long long)sms * 32;
  if (blocks > cap) blocks = cap;
  if (bits == 4)
    fmoe::pack_kernel<4><<<(unsigned)blocks, 128, 0, stream>>>(w, rows, cols, (uint8_t*)dst);
  else
    fmoe::pack_kernel<2><<<(unsigned)blocks, 128, 0, stream>>>(w, rows, cols, (uint8_t*)dst);
  return cudaGetLastError();
}
