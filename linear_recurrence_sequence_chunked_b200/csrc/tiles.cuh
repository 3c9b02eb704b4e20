// tiles.cuh -- operand-tile helpers shared by the tensor-core chunk kernels:
// offsets in the no-swizzle "TL" layout (8-row x 16-byte core matrices, row
// groups major) and bf16 packing.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace pdn {

// TL tile offsets (bytes) of the 16-byte row segment (row, 8-column group).
__device__ __forceinline__ uint32_t tl128(int row, int c8) {
  return (uint32_t)(((row >> 3) * 16 + c8) * 128 + (row & 7) * 16);
}
__device__ __forceinline__ uint32_t tl64(int row, int c8) {
  return (uint32_t)(((row >> 3) * 8 + c8) * 128 + (row & 7) * 16);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ uint4 pack8(const float (&v)[8]) {
  return make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                    pack_bf16(v[6], v[7]));
}
__device__ __forceinline__ void unpack8(uint4 u, float (&v)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&w[i]);
    v[2 * i] = __low2float(b);
    v[2 * i + 1] = __high2float(b);
  }
}
__device__ __forceinline__ void ld8f(const float *p, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4 *>(p);
  const float4 b = *reinterpret_cast<const float4 *>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

}  // namespace pdn
