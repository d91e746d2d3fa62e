// Device side of the seeded input generator (see gen.h): the same counter
// hash and fp32 transforms, one thread per element, grid-stride.
#include <cuda_runtime.h>
#include <stdint.h>
#include "gen.h"

namespace {
__global__ void gen_fill_kernel(void* out, int64_t n, int64_t start, uint64_t seed,
                                uint32_t tensor_id, int dist, float p0, float p1, int dtype) {
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    float v = moe_gen_value(seed, tensor_id, (uint64_t)(start + i), dist, p0, p1);
    if (dtype == MOE_GEN_F32)
      ((float*)out)[i] = v;
    else
      ((uint16_t*)out)[i] = moe_gen_f32_to_bf16(v);
  }
}
}  // namespace

extern "C" int moe_gen_fill_cuda(void* out, int64_t n, int64_t start, uint64_t seed,
                                 uint32_t tensor_id, int dist, float p0, float p1, int dtype,
                                 void* stream) {
  if (n <= 0) return 0;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  gen_fill_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(out, n, start, seed, tensor_id,
                                                                     dist, p0, p1, dtype);
  return (int)cudaGetLastError();
}
