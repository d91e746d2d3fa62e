/* Host side of the seeded input generator (see gen.h).  Fills n elements,
 * element i taking counter index start + i.  Built with -ffp-contract=off so
 * that the fp32 operations in gen.h round exactly as the device ones do. */
#include <stddef.h>
#include <stdint.h>
#include "gen.h"

void moe_gen_fill_host(void* out, int64_t n, int64_t start, uint64_t seed, uint32_t tensor_id,
                       int dist, float p0, float p1, int dtype) {
  if (dtype == MOE_GEN_F32) {
    float* o = (float*)out;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
      o[i] = moe_gen_value(seed, tensor_id, (uint64_t)(start + i), dist, p0, p1);
  } else {
    uint16_t* o = (uint16_t*)out;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
      o[i] = moe_gen_f32_to_bf16(moe_gen_value(seed, tensor_id, (uint64_t)(start + i), dist, p0, p1));
  }
}

uint64_t moe_gen_hash_host(uint64_t seed, uint32_t tensor_id, uint64_t index) {
  return moe_gen_hash(seed, tensor_id, index);
}
