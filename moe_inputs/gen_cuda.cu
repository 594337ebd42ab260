/*
 * CUDA implementation of the seeded input generator (formulas in gen_core.h),
 * bit-identical to gen_host.c.  Used to fill device tensors directly, so that
 * multi-GB weight sets never cross PCIe.
 */
#include <cuda_runtime.h>
#include <stdint.h>

#include "gen_core.h"

namespace {

__global__ void gen_kernel(uint64_t key, uint64_t first, size_t count, float scale, void* out,
                           int kind) {
  size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride) {
    uint64_t idx = first + (uint64_t)i;
    if (kind == 0)
      ((uint16_t*)out)[i] = gen_f32_to_bf16(gen_normal_f32(key, idx, scale));
    else if (kind == 1)
      ((float*)out)[i] = gen_normal_f32(key, idx, scale);
    else
      ((float*)out)[i] = gen_uniform01(key, idx);
  }
}

int launch(uint64_t key, uint64_t first, size_t count, float scale, void* out, int kind,
           void* stream) {
  if (count == 0) return 0;
  if (out == nullptr) return (int)cudaErrorInvalidValue;
  size_t blocks = (count + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  gen_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(key, first, count, scale, out, kind);
  return (int)cudaGetLastError();
}

}  // namespace

extern "C" {
int gen_normal_bf16_cuda(uint64_t key, uint64_t first, size_t count, float scale, uint16_t* out,
                         void* stream) {
  return launch(key, first, count, scale, out, 0, stream);
}
int gen_normal_f32_cuda(uint64_t key, uint64_t first, size_t count, float scale, float* out,
                        void* stream) {
  return launch(key, first, count, scale, out, 1, stream);
}
int gen_uniform_f32_cuda(uint64_t key, uint64_t first, size_t count, float* out, void* stream) {
  return launch(key, first, count, 0.0f, out, 2, stream);
}
}
