// synth_cuda.cu - device fill of the seeded input generator (definition in synth.h).
// Produces the same bits as synth_fill_host for the same arguments.
#include <cuda_runtime.h>
#include <stdint.h>

#include "synth.h"

namespace {

__global__ void synth_fill_kernel(void* dst, int64_t n, uint64_t key, uint64_t offset, double stdv,
                                  int dtype) {
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    double z = synth_mul(synth_normal(key, offset + (uint64_t)i), stdv);
    float f = synth_to_f32(z);
    if (dtype == SYNTH_BF16) {
      static_cast<uint16_t*>(dst)[i] = synth_f32_to_bf16(f);
    } else {
      static_cast<float*>(dst)[i] = f;
    }
  }
}

}  // namespace

extern "C" {

// Device counterpart of synth_fill_host: dst is a device pointer, the fill is asynchronous on
// `stream` (a cudaStream_t, 0 = legacy default stream).  Returns 0, -1 on a bad argument, or
// the cudaError_t of the launch.
int synth_fill_cuda(void* dst, int64_t n, uint64_t seed, uint64_t tensor_id, uint64_t offset,
                    double stdv, int dtype, void* stream) {
  if (n < 0 || (n > 0 && dst == nullptr) || (dtype != SYNTH_BF16 && dtype != SYNTH_F32)) return -1;
  if (n == 0) return 0;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (n + 255) / 256;
  int64_t cap = (int64_t)sms * 16;
  if (blocks > cap) blocks = cap;
  synth_fill_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(dst, n, synth_key(seed, tensor_id),
                                                                     offset, stdv, dtype);
  return (int)cudaGetLastError();
}

}  // extern "C"
