// The QJL matrix S generated on the device from the quantizer seed
// (TurboQuant article 2.3.2), entry by entry with the counter-based
// generator of tq_rng.cuh: the numbers the host set-up stores.
#include <algorithm>

#include "tq_kernels.h"
#include "tq_sm100.cuh"
#include "tq_rng.cuh"

namespace tq {

namespace {

__global__ void __launch_bounds__(256) k_qjl_matrix(uint64_t key, int64_t count, uint16_t *s16) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x)
    s16[i] = qjl_entry_f16(key, (uint64_t)i);
}

}  // namespace

tq_status qjl_matrix_launch(uint64_t key, int64_t count, uint16_t *s16, cudaStream_t st) {
  if (count <= 0) return TQ_OK;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t blocks = std::min<int64_t>((count + 255) / 256, (int64_t)sms * 8);
  k_qjl_matrix<<<(unsigned)blocks, 256, 0, st>>>(key, count, s16);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

}  // namespace tq
