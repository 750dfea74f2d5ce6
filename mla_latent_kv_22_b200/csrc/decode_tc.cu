// Split-KV absorbed-MLA decode on the tcgen05 tensor cores (placeholder until the
// kernel lands: reports the shape unsupported so the mma.sync kernel runs).
#include "mla_device.cuh"
#include "mla_internal.h"

namespace mla {

bool decode_tc_supported(int heads) {
  (void)heads;
  return false;
}

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream) {
  (void)a;
  (void)stream;
  return cudaErrorNotSupported;
}

}  // namespace mla
