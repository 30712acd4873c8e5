// Tensor-core (tcgen05 / TMEM / TMA) chunked prefill for bf16 io.
#include "dn_common.cuh"

namespace dn {

bool chunk_tc_supported(const Args& a) {
  (void)a;
  return false;
}

cudaError_t launch_chunk_tc(const Args& a, cudaStream_t s) {
  (void)a;
  (void)s;
  return cudaErrorNotSupported;
}

}  // namespace dn
