// Chunked KDA prefill on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
// Not yet available: every call is routed to the SIMT kernel.
#include "kda_internal.cuh"

namespace kda {

bool prefill_tc_supported(int dk, int dv, kda_dtype in_dtype) {
  (void)dk;
  (void)dv;
  (void)in_dtype;
  return false;
}

cudaError_t launch_prefill_tc(const PrefillParams &p, kda_dtype in_dtype, kda_dtype out_dtype,
                              cudaStream_t stream) {
  (void)p;
  (void)in_dtype;
  (void)out_dtype;
  (void)stream;
  return cudaErrorNotSupported;
}

}  // namespace kda
