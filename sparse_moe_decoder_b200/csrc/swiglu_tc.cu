// Grouped SwiGLU on the 5th-generation tensor cores (tcgen05 / TMEM / TMA) for prefill-size
// batches.  Not built yet: reports itself unsupported, so every bf16 shape takes the
// weight-streaming path.
#include "common.cuh"

namespace zmoe {

bool grouped_swiglu_tc_supported(int, int) { return false; }

size_t grouped_swiglu_tc_workspace(int, int, int, int) { return 0; }

zmoe_status grouped_swiglu_tc(const uint16_t*, const int32_t*, int, const uint16_t*, const uint16_t*,
                              const uint16_t*, int, int, int, uint16_t*, float*, void*, size_t, cudaStream_t) {
  return fail(ZMOE_ERR_UNSUPPORTED, "grouped_swiglu (tcgen05): not built");
}

}  // namespace zmoe
