// Fused transform + 3-bit group quantization along rows.
#include "kernels.h"
#include "rows_ops.cuh"

namespace hit {
template <typename Tin>
static cudaError_t dispatch(int logn, const RowArgs& a, cudaStream_t st) {
  switch (logn) {
#define HIT_CASE(L) \
  case L:           \
    return launch_a2b<L, Tin, float, EPI_QUANT, 3>(a, st);
    HIT_CASE(5) HIT_CASE(6) HIT_CASE(7) HIT_CASE(8) HIT_CASE(9) HIT_CASE(10)
    HIT_CASE(11) HIT_CASE(12) HIT_CASE(13) HIT_CASE(14) HIT_CASE(15)
#undef HIT_CASE
  }
  return cudaErrorInvalidValue;
}

cudaError_t rows_quant_b3(int logn, int dt_in, const RowArgs& a, cudaStream_t st) {
  return dt_in == DT_F32 ? dispatch<float>(logn, a, st) : dispatch<__nv_bfloat16>(logn, a, st);
}
}  // namespace hit
