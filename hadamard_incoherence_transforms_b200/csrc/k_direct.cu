// Persistent direct-load row kernels for n = 8192 (see rows_direct.cuh).
#include "kernels.h"
#include "rows_direct.cuh"

namespace hit {

template <typename Tin>
static cudaError_t quant_bits(int bits, const RowArgs& a, cudaStream_t st) {
  if (bits == 4) return launch_direct<13, Tin, float, EPI_QUANT, 4, 8, 1>(a, st);
  if (bits == 3) return launch_direct<13, Tin, float, EPI_QUANT, 3, 8, 1>(a, st);
  return launch_direct<13, Tin, float, EPI_QUANT, 2, 8, 1>(a, st);
}

cudaError_t rows_direct_quant(int logn, int dt_in, int bits, const RowArgs& a, cudaStream_t st) {
  if (logn != 13) return cudaErrorInvalidValue;
  return dt_in == DT_F32 ? quant_bits<float>(bits, a, st) : quant_bits<__nv_bfloat16>(bits, a, st);
}

template <typename Tin, typename Tout>
static cudaError_t store_logn(int logn, const RowArgs& a, cudaStream_t st) {
  return launch_direct<13, Tin, Tout, EPI_STORE, 0, 8, 1>(a, st);
}

cudaError_t rows_direct_store(int logn, int dt_in, int dt_out, const RowArgs& a, cudaStream_t st) {
  if (logn != 13) return cudaErrorInvalidValue;
  if (dt_in == DT_F32)
    return dt_out == DT_F32 ? store_logn<float, float>(logn, a, st) : store_logn<float, __nv_bfloat16>(logn, a, st);
  return dt_out == DT_F32 ? store_logn<__nv_bfloat16, float>(logn, a, st)
                          : store_logn<__nv_bfloat16, __nv_bfloat16>(logn, a, st);
}

}  // namespace hit
