// Persistent TMA-fed row kernels for n = 4096 (see rows_stream.cuh).
#include "kernels.h"
#include "rows_stream.cuh"

namespace hit {

template <typename Tin>
static cudaError_t quant_bits(int bits, const RowArgs& a, cudaStream_t st) {
  if (bits == 4) return launch_stream<12, Tin, float, EPI_QUANT, 4>(a, st);
  if (bits == 3) return launch_stream<12, Tin, float, EPI_QUANT, 3>(a, st);
  return launch_stream<12, Tin, float, EPI_QUANT, 2>(a, st);
}

cudaError_t rows_stream_quant(int logn, int dt_in, int bits, const RowArgs& a, cudaStream_t st) {
  if (logn != 12) return cudaErrorInvalidValue;
  return dt_in == DT_F32 ? quant_bits<float>(bits, a, st) : quant_bits<__nv_bfloat16>(bits, a, st);
}

template <typename Tin, typename Tout>
static cudaError_t store_logn(int logn, const RowArgs& a, cudaStream_t st) {
  return launch_stream<12, Tin, Tout, EPI_STORE, 0>(a, st);
}

cudaError_t rows_stream_store(int logn, int dt_in, int dt_out, const RowArgs& a, cudaStream_t st) {
  if (logn != 12) return cudaErrorInvalidValue;
  if (dt_in == DT_F32) return dt_out == DT_F32 ? store_logn<float, float>(logn, a, st) : store_logn<float, __nv_bfloat16>(logn, a, st);
  return dt_out == DT_F32 ? store_logn<__nv_bfloat16, float>(logn, a, st)
                          : store_logn<__nv_bfloat16, __nv_bfloat16>(logn, a, st);
}

unsigned int read_wait_timeouts() {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_wait_timeouts, sizeof v) != cudaSuccess) return 0xffffffffu;
  return v;
}

}  // namespace hit
