// Fused d = 5120 randomized transform + 4-bit group quantization (see
// rows_mixed.cuh).
#include "kernels.h"
#include "rows_mixed.cuh"

namespace hit {

cudaError_t rows_mixed5120_quant(const float* x, int64_t rows, int64_t ldx, const int8_t* signs, const float* g5,
                                 uint8_t* codes, float* scales, cudaStream_t st) {
  MixArgs a;
  a.x = x;
  a.rows = rows;
  a.ldx = ldx;
  a.signs = signs;
  for (int i = 0; i < 25; ++i) a.g5[i] = g5[i] * 0.03125f;  // 1/sqrt(1024), exact
  a.codes = codes;
  a.scales = scales;
  return launch_mixed5120_q4(a, st);
}

cudaError_t wait_timeouts_mixed(unsigned long long* count, bool reset) {
  unsigned int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_wait_timeouts_mixed, sizeof v);
  if (e != cudaSuccess) return e;
  *count += v;
  if (reset && v != 0) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_wait_timeouts_mixed, &zero, sizeof zero);
  }
  return e;
}

}  // namespace hit
