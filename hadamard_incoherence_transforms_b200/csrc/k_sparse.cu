// Sparse Walsh-Hadamard adapter: scatter + transform (forward) and
// transform + gather (backward) along rows.
#include "kernels.h"
#include "rows_ops.cuh"

namespace hit {
cudaError_t rows_sparse_all(int logn, int mode, const RowArgs& a, cudaStream_t st) {
  switch (logn) {
#define HIT_CASE(L)                                                    \
  case L:                                                              \
    return mode == 0 ? launch_b2a<L, float, PRO_SCATTER, 0>(a, st)     \
                     : launch_a2b<L, float, float, EPI_GATHER, 0>(a, st);
    HIT_CASE(5) HIT_CASE(6) HIT_CASE(7) HIT_CASE(8) HIT_CASE(9) HIT_CASE(10)
    HIT_CASE(11) HIT_CASE(12) HIT_CASE(13) HIT_CASE(14) HIT_CASE(15)
#undef HIT_CASE
  }
  return cudaErrorInvalidValue;
}
}  // namespace hit
