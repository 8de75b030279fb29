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

// A bounded wait that gives up bumps g_wait_timeouts (this translation unit's
// copy; every kernel with bounded waits is instantiated here).
cudaError_t wait_timeouts_stream(unsigned long long* count, bool reset) {
  unsigned int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_wait_timeouts, sizeof v);
  if (e != cudaSuccess) return e;
  *count += v;
  if (reset && v != 0) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_wait_timeouts, &zero, sizeof zero);
  }
  return e;
}

// One warp waits, with the given limit, for a phase of an mbarrier that nothing
// ever completes (no arrival, no copy), so the wait runs out and is counted
// exactly like a lost copy completion in the row kernels.  Nothing is in
// flight when the warp leaves.
__global__ void k_wait_selftest(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_init_fence();
  }
  __syncwarp();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0u, limit_ns)) atomicAdd(&g_wait_timeouts, 1u);
}

cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t st) {
  k_wait_selftest<<<1, 32, 0, st>>>(limit_ns);
  return cudaGetLastError();
}

}  // namespace hit
