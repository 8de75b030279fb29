// Per-translation-unit row-kernel entry points (compiled in parallel).
#pragma once
#include "internal.h"

namespace hit {
cudaError_t rows_store_from_f32(int logn, int dt_out, const RowArgs& a, cudaStream_t st);
cudaError_t rows_store_from_bf16(int logn, int dt_out, const RowArgs& a, cudaStream_t st);
cudaError_t rows_quant_b2(int logn, int dt_in, const RowArgs& a, cudaStream_t st);
cudaError_t rows_quant_b3(int logn, int dt_in, const RowArgs& a, cudaStream_t st);
cudaError_t rows_quant_b4(int logn, int dt_in, const RowArgs& a, cudaStream_t st);
cudaError_t rows_dequant_b2(int logn, int dt_out, const RowArgs& a, cudaStream_t st);
cudaError_t rows_dequant_b3(int logn, int dt_out, const RowArgs& a, cudaStream_t st);
cudaError_t rows_dequant_b4(int logn, int dt_out, const RowArgs& a, cudaStream_t st);
cudaError_t rows_sparse_all(int logn, int mode, const RowArgs& a, cudaStream_t st);
// Persistent TMA-fed variants for n = 4096 / 8192.
cudaError_t rows_stream_quant(int logn, int dt_in, int bits, const RowArgs& a, cudaStream_t st);
cudaError_t rows_stream_store(int logn, int dt_in, int dt_out, const RowArgs& a, cudaStream_t st);
// Bounded-wait timeouts counted on the current device (added to *count; reset
// clears the counter), and a kernel whose one wait runs out after limit_ns.
cudaError_t wait_timeouts_stream(unsigned long long* count, bool reset);
cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t st);
// Fused d = 5120 (radices 8, 8, 8, 5, 2) transform + 4-bit quantization in
// groups of 128; g5 = the host's 5 x 5 mixer (row-major), and its own
// bounded-wait counter.
cudaError_t rows_mixed5120_quant(const float* x, int64_t rows, int64_t ldx, const int8_t* signs, const float* g5,
                                 uint8_t* codes, float* scales, cudaStream_t st);
cudaError_t wait_timeouts_mixed(unsigned long long* count, bool reset);
// Persistent direct-load variants for n = 4096 / 8192.
cudaError_t rows_direct_quant(int logn, int dt_in, int bits, const RowArgs& a, cudaStream_t st);
cudaError_t rows_direct_store(int logn, int dt_in, int dt_out, const RowArgs& a, cudaStream_t st);
}  // namespace hit
