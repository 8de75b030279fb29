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
unsigned int read_wait_timeouts();
// Persistent direct-load variants for n = 4096 / 8192.
cudaError_t rows_direct_quant(int logn, int dt_in, int bits, const RowArgs& a, cudaStream_t st);
cudaError_t rows_direct_store(int logn, int dt_in, int dt_out, const RowArgs& a, cudaStream_t st);
}  // namespace hit
