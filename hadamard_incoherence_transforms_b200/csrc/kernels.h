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
}  // namespace hit
