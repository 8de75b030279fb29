// Internal launcher interface between the C ABI (api.cu) and the kernel
// translation units.  Host-side C++ only; no torch types anywhere.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace hit {

// Arguments of the row kernels (one CUDA thread team per row; the row length
// n = 2^logn is a template parameter of the kernel).
struct RowArgs {
  const void* x = nullptr;  // dense input rows [rows, ldx]
  void* y = nullptr;        // dense output rows [rows, ldy]
  int64_t rows = 0, ldx = 0, ldy = 0;
  const int8_t* pre_signs = nullptr;   // diag(s) applied on load (forward)
  const int8_t* post_signs = nullptr;  // diag(s) applied before the store (inverse)
  float norm = 1.0f;                   // 1/sqrt(n) (or a caller scale)
  // group quantization (output) / dequantization (input)
  uint8_t* codes = nullptr;
  float* scales = nullptr;
  const uint8_t* codes_in = nullptr;
  const float* scales_in = nullptr;
  int log2g = 0;
  // sparse adapter
  const float* sp_values = nullptr;
  const int32_t* sp_cols = nullptr;
  float* sp_out = nullptr;
  int nnz = 0;
  float sp_scale = 1.0f;
};

// Record the message hit_last_error() returns on this host thread.
void set_last_error(const char* msg);

// dtype codes (same values as the C ABI)
enum { DT_F32 = 0, DT_BF16 = 1 };

// y = post(H (pre(x))) * norm along rows, dense in and out.
cudaError_t launch_rows_store(int logn, int dt_in, int dt_out, const RowArgs& a, cudaStream_t st);
// Fused transform + group quantization + packing along rows.
cudaError_t launch_rows_quant(int logn, int dt_in, int bits, const RowArgs& a, cudaStream_t st);
// Dequantization + inverse transform along rows.
cudaError_t launch_rows_dequant(int logn, int dt_out, int bits, const RowArgs& a, cudaStream_t st);
// Sparse adapter: mode 0 scatter + transform, mode 1 transform + gather.
cudaError_t launch_rows_sparse(int logn, int mode, const RowArgs& a, cudaStream_t st);

// Column (axis 0) transform pass over row-index bits [lo, lo + nb), nb <= 7.
struct ColArgs {
  const void* x = nullptr;
  void* y = nullptr;
  int64_t m = 0;      // transform length (number of rows), power of two
  int64_t cols = 0;   // number of columns
  int64_t ldx = 0, ldy = 0;
  int lo = 0;         // first row bit of this pass
  const int8_t* pre_signs = nullptr;
  const int8_t* post_signs = nullptr;
  float norm = 1.0f;  // applied on store when != 1
};
cudaError_t launch_cols_pass(int nb, int dt_in, int dt_out, const ColArgs& a, cudaStream_t st);
// Whole column transform in one pass for 2^8 <= m <= 2^13 (4-column strips;
// needs cols % 4 == 0 and 16-byte (fp32) / 8-byte (bf16) aligned strip rows).
cudaError_t launch_cols_full(int logm, int dt_in, int dt_out, const ColArgs& a, cudaStream_t st);
// Whole column transform for 2^10 <= m <= 2^13 with thread-block clusters of
// m/1024 CTAs (32-column strips; needs cols % 32 == 0, aligned strip rows).
cudaError_t launch_cols_cluster(int logm, int dt_in, int dt_out, const ColArgs& a, cudaStream_t st);

// One pass of mixed-radix butterfly stages over consecutive digits (see
// butterfly.cu for the tiling).
// Unsigned division by a run-time constant d (d >= 1, numerators < 2^31):
// q = (umulhi(n, mul) + n) >> shr.
struct FastDiv {
  uint32_t d = 1, mul = 0, shr = 0;
};
inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  uint32_t s = 0;
  while ((1ull << s) < d) ++s;
  f.shr = s;
  f.mul = static_cast<uint32_t>(((1ull << 32) * ((1ull << s) - d)) / d + 1);
  if (d == 1) f.mul = 0;
  return f;
}
struct BflyStage {
  const float* blocks = nullptr;  // [G, b, b] fp32, or one shared block
  int b = 1;                      // radix
  int bp = 4;                     // b rounded up to a multiple of 4 (shared-memory row length)
  int ls = 1;                     // stride of this digit inside the group index mid
  FastDiv div_ls;                 // division by ls
  FastDiv div_bp;                 // division by bp
  int sofs = 0;                   // float offset of the stage's blocks in shared memory
  int shared_block = 0;
  int transpose = 0;              // use B^T
};
constexpr int kMaxPassStages = 16;
struct BflyPass {
  const void* x = nullptr;
  void* y = nullptr;
  int64_t outer = 0;          // rows (axis 1) or columns (axis 0)
  int64_t ldx = 0, ldy = 0;
  int axis = 1;
  int P = 1;                  // positions per group (product of the pass's radices)
  int64_t S_in = 1;           // stride of the pass's last digit
  int NL = 1;                 // consecutive lo values per tile (power of two)
  int log_nl = 0;
  int NB = 1;                 // rows / columns per chunk (power of two)
  int log_nb = 0;
  FastDiv div_pnl;            // division by P * NL
  int pitch = 1;              // floats per tile row in shared memory (odd)
  int64_t n_tiles = 1;
  int64_t chunks_per_split = 1;
  int blk_floats = 0;
  int ns = 0;
  BflyStage st[kMaxPassStages];
};
cudaError_t launch_butterfly_pass(int dt_in, int dt_out, const BflyPass& p, cudaStream_t st);

// Tensor-core butterfly passes (bfly_tc.cu).  A pass's window holds Pw
// positions base(w) + p * step, base(w) = (w / step) * Pw * step + (w % step);
// its stages are composed into one bf16 Pw x Pw matrix per window.
struct TcStage {
  const float* blocks = nullptr;  // [G, b, b] fp32 (or one shared block)
  int b = 1;
  int64_t stride = 1;             // digit stride S_t of the whole transform
  int shared_block = 0;
  int transpose = 0;              // use B^T
  FastDiv div_s, div_b;           // division by S_t and by b (positions < 2^31)
};
struct TcComposeArgs {
  int Pw = 0;
  int64_t step = 1;
  int ns = 0;
  TcStage st[kMaxPassStages];     // in application order
};
struct TcPassArgs {
  int cols = 0;           // 0: row pass over contiguous windows, 1: column pass
  int Pw = 0, K = 0, N = 0;
  int64_t step = 1;
  int64_t L = 0;          // transform length
  int64_t outer = 0;      // row pass: rows
  int64_t ncols = 0;      // column pass: columns
  int n_windows = 0, m_halves = 1, tmem_cols = 0;
  int bytes_mat = 0, bytes_stage = 0;  // window matrix / one data tile in shared memory
  int bytes_out = 0;                   // one output tile staged for its TMA store
  int out_bufs = 2;                    // output staging buffers (2: a tile's stores drain under the next)
  int stages = 1;                      // data tiles in flight per CTA
  int64_t tiles = 0, tiles_per_key = 1;  // tiles of the pass; consecutive tiles sharing a window matrix
  void* y = nullptr;
  int64_t ldy = 0;
};
cudaError_t launch_bfly_compose(const TcComposeArgs& a, int64_t n_windows, __nv_bfloat16* mats, cudaStream_t st);
cudaError_t launch_bfly_tc(const TcPassArgs& a, const void* x, int64_t ldx, const __nv_bfloat16* mats, int dt_out,
                           cudaStream_t st);
cudaError_t wait_timeouts_tc(unsigned long long* count, bool reset);
// Tiled TMA tensor map (bf16 for esize 2, fp32 for 4), dims and strides in
// elements with dim 0 contiguous, 128-byte swizzle (or a dense box without);
// false if the driver rejects it.
bool make_tensor_map(CUtensorMap* m, const void* base, int rank, const int64_t* dims, const int64_t* strides_el,
                     const uint32_t* box, int esize, bool swizzle);

// Two adjacent digits H (radix bh) and L (radix bl) along rows at a stride s
// (bfly_strided.cu): positions hi * P * s + (iH * bl + iL) * s + lo.
struct StridedArgs {
  const void* x = nullptr;
  void* y = nullptr;
  int64_t ldx = 0, ldy = 0, rows = 0;
  int64_t s = 8;        // stride of digit L (a multiple of 8)
  int64_t n_hi = 1;     // L / (P s)
  const float* blocks_h = nullptr;  // stage on H: [groups, bh, bh]
  const float* blocks_l = nullptr;  // stage on L: [groups, bl, bl]
  int shared_h = 0, shared_l = 0;   // one block for every group
  int transpose = 0;                // transposed blocks
  int h_first = 1;                  // stage on H applied before the stage on L
  int64_t parts = 1;                // CTAs per key (row ranges), set by the launcher
};
// Whether (bh, bl) has a kernel for these element sizes, strides (elements)
// and 16-byte aligned bases.
bool strided_supported(int bh, int bl, int es_in, int es_out);
cudaError_t wait_timeouts_strided(unsigned long long* count, bool reset);
cudaError_t launch_bfly_strided(int bh, int bl, int dt_in, int dt_out, const StridedArgs& a, cudaStream_t st);

}  // namespace hit
