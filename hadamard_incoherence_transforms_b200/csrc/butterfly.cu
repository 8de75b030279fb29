// Mixed-radix stride butterfly stages (HARP explainer, technical summary
// §2.1: each stage applies a block-diagonal orthogonal matrix to coordinate
// groups separated by a stride; §2.4: stride stages applied without
// materialising the permutation).
//
// Stage t of a length-L transform with radix b and stride S (the product of
// the later radices): group c = hi * S + lo owns the b elements
// i_k = hi * b * S + k * S + lo (k = 0 .. b-1) and maps them through its own
// b x b block: y_{i_j} = sum_k B_c[j][k] x_{i_k} (B_c^T for the transpose).
// One thread owns one (group, row) pair along rows or one (group, column)
// pair along columns; it loads its b inputs into registers before writing
// any output, and groups are disjoint, so a stage can run in place.  Along
// columns consecutive threads take consecutive columns of the same group, so
// loads are coalesced and the block entries are warp-uniform.
#include "device.cuh"
#include "internal.h"
#include "rows.cuh"

namespace hit {

template <int BM, typename Tin, typename Tout>
__global__ void __launch_bounds__(256) k_bfly_stage(const StageArgs a) {
  const int b = a.b;
  const int64_t groups = a.len / b;
  const int64_t items = groups * a.outer;
  const Tin* src = static_cast<const Tin*>(a.x);
  Tout* dst = static_cast<Tout*>(a.y);
  for (int64_t it = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; it < items;
       it += int64_t(gridDim.x) * blockDim.x) {
    int64_t o, c;
    if (a.axis == 1) {
      c = it % groups;
      o = it / groups;
    } else {
      o = it % a.outer;
      c = it / a.outer;
    }
    const int64_t lo = c % a.stride, hi = c / a.stride;
    const int64_t i0 = hi * b * a.stride + lo;
    const int64_t xs = a.axis == 1 ? a.stride : a.stride * a.ldx;
    const int64_t ys = a.axis == 1 ? a.stride : a.stride * a.ldy;
    const int64_t xb = a.axis == 1 ? o * a.ldx + i0 : i0 * a.ldx + o;
    const int64_t yb = a.axis == 1 ? o * a.ldy + i0 : i0 * a.ldy + o;
    float v[BM];
#pragma unroll
    for (int k = 0; k < BM; ++k) v[k] = k < b ? to_f32(src[xb + k * xs]) : 0.0f;
    const float* blk = a.blocks + (a.shared_block ? 0 : c * int64_t(b) * b);
    const int rs = a.transpose ? 1 : b;  // step between entries of one output
    const int os = a.transpose ? b : 1;  // step between consecutive k
#pragma unroll 1
    for (int j = 0; j < b; ++j) {
      const float* row = blk + j * rs;
      float acc = 0.0f;
#pragma unroll
      for (int k = 0; k < BM; ++k)
        if (k < b) acc = fmaf(__ldg(row + k * os), v[k], acc);
      dst[yb + j * ys] = from_f32<Tout>(acc);
    }
  }
}

template <int BM>
static cudaError_t launch_bm(int dt_in, int dt_out, const StageArgs& a, cudaStream_t st) {
  const int64_t items = (a.len / a.b) * a.outer;
  if (items <= 0) return cudaSuccess;
  int64_t grid = (items + 255) / 256;
  if (grid > 148 * 16) grid = 148 * 16;
  const dim3 g(static_cast<unsigned>(grid));
  if (dt_in == DT_F32 && dt_out == DT_F32) k_bfly_stage<BM, float, float><<<g, 256, 0, st>>>(a);
  else if (dt_in == DT_F32) k_bfly_stage<BM, float, __nv_bfloat16><<<g, 256, 0, st>>>(a);
  else if (dt_out == DT_F32) k_bfly_stage<BM, __nv_bfloat16, float><<<g, 256, 0, st>>>(a);
  else k_bfly_stage<BM, __nv_bfloat16, __nv_bfloat16><<<g, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_butterfly_stage(int dt_in, int dt_out, const StageArgs& a, cudaStream_t st) {
  if (a.b <= 4) return launch_bm<4>(dt_in, dt_out, a, st);
  if (a.b <= 8) return launch_bm<8>(dt_in, dt_out, a, st);
  if (a.b <= 16) return launch_bm<16>(dt_in, dt_out, a, st);
  if (a.b <= 32) return launch_bm<32>(dt_in, dt_out, a, st);
  if (a.b <= 64) return launch_bm<64>(dt_in, dt_out, a, st);
  return cudaErrorInvalidValue;
}

}  // namespace hit
