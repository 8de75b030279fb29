// Column (axis 0) Walsh-Hadamard transform passes.
//
// Transforming every column of an [m, cols] row-major matrix is the same
// product of log2(m) butterfly stages, now on the bits of the row index.  One
// pass handles up to 7 consecutive row bits [lo, lo + nb): a thread owns one
// column and the 2^nb rows base + k * 2^lo (k = 0 .. 2^nb - 1), holds them in
// registers and runs the nb stages there.  A warp covers 32 consecutive
// columns, so every register load / store is one 128-byte (fp32) or 64-byte
// (bf16) coalesced row segment.  A transform of length m = 2^k takes
// ceil(k / 7) passes; the first pass applies the signs on load (forward), the
// last applies 1/sqrt(m) and, for the inverse, the signs before the store.
// Each thread reads all its elements before writing them and the threads'
// element sets are disjoint, so a pass may run in place.
#include "device.cuh"
#include "internal.h"
#include "rows.cuh"

namespace hit {

template <int NB, typename Tin, typename Tout>
__global__ void __launch_bounds__(128) k_cols_pass(const ColArgs a) {
  constexpr int R = 1 << NB;
  const int64_t colblocks = (a.cols + 127) / 128;
  const int64_t cb = int64_t(blockIdx.x) % colblocks;
  const int64_t bi = int64_t(blockIdx.x) / colblocks;  // which row base
  const int64_t col = cb * 128 + threadIdx.x;
  if (col >= a.cols) return;
  const int64_t lo_mask = (int64_t(1) << a.lo) - 1;
  // base has zero bits in [lo, lo + NB): low part from bi's low bits, the rest shifted up
  const int64_t base = (bi & lo_mask) | ((bi >> a.lo) << (a.lo + NB));
  const int64_t step = int64_t(1) << a.lo;

  const Tin* src = static_cast<const Tin*>(a.x);
  float v[R];
#pragma unroll
  for (int k = 0; k < R; ++k) {
    const int64_t r = base + k * step;
    float f = to_f32(src[r * a.ldx + col]);
    if (a.pre_signs != nullptr && a.pre_signs[r] < 0) f = -f;
    v[k] = f;
  }
  reg_stages<R, 0, NB>(v);
  Tout* dst = static_cast<Tout*>(a.y);
#pragma unroll
  for (int k = 0; k < R; ++k) {
    const int64_t r = base + k * step;
    float f = v[k] * a.norm;
    if (a.post_signs != nullptr && a.post_signs[r] < 0) f = -f;
    dst[r * a.ldy + col] = from_f32<Tout>(f);
  }
}

template <int NB>
static cudaError_t launch_nb(int dt_in, int dt_out, const ColArgs& a, cudaStream_t st) {
  const int64_t colblocks = (a.cols + 127) / 128;
  const int64_t bases = a.m >> NB;
  const int64_t grid = colblocks * bases;
  if (grid <= 0) return cudaSuccess;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const dim3 g(static_cast<unsigned>(grid));
  if (dt_in == DT_F32 && dt_out == DT_F32) k_cols_pass<NB, float, float><<<g, 128, 0, st>>>(a);
  else if (dt_in == DT_F32) k_cols_pass<NB, float, __nv_bfloat16><<<g, 128, 0, st>>>(a);
  else if (dt_out == DT_F32) k_cols_pass<NB, __nv_bfloat16, float><<<g, 128, 0, st>>>(a);
  else k_cols_pass<NB, __nv_bfloat16, __nv_bfloat16><<<g, 128, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_cols_pass(int nb, int dt_in, int dt_out, const ColArgs& a, cudaStream_t st) {
  switch (nb) {
    case 0: return launch_nb<0>(dt_in, dt_out, a, st);
    case 1: return launch_nb<1>(dt_in, dt_out, a, st);
    case 2: return launch_nb<2>(dt_in, dt_out, a, st);
    case 3: return launch_nb<3>(dt_in, dt_out, a, st);
    case 4: return launch_nb<4>(dt_in, dt_out, a, st);
    case 5: return launch_nb<5>(dt_in, dt_out, a, st);
    case 6: return launch_nb<6>(dt_in, dt_out, a, st);
    case 7: return launch_nb<7>(dt_in, dt_out, a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace hit
