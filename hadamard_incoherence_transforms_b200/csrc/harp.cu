// HARP stage blocks from their learnable parameters, on the device.
//
// HARP explainer, technical summary §2.2: every block of a stride stage is a
// learnable orthogonal factor times a fixed base mixer, B_c = Q(theta_c) G_b.
// Q is a Givens rotation for b = 2 and the Cayley map (I - A)^-1 (I + A) of a
// skew-symmetric A for b > 2; all parameters at zero give Q = I, so the
// processor starts exactly at the randomized Hadamard transform.  §2.4: the
// parameters may be stored as int8.
//
// One warp builds one block.  For b > 2 the Cayley solve is Gauss-Jordan
// elimination on [I - A | I + A] with lane j owning column j (2b <= 32
// columns, so b <= 16); no pivoting is needed because the symmetric part of
// I - A is I: every pivot, and every pivot of the later Schur complements, is
// positive.  B = Q G is then formed column by column, lane j holding column j.
// For the first stage of a transform, the sign diagonal of the randomized
// transform can be folded into the blocks: the column k of group c's block
// multiplies input position k * groups + c, so scaling that column by the
// position's sign (exact, +-1) gives R(theta) diag(s) from the stages alone.
#include <cuda_runtime.h>
#include <stdint.h>

#include "hit.h"
#include "internal.h"

namespace hit {
namespace {

struct HarpArgs {
  const float* theta = nullptr;   // [groups, P] fp32, or NULL
  const int8_t* theta_q = nullptr;  // [groups, P] int8, or NULL
  float theta_scale = 1.0f;       // int8 parameters stand for fp32(q) * scale
  int64_t groups = 0;
  const float* mixer = nullptr;   // [b, b] row-major, NULL = Sylvester / sqrt(b)
  const int8_t* signs = nullptr;  // [b * groups] or NULL (first stage only)
  float* blocks = nullptr;        // [groups, b, b] row-major
};

template <int B>
__device__ __forceinline__ float mixer_at(const HarpArgs& a, int k, int j) {
  if (a.mixer != nullptr) return __ldg(a.mixer + k * B + j);
  // normalized Sylvester Hadamard: H[k][j] = (-1)^popcount(k & j), scaled by RN(1/sqrt(b))
  constexpr float INV = B == 1 ? 1.0f
                        : B == 2 ? 0.70710678118654752f
                        : B == 4 ? 0.5f
                        : B == 8 ? 0.35355339059327376f
                                 : 0.25f;
  return (__popc(k & j) & 1) ? -INV : INV;
}

__device__ __forceinline__ float theta_at(const HarpArgs& a, int64_t idx) {
  return a.theta_q != nullptr ? float(a.theta_q[idx]) * a.theta_scale : __ldg(a.theta + idx);
}

template <int B>
__global__ void __launch_bounds__(256) k_harp_blocks(const HarpArgs a) {
  static_assert(B >= 1 && B <= 16, "one warp holds the 2b columns of [I - A | I + A]");
  constexpr int P = B <= 1 ? 0 : (B == 2 ? 1 : B * (B - 1) / 2);
  const int lane = threadIdx.x & 31;
  const int64_t c = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (c >= a.groups) return;  // whole warps leave together
  const int64_t tb = c * P;
  float q[B];  // lane j < B: column j of Q (q[i] = Q[i][j])
  if constexpr (B == 1) {
    q[0] = 1.0f;
  } else if constexpr (B == 2) {
    // Q = [[cos p, -sin p], [sin p, cos p]]: column 0 = (cos, sin), column 1 = (-sin, cos)
    float sn, cs;
    sincosf(theta_at(a, tb), &sn, &cs);
    q[0] = lane == 0 ? cs : -sn;
    q[1] = lane == 0 ? sn : cs;
  } else {
    // col[i] = row i of this lane's column of [I - A | I + A]; lanes 2B..31
    // carry a unit column and read no parameters (they only take part in the
    // full-warp shuffles).
    const bool live = lane < 2 * B;
    const int j = lane < B ? lane : (live ? lane - B : 0);
    const float sgn = lane < B ? -1.0f : 1.0f;
    float col[B];
#pragma unroll
    for (int i = 0; i < B; ++i) {
      float aij = 0.0f;  // A[i][j]: theta on the strict upper triangle, pairs numbered row by row
      if (live && i < j) aij = theta_at(a, tb + i * (2 * B - i - 1) / 2 + (j - i - 1));
      else if (live && i > j) aij = -theta_at(a, tb + j * (2 * B - j - 1) / 2 + (i - j - 1));
      col[i] = (i == j ? 1.0f : 0.0f) + sgn * aij;
    }
#pragma unroll
    for (int p = 0; p < B; ++p) {
      float f[B];  // the pivot column (lane p) before this step
#pragma unroll
      for (int i = 0; i < B; ++i) f[i] = __shfl_sync(0xffffffffu, col[i], p);
      col[p] = col[p] / f[p];
#pragma unroll
      for (int i = 0; i < B; ++i)
        if (i != p) col[i] = fmaf(-f[i], col[p], col[i]);
    }
    // lanes B .. 2B-1 now hold the columns of Q; bring column j to lane j
#pragma unroll
    for (int i = 0; i < B; ++i) q[i] = __shfl_sync(0xffffffffu, col[i], (lane + B) & 31);
  }
  // B_c = Q G: lane j < B forms column j as sum_k Q[:, k] G[k][j]
  float acc[B];
#pragma unroll
  for (int i = 0; i < B; ++i) acc[i] = 0.0f;
#pragma unroll
  for (int k = 0; k < B; ++k) {
    const float gkj = lane < B ? mixer_at<B>(a, k, lane) : 0.0f;
#pragma unroll
    for (int i = 0; i < B; ++i) acc[i] = fmaf(__shfl_sync(0xffffffffu, q[i], k), gkj, acc[i]);
  }
  if (lane < B) {
    if (a.signs != nullptr && a.signs[int64_t(lane) * a.groups + c] < 0) {
#pragma unroll
      for (int i = 0; i < B; ++i) acc[i] = -acc[i];
    }
    float* out = a.blocks + c * (B * B);
#pragma unroll
    for (int i = 0; i < B; ++i) out[i * B + lane] = acc[i];
  }
}

template <int B>
cudaError_t launch(const HarpArgs& a, cudaStream_t st) {
  const int64_t threads = a.groups * 32;
  const unsigned grid = unsigned((threads + 255) / 256);
  k_harp_blocks<B><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_harp(int b, const HarpArgs& a, cudaStream_t st) {
  switch (b) {
    case 1: return launch<1>(a, st);
    case 2: return launch<2>(a, st);
    case 3: return launch<3>(a, st);
    case 4: return launch<4>(a, st);
    case 5: return launch<5>(a, st);
    case 6: return launch<6>(a, st);
    case 7: return launch<7>(a, st);
    case 8: return launch<8>(a, st);
    case 9: return launch<9>(a, st);
    case 10: return launch<10>(a, st);
    case 11: return launch<11>(a, st);
    case 12: return launch<12>(a, st);
    case 13: return launch<13>(a, st);
    case 14: return launch<14>(a, st);
    case 15: return launch<15>(a, st);
    case 16: return launch<16>(a, st);
  }
  return cudaErrorInvalidValue;
}

bool aligned(const void* p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

}  // namespace
}  // namespace hit

extern "C" HIT_API int harp_blocks(const float* theta, const int8_t* theta_q, float theta_scale, int64_t groups, int b,
                                   const float* mixer, const int8_t* signs, float* blocks, void* stream) {
  if (b < 1 || b > 16) {
    hit::set_last_error("harp_blocks: radix must be in [1, 16]");
    return HIT_EUNSUPPORTED;
  }
  if (groups < 0 || groups > (int64_t(1) << 40)) {
    hit::set_last_error("harp_blocks: bad group count");
    return HIT_EINVAL;
  }
  if (groups == 0) return HIT_OK;
  if (blocks == nullptr || !hit::aligned(blocks, 4)) {
    hit::set_last_error("harp_blocks: blocks missing or not 4-byte aligned");
    return blocks == nullptr ? HIT_EINVAL : HIT_EALIGN;
  }
  if (b >= 2 && (theta == nullptr) == (theta_q == nullptr)) {
    hit::set_last_error("harp_blocks: give exactly one of theta (fp32) and theta_q (int8)");
    return HIT_EINVAL;
  }
  if (theta != nullptr && !hit::aligned(theta, 4)) {
    hit::set_last_error("harp_blocks: theta must be 4-byte aligned");
    return HIT_EALIGN;
  }
  const bool pow2 = (b & (b - 1)) == 0;
  if (!pow2 && mixer == nullptr) {
    hit::set_last_error("harp_blocks: a radix that is not a power of two needs its orthogonal mixer");
    return HIT_EINVAL;
  }
  if (mixer != nullptr && !hit::aligned(mixer, 4)) {
    hit::set_last_error("harp_blocks: mixer must be 4-byte aligned");
    return HIT_EALIGN;
  }
  hit::HarpArgs a;
  a.theta = theta_q != nullptr ? nullptr : theta;
  a.theta_q = theta_q;
  a.theta_scale = theta_scale;
  a.groups = groups;
  a.mixer = mixer;
  a.signs = signs;
  a.blocks = blocks;
  const cudaError_t e = hit::launch_harp(b, a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    hit::set_last_error(cudaGetErrorString(e));
    return HIT_ECUDA;
  }
  return HIT_OK;
}
