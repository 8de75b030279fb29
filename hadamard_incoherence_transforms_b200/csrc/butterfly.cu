// Mixed-radix stride butterfly passes (HARP explainer, technical summary
// §2.1: each stage applies a block-diagonal orthogonal matrix to coordinate
// groups separated by a stride permutation; §2.4: the stride stages run fused,
// without materialising the permutation).
//
// A transform of length L = b_0 * ... * b_{m-1} has row-major digits with
// strides S_t = prod_{u>t} b_u.  One pass applies a run of consecutive stages
// whose digits [dlo, dhi] form a "group": with P = prod_{t=dlo..dhi} b_t and
// S_in = S_dhi every index is pos = hi * P * S_in + mid * S_in + lo, and the
// run of stages only mixes positions that share (hi, lo).  A CTA owns one tile
// -- a fixed hi and NL consecutive lo values, i.e. P * NL positions -- and
// streams the other dimension (rows for a row transform, columns for a column
// transform) through shared memory NB at a time.  The blocks the tile's groups
// use are loaded into shared memory once per CTA and reused for every row or
// column, so the block traffic is independent of the batch size.
//
// Within a stage, an item is one (row-or-column, group) pair: it reads its b
// inputs into registers and writes its b outputs to the same positions, and
// items are disjoint, so stages run in place on the tile.  Consecutive threads
// take consecutive rows/columns of the same group: block reads are warp
// uniform and the tile pitch is odd, so tile accesses are conflict free.
#include <atomic>

#include "device.cuh"
#include "internal.h"
#include "rows_ops.cuh"

namespace hit {

template <int BM, typename Tin, typename Tout>
__global__ void __launch_bounds__(256) k_bfly_pass(const BflyPass p) {
  extern __shared__ float bf_smem[];
  float* sblk = bf_smem;                 // blocks of every stage of the pass
  float* tile = bf_smem + p.blk_floats;  // [NB][pitch]
  const int tid = threadIdx.x;
  const int64_t tiles_lo = p.S_in / p.NL;
  const int64_t tile_id = int64_t(blockIdx.x) % p.n_tiles;
  const int64_t split = int64_t(blockIdx.x) / p.n_tiles;
  const int64_t hi = tile_id / tiles_lo;
  const int64_t lo0 = (tile_id % tiles_lo) * p.NL;
  const int64_t base = hi * p.P * p.S_in + lo0;  // position of (mid = 0, l = 0)
  const int PNL = p.P * p.NL;

  // 1. this tile's blocks -> shared memory: stage s, local group (m', l)
  for (int s = 0; s < p.ns; ++s) {
    const BflyStage& st = p.st[s];
    const int b = st.b, bb = b * b;
    const int groups = (p.P / b) * p.NL;
    float* dst = sblk + st.sofs;
    if (st.shared_block) {
      for (int i = tid; i < bb; i += blockDim.x) dst[i] = __ldg(st.blocks + i);
    } else {
      for (int i = tid; i < groups * bb; i += blockDim.x) {
        const int g = i / bb, e = i - g * bb;
        const int mp = g / p.NL, l = g - mp * p.NL;
        const int64_t c = hi * (p.P / b) * p.S_in + int64_t(mp) * p.S_in + lo0 + l;
        dst[i] = __ldg(st.blocks + c * bb + e);
      }
    }
  }

  const Tin* src = static_cast<const Tin*>(p.x);
  Tout* out = static_cast<Tout*>(p.y);
  const int64_t chunk0 = split * p.chunks_per_split;
  for (int64_t ch = chunk0; ch < chunk0 + p.chunks_per_split; ++ch) {
    const int64_t o0 = ch * p.NB;  // first row (axis 1) / column (axis 0) of this chunk
    if (o0 >= p.outer) break;
    const int nb = int(p.outer - o0 < p.NB ? p.outer - o0 : p.NB);
    __syncthreads();  // blocks ready / previous chunk stored
    // 2. load the tile
    for (int e = tid; e < p.NB * PNL; e += blockDim.x) {
      int bi, q;
      if (p.axis == 1) {
        bi = e / PNL;
        q = e - bi * PNL;
      } else {
        bi = e % p.NB;
        q = e / p.NB;
      }
      if (bi >= nb) continue;
      const int mid = q / p.NL, l = q - mid * p.NL;
      const int64_t pos = base + int64_t(mid) * p.S_in + l;
      const int64_t g = p.axis == 1 ? (o0 + bi) * p.ldx + pos : pos * p.ldx + (o0 + bi);
      tile[bi * p.pitch + q] = to_f32(src[g]);
    }
    __syncthreads();
    // 3. the stages, in application order
    for (int s = 0; s < p.ns; ++s) {
      const BflyStage& st = p.st[s];
      const int b = st.b;
      const int ls = st.ls;  // stride of this digit inside mid
      const int per = p.P / b;
      const int items = p.NB * per * p.NL;
      for (int it = tid; it < items; it += blockDim.x) {
        const int bi = it % p.NB;
        const int g = it / p.NB;  // (m', l)
        const int mp = g / p.NL, l = g - mp * p.NL;
        const int mh = mp / ls, ml = mp - mh * ls;
        const int mid0 = mh * b * ls + ml;
        float* row = tile + bi * p.pitch + l;
        float v[BM];
#pragma unroll
        for (int k = 0; k < BM; ++k) v[k] = k < b ? row[(mid0 + k * ls) * p.NL] : 0.0f;
        const float* blk = sblk + st.sofs + (st.shared_block ? 0 : g * b * b);
        const int js = st.transpose ? 1 : b, ks = st.transpose ? b : 1;
#pragma unroll 1
        for (int j = 0; j < b; ++j) {
          const float* br = blk + j * js;
          float acc = 0.0f;
#pragma unroll
          for (int k = 0; k < BM; ++k)
            if (k < b) acc = fmaf(br[k * ks], v[k], acc);
          row[(mid0 + j * ls) * p.NL] = acc;
        }
      }
      __syncthreads();
    }
    // 4. store the tile
    for (int e = tid; e < p.NB * PNL; e += blockDim.x) {
      int bi, q;
      if (p.axis == 1) {
        bi = e / PNL;
        q = e - bi * PNL;
      } else {
        bi = e % p.NB;
        q = e / p.NB;
      }
      if (bi >= nb) continue;
      const int mid = q / p.NL, l = q - mid * p.NL;
      const int64_t pos = base + int64_t(mid) * p.S_in + l;
      const int64_t g = p.axis == 1 ? (o0 + bi) * p.ldy + pos : pos * p.ldy + (o0 + bi);
      out[g] = from_f32<Tout>(tile[bi * p.pitch + q]);
    }
  }
}

template <int BM>
static cudaError_t launch_bm(int dt_in, int dt_out, const BflyPass& p, size_t smem, int64_t grid, cudaStream_t st) {
  static std::atomic<unsigned long long> d0{0}, d1{0}, d2{0}, d3{0};
  const dim3 g(static_cast<unsigned>(grid));
  cudaError_t e;
  if (dt_in == DT_F32 && dt_out == DT_F32) {
    if ((e = set_smem_attr(k_bfly_pass<BM, float, float>, smem, d0)) != cudaSuccess) return e;
    k_bfly_pass<BM, float, float><<<g, 256, smem, st>>>(p);
  } else if (dt_in == DT_F32) {
    if ((e = set_smem_attr(k_bfly_pass<BM, float, __nv_bfloat16>, smem, d1)) != cudaSuccess) return e;
    k_bfly_pass<BM, float, __nv_bfloat16><<<g, 256, smem, st>>>(p);
  } else if (dt_out == DT_F32) {
    if ((e = set_smem_attr(k_bfly_pass<BM, __nv_bfloat16, float>, smem, d2)) != cudaSuccess) return e;
    k_bfly_pass<BM, __nv_bfloat16, float><<<g, 256, smem, st>>>(p);
  } else {
    if ((e = set_smem_attr(k_bfly_pass<BM, __nv_bfloat16, __nv_bfloat16>, smem, d3)) != cudaSuccess) return e;
    k_bfly_pass<BM, __nv_bfloat16, __nv_bfloat16><<<g, 256, smem, st>>>(p);
  }
  return cudaGetLastError();
}

cudaError_t launch_butterfly_pass(int dt_in, int dt_out, const BflyPass& p, cudaStream_t st) {
  int bmax = 1;
  for (int s = 0; s < p.ns; ++s) bmax = p.st[s].b > bmax ? p.st[s].b : bmax;
  const size_t smem = (size_t(p.blk_floats) + size_t(p.NB) * p.pitch) * sizeof(float);
  const int64_t splits = (p.outer + p.NB * p.chunks_per_split - 1) / (p.NB * p.chunks_per_split);
  const int64_t grid = p.n_tiles * splits;
  if (grid <= 0) return cudaSuccess;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (bmax <= 8) return launch_bm<8>(dt_in, dt_out, p, smem, grid, st);
  if (bmax <= 16) return launch_bm<16>(dt_in, dt_out, p, smem, grid, st);
  if (bmax <= 32) return launch_bm<32>(dt_in, dt_out, p, smem, grid, st);
  return launch_bm<64>(dt_in, dt_out, p, smem, grid, st);
}

}  // namespace hit
