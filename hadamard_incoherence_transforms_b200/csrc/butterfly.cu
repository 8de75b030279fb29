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

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  return (__umulhi(n, f.mul) + n) >> f.shr;
}

template <int BM, typename Tin, typename Tout>
__global__ void __launch_bounds__(256, 2) k_bfly_pass(const BflyPass p) {  // launched with 256 threads, up to two CTAs per SM
  extern __shared__ float4 bf_smem4[];
  float* sblk = reinterpret_cast<float*>(bf_smem4);  // per stage: [group][k][bp] (bp >= b, zero padded)
  float* tile = sblk + p.blk_floats;                  // [NB][pitch]
  const int tid = threadIdx.x;
  const int64_t tiles_lo = p.S_in >> p.log_nl;
  const int64_t tile_id = int64_t(blockIdx.x) % p.n_tiles;
  const int64_t split = int64_t(blockIdx.x) / p.n_tiles;
  const int64_t hi = tile_id / tiles_lo;
  const int64_t lo0 = (tile_id % tiles_lo) << p.log_nl;
  const int64_t base = hi * p.P * p.S_in + lo0;  // position of (mid = 0, l = 0)
  const int PNL = p.P << p.log_nl;
  const int nlm = p.NL - 1, nbm = p.NB - 1;

  // 1. this tile's blocks -> shared memory, laid out so that for a fixed input
  //    index k the b output coefficients are contiguous: row k holds
  //    B[j][k] (forward) or B[k][j] (transpose) for j = 0 .. b-1.
  for (int s = 0; s < p.ns; ++s) {
    const BflyStage& st = p.st[s];
    const int b = st.b, bb = b * b, bp = st.bp;
    const int groups = st.shared_block ? 1 : (p.P / b) << p.log_nl;
    float* dst = sblk + st.sofs;
    for (int i = tid; i < groups * b * bp; i += blockDim.x) {
      const int g = i / (b * bp), r = i - g * (b * bp);
      const int k = r / bp, j = r - k * bp;
      float v = 0.0f;
      if (j < b) {
        int64_t c = 0;
        if (!st.shared_block) {
          const int mp = g >> p.log_nl, l = g & nlm;
          c = hi * (p.P / b) * p.S_in + int64_t(mp) * p.S_in + lo0 + l;
        }
        v = __ldg(st.blocks + c * bb + (st.transpose ? k * b + j : j * b + k));
      }
      dst[i] = v;
    }
  }

  const Tin* src = static_cast<const Tin*>(p.x);
  Tout* out = static_cast<Tout*>(p.y);
  const int64_t chunk0 = split * p.chunks_per_split;
  for (int64_t ch = chunk0; ch < chunk0 + p.chunks_per_split; ++ch) {
    const int64_t o0 = ch << p.log_nb;  // first row (axis 1) / column (axis 0) of this chunk
    if (o0 >= p.outer) break;
    const int nb = int(p.outer - o0 < p.NB ? p.outer - o0 : p.NB);
    __syncthreads();  // blocks ready / previous chunk stored
    // 2. load the tile (consecutive threads: consecutive memory),
    //    sixteen independent loads in flight per thread before they land in shared memory
    constexpr int U = 16;
    const int total = PNL << p.log_nb;
    for (int e0 = tid; e0 < total; e0 += U * blockDim.x) {
      float val[U];
      int dst[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int e = e0 + u * blockDim.x;
        dst[u] = -1;
        val[u] = 0.0f;
        if (e < total) {
          int bi, q;
          if (p.axis == 1) {
            bi = int(fdiv(uint32_t(e), p.div_pnl));
            q = e - bi * PNL;
          } else {
            bi = e & nbm;
            q = e >> p.log_nb;
          }
          if (bi < nb) {
            const int64_t pos = base + int64_t(q >> p.log_nl) * p.S_in + (q & nlm);
            const int64_t g = p.axis == 1 ? (o0 + bi) * p.ldx + pos : pos * p.ldx + (o0 + bi);
            val[u] = to_f32(__ldcs(src + g));
            dst[u] = bi * p.pitch + q;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (dst[u] >= 0) tile[dst[u]] = val[u];
    }
    __syncthreads();
    // 3. the stages, in application order
    for (int s = 0; s < p.ns; ++s) {
      const BflyStage& st = p.st[s];
      const int b = st.b, bp = st.bp, ls = st.ls;
      const int items = ((p.P / b) << p.log_nl) << p.log_nb;
      for (int it = tid; it < items; it += blockDim.x) {
        const int bi = it & nbm;
        const int g = it >> p.log_nb;  // local group (m', l)
        const int mp = g >> p.log_nl, l = g & nlm;
        const int mh = int(fdiv(uint32_t(mp), st.div_ls)), ml = mp - mh * ls;
        const int mid0 = mh * b * ls + ml;
        float* row = tile + bi * p.pitch + l;
        const int step = ls << p.log_nl;
        float v[BM];
#pragma unroll
        for (int k = 0; k < BM; ++k) v[k] = k < b ? row[(mid0 << p.log_nl) + k * step] : 0.0f;
        float acc[BM];
#pragma unroll
        for (int j = 0; j < BM; ++j) acc[j] = 0.0f;
        const float4* blk = reinterpret_cast<const float4*>(sblk + st.sofs + (st.shared_block ? 0 : g * b * bp));
#pragma unroll
        for (int k = 0; k < BM; ++k) {
          if (k < b) {
#pragma unroll
            for (int j4 = 0; j4 < BM / 4; ++j4) {
              if (4 * j4 < bp) {
                const float4 w = blk[(k * bp >> 2) + j4];
                fma_x2(w.x, w.y, v[k], v[k], acc[4 * j4], acc[4 * j4 + 1], acc[4 * j4], acc[4 * j4 + 1]);
                fma_x2(w.z, w.w, v[k], v[k], acc[4 * j4 + 2], acc[4 * j4 + 3], acc[4 * j4 + 2], acc[4 * j4 + 3]);
              }
            }
          }
        }
#pragma unroll
        for (int j = 0; j < BM; ++j)
          if (j < b) row[(mid0 << p.log_nl) + j * step] = acc[j];
      }
      __syncthreads();
    }
    // 4. store the tile
#pragma unroll 4
    for (int e = tid; e < (PNL << p.log_nb); e += blockDim.x) {
      int bi, q;
      if (p.axis == 1) {
        bi = int(fdiv(uint32_t(e), p.div_pnl));
        q = e - bi * PNL;
      } else {
        bi = e & nbm;
        q = e >> p.log_nb;
      }
      if (bi >= nb) continue;
      const int64_t pos = base + int64_t(q >> p.log_nl) * p.S_in + (q & nlm);
      const int64_t g = p.axis == 1 ? (o0 + bi) * p.ldy + pos : pos * p.ldy + (o0 + bi);
      __stcs(out + g, from_f32<Tout>(tile[bi * p.pitch + q]));
    }
  }
}

// The pass's shared-memory size depends on the call, so each kernel is opted
// in to the largest size the planner can ask for, once per device.
constexpr size_t kBflySmemMax = 227 * 1024;

template <int BM>
static cudaError_t launch_bm(int dt_in, int dt_out, const BflyPass& p, size_t smem, int64_t grid, cudaStream_t st) {
  static std::atomic<unsigned long long> d0{0}, d1{0}, d2{0}, d3{0};
  const dim3 g(static_cast<unsigned>(grid));
  if (smem > kBflySmemMax) return cudaErrorInvalidValue;
  cudaError_t e;
  if (dt_in == DT_F32 && dt_out == DT_F32) {
    if ((e = set_smem_attr(k_bfly_pass<BM, float, float>, kBflySmemMax, d0)) != cudaSuccess) return e;
    k_bfly_pass<BM, float, float><<<g, 256, smem, st>>>(p);
  } else if (dt_in == DT_F32) {
    if ((e = set_smem_attr(k_bfly_pass<BM, float, __nv_bfloat16>, kBflySmemMax, d1)) != cudaSuccess) return e;
    k_bfly_pass<BM, float, __nv_bfloat16><<<g, 256, smem, st>>>(p);
  } else if (dt_out == DT_F32) {
    if ((e = set_smem_attr(k_bfly_pass<BM, __nv_bfloat16, float>, kBflySmemMax, d2)) != cudaSuccess) return e;
    k_bfly_pass<BM, __nv_bfloat16, float><<<g, 256, smem, st>>>(p);
  } else {
    if ((e = set_smem_attr(k_bfly_pass<BM, __nv_bfloat16, __nv_bfloat16>, kBflySmemMax, d3)) != cudaSuccess) return e;
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
