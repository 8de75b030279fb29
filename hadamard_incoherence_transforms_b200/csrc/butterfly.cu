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

// One fp32 element global -> shared without passing through registers, so a
// thread can have all of its tile loads in flight at once.
__device__ __forceinline__ void cp_async4(float* smem, const float* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}

// Offset, inside a tile row, of the first position of local group g of a
// stage with radix b (the group's positions follow at stride ls << log_nl).
__device__ __forceinline__ int group_offset(int g, int b, const BflyStage& st, int log_nl, int nlm) {
  const int mp = g >> log_nl, l = g & nlm;
  const int mh = int(fdiv(uint32_t(mp), st.div_ls)), ml = mp - mh * st.ls;
  return ((mh * b * st.ls + ml) << log_nl) + l;
}

// A stage of fixed radix B: a thread takes R rows of one group (rows rq,
// rq + NB/R, ...) and streams the B inputs: per input k it loads its R input
// values and the block's row k (the coefficients of all B outputs, one
// 16-byte broadcast per four outputs) and updates R x B accumulators with
// packed FMAs, so every coefficient loaded feeds R rows.  Items own disjoint
// (row, position) sets and read all their inputs before writing, so the stage
// runs in place.
template <int B, int R>
__device__ __forceinline__ void stage_fixed(float* tile, const float* sblk, const BflyStage& st, int groups,
                                            int log_nb, int pitch, int log_nl, int nlm) {
  constexpr int BP = (B + 3) / 4 * 4;
  constexpr int LR = R == 4 ? 2 : (R == 2 ? 1 : 0);
  const int log_nbr = log_nb - LR;
  const int nbr = 1 << log_nbr;
  const int items = groups << log_nbr;
  const int step = st.ls << log_nl;
  for (int it = threadIdx.x; it < items; it += blockDim.x) {
    const int rq = it & (nbr - 1);
    const int g = it >> log_nbr;
    const int off = group_offset(g, B, st, log_nl, nlm);
    int rows[R];  // tile offsets of the item's rows
#pragma unroll
    for (int r = 0; r < R; ++r) rows[r] = (rq + r * nbr) * pitch + off;
    const float4* blk = reinterpret_cast<const float4*>(sblk + st.sofs + (st.shared_block ? 0 : g * B * BP));
    float acc[R][BP];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int j = 0; j < BP; ++j) acc[r][j] = 0.0f;
#pragma unroll
    for (int k = 0; k < B; ++k) {
      float xk[R];
#pragma unroll
      for (int r = 0; r < R; ++r) xk[r] = tile[rows[r] + k * step];
#pragma unroll
      for (int j4 = 0; j4 < BP / 4; ++j4) {
        const float4 w = blk[(k * BP >> 2) + j4];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          fma_x2(w.x, w.y, xk[r], xk[r], acc[r][4 * j4], acc[r][4 * j4 + 1], acc[r][4 * j4], acc[r][4 * j4 + 1]);
          fma_x2(w.z, w.w, xk[r], xk[r], acc[r][4 * j4 + 2], acc[r][4 * j4 + 3], acc[r][4 * j4 + 2],
                 acc[r][4 * j4 + 3]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int j = 0; j < B; ++j) tile[rows[r] + j * step] = acc[r][j];
  }
}

// Any radix b <= BM: one thread per (row, group) item, all b accumulators in
// registers.
template <int BM>
__device__ __forceinline__ void stage_generic(float* tile, const float* sblk, const BflyStage& st, int groups,
                                              int log_nb, int pitch, int log_nl, int nlm) {
  const int b = st.b, bp = st.bp;
  const int items = groups << log_nb;
  const int nbm = (1 << log_nb) - 1;
  const int step = st.ls << log_nl;
  for (int it = threadIdx.x; it < items; it += blockDim.x) {
    const int bi = it & nbm;
    const int g = it >> log_nb;
    float* row = tile + bi * pitch + group_offset(g, b, st, log_nl, nlm);
    float v[BM];
#pragma unroll
    for (int k = 0; k < BM; ++k) v[k] = k < b ? row[k * step] : 0.0f;
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
      if (j < b) row[j * step] = acc[j];
  }
}

template <int BM, int B>
__device__ __forceinline__ bool try_fixed(float* tile, const float* sblk, const BflyStage& st, int groups, int log_nb,
                                          int pitch, int log_nl, int nlm) {
  // four rows per thread (two for radix 16, whose 64 accumulators would not
  // leave room for two CTAs per SM)
  constexpr int R = B >= 16 ? 2 : 4;
  if constexpr (B <= BM) {
    if (st.b == B && log_nb >= (R == 4 ? 2 : 1)) {
      stage_fixed<B, R>(tile, sblk, st, groups, log_nb, pitch, log_nl, nlm);
      return true;
    }
  }
  return false;
}

template <int BM, typename Tin, typename Tout>
__global__ void __launch_bounds__(256, 2) k_bfly_pass(const BflyPass p) {  // launched with 256 threads, up to two CTAs per SM
  extern __shared__ float4 bf_smem4[];
  float* sblk = reinterpret_cast<float*>(bf_smem4);  // per stage: [group][k][bp] (bp >= b, zero padded)
  float* tile = sblk + p.blk_floats;                  // [NB][pitch]
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, nwarps = blockDim.x >> 5;
  const int64_t tiles_lo = p.S_in >> p.log_nl;
  const int64_t tile_id = int64_t(blockIdx.x) % p.n_tiles;
  const int64_t split = int64_t(blockIdx.x) / p.n_tiles;
  const int64_t hi = tile_id / tiles_lo;
  const int64_t lo0 = (tile_id % tiles_lo) << p.log_nl;
  const int64_t base = hi * p.P * p.S_in + lo0;  // position of (mid = 0, l = 0)
  const int PNL = p.P << p.log_nl;
  const int nlm = p.NL - 1;

  // 1. this tile's blocks -> shared memory, laid out so that for a fixed input
  //    index k the b output coefficients are contiguous: row k holds
  //    B[j][k] (forward) or B[k][j] (transpose) for j = 0 .. b-1.  One warp
  //    per group.
  for (int s = 0; s < p.ns; ++s) {
    const BflyStage& st = p.st[s];
    const int b = st.b, bp = st.bp, kjn = b * bp;
    const int groups = st.shared_block ? 1 : (p.P / b) << p.log_nl;
    float* dst = sblk + st.sofs;
    for (int g = warp; g < groups; g += nwarps) {
      const float* src_blk = st.blocks;
      if (!st.shared_block) {
        const int mp = g >> p.log_nl, l = g & nlm;
        src_blk += (hi * (p.P / b) * p.S_in + int64_t(mp) * p.S_in + lo0 + l) * int64_t(b) * b;
      }
      for (int kj = lane; kj < kjn; kj += 32) {
        const int k = int(fdiv(uint32_t(kj), st.div_bp)), j = kj - k * bp;
        dst[g * kjn + kj] = j < b ? __ldg(src_blk + (st.transpose ? k * b + j : j * b + k)) : 0.0f;
      }
    }
  }

  const Tin* src = static_cast<const Tin*>(p.x);
  Tout* out = static_cast<Tout*>(p.y);
  // Fixed per-thread share of the tile for loads and stores.  Along rows
  // (axis 1) a thread keeps position q and walks rows bi, bi + R0, ...;
  // along columns (axis 0) the lanes walk consecutive columns bi (contiguous
  // in memory) and the warps take positions.
  const int QS = PNL < int(blockDim.x) ? PNL : int(blockDim.x);
  const int R0 = int(blockDim.x) / QS;
  const int qi = tid % QS, ri = tid / QS;
  const int BS = p.NB < 32 ? p.NB : 32;
  const int bl = tid % BS, qw0 = tid / BS, QW = int(blockDim.x) / BS;

  const int64_t chunk0 = split * p.chunks_per_split;
  for (int64_t ch = chunk0; ch < chunk0 + p.chunks_per_split; ++ch) {
    const int64_t o0 = ch << p.log_nb;  // first row (axis 1) / column (axis 0) of this chunk
    if (o0 >= p.outer) break;
    const int nb = int(p.outer - o0 < p.NB ? p.outer - o0 : p.NB);
    __syncthreads();  // blocks ready / previous chunk stored
    // 2. load the tile
    if constexpr (std::is_same<Tin, float>::value) {
      // fp32 input: every element of the tile is an asynchronous copy
      if (p.axis == 1) {
        if (ri < R0) {
          for (int q = qi; q < PNL; q += QS) {
            const int64_t coff = base + int64_t(q >> p.log_nl) * p.S_in + (q & nlm);
            const float* sp = src + (o0 + ri) * p.ldx + coff;
            float* tp = tile + ri * p.pitch + q;
            const int64_t sstep = int64_t(R0) * p.ldx;
            const int tstep = R0 * p.pitch;
            for (int bi = ri; bi < nb; bi += R0) {
              cp_async4(tp, sp);
              sp += sstep;
              tp += tstep;
            }
          }
        }
      } else {
        for (int q = qw0; q < PNL; q += QW) {
          const int64_t r = base + int64_t(q >> p.log_nl) * p.S_in + (q & nlm);
          const float* sp = src + r * p.ldx + o0;
          for (int bi = bl; bi < nb; bi += BS) cp_async4(tile + bi * p.pitch + q, sp + bi);
        }
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    } else if (p.axis == 1) {
      if (ri < R0) {
        for (int q = qi; q < PNL; q += QS) {
          const int64_t coff = base + int64_t(q >> p.log_nl) * p.S_in + (q & nlm);
          const Tin* sp = src + (o0 + ri) * p.ldx + coff;
          float* tp = tile + ri * p.pitch + q;
          const int64_t sstep = int64_t(R0) * p.ldx;
          const int tstep = R0 * p.pitch;
          int bi = ri;
          for (; bi + 7 * R0 < nb; bi += 8 * R0) {  // eight loads in flight
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              v[u] = to_f32(__ldcs(sp));
              sp += sstep;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) tp[u * tstep] = v[u];
            tp += 8 * tstep;
          }
          for (; bi < nb; bi += R0) {
            *tp = to_f32(__ldcs(sp));
            sp += sstep;
            tp += tstep;
          }
        }
      }
    } else {
      for (int q = qw0; q < PNL; q += QW) {
        const int64_t r = base + int64_t(q >> p.log_nl) * p.S_in + (q & nlm);
        const Tin* sp = src + r * p.ldx + o0;
        int bi = bl;
        for (; bi + 7 * BS < nb; bi += 8 * BS) {  // eight loads in flight
          float v[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) v[u] = to_f32(__ldcs(sp + bi + u * BS));
#pragma unroll
          for (int u = 0; u < 8; ++u) tile[(bi + u * BS) * p.pitch + q] = v[u];
        }
        for (; bi < nb; bi += BS) tile[bi * p.pitch + q] = to_f32(__ldcs(sp + bi));
      }
    }
    __syncthreads();
    // 3. the stages, in application order
    for (int s = 0; s < p.ns; ++s) {
      const BflyStage& st = p.st[s];
      const int groups = (p.P / st.b) << p.log_nl;
      if (!(try_fixed<BM, 16>(tile, sblk, st, groups, p.log_nb, p.pitch, p.log_nl, nlm) ||
            try_fixed<BM, 8>(tile, sblk, st, groups, p.log_nb, p.pitch, p.log_nl, nlm) ||
            try_fixed<BM, 7>(tile, sblk, st, groups, p.log_nb, p.pitch, p.log_nl, nlm) ||
            try_fixed<BM, 4>(tile, sblk, st, groups, p.log_nb, p.pitch, p.log_nl, nlm) ||
            try_fixed<BM, 2>(tile, sblk, st, groups, p.log_nb, p.pitch, p.log_nl, nlm)))
        stage_generic<BM>(tile, sblk, st, groups, p.log_nb, p.pitch, p.log_nl, nlm);
      __syncthreads();
    }
    // 4. store the tile
    if (p.axis == 1) {
      if (ri < R0) {
        for (int q = qi; q < PNL; q += QS) {
          const int64_t coff = base + int64_t(q >> p.log_nl) * p.S_in + (q & nlm);
          Tout* dp = out + (o0 + ri) * p.ldy + coff;
          const float* tp = tile + ri * p.pitch + q;
          const int64_t dstep = int64_t(R0) * p.ldy;
          const int tstep = R0 * p.pitch;
          for (int bi = ri; bi < nb; bi += R0) {
            __stcs(dp, from_f32<Tout>(*tp));
            dp += dstep;
            tp += tstep;
          }
        }
      }
    } else {
      for (int q = qw0; q < PNL; q += QW) {
        const int64_t r = base + int64_t(q >> p.log_nl) * p.S_in + (q & nlm);
        Tout* dp = out + r * p.ldy + o0;
        for (int bi = bl; bi < nb; bi += BS) __stcs(dp + bi, from_f32<Tout>(tile[bi * p.pitch + q]));
      }
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
