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
#include <cooperative_groups.h>

#include <atomic>

#include "device.cuh"
#include "internal.h"
#include "rows_ops.cuh"

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

// ---------------------------------------------------------------------------
// Single-pass column transform for 2^8 <= m <= 2^13.
//
// A CTA owns complete columns: a strip of 4 adjacent columns per team of
// T = m/32 threads (256 / T strips per CTA, 256 threads).  Every element moves
// as part of a 4-column vector (one 16-byte fp32 / 8-byte bf16 access per
// row), and a thread holds 32 rows x 4 columns = 128 values.  The row index
// bits are processed in windows of five bits from the top: in phase p the
// thread's 32 rows differ in the window's bits (register bits), while its
// thread index supplies the other bits.  Between phases the strip goes
// through shared memory (row r of a strip is 16-byte chunk r, stored at
// r ^ ((r >> 5) & 7)).  The last window is widened down to bit 0 and only runs
// the stages not done yet.  The strip's data crosses HBM exactly once in each
// direction.
// ---------------------------------------------------------------------------
template <int LOGM>
struct ColFull {
  static constexpr int M = 1 << LOGM;
  static constexpr int LOGT = LOGM - 5;
  static constexpr int T = 1 << LOGT;   // threads per strip
  static constexpr int STRIPS = 256 / T; // strips per CTA
  static constexpr int NP = (LOGM + 4) / 5;
  static constexpr size_t SMEM = size_t(256) * 32 * 16;  // 128 KB
};

// window (lowest register bit) of phase P
template <int LOGM, int P>
struct ColWin {
  static constexpr int HI = LOGM - 5 * P;                  // exclusive top of the window
  static constexpr int LO = HI - 5 > 0 ? HI - 5 : 0;       // register window [LO, LO+5)
  static constexpr int STAGE_LO = HI - 5 > 0 ? 0 : LO;     // new stages: window bits below HI
  static constexpr int NSTAGE = HI - LO;                   // bits of the window still to do
};

template <int LOGM, int P>
__device__ __forceinline__ int64_t colfull_row(int t, int k) {
  constexpr int LO = ColWin<LOGM, P>::LO;
  const int low = t & ((1 << LO) - 1);
  const int high = t >> LO;
  return int64_t(low | (k << LO) | (high << (LO + 5)));
}

__device__ __forceinline__ int colfull_chunk(int r) { return r ^ ((r >> 5) & 7); }

template <int LOGM, int P>
__device__ __forceinline__ void colfull_stages(float (&x)[128]) {
  // register index 4k + c; row-window bit q <-> register bit q + 2
  reg_stages<128, 2, 2 + ColWin<LOGM, P>::NSTAGE>(x);
}

template <int LOGM, int P>
__device__ __forceinline__ void colfull_get(const float4* strip, float (&x)[128], int t) {
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const float4 v = strip[colfull_chunk(int(colfull_row<LOGM, P>(t, k)))];
    x[4 * k] = v.x;
    x[4 * k + 1] = v.y;
    x[4 * k + 2] = v.z;
    x[4 * k + 3] = v.w;
  }
}
template <int LOGM, int P>
__device__ __forceinline__ void colfull_put(float4* strip, const float (&x)[128], int t) {
#pragma unroll
  for (int k = 0; k < 32; ++k)
    strip[colfull_chunk(int(colfull_row<LOGM, P>(t, k)))] = make_float4(x[4 * k], x[4 * k + 1], x[4 * k + 2], x[4 * k + 3]);
}

template <int LOGM, typename Tin, typename Tout>
__global__ void __launch_bounds__(256, 1) k_cols_full(const ColArgs a) {
  using F = ColFull<LOGM>;
  extern __shared__ float4 cf_smem[];
  const int tid = threadIdx.x;
  const int strip_in_cta = tid >> F::LOGT;
  const int t = tid & (F::T - 1);
  const int64_t col0 = (int64_t(blockIdx.x) * F::STRIPS + strip_in_cta) * 4;
  const bool active = col0 < a.cols;
  float4* strip = cf_smem + size_t(strip_in_cta) * F::M;
  float x[128];
  if (active) {
    const Tin* src = static_cast<const Tin*>(a.x) + col0;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const int64_t r = colfull_row<LOGM, 0>(t, k);
      float v0, v1, v2, v3;
      if constexpr (std::is_same<Tin, float>::value) {
        const float4 v = __ldcs(reinterpret_cast<const float4*>(src + r * a.ldx));
        v0 = v.x; v1 = v.y; v2 = v.z; v3 = v.w;
      } else {
        const uint2 v = __ldcs(reinterpret_cast<const uint2*>(src + r * a.ldx));
        bf16x2_to_f32(v.x, v0, v1);
        bf16x2_to_f32(v.y, v2, v3);
      }
      if (a.pre_signs != nullptr && a.pre_signs[r] < 0) {
        v0 = -v0; v1 = -v1; v2 = -v2; v3 = -v3;
      }
      x[4 * k] = v0; x[4 * k + 1] = v1; x[4 * k + 2] = v2; x[4 * k + 3] = v3;
    }
    colfull_stages<LOGM, 0>(x);
  }
  if constexpr (F::NP > 1) {
    if (active) colfull_put<LOGM, 0>(strip, x, t);
    __syncthreads();
    if (active) {
      colfull_get<LOGM, 1>(strip, x, t);
      colfull_stages<LOGM, 1>(x);
    }
  }
  if constexpr (F::NP > 2) {
    __syncthreads();  // all phase-1 reads done before the phase-1 writes
    if (active) colfull_put<LOGM, 1>(strip, x, t);
    __syncthreads();
    if (active) {
      colfull_get<LOGM, 2>(strip, x, t);
      colfull_stages<LOGM, 2>(x);
    }
  }
  if (!active) return;
  constexpr int PL = F::NP - 1;
  Tout* dst = static_cast<Tout*>(a.y) + col0;
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const int64_t r = colfull_row<LOGM, PL>(t, k);
    float v0 = x[4 * k] * a.norm, v1 = x[4 * k + 1] * a.norm, v2 = x[4 * k + 2] * a.norm, v3 = x[4 * k + 3] * a.norm;
    if (a.post_signs != nullptr && a.post_signs[r] < 0) {
      v0 = -v0; v1 = -v1; v2 = -v2; v3 = -v3;
    }
    if constexpr (std::is_same<Tout, float>::value) {
      __stcs(reinterpret_cast<float4*>(dst + r * a.ldy), make_float4(v0, v1, v2, v3));
    } else {
      __stcs(reinterpret_cast<uint2*>(dst + r * a.ldy), make_uint2(f32_to_bf16x2(v0, v1), f32_to_bf16x2(v2, v3)));
    }
  }
}

template <int LOGM, typename Tin, typename Tout>
static cudaError_t launch_full_t(const ColArgs& a, cudaStream_t st) {
  using F = ColFull<LOGM>;
  auto kern = k_cols_full<LOGM, Tin, Tout>;
  static std::atomic<unsigned long long> done{0};
  cudaError_t e = set_smem_attr(kern, F::SMEM, done);
  if (e != cudaSuccess) return e;
  const int64_t strips = (a.cols + 3) / 4;
  const int64_t grid = (strips + F::STRIPS - 1) / F::STRIPS;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  kern<<<dim3(unsigned(grid)), 256, F::SMEM, st>>>(a);
  return cudaGetLastError();
}

template <int LOGM>
static cudaError_t launch_full_m(int dt_in, int dt_out, const ColArgs& a, cudaStream_t st) {
  if (dt_in == DT_F32 && dt_out == DT_F32) return launch_full_t<LOGM, float, float>(a, st);
  if (dt_in == DT_F32) return launch_full_t<LOGM, float, __nv_bfloat16>(a, st);
  if (dt_out == DT_F32) return launch_full_t<LOGM, __nv_bfloat16, float>(a, st);
  return launch_full_t<LOGM, __nv_bfloat16, __nv_bfloat16>(a, st);
}

cudaError_t launch_cols_full(int logm, int dt_in, int dt_out, const ColArgs& a, cudaStream_t st) {
  switch (logm) {
    case 8: return launch_full_m<8>(dt_in, dt_out, a, st);
    case 9: return launch_full_m<9>(dt_in, dt_out, a, st);
    case 10: return launch_full_m<10>(dt_in, dt_out, a, st);
    case 11: return launch_full_m<11>(dt_in, dt_out, a, st);
    case 12: return launch_full_m<12>(dt_in, dt_out, a, st);
    case 13: return launch_full_m<13>(dt_in, dt_out, a, st);
  }
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------
// Column transform for 1024 <= m <= 8192 with thread-block clusters.
//
// A cluster of CL = m / 1024 CTAs owns a strip of 16 (bf16 source) or 8 (fp32
// source) adjacent columns over all m rows; CTA c of the cluster holds rows
// [1024 c, 1024 c + 1024) of the strip (64 or 32 KB fp32).  Row segments are
// 32 bytes wide, so global accesses are whole sectors.  Within a CTA a thread owns
// one 4-column quad and 32 rows: first rows tr + 32k (the register bits are
// row bits 5..9), then, after one pass through shared memory, rows
// 32 tr + r (row bits 0..4).  The CL row blocks (row bits 10 and up) are then
// combined through distributed shared memory: each thread reads the CL
// vectors of one (row, quad) position from the cluster's CTAs, runs the
// remaining log2(CL) stages and writes the CL output rows.
//
// The clusters are persistent: cluster i takes strips i, i + clusters, ...,
// and while it transforms and stores one strip its rows of the next strip
// are already streaming into a staging buffer with 16-byte asynchronous
// copies (cp.async), so the loads of one strip overlap the arithmetic,
// exchange and stores of the previous one.
// ---------------------------------------------------------------------------
// Quads (4-column groups) per strip: 4 for bf16 sources (16 columns, 32-byte
// row segments), 2 for fp32 sources (8 columns, 32-byte row segments), so the
// fp32 staging buffer stays small enough for three CTAs per SM.
template <typename Tin>
struct ClusterQuads {
  static constexpr int QD = std::is_same<Tin, float>::value ? 2 : 4;
  static constexpr int LQD = QD == 4 ? 2 : 1;
};
// 16-byte chunk of (row, quad); the bits above the quad index are xor-ed with
// row bits 5.. so that rows 32 apart (the phase-2 pattern) fall in different
// bank groups.
template <int QD>
__device__ __forceinline__ int cs_idx(int row, int q) {
  constexpr int LQD = QD == 4 ? 2 : 1;
  return (row * QD + q) ^ (((row >> 5) & (8 / QD - 1)) << LQD);
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

template <typename Tin>
struct ClusterSmem {
  static constexpr int QD = ClusterQuads<Tin>::QD;
  static constexpr int THREADS = QD * 32;
  static constexpr int SROW = 4 * QD * int(sizeof(Tin));  // staged bytes per row of a strip
  static constexpr size_t WORK = size_t(1024) * QD * sizeof(float4);
  static constexpr size_t SMEM = WORK + size_t(1024) * SROW;
};

template <int CL, typename Tin, typename Tout>
__global__ void __launch_bounds__(ClusterSmem<Tin>::THREADS) k_cols_cluster(const ColArgs a) {
  using SM = ClusterSmem<Tin>;
  constexpr int kQuads = SM::QD;
  constexpr int kClusterThreads = SM::THREADS;
  extern __shared__ float4 cs_smem[];  // [1024 rows][kQuads quads] fp32, then the staging rows
  uint8_t* stage = reinterpret_cast<uint8_t*>(cs_smem) + SM::WORK;
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = static_cast<int>(cluster.block_rank());
  const int64_t clusters = gridDim.x / CL;
  const int64_t strips = a.cols / (4 * kQuads);
  const int tid = threadIdx.x;
  const int q = tid % kQuads;  // column quad within the strip
  const int tr = tid / kQuads;  // 0..31
  const int64_t row_base = int64_t(crank) * 1024;
  constexpr int CPR = SM::SROW / 16;  // 16-byte copies per staged row
  auto prefetch = [&](int64_t strip) {
    const uint8_t* src = static_cast<const uint8_t*>(a.x) + (row_base * a.ldx + strip * 4 * kQuads) * int64_t(sizeof(Tin));
    const int64_t pitch = a.ldx * int64_t(sizeof(Tin));
#pragma unroll 4
    for (int i = tid; i < 1024 * CPR; i += kClusterThreads) {
      const int r = i / CPR, c = i - r * CPR;
      cp_async16(stage + r * SM::SROW + 16 * c, src + r * pitch + 16 * c);
    }
    cp_async_commit();
  };

  int64_t strip = blockIdx.x / CL;
  if (strip < strips) prefetch(strip);
  // Every strip of this CTA uses the same rows, so each thread's signs become
  // two bit masks once: bit k of pre_m is the sign of phase-1 row tr + 32 k,
  // bit 4 u + c of post_m the sign of phase-3 row 1024 c + row_low(u).
  constexpr int SHARE = 1024 / CL;
  uint32_t pre_m = 0, post_m = 0;
  if (a.pre_signs != nullptr) {
#pragma unroll
    for (int k = 0; k < 32; ++k) pre_m |= uint32_t(a.pre_signs[row_base + tr + 32 * k] < 0) << k;
  }
  if (a.post_signs != nullptr) {
#pragma unroll
    for (int u = 0; u < SHARE / 32; ++u)
#pragma unroll
      for (int c = 0; c < CL; ++c)
        post_m |= uint32_t(a.post_signs[int64_t(c) * 1024 + crank * SHARE + tr + 32 * u] < 0) << (u * CL + c);
  }
  bool pending = false;  // this thread arrived on the cluster barrier after a strip's reads
  for (; strip < strips; strip += clusters) {
    cp_async_wait_all();
    __syncthreads();  // every thread's copies of this strip have landed
    float x[128];
    // phase 1: rows tr + 32 k of this CTA's block, from the staging rows
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const int r = tr + 32 * k;
      float v0, v1, v2, v3;
      if constexpr (std::is_same<Tin, float>::value) {
        const float4 v = *reinterpret_cast<const float4*>(stage + r * SM::SROW + 16 * q);
        v0 = v.x; v1 = v.y; v2 = v.z; v3 = v.w;
      } else {
        const uint2 v = *reinterpret_cast<const uint2*>(stage + r * SM::SROW + 8 * q);
        bf16x2_to_f32(v.x, v0, v1);
        bf16x2_to_f32(v.y, v2, v3);
      }
      const uint32_t sb = (pre_m >> k) << 31;
      x[4 * k] = __uint_as_float(__float_as_uint(v0) ^ sb);
      x[4 * k + 1] = __uint_as_float(__float_as_uint(v1) ^ sb);
      x[4 * k + 2] = __uint_as_float(__float_as_uint(v2) ^ sb);
      x[4 * k + 3] = __uint_as_float(__float_as_uint(v3) ^ sb);
    }
    __syncthreads();  // the staging rows are free: start streaming the next strip
    if (strip + clusters < strips) prefetch(strip + clusters);
    reg_stages<128, 2, 7>(x);  // row bits 5..9
    // the cluster's phase-3 reads of this CTA's previous block are done
    if (pending) asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
#pragma unroll
    for (int k = 0; k < 32; ++k)
      cs_smem[cs_idx<kQuads>(tr + 32 * k, q)] = make_float4(x[4 * k], x[4 * k + 1], x[4 * k + 2], x[4 * k + 3]);
    __syncthreads();
    // phase 2: rows 32 tr + r
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      const float4 v = cs_smem[cs_idx<kQuads>(32 * tr + r, q)];
      x[4 * r] = v.x; x[4 * r + 1] = v.y; x[4 * r + 2] = v.z; x[4 * r + 3] = v.w;
    }
    reg_stages<128, 2, 7>(x);  // row bits 0..4
    __syncthreads();           // every phase-2 read is done before the writes
#pragma unroll
    for (int r = 0; r < 32; ++r)
      cs_smem[cs_idx<kQuads>(32 * tr + r, q)] = make_float4(x[4 * r], x[4 * r + 1], x[4 * r + 2], x[4 * r + 3]);
    cluster.sync();  // all blocks of the strip are in shared memory
    // phase 3: this CTA combines rows (c', row_low) for row_low in its share
    Tout* dst = static_cast<Tout*>(a.y) + strip * 4 * kQuads + 4 * q;
    // every remote read of the strip is issued before the first is used
    float vall[SHARE / 32][4 * CL];
#pragma unroll
    for (int u = 0; u < SHARE / 32; ++u) {
      const int row_low = crank * SHARE + tr + 32 * u;
#pragma unroll
      for (int c = 0; c < CL; ++c) {
        const float4* rem = cluster.map_shared_rank(cs_smem, c);
        const float4 w = rem[cs_idx<kQuads>(row_low, q)];
        vall[u][4 * c] = w.x; vall[u][4 * c + 1] = w.y; vall[u][4 * c + 2] = w.z; vall[u][4 * c + 3] = w.w;
      }
    }
    // the remaining stages consume every value read (so the reads have
    // completed) before this CTA releases its hold on the cluster's blocks
    // with a relaxed arrive; the matching wait comes before the next strip's
    // first write to shared memory (or at exit)
    if constexpr (CL > 1) {
#pragma unroll
      for (int u = 0; u < SHARE / 32; ++u) reg_stages<4 * CL, 2, 2 + (CL == 2 ? 1 : (CL == 4 ? 2 : 3))>(vall[u]);
    }
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    pending = true;
#pragma unroll
    for (int u = 0; u < SHARE / 32; ++u) {
      const int row_low = crank * SHARE + tr + 32 * u;
      const float(&v)[4 * CL] = vall[u];
#pragma unroll
      for (int c = 0; c < CL; ++c) {
        const int64_t r = int64_t(c) * 1024 + row_low;
        const float nrm = __uint_as_float(__float_as_uint(a.norm) ^ (((post_m >> (u * CL + c)) & 1u) << 31));
        const float o0 = v[4 * c] * nrm, o1 = v[4 * c + 1] * nrm, o2 = v[4 * c + 2] * nrm, o3 = v[4 * c + 3] * nrm;
        if constexpr (std::is_same<Tout, float>::value) {
          __stcs(reinterpret_cast<float4*>(dst + r * a.ldy), make_float4(o0, o1, o2, o3));
        } else {
          __stcs(reinterpret_cast<uint2*>(dst + r * a.ldy), make_uint2(f32_to_bf16x2(o0, o1), f32_to_bf16x2(o2, o3)));
        }
      }
    }
  }
  // no CTA leaves while others may still read its block
  if (pending) asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  cp_async_wait_all();  // nothing in flight into this CTA's shared memory at exit
}

template <int CL, typename Tin, typename Tout>
static cudaError_t launch_cluster_t(const ColArgs& a, cudaStream_t st) {
  using SM = ClusterSmem<Tin>;
  auto kern = k_cols_cluster<CL, Tin, Tout>;
  static std::atomic<unsigned long long> done{0};
  cudaError_t e = set_smem_attr(kern, SM::SMEM, done);
  if (e != cudaSuccess) return e;
  const int64_t strips = a.cols / (4 * SM::QD);
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(SM::THREADS);
  cfg.dynamicSmemBytes = SM::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // Persistent clusters: as many as can be resident at once (queried once per
  // device), never more than there are strips.
  static std::atomic<int> resident[64];
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  int nres = dev < 64 ? resident[dev].load() : 0;
  if (nres <= 0) {
    cfg.gridDim = dim3(static_cast<unsigned>(CL));
    if ((e = cudaOccupancyMaxActiveClusters(&nres, kern, &cfg)) != cudaSuccess) return e;
    if (nres <= 0) nres = 1;
    if (dev < 64) resident[dev].store(nres);
  }
  const int64_t clusters = strips < nres ? strips : nres;
  cfg.gridDim = dim3(static_cast<unsigned>(clusters * CL));
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int CL>
static cudaError_t launch_cluster_cl(int dt_in, int dt_out, const ColArgs& a, cudaStream_t st) {
  if (dt_in == DT_F32 && dt_out == DT_F32) return launch_cluster_t<CL, float, float>(a, st);
  if (dt_in == DT_F32) return launch_cluster_t<CL, float, __nv_bfloat16>(a, st);
  if (dt_out == DT_F32) return launch_cluster_t<CL, __nv_bfloat16, float>(a, st);
  return launch_cluster_t<CL, __nv_bfloat16, __nv_bfloat16>(a, st);
}

cudaError_t launch_cols_cluster(int logm, int dt_in, int dt_out, const ColArgs& a, cudaStream_t st) {
  if (a.cols % 16 != 0 || a.cols / 8 > 0x7fffffffLL / 8) return cudaErrorInvalidValue;
  switch (logm) {
    case 10: return launch_cluster_cl<1>(dt_in, dt_out, a, st);
    case 11: return launch_cluster_cl<2>(dt_in, dt_out, a, st);
    case 12: return launch_cluster_cl<4>(dt_in, dt_out, a, st);
    case 13: return launch_cluster_cl<8>(dt_in, dt_out, a, st);
  }
  return cudaErrorInvalidValue;
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
