// Mixed-radix butterfly passes on the tensor cores (tcgen05, sm_100a).
//
// HARP explainer, technical summary §2.1: a stage applies a block-diagonal
// orthogonal matrix to coordinate groups separated by a stride; a run of
// consecutive stages mixes only the positions of a "window" -- the positions
// that differ in the run's digits.  Restricted to a window, the run is one
// dense P x P matrix (the product of the stages' blocks), different for every
// window because the blocks are per group.  A pass is then, per window, a
// dense matrix product over a batch (rows or columns):
//   row pass (axis 1, window = P contiguous columns):
//     Y[r, w0 + p'] = sum_p X[r, w0 + p] M_w[p', p]        D = X_tile M_w^T
//   column pass (axis 0, window = P rows at stride S):
//     Y[row(w, p'), c] = sum_p M_w[p', p] X[row(w, p), c]  D = M_w X_tile
// which is what the 5th-generation tensor cores compute: bf16 operands staged
// in shared memory by TMA (128-byte swizzle), fp32 accumulation in tensor
// memory, one thread issuing the MMAs.  The window matrices are composed on
// the device from the fp32 blocks (compose kernel below) and rounded to bf16
// once; data between passes is bf16.
//
// One CTA computes one 128 x N tile with the whole K (<= 256) in shared memory:
// TMA loads of the data tile and of the window matrix land on one mbarrier,
// the K/16 MMAs accumulate in tensor memory, a commit arrives on a second
// mbarrier, and four warps read the accumulator rows (one row per thread) and
// store them with 16/32-byte stores.  Several CTAs per SM overlap one
// another's loads, MMAs and stores.  Every wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "device.cuh"
#include "internal.h"

namespace hit {

__device__ unsigned int g_wait_timeouts_tc = 0;

namespace {

// ---------------------------------------------------------------------------
// Compose: Mat[w][p'][p] = pass operator restricted to window w, as bf16.
// Window w holds positions base(w) + p * step (p < Pw), base(w) =
// (w / step) * Pw * step + (w % step).  Column p of the matrix is the pass
// applied to the unit vector at position p, computed in fp32 in shared memory
// (CC columns per CTA, ping-pong buffers).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t fdiv_u32(uint32_t n, const FastDiv& f) {
  return (__umulhi(n, f.mul) + n) >> f.shr;
}

template <int CC>
__global__ void __launch_bounds__(256) k_bfly_compose(const TcComposeArgs a, __nv_bfloat16* __restrict__ mats) {
  extern __shared__ float cbuf[];  // [2][CC][Pw]
  const int Pw = a.Pw;
  const uint32_t w = blockIdx.x;
  const int j0 = blockIdx.y * CC;
  float* v = cbuf;
  float* u = cbuf + CC * Pw;
  const uint32_t step = uint32_t(a.step);
  const uint32_t base = (w / step) * uint32_t(Pw) * step + (w % step);
  for (int i = threadIdx.x; i < CC * Pw; i += blockDim.x) {
    const int j = i / Pw, q = i - j * Pw;
    v[i] = (q == j0 + j) ? 1.0f : 0.0f;
  }
  __syncthreads();
  for (int t = 0; t < a.ns; ++t) {
    const TcStage& st = a.st[t];
    const uint32_t S = uint32_t(st.stride);
    const int b = st.b;
    const int sw = int(S / step);  // the digit stride in window positions
    // every column of the chunk shares the position q: the block and the digit
    // are found once per position, then applied to the CC columns
    for (int q = threadIdx.x; q < Pw; q += blockDim.x) {
      const uint32_t g = base + uint32_t(q) * step;  // global position (< 2^31)
      const uint32_t q1 = fdiv_u32(g, st.div_s);     // g / S
      const uint32_t lo = g - q1 * S;                // g % S
      const uint32_t hi = fdiv_u32(q1, st.div_b);    // g / (b S)
      const int dig = int(q1 - hi * uint32_t(b));    // (g / S) % b
      const uint64_t c = st.shared_block ? 0 : uint64_t(hi) * S + lo;
      const float* blk = st.blocks + c * uint64_t(b) * uint64_t(b);
      const int q0 = q - dig * sw;
      float acc[CC];
#pragma unroll
      for (int j = 0; j < CC; ++j) acc[j] = 0.0f;
      if (b <= 16) {
        // the block row's coefficients are all loaded before the first use
        float mk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          mk[k] = k < b ? (st.transpose ? __ldg(blk + k * b + dig) : __ldg(blk + dig * b + k)) : 0.0f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          if (k < b) {
#pragma unroll
            for (int j = 0; j < CC; ++j) acc[j] = fmaf(mk[k], v[j * Pw + q0 + k * sw], acc[j]);
          }
        }
      } else {
        for (int k = 0; k < b; ++k) {
          const float mk = st.transpose ? __ldg(blk + k * b + dig) : __ldg(blk + dig * b + k);
#pragma unroll
          for (int j = 0; j < CC; ++j) acc[j] = fmaf(mk, v[j * Pw + q0 + k * sw], acc[j]);
        }
      }
#pragma unroll
      for (int j = 0; j < CC; ++j) u[j * Pw + q] = acc[j];
    }
    __syncthreads();
    float* tmp = v;
    v = u;
    u = tmp;
  }
  // row q, columns j0 .. j0 + CC - 1 of the window's matrix: one thread per
  // row reads its column of the buffer (consecutive lanes, consecutive words)
  // and writes the CC values as 16-byte pieces
  __nv_bfloat16* out = mats + uint64_t(w) * uint64_t(Pw) * Pw;
  for (int q = threadIdx.x; q < Pw; q += blockDim.x) {
    uint4* dst = reinterpret_cast<uint4*>(out + uint64_t(q) * Pw + j0);
#pragma unroll
    for (int c = 0; c < CC / 8; ++c) {
      uint32_t p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 8 * c + 2 * e;
        p[e] = f32_to_bf16x2(v[j * Pw + q], v[(j + 1) * Pw + q]);
      }
      dst[c] = make_uint4(p[0], p[1], p[2], p[3]);
    }
  }
}

// ---------------------------------------------------------------------------
// tcgen05 / TMA helpers (inline PTX).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];" ::
          "r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), sm_100
// descriptor version 1; addresses and offsets in 16-byte units.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= uint64_t((addr >> 4) & 0x3fff);
  d |= uint64_t((lbo_bytes >> 4) & 0x3fff) << 16;
  d |= uint64_t((sbo_bytes >> 4) & 0x3fff) << 32;
  d |= uint64_t(1) << 46;  // descriptor version
  d |= uint64_t(2) << 61;  // 128-byte swizzle
  return d;
}

// AND of a predicate over the 128 threads of warps 0-3 (named barrier 1).
__device__ __forceinline__ bool bar_and_128(bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(uint32_t(v ? 1 : 0))
      : "memory");
  return out != 0;
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(a_mn_major) << 15) | (uint32_t(b_mn_major) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// The pass kernel: persistent and warp-specialized.  COLS = 0: row pass
// (A = data tile [128 rows x K], K-major; B = window matrix [N = Pw x K],
// K-major).  COLS = 1: column pass (A = window matrix rows [128 x K], K-major;
// B = data tile [K positions x N columns], MN-major).  Tout: float or bf16.
//
// Each CTA owns a contiguous range of tiles, ordered so that consecutive tiles
// share their window matrix.  Warp 4 (one lane) streams the data tiles into a
// ring of NS shared-memory stages with TMA and reloads the window matrix only
// when the window changes; warp 5 (one lane) issues the K/16 MMAs of a tile
// into one of two tensor-memory accumulators and commits them to barriers that
// free the data stage, hand the accumulator to the epilogue and (after the
// window's last tile) free the matrix; warps 0-3 read an accumulator (warp w
// owns tensor-memory lanes 32w..32w+31, one output row per thread), store it,
// and hand it back, so the stores of tile i overlap the loads and MMAs of the
// tiles after it.
// ---------------------------------------------------------------------------
struct TcBars {
  uint64_t full[8], empty[8];  // data stages
  uint64_t mfull, mempty;      // window matrix
  uint64_t afull[2], aempty[2];  // accumulators
  uint64_t mdone;              // final drain of the MMAs
  long long issued;            // data tiles whose copies were issued
  int mat_loads;               // window matrices whose copies were issued
  uint32_t tmem;
  int abort;
};

template <int COLS, typename Tout>
__global__ void __launch_bounds__(192, 1) k_bfly_tc(const __grid_constant__ CUtensorMap map_x,
                                                    const __grid_constant__ CUtensorMap map_m,
                                                    const __grid_constant__ CUtensorMap map_y, const TcPassArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int K = a.K, N = a.N, NS = a.stages;
  uint8_t* smat = smem;                                   // window matrix (A for COLS 1, B for COLS 0)
  uint8_t* sdat = smem + size_t(a.bytes_mat);             // NS data stages
  uint8_t* sout = sdat + size_t(NS) * a.bytes_stage;       // two output tiles (TMA store sources)
  TcBars* bars = reinterpret_cast<TcBars*>(sout + size_t(a.out_bufs) * a.bytes_out);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // contiguous tile range of this CTA.  A column pass whose window spans two
  // 128-row halves gives the halves to neighbouring CTAs (half = block index
  // mod m_halves) that walk the same (window, column tile) sequence in step,
  // so each data tile is read from DRAM once and from L2 by the other half.
  const bool split = COLS == 1 && a.m_halves > 1;
  const int mh = split ? int(blockIdx.x % unsigned(a.m_halves)) : 0;
  const int64_t T = split ? a.tiles / a.m_halves : a.tiles;
  const int64_t G = split ? int64_t(gridDim.x / unsigned(a.m_halves)) : int64_t(gridDim.x);
  const int64_t bidx = split ? int64_t(blockIdx.x / unsigned(a.m_halves)) : int64_t(blockIdx.x);
  const int64_t t_begin = bidx < G ? bidx * T / G : T, t_end = bidx < G ? (bidx + 1) * T / G : T;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->mfull, 1);
    mbar_init(&bars->mempty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->afull[b], 1);
      mbar_init(&bars->aempty[b], 4);
    }
    mbar_init(&bars->mdone, 1);
    bars->abort = 0;
    bars->issued = 0;
    bars->mat_loads = 0;
    mbar_init_fence();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&bars->tmem)),
                 "r"(uint32_t(a.tmem_cols))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = bars->tmem;
  volatile int* abort = &bars->abort;

  auto decode = [&](int64_t t, int64_t& w, int& half, int64_t& t0) {
    const int64_t key = t / a.tiles_per_key, r = t % a.tiles_per_key;
    if (COLS == 0) {
      w = key;
      half = 0;
      t0 = r * 128;
    } else if (split) {
      w = key;
      half = mh;
      t0 = r * N;
    } else {
      w = key / a.m_halves;
      half = int(key % a.m_halves);
      t0 = r * N;
    }
  };

  if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int64_t cur = -1;
      int ver = 0;
      for (int64_t t = t_begin; t < t_end && !*abort; ++t) {
        int64_t w, t0;
        int half;
        decode(t, w, half, t0);
        const int64_t key = t / a.tiles_per_key;
        if (key != cur) {
          if (ver > 0 && !mbar_wait(&bars->mempty, uint32_t(ver - 1) & 1u)) {
            atomicAdd(&g_wait_timeouts_tc, 1u);
            *abort = 1;
            break;
          }
          mbar_expect_tx(&bars->mfull, uint32_t(a.bytes_mat));
          for (int j = 0; j < K / 64; ++j) {
            if (COLS == 0)
              tma_load_2d(smat + size_t(j) * N * 128, &map_m, 64 * j, int(w * a.Pw), &bars->mfull);
            else
              tma_load_2d(smat + size_t(j) * 128 * 128, &map_m, 64 * j, int(w * a.Pw + 128 * half), &bars->mfull);
          }
          ++ver;
          bars->mat_loads = ver;
          cur = key;
        }
        const int64_t i = t - t_begin;
        const int s = int(i % NS);
        const int64_t round = i / NS;
        if (round > 0 && !mbar_wait(&bars->empty[s], uint32_t(round - 1) & 1u)) {
          atomicAdd(&g_wait_timeouts_tc, 1u);
          *abort = 1;
          break;
        }
        uint8_t* st = sdat + size_t(s) * a.bytes_stage;
        mbar_expect_tx(&bars->full[s], uint32_t(a.bytes_stage));
        if (COLS == 0) {
          for (int j = 0; j < K / 64; ++j)
            tma_load_2d(st + size_t(j) * 128 * 128, &map_x, int(w * a.Pw + 64 * j), int(t0), &bars->full[s]);
        } else {
          const int lo = int(w % a.step), hi = int(w / a.step);
          for (int j = 0; j < N / 64; ++j)
            tma_load_4d(st + size_t(j) * K * 128, &map_x, int(t0 + 64 * j), 0, lo, hi, &bars->full[s]);
        }
        bars->issued = i + 1;
      }
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, N, 0, COLS);
      const uint32_t m0 = smem_u32(smat);
      int64_t cur = -1;
      int ver = 0;
      for (int64_t t = t_begin; t < t_end && !*abort; ++t) {
        const int64_t key = t / a.tiles_per_key;
        const int64_t i = t - t_begin;
        const int s = int(i % NS);
        const int64_t round = i / NS;
        const int ab = int(i & 1);
        const int64_t around = i >> 1;
        bool ok = true;
        if (key != cur) {
          ok = mbar_wait(&bars->mfull, uint32_t(ver) & 1u);
          ++ver;
          cur = key;
        }
        ok = ok && mbar_wait(&bars->full[s], uint32_t(round) & 1u);
        ok = ok && (around == 0 || mbar_wait(&bars->aempty[ab], uint32_t(around - 1) & 1u));
        if (!ok) {
          atomicAdd(&g_wait_timeouts_tc, 1u);
          *abort = 1;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t d0 = smem_u32(sdat + size_t(s) * a.bytes_stage);
        const uint32_t acc = tmem + uint32_t(ab * N);
        for (int k = 0; k < K / 16; ++k) {
          const int j = k >> 2, kk = k & 3;
          uint64_t ad, bd;
          if (COLS == 0) {
            ad = smem_desc_sw128(d0 + uint32_t(j) * 128 * 128 + 32 * kk, 16, 1024);        // data, K-major
            bd = smem_desc_sw128(m0 + uint32_t(j) * uint32_t(N) * 128 + 32 * kk, 16, 1024);  // matrix, K-major
          } else {
            ad = smem_desc_sw128(m0 + uint32_t(j) * 128 * 128 + 32 * kk, 16, 1024);        // matrix, K-major
            bd = smem_desc_sw128(d0 + uint32_t(k) * 16 * 128, uint32_t(K) * 128, 1024);     // data, MN-major
          }
          mma_bf16(acc, ad, bd, idesc, k > 0 ? 1u : 0u);
        }
        mma_commit(&bars->empty[s]);
        mma_commit(&bars->afull[ab]);
        const bool last_of_key = (t + 1 >= t_end) || ((t + 1) / a.tiles_per_key != key);
        if (last_of_key) mma_commit(&bars->mempty);
      }
      // every MMA issued above has completed before tensor memory is released
      mma_commit(&bars->mdone);
      if (!mbar_wait(&bars->mdone, 0u)) atomicAdd(&g_wait_timeouts_tc, 1u);
    }
  } else {
    // ---------------- epilogue: warps 0-3 ----------------
    // The accumulator row of this thread goes to a shared-memory copy of the
    // output tile laid out as the output tensor map's boxes (128 rows x 128
    // bytes, 128-byte swizzle); one thread then writes the whole tile with
    // TMA stores, so global writes are whole lines.  Two tile buffers: the
    // stores of tile i drain while tile i + 1 is staged.
    constexpr int ES = int(sizeof(Tout));
    constexpr int BOXC = 128 / ES;  // output columns per box
    const int r = 32 * warp + lane;  // accumulator row = row of the output box
    for (int64_t t = t_begin; t < t_end; ++t) {
      int64_t w, t0;
      int half;
      decode(t, w, half, t0);
      const int64_t i = t - t_begin;
      const int ab = int(i & 1);
      const int64_t around = i >> 1;
      bool ok = !*abort;
      if (ok && !mbar_wait(&bars->afull[ab], uint32_t(around) & 1u)) {
        ok = false;
        if (lane == 0) atomicAdd(&g_wait_timeouts_tc, 1u);
      }
      // the staging buffer of tile i - 2 must have been read by its stores
      // (with one staging buffer: the previous tile's)
      if (threadIdx.x == 0 && i >= a.out_bufs) {
        if (a.out_bufs == 2) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        else asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      }
      // one decision for the four warps (they meet at named barriers below)
      if (!bar_and_128(ok)) {
        *abort = 1;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      uint8_t* ob = sout + size_t(a.out_bufs == 2 ? ab : 0) * a.bytes_out;
      for (int c = 0; c < N / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + (uint32_t(32 * warp) << 16) + uint32_t(ab * N + 32 * c), v);
        // columns 32 c .. 32 c + 31: box (32 c) / BOXC, byte offset (32 c * ES) % 128 in its row
        const int col0 = 32 * c;
        uint8_t* rowp = ob + size_t(col0 / BOXC) * (128 * 128) + size_t(r) * 128;
        const int chunk0 = ((col0 % BOXC) * ES) / 16;
        if constexpr (ES == 4) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<uint4*>(rowp + 16 * ((chunk0 + q) ^ (r & 7))) =
                make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(rowp + 16 * ((chunk0 + q) ^ (r & 7))) =
                make_uint4(f32_to_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                           f32_to_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                           f32_to_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                           f32_to_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
        }
      }
      // the accumulator is free once its loads are done
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->aempty[ab]);
      // make the staged tile visible to the TMA engine, then store it
      fence_proxy_async_smem();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (threadIdx.x == 0) {
        for (int j = 0; j < N / BOXC; ++j) {
          const uint32_t src = smem_u32(ob + size_t(j) * (128 * 128));
          if (COLS == 0) {
            asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(&map_y),
                         "r"(int(w * a.Pw + BOXC * j)), "r"(int(t0)), "r"(src)
                         : "memory");
          } else {
            const int lo = int(w % a.step), hi = int(w / a.step);
            asm volatile(
                "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%1, %2, %3, %4}], [%5];" ::"l"(&map_y),
                "r"(int(t0 + BOXC * j)), "r"(128 * half), "r"(lo), "r"(hi), "r"(src)
                : "memory");
          }
        }
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }
    }
    // every store has finished reading shared memory (and completed) before exit
    if (threadIdx.x == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 4 * 32 && *abort) {
    // drain: every stage and matrix copy this CTA issued has landed before
    // its shared memory is released
    const int64_t n = bars->issued;
    for (int s = 0; s < NS && s < n; ++s) {
      const int64_t last_round = (n - 1 - s) / NS;
      if (!mbar_wait(&bars->full[s], uint32_t(last_round) & 1u)) atomicAdd(&g_wait_timeouts_tc, 1u);
    }
    const int v = bars->mat_loads;
    if (v > 0 && !mbar_wait(&bars->mfull, uint32_t(v - 1) & 1u)) atomicAdd(&g_wait_timeouts_tc, 1u);
  }
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(uint32_t(a.tmem_cols))
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// Host: tensor maps through the driver entry point (no link-time libcuda).
// ---------------------------------------------------------------------------
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
  static std::atomic<EncodeTiled> fn{nullptr};
  EncodeTiled f = fn.load();
  if (f == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    f = reinterpret_cast<EncodeTiled>(p);
    fn.store(f);
  }
  return f;
}

// bf16 (or fp32) tensor map, dims / strides in elements (dim 0 contiguous), 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int rank, const int64_t* dims, const int64_t* strides_el,
              const uint32_t* box, int esize = 2, bool swizzle = true) {
  EncodeTiled f = encode_fn();
  if (f == nullptr) return false;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bd[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = cuuint64_t(dims[i]);
    bd[i] = box[i];
    es[i] = 1;
    if (i > 0) gs[i - 1] = cuuint64_t(strides_el[i]) * cuuint64_t(esize);
  }
  const CUtensorMapDataType dt = esize == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return f(m, dt, cuuint32_t(rank), const_cast<void*>(base), gd, gs, bd, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Opt the kernel into the device's whole per-block shared memory (minus its
// static part) once per device, so every later launch of any size fits.
template <typename K>
cudaError_t smem_attr_once(K kernel, size_t smem, std::atomic<unsigned long long>& done_mask) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done_mask.load() & bit) return cudaSuccess;
  int optin = 0;
  if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  cudaFuncAttributes fa;
  if ((e = cudaFuncGetAttributes(&fa, kernel)) != cudaSuccess) return e;
  const int dyn = optin - int(fa.sharedSizeBytes);
  if (size_t(dyn) < smem) return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
  if (e == cudaSuccess) done_mask.fetch_or(bit);
  return e;
}

template <int COLS, typename Tout>
cudaError_t launch_tc(const CUtensorMap& mx, const CUtensorMap& mm, const CUtensorMap& my, const TcPassArgs& a,
                      size_t smem, cudaStream_t st) {
  static std::atomic<unsigned long long> done{0};
  auto kern = k_bfly_tc<COLS, Tout>;
  cudaError_t e = smem_attr_once(kern, smem, done);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 192, smem)) != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  // tensor memory: 512 columns per SM shared by the resident CTAs
  const int by_tmem = 512 / a.tmem_cols;
  per_sm = per_sm < by_tmem ? per_sm : by_tmem;
  int64_t grid = int64_t(sms) * per_sm;
  grid = grid < a.tiles ? grid : a.tiles;
  // column passes over two-half windows pair their CTAs (see the kernel)
  if (COLS == 1 && a.m_halves > 1) grid -= grid % a.m_halves;
  kern<<<dim3(unsigned(grid)), 192, smem, st>>>(mx, mm, my, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bfly_compose(const TcComposeArgs& a, int64_t n_windows, __nv_bfloat16* mats, cudaStream_t st) {
  // 64 columns per CTA up to 128-position windows, 32 for 256 (64 KB of
  // buffers either way); 16 for windows narrower than 64
  static std::atomic<unsigned long long> done16{0}, done32{0}, done64{0};
  const int threads = a.Pw >= 256 ? 256 : ((a.Pw + 31) / 32) * 32;
  cudaError_t e;
  if (a.Pw % 64 == 0 && a.Pw <= 128) {
    const size_t smem = size_t(2) * 64 * a.Pw * sizeof(float);
    if ((e = smem_attr_once(k_bfly_compose<64>, smem, done64)) != cudaSuccess) return e;
    k_bfly_compose<64><<<dim3(unsigned(n_windows), unsigned(a.Pw / 64)), threads, smem, st>>>(a, mats);
  } else if (a.Pw % 32 == 0) {
    const size_t smem = size_t(2) * 32 * a.Pw * sizeof(float);
    if ((e = smem_attr_once(k_bfly_compose<32>, smem, done32)) != cudaSuccess) return e;
    k_bfly_compose<32><<<dim3(unsigned(n_windows), unsigned(a.Pw / 32)), threads, smem, st>>>(a, mats);
  } else {
    const size_t smem = size_t(2) * 16 * a.Pw * sizeof(float);
    if ((e = smem_attr_once(k_bfly_compose<16>, smem, done16)) != cudaSuccess) return e;
    k_bfly_compose<16><<<dim3(unsigned(n_windows), unsigned(a.Pw / 16)), threads, smem, st>>>(a, mats);
  }
  return cudaGetLastError();
}

// x: bf16 data [.., ldx]; mats: bf16 [n_windows * Pw, Pw]; y: [.., ldy] (dt_out).
cudaError_t launch_bfly_tc(const TcPassArgs& args, const void* x, int64_t ldx, const __nv_bfloat16* mats, int dt_out,
                           cudaStream_t st) {
  TcPassArgs a = args;
  CUtensorMap mx, mm, my;
  const int K = a.K;
  const int eo = dt_out == DT_F32 ? 4 : 2;
  const uint32_t boxc = uint32_t(128 / eo);  // output columns per 128-byte box row
  if (K % 64 != 0 || K > 256 || a.N % 64 != 0 || a.N > 256) return cudaErrorInvalidValue;
  if (a.cols == 0) {
    // data [outer rows, L columns], box 64 columns x 128 rows
    const int64_t dx[2] = {a.L, a.outer}, sx[2] = {1, ldx};
    const uint32_t bx[2] = {64, 128};
    if (!make_map(&mx, x, 2, dx, sx, bx)) return cudaErrorInvalidValue;
    // matrices [n_windows * Pw rows, Pw columns], box 64 x N (the window's output rows)
    const int64_t dm[2] = {a.Pw, int64_t(a.n_windows) * a.Pw}, sm[2] = {1, a.Pw};
    const uint32_t bm[2] = {64, uint32_t(a.N)};
    if (!make_map(&mm, mats, 2, dm, sm, bm)) return cudaErrorInvalidValue;
    // output [outer rows, L columns], box 128 bytes x 128 rows
    const int64_t dy[2] = {a.L, a.outer}, sy[2] = {1, a.ldy};
    const uint32_t by[2] = {boxc, 128};
    if (!make_map(&my, a.y, 2, dy, sy, by, eo)) return cudaErrorInvalidValue;
    a.bytes_stage = 128 * K * 2;
    a.bytes_mat = a.N * K * 2;
    a.tiles_per_key = (a.outer + 127) / 128;
    a.tiles = int64_t(a.n_windows) * a.tiles_per_key;
  } else {
    // data [L rows, ncols columns] as (column, p, lo, hi): row = hi * Pw * step + p * step + lo
    const int64_t dx[4] = {a.ncols, a.Pw, a.step, a.L / (int64_t(a.Pw) * a.step)};
    const int64_t sx[4] = {1, a.step * ldx, ldx, int64_t(a.Pw) * a.step * ldx};
    const uint32_t bx[4] = {64, uint32_t(K), 1, 1};
    if (!make_map(&mx, x, 4, dx, sx, bx)) return cudaErrorInvalidValue;
    const int64_t dm[2] = {a.Pw, int64_t(a.n_windows) * a.Pw}, sm[2] = {1, a.Pw};
    const uint32_t bm[2] = {64, 128};
    if (!make_map(&mm, mats, 2, dm, sm, bm)) return cudaErrorInvalidValue;
    // output the same view of y, box 128 bytes x 128 window positions
    const int64_t sy[4] = {1, a.step * a.ldy, a.ldy, int64_t(a.Pw) * a.step * a.ldy};
    const uint32_t by[4] = {boxc, 128, 1, 1};
    if (!make_map(&my, a.y, 4, dx, sy, by, eo)) return cudaErrorInvalidValue;
    a.bytes_stage = a.N * K * 2;
    a.bytes_mat = 128 * K * 2;
    a.tiles_per_key = (a.ncols + a.N - 1) / a.N;
    a.tiles = int64_t(a.n_windows) * a.m_halves * a.tiles_per_key;
  }
  a.bytes_out = 128 * a.N * eo;
  a.tmem_cols = 2 * a.N <= 64 ? 64 : (2 * a.N <= 128 ? 128 : (2 * a.N <= 256 ? 256 : 512));
  // one CTA per SM: the window matrix, two output tiles and as many data
  // stages as fit (at most six); one output tile when two would leave fewer
  // than two data stages
  const size_t whole = 226 * 1024;
  size_t fixed = 0;
  int ns = 0;
  for (int ob = 2; ob >= 1; --ob) {
    fixed = 1024 + size_t(a.bytes_mat) + size_t(ob) * size_t(a.bytes_out) + 512;
    ns = fixed < whole ? int((whole - fixed) / size_t(a.bytes_stage)) : 0;
    a.out_bufs = ob;
    if (ns >= 2) break;
  }
  ns = ns > 6 ? 6 : ns;
  if (ns < 1) return cudaErrorInvalidValue;
  a.stages = ns;
  const size_t smem = fixed + size_t(ns) * a.bytes_stage;
  if (a.cols == 0)
    return dt_out == DT_F32 ? launch_tc<0, float>(mx, mm, my, a, smem, st)
                            : launch_tc<0, __nv_bfloat16>(mx, mm, my, a, smem, st);
  return dt_out == DT_F32 ? launch_tc<1, float>(mx, mm, my, a, smem, st)
                          : launch_tc<1, __nv_bfloat16>(mx, mm, my, a, smem, st);
}

bool make_tensor_map(CUtensorMap* m, const void* base, int rank, const int64_t* dims, const int64_t* strides_el,
                     const uint32_t* box, int esize, bool swizzle) {
  return make_map(m, base, rank, dims, strides_el, box, esize, swizzle);
}

cudaError_t wait_timeouts_tc(unsigned long long* count, bool reset) {
  unsigned int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_wait_timeouts_tc, sizeof v);
  if (e != cudaSuccess) return e;
  *count += v;
  if (reset && v != 0) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_wait_timeouts_tc, &zero, sizeof zero);
  }
  return e;
}

}  // namespace hit
