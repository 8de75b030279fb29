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
constexpr int kComposeCols = 16;

__global__ void __launch_bounds__(256) k_bfly_compose(const TcComposeArgs a, __nv_bfloat16* __restrict__ mats) {
  extern __shared__ float cbuf[];  // [2][kComposeCols][Pw]
  const int Pw = a.Pw;
  const int64_t w = blockIdx.x;
  const int j0 = blockIdx.y * kComposeCols;
  float* v = cbuf;
  float* u = cbuf + kComposeCols * Pw;
  const int64_t base = (w / a.step) * int64_t(Pw) * a.step + (w % a.step);
  for (int i = threadIdx.x; i < kComposeCols * Pw; i += blockDim.x) {
    const int j = i / Pw, q = i - j * Pw;
    v[i] = (q == j0 + j) ? 1.0f : 0.0f;
  }
  __syncthreads();
  for (int t = 0; t < a.ns; ++t) {
    const TcStage& st = a.st[t];
    const int64_t S = st.stride;           // global digit stride
    const int sw = int(S / a.step);        // the same stride in window positions
    for (int i = threadIdx.x; i < kComposeCols * Pw; i += blockDim.x) {
      const int j = i / Pw, q = i - j * Pw;
      const int64_t g = base + int64_t(q) * a.step;  // global position
      const int64_t hiq = g / (int64_t(st.b) * S);
      const int64_t loq = g % S;
      const int dig = int((g / S) % st.b);
      const int64_t c = st.shared_block ? 0 : hiq * S + loq;
      const float* blk = st.blocks + c * int64_t(st.b) * st.b;
      const float* col = v + j * Pw + (q - dig * sw);
      float acc = 0.0f;
      for (int k = 0; k < st.b; ++k) {
        const float m = st.transpose ? blk[k * st.b + dig] : blk[dig * st.b + k];
        acc = fmaf(m, col[k * sw], acc);
      }
      u[i] = acc;
    }
    __syncthreads();
    float* tmp = v;
    v = u;
    u = tmp;
  }
  // row q, column j0 + j of the window's matrix
  __nv_bfloat16* out = mats + w * int64_t(Pw) * Pw;
  for (int i = threadIdx.x; i < kComposeCols * Pw; i += blockDim.x) {
    const int q = i / kComposeCols, j = i - q * kComposeCols;
    out[int64_t(q) * Pw + j0 + j] = __float2bfloat16_rn(v[j * Pw + q]);
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
// The pass kernel.  COLS = 0: row pass (A = data, K-major; B = window matrix,
// K-major); COLS = 1: column pass (A = window matrix, K-major; B = data,
// MN-major).  Tout: float or bf16.
// ---------------------------------------------------------------------------
template <int COLS, typename Tout>
__global__ void __launch_bounds__(128) k_bfly_tc(const __grid_constant__ CUtensorMap map_x,
                                                 const __grid_constant__ CUtensorMap map_m, const TcPassArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int K = a.K, N = a.N;
  uint8_t* sa = smem;                                   // A operand
  uint8_t* sb = smem + size_t(a.bytes_a);               // B operand
  uint64_t* bars = reinterpret_cast<uint64_t*>(sb + a.bytes_b);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // tile coordinates
  int64_t w, t0;   // window; row tile (COLS 0) or column tile (COLS 1)
  int half = 0;    // COLS 1: which 128 output positions of the window
  if (COLS == 0) {
    w = blockIdx.x % a.n_windows;
    t0 = int64_t(blockIdx.x / a.n_windows) * 128;
  } else {
    const int64_t per = int64_t(a.n_windows) * a.m_halves;
    const int64_t r = blockIdx.x % per;
    w = r / a.m_halves;
    half = int(r % a.m_halves);
    t0 = int64_t(blockIdx.x / per) * N;
  }

  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init_fence();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(uint32_t(a.tmem_cols))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tslot;

  bool ok = true;
  if (threadIdx.x == 0) {
    mbar_expect_tx(&bars[0], uint32_t(a.bytes_a + a.bytes_b));
    const int kb = K / 64;  // 64-element (128-byte) boxes along K
    if (COLS == 0) {
      // A: data rows t0.., columns w*Pw + 64 j; B: window matrix rows w*Pw.., columns 64 j
      for (int j = 0; j < kb; ++j) {
        tma_load_2d(sa + size_t(j) * 128 * 128, &map_x, int(w * a.Pw + 64 * j), int(t0), &bars[0]);
        tma_load_2d(sb + size_t(j) * N * 128, &map_m, 64 * j, int(w * a.Pw), &bars[0]);
      }
    } else {
      // A: window matrix rows w*Pw + 128 half.., columns 64 j;
      // B: data columns t0 + 64 j, positions p (all K of them) of window w
      for (int j = 0; j < kb; ++j)
        tma_load_2d(sa + size_t(j) * 128 * 128, &map_m, 64 * j, int(w * a.Pw + 128 * half), &bars[0]);
      const int lo = int(w % a.step), hi = int(w / a.step);
      for (int j = 0; j < N / 64; ++j)
        tma_load_4d(sb + size_t(j) * K * 128, &map_x, int(t0 + 64 * j), 0, lo, hi, &bars[0]);
    }
    ok = mbar_wait(&bars[0], 0u);
    if (ok) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t idesc = idesc_bf16(128, N, 0, COLS);
      const uint32_t a0 = smem_u32(sa), b0 = smem_u32(sb);
      for (int s = 0; s < K / 16; ++s) {
        const int j = s >> 2, kk = s & 3;
        // K-major operand: box j (rows x 128 B), 32 bytes per 16 elements inside the row
        const uint64_t ad = smem_desc_sw128(a0 + uint32_t(j) * 128 * 128 + 32 * kk, 16, 1024);
        uint64_t bd;
        if (COLS == 0) bd = smem_desc_sw128(b0 + uint32_t(j) * uint32_t(N) * 128 + 32 * kk, 16, 1024);
        else bd = smem_desc_sw128(b0 + uint32_t(s) * 16 * 128, uint32_t(K) * 128, 1024);  // MN-major: 16 K-rows per step
        mma_bf16(tmem, ad, bd, idesc, s > 0 ? 1u : 0u);
      }
      mma_commit(&bars[1]);
    } else {
      atomicAdd(&g_wait_timeouts_tc, 1u);
      // do not leave with copies into shared memory in flight
      if (!mbar_wait(&bars[0], 0u)) atomicAdd(&g_wait_timeouts_tc, 1u);
    }
  }
  // broadcast the outcome of the load wait (lane 0 of warp 0 decided it)
  __shared__ int s_ok;
  if (threadIdx.x == 0) s_ok = ok ? 1 : 0;
  __syncthreads();
  ok = s_ok != 0;
  if (ok) {
    bool done = mbar_wait(&bars[1], 0u);
    if (!done) {
      if (lane == 0) atomicAdd(&g_wait_timeouts_tc, 1u);
      // the MMAs may still read shared memory / write tensor memory: wait once more
      done = mbar_wait(&bars[1], 0u);
    }
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (done) {
      // Epilogue: accumulator row = 32 warp + lane, 32 columns per load.
      int64_t grow;   // global output row
      int64_t gcol0;  // global column of accumulator column 0
      bool live;
      if (COLS == 0) {
        grow = t0 + 32 * warp + lane;
        gcol0 = w * a.Pw;
        live = grow < a.outer;
      } else {
        const int p = 128 * half + 32 * warp + lane;
        const int64_t base = (w / a.step) * int64_t(a.Pw) * a.step + (w % a.step);
        grow = base + int64_t(p) * a.step;
        gcol0 = t0;
        live = p < a.Pw;
      }
      Tout* yrow = static_cast<Tout*>(a.y) + grow * a.ldy + gcol0;
      for (int c = 0; c < N / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + (uint32_t(32 * warp) << 16) + uint32_t(32 * c), r);
        if (!live) continue;
        const int64_t col = gcol0 + 32 * c;
        Tout* dst = yrow + 32 * c;
        const int64_t lim = COLS == 0 ? int64_t(32) : a.ncols - col;  // columns of this chunk inside the matrix
        if (lim >= 32) {
          if constexpr (sizeof(Tout) == 4) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              __stcs(reinterpret_cast<uint4*>(dst) + q, make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]));
          } else {
            uint32_t h[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) h[q] = f32_to_bf16x2(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1]));
#pragma unroll
            for (int q = 0; q < 4; ++q)
              __stcs(reinterpret_cast<uint4*>(dst) + q, make_uint4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]));
          }
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            if (q < lim) {
              if constexpr (sizeof(Tout) == 4) dst[q] = __uint_as_float(r[q]);
              else dst[q] = __float2bfloat16_rn(__uint_as_float(r[q]));
            }
          }
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
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

// bf16 tensor map, dims / strides in elements (dim 0 contiguous), 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int rank, const int64_t* dims, const int64_t* strides_el,
              const uint32_t* box) {
  EncodeTiled f = encode_fn();
  if (f == nullptr) return false;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bd[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = cuuint64_t(dims[i]);
    bd[i] = box[i];
    es[i] = 1;
    if (i > 0) gs[i - 1] = cuuint64_t(strides_el[i]) * 2;
  }
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cuuint32_t(rank), const_cast<void*>(base), gd, gs, bd, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
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
cudaError_t launch_tc(const CUtensorMap& mx, const CUtensorMap& mm, const TcPassArgs& a, int64_t grid, size_t smem,
                      cudaStream_t st) {
  static std::atomic<unsigned long long> done{0};
  auto kern = k_bfly_tc<COLS, Tout>;
  cudaError_t e = smem_attr_once(kern, smem, done);
  if (e != cudaSuccess) return e;
  kern<<<dim3(unsigned(grid)), 128, smem, st>>>(mx, mm, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bfly_compose(const TcComposeArgs& a, int64_t n_windows, __nv_bfloat16* mats, cudaStream_t st) {
  static std::atomic<unsigned long long> done{0};
  const size_t smem = size_t(2) * kComposeCols * a.Pw * sizeof(float);
  cudaError_t e = smem_attr_once(k_bfly_compose, smem, done);
  if (e != cudaSuccess) return e;
  k_bfly_compose<<<dim3(unsigned(n_windows), unsigned(a.Pw / kComposeCols)), 256, smem, st>>>(a, mats);
  return cudaGetLastError();
}

// x: bf16 data [.., ldx]; mats: bf16 [n_windows * Pw, Pw]; y: [.., ldy] (dt_out).
cudaError_t launch_bfly_tc(const TcPassArgs& args, const void* x, int64_t ldx, const __nv_bfloat16* mats, int dt_out,
                           cudaStream_t st) {
  TcPassArgs a = args;
  CUtensorMap mx, mm;
  const int K = a.K;
  if (a.cols == 0) {
    // data [outer rows, L columns], box 64 columns x 128 rows
    const int64_t dx[2] = {a.L, a.outer}, sx[2] = {1, ldx};
    const uint32_t bx[2] = {64, 128};
    if (!make_map(&mx, x, 2, dx, sx, bx)) return cudaErrorInvalidValue;
    // matrices [n_windows * Pw rows, Pw columns], box 64 x N (the window's output rows)
    const int64_t dm[2] = {a.Pw, int64_t(a.n_windows) * a.Pw}, sm[2] = {1, a.Pw};
    const uint32_t bm[2] = {64, uint32_t(a.N)};
    if (!make_map(&mm, mats, 2, dm, sm, bm)) return cudaErrorInvalidValue;
    a.bytes_a = 128 * K * 2;
    a.bytes_b = a.N * K * 2;
  } else {
    // data [L rows, ncols columns] as (column, p, lo, hi): row = hi * Pw * step + p * step + lo
    const int64_t dx[4] = {a.ncols, a.Pw, a.step, a.L / (int64_t(a.Pw) * a.step)};
    const int64_t sx[4] = {1, a.step * ldx, ldx, int64_t(a.Pw) * a.step * ldx};
    const uint32_t bx[4] = {64, uint32_t(K), 1, 1};
    if (!make_map(&mx, x, 4, dx, sx, bx)) return cudaErrorInvalidValue;
    const int64_t dm[2] = {a.Pw, int64_t(a.n_windows) * a.Pw}, sm[2] = {1, a.Pw};
    const uint32_t bm[2] = {64, 128};
    if (!make_map(&mm, mats, 2, dm, sm, bm)) return cudaErrorInvalidValue;
    a.bytes_a = 128 * K * 2;
    a.bytes_b = a.N * K * 2;
  }
  const size_t smem = 1024 + size_t(a.bytes_a) + size_t(a.bytes_b) + 64;
  int64_t grid;
  if (a.cols == 0) grid = int64_t(a.n_windows) * ((a.outer + 127) / 128);
  else grid = int64_t(a.n_windows) * a.m_halves * ((a.ncols + a.N - 1) / a.N);
  if (a.cols == 0)
    return dt_out == DT_F32 ? launch_tc<0, float>(mx, mm, a, grid, smem, st)
                            : launch_tc<0, __nv_bfloat16>(mx, mm, a, grid, smem, st);
  return dt_out == DT_F32 ? launch_tc<1, float>(mx, mm, a, grid, smem, st)
                          : launch_tc<1, __nv_bfloat16>(mx, mm, a, grid, smem, st);
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
