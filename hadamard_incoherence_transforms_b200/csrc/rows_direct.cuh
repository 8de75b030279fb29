// Persistent row kernel for long rows (n = 4096 / 8192, one or two warps per
// row) that loads rows straight from global memory into registers.
//
// Every warp computes: a team of one (n = 4096) or two (n = 8192) warps takes
// the rows blockIdx.x + grid * (team + TEAMS * k), k = 0, 1, ..., so the last
// round of rows is spread over all SMs.  Per row a team
//   - reads the row in layout A with coalesced vector loads (the loads were
//     issued during the previous row's epilogue, and the row was prefetched
//     into L2 one row earlier still with a bulk prefetch),
//   - flips signs with an integer xor from sign-bit masks held in registers
//     (each thread always sees the same columns, so its signs fit in four
//     32-bit words),
//   - runs the layout-A stages, transposes through a per-team shared-memory
//     buffer, runs the layout-B stages (and the shuffle stage for n = 8192),
//   - runs the epilogue (quantize + pack, or scale + store) one 32-element
//     chunk at a time, and as soon as a chunk's registers are free it issues
//     the loads of the matching part of the team's next row.
// Shared memory carries only the transpose (one write and one read of the
// row), and no warp is set aside for data movement.  No wait in this kernel
// depends on another CTA or on an asynchronous copy.
#pragma once
#include "rows_ops.cuh"

namespace hit {

template <int LOGN, int WARPS>
struct DirectCfg {
  using G = Geom<LOGN>;
  static_assert(G::T == 32 || G::T == 64, "direct kernel needs one or two warps per row");
  static_assert(G::E == 128, "direct kernel holds 128 elements per thread");
  static constexpr int WPR = G::T / 32;
  static constexpr int TEAMS = WARPS / WPR;
  static constexpr int THREADS = WARPS * 32;
  static constexpr size_t SMEM = size_t(TEAMS) * G::N * sizeof(float);
  static_assert(TEAMS * WPR == WARPS && TEAMS <= 15, "whole teams, named barrier ids 1..15");
};

// L2 prefetch of a contiguous range (16-byte aligned start, size a multiple of 16).
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Layout-A vector j (elements 4*(tau + T*j) .. +3) of a row into x[4j .. 4j+3].
template <int LOGN, typename Tin>
__device__ __forceinline__ void load_vecA(float* x, const Tin* __restrict__ src, int tau, int j) {
  const int i0 = 4 * (tau + Geom<LOGN>::T * j);
  if constexpr (std::is_same<Tin, float>::value) {
    const float4 v = ld_stream_f4(src + i0);
    x[0] = v.x;
    x[1] = v.y;
    x[2] = v.z;
    x[3] = v.w;
  } else {
    const uint2 v = ld_stream_u2(src + i0);
    bf16x2_to_f32(v.x, x[0], x[1]);
    bf16x2_to_f32(v.y, x[2], x[3]);
  }
}

// Sign-bit masks of the layout-A columns of thread tau: bit j of m[c] is the
// sign of element 4*(tau + T*j) + c.
template <int LOGN>
__device__ __forceinline__ void sign_masks(uint32_t (&m)[4], const int8_t* __restrict__ s, int tau) {
  using G = Geom<LOGN>;
  m[0] = m[1] = m[2] = m[3] = 0u;
  if (s == nullptr) return;
  const bool al = (reinterpret_cast<uintptr_t>(s) & 3) == 0;
#pragma unroll
  for (int j = 0; j < G::NV; ++j) {
    const int i0 = 4 * (tau + G::T * j);
    uint32_t w;
    if (al) {
      w = __ldg(reinterpret_cast<const uint32_t*>(s + i0));
    } else {
      w = uint32_t(uint8_t(s[i0])) | (uint32_t(uint8_t(s[i0 + 1])) << 8) | (uint32_t(uint8_t(s[i0 + 2])) << 16) |
          (uint32_t(uint8_t(s[i0 + 3])) << 24);
    }
    m[0] |= ((w >> 7) & 1u) << j;
    m[1] |= ((w >> 15) & 1u) << j;
    m[2] |= ((w >> 23) & 1u) << j;
    m[3] |= ((w >> 31) & 1u) << j;
  }
}

template <int LOGN>
__device__ __forceinline__ void apply_sign_masks(float (&x)[Geom<LOGN>::E], const uint32_t (&m)[4]) {
#pragma unroll
  for (int j = 0; j < Geom<LOGN>::NV; ++j) {
#pragma unroll
    for (int c = 0; c < 4; ++c)
      x[4 * j + c] = __uint_as_float(__float_as_uint(x[4 * j + c]) ^ ((m[c] << (31 - j)) & 0x80000000u));
  }
}

template <int LOGN, int WARPS>
__device__ __forceinline__ void direct_team_sync(int team) {
  if constexpr (DirectCfg<LOGN, WARPS>::WPR == 1) {
    __syncwarp();
  } else {
    asm volatile("bar.sync %0, %1;" ::"r"(team + 1), "r"(Geom<LOGN>::T) : "memory");
  }
}

// Scale (and post-sign) + store a row held in layout B, 32 elements at a time;
// after chunk cc is stored, next(cc) may overwrite x[32cc .. 32cc+31].
template <int LOGN, typename Tout, typename Next>
__device__ __forceinline__ void store_rowB_next(float (&x)[Geom<LOGN>::E], Tout* __restrict__ dst, int tau,
                                                float norm, const int8_t* __restrict__ sg, Next&& next) {
  using G = Geom<LOGN>;
  constexpr int E = G::E;
  const int base = E * tau;
  const bool wide = (reinterpret_cast<uintptr_t>(dst + base) & 31) == 0;
#pragma unroll
  for (int cc = 0; cc < E / 32; ++cc) {
    float* xc = x + 32 * cc;
#pragma unroll
    for (int e = 0; e < 32; e += 2) mul_x2(xc[e], xc[e + 1], norm, norm);
    if (sg != nullptr) {
#pragma unroll
      for (int m = 0; m < 8; ++m)
        apply_sign4(xc[4 * m], xc[4 * m + 1], xc[4 * m + 2], xc[4 * m + 3],
                    __ldg(reinterpret_cast<const uint32_t*>(sg + base + 32 * cc + 4 * m)));
    }
    if constexpr (std::is_same<Tout, float>::value) {
      if (!wide) {
#pragma unroll
        for (int m = 0; m < 8; ++m)
          st_stream_f4(dst + base + 32 * cc + 4 * m,
                       make_float4(xc[4 * m], xc[4 * m + 1], xc[4 * m + 2], xc[4 * m + 3]));
      } else {
#pragma unroll
      for (int m = 0; m < 4; ++m)  // 32-byte stores (whole sectors)
        st_stream_v8(dst + base + 32 * cc + 8 * m, __float_as_uint(xc[8 * m]), __float_as_uint(xc[8 * m + 1]),
                     __float_as_uint(xc[8 * m + 2]), __float_as_uint(xc[8 * m + 3]), __float_as_uint(xc[8 * m + 4]),
                     __float_as_uint(xc[8 * m + 5]), __float_as_uint(xc[8 * m + 6]), __float_as_uint(xc[8 * m + 7]));
      }
    } else if (!wide) {
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        uint4 v;
        v.x = f32_to_bf16x2(xc[8 * m], xc[8 * m + 1]);
        v.y = f32_to_bf16x2(xc[8 * m + 2], xc[8 * m + 3]);
        v.z = f32_to_bf16x2(xc[8 * m + 4], xc[8 * m + 5]);
        v.w = f32_to_bf16x2(xc[8 * m + 6], xc[8 * m + 7]);
        __stcs(reinterpret_cast<uint4*>(dst + base + 32 * cc + 8 * m), v);
      }
    } else {
#pragma unroll
      for (int m = 0; m < 2; ++m)  // 32-byte stores (whole sectors)
        st_stream_v8(dst + base + 32 * cc + 16 * m, f32_to_bf16x2(xc[16 * m], xc[16 * m + 1]),
                     f32_to_bf16x2(xc[16 * m + 2], xc[16 * m + 3]), f32_to_bf16x2(xc[16 * m + 4], xc[16 * m + 5]),
                     f32_to_bf16x2(xc[16 * m + 6], xc[16 * m + 7]), f32_to_bf16x2(xc[16 * m + 8], xc[16 * m + 9]),
                     f32_to_bf16x2(xc[16 * m + 10], xc[16 * m + 11]), f32_to_bf16x2(xc[16 * m + 12], xc[16 * m + 13]),
                     f32_to_bf16x2(xc[16 * m + 14], xc[16 * m + 15]));
    }
    next(cc);
  }
}

template <int LOGN, typename Tin, typename Tout, int EPI, int BITS, int WARPS, int PF>
__global__ void __launch_bounds__(DirectCfg<LOGN, WARPS>::THREADS, 1) k_rows_direct(const RowArgs a) {
  using G = Geom<LOGN>;
  using C = DirectCfg<LOGN, WARPS>;
  extern __shared__ __align__(16) float4 dsm4[];
  const int warp = threadIdx.x >> 5;
  const int team = warp / C::WPR;
  const int tau = (warp % C::WPR) * 32 + (threadIdx.x & 31);
  const int64_t grid = gridDim.x;
  const int64_t stride = grid * C::TEAMS;
  int64_t row = blockIdx.x + grid * team;
  if (row >= a.rows) return;  // the whole team leaves together
  float4* buf = dsm4 + size_t(team) * (G::N / 4);
  const Tin* __restrict__ xin = static_cast<const Tin*>(a.x);
  constexpr uint32_t ROW_BYTES = uint32_t(G::N * sizeof(Tin));

  uint32_t sm[4];
  sign_masks<LOGN>(sm, a.pre_signs, tau);
  const bool has_signs = a.pre_signs != nullptr;

  float x[G::E];
  {
    const Tin* src = xin + row * a.ldx;
#pragma unroll
    for (int j = 0; j < G::NV; ++j) load_vecA<LOGN, Tin>(x + 4 * j, src, tau, j);
  }
  for (;;) {
    const int64_t nxt = row + stride;
    const bool more = nxt < a.rows;
    // L2 prefetch PF rows ahead of the row being computed (the row right
    // after it is loaded into registers during this row's epilogue).
    if constexpr (PF >= 1) {
      if (tau == 0) {
        const bool first = row == blockIdx.x + grid * team;
        for (int d = first ? 1 : PF; d <= PF; ++d)
          if (row + d * stride < a.rows) prefetch_l2_bulk(xin + (row + d * stride) * a.ldx, ROW_BYTES);
      }
    }
    if (has_signs) {
      // Redefine the masks every row: otherwise the compiler hoists the 128
      // shifted masks out of the row loop and runs out of registers.
#pragma unroll
      for (int c = 0; c < 4; ++c) asm volatile("mov.b32 %0, %0;" : "+r"(sm[c]));
      apply_sign_masks<LOGN>(x, sm);
    }
    reg_stages<G::E, 0, G::LOGE>(x);
    direct_team_sync<LOGN, WARPS>(team);  // the team's reads of the previous row's buffer are done
    smem_put_A<LOGN>(buf, x, tau);
    direct_team_sync<LOGN, WARPS>(team);
    smem_get_B<LOGN>(buf, x, tau);
    reg_stages<G::E, 2, G::B_FWD_HI>(x);
#pragma unroll
    for (int b = 0; b < G::NSH; ++b) shfl_stage<G::E>(x, b, (tau >> b) & 1);

    const Tin* nsrc = xin + (more ? nxt : row) * a.ldx;
    auto next = [&](int cc) {
      if (more) {
#pragma unroll
        for (int j = 8 * cc; j < 8 * cc + 8; ++j) load_vecA<LOGN, Tin>(x + 4 * j, nsrc, tau, j);
      }
    };
    if constexpr (EPI == EPI_STORE) {
      store_rowB_next<LOGN, Tout>(x, static_cast<Tout*>(a.y) + row * a.ldy, tau, a.norm, a.post_signs, next);
    } else {
      quant_rowB_next<LOGN, BITS>(x, a, row, tau, next);
    }
    if (!more) break;
    row = nxt;
  }
}

template <int LOGN, typename Tin, typename Tout, int EPI, int BITS, int WARPS = 8, int PF = 2>
cudaError_t launch_direct(const RowArgs& a, cudaStream_t st) {
  using C = DirectCfg<LOGN, WARPS>;
  static std::atomic<unsigned long long> done{0};
  auto kern = k_rows_direct<LOGN, Tin, Tout, EPI, BITS, WARPS, PF>;
  cudaError_t e = set_smem_attr(kern, C::SMEM, done);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int64_t need = (a.rows + C::TEAMS - 1) / C::TEAMS;
  const int64_t grid = need < sms ? need : sms;
  kern<<<dim3(unsigned(grid)), C::THREADS, C::SMEM, st>>>(a);
  return cudaGetLastError();
}

}  // namespace hit
