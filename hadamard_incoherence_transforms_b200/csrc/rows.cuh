// Row kernels: batched Walsh-Hadamard transforms along the contiguous
// dimension, fused with sign flips, normalization, group quantization and
// packing, dequantization, and the sparse adapter scatter / gather.
//
// The transform of a row of n = 2^LOGN elements is the product of LOGN
// butterfly stages, one per bit of the element index (the fast WHT of the HARP
// and QWHA explainers: +-1 kernel, additions only, O(n log n)).  The stages
// act on distinct index bits and commute, so any mapping of index bits to
// (register, thread) positions works.  A team of T = n/E threads owns one row
// and each thread holds E = 2^LOGE elements in registers in one of two layouts:
//
//   layout A  register bits = element bits {0,1} and the top LOGE-2 bits;
//             thread bits   = element bits [2, 2+LOGT).  Loads and stores in
//             this layout are 4-element vectors, consecutive threads touching
//             consecutive 16-byte chunks (fully coalesced).
//   layout B  register bits = element bits [0, LOGE): each thread holds one
//             contiguous run of E elements (quantization groups, code words).
//
// A row goes through "stages in layout A -> shared-memory transpose -> stages
// in layout B" (or the reverse).  LOGE is chosen so the two layouts' register
// bits cover every bit; for LOGN >= 13 the few element bits that are thread
// bits in both layouts are done with warp shuffles.
#pragma once
#include <type_traits>

#include "device.cuh"
#include "internal.h"

namespace hit {

template <int LOGN>
struct Geom {
  static constexpr int N = 1 << LOGN;
  static constexpr int LOGE = LOGN <= 7 ? LOGN : (LOGN == 8 ? 5 : (LOGN <= 10 ? 6 : 7));
  static constexpr int E = 1 << LOGE;
  static constexpr int LOGT = LOGN - LOGE;
  static constexpr int T = 1 << LOGT;
  static constexpr int VW = LOGN >= 2 ? 4 : (1 << LOGN);  // layout-A vector width (elements)
  static constexpr int NV = E / VW;
  static constexpr int NT = T > 128 ? T : 128;  // threads per CTA
  static constexpr int RPC = NT / T;            // rows per CTA
  static constexpr int NSH = (T > 1 && 2 + LOGT > LOGE) ? 2 + LOGT - LOGE : 0;
  static constexpr int LQ = LOGE - 2 >= 3 ? LOGE - 2 : 3;
  static constexpr int B_FWD_HI = LOGE < 2 + LOGT ? LOGE : 2 + LOGT;  // layout-B stages after A
  static constexpr int A_INV_LO = LOGE - LOGT > 2 ? LOGE - LOGT : 2;  // layout-A stages after B
  // CTAs per SM the register budget is shaped for (128-element threads: 3).
  static constexpr int MINB = (E == 128 && NT == 128) ? 3 : 1;
  static constexpr size_t smem_bytes(bool need_buf) {
    return (T > 1 || need_buf) ? size_t(RPC) * N * sizeof(float) : 0;
  }
};

template <int T>
__device__ __forceinline__ unsigned team_mask() {
  if constexpr (T >= 32) {
    return 0xffffffffu;
  } else {
    const int lane = threadIdx.x & 31;
    return ((1u << T) - 1u) << (lane & ~(T - 1));
  }
}

template <int T>
__device__ __forceinline__ void team_sync(int team) {
  if constexpr (T > 32) {
    asm volatile("bar.sync %0, %1;" ::"r"(team + 1), "r"(T) : "memory");
  } else {
    __syncwarp(team_mask<T>());
  }
}

template <typename Tv>
__device__ __forceinline__ float to_f32(Tv v) {
  if constexpr (std::is_same<Tv, float>::value) return v;
  else return __bfloat162float(v);
}
template <typename Tv>
__device__ __forceinline__ Tv from_f32(float v) {
  if constexpr (std::is_same<Tv, float>::value) return v;
  else return __float2bfloat16_rn(v);
}

// ----------------------------------------------------------------------------
// Dense rows in layout A (vector j of thread tau covers elements
// 4*(tau + T*j) .. +3), with the sign flip diag(s) fused into the load.
// ----------------------------------------------------------------------------
template <int LOGN, typename Tin>
__device__ __forceinline__ void load_rowA(float (&x)[Geom<LOGN>::E], const Tin* __restrict__ src, int tau,
                                          const int8_t* __restrict__ sg) {
  using G = Geom<LOGN>;
  if constexpr (G::VW == 4) {
#pragma unroll
    for (int j = 0; j < G::NV; ++j) {
      const int i0 = 4 * (tau + G::T * j);
      if constexpr (std::is_same<Tin, float>::value) {
        const float4 v = ld_stream_f4(src + i0);
        x[4 * j] = v.x;
        x[4 * j + 1] = v.y;
        x[4 * j + 2] = v.z;
        x[4 * j + 3] = v.w;
      } else {
        const uint2 v = ld_stream_u2(src + i0);
        bf16x2_to_f32(v.x, x[4 * j], x[4 * j + 1]);
        bf16x2_to_f32(v.y, x[4 * j + 2], x[4 * j + 3]);
      }
      if (sg != nullptr) {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(sg + i0));
        apply_sign4(x[4 * j], x[4 * j + 1], x[4 * j + 2], x[4 * j + 3], w);
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < G::E; ++e) {
      x[e] = to_f32(src[e]);
      if (sg != nullptr && sg[e] < 0) x[e] = -x[e];
    }
  }
}

template <int LOGN, typename Tout, bool NORM>
__device__ __forceinline__ void store_rowA(float (&x)[Geom<LOGN>::E], Tout* __restrict__ dst, int tau, float norm,
                                           const int8_t* __restrict__ sg) {
  using G = Geom<LOGN>;
  if constexpr (G::VW == 4) {
#pragma unroll
    for (int j = 0; j < G::NV; ++j) {
      const int i0 = 4 * (tau + G::T * j);
      float v0 = x[4 * j], v1 = x[4 * j + 1], v2 = x[4 * j + 2], v3 = x[4 * j + 3];
      if constexpr (NORM) {
        mul_x2(v0, v1, norm, norm);
        mul_x2(v2, v3, norm, norm);
      }
      if (sg != nullptr) apply_sign4(v0, v1, v2, v3, __ldg(reinterpret_cast<const uint32_t*>(sg + i0)));
      if constexpr (std::is_same<Tout, float>::value) {
        st_stream_f4(dst + i0, make_float4(v0, v1, v2, v3));
      } else {
        st_stream_u2(dst + i0, make_uint2(f32_to_bf16x2(v0, v1), f32_to_bf16x2(v2, v3)));
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < G::E; ++e) {
      float v = x[e];
      if constexpr (NORM) v *= norm;
      if (sg != nullptr && sg[e] < 0) v = -v;
      dst[e] = from_f32<Tout>(v);
    }
  }
}

// ----------------------------------------------------------------------------
// Dense rows in layout B (thread tau holds elements E*tau .. E*tau + E - 1).
// ----------------------------------------------------------------------------
template <int LOGN, typename Tout>
__device__ __forceinline__ void store_rowB(float (&x)[Geom<LOGN>::E], Tout* __restrict__ dst, int tau, float norm,
                                           const int8_t* __restrict__ sg) {
  using G = Geom<LOGN>;
  constexpr int E = G::E;
  const int base = E * tau;
  if constexpr (E >= 2) {
#pragma unroll
    for (int e = 0; e < E; e += 2) mul_x2(x[e], x[e + 1], norm, norm);
  } else {
    x[0] *= norm;
  }
  if (sg != nullptr) {
    if constexpr (E >= 4) {
#pragma unroll
      for (int m = 0; m < E / 4; ++m)
        apply_sign4(x[4 * m], x[4 * m + 1], x[4 * m + 2], x[4 * m + 3],
                    __ldg(reinterpret_cast<const uint32_t*>(sg + base + 4 * m)));
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e)
        if (sg[base + e] < 0) x[e] = -x[e];
    }
  }
  // A thread's run is contiguous: with 32-byte alignment it goes out as whole
  // 32-byte sectors, one per store.
  const bool wide = (reinterpret_cast<uintptr_t>(dst + base) & 31) == 0;
  if constexpr (std::is_same<Tout, float>::value && E >= 8) {
    if (wide) {
#pragma unroll
      for (int m = 0; m < E / 8; ++m)
        st_stream_v8(dst + base + 8 * m, __float_as_uint(x[8 * m]), __float_as_uint(x[8 * m + 1]),
                     __float_as_uint(x[8 * m + 2]), __float_as_uint(x[8 * m + 3]), __float_as_uint(x[8 * m + 4]),
                     __float_as_uint(x[8 * m + 5]), __float_as_uint(x[8 * m + 6]), __float_as_uint(x[8 * m + 7]));
      return;
    }
  }
  if constexpr (std::is_same<Tout, __nv_bfloat16>::value && E >= 16) {
    if (wide) {
#pragma unroll
      for (int m = 0; m < E / 16; ++m)
        st_stream_v8(dst + base + 16 * m, f32_to_bf16x2(x[16 * m], x[16 * m + 1]),
                     f32_to_bf16x2(x[16 * m + 2], x[16 * m + 3]), f32_to_bf16x2(x[16 * m + 4], x[16 * m + 5]),
                     f32_to_bf16x2(x[16 * m + 6], x[16 * m + 7]), f32_to_bf16x2(x[16 * m + 8], x[16 * m + 9]),
                     f32_to_bf16x2(x[16 * m + 10], x[16 * m + 11]), f32_to_bf16x2(x[16 * m + 12], x[16 * m + 13]),
                     f32_to_bf16x2(x[16 * m + 14], x[16 * m + 15]));
      return;
    }
  }
  if constexpr (std::is_same<Tout, float>::value && E >= 4) {
#pragma unroll
    for (int m = 0; m < E / 4; ++m)
      st_stream_f4(dst + base + 4 * m, make_float4(x[4 * m], x[4 * m + 1], x[4 * m + 2], x[4 * m + 3]));
  } else if constexpr (std::is_same<Tout, __nv_bfloat16>::value && E >= 8) {
#pragma unroll
    for (int m = 0; m < E / 8; ++m) {
      uint4 v;
      v.x = f32_to_bf16x2(x[8 * m], x[8 * m + 1]);
      v.y = f32_to_bf16x2(x[8 * m + 2], x[8 * m + 3]);
      v.z = f32_to_bf16x2(x[8 * m + 4], x[8 * m + 5]);
      v.w = f32_to_bf16x2(x[8 * m + 6], x[8 * m + 7]);
      __stcs(reinterpret_cast<uint4*>(dst + base + 8 * m), v);
    }
  } else if constexpr (std::is_same<Tout, __nv_bfloat16>::value && E == 4) {
    st_stream_u2(dst + base, make_uint2(f32_to_bf16x2(x[0], x[1]), f32_to_bf16x2(x[2], x[3])));
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) dst[base + e] = from_f32<Tout>(x[e]);
  }
}

// Shared-memory transposes between the layouts (row buffer of n floats).
template <int LOGN>
__device__ __forceinline__ void smem_put_A(float4* buf, const float (&x)[Geom<LOGN>::E], int tau) {
  using G = Geom<LOGN>;
#pragma unroll
  for (int j = 0; j < G::NV; ++j)
    buf[swz<G::LQ>(tau + G::T * j)] = make_float4(x[4 * j], x[4 * j + 1], x[4 * j + 2], x[4 * j + 3]);
}
template <int LOGN>
__device__ __forceinline__ void smem_get_A(const float4* buf, float (&x)[Geom<LOGN>::E], int tau) {
  using G = Geom<LOGN>;
#pragma unroll
  for (int j = 0; j < G::NV; ++j) {
    const float4 v = buf[swz<G::LQ>(tau + G::T * j)];
    x[4 * j] = v.x;
    x[4 * j + 1] = v.y;
    x[4 * j + 2] = v.z;
    x[4 * j + 3] = v.w;
  }
}
template <int LOGN>
__device__ __forceinline__ void smem_put_B(float4* buf, const float (&x)[Geom<LOGN>::E], int tau) {
  using G = Geom<LOGN>;
#pragma unroll
  for (int m = 0; m < G::E / 4; ++m)
    buf[swz<G::LQ>((G::E / 4) * tau + m)] = make_float4(x[4 * m], x[4 * m + 1], x[4 * m + 2], x[4 * m + 3]);
}
template <int LOGN>
__device__ __forceinline__ void smem_get_B(const float4* buf, float (&x)[Geom<LOGN>::E], int tau) {
  using G = Geom<LOGN>;
#pragma unroll
  for (int m = 0; m < G::E / 4; ++m) {
    const float4 v = buf[swz<G::LQ>((G::E / 4) * tau + m)];
    x[4 * m] = v.x;
    x[4 * m + 1] = v.y;
    x[4 * m + 2] = v.z;
    x[4 * m + 3] = v.w;
  }
}
template <int LOGN>
__device__ __forceinline__ int smem_elem(int i) {
  return swz<Geom<LOGN>::LQ>(i >> 2) * 4 + (i & 3);
}

}  // namespace hit
