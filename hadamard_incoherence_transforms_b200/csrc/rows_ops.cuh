// Epilogues / prologues of the row kernels and the kernels themselves.
#pragma once
#include <atomic>

#include "rows.cuh"

namespace hit {

// ----------------------------------------------------------------------------
// Group-wise symmetric absmax round-to-nearest, in layout B.
//
// Per group: a = max|y|, s = a / qmax (IEEE division), q = rint(y / s) with
// ties to even, stored code u = q + 2^(bits-1).
//
// The quotient t = RN(y / s) is computed without a divide instruction by
// Markstein's correction step (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990): with r = RN(1/s) and q0 = RN(y r) (within one ulp of y/s), the
// remainder e = y - s q0 is exact in one fma and RN(q0 + e r) is the
// correctly rounded quotient, barring underflow and overflow.  Groups whose
// scale lies outside [2^-100, 2^100] are rescaled by an exact power of two
// first (y/s is unchanged; elements that underflow in the rescale have
// |y/s| far below 1/2 and quantize to 0 either way).  Every element is then
// rounded to an integer by adding 1.5*2^23 + 2^(bits-1): the sum lies in
// [2^23, 2^24) where the float spacing is 1, so the add rounds t to the
// nearest integer with ties to even (the offset is even) and the low byte of
// the sum's bit pattern is the stored code.  |t| <= qmax (1 + 2^-23), so no
// clamp is needed.  The fp32 operations are packed two per instruction.
//
// When log2(n) is even, 1/sqrt(n) is a power of two and is folded exactly
// into the scale: y = acc * 2^-k, s = s_acc * 2^-k, y/s = acc/s_acc.
// ----------------------------------------------------------------------------
template <int BITS>
struct QConst {
  static constexpr float QMAX = float((1 << (BITS - 1)) - 1);
  static constexpr float MAGIC = 12582912.0f + float(1 << (BITS - 1));
};

// s = RN(a / qmax) for the group scale.  qmax is 1, 3 or 7.  For a >= 2^-120
// the quotient is formed with the same correction step as the codes (with
// r = RN(1/qmax) a compile-time constant): q0 = RN(a r) is within one ulp of
// a/qmax, the remainder a - qmax q0 is exact, and RN(q0 + e r) is the
// correctly rounded quotient; smaller a (where the remainder could underflow)
// takes the IEEE division.
template <int BITS>
__device__ __forceinline__ float group_scale(float a) {
  constexpr float QMAX = QConst<BITS>::QMAX;
  if constexpr (BITS == 2) {
    return a;  // qmax = 1
  } else {
    constexpr float R = 1.0f / QMAX;  // RN(1/qmax): 1/3 and 1/7 rounded once at compile time
    if (a >= 0x1p-120f) {
      const float q0 = a * R;
      const float e = fmaf(-QMAX, q0, a);
      return fmaf(e, R, q0);
    }
    return __fdiv_rn(a, QMAX);
  }
}

// Codes of 8 elements of one group with scale s and r = RN(1/s).  An all-zero
// group passes r = 0 (and s = 1): every quotient is then 0 and the code is
// the offset 2^(bits-1).
template <int BITS>
__device__ __forceinline__ void quant8(const float* xc, float s, float r, uint32_t* ub) {
  constexpr float MAGIC = QConst<BITS>::MAGIC;
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    float q0, q1, e0, e1, t0, t1, m0, m1;
    fma_x2(xc[e], xc[e + 1], r, r, 0.0f, 0.0f, q0, q1);      // q0 = RN(y r)
    fma_x2(q0, q1, -s, -s, xc[e], xc[e + 1], e0, e1);         // e = y - s q0 (exact)
    fma_x2(e0, e1, r, r, q0, q1, t0, t1);                     // t = RN(q0 + e r) = RN(y / s)
    fma_x2(t0, t1, 1.0f, 1.0f, MAGIC, MAGIC, m0, m1);         // RN(t + MAGIC) = rint(t) + MAGIC
    ub[e] = __float_as_uint(m0);
    ub[e + 1] = __float_as_uint(m1);
  }
}

// next(cc) runs after chunk cc's values are consumed; a persistent kernel uses
// it to refill x[32cc .. 32cc+31] with its next row.
template <int LOGN, int BITS, typename Next>
__device__ __forceinline__ void quant_rowB_next(float (&x)[Geom<LOGN>::E], const RowArgs& a, int64_t row, int tau,
                                                Next&& next) {
  using G = Geom<LOGN>;
  constexpr int E = G::E;
  constexpr int NCH = E / 32;
  constexpr bool FOLD = (LOGN % 2) == 0;
  constexpr float QMAX = QConst<BITS>::QMAX;
  constexpr float MAGIC = QConst<BITS>::MAGIC;
  static_assert(E >= 32, "quantization needs at least 32 elements per thread");

  if constexpr (!FOLD) {
#pragma unroll
    for (int e = 0; e < E; e += 2) mul_x2(x[e], x[e + 1], a.norm, a.norm);
  }
  float mx[NCH];
#pragma unroll
  for (int cc = 0; cc < NCH; ++cc) {  // |max| over 32 elements as a tree (independent chains)
    float t[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      t[k] = fmaxf(fmaxf(fabsf(x[32 * cc + k]), fabsf(x[32 * cc + 8 + k])),
                   fmaxf(fabsf(x[32 * cc + 16 + k]), fabsf(x[32 * cc + 24 + k])));
    mx[cc] = fmaxf(fmaxf(fmaxf(t[0], t[1]), fmaxf(t[2], t[3])), fmaxf(fmaxf(t[4], t[5]), fmaxf(t[6], t[7])));
  }
  const int lg = a.log2g;
#pragma unroll
  for (int L = 0; (1 << L) < NCH; ++L) {
    if (5 + L < lg) {
#pragma unroll
      for (int cc = 0; cc < NCH; ++cc) {
        if ((cc >> L) & 1) continue;
        const float m = fmaxf(mx[cc], mx[cc | (1 << L)]);
        mx[cc] = m;
        mx[cc | (1 << L)] = m;
      }
    }
  }
  if (lg > G::LOGE) {  // a group spans 2^(lg-LOGE) neighbouring threads
    float m = mx[0];
    const unsigned mask = team_mask<G::T>();
    for (int L = 0; L < lg - G::LOGE; ++L) m = fmaxf(m, __shfl_xor_sync(mask, m, 1 << L));
#pragma unroll
    for (int cc = 0; cc < NCH; ++cc) mx[cc] = m;
  }

  // 4- and 2-bit codes are packed as each 32-element chunk is done and stored
  // in 32-byte pieces (two 4-bit or four 2-bit chunks) when the thread's code
  // run is 32-byte aligned, else per chunk; 3-bit chunks (12 bytes) are
  // collected and stored as 16-byte vectors at the end.
  constexpr int NW = E * BITS / 32;  // packed words per thread
  constexpr int CW = BITS;           // packed words per 32-element chunk
  uint32_t W[BITS == 3 ? NW : 8];
  uint8_t* dst = a.codes + row * (int64_t(G::N) * BITS / 8) + int64_t(tau) * (E * BITS / 8);
  const bool wide = (reinterpret_cast<uintptr_t>(dst) & 31) == 0;
  const int64_t spr = int64_t(G::N) >> lg;
  float s = 0.0f, ss = 0.0f, r = 0.0f, k = 1.0f;
#pragma unroll
  for (int cc = 0; cc < NCH; ++cc) {
    const int e0 = E * tau + 32 * cc;
    if (cc == 0 || (e0 & ((1 << lg) - 1)) == 0) {  // first chunk of a group: its scale
      s = group_scale<BITS>(mx[cc]);
      if ((e0 & ((1 << lg) - 1)) == 0) a.scales[row * spr + (e0 >> lg)] = FOLD ? s * a.norm : s;
      k = s < 0x1p-100f ? 0x1p100f : (s > 0x1p100f ? 0x1p-100f : 1.0f);
      ss = s * k;
      r = s > 0.0f ? __frcp_rn(ss) : 0.0f;
    }
    float* xc = x + 32 * cc;
    if (k != 1.0f) {
#pragma unroll
      for (int e = 0; e < 32; e += 2) mul_x2(xc[e], xc[e + 1], k, k);
    }
    const float rr = s > 0.0f ? r : 0.0f;
    const float sx = s > 0.0f ? ss : 1.0f;
    if constexpr (BITS == 4) {
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint32_t ub[8];
        quant8<BITS>(xc + 8 * v, sx, rr, ub);
        W[4 * (cc & 1) + v] = pack4x8(ub);
      }
      // 32 bytes (two chunks) per store when aligned: whole sectors
      if (NCH >= 2 && wide) {
        if (cc & 1)
          st_stream_v8(dst + 16 * (cc - 1), W[0], W[1], W[2], W[3], W[4], W[5], W[6], W[7]);
      } else {
        __stcs(reinterpret_cast<uint4*>(dst) + cc, make_uint4(W[4 * (cc & 1)], W[4 * (cc & 1) + 1],
                                                             W[4 * (cc & 1) + 2], W[4 * (cc & 1) + 3]));
      }
    } else if constexpr (BITS == 2) {
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        uint32_t ub[16];
        quant8<BITS>(xc + 16 * v, sx, rr, ub);
        quant8<BITS>(xc + 16 * v + 8, sx, rr, ub + 8);
        W[2 * (cc & 3) + v] = pack2x16(ub);
      }
      // 32 bytes (four chunks) per store when aligned
      if (NCH >= 4 && wide) {
        if ((cc & 3) == 3)
          st_stream_v8(dst + 8 * (cc - 3), W[0], W[1], W[2], W[3], W[4], W[5], W[6], W[7]);
      } else {
        __stcs(reinterpret_cast<uint2*>(dst) + cc, make_uint2(W[2 * (cc & 3)], W[2 * (cc & 3) + 1]));
      }
    } else {
      uint32_t ub[32];
#pragma unroll
      for (int v = 0; v < 4; ++v) quant8<BITS>(xc + 8 * v, sx, rr, ub + 8 * v);
      pack3x32(ub, W + CW * cc);
    }
    next(cc);
  }
  if constexpr (BITS == 3) {
    if constexpr (NW % 4 == 0) {
#pragma unroll
      for (int v = 0; v < NW / 4; ++v)
        __stcs(reinterpret_cast<uint4*>(dst) + v, make_uint4(W[4 * v], W[4 * v + 1], W[4 * v + 2], W[4 * v + 3]));
    } else {
#pragma unroll
      for (int v = 0; v < NW; ++v) __stcs(reinterpret_cast<uint32_t*>(dst) + v, W[v]);
    }
  }
}

template <int LOGN, int BITS>
__device__ __forceinline__ void quant_rowB(float (&x)[Geom<LOGN>::E], const RowArgs& a, int64_t row, int tau) {
  quant_rowB_next<LOGN, BITS>(x, a, row, tau, [](int) {});
}

// Dequantization into layout B: yhat = (u - 2^(bits-1)) * s, with the
// transform's 1/sqrt(n) folded into s (exact when log2 n is even).
template <int LOGN, int BITS>
__device__ __forceinline__ void dequant_rowB(float (&x)[Geom<LOGN>::E], const RowArgs& a, int64_t row, int tau) {
  using G = Geom<LOGN>;
  constexpr int E = G::E;
  constexpr int NCH = E / 32;
  constexpr int NW = E * BITS / 32;
  constexpr float MAGIC = QConst<BITS>::MAGIC;
  uint32_t W[NW];
  const uint8_t* src = a.codes_in + row * (int64_t(G::N) * BITS / 8) + int64_t(tau) * (E * BITS / 8);
  if constexpr (NW % 4 == 0) {
#pragma unroll
    for (int v = 0; v < NW / 4; ++v) {
      const uint4 q = __ldcs(reinterpret_cast<const uint4*>(src) + v);
      W[4 * v] = q.x;
      W[4 * v + 1] = q.y;
      W[4 * v + 2] = q.z;
      W[4 * v + 3] = q.w;
    }
  } else if constexpr (NW % 2 == 0) {
#pragma unroll
    for (int v = 0; v < NW / 2; ++v) {
      const uint2 q = __ldcs(reinterpret_cast<const uint2*>(src) + v);
      W[2 * v] = q.x;
      W[2 * v + 1] = q.y;
    }
  } else {
#pragma unroll
    for (int v = 0; v < NW; ++v) W[v] = __ldcs(reinterpret_cast<const uint32_t*>(src) + v);
  }
  const int lg = a.log2g;
  const int64_t spr = int64_t(G::N) >> lg;
#pragma unroll
  for (int cc = 0; cc < NCH; ++cc) {
    const float s = __ldg(a.scales_in + row * spr + ((E * tau + 32 * cc) >> lg)) * a.norm;
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      float q0 = __uint_as_float(0x4B400000u | code_at<BITS>(W + BITS * cc, e)) - MAGIC;
      float q1 = __uint_as_float(0x4B400000u | code_at<BITS>(W + BITS * cc, e + 1)) - MAGIC;
      mul_x2(q0, q1, s, s);
      x[32 * cc + e] = q0;
      x[32 * cc + e + 1] = q1;
    }
  }
}

// Sparse adapter, forward: F_r = scatter-add of (values * scale) at cols into
// a zeroed row buffer, then read back in layout B.
// Up to kScatterPre entries per thread are held in registers, loaded before
// the row buffer is cleared so that their latency overlaps the clearing.
constexpr int kScatterPre = 4;
template <int LOGN>
__device__ __forceinline__ void scatter_load(int (&cols)[kScatterPre], float (&vals)[kScatterPre], const RowArgs& a,
                                             int64_t row, int tau) {
  using G = Geom<LOGN>;
  const int64_t base = row * a.nnz;
#pragma unroll
  for (int j = 0; j < kScatterPre; ++j) {
    const int k = tau + j * G::T;
    cols[j] = -1;
    vals[j] = 0.0f;
    if (k < a.nnz) {
      cols[j] = __ldg(a.sp_cols + base + k);
      vals[j] = __ldg(a.sp_values + base + k);
    }
  }
}
// Clear the row buffer, add the row's entries (held in registers when `fast`,
// else read here) and read the row back in layout B.
template <int LOGN>
__device__ __forceinline__ void scatter_apply(float (&x)[Geom<LOGN>::E], const RowArgs& a, int64_t row, int tau,
                                              int team, float4* buf, bool fast, const int (&cols)[kScatterPre],
                                              const float (&vals)[kScatterPre]) {
  using G = Geom<LOGN>;
  float* bf = reinterpret_cast<float*>(buf);
#pragma unroll
  for (int m = 0; m < G::E / 4; ++m) buf[swz<G::LQ>((G::E / 4) * tau + m)] = make_float4(0.f, 0.f, 0.f, 0.f);
  team_sync<G::T>(team);
  if (fast) {
#pragma unroll
    for (int j = 0; j < kScatterPre; ++j)
      if (static_cast<unsigned>(cols[j]) < static_cast<unsigned>(G::N))
        atomicAdd(bf + smem_elem<LOGN>(cols[j]), vals[j] * a.sp_scale);
  } else {
    const int64_t base = row * a.nnz;
    for (int k = tau; k < a.nnz; k += G::T) {
      const int col = __ldg(a.sp_cols + base + k);
      if (static_cast<unsigned>(col) < static_cast<unsigned>(G::N))
        atomicAdd(bf + smem_elem<LOGN>(col), __ldg(a.sp_values + base + k) * a.sp_scale);
    }
  }
  team_sync<G::T>(team);
  smem_get_B<LOGN>(buf, x, tau);
}
template <int LOGN>
__device__ __forceinline__ void scatter_rowB(float (&x)[Geom<LOGN>::E], const RowArgs& a, int64_t row, int tau,
                                             int team, float4* buf) {
  using G = Geom<LOGN>;
  int cols[kScatterPre];
  float vals[kScatterPre];
  const bool fast = a.nnz <= kScatterPre * G::T;
  if (fast) scatter_load<LOGN>(cols, vals, a, row, tau);
  scatter_apply<LOGN>(x, a, row, tau, team, buf, fast, cols, vals);
}

// Sparse adapter, backward: out[k] = (row transform * scale)[cols[k]].
// Up to kGatherPre column indices per thread are read before the row (see
// k_rows_a2b), so their latency overlaps the row's load and transform.
constexpr int kGatherPre = 4;
template <int LOGN>
__device__ __forceinline__ void gather_cols_pre(int (&cols)[kGatherPre], const RowArgs& a, int64_t row, int tau) {
  using G = Geom<LOGN>;
  const int64_t base = row * a.nnz;
#pragma unroll
  for (int j = 0; j < kGatherPre; ++j) {
    const int k = tau + j * G::T;
    cols[j] = k < a.nnz ? __ldg(a.sp_cols + base + k) : -1;
  }
}
template <int LOGN>
__device__ __forceinline__ void gather_rowB(const float (&x)[Geom<LOGN>::E], const RowArgs& a, int64_t row, int tau,
                                            int team, float4* buf, const int (&cols)[kGatherPre]) {
  using G = Geom<LOGN>;
  smem_put_B<LOGN>(buf, x, tau);
  team_sync<G::T>(team);
  const float* bf = reinterpret_cast<const float*>(buf);
  const int64_t base = row * a.nnz;
#pragma unroll
  for (int j = 0; j < kGatherPre; ++j) {
    const int k = tau + j * G::T;
    if (k < a.nnz) {
      float v = 0.0f;
      if (static_cast<unsigned>(cols[j]) < static_cast<unsigned>(G::N)) v = bf[smem_elem<LOGN>(cols[j])] * a.sp_scale;
      a.sp_out[base + k] = v;
    }
  }
  for (int k = tau + kGatherPre * G::T; k < a.nnz; k += G::T) {
    const int col = __ldg(a.sp_cols + base + k);
    float v = 0.0f;
    if (static_cast<unsigned>(col) < static_cast<unsigned>(G::N)) v = bf[smem_elem<LOGN>(col)] * a.sp_scale;
    a.sp_out[base + k] = v;
  }
}

enum { EPI_STORE = 0, EPI_QUANT = 1, EPI_GATHER = 2 };
enum { PRO_DEQUANT = 0, PRO_SCATTER = 1 };

// Dense rows in (layout A), transform, result in layout B.
template <int LOGN, typename Tin, typename Tout, int EPI, int BITS>
__global__ void __launch_bounds__(Geom<LOGN>::NT, Geom<LOGN>::MINB) k_rows_a2b(const RowArgs a) {
  using G = Geom<LOGN>;
  extern __shared__ float4 smem4[];
  const int tid = threadIdx.x;
  const int team = tid >> G::LOGT;
  const int tau = tid & (G::T - 1);
  const int64_t row = int64_t(blockIdx.x) * G::RPC + team;
  if (row >= a.rows) return;  // whole teams leave together
  float4* buf = smem4 + size_t(team) * (G::N / 4);

  float x[G::E];
  int gcols[kGatherPre];
  if constexpr (EPI == EPI_GATHER) gather_cols_pre<LOGN>(gcols, a, row, tau);
  load_rowA<LOGN, Tin>(x, static_cast<const Tin*>(a.x) + row * a.ldx, tau, a.pre_signs);
  reg_stages<G::E, 0, G::LOGE>(x);
  if constexpr (G::T > 1) {
    smem_put_A<LOGN>(buf, x, tau);
    team_sync<G::T>(team);
    smem_get_B<LOGN>(buf, x, tau);
    reg_stages<G::E, 2, G::B_FWD_HI>(x);
#pragma unroll
    for (int b = 0; b < G::NSH; ++b) shfl_stage<G::E>(x, b, (tau >> b) & 1);
  }
  if constexpr (EPI == EPI_STORE) {
    store_rowB<LOGN, Tout>(x, static_cast<Tout*>(a.y) + row * a.ldy, tau, a.norm, a.post_signs);
  } else if constexpr (EPI == EPI_QUANT) {
    quant_rowB<LOGN, BITS>(x, a, row, tau);
  } else {
    gather_rowB<LOGN>(x, a, row, tau, team, buf, gcols);
  }
}

// Rows produced in layout B (dequantized codes or a scattered sparse row),
// transform, dense result stored in layout A.
template <int LOGN, typename Tout, int PRO, int BITS>
__global__ void __launch_bounds__(Geom<LOGN>::NT, Geom<LOGN>::MINB) k_rows_b2a(const RowArgs a) {
  using G = Geom<LOGN>;
  extern __shared__ float4 smem4[];
  const int tid = threadIdx.x;
  const int team = tid >> G::LOGT;
  const int tau = tid & (G::T - 1);
  const int64_t row = int64_t(blockIdx.x) * G::RPC + team;
  if (row >= a.rows) return;
  float4* buf = smem4 + size_t(team) * (G::N / 4);

  float x[G::E];
  if constexpr (PRO == PRO_DEQUANT) {
    dequant_rowB<LOGN, BITS>(x, a, row, tau);
  } else {
    scatter_rowB<LOGN>(x, a, row, tau, team, buf);
  }
  reg_stages<G::E, 0, G::LOGE>(x);
  if constexpr (G::T > 1) {
#pragma unroll
    for (int b = 0; b < G::NSH; ++b) shfl_stage<G::E>(x, b, (tau >> b) & 1);
    smem_put_B<LOGN>(buf, x, tau);
    team_sync<G::T>(team);
    smem_get_A<LOGN>(buf, x, tau);
    reg_stages<G::E, G::A_INV_LO, G::LOGE>(x);
  }
  store_rowA<LOGN, Tout, false>(x, static_cast<Tout*>(a.y) + row * a.ldy, tau, 1.0f, a.post_signs);
}

// ----------------------------------------------------------------------------
// Host launch helpers.
// ----------------------------------------------------------------------------
// Opt a kernel into more than 48 KB of dynamic shared memory, once per device.
template <typename K>
inline cudaError_t set_smem_attr(K kernel, size_t smem, std::atomic<unsigned long long>& done_mask) {
  if (smem <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done_mask.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e == cudaSuccess) done_mask.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

template <int LOGN, typename Tin, typename Tout, int EPI, int BITS>
cudaError_t launch_a2b(const RowArgs& a, cudaStream_t st) {
  using G = Geom<LOGN>;
  static std::atomic<unsigned long long> done{0};
  auto kern = k_rows_a2b<LOGN, Tin, Tout, EPI, BITS>;
  const size_t smem = G::smem_bytes(EPI == EPI_GATHER);
  cudaError_t e = set_smem_attr(kern, smem, done);
  if (e != cudaSuccess) return e;
  const int64_t grid = (a.rows + G::RPC - 1) / G::RPC;
  kern<<<dim3(unsigned(grid)), G::NT, smem, st>>>(a);
  return cudaGetLastError();
}

template <int LOGN, typename Tout, int PRO, int BITS>
cudaError_t launch_b2a(const RowArgs& a, cudaStream_t st) {
  using G = Geom<LOGN>;
  static std::atomic<unsigned long long> done{0};
  auto kern = k_rows_b2a<LOGN, Tout, PRO, BITS>;
  const size_t smem = G::smem_bytes(PRO == PRO_SCATTER);
  cudaError_t e = set_smem_attr(kern, smem, done);
  if (e != cudaSuccess) return e;
  const int64_t grid = (a.rows + G::RPC - 1) / G::RPC;
  kern<<<dim3(unsigned(grid)), G::NT, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace hit
