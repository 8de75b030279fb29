// Device helpers shared by the kernels of libhit.so (sm_100a only).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libhit targets sm_100a (Blackwell) only"
#endif

namespace hit {

// ---------------------------------------------------------------------------
// Packed fp32 pairs.  sm_100a executes add/sub/fma on two fp32 lanes held in
// one 64-bit register pair, halving the issue slots of the butterfly stages.
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned long long pk2(float a, float b) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk2(unsigned long long r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}

// (a, b) <- (a + b, a - b) on two element pairs {a0,a1} and {b0,b1}.
__device__ __forceinline__ void bfly_x2(float& a0, float& a1, float& b0, float& b1) {
  unsigned long long A = pk2(a0, a1), B = pk2(b0, b1), S, D;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(S) : "l"(A), "l"(B));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(D) : "l"(A), "l"(B));
  upk2(S, a0, a1);
  upk2(D, b0, b1);
}
__device__ __forceinline__ void bfly_x1(float& a, float& b) {
  const float s = a + b, d = a - b;
  a = s;
  b = d;
}
// {a0, a1} *= {m0, m1}
__device__ __forceinline__ void mul_x2(float& a0, float& a1, float m0, float m1) {
  unsigned long long A = pk2(a0, a1), M = pk2(m0, m1), R;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(R) : "l"(A), "l"(M));
  upk2(R, a0, a1);
}

// {d0, d1} = {a0, a1} * {b0, b1} + {c0, c1}, one rounding per lane
__device__ __forceinline__ void fma_x2(float a0, float a1, float b0, float b1, float c0, float c1, float& d0,
                                       float& d1) {
  unsigned long long A = pk2(a0, a1), B = pk2(b0, b1), C = pk2(c0, c1), D;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(D) : "l"(A), "l"(B), "l"(C));
  upk2(D, d0, d1);
}
// {d0, d1} = {a0, a1} - {b0, b1}
__device__ __forceinline__ void sub_x2(float a0, float a1, float b0, float b1, float& d0, float& d1) {
  unsigned long long A = pk2(a0, a1), B = pk2(b0, b1), D;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(D) : "l"(A), "l"(B));
  upk2(D, d0, d1);
}

// One Hadamard stage on register-index bit Q of a thread-private array: for
// every r with bit Q clear, (x[r], x[r + 2^Q]) <- (x[r] + x[r+2^Q], x[r] - x[r+2^Q]).
template <int E, int Q>
__device__ __forceinline__ void reg_stage(float (&x)[E]) {
  constexpr int h = 1 << Q;
  if constexpr (Q == 0) {
#pragma unroll
    for (int r = 0; r < E; r += 2) bfly_x1(x[r], x[r + 1]);
  } else {
#pragma unroll
    for (int r = 0; r < E; r += 2 * h) {
#pragma unroll
      for (int u = 0; u < h; u += 2) bfly_x2(x[r + u], x[r + u + 1], x[r + u + h], x[r + u + h + 1]);
    }
  }
}
// Stages on register bits [LO, HI).
template <int E, int LO, int HI>
__device__ __forceinline__ void reg_stages(float (&x)[E]) {
  if constexpr (LO < HI) {
    reg_stage<E, LO>(x);
    reg_stages<E, LO + 1, HI>(x);
  }
}

// Stage on thread bit `bit` (partner lane = lane ^ 2^bit, same warp).
template <int E>
__device__ __forceinline__ void shfl_stage(float (&x)[E], int bit, bool upper) {
  const int m = 1 << bit;
#pragma unroll
  for (int r = 0; r < E; ++r) {
    const float v = __shfl_xor_sync(0xffffffffu, x[r], m);
    x[r] = upper ? (v - x[r]) : (x[r] + v);
  }
}

// ---------------------------------------------------------------------------
// Sign flips from int8 +-1 signs packed four per 32-bit word (byte c = element
// c).  The sign bit of byte c is moved to bit 31 and xor-ed into the float.
// ---------------------------------------------------------------------------
template <int C>
__device__ __forceinline__ float apply_sign_byte(float v, uint32_t w) {
  const uint32_t m = (w << (24 - 8 * C)) & 0x80000000u;
  return __uint_as_float(__float_as_uint(v) ^ m);
}
__device__ __forceinline__ void apply_sign4(float& a, float& b, float& c, float& d, uint32_t w) {
  a = apply_sign_byte<0>(a, w);
  b = apply_sign_byte<1>(b, w);
  c = apply_sign_byte<2>(c, w);
  d = apply_sign_byte<3>(d, w);
}

// ---------------------------------------------------------------------------
// bf16 <-> fp32
// ---------------------------------------------------------------------------
__device__ __forceinline__ void bf16x2_to_f32(uint32_t w, float& lo, float& hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xffff0000u);
}
__device__ __forceinline__ uint32_t f32_to_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------------------------
// Streaming global memory access (read-once inputs, write-once outputs).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float4 ld_stream_f4(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ uint2 ld_stream_u2(const void* p) { return __ldcs(reinterpret_cast<const uint2*>(p)); }
__device__ __forceinline__ void st_stream_f4(float* p, float4 v) { __stcs(reinterpret_cast<float4*>(p), v); }
__device__ __forceinline__ void st_stream_u2(void* p, uint2 v) { __stcs(reinterpret_cast<uint2*>(p), v); }
// 32-byte streaming store (one whole sector per thread); p must be 32-byte aligned.
__device__ __forceinline__ void st_stream_v8(void* p, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t a4,
                                             uint32_t a5, uint32_t a6, uint32_t a7) {
  asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a0), "r"(a1), "r"(a2),
               "r"(a3), "r"(a4), "r"(a5), "r"(a6), "r"(a7)
               : "memory");
}

// ---------------------------------------------------------------------------
// Row-buffer swizzle for the register-layout transposes.  The buffer is
// addressed in 16-byte chunks q; chunk q lives at q ^ ((q >> LQ) & 7).  With
// LQ = log2(elements per thread / 4) >= 3 both the "consecutive chunks per
// consecutive thread" and the "one contiguous run of chunks per thread"
// access patterns hit 8 distinct 16-byte bank groups per quarter warp.
// ---------------------------------------------------------------------------
template <int LQ>
__device__ __forceinline__ int swz(int q) {
  return q ^ ((q >> LQ) & 7);
}

// ---------------------------------------------------------------------------
// Code packing.  Inputs are the raw bit patterns of floats whose low byte
// holds a stored code u (see the quantizer); only that byte is used.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t low_bytes4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}
// 8 four-bit codes -> one word, element e at bits [4e, 4e+4).
__device__ __forceinline__ uint32_t pack4x8(const uint32_t* u) {
  const uint32_t ev = low_bytes4(u[0], u[2], u[4], u[6]);
  const uint32_t od = low_bytes4(u[1], u[3], u[5], u[7]);
  return ev | (od << 4);
}
// 16 two-bit codes -> one word, element e at bits [2e, 2e+2).
__device__ __forceinline__ uint32_t pack2x16(const uint32_t* u) {
  const uint32_t a = low_bytes4(u[0], u[4], u[8], u[12]);
  const uint32_t b = low_bytes4(u[1], u[5], u[9], u[13]);
  const uint32_t c = low_bytes4(u[2], u[6], u[10], u[14]);
  const uint32_t d = low_bytes4(u[3], u[7], u[11], u[15]);
  return a | (b << 2) | (c << 4) | (d << 6);
}
// 4 three-bit codes (low bytes of a word) -> 12 bits.
__device__ __forceinline__ uint32_t squeeze3x4(uint32_t w) {
  const uint32_t p = (w & 0x00070007u) | ((w >> 5) & 0x00380038u);
  return (p & 0x3fu) | ((p >> 10) & 0xfc0u);
}
// 32 three-bit codes -> three words (96-bit stream), element e at bits [3e, 3e+3).
__device__ __forceinline__ void pack3x32(const uint32_t* u, uint32_t* w) {
  uint32_t v[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t lo = squeeze3x4(low_bytes4(u[8 * k + 0], u[8 * k + 1], u[8 * k + 2], u[8 * k + 3]));
    const uint32_t hi = squeeze3x4(low_bytes4(u[8 * k + 4], u[8 * k + 5], u[8 * k + 6], u[8 * k + 7]));
    v[k] = lo | (hi << 12);
  }
  w[0] = v[0] | (v[1] << 24);
  w[1] = (v[1] >> 8) | (v[2] << 16);
  w[2] = (v[2] >> 16) | (v[3] << 8);
}

// Stored code e of a packed stream (bits per code B), returned as uint32.
template <int B>
__device__ __forceinline__ uint32_t code_at(const uint32_t* w, int e) {
  const int bit = B * e;
  const int wi = bit >> 5, sh = bit & 31;
  uint32_t v = w[wi] >> sh;
  if (sh + B > 32) v |= w[wi + 1] << (32 - sh);
  return v & ((1u << B) - 1u);
}

}  // namespace hit

namespace hit {
// ---------------------------------------------------------------------------
// mbarrier + 1-D bulk async copy (TMA) helpers.  Every wait is bounded in
// time: it gives up after about two seconds (global timer) and reports
// failure to the caller, which records it in a device counter and stops.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Time limit of every production wait: far above any legitimate wait (a copy
// lands in microseconds), short enough that a lost completion ends the kernel.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
// Wait for phase `parity` of an mbarrier; false once `limit_ns` has passed.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0 && global_ns() - t0 > limit_ns) return false;
  }
}
// global -> shared bulk copy; dst and src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// order this thread's generic-proxy shared-memory accesses before later async-proxy (TMA) writes
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
}  // namespace hit
