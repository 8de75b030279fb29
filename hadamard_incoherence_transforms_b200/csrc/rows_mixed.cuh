// Fused randomized transform + 4-bit group quantization for rows of the
// non-power-of-two length d = 5120 = 8 * 8 * 8 * 5 * 2.
//
// HARP explainer, technical summary §2.1: dimensions that are not powers of two
// (5120 with the schedule (8, 8, 8, 5, 2)) are handled by a mixed-radix stride
// schedule whose non-power-of-two radices use orthogonal QR-of-Gaussian mixers.
// With the Hadamard blocks H_b / sqrt(b) for the power-of-two radices and one
// shared 5 x 5 mixer G_5, the stage product is the Kronecker product
//     R = (H_512 / sqrt 512) (x) G_5 (x) (H_2 / sqrt 2)
// on the index i = 10 j + 2 i3 + i4 (j < 512, i3 < 5, i4 < 2): the three radix-8
// stages together are the Sylvester H_512 on j, so the stages commute and can
// run in any order.  y = R diag(s) x; the factor 1/sqrt(1024) = 1/32 is exact
// and folded into the mixer coefficients, which ride in the kernel parameters.
//
// One warp per row, 160 values per lane, rows streamed through a ring of
// shared-memory slots by bulk copies (four quarter copies per row, one mbarrier
// each), a producer warp and seven consumer warps per CTA (the protocol of the
// power-of-two streaming kernel; every wait bounded).
//   layout A: lane = 2 jg + i4 holds j = jg + 16 a (a = 0..31) for i3 = 0..4 in
//             v[32 i3 + a] (conflict-free 32-bit reads of the landed row);
//             signs, G_5 on i3, WHT over a (j bits 4..8);
//   transpose through the row's own slot (16-byte chunk index xor (a & 7));
//   layout B: lane t holds elements 160 t .. 160 t + 159, v[10 b + r] with
//             j = 16 t + b; WHT over b (j bits 0..3), then H_2 on i4;
//   quantize: every 32-element chunk lies inside one group of 128; a lane's
//             first 4 - (t & 3) chunks belong to group (5 t) / 4, the rest to
//             the next one; the two partial group maxima meet the neighbouring
//             lanes' by one shuffle each way.
#pragma once
#include "rows_ops.cuh"

namespace hit {

__device__ unsigned int g_wait_timeouts_mixed = 0;

struct MixArgs {
  const float* x = nullptr;       // [rows, ldx] fp32
  int64_t rows = 0, ldx = 0;      // ldx in elements, multiple of 4
  const int8_t* signs = nullptr;  // [5120] +-1, or NULL
  float g5[25] = {};              // G_5 row-major, times 1/32
  uint8_t* codes = nullptr;       // [rows, 2560]
  float* scales = nullptr;        // [rows, 40]
};

struct MixCfg {
  static constexpr int N = 5120;
  static constexpr int E = 160;
  static constexpr int NCW = 7;  // consumer warps, one row each
  static constexpr int THREADS = (NCW + 1) * 32;
  static constexpr uint32_t ROW = uint32_t(N) * 4;
  static constexpr int NQ = 4;
  static constexpr uint32_t QROW = ROW / NQ;
  static constexpr uint32_t SMEM_MAX = 232448;
  static constexpr int S = int((SMEM_MAX - 1024) / ROW);
  static constexpr size_t SMEM = 1024 + size_t(S) * ROW;
  static_assert(S + 1 >= NCW, "ring too shallow for the ticket protocol");
  static_assert(S <= 32, "the ramp issues one slot per producer lane");
  static_assert((NQ + 1) * S * 8 + 8 <= 1024, "barriers fit in the first kilobyte");
  static_assert(QROW % 16 == 0, "quarter copies are whole 16-byte units");
};

__global__ void __launch_bounds__(MixCfg::THREADS, 1) k_rows_mixed5120_q4(const MixArgs a) {
  using C = MixCfg;
  constexpr int BITS = 4;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + C::S * C::NQ;
  int* ticket = reinterpret_cast<int*>(empty + C::S);
  uint8_t* slots = smem + 1024;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // programmatic dependent launch: the CTA may start while the previous kernel
  // in the stream finishes; every global access comes after griddepcontrol.wait
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::S; ++s) {
      for (int q = 0; q < C::NQ; ++q) mbar_init(&full[s * C::NQ + q], 1);
      mbar_init(&empty[s], 1);
    }
    ticket[0] = 0;
    mbar_init_fence();
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __syncthreads();
  const int64_t grid = gridDim.x;
  const int64_t nrows = a.rows > blockIdx.x ? (a.rows - blockIdx.x + grid - 1) / grid : 0;

  if (warp == C::NCW) {  // producer: row k of this CTA goes to slot k % S
    const uint8_t* src = reinterpret_cast<const uint8_t*>(a.x);
    auto issue_q = [&](int64_t k, int q) {
      const int s = int(k % C::S);
      const int64_t row = blockIdx.x + k * grid;
      mbar_expect_tx(&full[s * C::NQ + q], C::QROW);
      bulk_g2s(slots + size_t(s) * C::ROW + size_t(q) * C::QROW, src + row * a.ldx * 4 + size_t(q) * C::QROW, C::QROW,
               &full[s * C::NQ + q]);
    };
    auto issue = [&](int64_t k) {
#pragma unroll
      for (int q = 0; q < C::NQ; ++q) issue_q(k, q);
    };
    // first wave quarter by quarter from parallel lanes, the rest of the ring
    // once the first row has landed
    const int64_t wave1 = nrows < C::NCW ? nrows : C::NCW;
    const int64_t wave2 = nrows < C::S ? nrows : C::S;
#pragma unroll
    for (int q = 0; q < C::NQ; ++q) {
      if (lane < wave1) issue_q(lane, q);
      __syncwarp();
    }
    bool ok = true;
    if (wave2 > wave1) {
      if (lane == 0) ok = mbar_wait(&full[C::NQ - 1], 0u);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok && lane >= wave1 && lane < wave2) issue(lane);
      __syncwarp();
    }
    if (lane == 0) {
      int64_t issued = ok ? wave2 : wave1;
      if (!ok) atomicAdd(&g_wait_timeouts_mixed, 1u);
      for (int64_t k = issued; ok && k < nrows; ++k) {
        if (!mbar_wait(&empty[k % C::S], uint32_t((k / C::S) - 1) & 1u)) {
          atomicAdd(&g_wait_timeouts_mixed, 1u);
          break;
        }
        issue(k);
        issued = k + 1;
      }
      // do not leave while a copy into this CTA's shared memory is in flight
      for (int64_t k = issued > C::S ? issued - C::S : 0; k < issued; ++k)
        for (int q = 0; q < C::NQ; ++q)
          if (!mbar_wait(&full[(k % C::S) * C::NQ + q], uint32_t(k / C::S) & 1u))
            atomicAdd(&g_wait_timeouts_mixed, 1u);
    }
    return;
  }

  // Per-lane constants: sign masks (bit a of m[i3] = sign of column
  // 10 (jg + 16 a) + 2 i3 + i4) and the layout-A word offset.
  const int jg = lane >> 1;
  const int baseA = 10 * jg + (lane & 1);
  uint32_t m[5];
#pragma unroll
  for (int i3 = 0; i3 < 5; ++i3) {
    uint32_t w = 0;
    if (a.signs != nullptr)
      for (int aa = 0; aa < 32; ++aa) w |= uint32_t(a.signs[baseA + 160 * aa + 2 * i3] < 0) << aa;
    m[i3] = w;
  }
  const int keyB = lane & 7;

  for (;;) {
    int tk = 0;
    if (lane == 0) tk = atomicAdd(ticket, 1);
    const int64_t k = __shfl_sync(0xffffffffu, tk, 0);
    if (k >= nrows) break;
    const int s = int(k % C::S);
    const int64_t row = blockIdx.x + k * grid;
    float* slot = reinterpret_cast<float*>(slots + size_t(s) * C::ROW);
    float v[C::E];
    bool stop = false;
    // ---- layout A, quarter by quarter (quarter q holds a in [8q, 8q + 8)) ----
#pragma unroll
    for (int q = 0; q < C::NQ; ++q) {
      if (!mbar_wait(&full[s * C::NQ + q], uint32_t(k / C::S) & 1u)) {
        if (lane == 0) atomicAdd(&g_wait_timeouts_mixed, 1u);
        stop = true;
        break;
      }
#pragma unroll
      for (int aa = 8 * q; aa < 8 * q + 8; ++aa) {
#pragma unroll
        for (int i3 = 0; i3 < 5; ++i3) {
          uint32_t mk = m[i3];
          asm volatile("mov.b32 %0, %0;" : "+r"(mk));  // keep the shifted masks out of registers across rows
          const float u = slot[baseA + 160 * aa + 2 * i3];
          v[32 * i3 + aa] = __uint_as_float(__float_as_uint(u) ^ ((mk << (31 - aa)) & 0x80000000u));
        }
      }
      // G_5 / 32 on i3, two a-values per packed fma
#pragma unroll
      for (int aa = 8 * q; aa < 8 * q + 8; aa += 2) {
        float i0[5], i1[5];
#pragma unroll
        for (int i3 = 0; i3 < 5; ++i3) {
          i0[i3] = v[32 * i3 + aa];
          i1[i3] = v[32 * i3 + aa + 1];
        }
#pragma unroll
        for (int o = 0; o < 5; ++o) {
          float r0 = i0[0], r1 = i1[0];
          mul_x2(r0, r1, a.g5[5 * o], a.g5[5 * o]);
#pragma unroll
          for (int kk = 1; kk < 5; ++kk) fma_x2(i0[kk], i1[kk], a.g5[5 * o + kk], a.g5[5 * o + kk], r0, r1, r0, r1);
          v[32 * o + aa] = r0;
          v[32 * o + aa + 1] = r1;
        }
      }
#pragma unroll
      for (int i3 = 0; i3 < 5; ++i3) reg_stages<8, 0, 3>(*reinterpret_cast<float(*)[8]>(v + 32 * i3 + 8 * q));
    }
    if (stop) return;
#pragma unroll
    for (int i3 = 0; i3 < 5; ++i3) reg_stages<32, 3, 5>(*reinterpret_cast<float(*)[32]>(v + 32 * i3));
    __syncwarp();  // every lane has read its layout-A words of this slot
    // ---- transpose: element (i3, a) to word 4 (c0 ^ (a & 7)) + w + 160 a ----
#pragma unroll
    for (int sw = 0; sw < 8; ++sw) {
#pragma unroll
      for (int i3 = 0; i3 < 5; ++i3) {
        const int li = baseA + 2 * i3;
        const int p = 4 * ((li >> 2) ^ sw) + (li & 3);
#pragma unroll
        for (int aa = sw; aa < 32; aa += 8) slot[p + 160 * aa] = v[32 * i3 + aa];
      }
    }
    __syncwarp();
    // ---- layout B: chunks 40 t + (kk ^ (t & 7)) ----
    const float4* s4 = reinterpret_cast<const float4*>(slot) + 40 * lane;
#pragma unroll
    for (int kk = 0; kk < 40; ++kk) {
      const float4 f = s4[(kk & ~7) | ((kk & 7) ^ keyB)];
      v[4 * kk] = f.x;
      v[4 * kk + 1] = f.y;
      v[4 * kk + 2] = f.z;
      v[4 * kk + 3] = f.w;
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    // WHT over b (element stride 10), packed over r pairs
#pragma unroll
    for (int L = 0; L < 4; ++L) {
#pragma unroll
      for (int b = 0; b < 16; ++b) {
        if ((b >> L) & 1) continue;
#pragma unroll
        for (int r = 0; r < 10; r += 2)
          bfly_x2(v[10 * b + r], v[10 * b + r + 1], v[10 * (b + (1 << L)) + r], v[10 * (b + (1 << L)) + r + 1]);
      }
    }
    // H_2 on i4
#pragma unroll
    for (int e = 0; e < C::E; e += 2) bfly_x1(v[e], v[e + 1]);

    // ---- quantize: two groups per lane ----
    float mx[5];
#pragma unroll
    for (int cc = 0; cc < 5; ++cc) {
      float t[8];
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        t[kk] = fmaxf(fmaxf(fabsf(v[32 * cc + kk]), fabsf(v[32 * cc + 8 + kk])),
                      fmaxf(fabsf(v[32 * cc + 16 + kk]), fabsf(v[32 * cc + 24 + kk])));
      mx[cc] = fmaxf(fmaxf(fmaxf(t[0], t[1]), fmaxf(t[2], t[3])), fmaxf(fmaxf(t[4], t[5]), fmaxf(t[6], t[7])));
    }
    const int ph = lane & 3;
    const int nl = 4 - ph;  // chunks in the left group
    float lm = 0.0f, rm = 0.0f;
#pragma unroll
    for (int cc = 0; cc < 5; ++cc) {
      if (cc < nl) lm = fmaxf(lm, mx[cc]);
      else rm = fmaxf(rm, mx[cc]);
    }
    const float up = __shfl_up_sync(0xffffffffu, rm, 1);
    const float dn = __shfl_down_sync(0xffffffffu, lm, 1);
    const float mL = ph != 0 ? fmaxf(lm, up) : lm;
    const float mR = ph != 3 ? fmaxf(rm, dn) : rm;
    const int gL = (5 * lane) >> 2;
    const float sL = group_scale<BITS>(mL), sR = group_scale<BITS>(mR);
    if (ph == 0) a.scales[row * 40 + gL] = sL;
    a.scales[row * 40 + gL + 1] = sR;
    uint8_t* dst = a.codes + row * 2560 + 80 * lane;
#pragma unroll
    for (int cc = 0; cc < 5; ++cc) {
      const float sg = cc < nl ? sL : sR;
      const float kf = sg < 0x1p-100f ? 0x1p100f : (sg > 0x1p100f ? 0x1p-100f : 1.0f);
      const float ss = sg * kf;
      const float rr = sg > 0.0f ? __frcp_rn(ss) : 0.0f;
      const float sx = sg > 0.0f ? ss : 1.0f;
      float* xc = v + 32 * cc;
      if (kf != 1.0f) {
#pragma unroll
        for (int e = 0; e < 32; e += 2) mul_x2(xc[e], xc[e + 1], kf, kf);
      }
      uint32_t W[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t ub[8];
        quant8<BITS>(xc + 8 * q, sx, rr, ub);
        W[q] = pack4x8(ub);
      }
      __stcs(reinterpret_cast<uint4*>(dst) + cc, make_uint4(W[0], W[1], W[2], W[3]));
    }
  }
}

inline cudaError_t launch_mixed5120_q4(const MixArgs& a, cudaStream_t st) {
  using C = MixCfg;
  static std::atomic<unsigned long long> done{0};
  cudaError_t e = set_smem_attr(k_rows_mixed5120_q4, C::SMEM, done);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int64_t grid = a.rows < sms ? a.rows : sms;
  if (grid == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid));
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_rows_mixed5120_q4, a);
}

}  // namespace hit
