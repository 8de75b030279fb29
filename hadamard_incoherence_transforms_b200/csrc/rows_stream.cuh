// Persistent, TMA-fed row kernel for long rows (n = 4096 / 8192, one or two
// warps per row).
//
// One CTA per SM.  A producer warp keeps a ring of S shared-memory row slots
// full with 1-D bulk async copies (cp.async.bulk, completion counted on an
// mbarrier per slot); consumer warps take rows from the ring in order.  A
// consumer team reads its row from the slot in layout A (4-element vectors,
// conflict-free), runs the layout-A stages in registers, writes the values
// back transposed into the same slot (swizzled), reads layout B, finishes the
// stages, releases the slot to the producer and runs the epilogue (store or
// quantize + pack) from registers.  Rows in flight per SM = slots being
// filled, so the HBM pipe stays busy while other rows are being computed.
// Each row is copied as four quarter-row copies with a barrier each, and the
// first wave is issued quarter by quarter: a team runs the layout-A stages
// that stay inside a quarter (register bits 0..4) as soon as that quarter has
// landed, so the first round of rows does not wait for whole rows.
// Every mbarrier wait is bounded; a wait that gives up bumps a device
// counter and the warp stops.
#pragma once
#include "rows_ops.cuh"

namespace hit {

__device__ unsigned int g_wait_timeouts = 0;

// Warps per CTA: one producer plus consumers.  Eight warps keep two warps per
// SM sub-partition, which leaves each thread the full 255 registers for its
// row elements.
#ifndef HIT_STREAM_WARPS
#define HIT_STREAM_WARPS 8
#endif

// Ring protocol.  The producer copies this CTA's rows k = 0, 1, 2, ... in
// order into slot k % S, refilling a slot only after its "empty" barrier has
// completed the previous phase.  Consumer teams take rows by ticket: a team
// draws the next k from a shared counter when it starts a row, so tickets in
// use are handed out in increasing order and every team holds one at a time.
// A parity wait for row k on slot k % S could only be fooled if row k - S had
// not been copied yet; the producer would then be stalled at some row r <= k - S
// whose slot is held by ticket r - S, and every ticket in [r, k] would belong
// to a team blocked on an uncopied row, i.e. S + 2 teams at least.  So any ring
// with S >= TEAMS - 1 is safe, and the ring takes every slot that fits.
template <int LOGN, typename Tin>
struct StreamCfg {
  using G = Geom<LOGN>;
  static_assert(G::T == 32 || G::T == 64, "streaming kernel needs one or two warps per row");
  static constexpr int WPR = G::T / 32;                        // warps per row
  static constexpr int NCW = ((HIT_STREAM_WARPS - 1) / WPR) * WPR;  // consumer warps
  static constexpr int TEAMS = NCW / WPR;                      // rows in compute at once
  static constexpr uint32_t SLOT = uint32_t(G::N) * 4;         // fp32 row (transpose space)
  static constexpr uint32_t ROW = uint32_t(G::N) * sizeof(Tin);
  static constexpr uint32_t SIGNS = uint32_t(G::N) * 4;        // sign-bit mask per column
  static constexpr uint32_t SMEM_MAX = 232448;                 // opt-in limit per CTA on sm_100
  static constexpr int S = int((SMEM_MAX - 1024 - SIGNS) / SLOT);  // ring depth
  static constexpr int NQ = 4;                                 // quarter copies per row
  static constexpr uint32_t QROW = ROW / NQ;
  static constexpr size_t SMEM = 1024 + SIGNS + size_t(S) * SLOT;
  static constexpr int THREADS = (NCW + 1) * 32;
  static constexpr int BAR_CONSUMERS = 15;                     // named barrier of all consumer warps
  static_assert(TEAMS >= 1 && S + 1 >= TEAMS, "ring too shallow for the ticket protocol");
  static_assert(TEAMS + 1 < BAR_CONSUMERS, "named barrier ids");
  static_assert(S <= 32, "the ramp issues one ring slot per producer lane");
  static_assert((NQ + 1) * S * 8 + 8 + 4 * TEAMS <= 1024, "barriers and tickets must fit in the first kilobyte");
  static_assert(QROW % 16 == 0, "quarter copies are whole 16-byte units");
  static_assert(G::E == 128, "quarters are the 32-register blocks of layout A");
};

template <int LOGN, typename Tin>
__device__ __forceinline__ void stream_team_sync(int team) {
  if constexpr (StreamCfg<LOGN, Tin>::WPR == 1) {
    __syncwarp();
  } else {
    asm volatile("bar.sync %0, %1;" ::"r"(team + 1), "r"(Geom<LOGN>::T) : "memory");
  }
}

// The sign vector as sign-bit masks (0 or 0x80000000 per column), one
// shared-memory table per CTA.  Each consumer thread loads its (at most two)
// 16-byte pieces of the int8 signs before the producer starts its copies, so
// these loads are not queued behind the first wave of row copies.
template <int N, int NTHREADS>
struct SignLoad {
  static constexpr int PIECES = N / 16;
  static constexpr int PER = (PIECES + NTHREADS - 1) / NTHREADS;
  uint4 v[PER];
  __device__ __forceinline__ void load(const int8_t* __restrict__ s, int t) {
    if ((reinterpret_cast<uintptr_t>(s) & 15) != 0) return;  // unaligned signs: store() reads bytes
#pragma unroll
    for (int p = 0; p < PER; ++p)
      if (t + p * NTHREADS < PIECES) v[p] = __ldg(reinterpret_cast<const uint4*>(s) + t + p * NTHREADS);
  }
  __device__ __forceinline__ void store(uint32_t* sgn, const int8_t* __restrict__ s, int t) const {
    if ((reinterpret_cast<uintptr_t>(s) & 15) != 0) {
      for (int i = t; i < N; i += NTHREADS) sgn[i] = s[i] < 0 ? 0x80000000u : 0u;
      return;
    }
#pragma unroll
    for (int p = 0; p < PER; ++p) {
      const int i = t + p * NTHREADS;
      if (i >= PIECES) break;
      const uint32_t w[4] = {v[p].x, v[p].y, v[p].z, v[p].w};
#pragma unroll
      for (int k = 0; k < 4; ++k)
        reinterpret_cast<uint4*>(sgn)[4 * i + k] =
            make_uint4((w[k] << 24) & 0x80000000u, (w[k] << 16) & 0x80000000u, (w[k] << 8) & 0x80000000u,
                       w[k] & 0x80000000u);
    }
  }
};

template <int LOGN, typename Tin, typename Tout, int EPI, int BITS, bool SIGNS>
__global__ void __launch_bounds__(StreamCfg<LOGN, Tin>::THREADS, 1) k_rows_stream(const RowArgs a) {
  using G = Geom<LOGN>;
  using C = StreamCfg<LOGN, Tin>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);  // [S][NQ], one per quarter copy
  uint64_t* empty = full + C::S * C::NQ;
  int* ticket = reinterpret_cast<int*>(empty + C::S);
  volatile int* abort = ticket + 1;
  int* team_ticket = ticket + 2;
  uint32_t* sgn = reinterpret_cast<uint32_t*>(smem + 1024);
  uint8_t* slots = smem + 1024 + C::SIGNS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Launched as a programmatic dependent of the previous kernel in the stream:
  // this CTA may start while that kernel's last CTAs still run (it only needs
  // the SM), so it lets the next launch do the same, sets up its barriers,
  // and waits for the previous kernel to complete (and its writes to become
  // visible) before its first global-memory access.  Launched without that
  // attribute, both instructions do nothing.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::S; ++s) {
      for (int q = 0; q < C::NQ; ++q) mbar_init(&full[s * C::NQ + q], 1);
      mbar_init(&empty[s], C::WPR);
    }
    ticket[0] = 0;
    ticket[1] = 0;
    mbar_init_fence();
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  SignLoad<G::N, C::NCW * 32> sl;
  if (SIGNS && warp < C::NCW) sl.load(a.pre_signs, threadIdx.x);
  __syncthreads();
  const int64_t grid = gridDim.x;
  const int64_t nrows = a.rows > blockIdx.x ? (a.rows - blockIdx.x + grid - 1) / grid : 0;

  if (warp == C::NCW) {  // producer
    const uint8_t* src = static_cast<const uint8_t*>(a.x);
    auto issue_q = [&](int64_t k, int q) {
      const int s = int(k % C::S);
      const int64_t row = blockIdx.x + k * grid;
      mbar_expect_tx(&full[s * C::NQ + q], C::QROW);
      bulk_g2s(slots + size_t(s) * C::SLOT + size_t(q) * C::QROW,
               src + row * a.ldx * int64_t(sizeof(Tin)) + size_t(q) * C::QROW, C::QROW, &full[s * C::NQ + q]);
    };
    auto issue = [&](int64_t k) {
#pragma unroll
      for (int q = 0; q < C::NQ; ++q) issue_q(k, q);
    };
    // Ramp: one row per team from parallel lanes, quarter by quarter (all
    // first quarters, then all second quarters, ...), and the rest of the
    // ring once the first row has landed (a smaller first wave arrives sooner).
    const int64_t wave1 = nrows < C::TEAMS ? nrows : C::TEAMS;
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
      if (!ok) atomicAdd(&g_wait_timeouts, 1u);
      for (int64_t k = issued; ok && k < nrows; ++k) {
        if (!mbar_wait(&empty[k % C::S], uint32_t((k / C::S) - 1) & 1u)) {
          atomicAdd(&g_wait_timeouts, 1u);
          break;
        }
        issue(k);
        issued = k + 1;
      }
      // Do not leave while a copy into this CTA's shared memory is in flight.
      for (int64_t k = issued > C::S ? issued - C::S : 0; k < issued; ++k)
        for (int q = 0; q < C::NQ; ++q)
          if (!mbar_wait(&full[(k % C::S) * C::NQ + q], uint32_t(k / C::S) & 1u)) atomicAdd(&g_wait_timeouts, 1u);
    }
    return;
  }

  if constexpr (SIGNS) {
    sl.store(sgn, a.pre_signs, threadIdx.x);
    asm volatile("bar.sync %0, %1;" ::"r"(C::BAR_CONSUMERS), "r"(C::NCW * 32) : "memory");
  }
  const int team = warp / C::WPR;
  const int tau = (warp % C::WPR) * 32 + lane;
  for (;;) {
    int64_t k;
    if constexpr (C::WPR == 1) {
      int t = 0;
      if (lane == 0) t = atomicAdd(ticket, 1);
      k = __shfl_sync(0xffffffffu, t, 0);
    } else {
      // The leader's write for the next row comes after this row's two team
      // barriers, so the partner warp has read this value by then.
      if (tau == 0) team_ticket[team] = atomicAdd(ticket, 1);
      stream_team_sync<LOGN, Tin>(team);
      k = *abort ? nrows : team_ticket[team];
    }
    if (k >= nrows) break;
    const int s = int(k % C::S);
    const int64_t row = blockIdx.x + k * grid;
    uint8_t* slot = slots + size_t(s) * C::SLOT;
    float x[G::E];
    // Layout A straight from the copied row (linear layout), one quarter at a
    // time: quarter q holds vectors j = 8q .. 8q+7, i.e. registers 32q .. 32q+31,
    // and register bits 0..4 stay inside a quarter.
    bool stop = false;
#pragma unroll
    for (int q = 0; q < C::NQ; ++q) {
      if (!mbar_wait(&full[s * C::NQ + q], uint32_t(k / C::S) & 1u)) {
        if (lane == 0) atomicAdd(&g_wait_timeouts, 1u);
        // A one-warp team stops.  A two-warp team finishes the row (its
        // partner is at the same team barriers) and both warps stop at the
        // next ticket; the row's output is then undefined and the counter
        // says so.
        if constexpr (C::WPR == 1) stop = true;
        else *abort = 1;
      }
      if constexpr (C::WPR == 1) {
        if (stop) break;
      }
#pragma unroll
      for (int j = 8 * q; j < 8 * q + 8; ++j) {
        const int i0 = 4 * (tau + G::T * j);
        if constexpr (std::is_same<Tin, float>::value) {
          const float4 v = reinterpret_cast<const float4*>(slot)[i0 >> 2];
          x[4 * j] = v.x;
          x[4 * j + 1] = v.y;
          x[4 * j + 2] = v.z;
          x[4 * j + 3] = v.w;
        } else {
          const uint2 v = reinterpret_cast<const uint2*>(slot)[i0 >> 2];
          bf16x2_to_f32(v.x, x[4 * j], x[4 * j + 1]);
          bf16x2_to_f32(v.y, x[4 * j + 2], x[4 * j + 3]);
        }
        if constexpr (SIGNS) {  // xor of the sign bit runs on the integer pipe, not the FP32 pipe
          const uint4 sv = reinterpret_cast<const uint4*>(sgn)[i0 >> 2];
          x[4 * j] = __uint_as_float(__float_as_uint(x[4 * j]) ^ sv.x);
          x[4 * j + 1] = __uint_as_float(__float_as_uint(x[4 * j + 1]) ^ sv.y);
          x[4 * j + 2] = __uint_as_float(__float_as_uint(x[4 * j + 2]) ^ sv.z);
          x[4 * j + 3] = __uint_as_float(__float_as_uint(x[4 * j + 3]) ^ sv.w);
        }
      }
      reg_stages<32, 0, 5>(*reinterpret_cast<float(*)[32]>(x + 32 * q));
    }
    if constexpr (C::WPR == 1) {
      if (stop) return;
    }
    reg_stages<G::E, 5, G::LOGE>(x);
    stream_team_sync<LOGN, Tin>(team);  // every thread has read its layout-A data
    float4* buf = reinterpret_cast<float4*>(slot);
    smem_put_A<LOGN>(buf, x, tau);
    stream_team_sync<LOGN, Tin>(team);
    smem_get_B<LOGN>(buf, x, tau);
    // the slot is free once this warp's layout-B reads are done
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    reg_stages<G::E, 2, G::B_FWD_HI>(x);
#pragma unroll
    for (int b = 0; b < G::NSH; ++b) shfl_stage<G::E>(x, b, (tau >> b) & 1);
    if constexpr (EPI == EPI_STORE) {
      store_rowB<LOGN, Tout>(x, static_cast<Tout*>(a.y) + row * a.ldy, tau, a.norm, a.post_signs);
    } else {
      quant_rowB<LOGN, BITS>(x, a, row, tau);
    }
  }
}

template <int LOGN, typename Tin, typename Tout, int EPI, int BITS, bool SIGNS>
cudaError_t launch_stream_k(const RowArgs& a, cudaStream_t st) {
  using C = StreamCfg<LOGN, Tin>;
  static std::atomic<unsigned long long> done{0};
  auto kern = k_rows_stream<LOGN, Tin, Tout, EPI, BITS, SIGNS>;
  cudaError_t e = set_smem_attr(kern, C::SMEM, done);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int64_t grid = a.rows < sms ? a.rows : sms;
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
  return cudaLaunchKernelEx(&cfg, kern, a);
}

// The sign flip is compiled in or out, so the row loop carries no branch on it.
template <int LOGN, typename Tin, typename Tout, int EPI, int BITS>
cudaError_t launch_stream(const RowArgs& a, cudaStream_t st) {
  return a.pre_signs != nullptr ? launch_stream_k<LOGN, Tin, Tout, EPI, BITS, true>(a, st)
                                : launch_stream_k<LOGN, Tin, Tout, EPI, BITS, false>(a, st);
}

}  // namespace hit
