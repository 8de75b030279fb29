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

// Ring protocol.  Row k of this CTA goes to slot k % S and is consumed by team
// k % TEAMS.  S is a multiple of TEAMS, so every slot is always served by the
// same team, which takes the slot's phases strictly in order: when a team
// waits for phase j of a slot's "full" barrier it has itself consumed phase
// j-1, and the producer refills a slot only after its "empty" barrier
// completed the previous phase.  A parity wait therefore never sees a barrier
// two phases behind or ahead of the phase it asks for.
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
  static constexpr int S = TEAMS * int((SMEM_MAX - 1024 - SIGNS) / (SLOT * TEAMS));  // ring depth
  static constexpr size_t SMEM = 1024 + SIGNS + size_t(S) * SLOT;
  static constexpr int THREADS = (NCW + 1) * 32;
  static_assert(TEAMS >= 1 && S >= TEAMS && S % TEAMS == 0, "ring depth must be a multiple of the team count");
  static_assert(2 * S * 8 <= 1024, "barriers must fit in the first kilobyte");
};

template <int LOGN, typename Tin>
__device__ __forceinline__ void stream_team_sync(int team) {
  if constexpr (StreamCfg<LOGN, Tin>::WPR == 1) {
    __syncwarp();
  } else {
    asm volatile("bar.sync %0, %1;" ::"r"(team + 1), "r"(Geom<LOGN>::T) : "memory");
  }
}

template <int LOGN, typename Tin, typename Tout, int EPI, int BITS>
__global__ void __launch_bounds__(StreamCfg<LOGN, Tin>::THREADS, 1) k_rows_stream(const RowArgs a) {
  using G = Geom<LOGN>;
  using C = StreamCfg<LOGN, Tin>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + C::S;
  uint32_t* sgn = reinterpret_cast<uint32_t*>(smem + 1024);
  uint8_t* slots = smem + 1024 + C::SIGNS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool has_signs = a.pre_signs != nullptr;
  if (has_signs) {  // the sign vector as sign-bit masks, shared by every row of this CTA
    for (int i = threadIdx.x; i < G::N; i += blockDim.x) sgn[i] = a.pre_signs[i] < 0 ? 0x80000000u : 0u;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::WPR);
    }
    mbar_init_fence();
  }
  __syncthreads();
  const int64_t grid = gridDim.x;
  const int64_t nrows = a.rows > blockIdx.x ? (a.rows - blockIdx.x + grid - 1) / grid : 0;

  if (warp == C::NCW) {  // producer
    if (lane == 0) {
      const uint8_t* src = static_cast<const uint8_t*>(a.x);
      int64_t issued = 0;
      for (int64_t k = 0; k < nrows; ++k) {
        const int s = int(k % C::S);
        if (k >= C::S && !mbar_wait(&empty[s], uint32_t((k / C::S) - 1) & 1u)) {
          atomicAdd(&g_wait_timeouts, 1u);
          break;
        }
        const int64_t row = blockIdx.x + k * grid;
        mbar_expect_tx(&full[s], C::ROW);
        bulk_g2s(slots + size_t(s) * C::SLOT, src + row * a.ldx * int64_t(sizeof(Tin)), C::ROW, &full[s]);
        issued = k + 1;
      }
      // Do not leave while a copy into this CTA's shared memory is in flight.
      for (int64_t k = issued > C::S ? issued - C::S : 0; k < issued; ++k)
        if (!mbar_wait(&full[k % C::S], uint32_t(k / C::S) & 1u)) atomicAdd(&g_wait_timeouts, 1u);
    }
    return;
  }

  const int team = warp / C::WPR;
  const int tau = (warp % C::WPR) * 32 + lane;
  for (int64_t k = team; k < nrows; k += C::TEAMS) {
    const int s = int(k % C::S);
    if (!mbar_wait(&full[s], uint32_t(k / C::S) & 1u)) {
      if (lane == 0) atomicAdd(&g_wait_timeouts, 1u);
      return;
    }
    const int64_t row = blockIdx.x + k * grid;
    uint8_t* slot = slots + size_t(s) * C::SLOT;
    float x[G::E];
    // layout A straight from the copied row (linear layout)
#pragma unroll
    for (int j = 0; j < G::NV; ++j) {
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
      if (has_signs) {  // xor of the sign bit runs on the integer pipe, not the FP32 pipe
        const uint4 sv = reinterpret_cast<const uint4*>(sgn)[i0 >> 2];
        x[4 * j] = __uint_as_float(__float_as_uint(x[4 * j]) ^ sv.x);
        x[4 * j + 1] = __uint_as_float(__float_as_uint(x[4 * j + 1]) ^ sv.y);
        x[4 * j + 2] = __uint_as_float(__float_as_uint(x[4 * j + 2]) ^ sv.z);
        x[4 * j + 3] = __uint_as_float(__float_as_uint(x[4 * j + 3]) ^ sv.w);
      }
    }
    reg_stages<G::E, 0, G::LOGE>(x);
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

template <int LOGN, typename Tin, typename Tout, int EPI, int BITS>
cudaError_t launch_stream(const RowArgs& a, cudaStream_t st) {
  using C = StreamCfg<LOGN, Tin>;
  static std::atomic<unsigned long long> done{0};
  auto kern = k_rows_stream<LOGN, Tin, Tout, EPI, BITS>;
  cudaError_t e = set_smem_attr(kern, C::SMEM, done);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int64_t grid = a.rows < sms ? a.rows : sms;
  kern<<<dim3(unsigned(grid)), C::THREADS, C::SMEM, st>>>(a);
  return cudaGetLastError();
}

}  // namespace hit
