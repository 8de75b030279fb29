// Two-stage butterfly runs along rows whose digits sit at a stride (SIMT,
// register resident, TMA tiles).
//
// HARP explainer, technical summary §2.1: each stage mixes, with a per-group
// block, the coordinates that differ in one digit.  For a run of two adjacent
// digits H (radix BH) and L (radix BL, even) whose positions in a row are
//   g = hi * P * S + (iH * BL + iL) * S + lo,   P = BH * BL, S >= 8,
// every (row, hi, lo) vector of P values is transformed on its own:
//   stage on H: for each iL, x[. * BL + iL] <- B_H(c) x[. * BL + iL],
//               c = (hi * BL + iL) * S + lo
//   stage on L: for each iH, x[iH * BL + .] <- B_L(c) x[iH * BL + .],
//               c = (hi * BH + iH) * S + lo
// (the group numbering of the stage convention, digit removed).
//
// A CTA owns one (hi, 8-lo group) at a time and keeps the blocks of its eight
// lo values in shared memory.  The data arrive as TMA boxes of 8 lo x (P + 1)
// positions x R rows (dense 16-byte rows; the extra position skews the rows
// across the shared-memory banks and is never used): one box loads while the
// previous one is computed.  A lane holds half of the vector (the iL of one
// parity, h, for every iH) of two rows of one lo: the stage on H is local, the
// stage on L takes the partner half (lane ^ 16) by shuffles, and every
// coefficient read from shared memory (bf16, eight per 16-byte read) feeds
// both rows with packed fp32 FMAs.
// Lane = h * 16 + rp * 8 + lo: the eight lo values of a half-warp read eight
// different blocks laid out 4 words apart in the banks (one wavefront), and the
// four (row, parity) pairs of a lo value read 16-byte rows in four distinct
// bank groups.  Results go through a padded shared-memory tile to 16-byte
// global stores.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <type_traits>

#include "device.cuh"
#include "internal.h"
#include "rows_ops.cuh"

namespace hit {

__device__ unsigned int g_wait_timeouts_strided = 0;

namespace {

// Coefficients of one lo value in shared memory, as bf16 (the tensor-core
// path's operand precision; every read then carries eight coefficients).
// Stage on H: block iL at iL BH BHP, entry (k, a) at k BHP + a = coefficient
// of output a from input k.  Stage on L: block iH at HF + iH BL BLP, entry
// (k, a) at k BLP + perm(a) with the even outputs first, perm(a) = (a & 1) HL +
// a / 2, so that the outputs of one parity are contiguous.  PER_LO is 8 mod 64
// elements (16 mod 128 bytes): the blocks of eight lo values start in eight
// different 4-bank groups.
template <int BH, int BL>
struct StridedBlocks {
  static constexpr int BHP = (BH + 3) / 4 * 4;
  static constexpr int BLP = (BL + 3) / 4 * 4;
  static constexpr int HL = BL / 2;
  static constexpr int HF0 = BL * BH * BHP;
  static constexpr int LF = BH * BL * BLP;
  static constexpr int PAD = ((8 - (HF0 + LF) % 64) + 64) % 64;
  static constexpr int HF = HF0 + PAD;
  static constexpr int PER_LO = HF + LF;
  static_assert(BL % 2 == 0, "the radix of L is split by parity");
  static_assert(PER_LO % 64 == 8 && HF % 8 == 0, "block layout must start the lo values in distinct bank groups");
};

// Stage the coefficients of one stage for the eight lo values of a group.  The
// blocks of groups run0 + d * run_stride + l (l = 0..7) are eight consecutive
// blocks in global memory for each of the NR run digits d, so every run is one
// contiguous stretch of 8 B^2 floats: read coalesced, eight loads in flight per
// thread, rounded to bf16.
template <int B, int BP, int NR, bool PERM, int NT>
__device__ __forceinline__ void stage_blocks(uint16_t* s_blk, int per_lo, int ofs, const float* blocks, int64_t run0,
                                             int64_t run_stride, bool shared, bool transpose) {
  constexpr int BB = B * B;
  constexpr int RUN = 8 * BB;
  constexpr int TOTAL = NR * RUN;
  for (int base = 0; base < TOTAL; base += 8 * NT) {
    float g[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + int(threadIdx.x) + NT * u;
      g[u] = 0.0f;
      if (i < TOTAL) {
        const int d = i / RUN, e = i - d * RUN;
        g[u] = shared ? __ldg(blocks + e % BB) : __ldg(blocks + (run0 + int64_t(d) * run_stride) * BB + e);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + int(threadIdx.x) + NT * u;
      if (i < TOTAL) {
        const int d = i / RUN, e = i - d * RUN;
        const int l = e / BB, f = e - l * BB, rr = f / B, cc = f - rr * B;  // entry (rr, cc) of block l
        const int k = transpose ? rr : cc, aa = transpose ? cc : rr;
        const int col = PERM ? (aa & 1) * (B / 2) + (aa >> 1) : aa;
        s_blk[l * per_lo + ofs + d * B * BP + k * BP + col] = __bfloat16_as_ushort(__float2bfloat16_rn(g[u]));
      }
    }
  }
}

// Byte offset of element (row, p, lo) in a dense box (or tile) of 8 lo x
// (P + 1) positions x rows with E-byte elements.
template <int P, int E>
__device__ __forceinline__ int box_offset(int row, int p, int lo) {
  return ((row * (P + 1) + p) * 8 + lo) * E;
}

template <typename T>
__device__ __forceinline__ float ld_elem(const uint8_t* p) {
  if constexpr (std::is_same<T, float>::value) return *reinterpret_cast<const float*>(p);
  else return __uint_as_float(uint32_t(*reinterpret_cast<const uint16_t*>(p)) << 16);
}
template <typename T>
__device__ __forceinline__ void st_elem(uint8_t* p, float v) {
  if constexpr (std::is_same<T, float>::value) *reinterpret_cast<float*>(p) = v;
  else *reinterpret_cast<uint16_t*>(p) = __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// o_r[q] += b[q] * s[r] for the RPL rows of a lane, q < N, from the N (padded
// to a multiple of four) consecutive bf16 coefficients at b: 16-byte reads of
// eight coefficients (8 or 4 bytes for four or two), packed fp32 FMAs on
// coefficient pairs.
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
template <int N, int RPL>
__device__ __forceinline__ void pair_fma(uint32_t w, int q, const float (&s)[RPL], float (&o)[RPL][N]) {
  if (q + 1 < N) {
#pragma unroll
    for (int r = 0; r < RPL; ++r) fma_x2(bf_lo(w), bf_hi(w), s[r], s[r], o[r][q], o[r][q + 1], o[r][q], o[r][q + 1]);
  } else if (q < N) {
#pragma unroll
    for (int r = 0; r < RPL; ++r) o[r][q] = fmaf(bf_lo(w), s[r], o[r][q]);
  }
}
template <int N, int RPL>
__device__ __forceinline__ void axpy_bf(const uint16_t* b, const float (&s)[RPL], float (&o)[RPL][N]) {
  if constexpr (N > 4) {
#pragma unroll
    for (int c8 = 0; c8 < (N + 7) / 8; ++c8) {
      const uint4 w = *reinterpret_cast<const uint4*>(b + 8 * c8);
      pair_fma<N, RPL>(w.x, 8 * c8, s, o);
      pair_fma<N, RPL>(w.y, 8 * c8 + 2, s, o);
      pair_fma<N, RPL>(w.z, 8 * c8 + 4, s, o);
      pair_fma<N, RPL>(w.w, 8 * c8 + 6, s, o);
    }
  } else if constexpr (N > 2) {
    const uint2 w = *reinterpret_cast<const uint2*>(b);
    pair_fma<N, RPL>(w.x, 0, s, o);
    pair_fma<N, RPL>(w.y, 2, s, o);
  } else {
    static_assert(N == 2, "row segment of 2 or more coefficients");
    pair_fma<N, RPL>(*reinterpret_cast<const uint32_t*>(b), 0, s, o);
  }
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::
          "r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}
template <int BH, int BL, int RPL, typename Tout>
struct StridedGeom {
  static constexpr int P = BH * BL;
  static constexpr int NT = 256;       // 8 warps x (2 row groups x 8 lo x 2 halves)
  static constexpr int R = 16 * RPL;   // rows per box: RPL rows per lane
  static constexpr int IN_BYTES = R * (P + 1) * 8 * 2;
  static constexpr int OUT_BYTES = R * (P + 1) * 8 * int(sizeof(Tout));
  static constexpr int IN_OFS = 0;  // 1024-byte aligned box
  static constexpr int OUT_OFS = (IN_BYTES + 1023) / 1024 * 1024;
  static constexpr int BLK_OFS = OUT_OFS + (OUT_BYTES + 15) / 16 * 16;
  static constexpr int BAR_OFS = BLK_OFS + 8 * StridedBlocks<BH, BL>::PER_LO * 2;
  static constexpr int SMEM = BAR_OFS + 16 + 1024;  // + slack to align the base
};

template <int BH, int BL, int RPL, typename Tout>
__global__ void __launch_bounds__(256, 1)
    k_bfly_strided(const __grid_constant__ CUtensorMap map_x, const StridedArgs a) {
  using SB = StridedBlocks<BH, BL>;
  using G = StridedGeom<BH, BL, RPL, Tout>;
  constexpr int P = G::P;
  constexpr int R = G::R;
  constexpr int HL = SB::HL;
  constexpr int NV = BH * HL;  // values per lane and row
  constexpr int EO = int(sizeof(Tout));
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* s_in = sm + G::IN_OFS;
  uint8_t* s_out = sm + G::OUT_OFS;
  uint16_t* s_blk = reinterpret_cast<uint16_t*>(sm + G::BLK_OFS);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + G::BAR_OFS);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = lane >> 4, rp = (lane >> 3) & 1, lo = lane & 7;
  const int row0 = (2 * warp + rp) * RPL;  // this lane's rows row0 .. row0 + RPL - 1 of the box
  const int64_t S = a.s;
  const int64_t groups8 = S / 8;
  const int64_t n_keys = a.n_hi * groups8;
  const int64_t row_tiles = (a.rows + R - 1) / R;
  // CTA b works on keys ks, ks + kslots, ... and, for each, on row-tile range
  // `part` of `parts`.  CTAs with consecutive b hold consecutive keys, so the
  // ones in flight together read and write the same rows at the same time: the
  // 16-byte rows of neighbouring lo groups fill the same DRAM lines while those
  // are in L2.
  const int64_t kslots = int64_t(gridDim.x) / a.parts;
  const int64_t ks = blockIdx.x % kslots, part = blockIdx.x / kslots;
  const int64_t rt_begin = part * row_tiles / a.parts, rt_end = (part + 1) * row_tiles / a.parts;
  if (ks >= n_keys || rt_begin >= rt_end) return;
  Tout* y = static_cast<Tout*>(a.y);
  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init_fence();
    mbar_expect_tx(full, uint32_t(G::IN_BYTES));
    tma_load_3d(s_in, &map_x, int((ks % groups8) * 8), int((ks / groups8) * P), int(rt_begin * R), full);
  }
  uint32_t phase = 0;
  const uint16_t* bl = s_blk + lo * SB::PER_LO;
  for (int64_t key = ks; key < n_keys; key += kslots) {
    const int64_t hi = key / groups8, lo0 = (key % groups8) * 8;
    const int64_t col0 = hi * int64_t(P) * S + lo0;  // column of (iH, iL) = (0, 0), lo = lo0
    __syncthreads();  // every lane done with the previous key's blocks
    stage_blocks<BH, SB::BHP, BL, false, G::NT>(s_blk, SB::PER_LO, 0, a.blocks_h, hi * BL * S + lo0, S,
                                                a.shared_h != 0, a.transpose != 0);
    stage_blocks<BL, SB::BLP, BH, true, G::NT>(s_blk, SB::PER_LO, SB::HF, a.blocks_l, hi * BH * S + lo0, S,
                                               a.shared_l != 0, a.transpose != 0);
    __syncthreads();
    for (int64_t rt = rt_begin; rt < rt_end; ++rt) {
      const bool ok = mbar_wait(full, phase);
      phase ^= 1u;
      // this lane's half vectors: v[r][iH * HL + j] = position iH BL + 2 j + h of row row0 + r
      float v[RPL][NV];
#pragma unroll
      for (int r = 0; r < RPL; ++r)
#pragma unroll
        for (int iH = 0; iH < BH; ++iH)
#pragma unroll
          for (int j = 0; j < HL; ++j)
            v[r][iH * HL + j] = ld_elem<__nv_bfloat16>(s_in + box_offset<P, 2>(row0 + r, iH * BL + 2 * j + h, lo));
      // every lane has read the box (and the previous tile's results have
      // left the output tile): the next box may land
      if (!__syncthreads_and(ok)) {
        if (threadIdx.x == 0) atomicAdd(&g_wait_timeouts_strided, 1u);
        return;
      }
      if (threadIdx.x == 0) {
        int64_t nkey = key, nrt = rt + 1;
        if (nrt == rt_end) {
          nkey = key + kslots;
          nrt = rt_begin;
        }
        if (nkey < n_keys) {
          mbar_expect_tx(full, uint32_t(G::IN_BYTES));
          tma_load_3d(s_in, &map_x, int((nkey % groups8) * 8), int((nkey / groups8) * P), int(nrt * R), full);
        }
      }
      auto stage_h = [&]() {
#pragma unroll
        for (int j = 0; j < HL; ++j) {
          const uint16_t* b = bl + (2 * j + h) * BH * SB::BHP;  // block iL = 2 j + h
          float o[RPL][BH];
#pragma unroll
          for (int r = 0; r < RPL; ++r)
#pragma unroll
            for (int q = 0; q < BH; ++q) o[r][q] = 0.0f;
#pragma unroll
          for (int k = 0; k < BH; ++k) {
            float in[RPL];
#pragma unroll
            for (int r = 0; r < RPL; ++r) in[r] = v[r][k * HL + j];
            axpy_bf<BH, RPL>(b + k * SB::BHP, in, o);
          }
#pragma unroll
          for (int r = 0; r < RPL; ++r)
#pragma unroll
            for (int q = 0; q < BH; ++q) v[r][q * HL + j] = o[r][q];
        }
      };
      auto stage_l = [&]() {
#pragma unroll
        for (int iH = 0; iH < BH; ++iH) {
          float o[RPL][HL];
#pragma unroll
          for (int r = 0; r < RPL; ++r)
#pragma unroll
            for (int q = 0; q < HL; ++q) o[r][q] = 0.0f;
          // outputs 2 q + h of block iH (contiguous after the column
          // permutation); inputs 2 j + h (own) and 2 j + 1 - h (partner)
          const uint16_t* b = bl + SB::HF + iH * BL * SB::BLP + h * HL;
#pragma unroll
          for (int j = 0; j < HL; ++j) {
            float own[RPL], oth[RPL];
#pragma unroll
            for (int r = 0; r < RPL; ++r) {
              own[r] = v[r][iH * HL + j];
              oth[r] = __shfl_xor_sync(0xffffffffu, own[r], 16);
            }
            axpy_bf<HL, RPL>(b + (2 * j + h) * SB::BLP, own, o);
            axpy_bf<HL, RPL>(b + (2 * j + 1 - h) * SB::BLP, oth, o);
          }
#pragma unroll
          for (int r = 0; r < RPL; ++r)
#pragma unroll
            for (int q = 0; q < HL; ++q) v[r][iH * HL + q] = o[r][q];
        }
      };
      if (a.h_first) {
        stage_h();
        stage_l();
      } else {
        stage_l();
        stage_h();
      }
#pragma unroll
      for (int r = 0; r < RPL; ++r)
#pragma unroll
        for (int iH = 0; iH < BH; ++iH)
#pragma unroll
          for (int j = 0; j < HL; ++j)
            st_elem<Tout>(s_out + box_offset<P, EO>(row0 + r, iH * BL + 2 * j + h, lo), v[r][iH * HL + j]);
      __syncthreads();
      // 16-byte global stores: piece (row, p) = the 8 lo values of one position
      constexpr int WO = 8 * EO / 16;  // 16-byte words per piece
      const int64_t r0 = rt * R;
      for (int i = threadIdx.x; i < R * P * WO; i += G::NT) {
        const int w = i % WO, pc = i / WO;
        const int rr = pc / P, p = pc - rr * P;
        const int64_t row = r0 + rr;
        if (row >= a.rows) continue;
        const uint4 val = *reinterpret_cast<const uint4*>(s_out + box_offset<P, EO>(rr, p, 0) + 16 * w);
        __stcs(reinterpret_cast<uint4*>(y + row * a.ldy + col0 + int64_t(p) * S) + w, val);
      }
    }
  }
}

template <int BH, int BL, int RPL, typename Tout>
cudaError_t launch_strided_t(const StridedArgs& a, cudaStream_t st) {
  using G = StridedGeom<BH, BL, RPL, Tout>;
  constexpr int R = G::R;
  static_assert(G::SMEM <= 227 * 1024, "shared memory");
  static std::atomic<unsigned long long> done{0};
  auto kern = k_bfly_strided<BH, BL, RPL, Tout>;
  cudaError_t e = set_smem_attr(kern, G::SMEM, done);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int64_t n_keys = a.n_hi * (a.s / 8), row_tiles = (a.rows + R - 1) / R;
  if (n_keys <= 0 || row_tiles <= 0) return cudaSuccess;
  // input boxes: dim 0 = lo (S, contiguous), dim 1 = position P hi + p
  // (stride S), dim 2 = row (stride ldx); a box of P + 1 positions reaches
  // one position into the next hi block (or past the end: zero fill)
  const int64_t len = a.n_hi * int64_t(G::P) * a.s;
  CUtensorMap mx;
  const int64_t dims[3] = {a.s, len / a.s, a.rows};
  const int64_t sx[3] = {1, a.s, a.ldx};
  const uint32_t box[3] = {8u, uint32_t(G::P + 1), uint32_t(R)};
  if (!make_tensor_map(&mx, a.x, 3, dims, sx, box, 2, false)) return cudaErrorInvalidValue;
  StridedArgs b = a;
  int64_t kslots = n_keys;
  if (n_keys <= sms) {
    b.parts = sms / n_keys;
    if (b.parts > row_tiles) b.parts = row_tiles;
  } else {
    b.parts = 1;
    kslots = sms;
  }
  kern<<<dim3(unsigned(kslots * b.parts)), G::NT, G::SMEM, st>>>(mx, b);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Tensor-core variant for BL = 16 with bf16 results (mma.sync m16n8k16, bf16
// operands, fp32 accumulation).  For one lo value the two stages are products
// with block-diagonal P x P matrices on the positions p = iH 16 + iL:
//   stage on H: Y = X M_H, M_H[(iH, iL), (a, iL')] = [iL = iL'] B_H(iL)[a, iH]
//   stage on L: Y = X M_L, M_L[(iH, iL), (iH', q)] = [iH = iH'] B_L(iH)[q, iL]
// A warp holds 16 rows of two lo values.  K steps of 16 run over iL at one iH
// and N tiles of 8 over (a or iH', half of iL' or q), so the accumulators of
// the first stage are, pairwise rounded to bf16, the A operands of the second
// (the column order of one product is the row order of the next).  Only the
// nonzero N tiles of each K step are issued: for M_H all BH of them (one
// nonzero per eight lanes, read from shared memory per MMA, and only the K
// half that holds them: m16n8k8), for M_L the two of its own diagonal block
// (dense, two registers per lane read per MMA).
// The A operands of the first stage come from the TMA box: the 32-bit word of
// the warp's lo pair in each (row, position) row of 8 lo values.  Results go
// to a shared-memory tile laid out per lo pair ([row][pair][position] words,
// rows skewed so a warp's 32 stores hit 32 banks) and leave as 16-byte global
// stores.
// ---------------------------------------------------------------------------
template <int BH>
struct MmaBlocks {
  static constexpr int HF = 16 * BH * 8;  // stage on H: [iL][a][k (8)]
  static constexpr int LF = BH * 256;     // stage on L: [iH][q][k (16)]
  static constexpr int PER_LO = HF + LF;  // bf16 elements
};

// Stage one stage's coefficients for the eight lo values of a group as bf16,
// entry (output a, input k) of run digit d at ofs + d B ROWP + a ROWP + k.
template <int B, int ROWP, int NR, int NT>
__device__ __forceinline__ void stage_blocks_ak(uint16_t* s_blk, int per_lo, int ofs, const float* blocks,
                                                int64_t run0, int64_t run_stride, bool shared, bool transpose) {
  constexpr int BB = B * B;
  constexpr int RUN = 8 * BB;
  constexpr int TOTAL = NR * RUN;
  for (int base = 0; base < TOTAL; base += 8 * NT) {
    float g[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + int(threadIdx.x) + NT * u;
      g[u] = 0.0f;
      if (i < TOTAL) {
        const int d = i / RUN, e = i - d * RUN;
        g[u] = shared ? __ldg(blocks + e % BB) : __ldg(blocks + (run0 + int64_t(d) * run_stride) * BB + e);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + int(threadIdx.x) + NT * u;
      if (i < TOTAL) {
        const int d = i / RUN, e = i - d * RUN;
        const int l = e / BB, f = e - l * BB, rr = f / B, cc = f - rr * B;  // entry (rr, cc) of block l
        const int k = transpose ? rr : cc, aa = transpose ? cc : rr;
        s_blk[l * per_lo + ofs + d * B * ROWP + aa * ROWP + k] = __bfloat16_as_ushort(__float2bfloat16_rn(g[u]));
      }
    }
  }
}

// m16n8k8: A = {a0, a1} (rows g, g + 8; k = 2 t, 2 t + 1), B = b0
__device__ __forceinline__ void mma_1688(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int BH>
struct MmaGeom {
  static constexpr int P = BH * 16;
  static constexpr int NT = 256;
  static constexpr int R = 32;                                // two groups of 16 rows
  static constexpr int IN_BYTES = R * (P + 1) * 8 * 2;        // TMA box (dense, P + 1 positions)
  static constexpr int PQ = P;                                // words per (row, lo pair) plane
  static constexpr int RP = 4 * PQ + ((8 - (4 * PQ) % 32) + 32) % 32;  // words per row, 8 mod 32
  static constexpr int OUT_WORDS = R * RP;
  static constexpr int IN_OFS = 0;
  static constexpr int OUT_OFS = (IN_BYTES + 1023) / 1024 * 1024;
  static constexpr int BLK_OFS = OUT_OFS + OUT_WORDS * 4;
  static constexpr int BAR_OFS = BLK_OFS + 8 * MmaBlocks<BH>::PER_LO * 2;
  static constexpr int SMEM = BAR_OFS + 16 + 1024;
  static_assert(RP % 32 == 8 && RP >= 4 * PQ + 1, "output rows must start 8 banks apart with room for the skew");
};

// word of (row, lo pair, position) in the output tile; rows 4..7 of every 8
// move one bank so that rows 0..7 start in banks 0, 8, 16, 24, 1, 9, 17, 25
template <int BH>
__device__ __forceinline__ int out_word(int row, int lq, int p) {
  using G = MmaGeom<BH>;
  return row * G::RP + lq * G::PQ + p + ((row >> 2) & 1);
}

template <int BH>
__global__ void __launch_bounds__(256, 1)
    k_bfly_strided_mma(const __grid_constant__ CUtensorMap map_x, const StridedArgs a) {
  using MB = MmaBlocks<BH>;
  using G = MmaGeom<BH>;
  constexpr int P = G::P;
  constexpr int R = G::R;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint8_t* s_in = sm + G::IN_OFS;
  uint32_t* s_out = reinterpret_cast<uint32_t*>(sm + G::OUT_OFS);
  uint16_t* s_blk = reinterpret_cast<uint16_t*>(sm + G::BLK_OFS);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + G::BAR_OFS);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rg = warp >> 2, lq = warp & 3;  // 16-row group, lo pair (2 lq, 2 lq + 1)
  const int g = lane >> 2, t = lane & 3;    // fragment group and thread in group
  const int rowA = 16 * rg + g, rowB = rowA + 8;
  // M_H's nonzero in this lane's B fragment: lanes with g / 2 == t carry the
  // coefficient of iL = g (+ 8), in the low (g even) or high half
  const bool hact = (g >> 1) == t;
  const int hsh = (g & 1) * 16;
  const int64_t S = a.s;
  const int64_t groups8 = S / 8;
  const int64_t n_keys = a.n_hi * groups8;
  const int64_t row_tiles = (a.rows + R - 1) / R;
  const int64_t kslots = int64_t(gridDim.x) / a.parts;
  const int64_t ks = blockIdx.x % kslots, part = blockIdx.x / kslots;
  const int64_t rt_begin = part * row_tiles / a.parts, rt_end = (part + 1) * row_tiles / a.parts;
  if (ks >= n_keys || rt_begin >= rt_end) return;
  __nv_bfloat16* y = static_cast<__nv_bfloat16*>(a.y);
  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init_fence();
    mbar_expect_tx(full, uint32_t(G::IN_BYTES));
    tma_load_3d(sm + G::IN_OFS, &map_x, int((ks % groups8) * 8), int((ks / groups8) * P), int(rt_begin * R), full);
  }
  uint32_t phase = 0;
  for (int64_t key = ks; key < n_keys; key += kslots) {
    const int64_t hi = key / groups8, lo0 = (key % groups8) * 8;
    const int64_t col0 = hi * int64_t(P) * S + lo0;
    __syncthreads();
    stage_blocks_ak<BH, 8, 16, G::NT>(s_blk, MB::PER_LO, 0, a.blocks_h, hi * 16 * S + lo0, S, a.shared_h != 0,
                                      a.transpose != 0);
    stage_blocks_ak<16, 16, BH, G::NT>(s_blk, MB::PER_LO, MB::HF, a.blocks_l, hi * BH * S + lo0, S,
                                       a.shared_l != 0, a.transpose != 0);
    __syncthreads();
    for (int64_t rt = rt_begin; rt < rt_end; ++rt) {
      const bool ok = mbar_wait(full, phase);
      phase ^= 1u;
      // words of the lo pair at rows rowA, rowB, positions j 16 + 2 t + {0, 1, 8, 9}
      uint32_t xw[BH][8];
#pragma unroll
      for (int j = 0; j < BH; ++j) {
        const int p = j * 16 + 2 * t;
        xw[j][0] = *reinterpret_cast<const uint32_t*>(s_in + box_offset<P, 2>(rowA, p, 2 * lq));
        xw[j][1] = *reinterpret_cast<const uint32_t*>(s_in + box_offset<P, 2>(rowA, p + 1, 2 * lq));
        xw[j][2] = *reinterpret_cast<const uint32_t*>(s_in + box_offset<P, 2>(rowB, p, 2 * lq));
        xw[j][3] = *reinterpret_cast<const uint32_t*>(s_in + box_offset<P, 2>(rowB, p + 1, 2 * lq));
        xw[j][4] = *reinterpret_cast<const uint32_t*>(s_in + box_offset<P, 2>(rowA, p + 8, 2 * lq));
        xw[j][5] = *reinterpret_cast<const uint32_t*>(s_in + box_offset<P, 2>(rowA, p + 9, 2 * lq));
        xw[j][6] = *reinterpret_cast<const uint32_t*>(s_in + box_offset<P, 2>(rowB, p + 8, 2 * lq));
        xw[j][7] = *reinterpret_cast<const uint32_t*>(s_in + box_offset<P, 2>(rowB, p + 9, 2 * lq));
      }
      if (!__syncthreads_and(ok)) {
        if (threadIdx.x == 0) atomicAdd(&g_wait_timeouts_strided, 1u);
        return;
      }
      if (threadIdx.x == 0) {
        int64_t nkey = key, nrt = rt + 1;
        if (nrt == rt_end) {
          nkey = key + kslots;
          nrt = rt_begin;
        }
        if (nkey < n_keys) {
          mbar_expect_tx(full, uint32_t(G::IN_BYTES));
          tma_load_3d(sm + G::IN_OFS, &map_x, int((nkey % groups8) * 8), int((nkey / groups8) * P), int(nrt * R),
                      full);
        }
      }
      uint32_t ow0[2 * BH][2];  // lo 2 lq results, bf16 pairs (rowA, rowB)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const uint32_t sel = e ? 0x7632u : 0x5410u;  // high or low halves: lo 2 lq + e
        const uint16_t* bh = s_blk + (2 * lq + e) * MB::PER_LO;
        const uint16_t* blt = bh + MB::HF;
        // stage with M_H on A fragments a(j): all BH N tiles of each K step
        auto stage_h = [&](auto&& afrag, float (&acc)[2 * BH][4]) {
#pragma unroll
          for (int j = 0; j < BH; ++j) {
            uint32_t a0, a1, a2, a3;
            afrag(j, a0, a1, a2, a3);
#pragma unroll
            for (int aa = 0; aa < BH; ++aa) {
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                // the tile's nonzeros lie in K half hh: one m16n8k8 on that half
                const uint32_t c = bh[(g + 8 * hh) * (BH * 8) + aa * 8 + j];
                const uint32_t w = hact ? (c << hsh) : 0u;
                if (hh == 0) mma_1688(acc[2 * aa], a0, a1, w);
                else mma_1688(acc[2 * aa + 1], a2, a3, w);
              }
            }
          }
        };
        // stage with M_L: the two N tiles of the diagonal block of each K step
        auto stage_l = [&](auto&& afrag, float (&acc)[2 * BH][4]) {
#pragma unroll
          for (int j = 0; j < BH; ++j) {
            uint32_t a0, a1, a2, a3;
            afrag(j, a0, a1, a2, a3);
#pragma unroll
            for (int hq = 0; hq < 2; ++hq) {
              const uint16_t* brow = blt + j * 256 + (8 * hq + g) * 16 + 2 * t;
              const uint32_t b0 = *reinterpret_cast<const uint32_t*>(brow);
              const uint32_t b1 = *reinterpret_cast<const uint32_t*>(brow + 8);
              mma_16816(acc[2 * j + hq], a0, a1, a2, a3, b0, b1);
            }
          }
        };
        auto from_x = [&](int j, uint32_t& a0, uint32_t& a1, uint32_t& a2, uint32_t& a3) {
          a0 = __byte_perm(xw[j][0], xw[j][1], sel);
          a1 = __byte_perm(xw[j][2], xw[j][3], sel);
          a2 = __byte_perm(xw[j][4], xw[j][5], sel);
          a3 = __byte_perm(xw[j][6], xw[j][7], sel);
        };
        float acc[2 * BH][4];
#pragma unroll
        for (int n = 0; n < 2 * BH; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;
        if (a.h_first) stage_h(from_x, acc);
        else stage_l(from_x, acc);
        // the first stage's N tiles (j, 0) and (j, 1) are the second stage's K step j
        uint32_t a2f[BH][4];
#pragma unroll
        for (int j = 0; j < BH; ++j) {
          a2f[j][0] = f32_to_bf16x2(acc[2 * j][0], acc[2 * j][1]);
          a2f[j][1] = f32_to_bf16x2(acc[2 * j][2], acc[2 * j][3]);
          a2f[j][2] = f32_to_bf16x2(acc[2 * j + 1][0], acc[2 * j + 1][1]);
          a2f[j][3] = f32_to_bf16x2(acc[2 * j + 1][2], acc[2 * j + 1][3]);
        }
        auto from_acc = [&](int j, uint32_t& a0, uint32_t& a1, uint32_t& a2, uint32_t& a3) {
          a0 = a2f[j][0];
          a1 = a2f[j][1];
          a2 = a2f[j][2];
          a3 = a2f[j][3];
        };
#pragma unroll
        for (int n = 0; n < 2 * BH; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;
        if (a.h_first) stage_l(from_acc, acc);
        else stage_h(from_acc, acc);
        if (e == 0) {
#pragma unroll
          for (int n = 0; n < 2 * BH; ++n) {
            ow0[n][0] = f32_to_bf16x2(acc[n][0], acc[n][1]);
            ow0[n][1] = f32_to_bf16x2(acc[n][2], acc[n][3]);
          }
        } else {
          // tile n = (j, half): positions p, p + 1 with p = 16 j + 8 half + 2 t;
          // one word per (row, position) holds the pair's two lo values
#pragma unroll
          for (int n = 0; n < 2 * BH; ++n) {
            const int p = 16 * (n >> 1) + 8 * (n & 1) + 2 * t;
            const uint32_t wA = f32_to_bf16x2(acc[n][0], acc[n][1]);
            const uint32_t wB = f32_to_bf16x2(acc[n][2], acc[n][3]);
            s_out[out_word<BH>(rowA, lq, p)] = __byte_perm(ow0[n][0], wA, 0x5410);
            s_out[out_word<BH>(rowA, lq, p + 1)] = __byte_perm(ow0[n][0], wA, 0x7632);
            s_out[out_word<BH>(rowB, lq, p)] = __byte_perm(ow0[n][1], wB, 0x5410);
            s_out[out_word<BH>(rowB, lq, p + 1)] = __byte_perm(ow0[n][1], wB, 0x7632);
          }
        }
      }
      __syncthreads();
      // 16-byte global stores: piece (row, p) = the 8 lo values of one position
      const int64_t r0 = rt * R;
      for (int i = threadIdx.x; i < R * P; i += G::NT) {
        const int rr = i / P, p = i - rr * P;
        const int64_t row = r0 + rr;
        if (row >= a.rows) continue;
        const uint4 val = make_uint4(s_out[out_word<BH>(rr, 0, p)], s_out[out_word<BH>(rr, 1, p)],
                                     s_out[out_word<BH>(rr, 2, p)], s_out[out_word<BH>(rr, 3, p)]);
        __stcs(reinterpret_cast<uint4*>(y + row * a.ldy + col0 + int64_t(p) * S), val);
      }
    }
  }
}

template <int BH>
cudaError_t launch_strided_mma(const StridedArgs& a, cudaStream_t st) {
  using G = MmaGeom<BH>;
  constexpr int R = G::R;
  static_assert(G::SMEM <= 227 * 1024, "shared memory");
  static std::atomic<unsigned long long> done{0};
  auto kern = k_bfly_strided_mma<BH>;
  cudaError_t e = set_smem_attr(kern, G::SMEM, done);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int64_t n_keys = a.n_hi * (a.s / 8), row_tiles = (a.rows + R - 1) / R;
  if (n_keys <= 0 || row_tiles <= 0) return cudaSuccess;
  const int64_t len = a.n_hi * int64_t(G::P) * a.s;
  CUtensorMap mx;
  const int64_t dims[3] = {a.s, len / a.s, a.rows};
  const int64_t sx[3] = {1, a.s, a.ldx};
  const uint32_t box[3] = {8u, uint32_t(G::P + 1), uint32_t(R)};
  if (!make_tensor_map(&mx, a.x, 3, dims, sx, box, 2, false)) return cudaErrorInvalidValue;
  StridedArgs b = a;
  int64_t kslots = n_keys;
  if (n_keys <= sms) {
    b.parts = sms / n_keys;
    if (b.parts > row_tiles) b.parts = row_tiles;
  } else {
    b.parts = 1;
    kslots = sms;
  }
  kern<<<dim3(unsigned(kslots * b.parts)), G::NT, G::SMEM, st>>>(mx, b);
  return cudaGetLastError();
}

template <int BH, int BL>
cudaError_t launch_strided_b(int dt_out, const StridedArgs& a, cudaStream_t st) {
  // two rows per lane (32-row boxes); three ran slower (the vectors and
  // accumulators of three rows exceed the registers)
  return dt_out == DT_BF16 ? launch_strided_t<BH, BL, 2, __nv_bfloat16>(a, st)
                           : launch_strided_t<BH, BL, 2, float>(a, st);
}

}  // namespace

bool strided_supported(int bh, int bl, int es_in, int es_out) {
  // the radix of L is split between two lanes (even), P = bh bl <= 256 positions per box
  const bool known = (bh == 7 && bl == 16) || (bh == 8 && bl == 8) || (bh == 4 && bl == 16) || (bh == 16 && bl == 4);
  return known && es_in == 2 && (es_out == 2 || es_out == 4);
}

cudaError_t launch_bfly_strided(int bh, int bl, int dt_in, int dt_out, const StridedArgs& a, cudaStream_t st) {
  if (dt_in != DT_BF16) return cudaErrorInvalidValue;
  // runs with a radix-16 digit L and bf16 results take the tensor cores
  if (bh == 7 && bl == 16 && dt_out == DT_BF16) return launch_strided_mma<7>(a, st);
  if (bh == 4 && bl == 16 && dt_out == DT_BF16) return launch_strided_mma<4>(a, st);
  if (bh == 7 && bl == 16) return launch_strided_b<7, 16>(dt_out, a, st);
  if (bh == 8 && bl == 8) return launch_strided_b<8, 8>(dt_out, a, st);
  if (bh == 4 && bl == 16) return launch_strided_b<4, 16>(dt_out, a, st);
  if (bh == 16 && bl == 4) return launch_strided_b<16, 4>(dt_out, a, st);
  return cudaErrorInvalidValue;
}

cudaError_t wait_timeouts_strided(unsigned long long* count, bool reset) {
  unsigned int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_wait_timeouts_strided, sizeof v);
  if (e != cudaSuccess) return e;
  *count += v;
  if (reset && v != 0) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_wait_timeouts_strided, &zero, sizeof zero);
  }
  return e;
}

}  // namespace hit
