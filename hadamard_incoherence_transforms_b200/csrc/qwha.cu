// QWHA adapter initialisation around the sparse Walsh-Hadamard expansion.
//
// QWHA explainer, technical summary §2.1: the adapter is dW = F H^-1 with a
// sparse coefficient matrix F (values c at positions E); the two-transform
// form other Fourier-type adapters use is dW = H'^-1 F H^-1.  §2.2: AdaAlloc
// spreads a budget of coefficients over the output channels (rows) in
// proportion to each channel's error, keeping a minimum per channel, and
// inside a channel keeps the coefficients of largest magnitude.
//
// This file holds
//  - row_norms: ||x_r||_2 per row (fp64 accumulation), the channel errors;
//  - qwha_allocate: the budget split (host arithmetic on `rows` numbers);
//  - qwha_select: the per-row top-k by magnitude on the device, ties to the
//    lower column, written CSR-style in ascending column order;
//  - wht_expand_sparse_2d: the two-transform expansion and its gradient,
//    composed of the row kernels of wht_expand_sparse and the column kernels.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cmath>
#include <numeric>
#include <vector>

#include "hit.h"
#include "internal.h"

namespace hit {
namespace {

bool aligned(const void* p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }
bool is_pow2(int64_t v) { return v >= 1 && (v & (v - 1)) == 0; }

int fail(int status, const char* msg) {
  set_last_error(msg);
  return status;
}

int cuda_fail(cudaError_t e) {
  if (e == cudaSuccess) return HIT_OK;
  set_last_error(cudaGetErrorString(e));
  return HIT_ECUDA;
}

// ---------------------------------------------------------------------------
// Row norms: one warp per row, 16-byte loads, squares summed in fp64 (an fp32
// value squares exactly in fp64), then a warp tree.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_row_norms(const float* __restrict__ x, int64_t rows, int64_t n, int64_t ldx,
                                                   double* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (r >= rows) return;
  const float4* p = reinterpret_cast<const float4*>(x + r * ldx);
  double acc = 0.0;
  for (int64_t i = lane; i < n / 4; i += 32) {
    const float4 v = __ldg(p + i);
    acc = fma(double(v.x), double(v.x), acc);
    acc = fma(double(v.y), double(v.y), acc);
    acc = fma(double(v.z), double(v.z), acc);
    acc = fma(double(v.w), double(v.w), acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) out[r] = sqrt(acc);
}

// ---------------------------------------------------------------------------
// Per-row top-k.  One CTA of 256 threads per row; thread t holds elements
// E t .. E t + E - 1.  The k-th largest |f| is found exactly by a radix select
// over the fp32 bit patterns (non-negative floats order like their patterns),
// one byte per pass from the top; every element above it is kept, and of the
// elements equal to it the lowest-indexed ones, as many as are still needed.
// ---------------------------------------------------------------------------
constexpr int TK_THREADS = 256;

struct TopkArgs {
  const float* f = nullptr;          // [rows, ldf]
  int64_t rows = 0, ldf = 0;         // ldf a multiple of 4
  const int64_t* offsets = nullptr;  // [rows + 1] CSR offsets (counts = differences)
  int32_t* cols = nullptr;           // [offsets[rows]]
  float* values = nullptr;           // [offsets[rows]]
};

// Exclusive block scan of one int per thread; returns this thread's prefix and the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) warp_sums[warp] = inc;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < TK_THREADS / 32; ++w) {
    const int s = warp_sums[w];
    if (w < warp) before += s;
    all += s;
  }
  __syncthreads();  // warp_sums is reused by the next scan
  total = all;
  return before + inc - v;
}

template <int N>
__global__ void __launch_bounds__(TK_THREADS) k_row_topk(const TopkArgs a) {
  static_assert(N % (TK_THREADS * 4) == 0, "whole float4 vectors per thread");
  constexpr int E = N / TK_THREADS;
  __shared__ int hist[256];
  __shared__ int warp_sums[TK_THREADS / 32];
  __shared__ int pick[2];  // chosen digit, count above it
  const int64_t row = blockIdx.x;
  const int t = threadIdx.x;
  const int64_t o0 = a.offsets[row];
  const int64_t kk = a.offsets[row + 1] - o0;
  if (kk <= 0) return;  // the whole block leaves together
  const int k = kk < N ? int(kk) : N;
  float v[E];
  uint32_t u[E];
  const float4* src = reinterpret_cast<const float4*>(a.f + row * a.ldf) + t * (E / 4);
#pragma unroll
  for (int q = 0; q < E / 4; ++q) {
    const float4 w = __ldg(src + q);
    v[4 * q] = w.x;
    v[4 * q + 1] = w.y;
    v[4 * q + 2] = w.z;
    v[4 * q + 3] = w.w;
  }
#pragma unroll
  for (int i = 0; i < E; ++i) u[i] = __float_as_uint(v[i]) & 0x7fffffffu;

  uint32_t prefix = 0, mask = 0;
  int need = k;  // rank of the wanted magnitude from the top (1-based)
  if (k < N) {
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
      hist[t] = 0;
      __syncthreads();
#pragma unroll
      for (int i = 0; i < E; ++i)
        if ((u[i] & mask) == prefix) atomicAdd(&hist[(u[i] >> shift) & 255], 1);
      __syncthreads();
      // thread t looks at digit 255 - t; exclusive count of the digits above it
      const int h = hist[255 - t];
      int tot;
      const int ex = block_exclusive_scan(h, warp_sums, tot);
      if (ex < need && need <= ex + h) {  // exactly one thread
        pick[0] = 255 - t;
        pick[1] = ex;
      }
      __syncthreads();
      const uint32_t d = uint32_t(pick[0]);
      need -= pick[1];
      prefix |= d << shift;
      mask |= 0xffu << shift;
      __syncthreads();  // pick[] is rewritten by the next pass
    }
  }
  // keep: above the threshold, or equal to it and among the first `need` equal ones
  int n_eq = 0;
  if (k < N) {
#pragma unroll
    for (int i = 0; i < E; ++i) n_eq += u[i] == prefix;
  }
  int tot_eq;
  const int eq_before = block_exclusive_scan(n_eq, warp_sums, tot_eq);
  bool keep[E];
  int n_keep = 0, r_eq = eq_before;
#pragma unroll
  for (int i = 0; i < E; ++i) {
    bool kp;
    if (k >= N) {
      kp = true;
    } else if (u[i] > prefix) {
      kp = true;
    } else if (u[i] == prefix) {
      kp = r_eq < need;
      ++r_eq;
    } else {
      kp = false;
    }
    keep[i] = kp;
    n_keep += kp;
  }
  int tot_keep;
  int pos = block_exclusive_scan(n_keep, warp_sums, tot_keep);
#pragma unroll
  for (int i = 0; i < E; ++i) {
    if (keep[i]) {
      a.cols[o0 + pos] = t * E + i;
      a.values[o0 + pos] = v[i];
      ++pos;
    }
  }
}

template <int N>
cudaError_t launch_topk(const TopkArgs& a, cudaStream_t st) {
  k_row_topk<N><<<dim3(unsigned(a.rows)), TK_THREADS, 0, st>>>(a);
  return cudaGetLastError();
}

// Left-to-right float64 sum (the order the allocation is defined with).
double sum_left_to_right(const std::vector<double>& v) {
  double acc = 0.0;
  for (double x : v) acc += x;
  return acc;
}

}  // namespace
}  // namespace hit

extern "C" {

HIT_API int row_norms(const float* x, int64_t rows, int64_t n, int64_t ldx, double* norms, void* stream) {
  if (rows < 0 || n < 1) return hit::fail(HIT_EINVAL, "row_norms: bad shape");
  if (rows == 0) return HIT_OK;
  if (x == nullptr || norms == nullptr) return hit::fail(HIT_EINVAL, "row_norms: NULL operand");
  if (n % 4 != 0 || ldx < n || ldx % 4 != 0) return hit::fail(HIT_EINVAL, "row_norms: n and ldx must be multiples of 4, ldx >= n");
  if (!hit::aligned(x, 16) || !hit::aligned(norms, 8)) return hit::fail(HIT_EALIGN, "row_norms: x 16-byte, norms 8-byte aligned");
  const unsigned grid = unsigned((rows * 32 + 255) / 256);
  hit::k_row_norms<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, rows, n, ldx, norms);
  return hit::cuda_fail(cudaGetLastError());
}

HIT_API int qwha_allocate(const double* err, int64_t rows, int64_t budget, int64_t k_min, int64_t n, int64_t* counts) {
  if (rows < 0 || n < 1 || k_min < 0 || k_min > n) return hit::fail(HIT_EINVAL, "qwha_allocate: bad rows, n or k_min");
  if (rows == 0) return budget == 0 ? HIT_OK : hit::fail(HIT_EINVAL, "qwha_allocate: budget without rows");
  if (err == nullptr || counts == nullptr) return hit::fail(HIT_EINVAL, "qwha_allocate: NULL operand");
  if (budget < rows * k_min || budget > rows * n)
    return hit::fail(HIT_EINVAL, "qwha_allocate: budget must lie in [rows * k_min, rows * n]");
  for (int64_t r = 0; r < rows; ++r)
    if (!(err[r] >= 0.0) || !std::isfinite(err[r])) return hit::fail(HIT_EINVAL, "qwha_allocate: errors must be finite and >= 0");
  const int64_t room = n - k_min;
  const int64_t left = budget - rows * k_min;
  std::vector<char> capped(rows, 0);
  std::vector<double> share(rows, 0.0);
  for (;;) {
    int64_t n_capped = 0;
    std::vector<double> w;
    w.reserve(rows);
    for (int64_t r = 0; r < rows; ++r) {
      if (capped[r]) ++n_capped;
      else w.push_back(err[r]);
    }
    const double rest = double(left - room * n_capped);
    const bool equal = !(hit::sum_left_to_right(w) > 0.0);
    if (equal) std::fill(w.begin(), w.end(), 1.0);
    const double total = hit::sum_left_to_right(w);
    bool any_over = false;
    size_t wi = 0;
    for (int64_t r = 0; r < rows; ++r) {
      if (capped[r]) {
        share[r] = 0.0;
        continue;
      }
      share[r] = (rest * w[wi++]) / total;
    }
    for (int64_t r = 0; r < rows; ++r)
      if (!capped[r] && share[r] > double(room)) any_over = true;
    if (!any_over) break;
    for (int64_t r = 0; r < rows; ++r)
      if (!capped[r] && share[r] > double(room)) capped[r] = 1;
  }
  int64_t assigned = 0;
  std::vector<double> frac(rows, 0.0);
  for (int64_t r = 0; r < rows; ++r) {
    if (capped[r]) {
      share[r] = double(room);
      counts[r] = room;
    } else {
      const double fl = std::floor(share[r]);
      counts[r] = int64_t(fl);
      frac[r] = share[r] - fl;
    }
    assigned += counts[r];
  }
  // capped rows: share = room exactly, fraction 0
  int64_t spare = left - assigned;
  std::vector<int64_t> order;
  for (int64_t r = 0; r < rows; ++r)
    if (!capped[r] && counts[r] < room) order.push_back(r);
  std::stable_sort(order.begin(), order.end(), [&](int64_t p, int64_t q) { return frac[p] > frac[q]; });
  for (size_t i = 0; i < order.size() && spare > 0; ++i, --spare) ++counts[order[i]];
  for (int64_t r = 0; r < rows; ++r) counts[r] += k_min;
  return HIT_OK;
}

HIT_API int qwha_select(const float* f, int64_t rows, int64_t n, int64_t ldf, const int64_t* offsets, int32_t* cols,
                        float* values, void* stream) {
  if (rows < 0) return hit::fail(HIT_EINVAL, "qwha_select: rows < 0");
  if (n != 1024 && n != 2048 && n != 4096 && n != 8192)
    return hit::fail(HIT_EUNSUPPORTED, "qwha_select: n must be 1024, 2048, 4096 or 8192");
  if (rows == 0) return HIT_OK;
  if (f == nullptr || offsets == nullptr || cols == nullptr || values == nullptr)
    return hit::fail(HIT_EINVAL, "qwha_select: NULL operand");
  if (rows > 0x7fffffff) return hit::fail(HIT_EUNSUPPORTED, "qwha_select: too many rows");
  if (ldf < n || ldf % 4 != 0) return hit::fail(HIT_EINVAL, "qwha_select: ldf must be >= n and a multiple of 4");
  if (!hit::aligned(f, 16) || !hit::aligned(offsets, 8) || !hit::aligned(cols, 4) || !hit::aligned(values, 4))
    return hit::fail(HIT_EALIGN, "qwha_select: misaligned operand");
  hit::TopkArgs a;
  a.f = f;
  a.rows = rows;
  a.ldf = ldf;
  a.offsets = offsets;
  a.cols = cols;
  a.values = values;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  switch (n) {
    case 1024: e = hit::launch_topk<1024>(a, st); break;
    case 2048: e = hit::launch_topk<2048>(a, st); break;
    case 4096: e = hit::launch_topk<4096>(a, st); break;
    default: e = hit::launch_topk<8192>(a, st); break;
  }
  return hit::cuda_fail(e);
}

}  // extern "C"
