// rht_quantize_pack_noalloc: the fused (two-sided) RHT + group quantizer for
// callers that cannot allocate device memory.
//
// The two-sided quantizer needs an fp32 [rows, n] intermediate between its
// column pass and its row pass.  rht_quantize_pack takes that intermediate as
// a caller-supplied workspace; this entry point instead uses a fixed scratch
// array that the library itself carries as a static device variable.  Every
// GPU that loads libhit.so holds the array (16 MiB) from module load until
// the process exits.  The intermediate is written in full by the column pass
// before the row pass reads it, so nothing in the array needs clearing
// between calls.
#include <cuda_runtime.h>

#include <mutex>

#include "hit.h"
#include "internal.h"

namespace {

constexpr size_t kScratchElems = HIT_NOALLOC_MAX_ELEMS;

static __device__ __align__(256) float g_noalloc_scratch[kScratchElems];

// Device address of the scratch array, resolved once per device with that
// device current.  In host code the array's name is only a host-side stand-in,
// so kernels must be given this address instead.  The address belongs to the
// device's primary context: a process that destroys that context
// (cudaDeviceReset) must not call this entry point on the device again.
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return HIT_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return HIT_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return HIT_ECUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return HIT_OK;
}

}  // namespace

extern "C" HIT_API int rht_quantize_pack_noalloc(const void* x, int64_t rows, int64_t n, int64_t ldx, int dtype_in,
                                                 const int8_t* row_signs, const int8_t* col_signs, int bits,
                                                 int group, uint8_t* codes, float* scales, void* stream) {
  if (col_signs == nullptr)  // one-sided: there is no intermediate to place
    return rht_quantize_pack(x, rows, n, ldx, dtype_in, row_signs, nullptr, bits, group, codes, scales, nullptr, 0,
                             stream);
  // Every argument check of rht_quantize_pack first, with no workspace: that
  // call launches nothing and answers HIT_EWORKSPACE only when all other
  // arguments are valid (HIT_OK when there are no rows, else the status a bad
  // argument gets from rht_quantize_pack itself).
  const int pre = rht_quantize_pack(x, rows, n, ldx, dtype_in, row_signs, col_signs, bits, group, codes, scales,
                                    nullptr, 0, stream);
  if (pre != HIT_EWORKSPACE) return pre;
  // n is now a power of two in [32, 32768], so the bound cannot overflow.
  if (rows > static_cast<int64_t>(kScratchElems) / n) {
    hit::set_last_error("rht_quantize_pack_noalloc: rows * n exceeds the static scratch of HIT_NOALLOC_MAX_ELEMS "
                        "(4194304) elements; use rht_quantize_pack with a workspace");
    return HIT_EWORKSPACE;
  }
  void* ws = nullptr;
  const int r = scratch_address(&ws);
  if (r != HIT_OK) {
    hit::set_last_error("rht_quantize_pack_noalloc: could not resolve the scratch array on this device");
    return r;
  }
  return rht_quantize_pack(x, rows, n, ldx, dtype_in, row_signs, col_signs, bits, group, codes, scales, ws,
                           kScratchElems * sizeof(float), stream);
}
