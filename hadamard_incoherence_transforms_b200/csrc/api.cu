// C ABI of libhit.so (declared in include/hit.h): host-side argument checks,
// pass planning and kernel dispatch.  Every check runs before the first CUDA
// call, so a rejected call launches nothing; no path falls back to the CPU.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <string>
#include <vector>

#include "hit.h"
#include "internal.h"
#include "kernels.h"

namespace {

thread_local std::string g_last_error;

int fail(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return status;
}

int ok() { return HIT_OK; }

int cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return HIT_OK;
  return fail(HIT_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool is_pow2(int64_t v) { return v >= 1 && (v & (v - 1)) == 0; }
int ilog2(int64_t v) {
  int k = 0;
  while ((int64_t(1) << k) < v) ++k;
  return k;
}
size_t esize(int dt) { return dt == HIT_F32 ? 4 : 2; }
bool dtype_ok(int dt) { return dt == HIT_F32 || dt == HIT_BF16; }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
float inv_sqrt(int64_t n) { return static_cast<float>(1.0 / std::sqrt(static_cast<double>(n))); }

// Row alignment the vector accesses of a row kernel need.
size_t row_align(int dt, int64_t n) {
  const int64_t bytes = n * static_cast<int64_t>(esize(dt));
  return bytes >= 16 ? 16 : static_cast<size_t>(bytes);
}

// Column passes access single elements: only element alignment is needed.
int check_cols_operand(const void* p, int64_t ld, int64_t n, int dt, const char* name) {
  if (p == nullptr) return fail(HIT_EINVAL, "%s is NULL", name);
  if (ld < n) return fail(HIT_EINVAL, "%s: leading dimension %lld < n %lld", name, (long long)ld, (long long)n);
  if (!aligned(p, esize(dt))) return fail(HIT_EALIGN, "%s: base must be %zu-byte aligned", name, esize(dt));
  return HIT_OK;
}

int check_rows_operand(const void* p, int64_t ld, int64_t n, int dt, const char* name) {
  if (p == nullptr) return fail(HIT_EINVAL, "%s is NULL", name);
  if (ld < n) return fail(HIT_EINVAL, "%s: leading dimension %lld < n %lld", name, (long long)ld, (long long)n);
  const size_t ra = row_align(dt, n);
  if (!aligned(p, ra) || (static_cast<size_t>(ld) * esize(dt)) % ra != 0)
    return fail(HIT_EALIGN, "%s: base and row pitch must be %zu-byte aligned", name, ra);
  return HIT_OK;
}

// Rows of 4096 elements go through the persistent TMA-fed kernel, rows of
// 8192 through the persistent direct-load kernel; both need 16-byte aligned
// row starts (always true for the row pitches the checks accept when
// n >= 4096 and the base is 16-byte aligned).
bool use_persistent(int logn, const void* x, int64_t ld, int dt) {
  return (logn == 12 || logn == 13) && aligned(x, 16) && (static_cast<size_t>(ld) * esize(dt)) % 16 == 0;
}

// Column transform of length m on an [m, cols] matrix: ceil(log2(m)/7) passes.
// tmp (fp32, leading dim ld_tmp) carries the intermediate between passes; it
// may alias dst when dst is fp32.
int run_cols(const void* src, int dt_src, int64_t ld_src, void* dst, int dt_dst, int64_t ld_dst, int64_t m,
             int64_t cols, const int8_t* pre, const int8_t* post, float* tmp, int64_t ld_tmp, cudaStream_t st) {
  const int k = ilog2(m);
  const bool vec_ok = ld_src % 4 == 0 && ld_dst % 4 == 0 && aligned(src, 4 * esize(dt_src)) &&
                      aligned(dst, 4 * esize(dt_dst));
  // One pass with clusters over 16-column strips (its staging copies are 16-byte
  // asynchronous copies, so the source rows must start on 16-byte boundaries).
  const bool src16 = aligned(src, 16) && (static_cast<size_t>(ld_src) * esize(dt_src)) % 16 == 0;
  if (k >= 10 && k <= 13 && cols % 16 == 0 && vec_ok && src16) {
    hit::ColArgs a;
    a.x = src;
    a.y = dst;
    a.m = m;
    a.cols = cols;
    a.ldx = ld_src;
    a.ldy = ld_dst;
    a.pre_signs = pre;
    a.post_signs = post;
    a.norm = inv_sqrt(m);
    return cuda_status(hit::launch_cols_cluster(k, dt_src, dt_dst, a, st), "column transform launch");
  }
  // One pass over whole 4-column strips when the strip rows are vector aligned.
  if (k >= 8 && k <= 13 && cols % 4 == 0 && vec_ok) {
    hit::ColArgs a;
    a.x = src;
    a.y = dst;
    a.m = m;
    a.cols = cols;
    a.ldx = ld_src;
    a.ldy = ld_dst;
    a.pre_signs = pre;
    a.post_signs = post;
    a.norm = inv_sqrt(m);
    return cuda_status(hit::launch_cols_full(k, dt_src, dt_dst, a, st), "column transform launch");
  }
  const int np = k == 0 ? 1 : (k + 6) / 7;
  int lo = 0;
  for (int p = 0; p < np; ++p) {
    const int nb = (k - lo) / (np - p);  // spread the bits evenly, larger passes last
    hit::ColArgs a;
    a.m = m;
    a.cols = cols;
    a.lo = lo;
    const bool first = p == 0, last = p == np - 1;
    const int nbits = last ? k - lo : nb;
    a.x = first ? src : tmp;
    a.ldx = first ? ld_src : ld_tmp;
    a.y = last ? dst : tmp;
    a.ldy = last ? ld_dst : ld_tmp;
    a.pre_signs = first ? pre : nullptr;
    a.post_signs = last ? post : nullptr;
    a.norm = last ? inv_sqrt(m) : 1.0f;
    const cudaError_t e = hit::launch_cols_pass(nbits, first ? dt_src : hit::DT_F32, last ? dt_dst : hit::DT_F32, a, st);
    if (e != cudaSuccess) return cuda_status(e, "column transform launch");
    lo += nbits;
  }
  return HIT_OK;
}

int rht_impl(bool inverse, const void* x, void* y, int64_t rows, int64_t n, int64_t ldx, int64_t ldy, int dt_in,
             int dt_out, const int8_t* signs, int axis, void* ws, size_t ws_bytes, void* stream) {
  const char* fn = inverse ? "rht_inverse" : "rht_forward";
  if (!dtype_ok(dt_in) || !dtype_ok(dt_out)) return fail(HIT_EUNSUPPORTED, "%s: unknown dtype", fn);
  if (rows < 0 || n < 1) return fail(HIT_EINVAL, "%s: bad shape [%lld, %lld]", fn, (long long)rows, (long long)n);
  if (axis != 0 && axis != 1) return fail(HIT_EINVAL, "%s: axis must be 0 or 1", fn);
  if (rows == 0) return ok();  // empty input: nothing to read or write
  const int64_t len = axis == 1 ? n : rows;
  if (!is_pow2(len)) return fail(HIT_EINVAL, "%s: transform length %lld is not a power of two", fn, (long long)len);
  if (axis == 1 && len > 32768) return fail(HIT_EUNSUPPORTED, "%s: row length %lld > 32768", fn, (long long)len);
  if (axis == 0 && len > (int64_t(1) << 24)) return fail(HIT_EUNSUPPORTED, "%s: column length > 2^24", fn);
  int r = axis == 1 ? check_rows_operand(x, ldx, n, dt_in, "x") : check_cols_operand(x, ldx, n, dt_in, "x");
  if (r) return r;
  r = axis == 1 ? check_rows_operand(y, ldy, n, dt_out, "y") : check_cols_operand(y, ldy, n, dt_out, "y");
  if (r) return r;
  if (signs != nullptr && len >= 4 && !aligned(signs, 4)) return fail(HIT_EALIGN, "%s: signs must be 4-byte aligned", fn);
  if (rows == 0) return ok();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (axis == 1) {
    hit::RowArgs a;
    a.x = x;
    a.y = y;
    a.rows = rows;
    a.ldx = ldx;
    a.ldy = ldy;
    a.pre_signs = inverse ? nullptr : signs;
    a.post_signs = inverse ? signs : nullptr;
    a.norm = inv_sqrt(n);
    const int logn = ilog2(n);
    cudaError_t e;
    if (use_persistent(logn, x, ldx, dt_in))
      e = logn == 12 ? hit::rows_stream_store(logn, dt_in, dt_out, a, st) : hit::rows_direct_store(logn, dt_in, dt_out, a, st);
    else if (dt_in == HIT_F32) e = hit::rows_store_from_f32(logn, dt_out, a, st);
    else e = hit::rows_store_from_bf16(logn, dt_out, a, st);
    return cuda_status(e, fn);
  }
  // columns
  const int k = ilog2(rows);
  float* tmp = nullptr;
  int64_t ld_tmp = 0;
  if (k > 7) {
    if (dt_out == HIT_F32) {
      tmp = static_cast<float*>(y);
      ld_tmp = ldy;
    } else {
      const size_t need = static_cast<size_t>(rows) * static_cast<size_t>(n) * 4;
      if (ws == nullptr || ws_bytes < need) return fail(HIT_EWORKSPACE, "%s: needs %zu workspace bytes", fn, need);
      if (!aligned(ws, 16)) return fail(HIT_EALIGN, "%s: workspace must be 16-byte aligned", fn);
      tmp = static_cast<float*>(ws);
      ld_tmp = n;
    }
  }
  return run_cols(x, dt_in, ldx, y, dt_out, ldy, rows, n, inverse ? nullptr : signs, inverse ? signs : nullptr, tmp,
                  ld_tmp, st);
}

}  // namespace

namespace hit {
void set_last_error(const char* msg) { g_last_error = msg; }
}  // namespace hit

// Plan one butterfly pass applying stages order[0..cnt) (consecutive digits).
static bool plan_pass(const int* order, int cnt, const int32_t* radices, const int64_t* S, const float* const* blocks,
                      const int64_t* n_groups, int64_t len, int64_t outer, int axis, bool transpose,
                      hit::BflyPass& p) {
  if (cnt > hit::kMaxPassStages) return false;
  int dlo = order[0], dhi = order[0];
  for (int k = 1; k < cnt; ++k) {
    dlo = order[k] < dlo ? order[k] : dlo;
    dhi = order[k] > dhi ? order[k] : dhi;
  }
  int64_t P = 1;
  for (int t = dlo; t <= dhi; ++t) P *= radices[t];
  if (P > 16384) return false;
  const int64_t S_in = S[dhi];
  const size_t budget = 100 * 1024;  // two CTAs per SM overlap their load / compute / store phases
  // consecutive lo values per tile (a power of two dividing S_in); along rows
  // they are contiguous in memory, so up to eight of them per tile
  int max_nl = 0;
  if (axis == 1)
    while (max_nl < 3 && S_in % (int64_t(2) << max_nl) == 0) ++max_nl;
  // Among the (NL, NB) that fit, take the largest tile (fewest chunks and
  // barriers per element); on ties prefer more contiguous lo values.
  int best_nl = -1, best_nb = -1;
  int64_t best_elems = 0, best_blk = 0, best_pitch = 0;
  for (int log_nl = max_nl; log_nl >= 0; --log_nl) {
    const int NL = 1 << log_nl;
    int64_t blk = 0;
    for (int k = 0; k < cnt; ++k) {
      const int t = order[k];
      const int64_t b = radices[t], bp = (b + 3) / 4 * 4;
      const bool shared = n_groups[t] == 1 && len / b != 1;
      blk += (shared ? 1 : (P / b) * NL) * b * bp;
    }
    const int64_t pnl = P * NL;
    const int64_t pitch = (pnl % 2 == 0) ? pnl + 1 : pnl;
    for (int log_nb = 10; log_nb >= 0; --log_nb) {
      const int64_t nb = int64_t(1) << log_nb;
      const size_t bytes = static_cast<size_t>(blk + nb * pitch) * sizeof(float);
      if (bytes > budget || nb * pnl > 32768) continue;
      if (nb * pnl > best_elems) {
        best_elems = nb * pnl;
        best_nl = log_nl;
        best_nb = log_nb;
        best_blk = blk;
        best_pitch = pitch;
      }
      break;  // smaller NB only shrinks the tile for this NL
    }
  }
  if (best_nl < 0) return false;
  const int NL = 1 << best_nl, nb = 1 << best_nb;
  p = hit::BflyPass();
  p.outer = outer;
  p.axis = axis;
  p.P = static_cast<int>(P);
  p.S_in = S_in;
  p.NL = NL;
  p.log_nl = best_nl;
  p.NB = nb;
  p.log_nb = best_nb;
  p.div_pnl = hit::make_fastdiv(static_cast<uint32_t>(P * NL));
  p.pitch = static_cast<int>(best_pitch);
  p.n_tiles = (len / (P * S_in)) * (S_in / NL);
  p.blk_floats = static_cast<int>(best_blk);
  p.ns = cnt;
  int ofs = 0;
  for (int k = 0; k < cnt; ++k) {
    const int t = order[k];
    hit::BflyStage& st = p.st[k];
    st.blocks = blocks[t];
    st.b = radices[t];
    st.bp = (st.b + 3) / 4 * 4;
    st.ls = static_cast<int>(S[t] / S_in);
    st.div_ls = hit::make_fastdiv(static_cast<uint32_t>(st.ls));
    st.div_bp = hit::make_fastdiv(static_cast<uint32_t>(st.bp));
    st.sofs = ofs;
    st.shared_block = (n_groups[t] == 1 && len / radices[t] != 1) ? 1 : 0;
    st.transpose = transpose ? 1 : 0;
    ofs += (st.shared_block ? 1 : static_cast<int>((P / st.b) * NL)) * st.b * st.bp;
  }
  // enough CTAs to fill the machine a few times over
  const int64_t chunks = (outer + nb - 1) / nb;
  int64_t splits = (4 * 148 + p.n_tiles - 1) / p.n_tiles;
  splits = splits < 1 ? 1 : (splits > chunks ? chunks : splits);
  p.chunks_per_split = (chunks + splits - 1) / splits;
  return true;
}

extern "C" {

int hit_version(void) { return 100; }

const char* hit_status_string(int status) {
  switch (status) {
    case HIT_OK: return "ok";
    case HIT_EINVAL: return "invalid argument";
    case HIT_EUNSUPPORTED: return "unsupported dtype or size";
    case HIT_EALIGN: return "misaligned pointer or leading dimension";
    case HIT_ECUDA: return "CUDA error";
    case HIT_EWORKSPACE: return "workspace missing or too small";
    case HIT_ETIMEOUT: return "a bounded device-side wait gave up";
  }
  return "unknown status";
}

const char* hit_last_error(void) { return g_last_error.c_str(); }

int hit_wait_timeouts(unsigned long long* count, int reset) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_status(e, "hit_wait_timeouts: device synchronize");
  unsigned long long n = 0;
  e = hit::wait_timeouts_stream(&n, reset != 0);
  if (e == cudaSuccess) e = hit::wait_timeouts_mixed(&n, reset != 0);
  if (e == cudaSuccess) e = hit::wait_timeouts_tc(&n, reset != 0);
  if (e == cudaSuccess) e = hit::wait_timeouts_strided(&n, reset != 0);
  if (e != cudaSuccess) return cuda_status(e, "hit_wait_timeouts: counter read");
  if (count != nullptr) *count += n;
  if (n != 0)
    return fail(HIT_ETIMEOUT, "%llu bounded device wait(s) gave up; outputs written since the last check are undefined",
                n);
  return HIT_OK;
}

int hit_wait_selftest(int64_t limit_ns, void* stream) {
  if (limit_ns < 1000 || limit_ns > 1000000000)
    return fail(HIT_EINVAL, "hit_wait_selftest: limit_ns must be in [1000, 1000000000]");
  return cuda_status(hit::launch_wait_selftest(static_cast<uint64_t>(limit_ns), static_cast<cudaStream_t>(stream)),
                     "hit_wait_selftest");
}

size_t hit_workspace_bytes(int op, int64_t rows, int64_t n, int dtype_out, int flags) {
  if (rows <= 0 || n <= 0) return 0;
  const size_t full = static_cast<size_t>(rows) * static_cast<size_t>(n) * 4;
  switch (op) {
    case HIT_OP_RHT: return (flags == 0 && rows > 128 && dtype_out != HIT_F32) ? full : 0;
    case HIT_OP_QUANT: return flags ? full : 0;
    case HIT_OP_DEQUANT: return (flags && dtype_out != HIT_F32) ? full : 0;
    case HIT_OP_BUTTERFLY: return (flags > 1 && dtype_out != HIT_F32) ? full : 0;
  }
  return 0;
}

int rht_forward(const void* x, void* y, int64_t rows, int64_t n, int64_t ldx, int64_t ldy, int dtype_in,
                int dtype_out, const int8_t* signs, int axis, void* workspace, size_t workspace_bytes,
                void* stream) {
  return rht_impl(false, x, y, rows, n, ldx, ldy, dtype_in, dtype_out, signs, axis, workspace, workspace_bytes,
                  stream);
}

int rht_inverse(const void* x, void* y, int64_t rows, int64_t n, int64_t ldx, int64_t ldy, int dtype_in,
                int dtype_out, const int8_t* signs, int axis, void* workspace, size_t workspace_bytes,
                void* stream) {
  return rht_impl(true, x, y, rows, n, ldx, ldy, dtype_in, dtype_out, signs, axis, workspace, workspace_bytes,
                  stream);
}

int butterfly_apply(const void* x, void* y, int64_t rows, int64_t n, int64_t ldx, int64_t ldy, int dtype_in,
                    int dtype_out, int n_stages, const int32_t* radices, const float* const* blocks,
                    const int64_t* n_groups, int transpose, int axis, void* workspace, size_t workspace_bytes,
                    void* stream) {
  const char* fn = "butterfly_apply";
  if (!dtype_ok(dtype_in) || !dtype_ok(dtype_out)) return fail(HIT_EUNSUPPORTED, "%s: unknown dtype", fn);
  if (rows < 0 || n < 1) return fail(HIT_EINVAL, "%s: bad shape", fn);
  if (axis != 0 && axis != 1) return fail(HIT_EINVAL, "%s: axis must be 0 or 1", fn);
  if (n_stages < 1 || n_stages > 16) return fail(HIT_EINVAL, "%s: n_stages must be 1..16", fn);
  if (rows == 0) return ok();
  if (radices == nullptr || blocks == nullptr || n_groups == nullptr)
    return fail(HIT_EINVAL, "%s: radices, blocks and n_groups are required", fn);
  if (x == nullptr || y == nullptr) return fail(HIT_EINVAL, "%s: x and y are required", fn);
  if (ldx < n || ldy < n) return fail(HIT_EINVAL, "%s: leading dimension < n", fn);
  if (!aligned(x, esize(dtype_in)) || !aligned(y, esize(dtype_out))) return fail(HIT_EALIGN, "%s: misaligned x or y", fn);
  const int64_t len = axis == 1 ? n : rows;
  int64_t prod = 1;
  for (int t = 0; t < n_stages; ++t) {
    if (radices[t] < 1 || radices[t] > 64) return fail(HIT_EUNSUPPORTED, "%s: radix %d outside 1..64", fn, radices[t]);
    prod *= radices[t];
    if (prod > (int64_t(1) << 40)) return fail(HIT_EINVAL, "%s: radices overflow", fn);
  }
  if (prod != len) return fail(HIT_EINVAL, "%s: radices multiply to %lld, transform length is %lld", fn,
                               (long long)prod, (long long)len);
  for (int t = 0; t < n_stages; ++t) {
    if (blocks[t] == nullptr || !aligned(blocks[t], 4)) return fail(HIT_EINVAL, "%s: blocks[%d] missing or misaligned", fn, t);
    if (n_groups[t] != 1 && n_groups[t] != len / radices[t])
      return fail(HIT_EINVAL, "%s: n_groups[%d] must be 1 or %lld", fn, t, (long long)(len / radices[t]));
  }
  if (rows == 0) return ok();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* tmp = nullptr;
  int64_t ld_tmp = 0;
  if (n_stages > 1) {
    if (dtype_out == HIT_F32) {
      tmp = y;
      ld_tmp = ldy;
    } else {
      const size_t need = static_cast<size_t>(rows) * static_cast<size_t>(n) * 4;
      if (workspace == nullptr || workspace_bytes < need) return fail(HIT_EWORKSPACE, "%s: needs %zu workspace bytes", fn, need);
      if (!aligned(workspace, 16)) return fail(HIT_EALIGN, "%s: workspace must be 16-byte aligned", fn);
      tmp = workspace;
      ld_tmp = n;
    }
  }
  // Strides, then group consecutive stages (in application order) into passes
  // whose tile and blocks fit the shared-memory budget.
  int64_t S[16];
  {
    int64_t acc = 1;
    for (int t = n_stages - 1; t >= 0; --t) {
      S[t] = acc;
      acc *= radices[t];
    }
  }
  int order[16];
  for (int i = 0; i < n_stages; ++i) order[i] = transpose ? n_stages - 1 - i : i;
  const int64_t outer = axis == 1 ? rows : n;
  std::vector<hit::BflyPass> passes;
  int i = 0;
  while (i < n_stages) {
    hit::BflyPass best;
    bool have = false;
    for (int j = i; j < n_stages; ++j) {  // try to extend the run [i, j]
      hit::BflyPass cand;
      if (!plan_pass(order + i, j - i + 1, radices, S, blocks, n_groups, len, outer, axis, transpose != 0, cand))
        break;
      best = cand;
      have = true;
    }
    if (!have) return fail(HIT_EUNSUPPORTED, "%s: stage %d does not fit in shared memory", fn, order[i]);
    passes.push_back(best);
    i += best.ns;
  }
  const int np = static_cast<int>(passes.size());
  for (int q = 0; q < np; ++q) {
    hit::BflyPass& p = passes[q];
    const bool first = q == 0, last = q == np - 1;
    p.x = first ? x : tmp;
    p.ldx = first ? ldx : ld_tmp;
    p.y = last ? y : tmp;
    p.ldy = last ? ldy : ld_tmp;
    if (!first || !last) {
      if (tmp == nullptr) {  // several passes but a single stage run was expected
        const size_t need = static_cast<size_t>(rows) * static_cast<size_t>(n) * 4;
        return fail(HIT_EWORKSPACE, "%s: needs %zu workspace bytes", fn, need);
      }
    }
    const cudaError_t e = hit::launch_butterfly_pass(first ? dtype_in : HIT_F32, last ? dtype_out : HIT_F32, p, st);
    if (e != cudaSuccess) return cuda_status(e, fn);
  }
  return HIT_OK;
}

// ---------------------------------------------------------------------------
// Tensor-core butterfly planning.  A pass is a run of consecutive stages (in
// application order) whose digits form a range [dlo, dhi]; with P the product
// of its radices and S_in the stride of digit dhi it mixes only the positions
// of a window.  It runs on the tensor cores when its window matrix fits one
// MMA tile:
//   along rows (axis 1): S_in = 1 and P dividing 128: window = 128
//     contiguous positions holding 128 / P groups (a block-diagonal matrix);
//   along columns (axis 0): P in {128, 256} (window = P positions at stride
//     S_in), or S_in = 1 and P a divisor of 128 (window = 128 contiguous
//     positions holding 128 / P groups: a block-diagonal matrix).
// Any other run goes through the SIMT pass.
// ---------------------------------------------------------------------------
namespace {

struct TcPlanPass {
  bool tc = false;
  int kind = 0;              // 0: contiguous row window, 1: column window, 2: strided two-digit row run
  int first = 0, count = 0;  // stages order[first .. first + count)
  int Pw = 0;                // window positions (kind 2: per lo value)
  int64_t step = 1;          // stride of the window positions
  hit::BflyPass simt;
};

bool tc_window(const int* order, int cnt, const int32_t* radices, const int64_t* S, int axis, int64_t outer, int& kind,
               int& Pw, int64_t& step) {
  int dlo = order[0], dhi = order[0];
  for (int k = 1; k < cnt; ++k) {
    dlo = order[k] < dlo ? order[k] : dlo;
    dhi = order[k] > dhi ? order[k] : dhi;
  }
  if (dhi - dlo + 1 != cnt) return false;
  int64_t P = 1;
  for (int t = dlo; t <= dhi; ++t) P *= radices[t];
  const int64_t s_in = S[dhi];
  if (axis == 1) {
    if (s_in == 1) {
      // windows of 128 contiguous positions holding 128 / P groups
      if (P > 128 || 128 % P != 0) return false;
      kind = 0;
      Pw = 128;
      step = 1;
      return true;
    }
    // a strided run puts each window's positions S apart along the row: no
    // MMA operand layout holds them without a transposition (SIMT pass)
    (void)outer;
    return false;
  }
  kind = 1;
  if (P == 128 || P == 256) {
    Pw = int(P);
    step = s_in;
    return true;
  }
  if (s_in == 1 && P <= 128 && 128 % P == 0) {
    Pw = 128;
    step = 1;
    return true;
  }
  return false;
}

// Workspace bytes of a tensor-core pass's window matrices.
size_t tc_matrix_bytes(int kind, int64_t len, int Pw) {
  return kind == 2 ? 0 : size_t(len) * size_t(Pw) * 2;
}

// Passes of the tensor-core plan: from each stage, the longest run that is a
// tensor-core window; otherwise a SIMT pass that stops before the next stage
// at which a tensor-core run could start.
bool plan_tc(int n_stages, const int32_t* radices, const int64_t* S, const float* const* blocks,
             const int64_t* n_groups, int64_t len, int64_t outer, int axis, bool transpose, const int* order,
             std::vector<TcPlanPass>& out) {
  auto tc_from = [&](int i, int& cnt, int& kind, int& Pw, int64_t& step) {
    for (int j = n_stages; j > i; --j)
      if (tc_window(order + i, j - i, radices, S, axis, outer, kind, Pw, step)) {
        cnt = j - i;
        return true;
      }
    return false;
  };
  int i = 0;
  while (i < n_stages) {
    TcPlanPass p;
    int cnt = 0, kind = 0, Pw = 0;
    int64_t step = 1;
    if (tc_from(i, cnt, kind, Pw, step)) {
      p.tc = true;
      p.kind = kind;
      p.first = i;
      p.count = cnt;
      p.Pw = Pw;
      p.step = step;
      // the windows must tile the transform
      if (len % (int64_t(Pw) * step) != 0) return false;
      out.push_back(p);
      i += cnt;
      continue;
    }
    // two adjacent digits along rows at a stride: the register-resident kernel
    if (axis == 1 && i + 1 < n_stages) {
      const int d0 = order[i], d1 = order[i + 1];
      const int dh = d0 < d1 ? d0 : d1, dl = d0 < d1 ? d1 : d0;
      const int64_t s_in = S[dl];
      if (dl == dh + 1 && s_in % 8 == 0 && hit::strided_supported(radices[dh], radices[dl], 2, 4)) {
        p.tc = true;
        p.kind = 2;
        p.first = i;
        p.count = 2;
        p.Pw = radices[dh] * radices[dl];
        p.step = s_in;
        out.push_back(p);
        i += 2;
        continue;
      }
    }
    int limit = n_stages;
    for (int k = i + 1; k < n_stages; ++k) {
      int c2 = 0, k2 = 0, pw2 = 0;
      int64_t st2 = 1;
      if (tc_from(k, c2, k2, pw2, st2)) {
        limit = k;
        break;
      }
    }
    bool have = false;
    for (int j = i; j < limit; ++j) {
      hit::BflyPass cand;
      if (!plan_pass(order + i, j - i + 1, radices, S, blocks, n_groups, len, outer, axis, transpose, cand)) break;
      p.simt = cand;
      have = true;
    }
    if (!have) return false;
    p.tc = false;
    p.first = i;
    p.count = p.simt.ns;
    out.push_back(p);
    i += p.count;
  }
  return true;
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

}  // namespace

extern "C" {

size_t butterfly_tc_workspace_bytes(int64_t rows, int64_t n, int axis, int n_stages, const int32_t* radices,
                                    int transpose) {
  if (rows <= 0 || n <= 0 || n_stages < 1 || n_stages > 16 || radices == nullptr) return 0;
  const int64_t len = axis == 1 ? n : rows;
  int64_t S[16], acc = 1;
  for (int t = n_stages - 1; t >= 0; --t) {
    if (radices[t] < 1) return 0;
    S[t] = acc;
    acc *= radices[t];
  }
  if (acc != len) return 0;
  int order[16];
  for (int i = 0; i < n_stages; ++i) order[i] = transpose ? n_stages - 1 - i : i;
  size_t total = 0;
  int passes = 0, i = 0;
  const int64_t outer = axis == 1 ? rows : n;
  while (i < n_stages) {
    int kind = 0, Pw = 0, NT = 0;
    int64_t step = 1;
    int cnt = 0;
    for (int j = n_stages; j > i; --j)
      if (tc_window(order + i, j - i, radices, S, axis, outer, kind, Pw, step)) {
        cnt = j - i;
        break;
      }
    if (cnt > 0) total += align256(tc_matrix_bytes(kind, len, Pw));
    i += cnt > 0 ? cnt : 1;  // a bound: SIMT runs may merge several stages
    ++passes;
  }
  const size_t inter = align256(size_t(rows) * size_t(n) * 2);
  return total + (passes > 1 ? inter : 0) + (passes > 2 ? inter : 0);
}

}  // extern "C"

static int check_quant_common(const char* fn, int64_t rows, int64_t n, int bits, int group) {
  if (rows < 0) return fail(HIT_EINVAL, "%s: rows < 0", fn);
  if (!is_pow2(n) || n < 32 || n > 32768) return fail(HIT_EUNSUPPORTED, "%s: n must be a power of two in [32, 32768]", fn);
  if (bits < 2 || bits > 4) return fail(HIT_EUNSUPPORTED, "%s: bits must be 2, 3 or 4", fn);
  if (!is_pow2(group) || group < 32 || group > n || group > 4096)
    return fail(HIT_EUNSUPPORTED, "%s: group must be a power of two in [32, min(n, 4096)]", fn);
  return HIT_OK;
}

int rht_quantize_pack(const void* x, int64_t rows, int64_t n, int64_t ldx, int dtype_in, const int8_t* row_signs,
                      const int8_t* col_signs, int bits, int group, uint8_t* codes, float* scales, void* workspace,
                      size_t workspace_bytes, void* stream) {
  const char* fn = "rht_quantize_pack";
  if (!dtype_ok(dtype_in)) return fail(HIT_EUNSUPPORTED, "%s: unknown dtype", fn);
  int r = check_quant_common(fn, rows, n, bits, group);
  if (r) return r;
  if (rows == 0) return ok();
  r = check_rows_operand(x, ldx, n, dtype_in, "x");
  if (r) return r;
  if (codes == nullptr || scales == nullptr) return fail(HIT_EINVAL, "%s: codes and scales are required", fn);
  if (!aligned(codes, 16) || !aligned(scales, 4)) return fail(HIT_EALIGN, "%s: codes must be 16-byte, scales 4-byte aligned", fn);
  if ((row_signs && !aligned(row_signs, 4)) || (col_signs && !aligned(col_signs, 4)))
    return fail(HIT_EALIGN, "%s: signs must be 4-byte aligned", fn);
  const bool two_sided = col_signs != nullptr;
  if (two_sided) {
    if (!is_pow2(rows) || rows > (int64_t(1) << 24)) return fail(HIT_EINVAL, "%s: two-sided needs power-of-two rows", fn);
    const size_t need = static_cast<size_t>(rows) * static_cast<size_t>(n) * 4;
    if (workspace == nullptr || workspace_bytes < need) return fail(HIT_EWORKSPACE, "%s: needs %zu workspace bytes", fn, need);
    if (!aligned(workspace, 16)) return fail(HIT_EALIGN, "%s: workspace must be 16-byte aligned", fn);
  }
  if (rows == 0) return ok();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  hit::RowArgs a;
  a.rows = rows;
  a.pre_signs = row_signs;
  a.norm = inv_sqrt(n);
  a.codes = codes;
  a.scales = scales;
  a.log2g = ilog2(group);
  int dt_rows = dtype_in;
  if (two_sided) {
    float* w = static_cast<float*>(workspace);
    r = run_cols(x, dtype_in, ldx, w, HIT_F32, n, rows, n, col_signs, nullptr, w, n, st);
    if (r) return r;
    a.x = w;
    a.ldx = n;
    dt_rows = HIT_F32;
  } else {
    a.x = x;
    a.ldx = ldx;
  }
  const int logn = ilog2(n);
  cudaError_t e;
  if (use_persistent(logn, a.x, a.ldx, dt_rows))
    e = logn == 12 ? hit::rows_stream_quant(logn, dt_rows, bits, a, st) : hit::rows_direct_quant(logn, dt_rows, bits, a, st);
  else if (bits == 4) e = hit::rows_quant_b4(logn, dt_rows, a, st);
  else if (bits == 3) e = hit::rows_quant_b3(logn, dt_rows, a, st);
  else e = hit::rows_quant_b2(logn, dt_rows, a, st);
  return cuda_status(e, fn);
}

int butterfly_apply_tc(const void* x, void* y, int64_t rows, int64_t n, int64_t ldx, int64_t ldy, int dtype_in,
                       int dtype_out, int n_stages, const int32_t* radices, const float* const* blocks,
                       const int64_t* n_groups, int transpose, int axis, void* workspace, size_t workspace_bytes,
                       void* stream) {
  const char* fn = "butterfly_apply_tc";
  if (dtype_in != HIT_BF16) return fail(HIT_EUNSUPPORTED, "%s: the input must be bf16 (tensor-core operands)", fn);
  if (!dtype_ok(dtype_out)) return fail(HIT_EUNSUPPORTED, "%s: unknown output dtype", fn);
  if (rows < 0 || n < 1) return fail(HIT_EINVAL, "%s: bad shape", fn);
  if (axis != 0 && axis != 1) return fail(HIT_EINVAL, "%s: axis must be 0 or 1", fn);
  if (n_stages < 1 || n_stages > 16) return fail(HIT_EINVAL, "%s: n_stages must be 1..16", fn);
  if (rows == 0) return ok();
  if (radices == nullptr || blocks == nullptr || n_groups == nullptr)
    return fail(HIT_EINVAL, "%s: radices, blocks and n_groups are required", fn);
  if (x == nullptr || y == nullptr) return fail(HIT_EINVAL, "%s: x and y are required", fn);
  if (x == y) return fail(HIT_EINVAL, "%s: x and y must not alias", fn);
  if (ldx < n || ldy < n) return fail(HIT_EINVAL, "%s: leading dimension < n", fn);
  if (!aligned(x, 16) || ldx % 8 != 0 || !aligned(y, 16) || (ldy * int64_t(esize(dtype_out))) % 16 != 0 || n % 8 != 0)
    return fail(HIT_EALIGN, "%s: x, y and their row pitches must be 16-byte aligned and n a multiple of 8", fn);
  if (rows > (int64_t(1) << 31) || n > (int64_t(1) << 31)) return fail(HIT_EUNSUPPORTED, "%s: too large", fn);
  const int64_t len = axis == 1 ? n : rows;
  int64_t prod = 1;
  for (int t = 0; t < n_stages; ++t) {
    if (radices[t] < 1 || radices[t] > 64) return fail(HIT_EUNSUPPORTED, "%s: radix %d outside 1..64", fn, radices[t]);
    prod *= radices[t];
    if (prod > (int64_t(1) << 40)) return fail(HIT_EINVAL, "%s: radices overflow", fn);
  }
  if (prod != len) return fail(HIT_EINVAL, "%s: radices multiply to %lld, transform length is %lld", fn,
                               (long long)prod, (long long)len);
  for (int t = 0; t < n_stages; ++t) {
    if (blocks[t] == nullptr || !aligned(blocks[t], 4)) return fail(HIT_EINVAL, "%s: blocks[%d] missing or misaligned", fn, t);
    if (n_groups[t] != 1 && n_groups[t] != len / radices[t])
      return fail(HIT_EINVAL, "%s: n_groups[%d] must be 1 or %lld", fn, t, (long long)(len / radices[t]));
  }
  int64_t S[16];
  {
    int64_t acc = 1;
    for (int t = n_stages - 1; t >= 0; --t) {
      S[t] = acc;
      acc *= radices[t];
    }
  }
  int order[16];
  for (int i = 0; i < n_stages; ++i) order[i] = transpose ? n_stages - 1 - i : i;
  const int64_t outer = axis == 1 ? rows : n;
  std::vector<TcPlanPass> plan;
  if (!plan_tc(n_stages, radices, S, blocks, n_groups, len, outer, axis, transpose != 0, order, plan))
    return fail(HIT_EUNSUPPORTED, "%s: no pass plan for this schedule", fn);
  // workspace: window matrices of every tensor-core pass, then bf16 intermediates
  const int np = static_cast<int>(plan.size());
  std::vector<size_t> mat_ofs(np, 0);
  size_t need = 0;
  for (int q = 0; q < np; ++q)
    if (plan[q].tc) {
      mat_ofs[q] = need;
      need += align256(tc_matrix_bytes(plan[q].kind, len, plan[q].Pw));
    }
  const size_t inter = align256(size_t(rows) * size_t(n) * 2);
  const size_t inter_ofs = need;
  need += (np > 1 ? inter : 0) + (np > 2 ? inter : 0);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need))
    return fail(HIT_EWORKSPACE, "%s: needs %zu workspace bytes (butterfly_tc_workspace_bytes)", fn, need);
  if (need > 0 && !aligned(workspace, 256)) return fail(HIT_EALIGN, "%s: workspace must be 256-byte aligned", fn);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* buf[2] = {ws + inter_ofs, ws + inter_ofs + inter};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int q = 0; q < np; ++q) {
    const bool first = q == 0, last = q == np - 1;
    const void* src = first ? x : buf[(q - 1) & 1];
    const int64_t ld_src = first ? ldx : n;
    void* dst = last ? y : buf[q & 1];
    const int64_t ld_dst = last ? ldy : n;
    const int dt_dst = last ? dtype_out : HIT_BF16;
    TcPlanPass& p = plan[q];
    if (!p.tc) {
      p.simt.x = src;
      p.simt.ldx = ld_src;
      p.simt.y = dst;
      p.simt.ldy = ld_dst;
      const cudaError_t e = hit::launch_butterfly_pass(HIT_BF16, dt_dst, p.simt, st);
      if (e != cudaSuccess) return cuda_status(e, fn);
      continue;
    }
    if (p.kind == 2) {
      const int t0 = order[p.first], t1 = order[p.first + 1];
      const int dh = t0 < t1 ? t0 : t1, dl = t0 < t1 ? t1 : t0;
      hit::StridedArgs sa;
      sa.x = src;
      sa.y = dst;
      sa.ldx = ld_src;
      sa.ldy = ld_dst;
      sa.rows = rows;
      sa.s = p.step;
      sa.n_hi = len / (int64_t(p.Pw) * p.step);
      sa.blocks_h = blocks[dh];
      sa.blocks_l = blocks[dl];
      sa.shared_h = (n_groups[dh] == 1 && len / radices[dh] != 1) ? 1 : 0;
      sa.shared_l = (n_groups[dl] == 1 && len / radices[dl] != 1) ? 1 : 0;
      sa.transpose = transpose ? 1 : 0;
      sa.h_first = t0 == dh ? 1 : 0;
      const cudaError_t e = hit::launch_bfly_strided(radices[dh], radices[dl], HIT_BF16, dt_dst, sa, st);
      if (e != cudaSuccess) return cuda_status(e, fn);
      continue;
    }
    hit::TcComposeArgs c;
    c.Pw = p.Pw;
    c.step = p.step;
    c.ns = p.count;
    for (int k = 0; k < p.count; ++k) {
      const int t = order[p.first + k];
      c.st[k].blocks = blocks[t];
      c.st[k].b = radices[t];
      c.st[k].stride = S[t];
      c.st[k].shared_block = (n_groups[t] == 1 && len / radices[t] != 1) ? 1 : 0;
      c.st[k].transpose = transpose ? 1 : 0;
      c.st[k].div_s = hit::make_fastdiv(static_cast<uint32_t>(S[t]));
      c.st[k].div_b = hit::make_fastdiv(static_cast<uint32_t>(radices[t]));
    }
    auto* mats = reinterpret_cast<__nv_bfloat16*>(ws + mat_ofs[q]);
    const int64_t n_windows = len / p.Pw;
    cudaError_t e = hit::launch_bfly_compose(c, n_windows, mats, st);
    if (e != cudaSuccess) return cuda_status(e, fn);
    hit::TcPassArgs a;
    a.cols = axis == 0 ? 1 : 0;
    a.Pw = p.Pw;
    a.K = p.Pw;
    a.step = p.step;
    a.L = len;
    a.outer = rows;
    a.ncols = n;
    a.n_windows = static_cast<int>(n_windows);
    if (axis == 1) {
      a.N = p.Pw;
      a.m_halves = 1;
    } else {
      // 128-column data tiles (for K = 256 the output is staged in one
      // buffer so that two data stages fit next to the half window matrix);
      // 64 columns for K = 256 with fp32 results (a 64 KB staged tile)
      a.N = (p.Pw == 256 && dt_dst == HIT_F32) ? 64 : 128;
      a.m_halves = p.Pw / 128;
    }
    a.y = dst;
    a.ldy = ld_dst;
    e = hit::launch_bfly_tc(a, src, ld_src, mats, dt_dst, st);
    if (e != cudaSuccess) return cuda_status(e, fn);
  }
  return HIT_OK;
}

int rht_mixed_quantize_pack(const float* x, int64_t rows, int64_t n, int64_t ldx, const int8_t* signs,
                            const float* mixer, int bits, int group, uint8_t* codes, float* scales, void* stream) {
  const char* fn = "rht_mixed_quantize_pack";
  if (rows < 0) return fail(HIT_EINVAL, "%s: rows < 0", fn);
  if (n != 5120) return fail(HIT_EUNSUPPORTED, "%s: n must be 5120 (radices 8, 8, 8, 5, 2)", fn);
  if (bits != 4 || group != 128) return fail(HIT_EUNSUPPORTED, "%s: 4-bit codes in groups of 128 only", fn);
  if (mixer == nullptr) return fail(HIT_EINVAL, "%s: the 5 x 5 mixer is required", fn);
  if (rows == 0) return ok();
  if (x == nullptr || codes == nullptr || scales == nullptr) return fail(HIT_EINVAL, "%s: NULL operand", fn);
  if (ldx < n) return fail(HIT_EINVAL, "%s: leading dimension %lld < n", fn, (long long)ldx);
  if (!aligned(x, 16) || ldx % 4 != 0) return fail(HIT_EALIGN, "%s: x and its row pitch must be 16-byte aligned", fn);
  if (!aligned(codes, 16) || !aligned(scales, 4))
    return fail(HIT_EALIGN, "%s: codes must be 16-byte, scales 4-byte aligned", fn);
  for (int i = 0; i < 25; ++i)
    if (!std::isfinite(mixer[i])) return fail(HIT_EINVAL, "%s: mixer entries must be finite", fn);
  return cuda_status(hit::rows_mixed5120_quant(x, rows, ldx, signs, mixer, codes, scales,
                                               static_cast<cudaStream_t>(stream)),
                     fn);
}

int dequant_inverse(const uint8_t* codes, const float* scales, int64_t rows, int64_t n, int bits, int group,
                    const int8_t* row_signs, const int8_t* col_signs, void* y, int64_t ldy, int dtype_out,
                    void* workspace, size_t workspace_bytes, void* stream) {
  const char* fn = "dequant_inverse";
  if (!dtype_ok(dtype_out)) return fail(HIT_EUNSUPPORTED, "%s: unknown dtype", fn);
  int r = check_quant_common(fn, rows, n, bits, group);
  if (r) return r;
  if (rows == 0) return ok();
  r = check_rows_operand(y, ldy, n, dtype_out, "y");
  if (r) return r;
  if (codes == nullptr || scales == nullptr) return fail(HIT_EINVAL, "%s: codes and scales are required", fn);
  if (!aligned(codes, 16) || !aligned(scales, 4)) return fail(HIT_EALIGN, "%s: codes must be 16-byte, scales 4-byte aligned", fn);
  if ((row_signs && !aligned(row_signs, 4)) || (col_signs && !aligned(col_signs, 4)))
    return fail(HIT_EALIGN, "%s: signs must be 4-byte aligned", fn);
  const bool two_sided = col_signs != nullptr;
  if (two_sided && (!is_pow2(rows) || rows > (int64_t(1) << 24)))
    return fail(HIT_EINVAL, "%s: two-sided needs power-of-two rows", fn);
  if (two_sided && dtype_out != HIT_F32) {
    const size_t need = static_cast<size_t>(rows) * static_cast<size_t>(n) * 4;
    if (workspace == nullptr || workspace_bytes < need) return fail(HIT_EWORKSPACE, "%s: needs %zu workspace bytes", fn, need);
    if (!aligned(workspace, 16)) return fail(HIT_EALIGN, "%s: workspace must be 16-byte aligned", fn);
  }
  if (rows == 0) return ok();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  hit::RowArgs a;
  a.rows = rows;
  a.codes_in = codes;
  a.scales_in = scales;
  a.log2g = ilog2(group);
  a.norm = inv_sqrt(n);
  a.post_signs = row_signs;
  int dt_rows = dtype_out;
  float* mid = nullptr;
  int64_t ld_mid = 0;
  if (two_sided) {
    if (dtype_out == HIT_F32) {
      mid = static_cast<float*>(y);
      ld_mid = ldy;
    } else {
      mid = static_cast<float*>(workspace);
      ld_mid = n;
    }
    a.y = mid;
    a.ldy = ld_mid;
    dt_rows = HIT_F32;
  } else {
    a.y = y;
    a.ldy = ldy;
  }
  const int logn = ilog2(n);
  cudaError_t e;
  if (bits == 4) e = hit::rows_dequant_b4(logn, dt_rows, a, st);
  else if (bits == 3) e = hit::rows_dequant_b3(logn, dt_rows, a, st);
  else e = hit::rows_dequant_b2(logn, dt_rows, a, st);
  r = cuda_status(e, fn);
  if (r || !two_sided) return r;
  return run_cols(mid, HIT_F32, ld_mid, y, dtype_out, ldy, rows, n, nullptr, col_signs, mid, ld_mid, st);
}

int wht_expand_sparse(float* values, const int32_t* cols, int64_t batch, int64_t rows, int64_t n, int32_t nnz,
                      float scale, float* dense, int mode, void* stream) {
  const char* fn = "wht_expand_sparse";
  if (batch < 0 || rows < 0) return fail(HIT_EINVAL, "%s: negative batch or rows", fn);
  if (!is_pow2(n) || n < 32 || n > 32768) return fail(HIT_EUNSUPPORTED, "%s: n must be a power of two in [32, 32768]", fn);
  if (nnz < 1 || nnz > n) return fail(HIT_EINVAL, "%s: nnz must be in [1, n]", fn);
  if (mode != 0 && mode != 1) return fail(HIT_EINVAL, "%s: mode must be 0 or 1", fn);
  if (batch * rows == 0) return ok();
  if (values == nullptr || cols == nullptr || dense == nullptr) return fail(HIT_EINVAL, "%s: NULL operand", fn);
  if (!aligned(values, 4) || !aligned(cols, 4) || !aligned(dense, 16)) return fail(HIT_EALIGN, "%s: misaligned operand", fn);
  const int64_t total = batch * rows;
  if (total == 0) return ok();
  hit::RowArgs a;
  a.rows = total;
  a.nnz = nnz;
  a.sp_cols = cols;
  a.sp_scale = scale;
  if (mode == 0) {
    a.sp_values = values;
    a.y = dense;
    a.ldy = n;
  } else {
    a.x = dense;
    a.ldx = n;
    a.sp_out = values;
  }
  return cuda_status(hit::rows_sparse_all(ilog2(n), mode, a, static_cast<cudaStream_t>(stream)), fn);
}

int wht_expand_sparse_2d(float* values, const int32_t* cols, int64_t batch, int64_t m, int64_t n, int32_t nnz,
                         float scale, float* dense, int mode, void* workspace, size_t workspace_bytes, void* stream) {
  const char* fn = "wht_expand_sparse_2d";
  if (batch < 0 || m < 1) return fail(HIT_EINVAL, "%s: bad batch or m", fn);
  if (!is_pow2(m) || m > (int64_t(1) << 24)) return fail(HIT_EUNSUPPORTED, "%s: m must be a power of two <= 2^24", fn);
  if (!is_pow2(n) || n < 32 || n > 32768) return fail(HIT_EUNSUPPORTED, "%s: n must be a power of two in [32, 32768]", fn);
  if (nnz < 1 || nnz > n) return fail(HIT_EINVAL, "%s: nnz must be in [1, n]", fn);
  if (mode != 0 && mode != 1) return fail(HIT_EINVAL, "%s: mode must be 0 or 1", fn);
  if (batch == 0) return ok();
  if (values == nullptr || cols == nullptr || dense == nullptr) return fail(HIT_EINVAL, "%s: NULL operand", fn);
  if (!aligned(values, 4) || !aligned(cols, 4) || !aligned(dense, 16)) return fail(HIT_EALIGN, "%s: misaligned operand", fn);
  const size_t mat = static_cast<size_t>(m) * static_cast<size_t>(n);
  float* g = nullptr;
  if (mode == 1) {
    const size_t need = static_cast<size_t>(batch) * mat * 4;
    if (workspace == nullptr || workspace_bytes < need) return fail(HIT_EWORKSPACE, "%s: needs %zu workspace bytes", fn, need);
    if (!aligned(workspace, 16)) return fail(HIT_EALIGN, "%s: workspace must be 16-byte aligned", fn);
    g = static_cast<float*>(workspace);
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  hit::RowArgs a;
  a.rows = batch * m;
  a.nnz = nnz;
  a.sp_cols = cols;
  a.sp_scale = scale;
  if (mode == 0) {
    // rows: scatter + transform (times scale) into dense; then every column
    // of every matrix in place (orthonormal, 1/sqrt(m))
    a.sp_values = values;
    a.y = dense;
    a.ldy = n;
    int r = cuda_status(hit::rows_sparse_all(ilog2(n), 0, a, st), fn);
    if (r) return r;
    for (int64_t b = 0; b < batch; ++b) {
      float* d = dense + static_cast<size_t>(b) * mat;
      r = run_cols(d, HIT_F32, n, d, HIT_F32, n, m, n, nullptr, nullptr, d, n, st);
      if (r) return r;
    }
    return HIT_OK;
  }
  // gradient: columns of every matrix of the incoming dense gradient into the
  // workspace, then rows: transform (times scale) + gather
  for (int64_t b = 0; b < batch; ++b) {
    float* d = dense + static_cast<size_t>(b) * mat;
    float* w = g + static_cast<size_t>(b) * mat;
    const int r = run_cols(d, HIT_F32, n, w, HIT_F32, n, m, n, nullptr, nullptr, w, n, st);
    if (r) return r;
  }
  a.x = g;
  a.ldx = n;
  a.sp_out = values;
  return cuda_status(hit::rows_sparse_all(ilog2(n), 1, a, st), fn);
}

}  // extern "C"
