// wa_api.cu -- the extern "C" entry points of libwa (declared in include/wa.h):
// host-side argument validation, workspace carving, error reporting, tensor-map
// creation, and the sequencing of the kernels of one HSA decode step on a stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "wa_internal.h"

#define WA_VERSION "wa 0.1.0 (sm_100a)"

namespace wa {

namespace {
thread_local std::string g_last_error;

// Device error word: one per device, read and cleared by wa_device_error().
__device__ uint32_t g_err_word;

std::mutex g_mu;
uint32_t* g_err_ptr[64] = {};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// Bump allocator over the caller's workspace (sizes are computed with the same
// carving, so "measure" mode just counts).
struct Carver {
  char* base;
  size_t used = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <typename T>
  T* take(size_t count) {
    const size_t off = used;
    used = align_up(used + count * sizeof(T));
    return base ? reinterpret_cast<T*>(base + off) : nullptr;
  }
};

size_t elem_size(wa_dtype dt) { return dt == WA_BF16 ? 2 : 4; }
int ceil_div(int a, int b) { return (a + b - 1) / b; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

wa_status set_error(wa_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

wa_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(WA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return WA_OK;
}

uint32_t* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_err_word) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<uint32_t*>(p);
  }
  return g_err_ptr[dev];
}

bool make_tmap_bf16_2d(void* tmap, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
        return false;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  if (!aligned16(base) || row_bytes % 16 != 0) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(static_cast<CUtensorMap*>(tmap), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                              const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A second stream (and the fork / join events) per host thread and device, on
// which the decode step runs the projection and the linear branch concurrently with
// block selection.  Created on first use; no device memory is allocated.
// The step's internal streams: `stream` takes the projection and the linear branch;
// `hi` (the device's highest stream priority) takes block selection and the work
// list, so that when both have CTAs waiting for an SM the selection side, which the
// sparse branch waits for first, is served first.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr;
  cudaEvent_t join = nullptr;
  cudaStream_t hi = nullptr;
  cudaEvent_t hi_join = nullptr;
};
thread_local SideStream t_side[64];

wa_status side_stream(SideStream** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return set_error(WA_ERR_CUDA, "cudaGetDevice failed");
  SideStream& s = t_side[dev];
  if (!s.stream) {
    int least = 0, greatest = 0;
    cudaDeviceGetStreamPriorityRange(&least, &greatest);
    if (cudaStreamCreateWithFlags(&s.stream, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithPriority(&s.hi, cudaStreamNonBlocking, greatest) != cudaSuccess ||
        cudaEventCreateWithFlags(&s.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&s.join, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&s.hi_join, cudaEventDisableTiming) != cudaSuccess)
      return set_error(WA_ERR_CUDA, "could not create the side stream");
  }
  *out = &s;
  return WA_OK;
}

}  // namespace wa

using namespace wa;

#define WA_REQUIRE(cond, ...)                                     \
  do {                                                            \
    if (!(cond)) return set_error(WA_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)
#define WA_TRY(expr)                    \
  do {                                  \
    const wa_status s_ = (expr);        \
    if (s_ != WA_OK) return s_;         \
  } while (0)

namespace wa_detail {

wa_status check_shape(int H, int d, int B, wa_dtype dt) {
  WA_REQUIRE(H >= 1, "H must be >= 1");
  WA_REQUIRE(dt == WA_F32 || dt == WA_BF16, "dtype must be WA_F32 or WA_BF16");
  if (d != 64 && d != 128) return set_error(WA_ERR_UNSUPPORTED, "d must be 64 or 128 (got %d)", d);
  if (B != 64) return set_error(WA_ERR_UNSUPPORTED, "B must be 64 (got %d)", B);
  const int vec = dt == WA_BF16 ? 8 : 4;
  if (static_cast<long long>(H) * d / vec > 1024) return set_error(WA_ERR_UNSUPPORTED, "H*d too large");
  return WA_OK;
}

wa_status check_ws(void* ws, size_t have, size_t need) {
  if (need == 0) return WA_OK;
  if (!ws || have < need || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return set_error(WA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned (got %zu)", need,
                     have);
  return WA_OK;
}

uint32_t* errw() { return device_error_word(); }

// ---- S1 internals (shared by wa_page_score and wa_hsa_step)
struct PageScoreWs {
  double* q_blocksum;   // [n_qb][cols]
  double* qbar;         // [cols]
  double* q_blockmean;  // [n_qb][cols]
  double* k_blocksum;   // [n_c][nbp][cols] by candidate position (nullable: page index)
  double* scratch;      // column-sum parts and partial dot products of the page scores
  unsigned* counters;   // completion counters of the page-score kernel
};

PageScoreWs carve_page_score(Carver& c, int Nq, int H, int d, int n_c, int T_p, int B, bool k_blocks) {
  PageScoreWs w{};
  const int cols = H * d;
  const int n_qb = ceil_div(Nq, B);
  w.q_blocksum = c.take<double>(static_cast<size_t>(n_qb) * cols);
  w.qbar = c.take<double>(cols);
  w.q_blockmean = c.take<double>(static_cast<size_t>(n_qb) * cols);
  w.k_blocksum = k_blocks ? c.take<double>(static_cast<size_t>(n_c) * ceil_div(T_p, B) * cols) : nullptr;
  w.scratch = c.take<double>(page_alpha_scratch_doubles(cols, n_c));
  w.counters = c.take<unsigned>(page_alpha_counters(cols));
  return w;
}

// One pass over the queries and the candidate pages (block sums, float64), then the
// page scores and the top-K_p pages from those sums.  The candidate pages are row
// *chunk (or row 0) of chunk_pages [n_chunks][n_c].  With a page index the pass reads
// only the queries and the scores read the index's block sums of the candidates.
wa_status run_page_score(const PageScoreWs& w, const void* q, int Nq, int H, int d,
                         const void* k_pool, int n_pool_pages, int T_p, const int32_t* chunk_pages,
                         const int32_t* chunk, int n_chunks, int n_c, int K_p, int B, wa_dtype dt,
                         double* alpha, int32_t* sel, int32_t* sel_pos, cudaStream_t st,
                         const double* page_index = nullptr) {
  const int cols = H * d;
  uint32_t* err = errw();
  if (!err) return set_error(WA_ERR_CUDA, "no device error word (is a CUDA device present?)");
  const int n_qb = ceil_div(Nq, B), nbp = ceil_div(T_p, B);
  BlockSumSeg seg[2];
  seg[0].x = q; seg[0].rows = Nq; seg[0].n_blocks = n_qb; seg[0].sums = w.q_blocksum; seg[0].nb_out = n_qb;
  int n_segs = 1;
  if (!page_index) {
    BlockSumSeg& g = seg[1];
    g.x = k_pool; g.ids = chunk_pages; g.chunk = chunk; g.id_rows = n_chunks; g.n_src = n_c;
    g.n_pages = n_pool_pages; g.rows = T_p; g.n_blocks = nbp; g.sums = w.k_blocksum; g.nb_out = nbp;
    n_segs = 2;
  }
  WA_TRY(launch_block_sums(dt, cols, B, seg, n_segs, w.counters, page_alpha_counters(cols), err, st));
  return launch_page_alpha(w.q_blocksum, n_qb, Nq, B, cols, page_index ? page_index : w.k_blocksum,
                           page_index ? chunk_pages : nullptr, n_pool_pages, nbp, chunk_pages, chunk,
                           n_chunks, n_c, T_p, H, d, K_p, w.qbar, w.q_blockmean, w.scratch, w.counters,
                           alpha, sel, sel_pos, err, st);
}

// Block sums of one contiguous buffer of `rows` rows (all its blocks).
wa_status buffer_block_sums(const void* x, int rows, int cols, int B, wa_dtype dt, double* sums,
                            uint32_t* err, cudaStream_t st) {
  BlockSumSeg g;
  g.x = x; g.rows = rows; g.n_blocks = ceil_div(rows, B); g.sums = sums; g.nb_out = g.n_blocks;
  return launch_block_sums(dt, cols, B, &g, 1, nullptr, 0, err, st);
}

}  // namespace wa_detail
using namespace wa_detail;

extern "C" {

const char* wa_last_error(void) { return g_last_error.c_str(); }
const char* wa_version(void) { return WA_VERSION; }

wa_status wa_device_error(void* stream, uint32_t* flags) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* p = errw();
  if (!p) return set_error(WA_ERR_CUDA, "no CUDA device");
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return set_error(WA_ERR_CUDA, "stream sync: %s", cudaGetErrorString(e));
  uint32_t v = 0;
  e = cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return set_error(WA_ERR_CUDA, "read error word: %s", cudaGetErrorString(e));
  if (v) cudaMemset(p, 0, sizeof(uint32_t));
  if (flags) *flags = v;
  if (v) return set_error(WA_ERR_DEVICE, "device error flags 0x%x", v);
  return WA_OK;
}

// ------------------------------------------------------------------ S0
wa_status wa_prompt_select(const float* e_cur, const float* e_chunks, int n_chunks, int D,
                           int32_t* chunk_out, void* stream) {
  WA_REQUIRE(e_cur && e_chunks && chunk_out, "NULL pointer");
  WA_REQUIRE(n_chunks >= 1 && D >= 1, "n_chunks and D must be >= 1");
  WA_REQUIRE(n_chunks <= 4096, "at most 4096 chunks");
  uint32_t* err = errw();
  if (!err) return set_error(WA_ERR_CUDA, "no CUDA device");
  return launch_prompt_select(e_cur, e_chunks, n_chunks, D, chunk_out, err,
                              static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------ S1
size_t wa_page_score_workspace_size(int Nq, int H, int d, int n_c, int T_p, int B) {
  if (Nq < 1 || H < 1 || d < 1 || n_c < 1 || T_p < 1 || B < 1) return 0;
  Carver c(nullptr);
  carve_page_score(c, Nq, H, d, n_c, T_p, B, true);
  c.take<int32_t>(n_c);
  return c.used;
}

wa_status wa_page_score(const void* q, int Nq, int H, int d, const void* k_pool, int n_pool_pages,
                        int T_p, const int32_t* cand_pages, int n_c, int K_p, int B, wa_dtype dtype,
                        double* alpha, int32_t* sel, double* k_blockmean, void* ws, size_t ws_bytes,
                        void* stream) {
  WA_REQUIRE(q && k_pool && cand_pages && alpha && sel, "NULL pointer");
  WA_REQUIRE(Nq >= 1 && T_p >= 1 && n_pool_pages >= 1 && n_c >= 1, "sizes must be >= 1");
  WA_REQUIRE(K_p >= 1 && K_p <= n_c, "need 1 <= K_p <= n_c (K_p=%d, n_c=%d)", K_p, n_c);
  WA_REQUIRE(n_c <= 4096, "n_c must be <= 4096");
  WA_TRY(check_shape(H, d, B, dtype));
  if (k_blockmean && T_p % B != 0)
    return set_error(WA_ERR_UNSUPPORTED, "k_blockmean needs T_p %% B == 0");
  WA_TRY(check_ws(ws, ws_bytes, wa_page_score_workspace_size(Nq, H, d, n_c, T_p, B)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carver c(ws);
  PageScoreWs w = carve_page_score(c, Nq, H, d, n_c, T_p, B, true);
  int32_t* sel_pos = c.take<int32_t>(n_c);
  WA_TRY(run_page_score(w, q, Nq, H, d, k_pool, n_pool_pages, T_p, cand_pages, nullptr, 1, n_c, K_p, B,
                        dtype, alpha, sel, sel_pos, st));
  if (k_blockmean) {
    const size_t n = static_cast<size_t>(n_c) * (T_p / B) * H * d;
    WA_TRY(launch_scale_copy(w.k_blocksum, k_blockmean, n, 1.0 / B, st));
  }
  return WA_OK;
}

// ------------------------------------------------------------------ S2
wa_status wa_gather_pages(const void* k_pool, const void* v_pool, int n_pool_pages, int T_p, int H,
                          int d, const int32_t* sel, int K_p, wa_dtype dtype, void* k_act,
                          void* v_act, void* stream) {
  WA_REQUIRE(k_pool && v_pool && sel && k_act && v_act, "NULL pointer");
  WA_REQUIRE(n_pool_pages >= 1 && T_p >= 1 && H >= 1 && d >= 1 && K_p >= 1, "sizes must be >= 1");
  WA_REQUIRE(dtype == WA_F32 || dtype == WA_BF16, "bad dtype");
  const size_t page_bytes = static_cast<size_t>(T_p) * H * d * elem_size(dtype);
  if (page_bytes % 16 != 0 || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(k_act) ||
      !aligned16(v_act))
    return set_error(WA_ERR_UNSUPPORTED, "gather needs 16-byte aligned pages");
  uint32_t* err = errw();
  if (!err) return set_error(WA_ERR_CUDA, "no CUDA device");
  return launch_gather(k_pool, v_pool, n_pool_pages, page_bytes, sel, K_p, k_act, v_act, err,
                       static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------ token order
// Cube-tile order (Appendix A.1.3), in closed form: the cubes before cube (a, b, c)
// hold a*C_t*H_l*W_l tokens (whole frame slabs), then ct*b*C_h*W_l (whole row bands
// of slab a) and ct*ch*c*C_w (cubes to the left in band b), where ct and ch are the
// (possibly cut short) extents of slab a and band b; inside the cube a token's
// offset is raster over the cube's extents.
wa_status wa_cube_order(int T, int H_l, int W_l, int C_t, int C_h, int C_w, int32_t* perm) {
  WA_REQUIRE(perm, "NULL pointer");
  WA_REQUIRE(T >= 1 && H_l >= 1 && W_l >= 1 && C_t >= 1 && C_h >= 1 && C_w >= 1,
             "sizes must be >= 1");
  const long long n = static_cast<long long>(T) * H_l * W_l;
  WA_REQUIRE(n <= INT_MAX, "more than 2^31 - 1 tokens");
  const long long plane = static_cast<long long>(H_l) * W_l;
  for (int t = 0; t < T; ++t) {
    const int a = t / C_t, ct = std::min(C_t, T - a * C_t);
    for (int h = 0; h < H_l; ++h) {
      const int b = h / C_h, ch = std::min(C_h, H_l - b * C_h);
      for (int w = 0; w < W_l; ++w) {
        const int c = w / C_w, cw = std::min(C_w, W_l - c * C_w);
        const long long cube0 = static_cast<long long>(a) * C_t * plane +
                                static_cast<long long>(ct) * b * C_h * W_l +
                                static_cast<long long>(ct) * ch * c * C_w;
        const long long local =
            (static_cast<long long>(t - a * C_t) * ch + (h - b * C_h)) * cw + (w - c * C_w);
        perm[cube0 + local] = static_cast<int32_t>(t * plane + static_cast<long long>(h) * W_l + w);
      }
    }
  }
  return WA_OK;
}

wa_status wa_permute_rows(const void* src, void* dst, const int32_t* perm, int n_rows,
                          size_t row_bytes, int inverse, void* stream) {
  WA_REQUIRE(src && dst && perm, "NULL pointer");
  WA_REQUIRE(n_rows >= 1 && row_bytes >= 1, "sizes must be >= 1");
  WA_REQUIRE(n_rows <= INT_MAX - (1 << 20), "too many rows (at most 2^31 - 2^20)");
  if (row_bytes % 16 != 0 || !aligned16(src) || !aligned16(dst))
    return set_error(WA_ERR_UNSUPPORTED, "permute_rows needs 16-byte aligned rows");
  uint32_t* err = errw();
  if (!err) return set_error(WA_ERR_CUDA, "no CUDA device");
  return launch_permute_rows(src, dst, perm, n_rows, row_bytes, inverse, err,
                             static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------ S3
// ------------------------------------------------------------------ pool
wa_status wa_pool_index(const void* k_pool, int n_pool_pages, int T_p, int H, int d, int B,
                        wa_dtype dtype, const int32_t* pages, int n_pages, double* page_index,
                        void* stream) {
  WA_REQUIRE(k_pool && pages && page_index, "NULL pointer");
  WA_REQUIRE(n_pool_pages >= 1 && T_p >= 1 && n_pages >= 1, "sizes must be >= 1");
  WA_TRY(check_shape(H, d, B, dtype));
  if (T_p % B != 0) return set_error(WA_ERR_UNSUPPORTED, "the page index needs T_p %% B == 0");
  uint32_t* err = errw();
  if (!err) return set_error(WA_ERR_CUDA, "no CUDA device");
  BlockSumSeg g;
  g.x = k_pool; g.ids = pages; g.n_src = n_pages; g.n_pages = n_pool_pages; g.rows = T_p;
  g.n_blocks = T_p / B; g.sums = page_index; g.nb_out = T_p / B; g.by_page = 1;
  return launch_block_sums(dtype, H * d, B, &g, 1, nullptr, 0, err, static_cast<cudaStream_t>(stream));
}

wa_status wa_pool_append(void* k_pool, void* v_pool, int n_pool_pages, int T_p, int H, int d,
                         wa_dtype dtype, const void* k_new, const void* v_new, int n_tokens,
                         long long token_offset, double* page_index, int B, void* stream) {
  WA_REQUIRE(k_pool && v_pool && k_new && v_new, "NULL pointer");
  WA_REQUIRE(n_pool_pages >= 1 && T_p >= 1 && n_tokens >= 1, "sizes must be >= 1");
  WA_REQUIRE(dtype == WA_F32 || dtype == WA_BF16, "bad dtype");
  WA_REQUIRE(H >= 1 && d >= 1, "sizes must be >= 1");
  const long long rows = static_cast<long long>(n_pool_pages) * T_p;
  WA_REQUIRE(rows < (1LL << 31), "pool too large");
  WA_REQUIRE(token_offset >= 0 && token_offset + n_tokens <= rows,
             "rows [%lld, %lld) fall outside the pool's %lld rows", token_offset,
             token_offset + n_tokens, rows);
  if (page_index) {
    WA_TRY(check_shape(H, d, B, dtype));
    if (T_p % B != 0) return set_error(WA_ERR_UNSUPPORTED, "the page index needs T_p %% B == 0");
  }
  const size_t row_bytes = static_cast<size_t>(H) * d * elem_size(dtype);
  if (row_bytes % 16 != 0 || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(k_new) ||
      !aligned16(v_new))
    return set_error(WA_ERR_UNSUPPORTED, "pool append needs 16-byte aligned rows");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t off = static_cast<size_t>(token_offset) * row_bytes;
  const size_t n16 = static_cast<size_t>(n_tokens) * row_bytes / 16;
  WA_TRY(launch_copy16(k_new, static_cast<char*>(k_pool) + off, n16, st));
  WA_TRY(launch_copy16(v_new, static_cast<char*>(v_pool) + off, n16, st));
  if (!page_index) return WA_OK;
  uint32_t* err = errw();
  if (!err) return set_error(WA_ERR_CUDA, "no CUDA device");
  const int b_first = static_cast<int>(token_offset / B);
  const int b_last = static_cast<int>((token_offset + n_tokens - 1) / B);
  // the touched blocks of the pool's flat token space (T_p % B == 0: a block never
  // straddles pages, and flat block b is block b % (T_p/B) of page b / (T_p/B))
  BlockSumSeg g;
  g.x = k_pool; g.rows = static_cast<int>(rows); g.block0 = b_first; g.n_blocks = b_last - b_first + 1;
  g.sums = page_index; g.nb_out = static_cast<int>(rows / B);
  return launch_block_sums(dtype, H * d, B, &g, 1, nullptr, 0, err, st);
}

namespace wa_detail {
namespace {  // internal linkage: nothing here is exported from libwa
struct BlockSelectWs {
  double* qsum;
  double* qbar;
  double* qmean;
  double* ksum;
  double* scores;
};
BlockSelectWs carve_block_select(Carver& c, int Nq, int H, int d, int L, int B, wa_dtype dt) {
  BlockSelectWs w{};
  const int cols = H * d;
  const int n_qb = ceil_div(Nq, B), n_kb = ceil_div(L, B);
  (void)dt;
  w.qsum = c.take<double>(static_cast<size_t>(n_qb) * cols);
  w.qbar = c.take<double>(cols);
  w.qmean = c.take<double>(static_cast<size_t>(n_qb) * cols);
  w.ksum = c.take<double>(static_cast<size_t>(n_kb) * cols);
  w.scores = reinterpret_cast<double*>(c.take<char>(block_scores_bytes(H, n_qb, n_kb)));
  return w;
}
}  // namespace
}  // namespace wa_detail

size_t wa_block_select_workspace_size(int Nq, int H, int d, int L, int B) {
  if (Nq < 1 || H < 1 || d < 1 || L < 1 || B < 1) return 0;
  Carver c(nullptr);
  carve_block_select(c, Nq, H, d, L, B, WA_F32);
  return c.used;
}

wa_status wa_block_select(const void* q, int Nq, int H, int d, const void* k_act,
                          const double* k_blockmean, int L, int B, wa_dtype dtype, const float* tau,
                          int32_t* blk_idx, int32_t* blk_cnt, uint32_t* blk_mask, void* ws,
                          size_t ws_bytes, void* stream) {
  WA_REQUIRE(q && tau, "NULL pointer");
  WA_REQUIRE((k_act != nullptr) != (k_blockmean != nullptr),
             "exactly one of k_act and k_blockmean must be given");
  WA_REQUIRE(Nq >= 1 && L >= 1, "sizes must be >= 1");
  WA_TRY(check_shape(H, d, B, dtype));
  const int n_kb = ceil_div(L, B);
  WA_REQUIRE(n_kb <= 8192, "at most 8192 key blocks");
  WA_TRY(check_ws(ws, ws_bytes, wa_block_select_workspace_size(Nq, H, d, L, B)));
  uint32_t* err = errw();
  if (!err) return set_error(WA_ERR_CUDA, "no CUDA device");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carver c(ws);
  BlockSelectWs w = carve_block_select(c, Nq, H, d, L, B, dtype);
  const int cols = H * d;
  WA_TRY(buffer_block_sums(q, Nq, cols, B, dtype, w.qsum, err, st));
  WA_TRY(launch_qmeans(w.qsum, ceil_div(Nq, B), Nq, B, cols, w.qbar, w.qmean, st));
  KeyMeans km;
  km.L = L;
  if (k_act) {
    WA_TRY(buffer_block_sums(k_act, L, cols, B, dtype, w.ksum, err, st));
    km.data = w.ksum;
    km.is_sum = 1;
  } else {
    km.data = k_blockmean;
    km.is_sum = 0;
  }
  return launch_block_select(w.qmean, Nq, H, d, B, km, n_kb, n_kb, tau, w.scores, blk_idx, blk_cnt,
                             blk_mask, st);
}

// ------------------------------------------------------------------ S4a
size_t wa_linear_project_workspace_size(int L, int H, int d, int r, wa_dtype dtype) {
  if (L < 1 || H < 1 || d < 1 || r < 1) return 0;
  if (dtype == WA_BF16) return align_up(umma_project_ws_bytes(L, H, d, r));
  return 0;
}

wa_status wa_linear_project(const void* k_act, const void* v_act, const void* e_k, const void* e_v,
                            int L, int H, int d, int r, wa_dtype dtype, void* k_til, void* v_til,
                            void* ws, size_t ws_bytes, void* stream) {
  WA_REQUIRE(k_act && v_act && e_k && e_v && k_til && v_til, "NULL pointer");
  WA_REQUIRE(L >= 1 && r >= 1, "sizes must be >= 1");
  WA_TRY(check_shape(H, d, 64, dtype));
  WA_TRY(check_ws(ws, ws_bytes, wa_linear_project_workspace_size(L, H, d, r, dtype)));
  uint32_t* err = errw();
  if (!err) return set_error(WA_ERR_CUDA, "no CUDA device");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  RowSource rs;
  rs.k = k_act; rs.v = v_act; rs.page_rows = L; rs.n_pages = 1; rs.L = L;
  if (dtype == WA_BF16)
    return launch_umma_project(k_act, v_act, rs, e_k, e_v, L, H, d, r, k_til, v_til, ws, err, st);
  WA_TRY(launch_simt_project(static_cast<const float*>(k_act), nullptr, L, 1,
                             static_cast<const float*>(e_k), L, H * d, r, d, 0,
                             static_cast<float*>(k_til), err, st));
  return launch_simt_project(static_cast<const float*>(v_act), nullptr, L, 1,
                             static_cast<const float*>(e_v), L, H * d, r, d, 0,
                             static_cast<float*>(v_til), err, st);
}

wa_status wa_linear_project_heads(const void* k_act, const void* v_act, const void* e_k,
                                  const void* e_v, int L, int H, int d, int r, wa_dtype dtype,
                                  long long e_head_stride, void* k_til, void* v_til, void* ws,
                                  size_t ws_bytes, void* stream) {
  WA_REQUIRE(k_act && v_act && e_k && e_v && k_til && v_til, "NULL pointer");
  WA_REQUIRE(L >= 1 && r >= 1, "sizes must be >= 1");
  WA_TRY(check_shape(H, d, 64, dtype));
  WA_REQUIRE(e_head_stride == 0 || e_head_stride == static_cast<long long>(L) * r,
             "e_head_stride must be 0 (one E for all heads) or L*r (one per head)");
  if (e_head_stride == 0)
    return wa_linear_project(k_act, v_act, e_k, e_v, L, H, d, r, dtype, k_til, v_til, ws, ws_bytes, stream);
  WA_TRY(check_ws(ws, ws_bytes, wa_linear_project_workspace_size(L, H, d, r, dtype)));
  uint32_t* err = errw();
  if (!err) return set_error(WA_ERR_CUDA, "no CUDA device");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  RowSource rs;
  rs.k = k_act; rs.v = v_act; rs.page_rows = L; rs.n_pages = 1; rs.L = L;
  if (dtype == WA_BF16)
    return launch_umma_project(k_act, v_act, rs, e_k, e_v, L, H, d, r, k_til, v_til, ws, err, st, true);
  WA_TRY(launch_simt_project(static_cast<const float*>(k_act), nullptr, L, 1,
                             static_cast<const float*>(e_k), L, H * d, r, d, e_head_stride,
                             static_cast<float*>(k_til), err, st));
  return launch_simt_project(static_cast<const float*>(v_act), nullptr, L, 1,
                             static_cast<const float*>(e_v), L, H * d, r, d, e_head_stride,
                             static_cast<float*>(v_til), err, st);
}

// ------------------------------------------------------------------ S4b+S5+S6
size_t wa_hsa_attention_workspace_size(int Nq, int H, int d, int L, int B, int r, wa_dtype dtype) {
  if (Nq < 1 || H < 1 || d < 1 || L < 1 || B < 1 || r < 1) return 0;
  Carver c(nullptr);
  c.take<float>(static_cast<size_t>(Nq) * H * d);                  // gated linear branch
  if (dtype == WA_BF16) c.take<char>(sparse_attn_ws_bytes(H, Nq, d, B));
  return c.used;
}

namespace wa_detail {
namespace {  // internal linkage: nothing here is exported from libwa
wa_status run_attention(const void* q, int Nq, int H, int d, RowSource rs, int B,
                        const uint32_t* blk_mask, const void* k_til, const void* v_til, int r,
                        const float* gate, const float* gate_lin, wa_dtype dtype, void* out,
                        float* o_sp, float* o_lin, float* lin_ws, void* scratch, cudaStream_t st,
                        void* const* events = nullptr) {
  auto mark = [&](int k) {
    if (events && events[k]) cudaEventRecord(static_cast<cudaEvent_t>(events[k]), st);
  };
  uint32_t* err = errw();
  if (!err) return set_error(WA_ERR_CUDA, "no CUDA device");
  const int n_qb = ceil_div(Nq, B);
  const int n_kb = ceil_div(rs.L, B);
  const int W = ceil_div(n_kb, 32);
  RowSource lin;
  lin.k = k_til; lin.v = v_til; lin.page_rows = r; lin.n_pages = 1; lin.L = r;
  if (dtype == WA_BF16) {
    WA_TRY(launch_linear_attention(q, Nq, H, d, lin, B, gate, gate_lin, lin_ws, o_lin, err, st));
    mark(5);
    return launch_sparse_attention(q, Nq, H, d, rs, B, blk_mask, gate, lin_ws, out, o_sp, scratch,
                                   err, st, events);
  }
  WA_TRY(launch_simt_attention(0, static_cast<const float*>(q), Nq, H, d, lin, B, nullptr, 0, gate,
                               gate_lin, lin_ws, nullptr, o_lin, err, st));
  mark(5);
  mark(6);
  return launch_simt_attention(1, static_cast<const float*>(q), Nq, H, d, rs, B, blk_mask, W, gate,
                               nullptr, lin_ws, static_cast<float*>(out), o_sp, err, st);
}

wa_status check_rank(int r, wa_dtype dt) {
  if (dt == WA_BF16 && r != 128 && r != 256)
    return set_error(WA_ERR_UNSUPPORTED, "bf16 path needs r in {128, 256} (got %d)", r);
  if (dt == WA_F32 && (r > 4096)) return set_error(WA_ERR_UNSUPPORTED, "r too large");
  return WA_OK;
}
}  // namespace
}  // namespace wa_detail
using namespace wa_detail;

namespace wa_detail {
namespace {  // internal linkage: nothing here is exported from libwa
wa_status hsa_attention(const void* q, int Nq, int H, int d, const void* k_act, const void* v_act,
                        int L, int B, const uint32_t* blk_mask, const void* k_til, const void* v_til,
                        int r, const float* gate, const float* gate_lin, wa_dtype dtype, void* out,
                        float* o_sp, float* o_lin, void* ws, size_t ws_bytes, void* stream) {
  WA_REQUIRE(q && k_act && v_act && blk_mask && k_til && v_til && gate && out, "NULL pointer");
  WA_REQUIRE(Nq >= 1 && L >= 1 && r >= 1, "sizes must be >= 1");
  WA_TRY(check_shape(H, d, B, dtype));
  WA_TRY(check_rank(r, dtype));
  WA_REQUIRE(ceil_div(L, B) <= 8192, "at most 8192 key blocks");
  WA_TRY(check_ws(ws, ws_bytes, wa_hsa_attention_workspace_size(Nq, H, d, L, B, r, dtype)));
  Carver c(ws);
  float* lin_ws = c.take<float>(static_cast<size_t>(Nq) * H * d);
  void* scratch = dtype == WA_BF16 ? c.take<char>(sparse_attn_ws_bytes(H, Nq, d, B)) : nullptr;
  RowSource rs;
  rs.k = k_act; rs.v = v_act; rs.page_rows = L; rs.n_pages = 1; rs.L = L;
  return run_attention(q, Nq, H, d, rs, B, blk_mask, k_til, v_til, r, gate, gate_lin, dtype, out, o_sp,
                       o_lin, lin_ws, scratch, static_cast<cudaStream_t>(stream));
}
}  // namespace
}  // namespace wa_detail

wa_status wa_hsa_attention(const void* q, int Nq, int H, int d, const void* k_act, const void* v_act,
                           int L, int B, const uint32_t* blk_mask, const void* k_til,
                           const void* v_til, int r, const float* gate, wa_dtype dtype, void* out,
                           float* o_sp, float* o_lin, void* ws, size_t ws_bytes, void* stream) {
  return hsa_attention(q, Nq, H, d, k_act, v_act, L, B, blk_mask, k_til, v_til, r, gate, nullptr,
                       dtype, out, o_sp, o_lin, ws, ws_bytes, stream);
}

wa_status wa_hsa_attention_gated2(const void* q, int Nq, int H, int d, const void* k_act,
                                  const void* v_act, int L, int B, const uint32_t* blk_mask,
                                  const void* k_til, const void* v_til, int r, const float* gate_sp,
                                  const float* gate_lin, wa_dtype dtype, void* out, float* o_sp,
                                  float* o_lin, void* ws, size_t ws_bytes, void* stream) {
  WA_REQUIRE(gate_lin, "NULL pointer");
  return hsa_attention(q, Nq, H, d, k_act, v_act, L, B, blk_mask, k_til, v_til, r, gate_sp, gate_lin,
                       dtype, out, o_sp, o_lin, ws, ws_bytes, stream);
}

// ------------------------------------------------------------------ step
namespace wa_detail {
namespace {  // internal linkage: nothing here is exported from libwa
struct StepWs {
  int32_t* chunk;
  PageScoreWs ps;
  double* alpha;
  int32_t* sel;
  int32_t* sel_pos;
  uint32_t* mask;
  void* k_til;
  void* v_til;
  void* proj;
  float* lin;
  void* attn;         // sparse-attention work list and partials
  void* k_act;
  void* v_act;
  double* ksum;     // non-fused: block sums of the gathered keys
  double* scores;   // float64 pooled block scores
  double* cur_sum;  // block sums of the current chunk's keys (intra-chunk keys)
};

wa_status validate_step(const wa_step_args* a) {
  WA_REQUIRE(a, "NULL args");
  WA_REQUIRE(a->q && a->k_pool && a->v_pool && a->e_k && a->e_v && a->tau && a->gate && a->out &&
                 a->chunk_pages,
             "NULL pointer in wa_step_args");
  WA_REQUIRE(a->Nq >= 1 && a->T_p >= 1 && a->n_pool_pages >= 1 && a->n_c >= 1, "sizes must be >= 1");
  WA_REQUIRE(a->K_p >= 1 && a->K_p <= a->n_c, "need 1 <= K_p <= n_c");
  WA_REQUIRE(a->n_c <= 4096, "n_c must be <= 4096");
  WA_REQUIRE(!a->e_cur || (a->e_chunks && a->n_chunks >= 1 && a->n_chunks <= 4096 && a->D >= 1),
             "bad prompt arguments");
  WA_TRY(check_shape(a->H, a->d, a->B, a->dtype));
  WA_TRY(check_rank(a->r, a->dtype));
  const long long L = static_cast<long long>(a->K_p) * a->T_p;
  WA_REQUIRE(L < (1LL << 31), "K_p*T_p too large");
  WA_REQUIRE(ceil_div(static_cast<int>(L), a->B) <= 8192, "at most 8192 key blocks");
  if (a->fused_gather && a->T_p % a->B != 0)
    return set_error(WA_ERR_UNSUPPORTED, "fused gather needs T_p %% B == 0");
  if (a->page_index && (!a->fused_gather || a->T_p % a->B != 0))
    return set_error(WA_ERR_UNSUPPORTED, "the page index needs fused_gather and T_p %% B == 0");
  WA_REQUIRE(static_cast<long long>(a->n_pool_pages) * a->T_p < (1LL << 31), "pool too large");
  WA_REQUIRE(!a->k_cur == !a->v_cur, "k_cur and v_cur are given together");
  WA_REQUIRE(a->B_inter == 0 || a->B_inter == a->B || a->B_inter == 2 * a->B,
             "B_inter must be 0, B or 2*B (got %d)", a->B_inter);
  WA_REQUIRE(a->e_head_stride == 0 || a->e_head_stride == L * a->r,
             "e_head_stride must be 0 (one E for all heads) or K_p*T_p*r (one per head)");
  if (a->B_inter == 2 * a->B && L % a->B != 0)
    return set_error(WA_ERR_UNSUPPORTED, "B_inter = 2*B needs K_p*T_p %% B == 0");
  if (a->k_cur) {
    if (L % a->B != 0)
      return set_error(WA_ERR_UNSUPPORTED, "the chunk's keys need K_p*T_p %% B == 0");
    WA_REQUIRE(ceil_div(static_cast<int>(L) + a->Nq, a->B) <= 8192, "at most 8192 key blocks");
  }
  return WA_OK;
}

// key blocks of the sparse branch: the history, then (intra-chunk keys) the chunk's own
int sparse_key_rows(const wa_step_args* a) {
  return a->K_p * a->T_p + (a->k_cur ? a->Nq : 0);
}

StepWs carve_step(Carver& c, const wa_step_args* a) {
  StepWs w{};
  const int cols = a->H * a->d;
  const int L = a->K_p * a->T_p;
  const int n_qb = ceil_div(a->Nq, a->B), n_kb = ceil_div(sparse_key_rows(a), a->B),
            W = ceil_div(n_kb, 32);
  const size_t es = elem_size(a->dtype);
  w.chunk = c.take<int32_t>(1);
  // block sums of the candidate pages, unless the page index holds them
  w.ps = carve_page_score(c, a->Nq, a->H, a->d, a->n_c, a->T_p, a->B, a->page_index == nullptr);
  w.alpha = c.take<double>(a->n_c);
  w.sel = c.take<int32_t>(a->K_p);
  w.sel_pos = c.take<int32_t>(a->K_p);
  w.mask = c.take<uint32_t>(static_cast<size_t>(a->H) * n_qb * W);
  w.k_til = c.take<char>(static_cast<size_t>(a->r) * cols * es);
  w.v_til = c.take<char>(static_cast<size_t>(a->r) * cols * es);
  w.proj = c.take<char>(a->dtype == WA_BF16 ? umma_project_ws_bytes(L, a->H, a->d, a->r) : 0);
  w.lin = c.take<float>(static_cast<size_t>(a->Nq) * cols);
  w.scores = reinterpret_cast<double*>(c.take<char>(block_scores_bytes(a->H, n_qb, n_kb)));
  w.attn = c.take<char>(a->dtype == WA_BF16 ? sparse_attn_ws_bytes(a->H, a->Nq, a->d, a->B) : 0);
  if (!a->fused_gather) {
    w.k_act = c.take<char>(static_cast<size_t>(L) * cols * es);
    w.v_act = c.take<char>(static_cast<size_t>(L) * cols * es);
    // k block sums of the gathered buffer for selection
    w.ksum = c.take<double>(static_cast<size_t>(ceil_div(L, a->B)) * cols);
  }
  if (a->k_cur) w.cur_sum = c.take<double>(static_cast<size_t>(ceil_div(a->Nq, a->B)) * cols);
  return w;
}

}  // namespace
}  // namespace wa_detail
using namespace wa_detail;

size_t wa_hsa_step_workspace_size(const wa_step_args* a) {
  if (!a || validate_step(a) != WA_OK) return 0;
  Carver c(nullptr);
  carve_step(c, a);
  return c.used;
}

wa_status wa_hsa_step(const wa_step_args* a, void* ws, size_t ws_bytes, void* stream) {
  WA_TRY(validate_step(a));
  const size_t need = wa_hsa_step_workspace_size(a);
  WA_TRY(check_ws(ws, ws_bytes, need));
  uint32_t* err = errw();
  if (!err) return set_error(WA_ERR_CUDA, "no CUDA device");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carver c(ws);
  StepWs w = carve_step(c, a);
  auto mark = [&](int k) {
    if (a->stage_events && a->stage_events[k])
      cudaEventRecord(static_cast<cudaEvent_t>(a->stage_events[k]), st);
  };
  mark(0);
  const int cols = a->H * a->d;
  const int L = a->K_p * a->T_p;
  const int n_kb = ceil_div(sparse_key_rows(a), a->B);

  // S0: candidate chunk
  int32_t* chunk = a->chunk_out ? a->chunk_out : w.chunk;
  const int n_chunks = a->e_cur ? a->n_chunks : 1;
  if (a->e_cur)
    WA_TRY(launch_prompt_select(a->e_cur, a->e_chunks, a->n_chunks, a->D, chunk, err, st));
  else if (a->chunk_out)
    cudaMemsetAsync(a->chunk_out, 0, sizeof(int32_t), st);

  // S1: page scores + top-K_p, and the block sums of the candidate pages (S3 reads
  // them in place of a pass over the selected keys); the candidate pages are row
  // `chunk` of chunk_pages (a chunk index of -1 from a zero-norm embedding reads row 0)
  double* alpha = a->alpha_out ? a->alpha_out : w.alpha;
  int32_t* sel = a->sel_out ? a->sel_out : w.sel;
  WA_TRY(run_page_score(w.ps, a->q, a->Nq, a->H, a->d, a->k_pool, a->n_pool_pages, a->T_p,
                        a->chunk_pages, a->e_cur ? chunk : nullptr, n_chunks, a->n_c, a->K_p, a->B,
                        a->dtype, alpha, sel, w.sel_pos, st, a->page_index));

  mark(1);
  // S2: page table (fused) or explicit gather
  RowSource rs;
  KeyMeans km;
  km.L = L;
  km.is_sum = 1;
  if (a->fused_gather) {
    rs.k = a->k_pool; rs.v = a->v_pool; rs.page_ids = sel; rs.page_rows = a->T_p;
    rs.n_pages = a->n_pool_pages; rs.L = L;
    km.nbp = a->T_p / a->B;
    if (a->page_index) {
      km.data = a->page_index;   // indexed by pool page id
      km.page_pos = sel;
    } else {
      km.data = w.ps.k_blocksum; // indexed by candidate position
      km.page_pos = w.sel_pos;
    }
  } else {
    const size_t page_bytes = static_cast<size_t>(a->T_p) * cols * elem_size(a->dtype);
    WA_TRY(launch_gather(a->k_pool, a->v_pool, a->n_pool_pages, page_bytes, sel, a->K_p, w.k_act,
                         w.v_act, err, st));
    rs.k = w.k_act; rs.v = w.v_act; rs.page_rows = L; rs.n_pages = 1; rs.L = L;
    WA_TRY(buffer_block_sums(w.k_act, L, cols, a->B, a->dtype, w.ksum, err, st));
    km.data = w.ksum;
  }
  if (a->k_cur) {
    // intra-chunk keys: the chunk's own K/V follow the history in the sparse branch
    rs.k2 = a->k_cur; rs.v2 = a->v_cur; rs.L2 = a->Nq;
    WA_TRY(buffer_block_sums(a->k_cur, a->Nq, cols, a->B, a->dtype, w.cur_sum, err, st));
    km.data2 = w.cur_sum; km.n_kb1 = L / a->B; km.L2 = a->Nq;
  }

  // inter-chunk granularity: the history's selection blocks pair up B-row block sums
  int n_sel = n_kb;   // selection blocks (= mask blocks unless paired)
  if (a->B_inter == 2 * a->B) {
    km.pair = 1;
    km.n_sub = L / a->B;
    const int n_h = (km.n_sub + 1) / 2;
    n_sel = n_h + (a->k_cur ? ceil_div(a->Nq, a->B) : 0);
    km.n_kb1 = n_h;
  }

  mark(2);
  uint32_t* mask = a->blk_mask_out ? a->blk_mask_out : w.mask;
  void* kt = a->k_til_out ? a->k_til_out : w.k_til;
  void* vt = a->v_til_out ? a->v_til_out : w.v_til;
  RowSource lin;
  lin.k = kt; lin.v = vt; lin.page_rows = a->r; lin.n_pages = 1; lin.L = a->r;
  if (a->dtype == WA_BF16) {
    // S4a + S4b (HBM-bound projection, then the linear branch) on a side stream,
    // concurrently with S3 and the work list (latency-bound) on a high-priority one;
    // the sparse branch, on this stream, joins both.
    SideStream* side = nullptr;
    WA_TRY(side_stream(&side));
    cudaEventRecord(side->fork, st);
    cudaStreamWaitEvent(side->stream, side->fork, 0);
    auto mark_side = [&](int k) {
      if (a->stage_events && a->stage_events[k])
        cudaEventRecord(static_cast<cudaEvent_t>(a->stage_events[k]), side->stream);
    };
    WA_TRY(launch_umma_project(rs.k, rs.v, rs, a->e_k, a->e_v, L, a->H, a->d, a->r, kt, vt, w.proj,
                               err, side->stream, a->e_head_stride != 0));
    mark_side(4);
    WA_TRY(launch_linear_attention(a->q, a->Nq, a->H, a->d, lin, a->B, a->gate, a->gate_lin, w.lin,
                                   nullptr, err, side->stream));
    mark_side(5);
    cudaEventRecord(side->join, side->stream);
    // S3: block selection, then the work list
    cudaStreamWaitEvent(side->hi, side->fork, 0);
    WA_TRY(launch_block_select(w.ps.q_blockmean, a->Nq, a->H, a->d, a->B, km, n_sel, n_kb, a->tau,
                               w.scores, nullptr, nullptr, mask, side->hi));
    if (a->stage_events && a->stage_events[3])
      cudaEventRecord(static_cast<cudaEvent_t>(a->stage_events[3]), side->hi);
    WA_TRY(launch_attn_worklist(a->Nq, a->H, a->d, a->B, sparse_key_rows(a), mask, w.attn, side->hi));
    cudaEventRecord(side->hi_join, side->hi);
    cudaStreamWaitEvent(st, side->hi_join, 0);
    cudaStreamWaitEvent(st, side->join, 0);
    mark(6);
    // S5 + S6
    WA_TRY(launch_attn_sparse(a->q, a->Nq, a->H, a->d, rs, a->B, mask, a->gate, w.lin, a->out, nullptr,
                              w.attn, err, st));
  } else {
    WA_TRY(launch_block_select(w.ps.q_blockmean, a->Nq, a->H, a->d, a->B, km, n_sel, n_kb, a->tau,
                               w.scores, nullptr, nullptr, mask, st));
    mark(3);
    WA_TRY(launch_simt_project(static_cast<const float*>(rs.k), rs.page_ids, rs.page_rows,
                               rs.n_pages, static_cast<const float*>(a->e_k), L, cols, a->r, a->d,
                               a->e_head_stride, static_cast<float*>(kt), err, st));
    WA_TRY(launch_simt_project(static_cast<const float*>(rs.v), rs.page_ids, rs.page_rows,
                               rs.n_pages, static_cast<const float*>(a->e_v), L, cols, a->r, a->d,
                               a->e_head_stride, static_cast<float*>(vt), err, st));
    mark(4);
    WA_TRY(run_attention(a->q, a->Nq, a->H, a->d, rs, a->B, mask, kt, vt, a->r, a->gate, a->gate_lin,
                         a->dtype, a->out, nullptr, nullptr, w.lin, w.attn, st, a->stage_events));
  }
  mark(7);
  return WA_OK;
}

}  // extern "C"
