// k_blocksum.cu -- the HBM pass of page retrieval and the block pooling:
//   float64 sums of every B-row block of the queries and of the candidate pages
//   (WorldAttention §3.2 "Stage 2: page-level retrieval": Qbar and Kbar_j are means
//   over the chunk's queries and over a page's keys; §3.3 / summary step 5: block
//   pooling is the mean over a block's rows, so the same block sums serve both),
// and the page scores alpha_j = (1/H) sum_h Qbar_h . Kbar_{h,j} / sqrt(d) with the
// top-K_p pages, formed from those sums.
//
// The pass streams every block once.  Each CTA is persistent (three per SM) and walks
// a fixed list of blocks; one producer thread copies each block, a few rows at a
// time, into a ring of shared-memory stages with cp.async.bulk (the rows of a block
// are contiguous in memory, so one bulk copy moves whole rows), and the consumer
// threads reduce the staged rows: thread t owns 16 bytes of every row (8 bf16 or 4
// float columns) and adds its rows in order in float64, so every sum is
// deterministic (for inputs whose values span fewer than about 2^40 in magnitude the
// float64 sum of 64 rows is exact anyway).  No barrier spans the consumers: each
// consumer warp releases a stage on its own, and every wait is bounded.
#include <cuda_bf16.h>

#include <cfloat>
#include <climits>
#include <cmath>

#include "sm100.cuh"
#include "wa_internal.h"

namespace wa {
namespace {

using namespace sm100;

constexpr int kMaxSegs = 2;
constexpr int kMaxStages = 16;
// Three CTAs per SM, each with a ring of three 24 KB stages at the one-layer shape
// (a sweep over 2-6 CTAs per SM, 32-96 KB rings and 6-48 KB copies put this setting
// first, at 4.9 TB/s on the 307 MB pass of eight candidate pages).
constexpr int kRingBytes = 72 * 1024;     // shared-memory ring of one CTA
constexpr int kCtasPerSm = 3;
constexpr int kChunkBytesMax = 24 * 1024; // rows per bulk copy: at most this many bytes

struct PassSeg {
  const char* x;            // rows of row_bytes bytes
  const int32_t* ids;       // nullable: source s is pool page ids[s] (or ids[*chunk * n_src + s])
  const int32_t* chunk;     // nullable: row of ids (candidate chunk chosen on the device)
  int id_rows;              // rows of ids (a chunk index outside [0, id_rows) reads row 0)
  int n_src;                // sources
  int n_pages;              // pages addressable through ids
  int rows;                 // rows per source
  int block0;               // first block of every source
  int n_blocks;             // blocks per source
  double* sums;             // [(by_page ? page : s) * nb_out + block][cols]
  int nb_out;
  int by_page;
  int units;                // n_src * n_blocks
};

struct PassArgs {
  PassSeg seg[kMaxSegs];
  int n_segs;
  int total_units;
  int cols;                 // elements per row
  int row_bytes;
  int B;                    // rows per block
  int R;                    // rows per bulk copy (a power of two dividing B, or B)
  int S;                    // ring stages
  int G;                    // 16-byte groups per row = consumer threads
  unsigned* counter;        // nullable: n_counters words zeroed here for the page-score kernel
  int n_counters;
  uint64_t wait_ns;
};

struct PassShared {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  int abort_flag;
};

// unit -> (segment, source position, block)
__device__ __forceinline__ void unit_of(const PassArgs& a, int u, int& sg, int& s, int& b) {
  sg = 0;
  if (a.n_segs > 1 && u >= a.seg[0].units) { u -= a.seg[0].units; sg = 1; }
  const PassSeg& g = a.seg[sg];
  s = u / g.n_blocks;
  b = g.block0 + u % g.n_blocks;
}

__device__ __forceinline__ int page_of(const PassSeg& g, int s, uint32_t* err, bool& ok) {
  ok = true;
  if (!g.ids) return s;
  int row = g.chunk ? *g.chunk : 0;
  if (row < 0 || row >= g.id_rows) row = 0;
  int p = g.ids[static_cast<size_t>(row) * g.n_src + s];
  if (p < 0 || p >= g.n_pages) { ok = false; p = 0; }
  return p;
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ double bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ double bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <typename T>
__device__ __forceinline__ void add16(const uint4& r, double (&acc)[16 / sizeof(T)]);
template <>
__device__ __forceinline__ void add16<__nv_bfloat16>(const uint4& r, double (&acc)[8]) {
  acc[0] += bf_lo(r.x); acc[1] += bf_hi(r.x); acc[2] += bf_lo(r.y); acc[3] += bf_hi(r.y);
  acc[4] += bf_lo(r.z); acc[5] += bf_hi(r.z); acc[6] += bf_lo(r.w); acc[7] += bf_hi(r.w);
}
template <>
__device__ __forceinline__ void add16<float>(const uint4& r, double (&acc)[4]) {
  acc[0] += static_cast<double>(__uint_as_float(r.x)); acc[1] += static_cast<double>(__uint_as_float(r.y));
  acc[2] += static_cast<double>(__uint_as_float(r.z)); acc[3] += static_cast<double>(__uint_as_float(r.w));
}

// Thread layout: warp 0 is the producer (lane 0 issues the copies); the consumer
// warps follow, thread 32 + g owning 16-byte group g of every row (lanes past G idle
// but take part in the warp-level stage release).
template <typename T>
__global__ void __launch_bounds__(1024)
k_block_sums(const __grid_constant__ PassArgs a, uint32_t* err) {
  constexpr int V = 16 / sizeof(T);
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ PassShared sh;
  const int chunk_bytes = a.R * a.row_bytes;
  uint8_t* ring = smem_raw;                                              // [S][chunk_bytes]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_cons_warps = (a.G + 31) >> 5;
  if (tid == 0) {
    for (int s = 0; s < a.S; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], n_cons_warps);
    }
    sh.abort_flag = 0;
    fence_mbar_init();
    if (a.counter && blockIdx.x == 0)
      for (int i = 0; i < a.n_counters; ++i) a.counter[i] = 0u;
  }
  __syncthreads();

  int issued = 0;   // producer: chunks whose copies were issued (for the abort drain)
  if (warp == 0) {
    if (lane == 0) {
      int k = 0;    // running chunk index of this CTA
      bool go = true;
      for (int u = blockIdx.x; u < a.total_units && go; u += gridDim.x) {
        int sg, s, b;
        unit_of(a, u, sg, s, b);
        const PassSeg& g = a.seg[sg];
        bool ok;
        const int page = page_of(g, s, err, ok);
        if (!ok) atomicOr(err, WA_DEVERR_PAGE_ID);
        const int r0 = b * a.B, r1 = min(g.rows, r0 + a.B);
        const char* base = g.x + (static_cast<size_t>(page) * g.rows + r0) * a.row_bytes;
        for (int r = r0; r < r1; r += a.R, ++k) {
          const int st = k % a.S;
          const int w = mbar_wait_bounded(&sh.empty[st], ((k / a.S) & 1) ^ 1, &sh.abort_flag, a.wait_ns);
          if (w != kWaitOk) {
            if (w == kWaitTimeout) atomicOr(err, WA_DEVERR_TIMEOUT);
            go = false;
            break;
          }
          const uint32_t bytes = static_cast<uint32_t>(min(a.R, r1 - r) * a.row_bytes);
          mbar_arrive_expect_tx(&sh.full[st], bytes);
          bulk_g2s(ring + static_cast<size_t>(st) * chunk_bytes,
                   base + static_cast<size_t>(r - r0) * a.row_bytes, bytes, &sh.full[st]);
          issued = k + 1;
        }
      }
    }
  } else if (warp <= n_cons_warps) {
    const int grp = tid - 32;
    const bool active = grp < a.G;
    int k = 0;
    bool alive = true;
    for (int u = blockIdx.x; u < a.total_units && alive; u += gridDim.x) {
      int sg, s, b;
      unit_of(a, u, sg, s, b);
      const PassSeg& g = a.seg[sg];
      const int r0 = b * a.B, r1 = min(g.rows, r0 + a.B);
      double acc[V];
#pragma unroll
      for (int v = 0; v < V; ++v) acc[v] = 0.0;
      for (int r = r0; r < r1; r += a.R, ++k) {
        const int st = k % a.S;
        // every lane waits, so the warp's decision to go on is uniform
        const bool got = __all_sync(0xffffffffu, mbar_wait_bounded(&sh.full[st], (k / a.S) & 1,
                                                                   &sh.abort_flag, a.wait_ns) == kWaitOk);
        if (!got) {
          alive = false;
          break;
        }
        if (active) {
          const int nr = min(a.R, r1 - r);
          const uint8_t* src = ring + static_cast<size_t>(st) * chunk_bytes + grp * 16;
#pragma unroll 4
          for (int rr = 0; rr < nr; ++rr) {
            const uint4 w = *reinterpret_cast<const uint4*>(src + static_cast<size_t>(rr) * a.row_bytes);
            add16<T>(w, acc);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[st]);
      }
      if (!alive) break;
      if (active) {
        bool ok = true;
        const int page = page_of(g, s, err, ok);
        if (ok || !g.by_page) {
          double* out = g.sums +
                        (static_cast<size_t>(g.by_page ? page : s) * g.nb_out + b) * a.cols + grp * V;
#pragma unroll
          for (int v = 0; v < V; ++v) out[v] = acc[v];
        }
      }
    }
  }
  __syncthreads();
  if (sh.abort_flag && warp == 0 && lane == 0) {
    // a wait gave up: wait (bounded) for the copies this CTA still has in flight
    int never = 0;
    for (int k = issued > a.S ? issued - a.S : 0; k < issued; ++k)
      if (mbar_wait_bounded(&sh.full[k % a.S], (k / a.S) & 1, &never, a.wait_ns) == kWaitTimeout)
        atomicOr(err, WA_DEVERR_TIMEOUT);
  }
}

// ------------------------------------------------------------------ page scores
// One CTA per slice of kAlphaCols columns; thread (tx, gy) takes column tx of the
// slice and the rows gy, gy + kAlphaGroups, ... of each sum it forms:
//   Qbar for the slice (the query block sums added / Nq; also written out, with the
//   query block means), then, kAlphaPages pages at a time, every candidate page's
//   column sum over its block sums (page kpage[row][j], or position j), each combined
//   over the row groups in order and dotted with Qbar over the slice -> partial[j][cs].
// The last CTA to finish adds the slices in order, forms
//   alpha_j = Qbar . colsum_j / (T_p sqrt(d) H)
// and takes the top-K_p pages (ties -> lower position), emitted in ascending position.
constexpr int kAlphaCols = 16;
constexpr int kAlphaThreads = 512;
constexpr int kAlphaGroups = kAlphaThreads / kAlphaCols;   // row groups
constexpr int kAlphaPages = 8;                             // pages whose loads are in flight together
constexpr int kAlphaBatch = 4;                             // blocks per page per thread per batch

__global__ void __launch_bounds__(kAlphaThreads)
k_page_alpha(const double* __restrict__ qsum, int n_qb, int Nq, int B, int cols,
             const double* __restrict__ ksum, const int32_t* __restrict__ kpage, int n_pages,
             int nbp, const int32_t* __restrict__ cand, const int32_t* __restrict__ chunk,
             int n_chunks, int n_c, int T_p, int H, int d, int K_p, double* __restrict__ qbar,
             double* __restrict__ qmean, double* __restrict__ partial, unsigned* counter,
             double* __restrict__ alpha, int32_t* __restrict__ sel, int32_t* __restrict__ sel_pos,
             uint32_t* err) {
  extern __shared__ double red[];            // [kAlphaPages][kAlphaGroups][kAlphaCols]
  __shared__ double qb[kAlphaCols];
  __shared__ bool last;
  const int cs = blockIdx.x, n_cs = gridDim.x;
  const int tx = threadIdx.x % kAlphaCols, gy = threadIdx.x / kAlphaCols;
  const int col = cs * kAlphaCols + tx;
  const bool cv = col < cols;
  const int lanei = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int row = chunk ? *chunk : 0;
  if (row < 0 || row >= n_chunks) row = 0;
  // Qbar of the slice
  {
    double t = 0.0;
    if (cv)
      for (int i = gy; i < n_qb; i += kAlphaGroups) {
        const double v = qsum[static_cast<size_t>(i) * cols + col];
        t += v;
        if (qmean) qmean[static_cast<size_t>(i) * cols + col] = v / (min(Nq, (i + 1) * B) - i * B);
      }
    red[gy * kAlphaCols + tx] = t;
    __syncthreads();
    if (gy == 0) {
      double s = 0.0;
      for (int g = 0; g < kAlphaGroups; ++g) s += red[g * kAlphaCols + tx];
      s /= Nq;
      qb[tx] = cv ? s : 0.0;
      if (cv) qbar[col] = s;
    }
    __syncthreads();
  }
  // the pages' column sums, kAlphaPages at a time; each thread issues the loads of
  // kAlphaBatch of its blocks for every page of the group before adding them (in
  // block order)
  for (int j0 = 0; j0 < n_c; j0 += kAlphaPages) {
    const double* kp[kAlphaPages];
#pragma unroll
    for (int jj = 0; jj < kAlphaPages; ++jj) {
      const int j = j0 + jj;
      int page = j < n_c ? j : 0;
      if (kpage && j < n_c) {
        page = kpage[static_cast<size_t>(row) * n_c + j];
        if (page < 0 || page >= n_pages) {
          if (threadIdx.x == 0 && cs == 0) atomicOr(err, WA_DEVERR_PAGE_ID);
          page = 0;
        }
      }
      kp[jj] = (j < n_c && cv) ? ksum + static_cast<size_t>(page) * nbp * cols + col : nullptr;
    }
    double acc[kAlphaPages];
#pragma unroll
    for (int jj = 0; jj < kAlphaPages; ++jj) acc[jj] = 0.0;
    for (int b0 = gy; b0 < nbp; b0 += kAlphaBatch * kAlphaGroups) {
      double v[kAlphaPages][kAlphaBatch];
#pragma unroll
      for (int jj = 0; jj < kAlphaPages; ++jj)
#pragma unroll
        for (int e = 0; e < kAlphaBatch; ++e) {
          const int b = b0 + e * kAlphaGroups;
          v[jj][e] = (kp[jj] && b < nbp) ? kp[jj][static_cast<size_t>(b) * cols] : 0.0;
        }
#pragma unroll
      for (int jj = 0; jj < kAlphaPages; ++jj)
#pragma unroll
        for (int e = 0; e < kAlphaBatch; ++e) acc[jj] += v[jj][e];
    }
#pragma unroll
    for (int jj = 0; jj < kAlphaPages; ++jj) red[(jj * kAlphaGroups + gy) * kAlphaCols + tx] = acc[jj];
    __syncthreads();
    // warp jj: page j0 + jj; lanes 0-15 combine the row groups of one column each
    if (warp < kAlphaPages && j0 + warp < n_c) {
      double dot = 0.0;
      if (lanei < kAlphaCols) {
        double c = 0.0;
        for (int g = 0; g < kAlphaGroups; ++g) c += red[(warp * kAlphaGroups + g) * kAlphaCols + lanei];
        dot = c * qb[lanei];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      if (lanei == 0) partial[static_cast<size_t>(j0 + warp) * n_cs + cs] = dot;
    }
    __syncthreads();
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(counter, 1u) == static_cast<unsigned>(n_cs) - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  // the last CTA: alpha for every page, then the top-K_p
  const double den = static_cast<double>(T_p) * sqrt(static_cast<double>(d)) * H;
  for (int c = warp; c < n_c; c += nw) {
    // lane l adds slices l, l + 32, ... in order, then a fixed butterfly
    const double* pr = partial + static_cast<size_t>(c) * n_cs;
    double s = 0.0;
    for (int k = lanei; k < n_cs; k += 32) s += __ldcg(pr + k);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lanei == 0) alpha[c] = s / den;
  }
  unsigned char* chosen = reinterpret_cast<unsigned char*>(red);   // [n_c], reuses the reduction buffer
  __syncthreads();
  for (int c = threadIdx.x; c < n_c; c += blockDim.x) chosen[c] = 0;
  __syncthreads();
  if (warp != 0) return;
  // top-K_p by repeated arg-max over the pages not yet taken (ties -> lower position)
  for (int k = 0; k < K_p; ++k) {
    double best = -DBL_MAX;
    int bi = INT_MAX;
    for (int c = lanei; c < n_c; c += 32) {
      if (chosen[c]) continue;
      const double v = const_cast<const volatile double*>(alpha)[c];
      if (bi == INT_MAX || v > best) { best = v; bi = c; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (oi != INT_MAX && (bi == INT_MAX || ob > best || (ob == best && oi < bi))) { best = ob; bi = oi; }
    }
    if (lanei == 0 && bi != INT_MAX) chosen[bi] = 1;
    __syncwarp();
  }
  if (lanei == 0) {
    // the chosen pages in ascending candidate position, as pool ids
    int k = 0;
    for (int c = 0; c < n_c && k < K_p; ++c)
      if (chosen[c]) {
        sel[k] = cand ? cand[static_cast<size_t>(row) * n_c + c] : c;
        if (sel_pos) sel_pos[k] = c;
        ++k;
      }
    *counter = 0u;
  }
}

constexpr size_t kAlphaSmem = static_cast<size_t>(kAlphaPages) * kAlphaGroups * kAlphaCols * sizeof(double);

int g_n_sm = 0;
int n_sm() {
  if (g_n_sm == 0) {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 148;
    g_n_sm = n;
  }
  return g_n_sm;
}

}  // namespace

wa_status launch_block_sums(wa_dtype dt, int cols, int B, const BlockSumSeg* segs, int n_segs,
                            unsigned* counter, int n_counters, uint32_t* err, cudaStream_t st) {
  if (n_segs < 1 || n_segs > kMaxSegs) return set_error(WA_ERR_INVALID_ARG, "block sums: 1 or 2 segments");
  PassArgs a{};
  const int es = dt == WA_BF16 ? 2 : 4;
  a.cols = cols;
  a.row_bytes = cols * es;
  if (a.row_bytes % 16 != 0) return set_error(WA_ERR_UNSUPPORTED, "block sums need rows of 16-byte multiples");
  a.B = B;
  a.n_segs = n_segs;
  a.counter = counter;
  a.n_counters = n_counters;
  a.wait_ns = wait_limit_ns();
  long long total = 0;
  for (int i = 0; i < n_segs; ++i) {
    const BlockSumSeg& s = segs[i];
    PassSeg& g = a.seg[i];
    g.x = static_cast<const char*>(s.x);
    g.ids = s.ids; g.chunk = s.chunk; g.id_rows = s.id_rows < 1 ? 1 : s.id_rows; g.n_src = s.n_src; g.n_pages = s.n_pages; g.rows = s.rows;
    g.block0 = s.block0; g.n_blocks = s.n_blocks; g.sums = s.sums; g.nb_out = s.nb_out;
    g.by_page = s.by_page;
    if (reinterpret_cast<uintptr_t>(s.x) % 16 != 0)
      return set_error(WA_ERR_UNSUPPORTED, "block sums need 16-byte aligned inputs");
    const long long u = static_cast<long long>(s.n_src) * s.n_blocks;
    if (u < 0 || u > INT_MAX) return set_error(WA_ERR_INVALID_ARG, "block sums: too many blocks");
    g.units = static_cast<int>(u);
    total += u;
  }
  if (total > INT_MAX) return set_error(WA_ERR_INVALID_ARG, "block sums: too many blocks");
  a.total_units = static_cast<int>(total);
  if (a.total_units == 0) return WA_OK;
  // rows per bulk copy: a power of two dividing B, at most kChunkBytesMax bytes
  int R = 1;
  while (R * 2 <= B && B % (R * 2) == 0 && (R * 2) * a.row_bytes <= kChunkBytesMax) R *= 2;
  a.R = R;
  const int chunk_bytes = R * a.row_bytes;
  a.G = a.row_bytes / 16;
  if (a.G > 992) return set_error(WA_ERR_UNSUPPORTED, "block sums: rows longer than 15872 bytes");
  int S = static_cast<int>(kRingBytes / chunk_bytes);
  if (S > kMaxStages) S = kMaxStages;
  if (S < 2) S = 2;
  a.S = S;
  const size_t smem = static_cast<size_t>(S) * chunk_bytes;
  const int threads = 32 + ((a.G + 31) / 32) * 32;
  const int max_grid = kCtasPerSm * n_sm();
  const int grid = a.total_units < max_grid ? a.total_units : max_grid;
  cudaError_t e;
  if (dt == WA_BF16) {
    e = cudaFuncSetAttribute(k_block_sums<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e == cudaSuccess)
      k_block_sums<__nv_bfloat16><<<grid, threads, smem, st>>>(a, err);
  } else {
    e = cudaFuncSetAttribute(k_block_sums<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e == cudaSuccess) k_block_sums<float><<<grid, threads, smem, st>>>(a, err);
  }
  if (e != cudaSuccess) return set_error(WA_ERR_CUDA, "block sums smem attr: %s", cudaGetErrorString(e));
  return check_launch("block_sums");
}

size_t page_alpha_scratch_doubles(int cols, int n_c) {
  const size_t n_cs = (cols + kAlphaCols - 1) / kAlphaCols;
  return static_cast<size_t>(n_c) * n_cs;   // slice dots [n_c][n_cs]
}

int page_alpha_counters(int) { return 1; }

wa_status launch_page_alpha(const double* qsum, int n_qb, int Nq, int B, int cols, const double* ksum,
                            const int32_t* kpage, int n_pages, int nbp, const int32_t* cand,
                            const int32_t* chunk, int n_chunks, int n_c, int T_p, int H, int d,
                            int K_p, double* qbar, double* qmean, double* scratch, unsigned* counters,
                            double* alpha, int32_t* sel, int32_t* sel_pos, uint32_t* err,
                            cudaStream_t st) {
  if (static_cast<size_t>(n_c) > kAlphaSmem)
    return set_error(WA_ERR_UNSUPPORTED, "page scores: too many candidate pages");
  const int n_cs = (cols + kAlphaCols - 1) / kAlphaCols;
  cudaError_t e = cudaFuncSetAttribute(k_page_alpha, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kAlphaSmem));
  if (e != cudaSuccess) return set_error(WA_ERR_CUDA, "page scores smem attr: %s", cudaGetErrorString(e));
  k_page_alpha<<<n_cs, kAlphaThreads, kAlphaSmem, st>>>(
      qsum, n_qb, Nq, B, cols, ksum, kpage, n_pages, nbp, cand, chunk, n_chunks, n_c, T_p, H, d, K_p,
      qbar, qmean, scratch, counters, alpha, sel, sel_pos, err);
  return check_launch("page_alpha");
}

}  // namespace wa
