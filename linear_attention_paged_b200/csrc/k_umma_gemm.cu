// k_umma_gemm.cu -- the Linformer projection of the linear branch on tcgen05
// tensor cores (WorldAttention §3.3 "Linear branch": K~ = E_K^T K, V~ = E_V^T V,
// E shared by the heads):
//     C[c][n] = sum_l E[l][c] * X[l][n]      c < r, n < H*d, l < L
// As stored, both operands have the reduction index l as their outer (strided)
// dimension, so A = E^T and B = X are read MN-major straight from the TMA tiles.
// L (49,920 at the bench shape) is split across CTAs; each CTA accumulates an
// r x TN tile in TMEM (two M=128 accumulators when r = 256) and writes an fp32
// partial; a second kernel sums the partials in a fixed order and rounds to bf16,
// so the result is deterministic.  K/V rows can be read through the page table,
// which removes the K_active / V_active copy.
#include <cuda.h>
#include <cuda_bf16.h>

#include <mutex>

#include "sm100.cuh"
#include "wa_internal.h"

namespace wa {

bool make_tmap_bf16_2d(void* tmap, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer);

namespace {

using namespace sm100;

constexpr int kThreads = 256;
constexpr int kKB = 64;  // rows of L per stage

template <int NSUB, int TN>
struct GCfg {
  static constexpr int kR = NSUB * 128;
  static constexpr int kABytes = kKB * kR * 2;    // r/64 panels of 64 x 128 B
  static constexpr int kBBytes = kKB * TN * 2;    // TN/64 panels
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (200 * 1024) / kStageBytes > 6 ? 6 : (200 * 1024) / kStageBytes;
  static constexpr int kSmem = kStages * kStageBytes + 1024;
  static constexpr uint32_t kCols = NSUB * TN;
  static constexpr uint32_t kTmem = kCols <= 32 ? 32 : kCols <= 64 ? 64 : kCols <= 128 ? 128
                                    : kCols <= 256 ? 256 : 512;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(128, TN, true, true);
};

struct GShared {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full;
  uint64_t drain;        // abort path: every MMA of the issuer complete
  uint64_t wait_ns;      // bound of every wait (wa_set_wait_limit_ns)
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ bool gwait(uint64_t* bar, uint32_t parity, GShared& sh, uint32_t* err) {
  const int r = mbar_wait_bounded(bar, parity, &sh.abort_flag, sh.wait_ns);
  if (r == kWaitTimeout) atomicOr(err, WA_DEVERR_TIMEOUT);
  return r == kWaitOk;
}

template <int NSUB, int TN>
__global__ void __launch_bounds__(kThreads, 1)
k_umma_project(const __grid_constant__ CUtensorMap tmEK, const __grid_constant__ CUtensorMap tmEV,
               const __grid_constant__ CUtensorMap tmXK, const __grid_constant__ CUtensorMap tmXV,
               RowSource rs, int L, int cols, int n_split, float* __restrict__ part,
               uint32_t* err, uint64_t wait_ns, int d, int e_head_rows) {
  using C = GCfg<NSUB, TN>;
  extern __shared__ uint8_t smem_dyn[];
  __shared__ GShared sh;
  uint8_t* tiles = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_nt = cols / TN;
  const int m = blockIdx.x / n_nt;     // 0: K, 1: V
  const int nt = blockIdx.x % n_nt;
  const int sp = blockIdx.y;
  const int n_kb = (L + kKB - 1) / kKB;
  const int per = (n_kb + n_split - 1) / n_split;
  const int kb0 = sp * per, kb1 = min(n_kb, kb0 + per);
  const int nk = kb1 > kb0 ? kb1 - kb0 : 0;
  const CUtensorMap* tE = m ? &tmEV : &tmEK;
  const CUtensorMap* tX = m ? &tmXV : &tmXK;
  // one E per head (e_head_rows = L): a tile lies within one head (TN <= d), whose E
  // rows start at head * L of the [H*L][r] view
  const int e_row0 = e_head_rows ? (nt * TN / d) * e_head_rows : 0;

  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) { mbar_init(&sh.full[s], 1); mbar_init(&sh.empty[s], 1); }
    mbar_init(&sh.acc_full, 1);
    mbar_init(&sh.drain, 1);
    sh.wait_ns = wait_ns;
    sh.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, C::kTmem);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sh.tmem_base;
  int issued = 0;   // producer: stages whose loads were issued (for the abort drain)

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(tE);
      prefetch_tmap(tX);
      for (int t = 0; t < nk; ++t) {
        const int s = t % C::kStages;
        if (!gwait(&sh.empty[s], ((t / C::kStages) & 1) ^ 1, sh, err)) break;
        const int l0 = (kb0 + t) * kKB;
        int row = l0;
        if (rs.page_ids) {
          int pg = rs.page_ids[l0 / rs.page_rows];
          if (pg < 0 || pg >= rs.n_pages) { atomicOr(err, WA_DEVERR_PAGE_ID); pg = 0; }
          row = pg * rs.page_rows + l0 % rs.page_rows;
        }
        uint8_t* As = tiles + s * C::kStageBytes;
        uint8_t* Bs = As + C::kABytes;
        mbar_arrive_expect_tx(&sh.full[s], C::kStageBytes);
        for (int p = 0; p < C::kR / 64; ++p) tma_load_2d(As + p * 8192, tE, &sh.full[s], p * 64, e_row0 + l0);
        for (int p = 0; p < TN / 64; ++p)
          tma_load_2d(Bs + p * 8192, tX, &sh.full[s], nt * TN + p * 64, row);
        issued = t + 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = true;
      for (int t = 0; t < nk; ++t) {
        const int s = t % C::kStages;
        if (!gwait(&sh.full[s], (t / C::kStages) & 1, sh, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_base = smem_u32(tiles + s * C::kStageBytes);
        const uint32_t b_base = a_base + C::kABytes;
#pragma unroll
        for (int ks = 0; ks < kKB / 16; ++ks) {
          const uint64_t bdesc = smem_desc_sw128(b_base + ks * 2048, 8192, 1024);
#pragma unroll
          for (int sub = 0; sub < NSUB; ++sub) {
            const uint64_t adesc = smem_desc_sw128(a_base + sub * 2 * 8192 + ks * 2048, 8192, 1024);
            mma_ss(tbase + sub * TN, adesc, bdesc, C::kIdesc, (t > 0 || ks > 0) ? 1u : 0u);
          }
        }
        mma_commit(&sh.empty[s]);
      }
      if (ok) mma_commit(&sh.acc_full);
    }
  } else if (warp >= 4) {
    const int q4 = warp - 4;
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    bool ok = true;
    if (nk > 0) ok = __all_sync(0xffffffffu, gwait(&sh.acc_full, 0, sh, err));
    tc_fence_after();
    for (int sub = 0; sub < NSUB; ++sub) {
      const int row = sub * 128 + q4 * 32 + lane;  // c index of the output
      float* dst = part + ((static_cast<size_t>(m) * n_split + sp) * C::kR + row) * cols + nt * TN;
#pragma unroll 1
      for (int c0 = 0; c0 < TN; c0 += 32) {
        uint32_t v[32];
        if (nk > 0 && ok) {
          tmem_ld32(tbase + lane_base + sub * TN + c0, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
        float4* d4 = reinterpret_cast<float4*>(dst + c0);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          d4[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                              __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (sh.abort_flag) {
    // A role gave up: wait (bounded, whatever the flag says) for the loads the
    // producer issued (at most the last kStages can be outstanding) and for every
    // MMA of the issuer, before TMEM is freed and the shared memory reused.
    int never = 0;
    if (warp == 0 && lane == 0) {
      for (int t = issued > C::kStages ? issued - C::kStages : 0; t < issued; ++t)
        if (mbar_wait_bounded(&sh.full[t % C::kStages], (t / C::kStages) & 1, &never, sh.wait_ns) ==
            kWaitTimeout)
          atomicOr(err, WA_DEVERR_TIMEOUT);
    } else if (warp == 1 && lane == 0) {
      mma_commit(&sh.drain);
      if (mbar_wait_bounded(&sh.drain, 0, &never, sh.wait_ns) == kWaitTimeout)
        atomicOr(err, WA_DEVERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::kTmem);
  }
}

// out_m[c][n] = bf16( sum_{split} part[m][split][c][n] ), splits summed in order.
// One float4 per thread; the split loads are issued kBatch at a time (independent,
// so they overlap) and added in split order.
constexpr int kReduceThreads = 256;
__global__ void __launch_bounds__(kReduceThreads)
k_reduce_splits(const float* __restrict__ part, int n_split, size_t per_m,
                __nv_bfloat16* __restrict__ out_k, __nv_bfloat16* __restrict__ out_v) {
  constexpr int kBatch = 8;
  const size_t n4 = per_m / 4;
  const size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (i >= 2 * n4) return;
  const int m = i >= n4;
  const size_t e = (i - m * n4) * 4;
  const float* src = part + static_cast<size_t>(m) * n_split * per_m + e;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < n_split; s0 += kBatch) {
    float4 v[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b)
      if (s0 + b < n_split) v[b] = __ldcs(reinterpret_cast<const float4*>(src + (s0 + b) * per_m));
#pragma unroll
    for (int b = 0; b < kBatch; ++b)
      if (s0 + b < n_split) { acc.x += v[b].x; acc.y += v[b].y; acc.z += v[b].z; acc.w += v[b].w; }
  }
  __nv_bfloat16* o = (m ? out_v : out_k) + e;
  *reinterpret_cast<uint2*>(o) = make_uint2(sm100::pack_bf16x2(acc.x, acc.y), sm100::pack_bf16x2(acc.z, acc.w));
}

// one thread per float4 of the two outputs
unsigned reduce_grid(size_t per_m) {
  return static_cast<unsigned>((2 * (per_m / 4) + kReduceThreads - 1) / kReduceThreads);
}

int pick_tn(int cols) {
  if (cols % 256 == 0) return 256;
  if (cols % 128 == 0) return 128;
  if (cols % 64 == 0) return 64;
  return 0;
}

// with one E per head a tile must lie within one head: width d at most
int pick_tn_for(int cols, int d, bool e_per_head) {
  const int tn = pick_tn(cols);
  return (e_per_head && tn > d) ? d : tn;
}

int pick_splits(int L, int r, int cols, int tn_override = 0) {
  const int tn = tn_override ? tn_override : pick_tn(cols);
  const int tiles = 2 * (cols / tn);
  const int n_kb = (L + kKB - 1) / kKB;
  int s = 148 / tiles;
  if (s < 1) s = 1;
  if (s > n_kb) s = n_kb;
  (void)r;
  return s;
}

template <int NSUB, int TN>
void launch_proj(dim3 grid, cudaStream_t st, const CUtensorMap& a, const CUtensorMap& b,
                 const CUtensorMap& c, const CUtensorMap& d, RowSource rs, int L, int cols,
                 int n_split, float* part, uint32_t* err, int dh = 128, int e_head_rows = 0) {
  using C = GCfg<NSUB, TN>;
  cudaFuncSetAttribute(k_umma_project<NSUB, TN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  k_umma_project<NSUB, TN><<<grid, kThreads, C::kSmem, st>>>(a, b, c, d, rs, L, cols, n_split,
                                                             part, err, wait_limit_ns(), dh,
                                                             e_head_rows);
}

}  // namespace

size_t umma_project_ws_bytes(int L, int H, int d, int r, bool e_per_head) {
  const int cols = H * d;
  const int tn = pick_tn_for(cols, d, e_per_head);
  if (tn == 0) return 0;
  return 2ull * pick_splits(L, r, cols, tn) * r * cols * sizeof(float);
}

wa_status launch_umma_project(const void* k, const void* v, RowSource rs, const void* e_k,
                              const void* e_v, int L, int H, int d, int r, void* k_til,
                              void* v_til, void* ws, uint32_t* err, cudaStream_t st,
                              bool e_per_head) {
  const int cols = H * d;
  const int tn = pick_tn_for(cols, d, e_per_head);
  if (tn == 0) return set_error(WA_ERR_UNSUPPORTED, "projection needs H*d %% 64 == 0");
  if (r != 128 && r != 256) return set_error(WA_ERR_UNSUPPORTED, "bf16 projection needs r in {128, 256}");
  if (rs.page_ids && rs.page_rows % kKB != 0)
    return set_error(WA_ERR_UNSUPPORTED, "paged projection needs T_p %% 64 == 0");
  const int n_split = pick_splits(L, r, cols, tn);
  const uint64_t rows = rs.page_ids ? static_cast<uint64_t>(rs.n_pages) * rs.page_rows
                                    : static_cast<uint64_t>(L);
  // E as a 2-D [rows][r] tensor: L rows, or H * L rows when there is one E per head
  const uint64_t e_rows = e_per_head ? static_cast<uint64_t>(H) * L : static_cast<uint64_t>(L);
  const int e_head_rows = e_per_head ? L : 0;
  alignas(64) CUtensorMap tek, tev, txk, txv;
  if (!make_tmap_bf16_2d(&tek, e_k, r, e_rows, static_cast<uint64_t>(r) * 2, 64, 64) ||
      !make_tmap_bf16_2d(&tev, e_v, r, e_rows, static_cast<uint64_t>(r) * 2, 64, 64) ||
      !make_tmap_bf16_2d(&txk, k, cols, rows, static_cast<uint64_t>(cols) * 2, 64, 64) ||
      !make_tmap_bf16_2d(&txv, v, cols, rows, static_cast<uint64_t>(cols) * 2, 64, 64))
    return set_error(WA_ERR_CUDA, "cuTensorMapEncodeTiled failed for the projection operands");
  float* part = static_cast<float*>(ws);
  dim3 grid(2 * (cols / tn), n_split);
  const int nsub = r / 128;
  if (nsub == 2) {
    if (tn == 256) launch_proj<2, 256>(grid, st, tek, tev, txk, txv, rs, L, cols, n_split, part, err, d, e_head_rows);
    else if (tn == 128) launch_proj<2, 128>(grid, st, tek, tev, txk, txv, rs, L, cols, n_split, part, err, d, e_head_rows);
    else launch_proj<2, 64>(grid, st, tek, tev, txk, txv, rs, L, cols, n_split, part, err, d, e_head_rows);
  } else {
    if (tn == 256) launch_proj<1, 256>(grid, st, tek, tev, txk, txv, rs, L, cols, n_split, part, err, d, e_head_rows);
    else if (tn == 128) launch_proj<1, 128>(grid, st, tek, tev, txk, txv, rs, L, cols, n_split, part, err, d, e_head_rows);
    else launch_proj<1, 64>(grid, st, tek, tev, txk, txv, rs, L, cols, n_split, part, err, d, e_head_rows);
  }
  wa_status s = check_launch("umma_project");
  if (s != WA_OK) return s;
  const size_t per_m = static_cast<size_t>(r) * cols;
  k_reduce_splits<<<reduce_grid(per_m), kReduceThreads, 0, st>>>(part, n_split, per_m,
                                                                  static_cast<__nv_bfloat16*>(k_til),
                                                                  static_cast<__nv_bfloat16*>(v_til));
  return check_launch("reduce_splits");
}

}  // namespace wa

// ============================================================================
// Projection without any allocation.
//
// Some callers cannot allocate device memory at all: code that runs inside a
// host framework which owns every device allocation through its own pool and
// forbids cudaMalloc, or a real-time loop where an allocation (which can
// synchronise the device) is not allowed.  They also may not have a workspace to
// hand over.  wa_linear_project_noalloc serves them: it runs the same tcgen05
// projection kernels as wa_linear_project, but keeps the split-L partial sums in
// one fixed, file-scope device array instead of a caller workspace.  The caller
// still passes its inputs and outputs.
//
// The array is kNoAllocScratchBytes (32 MiB) and is held by every GPU that loads
// this library until the process exits.  Its device address is looked up once per
// device and kept for the process: it belongs to the device's primary context and
// goes stale if that device is reset.  All calls share it, so calls that
// overlap on the GPU (for instance on two streams at once) race on it; callers
// must order them.  Each call overwrites every partial it reads before reading
// it, so the contents left by an earlier call never leak into a result.
// ============================================================================
namespace wa {
namespace {

constexpr size_t kNoAllocScratchBytes = 32ull << 20;
static __device__ __align__(256) float g_noalloc_partials[kNoAllocScratchBytes / sizeof(float)];

std::mutex g_noalloc_mu;
float* g_noalloc_ptr[64] = {};

// Device address of the static array for the current device.  In host code the
// array's name is only a host-side stand-in; the kernels need the address that
// cudaGetSymbolAddress returns, looked up once per device with that device current.
wa_status noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64)
    return set_error(WA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_partials);
    if (e != cudaSuccess || p == nullptr)
      return set_error(WA_ERR_CUDA, "cudaGetSymbolAddress(projection scratch): %s",
                       cudaGetErrorString(e));
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return WA_OK;
}

}  // namespace
}  // namespace wa

extern "C" wa_status wa_linear_project_noalloc(const void* k_act, const void* v_act,
                                               const void* e_k, const void* e_v, int L, int H,
                                               int d, int r, wa_dtype dtype, void* k_til,
                                               void* v_til, void* stream) {
  using namespace wa;
  if (!k_act || !v_act || !e_k || !e_v || !k_til || !v_til)
    return set_error(WA_ERR_INVALID_ARG, "NULL pointer");
  if (L < 1 || H < 1 || r < 1) return set_error(WA_ERR_INVALID_ARG, "sizes must be >= 1");
  if (dtype != WA_BF16)
    return set_error(WA_ERR_UNSUPPORTED, "wa_linear_project_noalloc takes bf16 inputs only");
  if (d != 64 && d != 128) return set_error(WA_ERR_UNSUPPORTED, "d must be 64 or 128");
  if (r != 128 && r != 256) return set_error(WA_ERR_UNSUPPORTED, "r must be 128 or 256");
  // as many splits of L as the default launch uses, but no more than the static
  // scratch holds (2 matrices x n_split x r x H*d floats); the product is formed in
  // 64 bits, so no H wraps around to a size that would pass
  const unsigned long long cols64 = static_cast<unsigned long long>(H) * d;
  const unsigned long long per_split = 2ull * r * cols64 * sizeof(float);
  if (per_split > kNoAllocScratchBytes)
    return set_error(WA_ERR_UNSUPPORTED,
                     "r*H*d = %llu needs %llu bytes of scratch per split; the static scratch holds %zu",
                     static_cast<unsigned long long>(r) * cols64, per_split, kNoAllocScratchBytes);
  const int cols = static_cast<int>(cols64);   // < 2^22 here
  const int tn = pick_tn(cols);
  if (tn == 0) return set_error(WA_ERR_UNSUPPORTED, "H*d must be a multiple of 64");
  const size_t fit = kNoAllocScratchBytes / per_split;
  int n_split = pick_splits(L, r, cols);
  if (static_cast<size_t>(n_split) > fit) n_split = static_cast<int>(fit);
  float* part = nullptr;
  wa_status s = noalloc_scratch(&part);
  if (s != WA_OK) return s;
  uint32_t* err = device_error_word();
  if (!err) return set_error(WA_ERR_CUDA, "no CUDA device");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  RowSource rs;
  rs.k = k_act; rs.v = v_act; rs.page_rows = L; rs.n_pages = 1; rs.L = L;
  alignas(64) CUtensorMap tek, tev, txk, txv;
  if (!make_tmap_bf16_2d(&tek, e_k, r, L, static_cast<uint64_t>(r) * 2, 64, 64) ||
      !make_tmap_bf16_2d(&tev, e_v, r, L, static_cast<uint64_t>(r) * 2, 64, 64) ||
      !make_tmap_bf16_2d(&txk, k_act, cols, L, static_cast<uint64_t>(cols) * 2, 64, 64) ||
      !make_tmap_bf16_2d(&txv, v_act, cols, L, static_cast<uint64_t>(cols) * 2, 64, 64))
    return set_error(WA_ERR_CUDA, "cuTensorMapEncodeTiled failed for the projection operands");
  dim3 grid(2 * (cols / tn), n_split);
  if (r == 256) {
    if (tn == 256) launch_proj<2, 256>(grid, st, tek, tev, txk, txv, rs, L, cols, n_split, part, err);
    else if (tn == 128) launch_proj<2, 128>(grid, st, tek, tev, txk, txv, rs, L, cols, n_split, part, err);
    else launch_proj<2, 64>(grid, st, tek, tev, txk, txv, rs, L, cols, n_split, part, err);
  } else {
    if (tn == 256) launch_proj<1, 256>(grid, st, tek, tev, txk, txv, rs, L, cols, n_split, part, err);
    else if (tn == 128) launch_proj<1, 128>(grid, st, tek, tev, txk, txv, rs, L, cols, n_split, part, err);
    else launch_proj<1, 64>(grid, st, tek, tev, txk, txv, rs, L, cols, n_split, part, err);
  }
  s = check_launch("umma_project (no-alloc)");
  if (s != WA_OK) return s;
  const size_t per_m = static_cast<size_t>(r) * cols;
  k_reduce_splits<<<reduce_grid(per_m), kReduceThreads, 0, st>>>(part, n_split, per_m,
                                                                  static_cast<__nv_bfloat16*>(k_til),
                                                                  static_cast<__nv_bfloat16*>(v_til));
  return check_launch("reduce_splits (no-alloc)");
}
