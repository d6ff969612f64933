// k_umma_attn.cu -- bf16 attention on the 5th-generation tensor cores (tcgen05,
// TMEM accumulators, TMA-fed shared memory) for the two HSA branches:
//   mode 0: linear branch, O_lin = softmax(Q K~^T / sqrt(d)) V~ over the r projected
//           keys (WorldAttention §3.3 "Linear branch"), stored as
//           (1 - sigmoid(g)) * O_lin in a float32 workspace;
//   mode 1: sparse branch, exact attention over the key blocks kept for each
//           (head, query block) (§3.3 "Sparse branch", Appendix A.1.3 "Block Sparse
//           Attention"), fused with the sigmoid gate (§3.3 "Gated fusion"):
//           out = bf16(sigmoid(g) * O_sp + workspace).
//
// The pages' kernels tile for Hopper WGMMA with 64-row query blocks.  The B200
// MMA wants M = 128, so one CTA takes a pair of query blocks of the same head
// (rows 0-63 and 64-127 of one tile) and walks the union of their two key-block
// sets, masking each half's unselected blocks to -inf.  Pairs are chosen to
// overlap as much as possible (k_pair_heads) and run longest first.
//
// CTA = 256 threads: warp 0 issues TMA loads (Q once, then K/V blocks through a
// 2-stage ring, straight from the pool pages via the page table), warp 1 owns
// TMEM and issues tcgen05.mma (S = Q K^T into one of two TMEM S buffers; O += P V
// with P read back from TMEM), warps 4-7 run the online softmax, one thread per
// TMEM lane (= query row), and the epilogue.  Two CTAs fit on an SM, so one CTA's
// softmax overlaps the other's MMAs.  Every wait is bounded in time.
#include <cuda.h>
#include <cuda_bf16.h>

#include <climits>
#include <cmath>

#include "sm100.cuh"
#include "wa_internal.h"

namespace wa {
namespace {

using namespace sm100;

constexpr int kBM = 128;          // query rows per tile (two 64-row blocks)
constexpr int kBN = 64;           // keys per block
constexpr int kStages = 2;
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 256;
constexpr int kColS = 0;          // two S/P buffers at columns 0 and 64
constexpr int kColO = 128;        // O accumulator at columns 128 .. 128+d
constexpr int kMaxW = 256;        // up to 8192 key blocks

template <int D>
struct Cfg {
  static constexpr int kPanels = D / 64;                 // 128-byte column panels
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kKVBytes = kBN * D * 2;
  static constexpr int kStageBytes = 2 * kKVBytes;
  static constexpr int kSmem = kQBytes + kStages * kStageBytes + 1024;  // + alignment slack
  static constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, false, false);
  static constexpr uint32_t kIdescO = idesc_bf16_f32(kBM, D, false, true);
};

struct Shared {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done;
  uint32_t tmem_base;
  int abort_flag;
  uint32_t mask[2][kMaxW];
};

// Bounded wait that also gives up when another role has aborted.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Shared& sh,
                                         uint32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0u) {
      if (*reinterpret_cast<volatile int*>(&sh.abort_flag)) return false;
      if (globaltimer_ns() - t0 > 2000000000ull) {
        atomicOr(err, WA_DEVERR_TIMEOUT);
        *reinterpret_cast<volatile int*>(&sh.abort_flag) = 1;
        return false;
      }
    }
  }
}

// Walks the key blocks of a tile in ascending order: the union of the two masks
// (mode 1) or every block (mode 0).
struct BlockIter {
  const uint32_t* a;
  const uint32_t* b;
  int W, n_kb, w, all;
  uint32_t bits;
  __device__ void init(const uint32_t* a_, const uint32_t* b_, int W_, int n_kb_, int all_) {
    a = a_; b = b_; W = W_; n_kb = n_kb_; all = all_; w = -1; bits = 0u;
  }
  __device__ int next() {
    if (all) { ++w; return w < n_kb ? w : -1; }
    while (bits == 0u) {
      if (++w >= W) return -1;
      bits = a[w] | b[w];
    }
    const int j = w * 32 + __ffs(bits) - 1;
    bits &= bits - 1u;
    return j;
  }
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
k_umma_attention(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, int mode, int Nq, int H, int Lk,
                 RowSource rs, const uint32_t* __restrict__ blk_mask, int W, int n_qb,
                 const int4* __restrict__ items, const float* __restrict__ gate,
                 float* __restrict__ lin_ws, __nv_bfloat16* __restrict__ out,
                 float* __restrict__ o_branch, uint32_t* err) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_dyn[];
  __shared__ Shared sh;
  uint8_t* tiles = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* Qs = tiles;
  auto Ks = [&](int s) { return tiles + C::kQBytes + s * C::kStageBytes; };
  auto Vs = [&](int s) { return tiles + C::kQBytes + s * C::kStageBytes + C::kKVBytes; };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int h, i0, i1;
  if (mode == 0) {
    const int n_pairs = (n_qb + 1) / 2;
    h = blockIdx.x / n_pairs;
    const int p = blockIdx.x % n_pairs;
    i0 = 2 * p;
    i1 = (2 * p + 1 < n_qb) ? 2 * p + 1 : -1;
  } else {
    const int4 it = items[blockIdx.x];
    h = it.x; i0 = it.y; i1 = it.z;
  }
  const int n_kb = (Lk + kBN - 1) / kBN;

  if (tid == 0) {
    mbar_init(&sh.q_full, 1);
    for (int s = 0; s < kStages; ++s) { mbar_init(&sh.kv_full[s], 1); mbar_init(&sh.kv_empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&sh.s_full[b], 1); mbar_init(&sh.p_full[b], 128); }
    mbar_init(&sh.o_done, 1);
    sh.abort_flag = 0;
    fence_mbar_init();
  }
  if (mode == 1) {
    const uint32_t* ma = blk_mask + (static_cast<size_t>(h) * n_qb + i0) * W;
    const uint32_t* mb = i1 >= 0 ? blk_mask + (static_cast<size_t>(h) * n_qb + i1) * W : nullptr;
    for (int w = tid; w < W; w += kThreads) {
      sh.mask[0][w] = ma[w];
      sh.mask[1][w] = mb ? mb[w] : 0u;
    }
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sh.tmem_base;

  // number of key blocks this tile walks
  int n_blk = 0;
  if (mode == 0) {
    n_blk = n_kb;
  } else {
    for (int w = 0; w < W; ++w) n_blk += __popc(sh.mask[0][w] | sh.mask[1][w]);
  }
  const int bpp = rs.page_ids ? rs.page_rows / kBN : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(&sh.q_full, C::kQBytes);
      const int y1 = i1 >= 0 ? i1 * 64 : Nq;  // out of range -> zero fill
      for (int p = 0; p < C::kPanels; ++p) {
        tma_load_2d(Qs + p * (kBM * 128), &tmQ, &sh.q_full, h * D + p * 64, i0 * 64);
        tma_load_2d(Qs + p * (kBM * 128) + 64 * 128, &tmQ, &sh.q_full, h * D + p * 64, y1);
      }
      BlockIter it;
      it.init(sh.mask[0], sh.mask[1], W, n_kb, mode == 0);
      int t = 0;
      for (int j = it.next(); j >= 0; j = it.next(), ++t) {
        const int s = t % kStages;
        if (!wait_bar(&sh.kv_empty[s], ((t / kStages) & 1) ^ 1, sh, err)) break;
        int row;
        if (rs.page_ids) {
          int pg = rs.page_ids[j / bpp];
          if (pg < 0 || pg >= rs.n_pages) { atomicOr(err, WA_DEVERR_PAGE_ID); pg = 0; }
          row = pg * rs.page_rows + (j % bpp) * kBN;
        } else {
          row = j * kBN;
        }
        mbar_arrive_expect_tx(&sh.kv_full[s], C::kStageBytes);
        for (int p = 0; p < C::kPanels; ++p) {
          tma_load_2d(Ks(s) + p * (kBN * 128), &tmK, &sh.kv_full[s], h * D + p * 64, row);
          tma_load_2d(Vs(s) + p * (kBN * 128), &tmV, &sh.kv_full[s], h * D + p * 64, row);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = wait_bar(&sh.q_full, 0, sh, err);
      tc_fence_after();
      const uint32_t q_base = smem_u32(Qs);
      auto issue_pv = [&](int u) -> bool {
        const int su = u & 1;
        if (!wait_bar(&sh.p_full[su], (u >> 1) & 1, sh, err)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(Vs(u % kStages));
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bdesc = smem_desc_sw128(v_base + kk * 2048, 64 * 128, 1024);
          mma_ts(tbase + kColO, tbase + kColS + su * 64 + kk * 8, bdesc, C::kIdescO,
                 (u > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&sh.kv_empty[u % kStages]);
        mma_commit(&sh.o_done);
        return true;
      };
      int t = 0;
      for (; ok && t < n_blk; ++t) {
        const int s = t % kStages;
        if (!wait_bar(&sh.kv_full[s], (t / kStages) & 1, sh, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_base = smem_u32(Ks(s));
        const int sb = t & 1;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t adesc = smem_desc_sw128(q_base + (k >> 2) * (kBM * 128) + (k & 3) * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(k_base + (k >> 2) * (kBN * 128) + (k & 3) * 32, 16, 1024);
          mma_ss(tbase + kColS + sb * 64, adesc, bdesc, C::kIdescS, k > 0 ? 1u : 0u);
        }
        mma_commit(&sh.s_full[sb]);
        if (t > 0 && !issue_pv(t - 1)) { ok = false; break; }
      }
      if (ok && n_blk > 0) ok = issue_pv(n_blk - 1);
      (void)ok;
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int q4 = warp - 4;
    const int row = q4 * 32 + lane;                 // TMEM lane = tile row
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const int half = row >> 6;
    const int ib = half ? i1 : i0;
    const int qrow = ib * 64 + (row & 63);
    const bool row_valid = ib >= 0 && qrow < Nq;
    const uint32_t* mymask = sh.mask[half];
    const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    BlockIter it;
    it.init(sh.mask[0], sh.mask[1], W, n_kb, mode == 0);
    int t = 0;
    for (int j = it.next(); j >= 0; j = it.next(), ++t) {
      const int sb = t & 1;
      if (!__all_sync(0xffffffffu, wait_bar(&sh.s_full[sb], (t >> 1) & 1, sh, err))) { ok = false; break; }
      tc_fence_after();
      uint32_t r[64];
      tmem_ld32(tbase + lane_base + kColS + sb * 64, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
      tmem_ld32(tbase + lane_base + kColS + sb * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
      tmem_wait_ld();
      const bool sel = mode == 0 || ((mymask[j >> 5] >> (j & 31)) & 1u);
      const int valid = min(kBN, Lk - j * kBN);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        float s = __uint_as_float(r[c]) * scale_log2;
        if (!sel || c >= valid) s = -INFINITY;
        r[c] = __float_as_uint(s);
        mx = fmaxf(mx, s);
      }
      float factor = 1.f;
      bool resc = false;
      if (m_run == -INFINITY) {
        m_run = mx;                        // no mass yet: O holds zeros for this row
      } else if (mx > m_run + 8.f) {       // keep a stale max unless it grows by > 2^8
        factor = ex2(m_run - mx);
        m_run = mx;
        resc = true;
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 64; c += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = ex2(__uint_as_float(r[c + 2 * e]) - m_use);
          const float p1 = ex2(__uint_as_float(r[c + 2 * e + 1]) - m_use);
          sum += p0 + p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tbase + lane_base + kColS + sb * 64 + c / 2, pk);
      }
      l_run = l_run * factor + sum;
      tmem_wait_st();
      if (t > 0) {
        if (!__all_sync(0xffffffffu, wait_bar(&sh.o_done, (t - 1) & 1, sh, err))) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tbase + lane_base + kColO + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
            tmem_st32(tbase + lane_base + kColO + c0, o);
          }
          tmem_wait_st();
        }
      }
      tc_fence_before();
      mbar_arrive(&sh.p_full[sb]);
    }
    if (ok && t > 0) ok = __all_sync(0xffffffffu, wait_bar(&sh.o_done, (t - 1) & 1, sh, err));
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    // epilogue
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    float sg = 0.f;
    size_t obase = 0;
    if (row_valid) {
      const float g = gate[static_cast<size_t>(qrow) * H + h];
      sg = 1.f / (1.f + expf(-g));
      obase = static_cast<size_t>(qrow) * H * D + static_cast<size_t>(h) * D;
    }
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t o[32];
      if (ok && t > 0) {
        tmem_ld32(tbase + lane_base + kColO + c0, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
      if (!row_valid) continue;
      float v[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(o[e]) * inv;
      if (o_branch) {
        float4* ob = reinterpret_cast<float4*>(o_branch + obase + c0);
#pragma unroll
        for (int e = 0; e < 8; ++e) ob[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
      }
      if (mode == 0) {
        float4* lw = reinterpret_cast<float4*>(lin_ws + obase + c0);
        const float a = 1.f - sg;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          lw[e] = make_float4(a * v[4 * e], a * v[4 * e + 1], a * v[4 * e + 2], a * v[4 * e + 3]);
      } else {
        const float4* lw = reinterpret_cast<const float4*>(lin_ws + obase + c0);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float4 l4 = lw[e];
          pk[2 * e] = pack_bf16x2(sg * v[4 * e] + l4.x, sg * v[4 * e + 1] + l4.y);
          pk[2 * e + 1] = pack_bf16x2(sg * v[4 * e + 2] + l4.z, sg * v[4 * e + 3] + l4.w);
        }
        uint4* op = reinterpret_cast<uint4*>(out + obase + c0);
#pragma unroll
        for (int e = 0; e < 4; ++e) op[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// ------------------------------------------------------------------ work items
// One CTA per head pairs its query blocks greedily by the smallest symmetric
// difference of their key-block sets (fewest masked half-blocks), falling back
// to neighbours when there are too many blocks for the distance table.
constexpr int kMaxPairTable = 144;  // 144^2 uint16 distances fit in static shared memory

__global__ void k_pair_heads(const uint32_t* __restrict__ mask, int n_qb, int W,
                             int4* __restrict__ items) {
  __shared__ uint16_t dist[kMaxPairTable * kMaxPairTable];
  __shared__ unsigned char paired[kMaxPairTable];
  const int h = blockIdx.x;
  const int n_pairs = (n_qb + 1) / 2;
  const uint32_t* mh = mask + static_cast<size_t>(h) * n_qb * W;
  auto union_count = [&](int a, int b) {
    int c = 0;
    for (int w = 0; w < W; ++w) c += __popc(mh[a * W + w] | (b >= 0 ? mh[b * W + w] : 0u));
    return c;
  };
  if (n_qb > kMaxPairTable) {
    for (int p = threadIdx.x; p < n_pairs; p += blockDim.x) {
      const int a = 2 * p, b = (2 * p + 1 < n_qb) ? 2 * p + 1 : -1;
      items[static_cast<size_t>(h) * n_pairs + p] = make_int4(h, a, b, union_count(a, b));
    }
    return;
  }
  for (int e = threadIdx.x; e < n_qb * n_qb; e += blockDim.x) {
    const int a = e / n_qb, b = e % n_qb;
    int c = 0;
    if (a < b)
      for (int w = 0; w < W; ++w) c += __popc(mh[a * W + w] ^ mh[b * W + w]);
    dist[e] = static_cast<uint16_t>(min(c, 65535));
  }
  for (int a = threadIdx.x; a < n_qb; a += blockDim.x) paired[a] = 0;
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int k = 0;
    for (int a = 0; a < n_qb; ++a) {
      if (paired[a]) continue;
      int best = INT_MAX, bi = -1;
      for (int b = a + 1 + lane; b < n_qb; b += 32) {
        if (paired[b]) continue;
        const int dv = dist[a * n_qb + b];
        if (dv < best) { best = dv; bi = b; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const int ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ob < best || (ob == best && oi >= 0 && (bi < 0 || oi < bi))) { best = ob; bi = oi; }
      }
      __syncwarp();
      if (lane == 0) {
        paired[a] = 1;
        if (bi >= 0) paired[bi] = 1;
        items[static_cast<size_t>(h) * n_pairs + k] = make_int4(h, a, bi, 0);
      }
      __syncwarp();
      ++k;
    }
  }
  __syncthreads();
  for (int p = threadIdx.x; p < n_pairs; p += blockDim.x) {
    int4 it = items[static_cast<size_t>(h) * n_pairs + p];
    it.w = union_count(it.y, it.z);
    items[static_cast<size_t>(h) * n_pairs + p] = it;
  }
}

// Longest-first order (ties by head, then first block) with one CTA's bitonic sort.
constexpr int kMaxSortItems = 4096;

__device__ __forceinline__ bool item_before(int4 a, int4 b) {
  if (a.w != b.w) return a.w > b.w;
  if (a.x != b.x) return a.x < b.x;
  return a.y < b.y;
}

__global__ void __launch_bounds__(1024) k_sort_items(int4* __restrict__ items, int n, int NP) {
  extern __shared__ int4 buf[];
  for (int e = threadIdx.x; e < NP; e += blockDim.x)
    buf[e] = e < n ? items[e] : make_int4(INT_MAX, INT_MAX, INT_MAX, -1);
  __syncthreads();
  for (int k = 2; k <= NP; k <<= 1) {
    for (int js = k >> 1; js > 0; js >>= 1) {
      for (int p = threadIdx.x; p < NP / 2; p += blockDim.x) {
        const int i = 2 * js * (p / js) + (p % js), l = i + js;
        const int4 a = buf[i], b = buf[l];
        const bool up = (i & k) == 0;
        const bool sw = up ? item_before(b, a) : item_before(a, b);
        if (sw) { buf[i] = b; buf[l] = a; }
      }
      __syncthreads();
    }
  }
  for (int e = threadIdx.x; e < n; e += blockDim.x) items[e] = buf[e];
}

}  // namespace

size_t attn_items_ws_bytes(int H, int n_qb) {
  return static_cast<size_t>(H) * ((n_qb + 1) / 2) * sizeof(int4);
}

wa_status launch_attn_items(const uint32_t* blk_mask, int H, int n_qb, int n_kb, int4* items,
                            void* /*scratch*/, cudaStream_t st) {
  const int W = (n_kb + 31) / 32;
  k_pair_heads<<<H, 256, 0, st>>>(blk_mask, n_qb, W, items);
  const int n = H * ((n_qb + 1) / 2);
  if (n <= kMaxSortItems) {
    int NP = 1;
    while (NP < n) NP <<= 1;
    if (NP < 2) NP = 2;
    cudaFuncSetAttribute(k_sort_items, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(NP * sizeof(int4)));
    k_sort_items<<<1, 1024, NP * sizeof(int4), st>>>(items, n, NP);
  }
  return check_launch("attn_items");
}

bool make_tmap_bf16_2d(void* tmap, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer);

wa_status launch_umma_attention(int mode, const void* q, int Nq, int H, int d, RowSource rs,
                                int B, const uint32_t* blk_mask, int W, const int4* items,
                                int n_items, const float* gate, float* lin_ws, void* out,
                                float* o_branch, uint32_t* err, cudaStream_t st) {
  if (B != kBN) return set_error(WA_ERR_UNSUPPORTED, "bf16 attention needs B == 64");
  if (d != 64 && d != 128) return set_error(WA_ERR_UNSUPPORTED, "bf16 attention needs d in {64,128}");
  if (W > kMaxW) return set_error(WA_ERR_UNSUPPORTED, "too many key blocks (max %d)", kMaxW * 32);
  const int cols = H * d;
  alignas(64) CUtensorMap tq, tk, tv;
  const uint64_t key_rows = rs.page_ids ? static_cast<uint64_t>(rs.n_pages) * rs.page_rows
                                        : static_cast<uint64_t>(rs.L);
  if (!make_tmap_bf16_2d(&tq, q, cols, Nq, static_cast<uint64_t>(cols) * 2, 64, 64) ||
      !make_tmap_bf16_2d(&tk, rs.k, cols, key_rows, static_cast<uint64_t>(cols) * 2, 64, 64) ||
      !make_tmap_bf16_2d(&tv, rs.v, cols, key_rows, static_cast<uint64_t>(cols) * 2, 64, 64))
    return set_error(WA_ERR_CUDA, "cuTensorMapEncodeTiled failed for the attention operands");
  const int n_qb = (Nq + B - 1) / B;
  const int grid = mode == 0 ? H * ((n_qb + 1) / 2) : n_items;
  if (grid == 0) return WA_OK;
  if (d == 128) {
    const int smem = Cfg<128>::kSmem;
    cudaFuncSetAttribute(k_umma_attention<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    k_umma_attention<128><<<grid, kThreads, smem, st>>>(
        tq, tk, tv, mode, Nq, H, rs.L, rs, blk_mask, W, n_qb, items, gate, lin_ws,
        static_cast<__nv_bfloat16*>(out), o_branch, err);
  } else {
    const int smem = Cfg<64>::kSmem;
    cudaFuncSetAttribute(k_umma_attention<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    k_umma_attention<64><<<grid, kThreads, smem, st>>>(
        tq, tk, tv, mode, Nq, H, rs.L, rs, blk_mask, W, n_qb, items, gate, lin_ws,
        static_cast<__nv_bfloat16*>(out), o_branch, err);
  }
  return check_launch("umma_attention");
}

}  // namespace wa
