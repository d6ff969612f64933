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
// MMA wants M = 128, so a tile is a pair of query blocks of the same head (rows
// 0-63 and 64-127) that walks the union of their two key-block sets, each half
// masking the blocks it did not select.  Pairs are chosen to overlap as much as
// possible (k_pair_heads).  A pair's key list is split in two work items when it
// is long enough, so that the work items fill whole waves of CTAs; the two
// partial results (unnormalised O, running max m, sum l per row) are merged by
// k_combine, which also applies the gate.  Items run longest first.
//
// CTA = 256 threads, two CTAs per SM: warp 0 loads Q and the K blocks, warp 2 the
// V blocks (TMA, 128-byte swizzle, straight from the pool pages through the page
// table, each through its own 2-slot ring: a K slot frees as soon as its S = Q K^T
// MMA completes, a V slot when its O += P V MMA completes); warp 1 owns TMEM and
// issues tcgen05.mma; warps 4-7 run the online softmax with one thread per TMEM
// lane (query row), write P back as bf16 into the S buffer, rescale O in TMEM only
// when the running max grows by more than 2^8, and run the epilogue.  One CTA's
// softmax overlaps the other CTA's MMAs.  Every wait is bounded in time.
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
constexpr int kRing = 2;          // slots of the K ring and of the V ring
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 256;
constexpr int kColS = 0;          // two S/P buffers at columns 0 and 64
constexpr int kColO = 128;        // O accumulator at columns 128 .. 128+d
constexpr int kMaxW = 256;        // up to 8192 key blocks
constexpr int kSplitMin = 8;      // pairs with at least this many key blocks are split in two

// item.y values
constexpr int kWhole = -1;        // the whole key list; writes the final output
constexpr int kEmpty = -2;        // placeholder: nothing to do

template <int D>
struct Cfg {
  static constexpr int kPanels = D / 64;                 // 128-byte column panels
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kKVBytes = kBN * D * 2;
  static constexpr int kSmem = kQBytes + 2 * kRing * kKVBytes + 1024;  // + alignment slack
  static constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, false, false);
  static constexpr uint32_t kIdescO = idesc_bf16_f32(kBM, D, false, true);
};

struct Shared {
  uint64_t q_full;
  uint64_t k_full[kRing], k_empty[kRing];
  uint64_t v_full[kRing], v_empty[kRing];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done[2];   // completion of O += P_u V_u, by the parity of u
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

// Walks key blocks [k0, k1) of a tile's list in ascending block order: the list is
// the union of the two masks (mode 1) or every block (mode 0).
struct BlockIter {
  const uint32_t* a;
  const uint32_t* b;
  int W, n_kb, w, all, pos, k1;
  uint32_t bits;
  __device__ int next_raw() {
    if (all) { ++w; return w < n_kb ? w : -1; }
    while (bits == 0u) {
      if (++w >= W) return -1;
      bits = a[w] | b[w];
    }
    const int j = w * 32 + __ffs(bits) - 1;
    bits &= bits - 1u;
    return j;
  }
  __device__ void init(const uint32_t* a_, const uint32_t* b_, int W_, int n_kb_, int all_, int k0_,
                       int k1_) {
    a = a_; b = b_; W = W_; n_kb = n_kb_; all = all_; w = -1; bits = 0u; pos = 0; k1 = k1_;
    for (; pos < k0_; ++pos) next_raw();
  }
  __device__ int next() {
    if (pos >= k1) return -1;
    ++pos;
    return next_raw();
  }
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ int key_row(const RowSource& rs, int bpp, int j, uint32_t* err) {
  if (!rs.page_ids) return j * kBN;
  int pg = rs.page_ids[j / bpp];
  if (pg < 0 || pg >= rs.n_pages) { atomicOr(err, WA_DEVERR_PAGE_ID); pg = 0; }
  return pg * rs.page_rows + (j % bpp) * kBN;
}

struct Partials {
  float* o;    // [slots][128][d]  unnormalised O
  float* ml;   // [slots][128][2]  running max (log2 units) and sum
};

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
k_umma_attention(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, int mode, int Nq, int H, int Lk,
                 RowSource rs, const uint32_t* __restrict__ blk_mask, int W, int n_qb,
                 const int4* __restrict__ pairs, const int4* __restrict__ items, Partials part,
                 const float* __restrict__ gate, float* __restrict__ lin_ws,
                 __nv_bfloat16* __restrict__ out, float* __restrict__ o_branch, uint32_t* err) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_dyn[];
  __shared__ Shared sh;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_kb = (Lk + kBN - 1) / kBN;
  int h, i0, i1, k0, k1, kind, slot;
  if (mode == 0) {
    const int n_pairs = (n_qb + 1) / 2;
    h = blockIdx.x / n_pairs;
    const int p = blockIdx.x % n_pairs;
    i0 = 2 * p;
    i1 = (2 * p + 1 < n_qb) ? 2 * p + 1 : -1;
    k0 = 0; k1 = n_kb; kind = kWhole; slot = 0;
  } else {
    const int4 it = items[blockIdx.x];
    kind = it.y;
    if (kind == kEmpty) return;
    const int4 pr = pairs[it.x];
    h = pr.x; i0 = pr.y; i1 = pr.z;
    k0 = it.z; k1 = it.w;
    slot = 2 * it.x + (kind < 0 ? 0 : kind);
  }
  uint8_t* tiles = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* Qs = tiles;
  auto Ks = [&](int s) { return tiles + C::kQBytes + s * C::kKVBytes; };
  auto Vs = [&](int s) { return tiles + C::kQBytes + (kRing + s) * C::kKVBytes; };

  if (tid == 0) {
    mbar_init(&sh.q_full, 1);
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&sh.k_full[s], 1); mbar_init(&sh.k_empty[s], 1);
      mbar_init(&sh.v_full[s], 1); mbar_init(&sh.v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) { mbar_init(&sh.s_full[b], 1); mbar_init(&sh.p_full[b], 128); }
    mbar_init(&sh.o_done[0], 1);
    mbar_init(&sh.o_done[1], 1);
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
  const int n_blk = k1 - k0;
  const int bpp = rs.page_ids ? rs.page_rows / kBN : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ Q + K producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      mbar_arrive_expect_tx(&sh.q_full, C::kQBytes);
      const int y1 = i1 >= 0 ? i1 * 64 : Nq;  // out of range -> zero fill
      for (int p = 0; p < C::kPanels; ++p) {
        tma_load_2d(Qs + p * (kBM * 128), &tmQ, &sh.q_full, h * D + p * 64, i0 * 64);
        tma_load_2d(Qs + p * (kBM * 128) + 64 * 128, &tmQ, &sh.q_full, h * D + p * 64, y1);
      }
      BlockIter it;
      it.init(sh.mask[0], sh.mask[1], W, n_kb, mode == 0, k0, k1);
      int t = 0;
      for (int j = it.next(); j >= 0; j = it.next(), ++t) {
        const int s = t % kRing;
        if (!wait_bar(&sh.k_empty[s], ((t / kRing) & 1) ^ 1, sh, err)) break;
        const int row = key_row(rs, bpp, j, err);
        mbar_arrive_expect_tx(&sh.k_full[s], C::kKVBytes);
        for (int p = 0; p < C::kPanels; ++p)
          tma_load_2d(Ks(s) + p * (kBN * 128), &tmK, &sh.k_full[s], h * D + p * 64, row);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ V producer
    if (lane == 0) {
      prefetch_tmap(&tmV);
      BlockIter it;
      it.init(sh.mask[0], sh.mask[1], W, n_kb, mode == 0, k0, k1);
      int t = 0;
      for (int j = it.next(); j >= 0; j = it.next(), ++t) {
        const int s = t % kRing;
        if (!wait_bar(&sh.v_empty[s], ((t / kRing) & 1) ^ 1, sh, err)) break;
        const int row = key_row(rs, bpp, j, err);
        mbar_arrive_expect_tx(&sh.v_full[s], C::kKVBytes);
        for (int p = 0; p < C::kPanels; ++p)
          tma_load_2d(Vs(s) + p * (kBN * 128), &tmV, &sh.v_full[s], h * D + p * 64, row);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = wait_bar(&sh.q_full, 0, sh, err);
      tc_fence_after();
      const uint32_t q_base = smem_u32(Qs);
      for (int t = 0; ok && t <= n_blk; ++t) {
        if (t < n_blk) {
          // S_t = Q K_t^T into S buffer t % 2 (its previous P was consumed by PV_{t-2},
          // issued earlier by this thread)
          const int s = t % kRing;
          if (!wait_bar(&sh.k_full[s], (t / kRing) & 1, sh, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_base = smem_u32(Ks(s));
          const int sb = t & 1;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint64_t adesc = smem_desc_sw128(q_base + (k >> 2) * (kBM * 128) + (k & 3) * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(k_base + (k >> 2) * (kBN * 128) + (k & 3) * 32, 16, 1024);
            mma_ss(tbase + kColS + sb * 64, adesc, bdesc, C::kIdescS, k > 0 ? 1u : 0u);
          }
          mma_commit(&sh.k_empty[s]);
          mma_commit(&sh.s_full[sb]);
        }
        if (t > 0) {
          // O += P_u V_u, P read from TMEM
          const int u = t - 1, su = u & 1, vs = u % kRing;
          if (!wait_bar(&sh.p_full[su], (u >> 1) & 1, sh, err)) { ok = false; break; }
          if (!wait_bar(&sh.v_full[vs], (u / kRing) & 1, sh, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t v_base = smem_u32(Vs(vs));
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            const uint64_t bdesc = smem_desc_sw128(v_base + kk * 2048, 64 * 128, 1024);
            mma_ts(tbase + kColO, tbase + kColS + su * 64 + kk * 8, bdesc, C::kIdescO,
                   (u > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&sh.v_empty[vs]);
          mma_commit(&sh.o_done[u & 1]);
        }
      }
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
    it.init(sh.mask[0], sh.mask[1], W, n_kb, mode == 0, k0, k1);
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
      if (!sel || valid < kBN) {
        // a block this half did not select, or the ragged last block: mask columns
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (!sel || c >= valid) r[c] = __float_as_uint(-INFINITY);
      }
      // row max of the raw scores: eight independent chains of 3-input maxima
      float mx8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(__uint_as_float(r[e]), __uint_as_float(r[8 + e]));
#pragma unroll
      for (int c = 16; c < 64; c += 16)
#pragma unroll
        for (int e = 0; e < 8; ++e)
          mx8[e] = max3f(mx8[e], __uint_as_float(r[c + e]), __uint_as_float(r[c + 8 + e]));
      const float mraw = max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]),
                               fmaxf(mx8[6], mx8[7]));
      const float mx = mraw * scale_log2;   // scale_log2 > 0: the max commutes with it
      float factor = 1.f;
      bool resc = false;
      if (m_run == -INFINITY) {
        m_run = mx;                        // no mass yet: O holds zeros for this row
      } else if (mx > m_run + 8.f) {       // keep a stale max unless it grows by > 2^8
        factor = ex2(m_run - mx);
        m_run = mx;
        resc = true;
      }
      const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
      // p = 2^(s * log2(e)/sqrt(d) - m) on column pairs (paired fp32 FMA and add),
      // summed in four two-lane chains, packed to bf16 pairs
      const float2 sc2 = make_float2(scale_log2, scale_log2);
      const float2 nm2 = make_float2(neg_m, neg_m);
      float2 acc2[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) acc2[e] = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < 64; c += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 x = make_float2(__uint_as_float(r[c + 2 * e]), __uint_as_float(r[c + 2 * e + 1]));
          const float2 y = __ffma2_rn(x, sc2, nm2);
          const float2 pp = make_float2(ex2(y.x), ex2(y.y));
          acc2[e & 3] = __fadd2_rn(acc2[e & 3], pp);
          pk[e] = pack_bf16x2(pp.x, pp.y);
        }
        tmem_st16(tbase + lane_base + kColS + sb * 64 + c / 2, pk);
      }
      const float2 a01 = __fadd2_rn(acc2[0], acc2[1]), a23 = __fadd2_rn(acc2[2], acc2[3]);
      const float2 a03 = __fadd2_rn(a01, a23);
      const float sum = a03.x + a03.y;
      l_run = l_run * factor + sum;
      tmem_wait_st();
      if (__any_sync(0xffffffffu, resc)) {
        // O may be rescaled only once PV_{t-1} has landed in it.  MMAs complete in
        // issue order and S_{t-1} (already waited for) was issued after PV_{t-3},
        // so on the barrier of PV_{t-1}'s parity at most PV_{t-1} is outstanding and
        // this parity wait is unambiguous although iterations without a rescale
        // skip it; S_t (waited for) also implies PV_{t-2} has landed.
        const int u = t - 1;
        if (!__all_sync(0xffffffffu, wait_bar(&sh.o_done[u & 1], (u >> 1) & 1, sh, err))) { ok = false; break; }
        tc_fence_after();
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
      tc_fence_before();
      mbar_arrive(&sh.p_full[sb]);
    }
    // the last two PVs may both be outstanding: one wait on each parity's barrier
    if (ok && t > 0) ok = __all_sync(0xffffffffu, wait_bar(&sh.o_done[(t - 1) & 1], ((t - 1) >> 1) & 1, sh, err));
    if (ok && t > 1) ok = __all_sync(0xffffffffu, wait_bar(&sh.o_done[(t - 2) & 1], ((t - 2) >> 1) & 1, sh, err));
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    const bool have_o = ok && t > 0;
    if (kind >= 0) {
      // one half of a split key list: hand the unnormalised state to k_combine
      float* po = part.o + (static_cast<size_t>(slot) * kBM + row) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        if (have_o) {
          tmem_ld32(tbase + lane_base + kColO + c0, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0u;
        }
        float4* p4 = reinterpret_cast<float4*>(po + c0);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          p4[e] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                              __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
      }
      *reinterpret_cast<float2*>(part.ml + (static_cast<size_t>(slot) * kBM + row) * 2) =
          make_float2(m_run, l_run);
    } else {
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
        if (have_o) {
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
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// Merge the two halves of a split pair: M = max(m0, m1), w_s = 2^(m_s - M),
// O = (w0 O0 + w1 O1) / (w0 l0 + w1 l1); then out = bf16(sigmoid(g) O + lin_ws).
// CTA = (pair, 32 tile rows); each thread takes 16 columns of one row (a warp
// covers 4 rows x 512 contiguous bytes), all its loads issued up front.
template <int D>
__global__ void __launch_bounds__(2 * D)
k_combine(const int4* __restrict__ pairs, Partials part, int Nq, int H,
          const float* __restrict__ gate, const float* __restrict__ lin_ws,
          __nv_bfloat16* __restrict__ out, float* __restrict__ o_branch) {
  constexpr int kSeg = D / 16;                 // 16-column segments per row
  const int4 pr = pairs[blockIdx.x];
  if (pr.w < kSplitMin) return;                // written whole by the attention kernel
  const int row = blockIdx.y * 32 + threadIdx.x / kSeg;
  const int c0 = (threadIdx.x % kSeg) * 16;
  const int half = row >> 6;
  const int ib = half ? pr.z : pr.y;
  const int qrow = ib * 64 + (row & 63);
  if (ib < 0 || qrow >= Nq) return;
  const int h = pr.x;
  const size_t s0 = 2 * static_cast<size_t>(blockIdx.x), s1 = s0 + 1;
  const float4* o0 = reinterpret_cast<const float4*>(part.o + (s0 * kBM + row) * D + c0);
  const float4* o1 = reinterpret_cast<const float4*>(part.o + (s1 * kBM + row) * D + c0);
  const size_t obase = static_cast<size_t>(qrow) * H * D + static_cast<size_t>(h) * D + c0;
  const float4* lw = reinterpret_cast<const float4*>(lin_ws + obase);
  float4 x[4], y[4], l4[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) { x[e] = o0[e]; y[e] = o1[e]; l4[e] = lw[e]; }
  const float2 a = *reinterpret_cast<const float2*>(part.ml + (s0 * kBM + row) * 2);
  const float2 b = *reinterpret_cast<const float2*>(part.ml + (s1 * kBM + row) * 2);
  const float g = gate[static_cast<size_t>(qrow) * H + h];
  const float M = fmaxf(a.x, b.x);
  const float w0 = a.x == -INFINITY ? 0.f : exp2f(a.x - M);
  const float w1 = b.x == -INFINITY ? 0.f : exp2f(b.x - M);
  const float lsum = w0 * a.y + w1 * b.y;
  const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
  const float c0w = w0 * inv, c1w = w1 * inv;
  const float sg = 1.f / (1.f + expf(-g));
  uint32_t pk[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float v0 = c0w * x[e].x + c1w * y[e].x, v1 = c0w * x[e].y + c1w * y[e].y;
    const float v2 = c0w * x[e].z + c1w * y[e].z, v3 = c0w * x[e].w + c1w * y[e].w;
    if (o_branch) reinterpret_cast<float4*>(o_branch + obase)[e] = make_float4(v0, v1, v2, v3);
    pk[2 * e] = pack_bf16x2(sg * v0 + l4[e].x, sg * v1 + l4[e].y);
    pk[2 * e + 1] = pack_bf16x2(sg * v2 + l4[e].z, sg * v3 + l4[e].w);
  }
  uint4* op = reinterpret_cast<uint4*>(out + obase);
  op[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  op[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}

// ------------------------------------------------------------------ work items
// One CTA per head pairs its query blocks by rounds of mutual nearest neighbours:
// distance = size of the symmetric difference of the two key-block sets (the
// half-blocks the pair computes and masks), ties broken by the lower block index.
// Each round pairs every two unpaired blocks that are each other's nearest
// unpaired neighbour; the closest remaining pair always qualifies, so every round
// makes progress.  Falls back to neighbours when there are too many blocks for the
// distance table.  pairs[h * n_pairs + k] = (h, first, second or -1, union size).
constexpr int kMaxPairTable = 128;
constexpr int kMaxPairMaskWords = 3072;   // staged masks of one head (n_qb * W words)

__global__ void __launch_bounds__(256)
k_pair_heads(const uint32_t* __restrict__ mask, int n_qb, int W, int4* __restrict__ pairs) {
  __shared__ uint16_t dist[kMaxPairTable * kMaxPairTable];
  __shared__ uint32_t ms[kMaxPairMaskWords];
  __shared__ int partner[kMaxPairTable];
  __shared__ int nn[kMaxPairTable];
  __shared__ int progress;
  const int h = blockIdx.x;
  const int n_pairs = (n_qb + 1) / 2;
  const uint32_t* mh = mask + static_cast<size_t>(h) * n_qb * W;
  const bool staged = n_qb * W <= kMaxPairMaskWords;
  if (staged)
    for (int e = threadIdx.x; e < n_qb * W; e += blockDim.x) ms[e] = mh[e];
  __syncthreads();
  const uint32_t* m = staged ? ms : mh;
  auto union_count = [&](int a, int b) {
    int c = 0;
    for (int w = 0; w < W; ++w) c += __popc(m[a * W + w] | (b >= 0 ? m[b * W + w] : 0u));
    return c;
  };
  if (n_qb > kMaxPairTable) {
    for (int p = threadIdx.x; p < n_pairs; p += blockDim.x) {
      const int a = 2 * p, b = (2 * p + 1 < n_qb) ? 2 * p + 1 : -1;
      pairs[static_cast<size_t>(h) * n_pairs + p] = make_int4(h, a, b, union_count(a, b));
    }
    return;
  }
  for (int e = threadIdx.x; e < n_qb * n_qb; e += blockDim.x) {
    const int a = e / n_qb, b = e - a * n_qb;
    int c = 0;
    if (a != b)
      for (int w = 0; w < W; ++w) c += __popc(m[a * W + w] ^ m[b * W + w]);
    dist[e] = static_cast<uint16_t>(min(c, 65535));
  }
  for (int a = threadIdx.x; a < n_qb; a += blockDim.x) partner[a] = -2;   // -2: unpaired
  __syncthreads();
  for (int round = 0; round < n_qb; ++round) {
    for (int a = threadIdx.x; a < n_qb; a += blockDim.x) {
      int best = INT_MAX, bi = -1;
      if (partner[a] == -2)
        for (int b = 0; b < n_qb; ++b) {
          if (b == a || partner[b] != -2) continue;
          const int dv = dist[a * n_qb + b];
          if (dv < best) { best = dv; bi = b; }   // increasing b: ties keep the lower index
        }
      nn[a] = bi;
    }
    if (threadIdx.x == 0) progress = 0;
    __syncthreads();
    for (int a = threadIdx.x; a < n_qb; a += blockDim.x) {
      const int b = nn[a];
      if (b > a && nn[b] == a) { partner[a] = b; partner[b] = a; progress = 1; }
    }
    __syncthreads();
    if (!progress) break;
  }
  // emit pairs in order of their first block (deterministic); a block left alone
  // (odd count) gets partner -1
  if (threadIdx.x == 0) {
    int k = 0;
    for (int a = 0; a < n_qb; ++a) {
      const int b = partner[a];
      if (b >= 0 && b < a) continue;
      pairs[static_cast<size_t>(h) * n_pairs + k] = make_int4(h, a, b >= 0 ? b : -1, 0);
      ++k;
    }
  }
  __syncthreads();
  for (int p = threadIdx.x; p < n_pairs; p += blockDim.x) {
    int4 it = pairs[static_cast<size_t>(h) * n_pairs + p];
    it.w = union_count(it.y, it.z);
    pairs[static_cast<size_t>(h) * n_pairs + p] = it;
  }
}

// Two work items per pair -- both halves of a split key list, or the whole list
// and an empty placeholder -- ordered longest first by a counting sort on the
// item length (order among equal lengths is arbitrary: it affects only the
// schedule, never a result).  One CTA.
constexpr int kLenBins = 1024;

__global__ void __launch_bounds__(1024)
k_make_items(const int4* __restrict__ pairs, int n_pairs, int shift, int4* __restrict__ items) {
  __shared__ int hist[kLenBins];
  __shared__ int base[kLenBins];
  __shared__ int wsum[32];
  for (int e = threadIdx.x; e < kLenBins; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  auto bin_of = [&](int len) { return kLenBins - 1 - min(kLenBins - 1, len >> shift); };  // long first
  for (int p = threadIdx.x; p < n_pairs; p += blockDim.x) {
    const int cnt = pairs[p].w;
    if (cnt >= kSplitMin) {
      atomicAdd(&hist[bin_of(cnt / 2)], 1);
      atomicAdd(&hist[bin_of(cnt - cnt / 2)], 1);
    } else {
      atomicAdd(&hist[bin_of(cnt)], 1);
      atomicAdd(&hist[kLenBins - 1], 1);
    }
  }
  __syncthreads();
  // exclusive scan of hist (1024 bins, one per thread)
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int v = threadIdx.x < kLenBins ? hist[threadIdx.x] : 0;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[wid] = incl;
  __syncthreads();
  int off = 0;
  for (int w = 0; w < wid; ++w) off += wsum[w];
  if (threadIdx.x < kLenBins) base[threadIdx.x] = off + incl - v;
  __syncthreads();
  for (int p = threadIdx.x; p < n_pairs; p += blockDim.x) {
    const int cnt = pairs[p].w;
    if (cnt >= kSplitMin) {
      const int hlf = cnt / 2;
      items[atomicAdd(&base[bin_of(hlf)], 1)] = make_int4(p, 0, 0, hlf);
      items[atomicAdd(&base[bin_of(cnt - hlf)], 1)] = make_int4(p, 1, hlf, cnt);
    } else {
      items[atomicAdd(&base[bin_of(cnt)], 1)] = make_int4(p, kWhole, 0, cnt);
      items[atomicAdd(&base[kLenBins - 1], 1)] = make_int4(p, kEmpty, 0, 0);
    }
  }
}

}  // namespace

size_t sparse_attn_ws_bytes(int H, int Nq, int d, int B) {
  const size_t n_pairs = static_cast<size_t>(H) * (((Nq + B - 1) / B + 1) / 2);
  auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  return al(n_pairs * sizeof(int4)) + al(2 * n_pairs * sizeof(int4)) +
         al(2 * n_pairs * kBM * d * sizeof(float)) + al(2 * n_pairs * kBM * 2 * sizeof(float));
}

bool make_tmap_bf16_2d(void* tmap, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer);

namespace {
template <int D>
void launch_attn_kernel(int grid, cudaStream_t st, const CUtensorMap& tq, const CUtensorMap& tk,
                        const CUtensorMap& tv, int mode, int Nq, int H, RowSource rs,
                        const uint32_t* blk_mask, int W, int n_qb, const int4* pairs,
                        const int4* items, Partials part, const float* gate, float* lin_ws,
                        void* out, float* o_branch, uint32_t* err) {
  const int smem = Cfg<D>::kSmem;
  cudaFuncSetAttribute(k_umma_attention<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  k_umma_attention<D><<<grid, kThreads, smem, st>>>(tq, tk, tv, mode, Nq, H, rs.L, rs, blk_mask, W,
                                                     n_qb, pairs, items, part, gate, lin_ws,
                                                     static_cast<__nv_bfloat16*>(out), o_branch, err);
}

wa_status make_maps(const void* q, int Nq, int H, int d, const RowSource& rs, CUtensorMap* tq,
                    CUtensorMap* tk, CUtensorMap* tv) {
  const int cols = H * d;
  const uint64_t key_rows = rs.page_ids ? static_cast<uint64_t>(rs.n_pages) * rs.page_rows
                                        : static_cast<uint64_t>(rs.L);
  if (!make_tmap_bf16_2d(tq, q, cols, Nq, static_cast<uint64_t>(cols) * 2, 64, 64) ||
      !make_tmap_bf16_2d(tk, rs.k, cols, key_rows, static_cast<uint64_t>(cols) * 2, 64, 64) ||
      !make_tmap_bf16_2d(tv, rs.v, cols, key_rows, static_cast<uint64_t>(cols) * 2, 64, 64))
    return set_error(WA_ERR_CUDA, "cuTensorMapEncodeTiled failed for the attention operands");
  return WA_OK;
}
}  // namespace

wa_status launch_linear_attention(const void* q, int Nq, int H, int d, RowSource lin, int B,
                                  const float* gate, float* lin_ws, float* o_lin, uint32_t* err,
                                  cudaStream_t st) {
  if (B != kBN) return set_error(WA_ERR_UNSUPPORTED, "bf16 attention needs B == 64");
  if (d != 64 && d != 128) return set_error(WA_ERR_UNSUPPORTED, "bf16 attention needs d in {64,128}");
  alignas(64) CUtensorMap tq, tk, tv;
  wa_status s = make_maps(q, Nq, H, d, lin, &tq, &tk, &tv);
  if (s != WA_OK) return s;
  const int n_qb = (Nq + B - 1) / B;
  const int grid = H * ((n_qb + 1) / 2);
  Partials none{nullptr, nullptr};
  if (d == 128)
    launch_attn_kernel<128>(grid, st, tq, tk, tv, 0, Nq, H, lin, nullptr, 0, n_qb, nullptr, nullptr,
                            none, gate, lin_ws, nullptr, o_lin, err);
  else
    launch_attn_kernel<64>(grid, st, tq, tk, tv, 0, Nq, H, lin, nullptr, 0, n_qb, nullptr, nullptr,
                           none, gate, lin_ws, nullptr, o_lin, err);
  return check_launch("linear attention");
}

namespace {
struct SparseLayout {
  int n_qb, n_kb, W, n_pairs;
  int4* pairs;
  int4* items;
  Partials part;
};
SparseLayout sparse_layout(void* scratch, int Nq, int H, int d, int B, int L) {
  SparseLayout s;
  s.n_qb = (Nq + B - 1) / B;
  s.n_kb = (L + B - 1) / B;
  s.W = (s.n_kb + 31) / 32;
  s.n_pairs = H * ((s.n_qb + 1) / 2);
  auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  char* p = static_cast<char*>(scratch);
  s.pairs = reinterpret_cast<int4*>(p);
  p += al(s.n_pairs * sizeof(int4));
  s.items = reinterpret_cast<int4*>(p);
  p += al(2 * static_cast<size_t>(s.n_pairs) * sizeof(int4));
  s.part.o = reinterpret_cast<float*>(p);
  p += al(2 * static_cast<size_t>(s.n_pairs) * kBM * d * sizeof(float));
  s.part.ml = reinterpret_cast<float*>(p);
  return s;
}
}  // namespace

wa_status launch_attn_worklist(int Nq, int H, int d, int B, int L, const uint32_t* blk_mask,
                               void* scratch, cudaStream_t st) {
  if (B != kBN) return set_error(WA_ERR_UNSUPPORTED, "bf16 attention needs B == 64");
  SparseLayout s = sparse_layout(scratch, Nq, H, d, B, L);
  if (s.W > kMaxW) return set_error(WA_ERR_UNSUPPORTED, "too many key blocks (max %d)", kMaxW * 32);
  k_pair_heads<<<H, 256, 0, st>>>(blk_mask, s.n_qb, s.W, s.pairs);
  int shift = 0;
  while ((s.n_kb >> shift) >= kLenBins) ++shift;
  k_make_items<<<1, 1024, 0, st>>>(s.pairs, s.n_pairs, shift, s.items);
  return check_launch("attention work list");
}

wa_status launch_attn_sparse(const void* q, int Nq, int H, int d, RowSource rs, int B,
                             const uint32_t* blk_mask, const float* gate, const float* lin_ws,
                             void* out, float* o_sp, void* scratch, uint32_t* err, cudaStream_t st) {
  if (B != kBN) return set_error(WA_ERR_UNSUPPORTED, "bf16 attention needs B == 64");
  if (d != 64 && d != 128) return set_error(WA_ERR_UNSUPPORTED, "bf16 attention needs d in {64,128}");
  SparseLayout s = sparse_layout(scratch, Nq, H, d, B, rs.L);
  if (s.W > kMaxW) return set_error(WA_ERR_UNSUPPORTED, "too many key blocks (max %d)", kMaxW * 32);
  alignas(64) CUtensorMap tq, tk, tv;
  wa_status e = make_maps(q, Nq, H, d, rs, &tq, &tk, &tv);
  if (e != WA_OK) return e;
  const int grid = 2 * s.n_pairs;
  float* lin_rw = const_cast<float*>(lin_ws);
  if (d == 128) {
    launch_attn_kernel<128>(grid, st, tq, tk, tv, 1, Nq, H, rs, blk_mask, s.W, s.n_qb, s.pairs, s.items,
                            s.part, gate, lin_rw, out, o_sp, err);
    k_combine<128><<<dim3(s.n_pairs, kBM / 32), 2 * 128, 0, st>>>(s.pairs, s.part, Nq, H, gate, lin_ws,
                                                                  static_cast<__nv_bfloat16*>(out), o_sp);
  } else {
    launch_attn_kernel<64>(grid, st, tq, tk, tv, 1, Nq, H, rs, blk_mask, s.W, s.n_qb, s.pairs, s.items,
                           s.part, gate, lin_rw, out, o_sp, err);
    k_combine<64><<<dim3(s.n_pairs, kBM / 32), 2 * 64, 0, st>>>(s.pairs, s.part, Nq, H, gate, lin_ws,
                                                                static_cast<__nv_bfloat16*>(out), o_sp);
  }
  return check_launch("sparse attention");
}

wa_status launch_sparse_attention(const void* q, int Nq, int H, int d, RowSource rs, int B,
                                  const uint32_t* blk_mask, const float* gate, const float* lin_ws,
                                  void* out, float* o_sp, void* scratch, uint32_t* err,
                                  cudaStream_t st, void* const* events) {
  wa_status e = launch_attn_worklist(Nq, H, d, B, rs.L, blk_mask, scratch, st);
  if (e != WA_OK) return e;
  if (events && events[6]) cudaEventRecord(static_cast<cudaEvent_t>(events[6]), st);
  return launch_attn_sparse(q, Nq, H, d, rs, B, blk_mask, gate, lin_ws, out, o_sp, scratch, err, st);
}

}  // namespace wa
