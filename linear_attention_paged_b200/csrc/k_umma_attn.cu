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
// possible (k_pair_heads).  When the pairs fill fewer than two waves of CTAs, a
// pair's key list is split in two work items whose partial results (unnormalised
// O, running max m, sum l per row) k_combine merges before applying the gate.
// Items run longest first.
//
// CTA = 384 threads, one CTA per SM.  The item's key blocks are listed once in
// shared memory; an iteration takes two consecutive blocks of the list (128 keys),
// so S = Q K^T is one M=128, N=128 MMA chain (with both operands in shared memory,
// N=64 chains ran at about two thirds of the tensor rate).  Roles:
//   warp 0  loads the K blocks, warp 2 the V blocks (TMA, 128-byte swizzle,
//           straight from the pool pages through a page table staged in shared
//           memory) into rings of 128-key slots (3 each);
//   warp 1  owns TMEM and issues the S MMAs with Q as the TMEM operand (the softmax
//           warps write the tile's Q rows into TMEM once), so an S MMA reads only K
//           from shared memory; warp 3 issues the P V MMAs.  TMEM holds one S
//           buffer, one P buffer, Q and two O accumulators.  S_{t+1} is issued as soon
//           as the softmax has loaded S_t into registers, so it runs during the
//           softmax of iteration t; P_t is stored once the P V MMAs of t-1 are done;
//   warps 4-7 / 8-11  two softmax groups, one per block of the iteration (S columns
//           0-63 / 64-127), one thread per TMEM lane (query row), each with its own
//           running max, sum and O accumulator, merged in the epilogue.  O is
//           rescaled in TMEM only when the running max grows by more than 2^8.
// Every wait is bounded in time.
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
constexpr int kIterKeys = 128;    // keys per iteration: two blocks of the tile's list
constexpr int kRingK = 3;         // 128-key slots of the K ring
constexpr int kRingV = 3;         // 128-key slots of the V ring
constexpr int kThreads = 384;     // warps 0-3: loads and MMA; 4-7 and 8-11: softmax
constexpr uint32_t kTmemCols = 512;
constexpr int kColS = 0;          // the S buffer: 128 fp32 columns
constexpr int kColP = 128;        // P (bf16 pairs): group g at columns 128 + 32g
constexpr int kColQ = 192;        // Q (bf16 pairs): d/2 columns
constexpr int kColO = 256;        // O accumulators: group g at columns 256 + g*d
constexpr int kMaxW = 256;        // up to 8192 key blocks
constexpr int kMaxList = kMaxW * 32;
constexpr int kMaxPages = 64;     // page-table entries staged in shared memory

// Key-list entries (16 bits): block index in bits 0-12, bit 13 / bit 14 set when
// the tile's first / second query block kept the block; kNoBlock pads an odd list.
constexpr uint32_t kSel0 = 1u << 13, kSel1 = 1u << 14;
constexpr uint32_t kNoBlock = 0xFFFFu;

// item.y values
constexpr int kWhole = -1;        // the whole key list; writes the final output
constexpr int kEmpty = -2;        // placeholder: nothing to do

template <int D>
struct Cfg {
  static constexpr int kPanels = D / 64;                 // 128-byte column panels
  static constexpr int kBlockBytes = kBN * D * 2;         // one 64-key block of K or V
  static constexpr int kSlotBytes = 2 * kBlockBytes;      // a 128-key slot
  static constexpr int kPanelBytes = kIterKeys * 128;     // one panel of a slot: 128 rows x 128 B
  static constexpr int kSmem = (kRingK + kRingV) * kSlotBytes + 1024;  // + alignment slack
  static constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kIterKeys, false, false);
  static constexpr uint32_t kIdescO = idesc_bf16_f32(kBM, D, false, true);
  static constexpr int kQWarps = 4 * (D / 64);            // softmax warps that write Q to TMEM
};

struct Shared {
  uint64_t q_full;        // Q rows in TMEM (one arrival per writing softmax warp)
  uint64_t k_full[kRingK], k_empty[kRingK];
  uint64_t v_full[kRingV], v_empty[kRingV];
  uint64_t s_full;        // S_t computed
  uint64_t s_free;        // S_t loaded by all eight softmax warps
  uint64_t p_full[2];     // P_t of group g stored, one arrival per warp of the group
  uint64_t o_done;        // O_g += P_t V_t complete (both groups)
  uint64_t drain[2];      // abort path: every MMA of issuer 0 (S) / 1 (P V) complete
  uint64_t wait_ns;       // bound of every wait (wa_set_wait_limit_ns)
  uint32_t tmem_base;
  int abort_flag;
  int scan[8];
  int page_row0[kMaxPages];  // first pool row of each page of the key sequence
  float xch[2][2][kBM];   // epilogue exchange of (m, l) between the two groups
  uint16_t list[kMaxList + 2];  // the item's key blocks, two per iteration
};

// Bounded wait that also gives up when another role has aborted.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Shared& sh,
                                         uint32_t* err) {
  const int r = mbar_wait_bounded(bar, parity, &sh.abort_flag, sh.wait_ns);
  if (r == kWaitTimeout) atomicOr(err, WA_DEVERR_TIMEOUT);
  return r == kWaitOk;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// One softmax pass over a 64-column half row held in r: p = 2^(s * scale_log2 - m)
// packed to bf16 pairs in pk, the sum of p in lsum and (kMax) the raw row maximum.
template <bool kMax>
__device__ __forceinline__ void softmax_pass(const uint32_t (&r)[64], float2 sc2, float2 nm2,
                                             uint32_t (&pk)[32], float& lsum, float& mraw) {
  float2 acc2[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) acc2[e] = make_float2(0.f, 0.f);
  float mx8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) mx8[e] = -INFINITY;
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const float2 x = make_float2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
    if (kMax) mx8[e & 7] = max3f(mx8[e & 7], x.x, x.y);
    const float2 y = __ffma2_rn(x, sc2, nm2);
    const float2 pp = make_float2(ex2(y.x), ex2(y.y));
    acc2[e & 3] = __fadd2_rn(acc2[e & 3], pp);
    pk[e] = pack_bf16x2(pp.x, pp.y);
  }
  const float2 a01 = __fadd2_rn(acc2[0], acc2[1]), a23 = __fadd2_rn(acc2[2], acc2[3]);
  const float2 a03 = __fadd2_rn(a01, a23);
  lsum = a03.x + a03.y;
  if (kMax)
    mraw = max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
}

__device__ __forceinline__ float rowmax64(const uint32_t (&r)[64]) {
  float mx8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(__uint_as_float(r[e]), __uint_as_float(r[8 + e]));
#pragma unroll
  for (int c = 16; c < 64; c += 16)
#pragma unroll
    for (int e = 0; e < 8; ++e)
      mx8[e] = max3f(mx8[e], __uint_as_float(r[c + e]), __uint_as_float(r[c + 8 + e]));
  return max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
}

__device__ __forceinline__ int page_row0(const RowSource& rs, int i, uint32_t* err) {
  int pg = rs.page_ids[i];
  if (pg < 0 || pg >= rs.n_pages) { atomicOr(err, WA_DEVERR_PAGE_ID); pg = 0; }
  return pg * rs.page_rows;
}

// First pool row of key block j: contiguous keys, or through the page table (staged
// in shared memory when it is short, so the loads never wait on global memory).
__device__ __forceinline__ int key_row(const RowSource& rs, const int* staged, int bpp, int j,
                                       uint32_t* err) {
  if (!rs.page_ids) return j * kBN;
  const int i = j / bpp;
  return (staged ? staged[i] : page_row0(rs, i, err)) + (j - i * bpp) * kBN;
}

struct Partials {
  float* o;    // [slots][128][d]  unnormalised O
  float* ml;   // [slots][128][2]  running max (log2 units) and sum
};

// One CTA per SM.  An iteration covers two consecutive blocks (ja, jb) of the
// tile's key list: S = Q K^T is one N=128 MMA chain with Q read from TMEM; K and V
// of the two blocks sit in one 128-key slot of their rings (the second half unused
// when the list is odd).
// Softmax group 0 (warps 4-7) owns the blocks at even list positions (S columns
// 0-63), group 1 (warps 8-11) those at odd positions (columns 64-127): each keeps
// its own running max and sum and its own O accumulator, so the groups never
// synchronise inside the loop; the epilogue merges the two (O, m, l) states.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
k_umma_attention(const __nv_bfloat16* __restrict__ q, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmK2,
                 const __grid_constant__ CUtensorMap tmV2, int mode, int Nq, int H, int Lk,
                 RowSource rs, const uint32_t* __restrict__ blk_mask, int W, int n_qb,
                 const int4* __restrict__ pairs, const int4* __restrict__ items, Partials part,
                 const float* __restrict__ gate, float lin_sign, float* __restrict__ lin_ws,
                 __nv_bfloat16* __restrict__ out, float* __restrict__ o_branch, uint32_t* err,
                 uint64_t wait_ns) {
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
  auto Ks = [&](int s) { return tiles + s * C::kSlotBytes; };
  auto Vs = [&](int s) { return tiles + (kRingK + s) * C::kSlotBytes; };

  if (tid == 0) {
    mbar_init(&sh.q_full, C::kQWarps);
    for (int s = 0; s < kRingK; ++s) { mbar_init(&sh.k_full[s], 1); mbar_init(&sh.k_empty[s], 1); }
    for (int s = 0; s < kRingV; ++s) { mbar_init(&sh.v_full[s], 1); mbar_init(&sh.v_empty[s], 1); }
    mbar_init(&sh.s_full, 1);
    mbar_init(&sh.s_free, 8);
    mbar_init(&sh.p_full[0], 4);
    mbar_init(&sh.p_full[1], 4);
    mbar_init(&sh.o_done, 1);
    mbar_init(&sh.drain[0], 1);
    mbar_init(&sh.drain[1], 1);
    sh.wait_ns = wait_ns;
    sh.abort_flag = 0;
    fence_mbar_init();
  }
  // The item's key blocks, positions [k0, k1) of the tile's list, with the
  // selection bits of both query blocks: one scan over the mask words (at most
  // kMaxW, one per thread).
  const int n_blk = k1 - k0;
  if (mode == 0) {
    for (int q = tid; q < n_blk; q += kThreads)
      sh.list[q] = static_cast<uint16_t>((k0 + q) | kSel0 | kSel1);
  } else {
    uint32_t ma = 0u, mb = 0u;
    if (tid < W) {
      ma = blk_mask[(static_cast<size_t>(h) * n_qb + i0) * W + tid];
      if (i1 >= 0) mb = blk_mask[(static_cast<size_t>(h) * n_qb + i1) * W + tid];
    }
    const uint32_t un = ma | mb;
    const int c = __popc(un);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31 && warp < 8) sh.scan[warp] = incl;
    __syncthreads();
    if (tid < W) {
      int pos = incl - c;
      for (int w = 0; w < warp; ++w) pos += sh.scan[w];
      for (uint32_t bits = un; bits != 0u; bits &= bits - 1u, ++pos) {
        if (pos < k0 || pos >= k1) continue;
        const int b = __ffs(bits) - 1;
        sh.list[pos - k0] = static_cast<uint16_t>((tid * 32 + b) | (((ma >> b) & 1u) ? kSel0 : 0u) |
                                                  (((mb >> b) & 1u) ? kSel1 : 0u));
      }
    }
  }
  if (tid == 0) sh.list[n_blk] = static_cast<uint16_t>(kNoBlock);
  // page-table entries cover the first segment only (rs.L rows)
  const int n_ids = rs.page_ids ? (rs.L + rs.page_rows - 1) / rs.page_rows : 0;
  const int* staged = (n_ids > 0 && n_ids <= kMaxPages) ? sh.page_row0 : nullptr;
  if (staged && tid < n_ids) sh.page_row0[tid] = page_row0(rs, tid, err);
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sh.tmem_base;
  const int n_it = (n_blk + 1) / 2;
  const uint32_t* list2 = reinterpret_cast<const uint32_t*>(sh.list);  // entries 2t, 2t+1
  const bool odd_tail = (n_blk & 1) != 0;   // the last iteration holds one block
  const int bpp = rs.page_ids ? rs.page_rows / kBN : 0;
  int issued = 0;   // producers: iterations whose loads were issued (for the abort drain)

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ producers:
    // warp 0 loads the K blocks, warp 2 the V blocks
    if (lane == 0) {
      const bool isK = warp == 0;
      const CUtensorMap* tm = isK ? &tmK : &tmV;
      const CUtensorMap* tm2 = isK ? &tmK2 : &tmV2;   // the chunk's own keys (second segment)
      const int n_kb1 = rs.k2 ? rs.L / kBN : INT_MAX;
      prefetch_tmap(tm);
      if (rs.k2) prefetch_tmap(tm2);
      const int ring = isK ? kRingK : kRingV;
      for (int t = 0; t < n_it; ++t) {
        const int s = t % ring;
        uint64_t* empty = isK ? &sh.k_empty[s] : &sh.v_empty[s];
        uint64_t* full = isK ? &sh.k_full[s] : &sh.v_full[s];
        if (!wait_bar(empty, ((t / ring) & 1) ^ 1, sh, err)) break;
        const uint32_t wrd = list2[t];
        const int ja = static_cast<int>(wrd & 0x1FFFu);
        const int jb = (wrd >> 16) == kNoBlock ? -1 : static_cast<int>((wrd >> 16) & 0x1FFFu);
        uint8_t* dst = isK ? Ks(s) : Vs(s);
        mbar_arrive_expect_tx(full, (jb >= 0 ? 2 : 1) * C::kBlockBytes);
        const bool a2 = ja >= n_kb1;
        const int ra = a2 ? (ja - n_kb1) * kBN : key_row(rs, staged, bpp, ja, err);
        for (int p = 0; p < C::kPanels; ++p)
          tma_load_2d(dst + p * C::kPanelBytes, a2 ? tm2 : tm, full, h * D + p * 64, ra);
        if (jb >= 0) {
          const bool b2 = jb >= n_kb1;
          const int rb = b2 ? (jb - n_kb1) * kBN : key_row(rs, staged, bpp, jb, err);
          for (int p = 0; p < C::kPanels; ++p)
            tma_load_2d(dst + p * C::kPanelBytes + kBN * 128, b2 ? tm2 : tm, full, h * D + p * 64, rb);
        }
        issued = t + 1;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S issuer
    if (lane == 0) {
      bool ok = wait_bar(&sh.q_full, 0, sh, err);
      tc_fence_after();
      for (int t = 0; ok && t < n_it; ++t) {
        // S_t = Q K_t^T (N = 128, Q from TMEM) once all softmax warps hold S_{t-1}
        // in registers
        const int s = t % kRingK;
        if (!wait_bar(&sh.k_full[s], (t / kRingK) & 1, sh, err)) break;
        if (t >= 1 && !wait_bar(&sh.s_free, (t - 1) & 1, sh, err)) break;
        tc_fence_after();
        const uint32_t k_base = smem_u32(Ks(s));
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t bdesc = smem_desc_sw128(k_base + (k >> 2) * C::kPanelBytes + (k & 3) * 32, 16, 1024);
          mma_ts(tbase + kColS, tbase + kColQ + k * 8, bdesc, C::kIdescS, k > 0 ? 1u : 0u);
        }
        mma_commit(&sh.k_empty[s]);
        mma_commit(&sh.s_full);
      }
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ P V issuer:
    // O_g += P_g V_g for each group's block of iteration u, P read from TMEM.  A
    // second issuing thread, so that S MMAs keep the tensor pipe busy while this one
    // waits for the softmax (an MMA's issue blocks behind the one executing).
    if (lane == 0) {
      for (int u = 0; u < n_it; ++u) {
        const int vs = u % kRingV;
        if (!wait_bar(&sh.v_full[vs], (u / kRingV) & 1, sh, err)) break;
        // group 1 has no block in an odd list's last iteration
        const int n_grp = (u == n_it - 1 && odd_tail) ? 1 : 2;
        bool ok = true;
        for (int g = 0; g < n_grp; ++g) {
          if (!wait_bar(&sh.p_full[g], u & 1, sh, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t v_base = smem_u32(Vs(vs)) + g * (kBN * 128);
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            const uint64_t bdesc = smem_desc_sw128(v_base + kk * 2048, C::kPanelBytes, 1024);
            mma_ts(tbase + kColO + g * D, tbase + kColP + g * (kBN / 2) + kk * 8, bdesc,
                   C::kIdescO, (u > 0 || kk > 0) ? 1u : 0u);
          }
        }
        if (!ok) break;
        mma_commit(&sh.v_empty[vs]);
        mma_commit(&sh.o_done);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int g = (warp - 4) >> 2;                  // softmax group
    const int q4 = warp & 3;                        // TMEM lane quarter of this warp
    const int row = q4 * 32 + lane;                 // TMEM lane = tile row
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t o_col = kColO + g * D;
    const int half = row >> 6;
    const int ib = half ? i1 : i0;
    const int qrow = ib * 64 + (row & 63);
    const bool row_valid = ib >= 0 && qrow < Nq;
    const uint32_t sel_bit = half ? kSel1 : kSel0;   // the same for the whole warp
    const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
    const float2 sc2 = make_float2(scale_log2, scale_log2);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    // one arrival per warp once all its lanes' TMEM accesses are complete
    auto arrive_warp = [&](uint64_t* bar) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    // Wait until the P V MMAs of iteration t-1 are done: P_t may then overwrite
    // P_{t-1} and O_g is stable for a rescale.  Every softmax warp waits once per
    // iteration, and P V of t needs this warp's P_t, so at this wait the barrier has
    // completed t-1 or t phases: its parity is unambiguous.
    auto wait_pv = [&](int t) -> bool {
      if (t == 0) return true;
      const bool w = __all_sync(0xffffffffu, wait_bar(&sh.o_done, (t - 1) & 1, sh, err));
      tc_fence_after();
      return w;
    };
    // The tile's Q rows into TMEM as bf16 pairs (the S MMA's A operand): one thread
    // per row, 64 elements per group; rows past Nq or of a missing second block are 0.
    if (g < D / 64) {
      uint32_t qv[32];
      if (row_valid) {
        const uint4* src =
            reinterpret_cast<const uint4*>(q + (static_cast<size_t>(qrow) * H + h) * D + g * 64);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint4 x = src[e];
          qv[4 * e] = x.x; qv[4 * e + 1] = x.y; qv[4 * e + 2] = x.z; qv[4 * e + 3] = x.w;
        }
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) qv[c] = 0u;
      }
      tmem_st32(tbase + lane_base + kColQ + g * 32, qv);
      tmem_wait_st();
      arrive_warp(&sh.q_full);
    }
    const uint32_t s_addr = tbase + lane_base + kColS + g * kBN;
    const uint32_t p_addr = tbase + lane_base + kColP + g * (kBN / 2);
    int t = 0;
    for (; t < n_it; ++t) {
      const uint32_t e = (list2[t] >> (16 * g)) & 0xFFFFu;
      if (!__all_sync(0xffffffffu, wait_bar(&sh.s_full, t & 1, sh, err))) { ok = false; break; }
      if (e == kNoBlock || !(e & sel_bit)) {
        // no block (group 1 in an odd list's last iteration), or this warp's query
        // block did not keep it: S is not read, P = 0, the state is unchanged
        arrive_warp(&sh.s_free);
        if (!wait_pv(t)) { ok = false; break; }
        if (e != kNoBlock) {
          uint32_t z[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) z[c] = 0u;
          tmem_st32(p_addr, z);
          tmem_wait_st();
          arrive_warp(&sh.p_full[g]);
        }
        continue;
      }
      tc_fence_after();
      uint32_t r[64];
      tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
      tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
      tmem_wait_ld();
      arrive_warp(&sh.s_free);   // S_{t+1} may now overwrite the buffer
      const int valid = min(kBN, Lk - static_cast<int>(e & 0x1FFFu) * kBN);
      const bool ragged = valid < kBN;   // the key sequence's last, partial block
      if (ragged) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= valid) r[c] = __float_as_uint(-INFINITY);
      }
      // A row's first kept block sets its reference max before any exponential;
      // afterwards the pass runs with the current (possibly stale) max and finds the
      // new one alongside, and is redone only if the max grew by more than 2^8.
      if (__any_sync(0xffffffffu, m_run == -INFINITY)) {
        const float m0 = rowmax64(r) * scale_log2;   // scale_log2 > 0: max commutes
        if (m_run == -INFINITY) m_run = m0;
      }
      uint32_t pk[32];
      float lsum, mraw;
      float2 nm2 = make_float2(-m_run, -m_run);
      softmax_pass<true>(r, sc2, nm2, pk, lsum, mraw);
      const float mx = mraw * scale_log2;
      float factor = 1.f;
      const bool resc = mx > m_run + 8.f;
      if (resc) {
        factor = ex2(m_run - mx);
        m_run = mx;
        nm2 = make_float2(-m_run, -m_run);
        softmax_pass<false>(r, sc2, nm2, pk, lsum, mraw);
      }
      l_run = l_run * factor + lsum;
      if (!wait_pv(t)) { ok = false; break; }
      if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tbase + lane_base + o_col + c0, o);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * factor);
          tmem_st32(tbase + lane_base + o_col + c0, o);
        }
      }
      tmem_st32(p_addr, pk);
      tmem_wait_st();
      arrive_warp(&sh.p_full[g]);
    }
    // the last iteration's P V MMAs
    if (ok && t > 0) ok = wait_pv(t);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    // merge the groups' states: M = max(m_0, m_1), w_g = 2^(m_g - M); each group then
    // writes half of the columns of  w_0 O_0 + w_1 O_1  and  l = w_0 l_0 + w_1 l_1
    sh.xch[0][g][row] = m_run;
    sh.xch[1][g][row] = l_run;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    const float m_o = sh.xch[0][g ^ 1][row], l_o = sh.xch[1][g ^ 1][row];
    const float m0 = g ? m_o : m_run, m1 = g ? m_run : m_o;
    const float l0 = g ? l_o : l_run, l1 = g ? l_run : l_o;
    const float M = fmaxf(m0, m1);
    const float w0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - M);
    const float w1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - M);
    const float l_tot = w0 * l0 + w1 * l1;
    // O_1 exists only if the item has at least two blocks
    const bool have0 = ok && n_blk >= 1, have1 = ok && n_blk >= 2;
    auto merged = [&](int c0, float (&v)[32]) {
      uint32_t a[32], b[32];
      if (have0) tmem_ld32(tbase + lane_base + kColO + c0, a);
      if (have1) tmem_ld32(tbase + lane_base + kColO + D + c0, b);
      if (have0 || have1) tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e)
        v[e] = (have0 ? w0 * __uint_as_float(a[e]) : 0.f) + (have1 ? w1 * __uint_as_float(b[e]) : 0.f);
    };
    const int cbeg = g * (D / 2), cend = cbeg + D / 2;
    if (kind >= 0) {
      // one half of a split key list: hand the unnormalised state to k_combine
      float* po = part.o + (static_cast<size_t>(slot) * kBM + row) * D;
#pragma unroll
      for (int c0 = cbeg; c0 < cend; c0 += 32) {
        float v[32];
        merged(c0, v);
        float4* p4 = reinterpret_cast<float4*>(po + c0);
#pragma unroll
        for (int e = 0; e < 8; ++e) p4[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
      }
      if (g == 0)
        *reinterpret_cast<float2*>(part.ml + (static_cast<size_t>(slot) * kBM + row) * 2) =
            make_float2(M, l_tot);
    } else {
      const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
      // mode 1: sg = sigmoid(g); mode 0: the linear branch's weight sigmoid(lin_sign * x)
      // (x = g and lin_sign = -1 for 1 - sigmoid(g); x = g_lin and +1 for two gates)
      float sg = 0.f;
      size_t obase = 0;
      if (row_valid) {
        const float gt = gate[static_cast<size_t>(qrow) * H + h];
        sg = 1.f / (1.f + expf(mode == 0 ? -lin_sign * gt : -gt));
        obase = static_cast<size_t>(qrow) * H * D + static_cast<size_t>(h) * D;
      }
#pragma unroll
      for (int c0 = cbeg; c0 < cend; c0 += 32) {
        float v[32];
        merged(c0, v);
        if (!row_valid) continue;
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] *= inv;
        if (o_branch) {
          float4* ob = reinterpret_cast<float4*>(o_branch + obase + c0);
#pragma unroll
          for (int e = 0; e < 8; ++e) ob[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
        }
        if (mode == 0) {
          float4* lw = reinterpret_cast<float4*>(lin_ws + obase + c0);
          const float a = sg;
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
  if (sh.abort_flag) {
    // A role gave up: before TMEM is freed and the shared memory handed to another
    // CTA, wait (bounded, whatever the flag says) for this CTA's own asynchronous
    // work -- the loads each producer issued into its ring (at most the last `ring`
    // can still be outstanding) and every MMA of both issuers (a commit to a drain
    // barrier arrives once all of the issuing thread's earlier MMAs are complete).
    int never = 0;
    if ((warp == 0 || warp == 2) && lane == 0) {
      const int ring = warp == 0 ? kRingK : kRingV;
      for (int t = issued > ring ? issued - ring : 0; t < issued; ++t) {
        uint64_t* full = warp == 0 ? &sh.k_full[t % ring] : &sh.v_full[t % ring];
        if (mbar_wait_bounded(full, (t / ring) & 1, &never, sh.wait_ns) == kWaitTimeout)
          atomicOr(err, WA_DEVERR_TIMEOUT);
      }
    } else if ((warp == 1 || warp == 3) && lane == 0) {
      uint64_t* bar = &sh.drain[warp == 1 ? 0 : 1];
      mma_commit(bar);
      if (mbar_wait_bounded(bar, 0, &never, sh.wait_ns) == kWaitTimeout) atomicOr(err, WA_DEVERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
  }
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
k_combine(const int4* __restrict__ pairs, Partials part, int Nq, int H, int split_min,
          const float* __restrict__ gate, const float* __restrict__ lin_ws,
          __nv_bfloat16* __restrict__ out, float* __restrict__ o_branch) {
  constexpr int kSeg = D / 16;                 // 16-column segments per row
  const int4 pr = pairs[blockIdx.x];
  if (pr.w < split_min) return;                // written whole by the attention kernel
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

constexpr int kPairThreads = 1024;

__global__ void __launch_bounds__(kPairThreads)
k_pair_heads(const uint32_t* __restrict__ mask, int n_qb, int W, int4* __restrict__ pairs) {
  __shared__ uint16_t dist[kMaxPairTable * kMaxPairTable];
  __shared__ uint32_t ms[kMaxPairMaskWords];
  __shared__ int partner[kMaxPairTable];
  __shared__ int nn[kMaxPairTable];
  const int h = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, n_warps = blockDim.x >> 5;
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
  // symmetric-difference distances, each unordered pair once
  const int n_tri = n_qb * (n_qb - 1) / 2;
  for (int e = threadIdx.x; e < n_tri; e += blockDim.x) {
    // e -> (a, b), a < b, row-major over the strict upper triangle
    int a = static_cast<int>((2 * n_qb - 1 - sqrtf(static_cast<float>((2 * n_qb - 1) * (2 * n_qb - 1) - 8 * e))) * 0.5f);
    if (a < 0) a = 0;
    while (a > 0 && a * (2 * n_qb - a - 1) / 2 > e) --a;
    while ((a + 1) * (2 * n_qb - a - 2) / 2 <= e) ++a;
    const int b = e - a * (2 * n_qb - a - 1) / 2 + a + 1;
    int c = 0;
    for (int w = 0; w < W; ++w) c += __popc(m[a * W + w] ^ m[b * W + w]);
    const uint16_t dv = static_cast<uint16_t>(min(c, 65535));
    dist[a * n_qb + b] = dv;
    dist[b * n_qb + a] = dv;
  }
  for (int a = threadIdx.x; a < n_qb; a += blockDim.x) partner[a] = -2;   // -2: unpaired
  __syncthreads();
  // rounds of mutual nearest neighbours among the unpaired blocks; a warp finds the
  // nearest of one block (ties: the lower index)
  for (int round = 0; round < n_qb; ++round) {
    for (int a = warp; a < n_qb; a += n_warps) {
      unsigned long long best = ~0ull;            // (distance << 32) | index
      if (partner[a] == -2)
        for (int b = lane; b < n_qb; b += 32)
          if (b != a && partner[b] == -2)
            best = min(best, (static_cast<unsigned long long>(dist[a * n_qb + b]) << 32) | b);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) best = min(best, __shfl_xor_sync(0xffffffffu, best, o));
      if (lane == 0) nn[a] = best == ~0ull ? -1 : static_cast<int>(best & 0xffffffffu);
    }
    __syncthreads();
    int paired = 0;
    for (int a = threadIdx.x; a < n_qb; a += blockDim.x) {
      const int b = nn[a];
      if (b > a && nn[b] == a) { partner[a] = b; partner[b] = a; paired = 1; }
    }
    // barrier and vote in one: every thread sees the same answer, and no shared flag
    // is reset while a slower thread may still be reading it
    if (!__syncthreads_or(paired)) break;
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
// and an empty placeholder (placed after every real item, so that a launch over the
// first n_pairs items covers them all) -- ordered longest first over all heads, by a counting
// sort (order among equal lengths is arbitrary: it affects only the schedule, never a
// result).  One CTA.  Ordering by head group first (so that a group's keys and values
// stay in L2 while its items run) halved the launch's DRAM reads but made the sparse
// branch 3.6 % slower at the one-layer shape and 12 % slower on the stress inputs: the
// heads' lists differ in length, and the longest then run last.
constexpr int kLenBins = 1024;

__global__ void __launch_bounds__(1024)
k_make_items(const int4* __restrict__ pairs, int n_pairs, int shift, int split_min,
             int4* __restrict__ items) {
  __shared__ int hist[kLenBins];
  __shared__ int base[kLenBins];
  __shared__ int wsum[32];
  for (int e = threadIdx.x; e < kLenBins; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  // long first: the longest lists in the lowest bins; the last bin holds only the
  // empty placeholders, so every real item comes before them
  auto bin_of = [&](int len) { return kLenBins - 2 - min(kLenBins - 2, len >> shift); };
  for (int p = threadIdx.x; p < n_pairs; p += blockDim.x) {
    const int cnt = pairs[p].w;
    if (cnt >= split_min) {
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
    if (cnt >= split_min) {
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
void launch_attn_kernel(int grid, cudaStream_t st, const void* q, const CUtensorMap& tk,
                        const CUtensorMap& tv, const CUtensorMap& tk2, const CUtensorMap& tv2,
                        int mode, int Nq, int H, RowSource rs,
                        const uint32_t* blk_mask, int W, int n_qb, const int4* pairs,
                        const int4* items, Partials part, const float* gate, float lin_sign,
                        float* lin_ws, void* out, float* o_branch, uint32_t* err) {
  const int smem = Cfg<D>::kSmem;
  cudaFuncSetAttribute(k_umma_attention<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  k_umma_attention<D><<<grid, kThreads, smem, st>>>(static_cast<const __nv_bfloat16*>(q), tk, tv, tk2, tv2, mode, Nq, H, rs.L + rs.L2, rs,
                                                     blk_mask, W,
                                                     n_qb, pairs, items, part, gate, lin_sign, lin_ws,
                                                     static_cast<__nv_bfloat16*>(out), o_branch, err,
                                                     wait_limit_ns());
}

// The keys/values of the first segment (pool pages or a contiguous buffer) and,
// when the row source has one, of the second (tk2/tv2 repeat tk/tv otherwise).
wa_status make_maps(int H, int d, const RowSource& rs, CUtensorMap* tk, CUtensorMap* tv,
                    CUtensorMap* tk2, CUtensorMap* tv2) {
  const int cols = H * d;
  const uint64_t key_rows = rs.page_ids ? static_cast<uint64_t>(rs.n_pages) * rs.page_rows
                                        : static_cast<uint64_t>(rs.L);
  const uint64_t rb = static_cast<uint64_t>(cols) * 2;
  if (!make_tmap_bf16_2d(tk, rs.k, cols, key_rows, rb, 64, 64) ||
      !make_tmap_bf16_2d(tv, rs.v, cols, key_rows, rb, 64, 64))
    return set_error(WA_ERR_CUDA, "cuTensorMapEncodeTiled failed for the attention operands");
  if (rs.k2) {
    if (!make_tmap_bf16_2d(tk2, rs.k2, cols, rs.L2, rb, 64, 64) ||
        !make_tmap_bf16_2d(tv2, rs.v2, cols, rs.L2, rb, 64, 64))
      return set_error(WA_ERR_CUDA, "cuTensorMapEncodeTiled failed for the chunk's keys");
  } else {
    *tk2 = *tk;
    *tv2 = *tv;
  }
  return WA_OK;
}
}  // namespace

wa_status launch_linear_attention(const void* q, int Nq, int H, int d, RowSource lin, int B,
                                  const float* gate, const float* gate_lin, float* lin_ws,
                                  float* o_lin, uint32_t* err, cudaStream_t st) {
  if (B != kBN) return set_error(WA_ERR_UNSUPPORTED, "bf16 attention needs B == 64");
  if (d != 64 && d != 128) return set_error(WA_ERR_UNSUPPORTED, "bf16 attention needs d in {64,128}");
  alignas(64) CUtensorMap tk, tv, tk2, tv2;
  wa_status s = make_maps(H, d, lin, &tk, &tv, &tk2, &tv2);
  if (s != WA_OK) return s;
  const int n_qb = (Nq + B - 1) / B;
  const int grid = H * ((n_qb + 1) / 2);
  Partials none{nullptr, nullptr};
  if (d == 128)
    launch_attn_kernel<128>(grid, st, q, tk, tv, tk2, tv2, 0, Nq, H, lin, nullptr, 0, n_qb, nullptr, nullptr,
                            none, gate_lin ? gate_lin : gate, gate_lin ? 1.f : -1.f, lin_ws, nullptr,
                            o_lin, err);
  else
    launch_attn_kernel<64>(grid, st, q, tk, tv, tk2, tv2, 0, Nq, H, lin, nullptr, 0, n_qb, nullptr, nullptr,
                           none, gate_lin ? gate_lin : gate, gate_lin ? 1.f : -1.f, lin_ws, nullptr,
                           o_lin, err);
  return check_launch("linear attention");
}

namespace {
struct SparseLayout {
  int n_qb, n_kb, W, n_pairs;
  int4* pairs;
  int4* items;
  Partials part;
};
// Key lists are split in two (and merged by k_combine) only when the pairs fill
// fewer than two waves of one CTA per SM: with more, the longest-first order
// already balances the SMs and a split only adds partial-state traffic.
int split_min_for(int n_pairs) {
  static int n_sm = 0;
  if (n_sm == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm < 1)
      n_sm = 148;
  }
  return n_pairs >= 2 * n_sm ? INT_MAX : 8;
}

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
  k_pair_heads<<<H, kPairThreads, 0, st>>>(blk_mask, s.n_qb, s.W, s.pairs);
  int shift = 0;
  while ((s.n_kb >> shift) >= kLenBins) ++shift;
  k_make_items<<<1, 1024, 0, st>>>(s.pairs, s.n_pairs, shift, split_min_for(s.n_pairs), s.items);
  return check_launch("attention work list");
}

wa_status launch_attn_sparse(const void* q, int Nq, int H, int d, RowSource rs, int B,
                             const uint32_t* blk_mask, const float* gate, const float* lin_ws,
                             void* out, float* o_sp, void* scratch, uint32_t* err, cudaStream_t st) {
  if (B != kBN) return set_error(WA_ERR_UNSUPPORTED, "bf16 attention needs B == 64");
  if (d != 64 && d != 128) return set_error(WA_ERR_UNSUPPORTED, "bf16 attention needs d in {64,128}");
  if (rs.k2 && rs.L % kBN != 0)
    return set_error(WA_ERR_UNSUPPORTED, "a second key segment needs the first to fill whole blocks");
  SparseLayout s = sparse_layout(scratch, Nq, H, d, B, rs.L + rs.L2);
  if (s.W > kMaxW) return set_error(WA_ERR_UNSUPPORTED, "too many key blocks (max %d)", kMaxW * 32);
  alignas(64) CUtensorMap tk, tv, tk2, tv2;
  wa_status e = make_maps(H, d, rs, &tk, &tv, &tk2, &tv2);
  if (e != WA_OK) return e;
  float* lin_rw = const_cast<float*>(lin_ws);
  const int split_min = split_min_for(s.n_pairs);
  // nothing split: the first n_pairs items are the whole lists and no CTA combines
  const bool split = split_min != INT_MAX;
  const int grid = split ? 2 * s.n_pairs : s.n_pairs;
  if (d == 128) {
    launch_attn_kernel<128>(grid, st, q, tk, tv, tk2, tv2, 1, Nq, H, rs, blk_mask, s.W, s.n_qb, s.pairs, s.items,
                            s.part, gate, 0.f, lin_rw, out, o_sp, err);
    if (split)
      k_combine<128><<<dim3(s.n_pairs, kBM / 32), 2 * 128, 0, st>>>(s.pairs, s.part, Nq, H, split_min, gate,
                                                                    lin_ws, static_cast<__nv_bfloat16*>(out), o_sp);
  } else {
    launch_attn_kernel<64>(grid, st, q, tk, tv, tk2, tv2, 1, Nq, H, rs, blk_mask, s.W, s.n_qb, s.pairs, s.items,
                           s.part, gate, 0.f, lin_rw, out, o_sp, err);
    if (split)
      k_combine<64><<<dim3(s.n_pairs, kBM / 32), 2 * 64, 0, st>>>(s.pairs, s.part, Nq, H, split_min, gate,
                                                                  lin_ws, static_cast<__nv_bfloat16*>(out), o_sp);
  }
  return check_launch("sparse attention");
}

wa_status launch_sparse_attention(const void* q, int Nq, int H, int d, RowSource rs, int B,
                                  const uint32_t* blk_mask, const float* gate, const float* lin_ws,
                                  void* out, float* o_sp, void* scratch, uint32_t* err,
                                  cudaStream_t st, void* const* events) {
  wa_status e = launch_attn_worklist(Nq, H, d, B, rs.L + rs.L2, blk_mask, scratch, st);
  if (e != WA_OK) return e;
  if (events && events[6]) cudaEventRecord(static_cast<cudaEvent_t>(events[6]), st);
  return launch_attn_sparse(q, Nq, H, d, rs, B, blk_mask, gate, lin_ws, out, o_sp, scratch, err, st);
}

}  // namespace wa
