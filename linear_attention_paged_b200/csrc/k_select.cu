// k_select.cu -- the index-producing steps of the HSA decode step:
//   S0 prompt-level retrieval (cosine top-1 chunk),
//   S1 page-level retrieval (mean-query . mean-key page scores, top-K_p),
//   S3 head-adaptive block selection (pooled block scores, minimal mass prefix).
// WorldAttention §3.2 "Stage 1", "Stage 2"; §3.3 "Head-level sparsity adaptation".
//
// Every quantity that decides an index is computed in float64, so the decision is
// taken in the same precision as the float64 reference; the HBM passes read the
// bf16/fp32 inputs once with 16-byte vector loads.
#include <cuda_bf16.h>

#include <cfloat>
#include <climits>
#include <cmath>

#include "wa_internal.h"

namespace wa {
namespace {

constexpr int kTargetCtas = 4 * 148;  // about four resident CTAs per SM on a B200

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum over a CTA of blockDim.x <= 1024 threads; result valid in every thread.
__device__ double block_sum(double v, double* red /*[32]*/) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
  for (int w = 0; w < nw; ++w) t += red[w];  // fixed order: deterministic
  return t;
}

// 16-byte vectors of inputs, widened to double.
__device__ __forceinline__ void load_raw(const float* p, uint4& r) {
  r = __ldg(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void widen(const float*, const uint4& r, double (&o)[4]) {
  o[0] = __uint_as_float(r.x); o[1] = __uint_as_float(r.y);
  o[2] = __uint_as_float(r.z); o[3] = __uint_as_float(r.w);
}
__device__ __forceinline__ void load_raw(const __nv_bfloat16* p, uint4& r) {
  r = __ldg(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ double bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ double bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ void widen(const __nv_bfloat16*, const uint4& r, double (&o)[8]) {
  o[0] = bf16_lo(r.x); o[1] = bf16_hi(r.x); o[2] = bf16_lo(r.y); o[3] = bf16_hi(r.y);
  o[4] = bf16_lo(r.z); o[5] = bf16_hi(r.z); o[6] = bf16_lo(r.w); o[7] = bf16_hi(r.w);
}

// ------------------------------------------------------------------ S0
// One CTA: warp w computes the cosine of chunks w, w+32, ... (lanes stride over
// the embedding, then a shuffle tree), then warp 0 takes the argmax.
constexpr int kMaxChunks = 4096;

__global__ void __launch_bounds__(1024)
k_prompt_select(const float* __restrict__ e_cur, const float* __restrict__ e_chunks, int n, int D,
                int32_t* chunk_out, uint32_t* err) {
  __shared__ double cosv[kMaxChunks];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int m = warp; m < n; m += nw) {
    const float* em = e_chunks + static_cast<size_t>(m) * D;
    double dot = 0.0, nm = 0.0, nc = 0.0;
    for (int i = lane; i < D; i += 32) {
      const double a = e_cur[i], b = em[i];
      dot += a * b; nm += b * b; nc += a * a;
    }
    dot = warp_sum(dot); nm = warp_sum(nm); nc = warp_sum(nc);
    if (lane == 0) cosv[m] = (nm == 0.0 || nc == 0.0) ? NAN : dot / (sqrt(nm) * sqrt(nc));
  }
  __syncthreads();
  if (warp != 0) return;
  double best = -DBL_MAX;
  int bi = INT_MAX;
  bool bad = false;
  for (int m = lane; m < n; m += 32) {
    const double c = cosv[m];
    if (isnan(c)) { bad = true; continue; }
    if (bi == INT_MAX || c > best) { best = c; bi = m; }  // increasing m: strict > keeps lowest
  }
  bad = __any_sync(0xffffffffu, bad);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (oi != INT_MAX && (bi == INT_MAX || ob > best || (ob == best && oi < bi))) {
      best = ob; bi = oi;
    }
  }
  if (lane == 0) {
    *chunk_out = bad ? -1 : bi;
    if (bad) atomicOr(err, WA_DEVERR_ZERO_NORM);
  }
}

// ------------------------------------------------------------------ S1 HBM pass
// One CTA sums blocks [b0, b1) of one source (pool page or buffer); thread t owns
// columns [t*V, t*V + V).  Rows are read with 16-byte loads, eight in flight.
template <typename T, int V>
__global__ void __launch_bounds__(1024)
k_rowblock_sum(const T* __restrict__ x, const int32_t* __restrict__ src_ids, int n_pages,
               int rows, int cols, int B, int nb, int bps, double* __restrict__ blocksum,
               double* __restrict__ partial, int n_split, uint32_t* err) {
  const int s = blockIdx.y, split = blockIdx.x;
  int page = src_ids ? src_ids[s] : s;
  const bool ok = page >= 0 && page < n_pages;
  if (!ok && threadIdx.x == 0) atomicOr(err, WA_DEVERR_PAGE_ID);
  if (!ok) page = 0;
  const T* base = x + static_cast<size_t>(page) * rows * cols + threadIdx.x * V;
  double part[V];
#pragma unroll
  for (int v = 0; v < V; ++v) part[v] = 0.0;
  const int b0 = split * bps, b1 = min(nb, b0 + bps);
  for (int b = b0; b < b1; ++b) {
    const int r0 = b * B, r1 = min(rows, r0 + B);
    double acc[V];
#pragma unroll
    for (int v = 0; v < V; ++v) acc[v] = 0.0;
    if (ok) {
      int r = r0;
      for (; r + 8 <= r1; r += 8) {
        uint4 raw[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) load_raw(base + static_cast<size_t>(r + u) * cols, raw[u]);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          double w[V];
          widen(base, raw[u], w);
#pragma unroll
          for (int v = 0; v < V; ++v) acc[v] += w[v];
        }
      }
      for (; r < r1; ++r) {
        uint4 raw;
        load_raw(base + static_cast<size_t>(r) * cols, raw);
        double w[V];
        widen(base, raw, w);
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] += w[v];
      }
    }
    if (blocksum) {
      double* o = blocksum + (static_cast<size_t>(s) * nb + b) * cols + threadIdx.x * V;
#pragma unroll
      for (int v = 0; v < V; ++v) o[v] = acc[v];
    }
#pragma unroll
    for (int v = 0; v < V; ++v) part[v] += acc[v];
  }
  double* o = partial + (static_cast<size_t>(s) * n_split + split) * cols + threadIdx.x * V;
#pragma unroll
  for (int v = 0; v < V; ++v) o[v] = part[v];
}

// ------------------------------------------------------------------ S1 scores
// alpha[c] = (1/(H*sqrt(d))) * sum_cols Qbar * Kbar_c, with Qbar = sum(q)/Nq and
// Kbar_c = sum(k_c)/T_p rebuilt from the per-CTA partial sums in a fixed order.
__global__ void k_page_alpha(const double* __restrict__ q_partial, int q_split, int Nq,
                             const double* __restrict__ k_partial, int k_split, int T_p, int H,
                             int d, double* __restrict__ alpha) {
  __shared__ double red[32];
  const int c = blockIdx.x, cols = H * d;
  double acc = 0.0;
  for (int col = threadIdx.x; col < cols; col += blockDim.x) {
    double qs = 0.0, ks = 0.0;
    for (int sp = 0; sp < q_split; ++sp) qs += q_partial[static_cast<size_t>(sp) * cols + col];
    for (int sp = 0; sp < k_split; ++sp)
      ks += k_partial[(static_cast<size_t>(c) * k_split + sp) * cols + col];
    acc += (qs / Nq) * (ks / T_p);
  }
  acc = block_sum(acc, red);
  if (threadIdx.x == 0) alpha[c] = acc / sqrt(static_cast<double>(d)) / H;
}

// Top-K_p of alpha (ties -> lower position), emitted in ascending position.
__global__ void k_page_topk(const double* __restrict__ alpha, int n_c, int K_p,
                            const int32_t* __restrict__ cand, int32_t* sel, int32_t* sel_pos) {
  extern __shared__ unsigned char chosen[];  // n_c bytes
  const int lane = threadIdx.x;
  for (int j = lane; j < n_c; j += 32) chosen[j] = 0;
  __syncwarp();
  for (int s = 0; s < K_p; ++s) {
    double best = -DBL_MAX;
    int bi = INT_MAX;
    for (int j = lane; j < n_c; j += 32) {
      if (chosen[j]) continue;
      const double a = alpha[j];
      if (bi == INT_MAX || a > best) { best = a; bi = j; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (oi != INT_MAX && (bi == INT_MAX || ob > best || (ob == best && oi < bi))) {
        best = ob; bi = oi;
      }
    }
    if (lane == 0 && bi != INT_MAX) chosen[bi] = 1;
    __syncwarp();
  }
  if (lane == 0) {
    int k = 0;
    for (int j = 0; j < n_c && k < K_p; ++j)
      if (chosen[j]) { sel[k] = cand[j]; if (sel_pos) sel_pos[k] = j; ++k; }
  }
}

__global__ void k_scale_copy(const double* __restrict__ src, double* __restrict__ dst, size_t n,
                             double scale) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    dst[i] = src[i] * scale;
}

// ------------------------------------------------------------------ S3
// CTA = (group of G query blocks, head).  Phases: pooled scores for every key block
// (float64), a bitonic sort per row (descending score, ascending block on ties), a
// warp scan of the softmax masses to find the shortest prefix reaching tau_h, then
// the mask / ascending index list.
constexpr int kSelThreads = 256;

struct SelSmem {
  double* qb;      // [G][d]
  double* kc;      // [32][d+1]
  double* key;     // [G][NP]
  int* idx;        // [G][NP]
  uint32_t* maskw; // [G][W]
  int* mstar;      // [G]
};

__device__ __forceinline__ bool before(double ka, int ia, double kb, int ib) {
  return ka > kb || (ka == kb && ia < ib);
}

__global__ void __launch_bounds__(kSelThreads)
k_block_select(const double* __restrict__ qsum, int Nq, int H, int d, int B, int n_qb,
               KeyMeans km, int n_kb, int NP, int G, int W, const float* __restrict__ tau,
               int32_t* __restrict__ blk_idx, int32_t* __restrict__ blk_cnt,
               uint32_t* __restrict__ blk_mask) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SelSmem sm;
  sm.qb = reinterpret_cast<double*>(smem_raw);
  sm.kc = sm.qb + G * d;
  sm.key = sm.kc + 32 * (d + 1);
  sm.idx = reinterpret_cast<int*>(sm.key + static_cast<size_t>(G) * NP);
  sm.maskw = reinterpret_cast<uint32_t*>(sm.idx + static_cast<size_t>(G) * NP);
  sm.mstar = reinterpret_cast<int*>(sm.maskw + G * W);

  const int h = blockIdx.y, i0 = blockIdx.x * G;
  const int cols = H * d;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const double sqrt_d = sqrt(static_cast<double>(d));

  // pooled query means
  for (int e = tid; e < G * d; e += kSelThreads) {
    const int g = e / d, c = e % d, i = i0 + g;
    double v = 0.0;
    if (i < n_qb) {
      const int cnt = min(Nq, (i + 1) * B) - i * B;
      v = qsum[static_cast<size_t>(i) * cols + h * d + c] / cnt;
    }
    sm.qb[e] = v;
  }
  // scores s[g][j] = qbar_g . kbar_j / sqrt(d), 32 key blocks per pass
  for (int j0 = 0; j0 < n_kb; j0 += 32) {
    __syncthreads();
    for (int e = tid; e < 32 * d; e += kSelThreads) {
      const int jj = e / d, c = e % d, j = j0 + jj;
      double v = 0.0;
      if (j < n_kb) {
        size_t row = j;
        if (km.page_pos) row = static_cast<size_t>(km.page_pos[j / km.nbp]) * km.nbp + j % km.nbp;
        v = km.data[row * cols + h * d + c];
        if (km.is_sum) v /= static_cast<double>(min(km.L, (j + 1) * B) - j * B);
      }
      sm.kc[jj * (d + 1) + c] = v;
    }
    __syncthreads();
    const int jj = tid & 31, g = tid >> 5, j = j0 + jj;
    if (g < G && j < n_kb) {
      const double* qg = sm.qb + g * d;
      const double* kr = sm.kc + jj * (d + 1);
      double s = 0.0;
      for (int c = 0; c < d; ++c) s += qg[c] * kr[c];
      sm.key[static_cast<size_t>(g) * NP + j] = s / sqrt_d;
      sm.idx[static_cast<size_t>(g) * NP + j] = j;
    }
  }
  for (int e = tid; e < G * NP; e += kSelThreads) {
    if (e % NP >= n_kb) { sm.key[e] = -INFINITY; sm.idx[e] = INT_MAX; }
  }
  __syncthreads();

  // bitonic sort of every row: "before" order first
  const int half = NP >> 1;
  for (int k = 2; k <= NP; k <<= 1) {
    for (int jstep = k >> 1; jstep > 0; jstep >>= 1) {
      for (int e = tid; e < G * half; e += kSelThreads) {
        const int g = e / half, p = e % half;
        const int i = 2 * jstep * (p / jstep) + (p % jstep);
        const int l = i + jstep;
        double* kr = sm.key + static_cast<size_t>(g) * NP;
        int* ir = sm.idx + static_cast<size_t>(g) * NP;
        const double ki = kr[i], kl = kr[l];
        const int ii = ir[i], il = ir[l];
        const bool up = (i & k) == 0;
        const bool swap = up ? before(kl, il, ki, ii) : before(ki, ii, kl, il);
        if (swap) { kr[i] = kl; kr[l] = ki; ir[i] = il; ir[l] = ii; }
      }
      __syncthreads();
    }
  }

  // shortest prefix reaching tau: one warp per row
  for (int g = warp; g < G; g += kSelThreads / 32) {
    const int i = i0 + g;
    if (i >= n_qb) { if (lane == 0) sm.mstar[g] = 0; continue; }
    const double th = static_cast<double>(tau[h]);
    const double* kr = sm.key + static_cast<size_t>(g) * NP;
    int m = n_kb;
    if (th < 1.0) {
      const double smax = kr[0];
      const int per = NP / 32;             // NP >= 32
      const int t0 = lane * per;
      double zl = 0.0;
      for (int t = t0; t < t0 + per && t < n_kb; ++t) zl += exp(kr[t] - smax);
      const double Z = warp_sum(zl);
      double pl = 0.0;
      for (int t = t0; t < t0 + per && t < n_kb; ++t) pl += exp(kr[t] - smax) / Z;
      // exclusive scan of the lane sums
      double incl = pl;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      double c = incl - pl;
      int first = INT_MAX;
      for (int t = t0; t < t0 + per && t < n_kb; ++t) {
        c += exp(kr[t] - smax) / Z;
        if (c >= th) { first = t; break; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) first = min(first, __shfl_xor_sync(0xffffffffu, first, o));
      if (first != INT_MAX) m = first + 1;
    }
    if (lane == 0) sm.mstar[g] = m;
  }
  for (int e = tid; e < G * W; e += kSelThreads) sm.maskw[e] = 0u;
  __syncthreads();
  for (int e = tid; e < G * NP; e += kSelThreads) {
    const int g = e / NP, t = e % NP;
    if (t < sm.mstar[g]) {
      const int j = sm.idx[e];
      atomicOr(&sm.maskw[g * W + (j >> 5)], 1u << (j & 31));
    }
  }
  __syncthreads();
  for (int g = warp; g < G; g += kSelThreads / 32) {
    const int i = i0 + g;
    if (i >= n_qb) continue;
    const size_t row = static_cast<size_t>(h) * n_qb + i;
    if (blk_mask)
      for (int w = lane; w < W; w += 32) blk_mask[row * W + w] = sm.maskw[g * W + w];
    if (blk_cnt && lane == 0) blk_cnt[row] = sm.mstar[g];
    if (blk_idx) {
      // lane owns words [lane*wpl, lane*wpl + wpl): ascending order follows lane order
      const int wpl = (W + 31) / 32;
      int cnt = 0;
      for (int w = lane * wpl; w < min(W, lane * wpl + wpl); ++w) cnt += __popc(sm.maskw[g * W + w]);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int pos = incl - cnt;
      int32_t* out = blk_idx + row * n_kb;
      for (int w = lane * wpl; w < min(W, lane * wpl + wpl); ++w) {
        uint32_t bits = sm.maskw[g * W + w];
        while (bits) {
          const int b = __ffs(bits) - 1;
          bits &= bits - 1;
          out[pos++] = w * 32 + b;
        }
      }
      const int m = sm.mstar[g];
      for (int t = m + lane; t < n_kb; t += 32) out[t] = -1;
    }
  }
}

}  // namespace

// ==================================================================== launchers
wa_status launch_prompt_select(const float* e_cur, const float* e_chunks, int n_chunks, int D,
                               int32_t* chunk_out, uint32_t* err, cudaStream_t st) {
  if (n_chunks > kMaxChunks) return set_error(WA_ERR_UNSUPPORTED, "at most %d chunks", kMaxChunks);
  k_prompt_select<<<1, 1024, 0, st>>>(e_cur, e_chunks, n_chunks, D, chunk_out, err);
  return check_launch("prompt_select");
}

int rowsum_splits(int n_src, int rows, int B) {
  const int nb = (rows + B - 1) / B;
  int want = (kTargetCtas + n_src - 1) / n_src;
  want = want < 1 ? 1 : (want > nb ? nb : want);
  const int bps = (nb + want - 1) / want;
  return (nb + bps - 1) / bps;
}

wa_status launch_rowblock_sum(const void* x, wa_dtype dt, const int32_t* src_ids, int n_src,
                              int n_pages, int rows, int cols, int B, double* blocksum,
                              double* partial, int n_split, uint32_t* err, cudaStream_t st) {
  const int nb = (rows + B - 1) / B;
  const int bps = (nb + n_split - 1) / n_split;
  dim3 grid(n_split, n_src);
  if (dt == WA_BF16) {
    k_rowblock_sum<__nv_bfloat16, 8><<<grid, cols / 8, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), src_ids, n_pages, rows, cols, B, nb, bps, blocksum,
        partial, n_split, err);
  } else {
    k_rowblock_sum<float, 4><<<grid, cols / 4, 0, st>>>(static_cast<const float*>(x), src_ids,
                                                        n_pages, rows, cols, B, nb, bps, blocksum,
                                                        partial, n_split, err);
  }
  return check_launch("rowblock_sum");
}

wa_status launch_page_alpha_topk(const double* q_partial, int q_split, int Nq,
                                 const double* k_partial, int k_split, int T_p, int n_c,
                                 int H, int d, int K_p, const int32_t* cand, double* alpha,
                                 int32_t* sel, int32_t* sel_pos, cudaStream_t st) {
  k_page_alpha<<<n_c, 256, 0, st>>>(q_partial, q_split, Nq, k_partial, k_split, T_p, H, d,
                                    alpha);
  k_page_topk<<<1, 32, n_c, st>>>(alpha, n_c, K_p, cand, sel, sel_pos);
  return check_launch("page_alpha_topk");
}

wa_status launch_scale_copy(const double* src, double* dst, size_t n, double scale,
                            cudaStream_t st) {
  k_scale_copy<<<4 * 148, 256, 0, st>>>(src, dst, n, scale);
  return check_launch("scale_copy");
}

size_t block_select_smem_bytes(int d, int n_kb, int* G_out) {
  int NP = 32;
  while (NP < n_kb) NP <<= 1;
  int G = 8;
  while (G > 1 && static_cast<size_t>(G) * NP * 12 > 98304) G >>= 1;
  const int W = (n_kb + 31) / 32;
  if (G_out) *G_out = G;
  return static_cast<size_t>(G) * d * 8 + 32 * static_cast<size_t>(d + 1) * 8 +
         static_cast<size_t>(G) * NP * 12 + static_cast<size_t>(G) * W * 4 + G * 4;
}

wa_status launch_block_select(const double* q_blocksum, int Nq, int H, int d, int B,
                              KeyMeans km, int n_kb, const float* tau, int32_t* blk_idx,
                              int32_t* blk_cnt, uint32_t* blk_mask, cudaStream_t st) {
  int G = 1;
  const size_t smem = block_select_smem_bytes(d, n_kb, &G);
  int NP = 32;
  while (NP < n_kb) NP <<= 1;
  const int W = (n_kb + 31) / 32;
  const int n_qb = (Nq + B - 1) / B;
  cudaError_t e = cudaFuncSetAttribute(k_block_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return set_error(WA_ERR_CUDA, "block_select smem attr: %s", cudaGetErrorString(e));
  dim3 grid((n_qb + G - 1) / G, H);
  k_block_select<<<grid, kSelThreads, smem, st>>>(q_blocksum, Nq, H, d, B, n_qb, km, n_kb, NP, G,
                                                  W, tau, blk_idx, blk_cnt, blk_mask);
  return check_launch("block_select");
}

}  // namespace wa
