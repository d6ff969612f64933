// k_select.cu -- the index-producing steps of the HSA decode step besides the page
// scores (those, and the block sums every step starts from, are in k_blocksum.cu):
//   S0 prompt-level retrieval (cosine top-1 chunk),
//   S3 head-adaptive block selection (pooled block scores, minimal mass prefix).
// WorldAttention §3.2 "Stage 1"; §3.3 "Head-level sparsity adaptation".
//
// Every quantity that decides an index is computed in float64, so the decision is
// taken in the same precision as the float64 reference.
#include <cuda_bf16.h>

#include <cfloat>
#include <climits>
#include <cmath>

#include "wa_internal.h"

namespace wa {
namespace {


__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
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

// Qbar[col] = sum of all query rows / Nq; qmean[i][col] = block sum / rows of block i.
// CTA = 32 columns x 8 row groups; group g sums blocks g, g+8, ...; the eight group
// sums are added in a fixed order (deterministic).
__global__ void __launch_bounds__(256)
k_qmeans(const double* __restrict__ qsum, int n_qb, int Nq, int B, int cols,
         double* __restrict__ qbar, double* __restrict__ qmean) {
  __shared__ double red[8][32];
  const int col = blockIdx.x * 32 + threadIdx.x;
  const int g = threadIdx.y;
  double t = 0.0;
  if (col < cols) {
#pragma unroll 4
    for (int i = g; i < n_qb; i += 8) {
      const double v = qsum[static_cast<size_t>(i) * cols + col];
      t += v;
      if (qmean) qmean[static_cast<size_t>(i) * cols + col] = v / (min(Nq, (i + 1) * B) - i * B);
    }
  }
  red[g][threadIdx.x] = t;
  __syncthreads();
  if (g == 0 && col < cols) {
    double s = 0.0;
    for (int k = 0; k < 8; ++k) s += red[k][threadIdx.x];
    qbar[col] = s / Nq;
  }
}

__global__ void k_scale_copy(const double* __restrict__ src, double* __restrict__ dst, size_t n,
                             double scale) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    dst[i] = src[i] * scale;
}

// ------------------------------------------------------------------ S3 scores
// s[h][i][j] = qbar_{h,i} . kbar_{h,j} / sqrt(d) in float64.  CTA = a 32 x 32 tile
// of (query block, key block) of one head; both 32-row operand tiles are staged in
// shared memory (key rows at pitch d+1 doubles against bank conflicts) and each
// thread accumulates a 2 x 2 register tile: rows ty, ty+16 and key blocks tx, tx+16.
__global__ void __launch_bounds__(256)
k_block_scores(const double* __restrict__ qmean, KeyMeans km, int n_qb, int n_kb, int H, int d,
               int B, double* __restrict__ scores) {
  extern __shared__ double sm_scores[];
  double* qs = sm_scores;                    // [32][d]
  double* kc = sm_scores + 32 * d;           // [32][d+1]
  const int j0 = blockIdx.x * 32, i0 = blockIdx.y * 32, h = blockIdx.z;
  const int cols = H * d;
  // a warp per row: the row's source (through the page position when the key means
  // come from the candidate pass) is resolved once, the d values load coalesced
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int rr = warp; rr < 32; rr += blockDim.x >> 5) {
    const int j = j0 + rr, i = i0 + rr;
    const double* ksrc = nullptr;
    const double* ksrc2 = nullptr;   // second B-row half of a 2B-row history block
    auto sub_row = [&](int jj) -> size_t {
      if (km.page_pos) return static_cast<size_t>(km.page_pos[jj / km.nbp]) * km.nbp + jj % km.nbp;
      return static_cast<size_t>(jj);
    };
    if (j < n_kb) {
      if (km.data2 && j >= km.n_kb1) {
        ksrc = km.data2 + static_cast<size_t>(j - km.n_kb1) * cols + h * d;
      } else if (km.pair) {
        ksrc = km.data + sub_row(2 * j) * cols + h * d;
        if (2 * j + 1 < km.n_sub) ksrc2 = km.data + sub_row(2 * j + 1) * cols + h * d;
      } else {
        ksrc = km.data + sub_row(j) * cols + h * d;
      }
    }
    const double* qsrc = i < n_qb ? qmean + static_cast<size_t>(i) * cols + h * d : nullptr;
    for (int c = lane; c < d; c += 32) {
      kc[rr * (d + 1) + c] = ksrc ? (ksrc2 ? ksrc[c] + ksrc2[c] : ksrc[c]) : 0.0;
      qs[rr * d + c] = qsrc ? qsrc[c] : 0.0;
    }
  }
  __syncthreads();
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const double* q0 = qs + ty * d;
  const double* q1 = qs + (ty + 16) * d;
  const double* k0 = kc + tx * (d + 1);
  const double* k1 = kc + (tx + 16) * (d + 1);
  double a00 = 0.0, a01 = 0.0, a10 = 0.0, a11 = 0.0;
#pragma unroll 4
  for (int c = 0; c < d; ++c) {
    const double x0 = q0[c], x1 = q1[c], y0 = k0[c], y1 = k1[c];
    a00 += x0 * y0; a01 += x0 * y1; a10 += x1 * y0; a11 += x1 * y1;
  }
  // key block sums become means here: q . (sum / n) / sqrt(d) = (q . sum) / (n sqrt(d))
  const double sqrt_d = sqrt(static_cast<double>(d));
  const double acc[2][2] = {{a00, a01}, {a10, a11}};
#pragma unroll
  for (int v = 0; v < 2; ++v) {
    const int j = j0 + tx + 16 * v;
    if (j >= n_kb) continue;
    double den = sqrt_d;
    if (km.data2 && j >= km.n_kb1) {
      const int jj = j - km.n_kb1;
      den = static_cast<double>(min(km.L2, (jj + 1) * B) - jj * B) * sqrt_d;
    } else if (km.is_sum) {
      const int Bk = km.pair ? 2 * B : B;   // rows of a history block
      den = static_cast<double>(min(km.L, (j + 1) * Bk) - j * Bk) * sqrt_d;
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = i0 + ty + 16 * u;
      if (i < n_qb) scores[(static_cast<size_t>(h) * n_qb + i) * n_kb + j] = acc[u][v] / den;
    }
  }
}

// ------------------------------------------------------------------ S3 choice
// CTA = one (head, query block) row: bitonic sort of the scores (descending,
// ascending block on ties), softmax masses exp(s - max)/Z, a block-wide scan of the
// masses in sorted order, the first position whose prefix reaches tau_h, then the
// mask and the ascending index list.
constexpr int kChooseThreads = 256;

__device__ __forceinline__ bool before(double ka, int ia, double kb, int ib) {
  return ka > kb || (ka == kb && ia < ib);
}

__global__ void __launch_bounds__(kChooseThreads)
k_block_choose(const double* __restrict__ scores, int n_qb, int n_kb, int lg_np, int W,
               const float* __restrict__ tau, int32_t* __restrict__ blk_idx,
               int32_t* __restrict__ blk_cnt, uint32_t* __restrict__ blk_mask, int n_h, int n_sub,
               int W_mask) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int NP = 1 << lg_np;
  double* key = reinterpret_cast<double*>(smem_raw);          // [NP]
  int* idx = reinterpret_cast<int*>(key + NP);                 // [NP]
  uint32_t* maskw = reinterpret_cast<uint32_t*>(idx + NP);     // [W] (selection blocks)
  uint32_t* maskx = maskw + W;                                  // [W_mask] (n_h > 0: B-row blocks)
  __shared__ double wred[kChooseThreads / 32];
  __shared__ int ired[kChooseThreads / 32];
  const int h = blockIdx.y, i = blockIdx.x;
  const size_t rowid = static_cast<size_t>(h) * n_qb + i;
  const double* srow = scores + rowid * n_kb;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < NP; e += kChooseThreads) {
    key[e] = e < n_kb ? srow[e] : -INFINITY;
    idx[e] = e < n_kb ? e : INT_MAX;
  }
  for (int w = tid; w < W; w += kChooseThreads) maskw[w] = 0u;
  for (int w = tid; w < W_mask && n_h > 0; w += kChooseThreads) maskx[w] = 0u;
  __syncthreads();
  for (int k = 2; k <= NP; k <<= 1) {
    for (int js = k >> 1; js > 0; js >>= 1) {
      for (int p = tid; p < (NP >> 1); p += kChooseThreads) {
        const int a = ((p & ~(js - 1)) << 1) | (p & (js - 1));   // bit js of a is 0
        const int b = a | js;
        const double ka = key[a], kb = key[b];
        const int ia = idx[a], ib = idx[b];
        const bool swap = (a & k) == 0 ? before(kb, ib, ka, ia) : before(ka, ia, kb, ib);
        if (swap) { key[a] = kb; key[b] = ka; idx[a] = ib; idx[b] = ia; }
      }
      __syncthreads();
    }
  }
  const double th = static_cast<double>(tau[h]);
  int m = n_kb;
  if (th < 1.0) {
    // every thread takes the maximum before thread 0 overwrites key[0] with its
    // exponential below (without this barrier a warp running ahead changes the
    // maximum that slower warps read, and the masses of their blocks come out wrong)
    const double smax = key[0];
    __syncthreads();
    const int per = NP / kChooseThreads > 0 ? NP / kChooseThreads : 1;
    const int t0 = tid * per;
    // z_t = exp(s_t - max), kept in place of the sorted scores
    double zl = 0.0;
    for (int t = t0; t < t0 + per && t < NP; ++t) {
      const double z = t < n_kb ? exp(key[t] - smax) : 0.0;
      key[t] = z;
      zl += z;
    }
    zl = warp_sum(zl);
    if (lane == 0) wred[warp] = zl;
    __syncthreads();
    double Z = 0.0;
    for (int w = 0; w < kChooseThreads / 32; ++w) Z += wred[w];
    __syncthreads();
    double pl = 0.0;
    for (int t = t0; t < t0 + per && t < NP; ++t) {
      const double pv = key[t] / Z;
      key[t] = pv;
      pl += pv;
    }
    // exclusive prefix of the per-thread sums, in thread order
    double incl = pl;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wred[warp] = incl;
    __syncthreads();
    double c = incl - pl;
    for (int w = 0; w < warp; ++w) c += wred[w];
    int first = INT_MAX;
    for (int t = t0; t < t0 + per && t < n_kb; ++t) {
      c += key[t];
      if (c >= th) { first = t; break; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) first = min(first, __shfl_xor_sync(0xffffffffu, first, o));
    if (lane == 0) ired[warp] = first;
    __syncthreads();
    first = INT_MAX;
    for (int w = 0; w < kChooseThreads / 32; ++w) first = min(first, ired[w]);
    if (first != INT_MAX) m = first + 1;
  }
  for (int t = tid; t < m; t += kChooseThreads) {
    const int j = idx[t];
    atomicOr(&maskw[j >> 5], 1u << (j & 31));
    if (n_h > 0) {
      // the same keys at B-row granularity: a 2B-row history block covers B-row blocks
      // 2j and 2j + 1, a chunk block one
      if (j < n_h) {
        atomicOr(&maskx[(2 * j) >> 5], 1u << ((2 * j) & 31));
        if (2 * j + 1 < n_sub) atomicOr(&maskx[(2 * j + 1) >> 5], 1u << ((2 * j + 1) & 31));
      } else {
        const int x = n_sub + (j - n_h);
        atomicOr(&maskx[x >> 5], 1u << (x & 31));
      }
    }
  }
  __syncthreads();
  if (blk_mask) {
    const uint32_t* src = n_h > 0 ? maskx : maskw;
    for (int w = tid; w < W_mask; w += kChooseThreads) blk_mask[rowid * W_mask + w] = src[w];
  }
  if (blk_cnt && tid == 0) blk_cnt[rowid] = m;
  if (blk_idx && warp == 0) {
    const int wpl = (W + 31) / 32;
    int cnt = 0;
    for (int w = lane * wpl; w < min(W, lane * wpl + wpl); ++w) cnt += __popc(maskw[w]);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = incl - cnt;
    int32_t* out = blk_idx + rowid * n_kb;
    for (int w = lane * wpl; w < min(W, lane * wpl + wpl); ++w) {
      uint32_t bits = maskw[w];
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        out[pos++] = w * 32 + b;
      }
    }
    for (int t = m + lane; t < n_kb; t += 32) out[t] = -1;
  }
}

// The same choice for rows of at most 1024 key blocks, without a barrier per stage of
// the sorting network: thread g of the row's NW warps holds positions g*E .. g*E+E-1
// in registers (NP = 32 * NW * E), strides below E compare inside a thread, strides
// below 32 E exchange with the partner lane by shuffles, and only larger ones (the
// last stages of the last phases when NW > 1) go through shared memory.  Padding
// positions carry score -inf and their own position as index, so the order stays
// strict.  The masses, their prefix and the cut follow the block kernel above (sums
// in another grouping: float64 rounding only).
template <int E>
__device__ __forceinline__ void ce_lane(double (&key)[E], int (&idx)[E], int a, int b, bool asc) {
  // a < b inside the thread; asc: position a must hold the element that comes first
  const bool b_first = key[b] > key[a] || (key[b] == key[a] && idx[b] < idx[a]);
  const bool a_first = key[a] > key[b] || (key[a] == key[b] && idx[a] < idx[b]);
  if (asc ? b_first : a_first) {
    const double tk = key[a]; key[a] = key[b]; key[b] = tk;
    const int ti = idx[a]; idx[a] = idx[b]; idx[b] = ti;
  }
}

template <int E, int NW>
__global__ void __launch_bounds__(32 * NW)
k_block_choose_net(const double* __restrict__ scores, int n_qb, int n_kb, int W,
                   const float* __restrict__ tau, int32_t* __restrict__ blk_idx,
                   int32_t* __restrict__ blk_cnt, uint32_t* __restrict__ blk_mask, int n_h,
                   int n_sub, int W_mask) {
  constexpr int NT = 32 * NW;
  constexpr int NP = NT * E;
  constexpr int LGE = E >= 8 ? 3 : E >= 4 ? 2 : E >= 2 ? 1 : 0;
  static_assert(E <= 8 && NP <= 1024, "positions per thread / row length");
  __shared__ double xk[NW > 1 ? E * NT : 1];   // exchange of the cross-warp stages,
  __shared__ int xi[NW > 1 ? E * NT : 1];      // position g*E+e at [e][g]
  __shared__ double red_d[NW];
  __shared__ int red_i[NW];
  __shared__ uint32_t maskw[32];                 // selection blocks (n_kb <= 1024)
  extern __shared__ uint32_t maskx[];            // [W_mask] (n_h > 0: B-row blocks)
  const int h = blockIdx.y, i = blockIdx.x, g = threadIdx.x, lane = g & 31, warp = g >> 5;
  const size_t rowid = static_cast<size_t>(h) * n_qb + i;
  const double* srow = scores + rowid * n_kb;
  const int p0 = g * E;
  double key[E];
  int idx[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    key[e] = p0 + e < n_kb ? srow[p0 + e] : -INFINITY;
    idx[e] = p0 + e;
  }
  for (int w = g; w < 32; w += NT) maskw[w] = 0u;
  for (int w = g; w < W_mask && n_h > 0; w += NT) maskx[w] = 0u;
  // phases k <= E: every stride is inside the thread
#pragma unroll
  for (int lk = 1; lk <= LGE; ++lk) {
    const int k = 1 << lk;
#pragma unroll
    for (int lj = lk - 1; lj >= 0; --lj) {
      const int j = 1 << lj;
#pragma unroll
      for (int e = 0; e < E; ++e)
        if ((e & j) == 0) ce_lane<E>(key, idx, e, e | j, ((p0 + e) & k) == 0);
    }
  }
  // phases k > E: strides across threads (shared memory, then shuffles), then inside
  for (int k = 2 * E; k <= NP; k <<= 1) {
    const bool asc = (p0 & k) == 0;   // the same for the thread's E positions
    for (int j = k >> 1; j >= E; j >>= 1) {
      const int gm = j / E;           // partner thread g ^ gm
      const bool keep_first = ((g & gm) == 0) == asc;
      if (NW > 1 && gm >= 32) {
        __syncthreads();              // the previous exchange has been read
#pragma unroll
        for (int e = 0; e < E; ++e) { xk[e * NT + g] = key[e]; xi[e * NT + g] = idx[e]; }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const double ok = xk[e * NT + (g ^ gm)];
          const int oi = xi[e * NT + (g ^ gm)];
          const bool other_first = ok > key[e] || (ok == key[e] && oi < idx[e]);
          if (keep_first == other_first) { key[e] = ok; idx[e] = oi; }
        }
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const double ok = __shfl_xor_sync(0xffffffffu, key[e], gm);
          const int oi = __shfl_xor_sync(0xffffffffu, idx[e], gm);
          const bool other_first = ok > key[e] || (ok == key[e] && oi < idx[e]);
          if (keep_first == other_first) { key[e] = ok; idx[e] = oi; }
        }
      }
    }
#pragma unroll
    for (int lj = LGE - 1; lj >= 0; --lj) {
      const int j = 1 << lj;
#pragma unroll
      for (int e = 0; e < E; ++e)
        if ((e & j) == 0) ce_lane<E>(key, idx, e, e | j, asc);
    }
  }
  const double th = static_cast<double>(tau[h]);
  int m = n_kb;
  if (th < 1.0) {
    if (g == 0) red_d[0] = key[0];    // position 0: the largest score
    __syncthreads();
    const double smax = red_d[0];
    __syncthreads();
    // z_t = exp(s_t - max) in place of the sorted scores, then p_t = z_t / Z
    double zl = 0.0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const double z = p0 + e < n_kb ? exp(key[e] - smax) : 0.0;
      key[e] = z;
      zl += z;
    }
    zl = warp_sum(zl);
    if (lane == 0) red_d[warp] = zl;
    __syncthreads();
    double Z = 0.0;
#pragma unroll
    for (int w = 0; w < NW; ++w) Z += red_d[w];
    __syncthreads();
    double pl = 0.0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      key[e] = key[e] / Z;
      pl += key[e];
    }
    // exclusive prefix of the per-thread sums, in thread order
    double incl = pl;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) red_d[warp] = incl;
    double c = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) c = 0.0;
    __syncthreads();
    for (int w = 0; w < warp; ++w) c += red_d[w];
    int first = INT_MAX;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if (p0 + e < n_kb && first == INT_MAX) {
        c += key[e];
        if (c >= th) first = p0 + e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) first = min(first, __shfl_xor_sync(0xffffffffu, first, o));
    if (lane == 0) red_i[warp] = first;
    __syncthreads();
    first = INT_MAX;
#pragma unroll
    for (int w = 0; w < NW; ++w) first = min(first, red_i[w]);
    if (first != INT_MAX) m = first + 1;
  }
  __syncthreads();
#pragma unroll
  for (int e = 0; e < E; ++e) {
    if (p0 + e >= m) continue;
    const int j = idx[e];
    atomicOr(&maskw[j >> 5], 1u << (j & 31));
    if (n_h > 0) {
      // the same keys at B-row granularity: a 2B-row history block covers B-row blocks
      // 2j and 2j + 1, a chunk block one
      if (j < n_h) {
        atomicOr(&maskx[(2 * j) >> 5], 1u << ((2 * j) & 31));
        if (2 * j + 1 < n_sub) atomicOr(&maskx[(2 * j + 1) >> 5], 1u << ((2 * j + 1) & 31));
      } else {
        const int x = n_sub + (j - n_h);
        atomicOr(&maskx[x >> 5], 1u << (x & 31));
      }
    }
  }
  __syncthreads();
  if (blk_mask) {
    const uint32_t* src = n_h > 0 ? maskx : maskw;
    for (int w = g; w < W_mask; w += NT) blk_mask[rowid * W_mask + w] = src[w];
  }
  if (warp == 0) {
    // W <= 32: one mask word per lane of the first warp
    const uint32_t bits0 = lane < W ? maskw[lane] : 0u;
    const int cnt = __popc(bits0);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (blk_cnt && lane == 0) blk_cnt[rowid] = total;
    if (blk_idx) {
      int32_t* out = blk_idx + rowid * n_kb;
      int pos = incl - cnt;
      for (uint32_t bits = bits0; bits != 0u; bits &= bits - 1u) out[pos++] = lane * 32 + __ffs(bits) - 1;
      for (int t = total + lane; t < n_kb; t += 32) out[t] = -1;
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

wa_status launch_qmeans(const double* qsum, int n_qb, int Nq, int B, int cols, double* qbar,
                        double* qmean, cudaStream_t st) {
  k_qmeans<<<(cols + 31) / 32, dim3(32, 8), 0, st>>>(qsum, n_qb, Nq, B, cols, qbar, qmean);
  return check_launch("qmeans");
}

wa_status launch_scale_copy(const double* src, double* dst, size_t n, double scale,
                            cudaStream_t st) {
  k_scale_copy<<<4 * 148, 256, 0, st>>>(src, dst, n, scale);
  return check_launch("scale_copy");
}

size_t block_scores_bytes(int H, int n_qb, int n_kb) {
  return static_cast<size_t>(H) * n_qb * n_kb * sizeof(double);
}

wa_status launch_block_select(const double* q_blockmean, int Nq, int H, int d, int B,
                              KeyMeans km, int n_kb, int n_kb_mask, const float* tau, double* scores,
                              int32_t* blk_idx, int32_t* blk_cnt, uint32_t* blk_mask,
                              cudaStream_t st) {
  const int n_qb = (Nq + B - 1) / B;
  const int W = (n_kb + 31) / 32;
  const int W_mask = (n_kb_mask + 31) / 32;
  if (km.pair && !km.is_sum) return set_error(WA_ERR_UNSUPPORTED, "2B-row history blocks need block sums");
  const size_t smem_s = (32 * static_cast<size_t>(d + 1) + 32 * static_cast<size_t>(d)) *
                        sizeof(double);
  cudaError_t e = cudaFuncSetAttribute(k_block_scores, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem_s));
  if (e != cudaSuccess) return set_error(WA_ERR_CUDA, "block_scores smem attr: %s", cudaGetErrorString(e));
  k_block_scores<<<dim3((n_kb + 31) / 32, (n_qb + 31) / 32, H), 256, smem_s, st>>>(
      q_blockmean, km, n_qb, n_kb, H, d, B, scores);
  int lg = 5;
  while ((1 << lg) < n_kb) ++lg;
  const int wm = km.pair ? W_mask : W;
  if (lg <= 10) {
    // rows of at most 1024 key blocks: the network in registers, 1, 2 or 4 warps a row
    const size_t smem_w = static_cast<size_t>(W_mask) * 4;
    const dim3 grid(n_qb, H);
    const int nh = km.pair ? km.n_kb1 : 0;
#define WA_CHOOSE(E_, NW_) \
  k_block_choose_net<E_, NW_><<<grid, 32 * NW_, smem_w, st>>>(scores, n_qb, n_kb, W, tau, blk_idx, \
                                                              blk_cnt, blk_mask, nh, km.n_sub, wm)
    switch (lg) {
      case 5: WA_CHOOSE(1, 1); break;
      case 6: WA_CHOOSE(2, 1); break;
      case 7: WA_CHOOSE(4, 1); break;
      case 8: WA_CHOOSE(8, 1); break;
      case 9: WA_CHOOSE(8, 2); break;
      default: WA_CHOOSE(8, 4); break;
    }
#undef WA_CHOOSE
    return check_launch("block_select");
  }
  const size_t smem_c = (static_cast<size_t>(1) << lg) * 12 + static_cast<size_t>(W + W_mask) * 4 + 16;
  e = cudaFuncSetAttribute(k_block_choose, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem_c));
  if (e != cudaSuccess) return set_error(WA_ERR_CUDA, "block_choose smem attr: %s", cudaGetErrorString(e));
  k_block_choose<<<dim3(n_qb, H), kChooseThreads, smem_c, st>>>(
      scores, n_qb, n_kb, lg, W, tau, blk_idx, blk_cnt, blk_mask, km.pair ? km.n_kb1 : 0, km.n_sub,
      km.pair ? W_mask : W);
  return check_launch("block_select");
}

}  // namespace wa
