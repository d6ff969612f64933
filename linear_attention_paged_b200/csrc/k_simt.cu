// k_simt.cu -- the float32 path (CUDA cores, FFMA), used when the inputs are fp32.
// A 1e-4 tolerance against float64 rules out TF32 tensor cores, and the fp32
// workloads are small, so these kernels favour plain, exact-order arithmetic:
//   * the Linformer projection K~ = E_K^T K (WorldAttention §3.3 "Linear branch"),
//     accumulated in float64, one thread per output element;
//   * attention of one (head, query block) per CTA, one thread per query row, with an
//     online softmax over 64-key tiles staged in shared memory: mode 0 is the linear
//     branch over (K~, V~), mode 1 the block-sparse branch over the kept key blocks
//     (§3.3 "Sparse branch", Appendix A.1.3), followed by the sigmoid gate
//     (§3.3 "Gated fusion of two branches").
#include <cmath>

#include "wa_internal.h"

namespace wa {
namespace {

__device__ __forceinline__ long long row_of(const RowSource& rs, int l, int B, bool& ok) {
  // row of token l of the active sequence in the base arrays
  if (!rs.page_ids) { ok = true; return l; }
  const int pg = rs.page_ids[l / rs.page_rows];
  ok = pg >= 0 && pg < rs.n_pages;
  return static_cast<long long>(ok ? pg : 0) * rs.page_rows + l % rs.page_rows;
}

__global__ void k_simt_project(const float* __restrict__ x, RowSource rs, const float* __restrict__ e,
                               int L, int cols, int r, int d, long long e_head_stride,
                               float* __restrict__ out, uint32_t* err) {
  const int col = blockIdx.x * blockDim.x + threadIdx.x;
  const int c = blockIdx.y;
  if (col >= cols) return;
  e += static_cast<long long>(col / d) * e_head_stride;   // this column's head's E (0: shared)
  double acc = 0.0;
  bool bad = false;
  for (int l = 0; l < L; ++l) {
    bool ok;
    const long long row = row_of(rs, l, 0, ok);
    bad |= !ok;
    acc += static_cast<double>(e[static_cast<size_t>(l) * r + c]) *
           static_cast<double>(x[row * cols + col]);
  }
  if (bad && col == 0) atomicOr(err, WA_DEVERR_PAGE_ID);
  out[static_cast<size_t>(c) * cols + col] = static_cast<float>(acc);
}

constexpr int kTile = 64;  // keys staged per pass

template <int D>
__global__ void __launch_bounds__(128)
k_simt_attention(int mode, const float* __restrict__ q, int Nq, int H, RowSource rs, int B,
                 const uint32_t* __restrict__ mask, int W, const float* __restrict__ gate,
                 float lin_sign, float* __restrict__ lin_ws, float* __restrict__ out,
                 float* __restrict__ o_branch, uint32_t* err) {
  extern __shared__ float sm[];
  float* Ks = sm;                 // [kTile][D]
  float* Vs = sm + kTile * D;     // [kTile][D]
  const int h = blockIdx.y, i = blockIdx.x;
  const int n_qb = (Nq + B - 1) / B;
  const int L = rs.L + rs.L2;      // the second segment (if any) follows the first
  const int n_kb = (L + B - 1) / B;
  const float* kb = static_cast<const float*>(rs.k);
  const float* vb = static_cast<const float*>(rs.v);
  const int cols = H * D;
  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  bool bad = false;

  // each thread owns one query row of the block
  const int row = i * B + threadIdx.x;
  const bool valid = threadIdx.x < B && row < Nq;
  float qr[D];
  float acc[D];
#pragma unroll
  for (int c = 0; c < D; ++c) { qr[c] = valid ? q[static_cast<size_t>(row) * cols + h * D + c] : 0.f; acc[c] = 0.f; }
  float m = -INFINITY, l = 0.f;

  for (int j = 0; j < n_kb; ++j) {
    if (mode == 1) {
      const uint32_t w = mask[(static_cast<size_t>(h) * n_qb + i) * W + (j >> 5)];
      if (!((w >> (j & 31)) & 1u)) continue;
    }
    const int k0 = j * B, k1 = min(L, k0 + B);
    for (int t0 = k0; t0 < k1; t0 += kTile) {
      const int cnt = min(kTile, k1 - t0);
      __syncthreads();
      for (int e = threadIdx.x; e < cnt * D; e += blockDim.x) {
        const int t = e / D, c = e % D;
        const int l = t0 + t;
        if (rs.k2 && l >= rs.L) {
          const size_t r2 = static_cast<size_t>(l - rs.L) * cols + h * D + c;
          Ks[t * D + c] = static_cast<const float*>(rs.k2)[r2];
          Vs[t * D + c] = static_cast<const float*>(rs.v2)[r2];
          continue;
        }
        bool ok;
        const long long r = row_of(rs, l, B, ok);
        bad |= !ok;
        Ks[t * D + c] = kb[r * cols + h * D + c];
        Vs[t * D + c] = vb[r * cols + h * D + c];
      }
      __syncthreads();
      if (!valid) continue;
      float sc[kTile];
      float mt = -INFINITY;
      for (int t = 0; t < cnt; ++t) {
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < D; ++c) s = fmaf(qr[c], Ks[t * D + c], s);
        s *= scale;
        sc[t] = s;
        mt = fmaxf(mt, s);
      }
      const float mn = fmaxf(m, mt);
      const float corr = (m == -INFINITY) ? 0.f : expf(m - mn);
      l *= corr;
#pragma unroll
      for (int c = 0; c < D; ++c) acc[c] *= corr;
      for (int t = 0; t < cnt; ++t) {
        const float p = expf(sc[t] - mn);
        l += p;
#pragma unroll
        for (int c = 0; c < D; ++c) acc[c] = fmaf(p, Vs[t * D + c], acc[c]);
      }
      m = mn;
    }
  }
  if (bad && threadIdx.x == 0) atomicOr(err, WA_DEVERR_PAGE_ID);
  if (!valid) return;
  const float inv = l > 0.f ? 1.0f / l : 0.f;
  // mode 1: sigmoid(g); mode 0: the linear branch's weight sigmoid(lin_sign * x), with
  // x = g, lin_sign = -1 (1 - sigmoid(g)) or x = g_lin, lin_sign = +1 (two gates)
  const float g = gate[static_cast<size_t>(row) * H + h];
  const float sg = 1.0f / (1.0f + expf(mode == 0 ? -lin_sign * g : -g));
  const size_t o = static_cast<size_t>(row) * cols + h * D;
#pragma unroll
  for (int c = 0; c < D; ++c) {
    const float v = acc[c] * inv;
    if (o_branch) o_branch[o + c] = v;
    if (mode == 0) lin_ws[o + c] = sg * v;
    else out[o + c] = sg * v + lin_ws[o + c];
  }
}

}  // namespace

wa_status launch_simt_project(const float* x, const int32_t* page_ids, int page_rows, int n_pages,
                              const float* e, int L, int cols, int r, int d, long long e_head_stride,
                              float* out, uint32_t* err, cudaStream_t st) {
  RowSource rs;
  rs.page_ids = page_ids;
  rs.page_rows = page_rows;
  rs.n_pages = n_pages;
  rs.L = L;
  dim3 grid((cols + 127) / 128, r);
  k_simt_project<<<grid, 128, 0, st>>>(x, rs, e, L, cols, r, d, e_head_stride, out, err);
  return check_launch("simt_project");
}

wa_status launch_simt_attention(int mode, const float* q, int Nq, int H, int d, RowSource rs,
                                int B, const uint32_t* blk_mask, int W, const float* gate,
                                const float* gate_lin, float* lin_ws, float* out, float* o_branch,
                                uint32_t* err, cudaStream_t st) {
  const float* gx = (mode == 0 && gate_lin) ? gate_lin : gate;
  const float lin_sign = gate_lin ? 1.f : -1.f;
  const int n_qb = (Nq + B - 1) / B;
  dim3 grid(n_qb, H);
  const size_t smem = 2 * static_cast<size_t>(kTile) * d * sizeof(float);
  if (B > 128) return set_error(WA_ERR_UNSUPPORTED, "fp32 attention needs B <= 128");
  if (d == 64) {
    cudaFuncSetAttribute(k_simt_attention<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k_simt_attention<64><<<grid, 128, smem, st>>>(mode, q, Nq, H, rs, B, blk_mask, W, gx, lin_sign,
                                                  lin_ws, out, o_branch, err);
  } else if (d == 128) {
    cudaFuncSetAttribute(k_simt_attention<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k_simt_attention<128><<<grid, 128, smem, st>>>(mode, q, Nq, H, rs, B, blk_mask, W, gx,
                                                   lin_sign, lin_ws, out, o_branch, err);
  } else {
    return set_error(WA_ERR_UNSUPPORTED, "fp32 attention supports d in {64,128}");
  }
  return check_launch("simt_attention");
}

}  // namespace wa
