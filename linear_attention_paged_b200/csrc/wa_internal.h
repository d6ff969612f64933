// wa_internal.h -- declarations shared by the translation units of libwa.
// Not part of the public ABI (see include/wa.h).
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/wa.h"

namespace wa {

// Where the rows of a key/value sequence live.  Block j (B rows) of the active
// sequence starts at row
//     page_ids[j / blocks_per_page] * page_rows + (j % blocks_per_page) * B
// of the base arrays; with page_ids == nullptr the sequence is one contiguous
// buffer (row = j * B).  page_ids are checked against n_pages.
struct RowSource {
  const void* k = nullptr;
  const void* v = nullptr;
  const int32_t* page_ids = nullptr;  // device, nullable
  int page_rows = 0;                  // T_p (paged) or L (contiguous)
  int n_pages = 1;                    // pool pages addressable from k / v
  int L = 0;                          // rows of the active sequence
  // optional second segment (the current chunk's own keys and values): rows
  // [L, L + L2) of the key sequence, contiguous [L2][H][d]; L is then a multiple of
  // the block size, so no block straddles the two segments
  const void* k2 = nullptr;
  const void* v2 = nullptr;
  int L2 = 0;
};

// Status of an internal launch: WA_OK or WA_ERR_CUDA with a message set.
wa_status set_error(wa_status s, const char* fmt, ...);
wa_status check_launch(const char* what);
uint32_t* device_error_word();  // current device's error word (device address)
// Bound, in nanoseconds of %globaltimer time, of every mbarrier wait in the kernels
// launched from now on (wa_set_wait_limit_ns; 2 s by default).
uint64_t wait_limit_ns();

// ---------------------------------------------------------------- selection
// S0: cosine of every chunk embedding with the current one, argmax -> chunk_out.
wa_status launch_prompt_select(const float* e_cur, const float* e_chunks, int n_chunks, int D,
                               int32_t* chunk_out, uint32_t* err, cudaStream_t st);

// Row-block sums in float64 over B-row blocks of `n_src` sources of `rows` rows
// each (a source is a pool page given by src_ids, or the buffer itself when
// src_ids == nullptr), cols = H*d columns:
//   blocksum[s][b][c]  (nullable)  sum of rows [b*B, min(rows,(b+1)*B)) of source s
//   kdot[s][split][cc] (with qbar) dot product of qbar with the CTA's column sums
struct RowsumPlan {
  int threads = 0;   // threads per CTA (V columns each)
  int n_cc = 1;      // column chunks
  int nb = 0;        // blocks per source (also the source stride of blocksum)
  int bps = 1;       // blocks per CTA
  int n_split = 1;   // CTAs per source and column chunk
  int block0 = 0;    // first block summed
  int n_blocks = 0;  // blocks summed (from block0)
  int by_page = 0;   // blocksum indexed by pool page id instead of source position
};
RowsumPlan rowsum_plan(int n_src, int rows, int cols, int B, wa_dtype dt);
// Plan over blocks [block0, block0 + n_blocks) of one source of `rows` rows.
RowsumPlan rowsum_plan_range(int rows, int cols, int B, wa_dtype dt, int block0, int n_blocks);
// kdot[c][b] = qbar . page_index[cand[c]][b] (page scores from the page index);
// cand == nullptr reads row c (block sums indexed by candidate position).
wa_status launch_index_dot(const double* page_index, const int32_t* cand, int n_c, int n_pages,
                           int nbp, int cols, const double* qbar, double* kdot, uint32_t* err,
                           cudaStream_t st);
wa_status launch_rowblock_sum(const void* x, wa_dtype dt, const int32_t* src_ids, int n_src,
                              int n_pages, int rows, int cols, int B, double* blocksum,
                              const double* qbar, double* kdot, const RowsumPlan& p, uint32_t* err,
                              cudaStream_t st);
// qbar[c] = sum_i qsum[i][c] / Nq; qmean[i][c] (nullable) = qsum[i][c] / rows of block i.
wa_status launch_qmeans(const double* qsum, int n_qb, int Nq, int B, int cols, double* qbar,
                        double* qmean, cudaStream_t st);
// S1 tail: alpha[c] from the K pass's dot products (per_page scalars per page), then
// top-K_p -> sel (pool ids) and sel_pos (candidate positions), ascending position.
wa_status launch_alpha_topk(const double* kdot, int per_page, int n_c, int T_p, int H, int d,
                            int K_p, const int32_t* cand, double* alpha, int32_t* sel,
                            int32_t* sel_pos, cudaStream_t st);

// dst[i] = src[i] * scale (float64).
wa_status launch_scale_copy(const double* src, double* dst, size_t n, double scale,
                            cudaStream_t st);

// Key block means source for block selection.
struct KeyMeans {
  const double* data = nullptr;   // [*][cols] fp64 means or sums
  const int32_t* page_pos = nullptr;  // nullable: block j -> row page_pos[j/nbp]*nbp + j%nbp
  int nbp = 0;                    // blocks per page (when page_pos != nullptr)
  int is_sum = 0;                 // data holds sums: divide by the block's row count
  int L = 0;                      // rows of the key sequence (for ragged counts)
  // optional second segment: blocks j >= n_kb1 read fp64 sums data2[j - n_kb1],
  // over L2 rows
  const double* data2 = nullptr;
  int n_kb1 = 0;
  int L2 = 0;
};
// S3: float64 pooled block scores into `scores` [H][n_qb][n_kb], then per (head,
// query block) the shortest descending prefix reaching tau_h.
size_t block_scores_bytes(int H, int n_qb, int n_kb);
wa_status launch_block_select(const double* q_blockmean, int Nq, int H, int d, int B,
                              KeyMeans km, int n_kb, const float* tau, double* scores,
                              int32_t* blk_idx, int32_t* blk_cnt, uint32_t* blk_mask,
                              cudaStream_t st);

// ---------------------------------------------------------------- gather
wa_status launch_gather(const void* k_pool, const void* v_pool, int n_pages, size_t page_bytes,
                        const int32_t* sel, int K_p, void* k_act, void* v_act, uint32_t* err,
                        cudaStream_t st);

// dst[0..n16) = src[0..n16) in 16-byte units.
wa_status launch_copy16(const void* src, void* dst, size_t n16, cudaStream_t st);
wa_status launch_permute_rows(const void* src, void* dst, const int32_t* perm, int n_rows,
                              size_t row_bytes, int inverse, uint32_t* err, cudaStream_t st);

// ---------------------------------------------------------------- fp32 SIMT path
wa_status launch_simt_project(const float* x, const int32_t* page_ids, int page_rows, int n_pages,
                              const float* e, int L, int cols, int r, float* out,
                              uint32_t* err, cudaStream_t st);
// mode 0: linear branch over (k_til, v_til), writes lin_ws = w * O_lin with
//         w = 1 - sigmoid(g), or sigmoid(g_lin) when gate_lin is given (two gates)
// mode 1: sparse branch over blk_mask, writes out = sigmoid(g)*O_sp + lin_ws
wa_status launch_simt_attention(int mode, const float* q, int Nq, int H, int d, RowSource rs,
                                int B, const uint32_t* blk_mask, int W, const float* gate,
                                const float* gate_lin, float* lin_ws, float* out, float* o_branch,
                                uint32_t* err, cudaStream_t st);

// ---------------------------------------------------------------- bf16 tcgen05 path
size_t umma_project_ws_bytes(int L, int H, int d, int r);
wa_status launch_umma_project(const void* k, const void* v, RowSource rs, const void* e_k,
                              const void* e_v, int L, int H, int d, int r, void* k_til,
                              void* v_til, void* ws, uint32_t* err, cudaStream_t st);

// Linear branch on tcgen05 (keys = k_til/v_til [r][H][d], every block): writes
//   lin_ws[n][h][:] = w * O_lin (fp32) and o_lin (nullable), with w = 1 - sigmoid(g),
//   or sigmoid(g_lin) when gate_lin is given (two independent gates).
wa_status launch_linear_attention(const void* q, int Nq, int H, int d, RowSource lin, int B,
                                  const float* gate, const float* gate_lin, float* lin_ws,
                                  float* o_lin, uint32_t* err, cudaStream_t st);
// Sparse branch on tcgen05 over the kept blocks of blk_mask, fused with the gate:
//   out = bf16(sigmoid(g) * O_sp + lin_ws), o_sp (nullable) = O_sp in fp32.
// `scratch` holds the work list and the split partials (sparse_attn_ws_bytes).
// events (nullable, WA_STEP_EVENTS entries): entry 6 is recorded after the work list.
size_t sparse_attn_ws_bytes(int H, int Nq, int d, int B);
// The two halves of launch_sparse_attention: the work list (pairs + items) from the
// masks, then the attention kernel and the combine.
wa_status launch_attn_worklist(int Nq, int H, int d, int B, int L, const uint32_t* blk_mask,
                               void* scratch, cudaStream_t st);
wa_status launch_attn_sparse(const void* q, int Nq, int H, int d, RowSource rs, int B,
                             const uint32_t* blk_mask, const float* gate, const float* lin_ws,
                             void* out, float* o_sp, void* scratch, uint32_t* err, cudaStream_t st);
wa_status launch_sparse_attention(const void* q, int Nq, int H, int d, RowSource rs, int B,
                                  const uint32_t* blk_mask, const float* gate, const float* lin_ws,
                                  void* out, float* o_sp, void* scratch, uint32_t* err,
                                  cudaStream_t st, void* const* events);

}  // namespace wa
