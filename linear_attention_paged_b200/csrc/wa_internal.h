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

// Float64 sums of B-row blocks, in one persistent pass fed by bulk copies (k_blocksum.cu).
// A segment is `n_src` sources of `rows` rows of `cols` elements: the buffer x itself
// (ids == nullptr, source s at row s * rows) or pool pages (source s is page
// ids[row * n_src + s], row = *chunk or 0).  Blocks [block0, block0 + n_blocks) of every
// source are summed (the last block of a source may be ragged) into
//   sums[((by_page ? page : s) * nb_out + block) * cols + c].
// Up to two segments per launch (e.g. the queries and the candidate pages).  With
// `counter` the launch also zeroes n_counters words for launch_page_alpha.
struct BlockSumSeg {
  const void* x = nullptr;
  const int32_t* ids = nullptr;
  const int32_t* chunk = nullptr;
  int id_rows = 1;        // rows of ids; a chunk index outside [0, id_rows) reads row 0
  int n_src = 1;
  int n_pages = 1;
  int rows = 0;
  int block0 = 0;
  int n_blocks = 0;
  double* sums = nullptr;
  int nb_out = 0;
  int by_page = 0;
};
wa_status launch_block_sums(wa_dtype dt, int cols, int B, const BlockSumSeg* segs, int n_segs,
                            unsigned* counter, int n_counters, uint32_t* err, cudaStream_t st);
// Page scores from block sums: Qbar = sum of qsum rows / Nq (written to qbar, and the
// query block means to qmean when non-null), column sums of each candidate page's
// block sums (ksum rows of page kpage[row][j], or of position j when kpage is null),
// alpha_j = Qbar . colsum_j / (T_p sqrt(d) H), then the top-K_p pages (sel: pool ids
// from cand[row][.], or positions when cand is null; sel_pos: positions), ascending.
// `scratch` holds page_alpha_scratch_doubles(cols, n_c) doubles; the
// page_alpha_counters(cols) words at `counters` must be zero (launch_block_sums zeroes
// them) and are left zero.
size_t page_alpha_scratch_doubles(int cols, int n_c);
int page_alpha_counters(int cols);
wa_status launch_page_alpha(const double* qsum, int n_qb, int Nq, int B, int cols, const double* ksum,
                            const int32_t* kpage, int n_pages, int nbp, const int32_t* cand,
                            const int32_t* chunk, int n_chunks, int n_c, int T_p, int H, int d,
                            int K_p, double* qbar, double* qmean, double* scratch, unsigned* counters,
                            double* alpha, int32_t* sel, int32_t* sel_pos, uint32_t* err,
                            cudaStream_t st);

// qbar[c] = sum_i qsum[i][c] / Nq; qmean[i][c] (nullable) = qsum[i][c] / rows of block i.
wa_status launch_qmeans(const double* qsum, int n_qb, int Nq, int B, int cols, double* qbar,
                        double* qmean, cudaStream_t st);
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
  // history blocks of 2B rows (inter-chunk granularity; needs is_sum): block j < n_kb1
  // is the sum of B-row blocks 2j and 2j + 1 (the latter when < n_sub) of `data`
  int pair = 0;
  int n_sub = 0;
};
// S3: float64 pooled block scores into `scores` [H][n_qb][n_kb], then per (head,
// query block) the shortest descending prefix reaching tau_h.
size_t block_scores_bytes(int H, int n_qb, int n_kb);
// With km.pair the n_kb selection blocks are mixed (history blocks of 2B rows, then
// chunk blocks of B); blk_idx / blk_cnt count them, and blk_mask is written at B-row
// granularity (n_kb_mask blocks: the history's n_sub, then the chunk's) for the
// attention kernel.  Without it n_kb_mask == n_kb.
wa_status launch_block_select(const double* q_blockmean, int Nq, int H, int d, int B,
                              KeyMeans km, int n_kb, int n_kb_mask, const float* tau, double* scores,
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
// out[c][col] = sum_l E_h[l][c] x[l][col], h = col / d, E_h = e + h * e_head_stride
// (e_head_stride 0: one E for every head)
wa_status launch_simt_project(const float* x, const int32_t* page_ids, int page_rows, int n_pages,
                              const float* e, int L, int cols, int r, int d, long long e_head_stride,
                              float* out, uint32_t* err, cudaStream_t st);
// mode 0: linear branch over (k_til, v_til), writes lin_ws = w * O_lin with
//         w = 1 - sigmoid(g), or sigmoid(g_lin) when gate_lin is given (two gates)
// mode 1: sparse branch over blk_mask, writes out = sigmoid(g)*O_sp + lin_ws
wa_status launch_simt_attention(int mode, const float* q, int Nq, int H, int d, RowSource rs,
                                int B, const uint32_t* blk_mask, int W, const float* gate,
                                const float* gate_lin, float* lin_ws, float* out, float* o_branch,
                                uint32_t* err, cudaStream_t st);

// ---------------------------------------------------------------- bf16 tcgen05 path
// e_per_head: E_K, E_V are [H][L][r] (one projection per head); else [L][r], shared.
// The workspace of the shared form is at least that of the per-head form.
size_t umma_project_ws_bytes(int L, int H, int d, int r, bool e_per_head = false);
wa_status launch_umma_project(const void* k, const void* v, RowSource rs, const void* e_k,
                              const void* e_v, int L, int H, int d, int r, void* k_til,
                              void* v_til, void* ws, uint32_t* err, cudaStream_t st,
                              bool e_per_head = false);

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
