/*
 * wa.h -- C ABI of libwa: the Hybrid Sparse Attention (HSA) decode step of
 * WorldAttention over Hierarchical-KV-Cache pages, for NVIDIA B200 (sm_100a).
 *
 * Method: "WorldAttention: An Efficient Attention Architecture for Interactive
 * Video World Models".  Each entry point below names the section of that paper
 * that defines what it computes.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Tensor pointers are DEVICE pointers, owned by the caller.  The library never
 *    allocates device memory on these paths: scratch comes from a caller-provided
 *    workspace `ws` of at least `*_workspace_size(...)` bytes (256-byte aligned).
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *    Every call is asynchronous on that stream; nothing synchronises.
 *  - Layouts are dense and token-major, row-major in the order written:
 *      q, out          [Nq][H][d]
 *      k_pool, v_pool  [n_pool_pages][T_p][H][d]
 *      k_act, v_act    [L][H][d]            (L = K_p * T_p)
 *      e_k, e_v        [L][r]               (shared by all heads)
 *      k_til, v_til    [r][H][d]
 *      gate            [Nq][H]   float32    (gate logits g)
 *      tau             [H]       float32
 *    Block b of a sequence covers rows [b*B, min(N, (b+1)*B)); the last block may be
 *    ragged.  n_qb = ceil(Nq/B), n_kb = ceil(L/B), W = ceil(n_kb/32).
 *  - `dtype` (WA_F32 or WA_BF16) applies to q, k/v, e_k/e_v, k_til/v_til and out.
 *    Scores, page/block means and every quantity that decides an index (page or
 *    block selection) are computed in float64; attention accumulates in float32.
 *  - Supported shapes: d in {64, 128}; B = 64; for WA_BF16 also r in {128, 256}
 *    (the projection's tensor-core tile height).  Others return WA_ERR_UNSUPPORTED.
 *  - Errors: every call validates its scalar arguments on the host and returns a
 *    wa_status; no C++ exception crosses the ABI.  `wa_last_error()` returns a
 *    message for the calling thread's last failure.  Index arguments that live in
 *    device memory (page ids) are checked by the kernels: an out-of-range id is
 *    skipped and recorded in a device error word that `wa_device_error()` reads.
 */
#ifndef WA_H_
#define WA_H_

#include <stddef.h>
#include <stdint.h>

/* Symbols of the C ABI; libwa is built with hidden visibility for everything else. */
#if defined(__GNUC__)
#define WA_API __attribute__((visibility("default")))
#else
#define WA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum wa_status {
  WA_OK = 0,
  WA_ERR_INVALID_ARG = 1,  /* a size, pointer or count is invalid                 */
  WA_ERR_UNSUPPORTED = 2,  /* valid, but outside the shapes this build implements */
  WA_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed          */
  WA_ERR_DEVICE = 4,       /* a kernel recorded a bad device-side index            */
  WA_ERR_WORKSPACE = 5     /* workspace NULL, too small or misaligned              */
} wa_status;

typedef enum wa_dtype { WA_F32 = 0, WA_BF16 = 1 } wa_dtype;

/* Device error word bits, returned through wa_device_error's *flags. */
#define WA_DEVERR_PAGE_ID   0x1u  /* a page id outside [0, n_pool_pages)            */
#define WA_DEVERR_ZERO_NORM 0x2u  /* a zero-norm prompt embedding in prompt select  */
#define WA_DEVERR_TIMEOUT   0x4u  /* a bounded wait inside a kernel gave up         */
#define WA_DEVERR_ROW_ID    0x8u  /* a row index outside [0, n_rows) in wa_permute_rows */

/* Bound of every mbarrier wait inside the kernels launched after this call, in
 * nanoseconds of %globaltimer time (process-wide; 2 s by default).  A wait that runs
 * out sets WA_DEVERR_TIMEOUT, makes the kernel's other roles stop, waits (within the
 * same bound) for the loads and MMAs the kernel itself had issued, frees its TMEM
 * and returns.  No counterpart in the paper: it is the runtime's failure detection.
 * INVALID_ARG outside [1e3, 6e10]. */
WA_API wa_status wa_set_wait_limit_ns(uint64_t limit_ns);
WA_API uint64_t wa_get_wait_limit_ns(void);

/* Failure-detection self-test (no counterpart in the paper).  Launches one CTA that
 * waits, through the kernels' bounded wait limited to limit_ns, on an mbarrier that no
 * thread ever arrives at.  The wait gives up: the kernel sets WA_DEVERR_TIMEOUT in the
 * device error word (read it with wa_device_error) and returns, with no load or MMA
 * in flight, so the context stays usable.  elapsed_ns (device, nullable) receives the
 * %globaltimer time the wait took.  INVALID_ARG: limit_ns outside [1e3, 1e9]. */
WA_API wa_status wa_check_bounded_wait(uint64_t limit_ns, uint64_t* elapsed_ns, void* stream);

/* Message describing the calling thread's most recent failure ("" if none). */
WA_API const char* wa_last_error(void);

/* Library version string. */
WA_API const char* wa_version(void);

/* Synchronise `stream`, read and clear the current device's error word.
 * *flags (may be NULL) receives the WA_DEVERR_* bits.  Returns WA_ERR_DEVICE when
 * any bit was set, WA_OK otherwise. */
WA_API wa_status wa_device_error(void* stream, uint32_t* flags);

/* ---------------------------------------------------------------------------
 * S0 -- prompt-level retrieval (WorldAttention §3.2, "Stage 1: prompt-level
 * retrieval"): the index of the history chunk whose prompt embedding has the
 * largest cosine similarity with the current prompt embedding (ties -> lowest).
 *   e_cur    [D] float32        current prompt embedding
 *   e_chunks [n_chunks][D] f32  one embedding per history chunk
 *   chunk_out[1] int32          the chosen chunk; -1 and WA_DEVERR_ZERO_NORM when a
 *                               norm is zero
 * Computed in float64.  INVALID_ARG: NULL pointer, n_chunks < 1, D < 1. */
WA_API wa_status wa_prompt_select(const float* e_cur, const float* e_chunks, int n_chunks, int D,
                           int32_t* chunk_out, void* stream);

/* ---------------------------------------------------------------------------
 * S1 -- page-level retrieval (WorldAttention §3.2, "Stage 2: page-level
 * retrieval", the equation alpha_{m,j} = Qbar^T Kbar_{m,j} / sqrt(d_k)): with
 * Qbar_h the mean query of head h over the chunk and Kbar_{h,j} the mean key of
 * candidate page j,  alpha_j = (1/H) sum_h Qbar_h . Kbar_{h,j} / sqrt(d); the
 * top-K_p pages (ties -> lower candidate position) are kept.
 *   q          [Nq][H][d]                queries of the current chunk
 *   k_pool     [n_pool_pages][T_p][H][d] key page pool
 *   cand_pages [n_c] int32 (device)      pool page ids of the candidate chunk
 *   alpha      [n_c] float64 (out)       page scores
 *   sel        [K_p] int32 (out)         chosen POOL PAGE IDS, in ascending
 *                                        candidate position (chronological order)
 *   k_blockmean[n_c][T_p/B][H][d] f64    (out, nullable) mean key of every B-row
 *                                        block of every candidate page; needs
 *                                        T_p % B == 0
 * One HBM pass over q and the candidate pages.  INVALID_ARG: K_p > n_c, sizes < 1,
 * NULL required pointer.  A candidate id outside the pool sets WA_DEVERR_PAGE_ID. */
WA_API size_t wa_page_score_workspace_size(int Nq, int H, int d, int n_c, int T_p, int B);
WA_API wa_status wa_page_score(const void* q, int Nq, int H, int d,
                        const void* k_pool, int n_pool_pages, int T_p,
                        const int32_t* cand_pages, int n_c, int K_p, int B, wa_dtype dtype,
                        double* alpha, int32_t* sel, double* k_blockmean,
                        void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * S2 -- active KV construction (WorldAttention §3.2, "Active KV construction";
 * summary step 4, the concatenation of the selected pages into K_active and
 * V_active): k_act[s*T_p + t] = k_pool[sel[s]][t], likewise for V.  A bit-exact
 * copy.  A page id outside the pool sets WA_DEVERR_PAGE_ID and that page is
 * skipped. */
WA_API wa_status wa_gather_pages(const void* k_pool, const void* v_pool, int n_pool_pages, int T_p,
                          int H, int d, const int32_t* sel, int K_p, wa_dtype dtype,
                          void* k_act, void* v_act, void* stream);

/* ---------------------------------------------------------------------------
 * Page pool maintenance (WorldAttention §3.2, "page-level KV abstraction" and the
 * L1 tier, which holds the retrieved KV pages "along with ... page indices
 * constructed from the keys K").
 *
 * The page index is a float64 array of B-row block SUMS of the keys:
 *   page_index [n_pool_pages][T_p/B][H][d]  (needs T_p % B == 0)
 * Block means, page means and therefore the page scores (S1) and the pooled block
 * scores (S3) follow from it without re-reading the keys.
 *
 * wa_pool_index: (re)compute the index entries of pages[0..n_pages) (device ids).
 * wa_pool_append: copy n_tokens new rows of K and V (k_new, v_new [n_tokens][H][d])
 *   into the pool's flat token space at rows [token_offset, token_offset + n_tokens)
 *   (a chunk may span page boundaries); when page_index is non-NULL, also refresh
 *   the index entries of every block the write touches (a block's entry is exact
 *   once all its rows are written).  INVALID_ARG: rows outside the pool. */
WA_API wa_status wa_pool_index(const void* k_pool, int n_pool_pages, int T_p, int H, int d, int B,
                        wa_dtype dtype, const int32_t* pages, int n_pages, double* page_index,
                        void* stream);
WA_API wa_status wa_pool_append(void* k_pool, void* v_pool, int n_pool_pages, int T_p, int H, int d,
                         wa_dtype dtype, const void* k_new, const void* v_new, int n_tokens,
                         long long token_offset, double* page_index, int B, void* stream);

/* ---------------------------------------------------------------------------
 * Token order: 3-D cube tiles (WorldAttention Appendix A.1.3, "Block Sparse
 * Attention": the flattened token sequence is re-indexed so that every contiguous
 * group of B tokens is one (C_t, C_h, C_w) cube of the video volume, so that a
 * selected or skipped block is a spatio-temporal cube).  The pages lost the index
 * formula; the reading implemented here: the tokens of a grid of T frames x H_l
 * rows x W_l columns (raster index (t*H_l + h)*W_l + w) are ordered cube by cube,
 * the cubes in raster order of their corners (t_c, h_c, w_c) and the tokens inside
 * a cube in raster order.  Where a grid side is not a multiple of the cube side the
 * last cube along it is cut short, so groups of C_t*C_h*C_w tokens are exact cubes
 * only when C_t | T, C_h | H_l and C_w | W_l (an 8-frame page of 30 x 52 latents
 * with (8, 2, 4) cubes: 195 cubes of 64 tokens, one per key block).  Attention over
 * cube-ordered keys is the same computation; only the blocks that selection pools
 * and keeps change.
 *
 * wa_cube_order: host function, no device work.  perm[n] (n in [0, T*H_l*W_l)) is
 *   the raster index of the token at cube-order position n; perm is caller-owned
 *   host memory of T*H_l*W_l int32.  INVALID_ARG: a size < 1, NULL perm, or more
 *   than 2^31 - 1 tokens.
 * wa_permute_rows: row permutation of [n_rows][row_bytes] device data on `stream`:
 *     inverse == 0:  dst[n] = src[perm[n]]   (raster -> cube order with wa_cube_order's perm)
 *     inverse != 0:  dst[perm[n]] = src[n]   (cube -> raster order)
 *   perm: device int32 [n_rows], a permutation of [0, n_rows); src and dst must not
 *   overlap; row_bytes a multiple of 16 and both pointers 16-byte aligned
 *   (UNSUPPORTED otherwise).  A bit-exact copy.  An entry of perm outside
 *   [0, n_rows) sets WA_DEVERR_ROW_ID and that row is skipped.  INVALID_ARG: NULL
 *   pointer, n_rows < 1 or above 2^31 - 2^20, row_bytes == 0. */
WA_API wa_status wa_cube_order(int T, int H_l, int W_l, int C_t, int C_h, int C_w, int32_t* perm);
WA_API wa_status wa_permute_rows(const void* src, void* dst, const int32_t* perm, int n_rows,
                                 size_t row_bytes, int inverse, void* stream);

/* ---------------------------------------------------------------------------
 * S3 -- head-adaptive block selection (WorldAttention §3.3, "Head-level sparsity
 * adaptation": per head the minimal set of blocks whose cumulative attention mass
 * reaches tau_h; summary step 5, block-pooled coarse selection).  For head h and
 * query block i: qbar, kbar are the means over the valid rows of each block;
 * s_j = qbar_i . kbar_j / sqrt(d); p = softmax_j(s); blocks sorted by s descending
 * (ties -> lower j); the shortest prefix whose mass sum reaches tau_h (>=) is kept.
 * tau_h >= 1, or a prefix sum that never reaches tau_h, keeps every block.
 *   q           [Nq][H][d]
 *   k_act       [L][H][d]        keys whose block means are pooled, or NULL
 *   k_blockmean [n_kb][H][d] f64 precomputed key block means, or NULL
 *                                (exactly one of k_act, k_blockmean is non-NULL)
 *   tau         [H] float32
 *   blk_idx     [H][n_qb][n_kb] int32 (out, nullable) kept blocks ascending, then -1
 *   blk_cnt     [H][n_qb] int32 (out, nullable)       number of kept blocks
 *   blk_mask    [H][n_qb][W] uint32 (out, nullable)   bit j of word j/32 = kept
 * INVALID_ARG: both or neither key sources, NULL q/tau, n_kb > 8192. */
WA_API size_t wa_block_select_workspace_size(int Nq, int H, int d, int L, int B);
WA_API wa_status wa_block_select(const void* q, int Nq, int H, int d,
                          const void* k_act, const double* k_blockmean, int L, int B,
                          wa_dtype dtype, const float* tau,
                          int32_t* blk_idx, int32_t* blk_cnt, uint32_t* blk_mask,
                          void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * S4a -- Linformer projection of the linear branch (WorldAttention §3.3, "Linear
 * branch": K~ = E_K^T K, V~ = E_V^T V with rank r << L, following Wang et al.
 * 2020): k_til[c][h][:] = sum_l e_k[l][c] * k_act[l][h][:], likewise v_til.
 * E is shared by all heads.  Accumulates in float32 (bf16 inputs on tcgen05
 * tensor cores with split-L and an ordered reduction); the result is rounded to
 * dtype. */
WA_API size_t wa_linear_project_workspace_size(int L, int H, int d, int r, wa_dtype dtype);
WA_API wa_status wa_linear_project(const void* k_act, const void* v_act, const void* e_k,
                            const void* e_v, int L, int H, int d, int r, wa_dtype dtype,
                            void* k_til, void* v_til, void* ws, size_t ws_bytes,
                            void* stream);

/* The same with one projection per head (main text §3.3, "Linear branch", writes
 * K~^(h) = E_K^T K^(h)): e_k, e_v are [H][L][r] with e_head_stride = L*r elements
 * (0 falls back to wa_linear_project: one E for every head).  The workspace is at most
 * wa_linear_project_workspace_size's.  INVALID_ARG: any other stride. */
WA_API wa_status wa_linear_project_heads(const void* k_act, const void* v_act, const void* e_k,
                                         const void* e_v, int L, int H, int d, int r,
                                         wa_dtype dtype, long long e_head_stride, void* k_til,
                                         void* v_til, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * The S4a projection for callers that cannot allocate device memory.  The paper
 * has no counterpart to this entry point.
 *
 * Some callers cannot call cudaMalloc and have no workspace to hand over: code
 * that runs inside a host framework which owns every device allocation through
 * its own pool, or a real-time loop where an allocation (which can synchronise
 * the device) is not allowed.  This call computes what wa_linear_project computes
 * for bf16 inputs, on the same tcgen05 kernels, to within the order of the float32
 * sums over L: when the scratch is the limit it uses fewer splits of L than the
 * workspace entry point, and the partials are then added in a different grouping.
 * It keeps its split-L partial sums in a fixed 32 MiB array that the library holds
 * as a file-scope device variable: every GPU that loads libwa holds those 32 MiB
 * until the process exits.  It calls no cudaMalloc, cudaFree or other allocating
 * routine.
 *   - The caller still passes inputs and outputs (same layouts as
 *     wa_linear_project; contiguous k_act / v_act [L][H][d], e_k / e_v [L][r]).
 *   - The first call on a device looks the array's device address up
 *     (cudaGetSymbolAddress, once per device, with that device current); make that
 *     first call before any stream capture.  The address is kept for the life of
 *     the process and belongs to the device's primary context: after a
 *     cudaDeviceReset on that device it is stale, so do not call this entry point
 *     on a device again once it has been reset.
 *   - All calls share the array, which keeps the last call's contents.  Each call
 *     writes every partial it later reads, so no earlier contents leak into a
 *     result; but calls that overlap on the GPU (two streams at once) race on it
 *     and must be ordered by the caller.
 *   - Sizes whose partials do not fit (2 * r * H * d * 4 bytes per split of L above
 *     32 MiB) are rejected with WA_ERR_UNSUPPORTED and a message; larger problems use
 *     fewer splits of L, down to one.
 *   - dtype must be WA_BF16, d in {64, 128}, r in {128, 256}, H*d % 64 == 0. */
WA_API wa_status wa_linear_project_noalloc(const void* k_act, const void* v_act, const void* e_k,
                                    const void* e_v, int L, int H, int d, int r, wa_dtype dtype,
                                    void* k_til, void* v_til, void* stream);

/* ---------------------------------------------------------------------------
 * S4b + S5 + S6 -- the two attention branches and their gate (WorldAttention
 * §3.3: "Linear branch" O_lin = softmax(Q K~^T / sqrt(d)) V~; "Sparse branch",
 * exact attention restricted to the selected key blocks, Appendix A.1.3;
 * "Gated fusion of two branches" with a sigmoid gate):
 *   out[n][h] = sigmoid(g[n][h]) * O_sp[n][h] + (1 - sigmoid(g[n][h])) * O_lin[n][h]
 *   q        [Nq][H][d]
 *   k_act, v_act [L][H][d]
 *   blk_mask [H][n_qb][W] uint32   key blocks kept for each (head, query block)
 *   k_til, v_til [r][H][d]
 *   gate     [Nq][H] float32
 *   out      [Nq][H][d] (dtype)
 *   o_sp, o_lin [Nq][H][d] float32 (out, nullable): the two branch outputs before
 *                                  the gate, for identity checks
 * A (head, query block) whose mask is empty gets O_sp = 0.  Masked key rows of a
 * ragged last block never enter a softmax. */
WA_API size_t wa_hsa_attention_workspace_size(int Nq, int H, int d, int L, int B, int r, wa_dtype dtype);
WA_API wa_status wa_hsa_attention(const void* q, int Nq, int H, int d,
                           const void* k_act, const void* v_act, int L, int B,
                           const uint32_t* blk_mask,
                           const void* k_til, const void* v_til, int r,
                           const float* gate, wa_dtype dtype,
                           void* out, float* o_sp, float* o_lin,
                           void* ws, size_t ws_bytes, void* stream);

/* The same with two independent gates, one per branch (WorldAttention §3.3, "Gated
 * fusion of two branches": sigmoid gates modulate both branches per token and head;
 * the section's formula O_lin ⊙ G_lin + O_sp ⊙ G_sp with G = sigmoid of the gate
 * logits):
 *   out[n][h] = sigmoid(gate_sp[n][h]) * O_sp[n][h] + sigmoid(gate_lin[n][h]) * O_lin[n][h]
 *   gate_sp, gate_lin [Nq][H] float32 (gate_lin must not be NULL); the logits are
 * inputs (the projection G = XW that makes them belongs to the model).  With
 * gate_lin = -gate_sp this is wa_hsa_attention.  Same workspace, errors and
 * layouts as wa_hsa_attention. */
WA_API wa_status wa_hsa_attention_gated2(const void* q, int Nq, int H, int d,
                                  const void* k_act, const void* v_act, int L, int B,
                                  const uint32_t* blk_mask,
                                  const void* k_til, const void* v_til, int r,
                                  const float* gate_sp, const float* gate_lin, wa_dtype dtype,
                                  void* out, float* o_sp, float* o_lin,
                                  void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * The whole decode step (WorldAttention §3.2 + §3.3; summary steps 2-6):
 * S0 (when e_cur != NULL) -> S1 -> S2 (or page-table addressing) -> S3 -> S4 ->
 * S5 -> S6, all on the device with no host round trip.
 * With fused_gather != 0 (needs T_p % B == 0) the projection and the sparse
 * branch read K/V straight from the pool pages through `sel`, so no K_active /
 * V_active copy is made; otherwise the selected pages are first gathered into
 * the workspace. */
typedef struct wa_step_args {
  /* S0, optional: when e_cur is NULL the candidate chunk is row 0 of chunk_pages */
  const float* e_cur;          /* [D] float32                                  */
  const float* e_chunks;       /* [n_chunks][D] float32                        */
  int n_chunks;
  int D;
  const int32_t* chunk_pages;  /* [n_chunks][n_c] pool page ids (device)       */
  int n_c;
  /* queries, pool and parameters */
  const void* q;               /* [Nq][H][d]                                   */
  int Nq, H, d;
  const void* k_pool;          /* [n_pool_pages][T_p][H][d]                    */
  const void* v_pool;
  int n_pool_pages, T_p;
  int K_p, B, r;
  const void* e_k;             /* [K_p*T_p][r]                                 */
  const void* e_v;
  const float* tau;            /* [H]                                          */
  const float* gate;           /* [Nq][H]                                      */
  wa_dtype dtype;
  int fused_gather;
  /* output */
  void* out;                   /* [Nq][H][d]                                   */
  /* optional outputs (NULL to skip) */
  int32_t* chunk_out;          /* [1]                                          */
  double* alpha_out;           /* [n_c]                                        */
  int32_t* sel_out;            /* [K_p]                                        */
  uint32_t* blk_mask_out;      /* [H][n_qb][W]                                 */
  void* k_til_out;             /* [r][H][d]                                    */
  void* v_til_out;
  /* optional timing: NULL, or WA_STEP_EVENTS cudaEvent_t handles (as void*) that
     are recorded on `stream` at the stage boundaries listed below */
  void* const* stage_events;
  /* optional page index (see wa_pool_index), [n_pool_pages][T_p/B][H][d] float64
     block sums kept current by the caller; with it S1 and S3 read the index instead
     of re-reducing the candidate pages (needs fused_gather and T_p % B == 0) */
  const double* page_index;
  /* optional second gate, [Nq][H] float32: with it the step fuses the branches as
     sigmoid(gate) * O_sp + sigmoid(gate_lin) * O_lin (see wa_hsa_attention_gated2);
     NULL keeps sigmoid(gate) * O_sp + (1 - sigmoid(gate)) * O_lin */
  const float* gate_lin;
  /* optional intra-chunk keys (main text §3.3, "Inter- and intra-chunk sparse
     granularity"): the current chunk's own keys and values, [Nq][H][d] in the step's
     dtype, both or neither.  With them the sparse branch's key sequence is the
     retrieved history followed by these Nq rows, block selection (S3) runs over all
     its blocks jointly, and blk_mask_out covers ceil((K_p*T_p + Nq)/B) blocks; the
     linear branch stays over the history.  Needs K_p*T_p % B == 0. */
  const void* k_cur;
  const void* v_cur;
  /* optional inter-chunk granularity (main text §3.3, "Inter- and intra-chunk sparse
     granularity": blocks of 128 tokens for the retrieved history pages, 64 for the
     current chunk): the block size of the history in block selection, 0 or B (the
     default: B everywhere) or 2*B.  With 2*B the history's selection blocks are
     consecutive 2B-token windows of the concatenated history (K_active; a block may
     span two adjacent pages), the chunk's own keys and the queries keep blocks of B,
     and one softmax runs over all key blocks of a row.  blk_mask_out stays at B-token
     granularity (a kept history block sets its two B-token blocks).  2*B needs
     K_p*T_p % B == 0. */
  int B_inter;
  /* optional per-head projections (main text §3.3, "Linear branch", K~^(h)): 0 (the
     default) when e_k / e_v are one [K_p*T_p][r] matrix for every head, or
     K_p*T_p*r when they are [H][K_p*T_p][r], one matrix per head (elements). */
  long long e_head_stride;
} wa_step_args;

/* Stage boundaries recorded into wa_step_args.stage_events:
 *   0 start | 1 after S0+S1 (page retrieval) | 2 after S2 (gather; = 1 when fused)
 *   3 after S3 (block selection) | 4 after S4a (projection) | 5 after S4b (linear
 *   branch) | 6 after the work list | 7 after S5+S6 (sparse branch + gate).
 * With bf16 inputs the step forks two internal streams after event 2 and joins them
 * before event 6: S4a and S4b run on one (events 4 and 5 are recorded there), S3 and
 * the work list on the other, which has the device's highest stream priority (event 3
 * is recorded there).  Events on different streams compare by time as usual. */
#define WA_STEP_EVENTS 8

WA_API size_t wa_hsa_step_workspace_size(const wa_step_args* a);
WA_API wa_status wa_hsa_step(const wa_step_args* a, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * A decode-step pipeline over host buffers (no counterpart in the pages: serving
 * plumbing).  Each submit uploads q and the gate logits from host memory, runs
 * wa_hsa_step and downloads out, on three streams so that step k+1's upload and step
 * k-1's download overlap step k.  Two device sets of (q, gate, out) alternate: set 0
 * is a->q / a->gate / a->out, set 1 is q1 / gate1 / out1 (same shapes).  Every
 * other field of *a (pool, E, tau, optional inputs) is copied once and used by every
 * step; ws (wa_hsa_step_workspace_size(a) bytes) is shared by the steps, which run in
 * order on `stream`.  Host buffers should be pinned for the copies to be
 * asynchronous; inputs must stay unchanged and outputs unread until wa_pipe_sync (or
 * work ordered after wa_pipe_end on `stream`).
 *   wa_pipe_begin   later copies wait for everything enqueued on `stream` so far
 *   wa_pipe_end     `stream` waits for every copy submitted so far
 *   wa_pipe_sync    waits on the host for everything submitted
 * A pipeline is driven from one host thread at a time (it keeps no lock). */
typedef struct wa_pipe wa_pipe;
WA_API wa_status wa_pipe_create(const wa_step_args* a, void* q1, const float* gate1, void* out1,
                                void* ws, size_t ws_bytes, void* stream, wa_pipe** out);
WA_API wa_status wa_pipe_destroy(wa_pipe* p);
WA_API wa_status wa_pipe_begin(wa_pipe* p);
WA_API wa_status wa_pipe_submit(wa_pipe* p, const void* q_host, const float* gate_host,
                                void* out_host);
WA_API wa_status wa_pipe_end(wa_pipe* p);
WA_API wa_status wa_pipe_sync(wa_pipe* p);

/* ---------------------------------------------------------------------------
 * L1 <-> L2 page tiering (WorldAttention §3.2, "Hierarchical KV Cache": pages that
 * are not active leave GPU memory for CPU DRAM by LRU and return on demand; pages
 * predicted to be needed are prefetched asynchronously).
 *
 * A tier owns no memory.  The caller gives
 *   slot_k, slot_v  device pool of n_slots page slots, [n_slots][page_bytes] each
 *                   (the L1 tier; a step uses it as its k_pool / v_pool)
 *   host_k, host_v  pinned host memory (cudaHostAlloc) holding every page,
 *                   [n_pages][page_bytes] each (the L2 tier)
 * and keeps all four alive until wa_tier_destroy.  With all four NULL the tier only
 * keeps the books (page -> slot map, LRU order, dirty bits, statistics), with no
 * copies.  One caller stream should be used for a tier's ensure / release / flush
 * calls and for the kernels that read its slots.
 *
 *   wa_tier_ensure    makes `pages` resident and writes their slots to slots_out
 *                     (host array of n).  Misses are filled in order on `stream`:
 *                     a free slot if any, else the least recently handed-out slot
 *                     not in this request; a dirty victim is first written back to
 *                     its host page.  A page whose prefetch is in flight makes
 *                     `stream` wait for it.  More distinct pages than slots is
 *                     WA_ERR_INVALID_ARG.
 *   wa_tier_release   the work that reads every slot handed out so far has been
 *                     enqueued on `stream`: those slots may now be evicted by
 *                     prefetches (which wait on this point of `stream`).
 *   wa_tier_prefetch  loads the non-resident `pages` on the tier's own stream into
 *                     free slots or released LRU slots; a hint: it stops when no
 *                     slot qualifies.  *issued (nullable) = pages started.
 *   wa_tier_mark_dirty  the resident `page` was written on the device (an appended
 *                     chunk): it is written back when evicted or flushed.
 *   wa_tier_flush     writes every dirty resident page back on `stream`.
 *   wa_tier_slot_of   the slot of `page`, or -1.
 * The calls of one tier may come from several host threads (an internal lock
 * orders them).  Errors: WA_ERR_INVALID_ARG (bad ids, sizes, NULL), WA_ERR_CUDA (a
 * copy or event call failed). */
typedef struct wa_tier wa_tier;
typedef struct wa_tier_stats {
  long long hits, misses, prefetch_hits, prefetches, evictions, writebacks;
  long long bytes_h2d, bytes_d2h;
} wa_tier_stats;
WA_API wa_status wa_tier_create(int n_pages, int n_slots, size_t page_bytes, void* host_k,
                                void* host_v, void* slot_k, void* slot_v, wa_tier** out);
WA_API wa_status wa_tier_destroy(wa_tier* t);
WA_API wa_status wa_tier_ensure(wa_tier* t, const int32_t* pages, int n, int32_t* slots_out,
                                void* stream);
WA_API wa_status wa_tier_release(wa_tier* t, void* stream);
WA_API wa_status wa_tier_prefetch(wa_tier* t, const int32_t* pages, int n, int* issued);
WA_API wa_status wa_tier_mark_dirty(wa_tier* t, int32_t page);
WA_API wa_status wa_tier_flush(wa_tier* t, void* stream);
WA_API wa_status wa_tier_slot_of(wa_tier* t, int32_t page, int32_t* slot);
WA_API wa_status wa_tier_get_stats(wa_tier* t, wa_tier_stats* out);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* WA_H_ */
