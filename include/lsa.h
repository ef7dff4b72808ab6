/*
 * lsa.h -- C ABI of the Lookahead Sparse Attention (LSA) decode hot path on B200.
 *
 * The method ("FlashMemory-DeepSeek-V4 Explained: Replacing Memory Sponge with a
 * Fortune Teller via Lookahead Sparse Attention", zhichai.net, section 2 "Core Idea of
 * LSA", steps 1-5): every tau = 64 decode steps a Neural Memory Indexer projects the
 * current hidden state with one small query encoder per indexer layer (section 3),
 * scores every historical KV block against its frozen compressed key, keeps a block
 * when sigmoid(score) > 0.5 and OR-combines three layers (section 4). The kept blocks
 * move from a host cold pool to the GPU, and the next 64 decode steps attend only to
 * them plus the recent window.
 *
 * Conventions (all entry points):
 *  - Every call returns an lsa_status. Calls never abort, never print, never allocate
 *    device or host memory, and never synchronise the stream they are given.
 *  - All device work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is
 *    the legacy default stream). Pointers marked "device" must be device memory of the
 *    current device; "pinned host" means page-locked host memory the device can map
 *    (cudaHostAlloc / torch pin_memory).
 *  - bf16 tensors are passed as uint16_t bit patterns. Ids and counts are int32,
 *    offsets int64. All layouts are dense row-major.
 *  - Errors found on the host (bad sizes, null pointers, unsupported shapes, a too
 *    small workspace) return LSA_ERR_INVALID_ARG before anything is enqueued.
 *    Errors found by a kernel (capacity overflow, an index out of range) are OR-ed as
 *    LSA_DEVERR_* bits into the caller's device int32 `err` word, which the caller
 *    reads after synchronising; the offending item is skipped, never accessed.
 *  - Ownership: the caller allocates and owns every buffer (inputs, outputs, pools,
 *    block tables, workspaces). A workspace must be zero-filled once before its first
 *    use; every call leaves it ready for the next call.
 *  - Calls that share a workspace or an output must not overlap on the GPU.
 */
#ifndef LSA_H
#define LSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t lsa_status;
#define LSA_OK                0
#define LSA_ERR_INVALID_ARG   1
#define LSA_ERR_CAPACITY      2
#define LSA_ERR_CUDA          3
#define LSA_ERR_TIMEOUT       4
#define LSA_ERR_UNIMPLEMENTED 5

/* bits of the device error word */
#define LSA_DEVERR_SEL_CAPACITY   1  /* a sequence kept more blocks than `cap`; ids past cap dropped */
#define LSA_DEVERR_POOL_CAPACITY  2  /* the HBM pool had no page left for a kept block; block skipped */
#define LSA_DEVERR_BAD_PAGE       4  /* a block-table entry or block id outside its pool; skipped */
#define LSA_DEVERR_BAD_SIZE       8  /* a device-side count (n_cand, n_entries, tail_len) out of range */
#define LSA_DEVERR_TIMEOUT       16  /* a bounded wait gave up */
#define LSA_DEVERR_NUMERIC       32  /* a top-p search did not converge (non-finite logits) */

#define LSA_BLOCK 64                 /* tokens per KV block / pool page */
#define LSA_TAU   64                 /* decode steps per indexer pass */

/* Text of a status code (static storage). */
const char* lsa_status_str(lsa_status s);
/* Library ABI version (major * 100 + minor). */
int32_t lsa_version(void);

/* ---------------------------------------------------------------------------------
 * lsa_index -- one indexer pass (section 2 steps 1-3; sections 3 and 4).
 *
 *   q_l        = W_q[l] . h[l][b]                       (fp32 accumulation, fp32 q)
 *   z_l[b][c]  = q_l . K_idx[kidx_off[b] + c] / sqrt(d_i) + bias[b],  c < n_cand[b]
 *   kept[b][c] = OR_l (z_l[b][c] > 0)                   (sigmoid(z) > 0.5, strict)
 *   sel_ids[b] = the kept c in ascending order; sel_cnt[b] = their number.
 *
 *   h         device bf16 [L][B][D]   hidden state each indexer layer reads
 *   w_q       device bf16 [L][d_i][D] query encoders (row j = weights of q component j)
 *   bias      device f32  [B]         per-sequence logit bias, shared by the layers
 *   k_idx     device bf16 [rows][d_i] frozen compressed block keys (shared by layers)
 *   kidx_off  device i64  [B]         row of block 0 of sequence b in k_idx
 *   n_cand    device i32  [B]         candidate blocks of sequence b (0 <= n <= max_cand)
 *   max_cand  host: bound on every n_cand[b] (sizes the grid and the optional outputs)
 *   sel_ids   device i32  [B][cap]    out; sel_cnt device i32 [B] out (clamped to cap,
 *                                     LSA_DEVERR_SEL_CAPACITY set if it overflowed)
 *   logits    nullable device f32 [L][B][max_cand] out: z_l[b][c] (entries c >= n_cand
 *                                     untouched)
 *   layer_mask nullable device u32 [L+1][B][ceil(max_cand/32)] out: bit c%32 of word
 *             c/32 = (z_l > 0) for l < L, and the OR for l = L
 *   ws        device workspace of lsa_index_workspace_size(B, L, d_i, max_cand) bytes,
 *             16-byte aligned, zero-filled before the first call. Its first 8 bytes are
 *             a grid-barrier counter that grows by twice the grid size per call; the
 *             caller must not change them between calls. A workspace sized for one shape
 *             serves any shape whose size is no larger, on the same device.
 * Supported: 1 <= L <= 4, d_i == 128, D % 256 == 0, B >= 1, cap >= 0. One cooperative
 * launch (one CTA per SM, all resident) with two grid-wide barriers: projection, then
 * scoring, then compaction.
 */
lsa_status lsa_index(const uint16_t* h, const uint16_t* w_q, const float* bias,
                     const uint16_t* k_idx, const int64_t* kidx_off, const int32_t* n_cand,
                     int32_t B, int32_t L, int32_t D, int32_t d_i, int32_t max_cand,
                     int32_t* sel_ids, int32_t* sel_cnt, int32_t cap,
                     float* logits, uint32_t* layer_mask,
                     void* ws, size_t ws_bytes, int32_t* err, void* stream);
size_t lsa_index_workspace_size(int32_t B, int32_t L, int32_t d_i, int32_t max_cand);

/* lsa_index_ex -- lsa_index where each indexer layer may score against its own frozen
 * compressed key table (section 3 of "FlashMemory-DeepSeek-V4 Explained": one small query
 * encoder per indexer layer against precomputed block keys; per-layer tables are the
 * reading where every indexer layer has its own keys):
 *
 *   z_l[b][c] = q_l . K_idx[l * kidx_layer_stride + kidx_off[b] + c] / sqrt(d_i) + bias[b]
 *
 *   kidx_layer_stride  rows between consecutive layers' tables in k_idx (each table laid
 *                      out like the shared one, sequence b's blocks from kidx_off[b]);
 *                      0 = one table shared by all layers (exactly lsa_index).
 * Every other argument, the workspace and the errors are as for lsa_index. Per-layer
 * tables read L x 256 bytes per candidate block instead of 256.
 */
lsa_status lsa_index_ex(const uint16_t* h, const uint16_t* w_q, const float* bias,
                        const uint16_t* k_idx, int64_t kidx_layer_stride,
                        const int64_t* kidx_off, const int32_t* n_cand,
                        int32_t B, int32_t L, int32_t D, int32_t d_i, int32_t max_cand,
                        int32_t* sel_ids, int32_t* sel_cnt, int32_t cap,
                        float* logits, uint32_t* layer_mask,
                        void* ws, size_t ws_bytes, int32_t* err, void* stream);

/* lsa_index_lowrank -- lsa_index_ex with factorised query encoders (section 4 of
 * "FlashMemory-DeepSeek-V4 Explained": a "low-rank query projection (r=2048)"; read here
 * as each layer's encoder being two stacked linear maps through an r-wide latent):
 *
 *   u_l = W_1[l] . h[l][b]          (fp32 accumulation, kept in fp32)
 *   q_l = W_2[l] . u_l              (fp32 accumulation)
 *
 * then scoring, sign test, OR and compaction exactly as lsa_index_ex.
 *   w_1   device bf16 [L][r][D]     down-projection
 *   w_2   device bf16 [L][d_i][r]   up-projection
 *   ws    device workspace of lsa_index_lowrank_workspace_size(B, L, d_i, r, max_cand)
 *         bytes (16-byte aligned, zero-filled before the first call; the same barrier
 *         counter rule as lsa_index, three grid barriers per call)
 * Supported: as lsa_index_ex, plus 256 <= r <= 8192, r % 256 == 0, D <= 16384. The W_1
 * stream (L r D 2 bytes) dominates the bytes read.
 */
lsa_status lsa_index_lowrank(const uint16_t* h, const uint16_t* w_1, const uint16_t* w_2,
                             int32_t r, const float* bias, const uint16_t* k_idx,
                             int64_t kidx_layer_stride, const int64_t* kidx_off,
                             const int32_t* n_cand, int32_t B, int32_t L, int32_t D,
                             int32_t d_i, int32_t max_cand, int32_t* sel_ids, int32_t* sel_cnt,
                             int32_t cap, float* logits, uint32_t* layer_mask,
                             void* ws, size_t ws_bytes, int32_t* err, void* stream);
size_t lsa_index_lowrank_workspace_size(int32_t B, int32_t L, int32_t d_i, int32_t r,
                                        int32_t max_cand);

/* ---------------------------------------------------------------------------------
 * lsa_gather -- move the kept blocks from the host cold pool into the HBM pool
 * (section 2 step 3) and build each sequence's block table.
 *
 *   Kept block j of sequence b (block id c = sel_ids[b][j]) is copied from host pool
 *   block host_blk_off[b] + c to HBM page sel_page_base + sum_{b'<b} sel_cnt[b'] + j
 *   and block_table[b][j] receives that page. Then the sequence's resident pages
 *   (its window, oldest first, with the partially filled tail page last) are appended:
 *   block_table[b][sel_cnt[b] + i] = res_pages[b][i], i < n_res[b];
 *   n_entries[b] = sel_cnt[b] + n_res[b].
 *
 *   host_pool     pinned host bf16 [host_blocks][2][64][d]  (K rows then V rows)
 *   host_blk_off  device i64 [B]
 *   sel_ids/sel_cnt/cap   as produced by lsa_index
 *   res_pages     device i32 [B][res_stride]; n_res device i32 [B] (<= res_stride)
 *   hbm_pool      device bf16 [n_pages][2][64][d]
 *   sel_page_base, sel_page_count   HBM pages reserved for kept blocks; a block that
 *                 does not fit sets LSA_DEVERR_POOL_CAPACITY and is left out
 *   block_table   device i32 [B][bt_stride] out (bt_stride >= cap + res_stride)
 *   n_entries     device i32 [B] out
 * The copy is done by a kernel that reads the pinned host pages over the host link.
 */
lsa_status lsa_gather(const uint16_t* host_pool, int64_t host_blocks,
                      const int64_t* host_blk_off,
                      const int32_t* sel_ids, const int32_t* sel_cnt, int32_t cap,
                      const int32_t* res_pages, const int32_t* n_res, int32_t res_stride,
                      int32_t B, int32_t d,
                      uint16_t* hbm_pool, int64_t n_pages,
                      int32_t sel_page_base, int32_t sel_page_count,
                      int32_t* block_table, int32_t bt_stride, int32_t* n_entries,
                      int32_t* err, void* stream);

/* ---------------------------------------------------------------------------------
 * lsa_gather_delta -- lsa_gather with resident-page reuse across passes (section 2 step 5,
 * "refresh the loaded set"): a block kept by this pass and by the previous one keeps its
 * HBM page and is not copied again; only blocks new to this pass cross the host link,
 * into pages no kept block holds any more. The block table is built as by lsa_gather.
 *
 *   kept_ids, kept_pages  device i32 [B][cap]: the previous pass's kept blocks (ascending)
 *                         and their pages; replaced by this pass's on return
 *   kept_cnt              device i32 [B]: their number (0 at the start of a run; the
 *                         step driver resets it at pass 0)
 *   ws                    device workspace of lsa_gather_delta_workspace_size(B, cap,
 *                         sel_page_count, n_sm) bytes, 16-byte aligned, zeroed before the
 *                         first call (its barrier counters are left at zero)
 *   copied                nullable device i32: incremented by the number of blocks copied
 * Other arguments and errors as for lsa_gather. One cooperative launch (2 CTAs per SM)
 * with three grid barriers; every wait is bounded.
 */
lsa_status lsa_gather_delta(const uint16_t* host_pool, int64_t host_blocks,
                            const int64_t* host_blk_off, const int32_t* sel_ids,
                            const int32_t* sel_cnt, int32_t cap, const int32_t* res_pages,
                            const int32_t* n_res, int32_t res_stride, int32_t B, int32_t d,
                            uint16_t* hbm_pool, int64_t n_pages, int32_t sel_page_base,
                            int32_t sel_page_count, int32_t* block_table, int32_t bt_stride,
                            int32_t* n_entries, int32_t* kept_ids, int32_t* kept_pages,
                            int32_t* kept_cnt, void* ws, size_t ws_bytes, int32_t* copied,
                            int32_t* err, void* stream);
size_t lsa_gather_delta_workspace_size(int32_t B, int32_t cap, int32_t sel_page_count,
                                       int32_t n_sm);

/* ---------------------------------------------------------------------------------
 * lsa_decode_attn -- one decode step of block-sparse MQA attention (section 2 step 4):
 * every query head of sequence b attends to the tokens of the pages listed in its
 * block table, one KV head shared by all heads:
 *
 *   out[b][h] = sum_t softmax_t(scale * q[b][h] . K_t) V_t
 *
 * over t in pages block_table[b][0 .. n_entries[b]-1]; every page holds 64 tokens
 * except the last, which holds tail_len[b] (1..64). A sequence with n_entries 0 gets
 * an all-zero output. The work is split over the SMs (split-K flash decoding on the
 * tensor cores) and the partial results are merged by log-sum-exp.
 *
 *   q           device bf16 [B][H][d]
 *   hbm_pool    device bf16 [n_pages][2][64][d]; tokens of the tail page past
 *               tail_len are read and given zero weight, so they must hold finite
 *               values (zero a page before its first token is appended)
 *   block_table device i32 [B][bt_stride]; entries outside [0, n_pages) set
 *               LSA_DEVERR_BAD_PAGE and are read as zero pages
 *   out         device bf16 [B][H][d] out
 *   ws          device workspace of lsa_decode_attn_workspace_size(B, H, d, n_sm)
 *               bytes, n_sm = multiprocessor count of the current device
 * Supported: d in {128, 256, 384, 512}, 1 <= H <= 64, scale > 0, n_pages <= 2^23,
 *            q, hbm_pool, ws and out 16-byte aligned. The launch is cooperative (one
 *            CTA per SM, all resident): the partial results are merged inside the same
 *            kernel behind a grid-wide barrier whose counters live in the first 256
 *            bytes of ws: they must be zero before the first call, and every call
 *            leaves them zero, so one workspace serves calls of any shape in turn.
 */
lsa_status lsa_decode_attn(const uint16_t* q, const uint16_t* hbm_pool, int64_t n_pages,
                           const int32_t* block_table, int32_t bt_stride,
                           const int32_t* n_entries, const int32_t* tail_len,
                           int32_t B, int32_t H, int32_t d, float scale,
                           uint16_t* out, void* ws, size_t ws_bytes,
                           int32_t* err, void* stream);
size_t lsa_decode_attn_workspace_size(int32_t B, int32_t H, int32_t d, int32_t n_sm);

/* ---------------------------------------------------------------------------------
 * lsa_decode_attn_noalloc -- lsa_decode_attn for callers that cannot allocate device
 * memory (no counterpart on the pages: it is a deployment convenience). Some callers
 * run inside a host framework that owns every allocation, or in a loop that must never
 * enter the CUDA allocator, or receive only their input and output buffers; they
 * cannot provide the workspace lsa_decode_attn needs for its split partials.
 *
 * This entry point takes the same arguments minus the workspace and uses instead one
 * fixed device array inside this library, LSA_NOALLOC_SCRATCH_BYTES large, which every
 * GPU that loads the library holds until the process exits. The call allocates nothing
 * (no cudaMalloc, cudaFree or allocating library routine).
 *  - Limit: lsa_decode_attn_workspace_size(B, H, d, n_sm) must not exceed
 *    LSA_NOALLOC_SCRATCH_BYTES (e.g. B <= 106 at H = 64, d = 512, 148 SMs); larger
 *    problems return LSA_ERR_CAPACITY before anything is enqueued.
 *  - The first call on a device looks up the array's device address and enqueues, on
 *    the caller's stream and ahead of the kernel, a clear of the array's first 256
 *    bytes (the merge barrier counters; the partials are always written before they
 *    are read). Make that first call before any stream capture.
 *  - Every call leaves the counters at zero. A call whose kernel reports
 *    LSA_DEVERR_TIMEOUT may leave them non-zero; later calls in the process are then
 *    unreliable.
 *  - Every call shares the array: calls that overlap on the GPU (other streams,
 *    other host threads) race and produce wrong results. Serialise them.
 *  - The caller still provides and owns q, the pool, the block table, out and err.
 */
#define LSA_NOALLOC_SCRATCH_BYTES (32u << 20)
lsa_status lsa_decode_attn_noalloc(const uint16_t* q, const uint16_t* hbm_pool, int64_t n_pages,
                                   const int32_t* block_table, int32_t bt_stride,
                                   const int32_t* n_entries, const int32_t* tail_len,
                                   int32_t B, int32_t H, int32_t d, float scale,
                                   uint16_t* out, int32_t* err, void* stream);

/* ---------------------------------------------------------------------------------
 * lsa_step -- the decode loop of section 2 (steps 1-5) for a batch of B sequences.
 *
 * Pass p covers global decode steps 64p .. 64p+63. When it starts, sequence b holds
 * N = 64 * nb tokens, nb = nb0[b] + p: blocks [0, nb - wb) are candidates that live
 * only in the host cold pool, blocks [nb - wb, nb) are the recent window (wb = W/64,
 * resident in HBM), and block nb is the tail page that receives the pass's 64 new
 * tokens. The window slides by one block per pass; the current token attends to
 * itself.
 *
 * HBM pool layout owned by the driver: pages [0, B*(wb+1)) are per-sequence window
 * rings (block j of sequence b lives in page b*(wb+1) + j % (wb+1)); pages
 * [B*(wb+1), n_pages) receive the kept blocks of the current pass.
 *
 *   step % 64 == 0: pass set-up kernel (n_cand, resident page lists, write-back of the
 *                   previous tail page to the host pool, zero the new tail page),
 *                   lsa_index on h, lsa_gather of the kept blocks;
 *   every step:     append k_new / v_new at slot step % 64 of each tail page, fused into
 *                   the decode-attention kernel, which writes out.
 * The tail page of the last pass of a run reaches the host pool only when a following
 * pass starts; the window keeps it resident in HBM meanwhile.
 *
 * All pointers in lsa_state are owned by the caller; the struct is plain data.
 */
typedef struct lsa_state {
  int32_t B, L, D, d_i, H, d, W;       /* W: window tokens, a multiple of 64 */
  int32_t cap;                         /* max kept blocks per sequence and pass */
  int32_t max_cand;                    /* >= every candidate count the run reaches */
  float scale;                         /* attention scale, e.g. 1/sqrt(d) */
  /* indexer inputs */
  const uint16_t* w_q;                 /* device bf16 [L][d_i][D] */
  const uint16_t* k_idx;               /* device bf16 [rows][d_i] */
  const int64_t* kidx_off;             /* device i64 [B] */
  const float* bias;                   /* device f32 [B] */
  /* cold pool */
  uint16_t* host_pool;                 /* pinned host bf16 [host_blocks][2][64][d] */
  int64_t host_blocks;
  const int64_t* host_blk_off;         /* device i64 [B+1]: blocks of seq b are
                                          [host_blk_off[b], host_blk_off[b+1]) */
  const int32_t* nb0;                  /* device i32 [B]: context blocks at pass 0 */
  /* HBM pool and per-pass buffers */
  uint16_t* hbm_pool;                  /* device bf16 [n_pages][2][64][d] */
  int64_t n_pages;
  int32_t* n_cand;                     /* device i32 [B] */
  int32_t* sel_ids;                    /* device i32 [B][cap] */
  int32_t* sel_cnt;                    /* device i32 [B] */
  int32_t* res_pages;                  /* device i32 [B][wb+1] */
  int32_t* n_res;                      /* device i32 [B] */
  int32_t* block_table;                /* device i32 [B][bt_stride], bt_stride >= cap+wb+1 */
  int32_t bt_stride;
  int32_t* n_entries;                  /* device i32 [B] */
  int32_t* tail_len;                   /* device i32 [B] */
  void* index_ws; size_t index_ws_bytes;   /* lsa_index_workspace_size(B, L, d_i, max_cand) */
  void* attn_ws;  size_t attn_ws_bytes;    /* lsa_decode_attn_workspace_size(B, H, d, n_sm) */
  int32_t* err;                        /* device i32 error word */
  int64_t kidx_layer_stride;           /* 0: K_idx shared by the layers; > 0: rows from
                                          layer l's key table to layer l+1's (lsa_index_ex) */
  /* resident-page reuse across passes (lsa_gather_delta); all null: plain lsa_gather */
  int32_t* kept_ids;                   /* device i32 [B][cap] */
  int32_t* kept_pages;                 /* device i32 [B][cap] */
  int32_t* kept_cnt;                   /* device i32 [B]; reset by lsa_pass_setup at pass 0 */
  void* gather_ws; size_t gather_ws_bytes; /* lsa_gather_delta_workspace_size(B, cap,
                                              n_pages - B*(W/64+1), n_sm), zeroed once */
} lsa_state;

/* Host-side validation of a state (no device work). */
lsa_status lsa_state_check(const lsa_state* st);
/* sizeof(lsa_state), for bindings that mirror the struct. */
size_t lsa_state_size(void);

/* Copy the window blocks of pass `pass` from the host pool into the window rings
   (set-up before the first lsa_step of a run; not part of the per-step path). */
lsa_status lsa_load_window(const lsa_state* st, int32_t pass, void* stream);

/* The pieces lsa_step is made of, for callers that schedule or time them separately:
   lsa_pass_setup  (pass start) candidate counts, resident page lists, a zeroed new tail
                   page; from pass 1 on it also writes the previous pass's completed tail
                   page back to the host pool;
   lsa_decode_step (every step) lsa_decode_attn with the token append fused into it: the
                   CTA that reads a sequence's tail page first stores k_new / v_new into
                   slot step % 64 of it; tail_len = step % 64 + 1.
   lsa_step(step) == [step % 64 == 0: lsa_pass_setup, lsa_index, lsa_gather],
                     lsa_decode_step, with the state's buffers.
   lsa_append is the stand-alone append (HBM tail page and host pool), for callers that
   run lsa_decode_attn themselves. */
lsa_status lsa_pass_setup(const lsa_state* st, int32_t pass, void* stream);
lsa_status lsa_decode_step(const lsa_state* st, int64_t step, const uint16_t* q,
                           const uint16_t* k_new, const uint16_t* v_new, uint16_t* out,
                           void* stream);
lsa_status lsa_append(const lsa_state* st, int64_t step, const uint16_t* k_new,
                      const uint16_t* v_new, void* stream);

/* One decode step. h: device bf16 [L][B][D], read only when step % 64 == 0;
   q: device bf16 [B][H][d]; k_new, v_new: device bf16 [B][d]; out: device bf16 [B][H][d]. */
lsa_status lsa_step(const lsa_state* st, int64_t step, const uint16_t* h, const uint16_t* q,
                    const uint16_t* k_new, const uint16_t* v_new, uint16_t* out, void* stream);

/* ---------------------------------------------------------------------------------
 * lsa_wait_selftest -- the library's bounded device wait, on its own: one thread polls
 * *flag (device u32, acquire at gpu scope) until it is >= target, the same wait every
 * grid barrier of the library uses. When limit_ns (1 .. 10^10) passes first, it ORs
 * LSA_DEVERR_TIMEOUT into the device word *err and returns, so a caller can make the
 * wait run out on a flag that nothing sets and check that the status arrives and the
 * context stays usable. (The library's own barriers wait at most 2 s.)
 */
lsa_status lsa_wait_selftest(const uint32_t* flag, uint32_t target, int64_t limit_ns,
                             int32_t* err, void* stream);

/* ---------------------------------------------------------------------------------
 * lsa_denoise_labels -- label denoising of the indexer's training targets (section 3
 * "Label Denoising Pipeline", three steps): for each token window w and CSA layer l,
 *
 *   prob = softmax(logits[w][l][:])                       (step 1)
 *   set[w][l] = the smallest set of blocks whose prob sums to >= top_p, taking blocks
 *               by decreasing prob, equal probs by increasing block id   (step 2)
 *   label[w][c] = 1 when block c is in set[w][l] for at least min_votes layers (step 3)
 *
 * The page's values are top_p = 0.6 and min_votes = 3 of 21 layers.
 *
 *   logits      device f32 [n_windows][n_layers][n_blocks], finite (a non-finite logit
 *               gives unspecified sets and may set LSA_DEVERR_NUMERIC; nothing faults)
 *   set_mask    device u32 [n_windows][n_layers][ceil(n_blocks/32)] out: bit (c % 32) of
 *               word c / 32 is block c; bits past n_blocks are zero
 *   set_cnt     nullable device i32 [n_windows][n_layers] out: the set sizes
 *   label_mask  nullable device u32 [n_windows][ceil(n_blocks/32)] out
 *   label_ids   device i32 [n_windows][label_cap] out: the labels in increasing id, the
 *               first label_cap of them (may be null when label_cap == 0)
 *   label_cnt   device i32 [n_windows] out: the number of labels (may exceed label_cap)
 * Supported: 1 <= n_layers <= 63, 1 <= n_blocks <= LSA_DENOISE_MAX_BLOCKS,
 * 0 < top_p <= 1; any min_votes (<= 0 keeps every block, > n_layers none).
 * Ties in probability are ties in the fp32 logit, so the tie order is exact; where the
 * running mass meets top_p within rounding (fp32 probabilities, fp64 sums) the boundary
 * block may differ from an exact computation. Two launches on `stream`: persistent CTAs
 * that take the (window, layer) rows in turn, then one CTA per window for the vote
 * (a programmatic dependent launch where the device allows it).
 */
#define LSA_DENOISE_MAX_BLOCKS 45056
lsa_status lsa_denoise_labels(const float* logits, int32_t n_windows, int32_t n_layers,
                              int32_t n_blocks, double top_p, int32_t min_votes,
                              uint32_t* set_mask, int32_t* set_cnt, uint32_t* label_mask,
                              int32_t* label_ids, int32_t label_cap, int32_t* label_cnt,
                              int32_t* err, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* LSA_H */
