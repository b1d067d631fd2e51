/*
 * flashblock.h -- C ABI of the FlashBlock denoise-step attention library (B200, sm_100a).
 *
 * What the library computes (FlashBlock, gist.science/es/paper/2602.05305,
 * "Mecanismo Central"): the queries of the active block attend to two key sets,
 * J_out (tokens outside the block: the cached prefix) and J_in (the block's own
 * tokens, bidirectional).  Each set gives a partial (A, L): A is softmax
 * attention over the set and L = log Z its natural-log normaliser.  The
 * out-of-block partial (A_out, L_out) is cached and reused on later steps; the
 * full output is the log-space composition
 *     A_full = (e^{L_out-m} A_out + e^{L_in-m} A_in) / (e^{L_out-m} + e^{L_in-m}),
 *     m = max(L_out, L_in),
 * with L_full = m + ln(e^{L_out-m} + e^{L_in-m}).
 * Reuse is decided per (sequence, q-head) by the gates of FlashBlock's
 * "Estrategias de Reutilizacion Adaptativa" (threshold tau on the updated-token
 * count; per-head similarity gamma) and only active query rows are computed
 * (SureLock, gist.science/es/paper/2602.06412, "Mecanismo de Funcionamiento":
 * locked rows compute no query but their K/V are still attended).  Several
 * requests or branches are packed into one call with cu_seqlens offsets
 * (BlockBatch, gist.science/fr/paper/2605.29233, "Optimisation Systeme").
 *
 * Conventions
 *  - Layout "THD": [tokens, heads, head_dim], head_dim contiguous, row-major.
 *  - bf16 tensors are passed as raw 16-bit patterns (fb_bf16).
 *  - Pointers marked (device) must be CUDA device memory of the current device;
 *    pointers marked (host) are host memory.  The caller owns every buffer; no
 *    call allocates device memory.  Every bf16/fp32 tensor must be 16-byte aligned.
 *  - Calls validate on the host and then enqueue on `stream` without
 *    synchronising (except fb_device_status).  They never abort or exit; on
 *    failure they return a non-zero fb_status and fb_last_error() describes it.
 *    Argument checks happen before any CUDA call, so they also work on a
 *    machine without a GPU.
 *  - softmax scale: scores are s = softmax_scale * q.k (usually 1/sqrt(d)).
 *  - Grouped heads: q-head h reads kv-head h / (num_heads_q / num_heads_kv).
 *  - Empty key set: A = 0, L = -inf.  Merging with an empty side returns the
 *    other side; two empty sides give A = 0, L = -inf.
 *  - A kernel that waits on an asynchronous copy gives up after about two
 *    seconds, records FB_ERR_TIMEOUT in a device status word and returns;
 *    fb_device_status() reads and clears it.  After a timeout the workspace
 *    must be re-initialised with fb_workspace_init().
 *  - Tracing: every call that enqueues device work (fb_workspace_init, the
 *    attention, merge, similarity, cache, layout and append calls, the
 *    self-test and fb_device_status) opens an NVTX range named for itself on
 *    entry and closes it on return, whatever it returns.  Without a tool
 *    attached to the process NVTX does nothing.
 */
#ifndef FLASHBLOCK_H
#define FLASHBLOCK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t fb_bf16;                /* bf16 bit pattern */
typedef struct CUstream_st* fb_stream_t; /* same type as cudaStream_t; NULL = default stream */

typedef enum fb_status {
  FB_OK = 0,
  FB_ERR_INVALID_ARG = 1, /* null pointer, negative size, misaligned buffer, bad offsets */
  FB_ERR_UNSUPPORTED = 2, /* head_dim not 64/128, num_heads_q % num_heads_kv != 0, group > 32,
                             sizes past 32-bit launch indices */
  FB_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed (message has the CUDA error) */
  FB_ERR_TIMEOUT = 4      /* a device-side bounded wait ran out (see fb_device_status) */
} fb_status;

/* Gate flags of fb_params.flags. */
#define FB_GATE_TAU 1u        /* reuse only if n_updated[b] < tau (strict)               */
#define FB_GATE_HEAD 2u       /* reuse head h only if cos(Q_bh, q_ref_bh) > gamma (strict);
                                 a head with no active rows has cos 0                  */
#define FB_FORCE_RECOMPUTE 4u /* recompute every head (dense step)                        */
#define FB_FORCE_REUSE 8u     /* reuse every head whose cache is valid                    */
/* Cumulative threshold gate: reuse only if cache->m_acc[b,h] + n_updated[b] < tau, i.e.
 * the block tokens updated since the head's cache was built (this step included) stay
 * below tau; the count is kept in cache->m_acc and restarts at 0 when the head
 * recomputes.  A reading of FlashBlock's updated-token count M ("Estrategias de
 * Reutilizacion Adaptativa", first bullet), whose per-step form is FB_GATE_TAU; the two
 * flags are exclusive.  The count is maintained on every call that sets the flag, forced
 * modes and caller masks included. */
#define FB_GATE_TAU_CUM 16u

/*
 * One step's problem.  Index arrays are int32 device arrays; the scalar bounds
 * are host values and must be exact totals / upper bounds of those arrays.
 *   cu_seqlens_q      [num_seqs+1] offsets of each sequence's ACTIVE query rows in Q
 *   q_rows            [total_q] block position (0..B_b-1) of each packed row, or
 *                     NULL meaning row r of sequence b is block position r - cu_seqlens_q[b]
 *   cu_seqlens_kv_out [num_seqs+1] offsets of each sequence's prefix (J_out) tokens
 *   cu_seqlens_kv_in  [num_seqs+1] offsets of each sequence's block (J_in) tokens
 * out_splits: number of key splits of the prefix pass; 0 lets the library choose.
 * Ordering: the attention calls read the index arrays (cu_seqlens_*, q_rows) before they
 *   wait for the previous kernel of the stream to finish, so that these loads overlap its
 *   tail; fb_step with early lean loads (fb_plan_info.lean_early) also reads its block
 *   inputs q, k_in and v_in there.  A kernel that precedes such a call on its stream
 *   and lets its dependents launch early (programmatic dependent launch,
 *   griddepcontrol.launch_dependents) must not write any of them; ordinary kernels
 *   and copies are waited for as usual.  The library's own
 *   kernels that write index arrays or block K/V (fb_sparse_layout, fb_prefix_append) do
 *   not launch dependents early, and none writes q.  The attention kernels themselves
 *   do launch their dependents early, so an output of one call (a_full, l_full, the
 *   cache) must not be read as q, k_in or v_in by the next attention call on the stream
 *   without an ordinary kernel or copy in between.  Everything else (the prefix K/V, the
 *   cache, kv_out_skip) is read after the wait.
 * kv_out_skip: NULL, or a bitmask over the prefix tokens (device, uint32 words, at least
 *   ceil(total_kv_out / 32) of them): bit t (bit t % 32 of word t / 32) set leaves prefix
 *   token t -- row t of k_out / v_out -- out of J_out.  The sparse-residual layout
 *   (fb_sparse_layout) sets the bits of the keys it moves into the block's key set.
 */
typedef struct fb_problem {
  int32_t num_seqs, num_heads_q, num_heads_kv, head_dim;
  float softmax_scale;
  const int32_t* cu_seqlens_q;
  const int32_t* q_rows;
  const int32_t* cu_seqlens_kv_out;
  const int32_t* cu_seqlens_kv_in;
  int32_t total_q, total_kv_out, total_kv_in; /* host: Q / prefix / block token counts   */
  int32_t max_q, max_kv_out, max_kv_in;       /* host: largest per-sequence count of each */
  int32_t out_splits;
  const uint32_t* kv_out_skip;
} fb_problem;

/*
 * The FlashBlock cache (FlashBlock, "Mecanismo Central": A_out and L_out are kept
 * from an earlier step and reused).  Rows are addressed by BLOCK POSITION, so a
 * row keeps its entry while the active set shrinks:  cache row of packed row r of
 * sequence b = cu_seqlens_kv_in[b] + q_rows[r].  All device memory, caller-owned.
 *   a_out [total_kv_in, H_q, d] fp32;  l_out [total_kv_in, H_q] fp32
 *   valid [num_seqs, H_q] uint8 (0 = empty: the head recomputes whatever the gates say)
 *   q_ref [total_kv_in, H_q, d] bf16: the queries each head's entry was built with
 *         (needed by FB_GATE_HEAD; may be NULL otherwise)
 *   m_acc [num_seqs, H_q] int32: block tokens updated since the head's last recompute
 *         (needed by FB_GATE_TAU_CUM, zero-initialised by the caller; may be NULL otherwise)
 */
typedef struct fb_cache {
  float* a_out;
  float* l_out;
  uint8_t* valid;
  fb_bf16* q_ref;
  int32_t* m_acc;
} fb_cache;

typedef struct fb_params {
  int32_t tau;    /* threshold of FB_GATE_TAU */
  float gamma;    /* threshold of FB_GATE_HEAD */
  uint32_t flags; /* FB_GATE_* | FB_FORCE_* (FB_GATE_TAU_CUM included) */
} fb_params;

/* Message of the last failing call on this thread (never NULL). */
const char* fb_last_error(void);

/* Library version (major*100 + minor). */
int32_t fb_version(void);

/* Calls whose launch plan fb_plan_query describes. */
#define FB_CALL_STEP 0 /* fb_step (and fb_step_noalloc)  */
#define FB_CALL_OUT 1  /* fb_out_attn                     */
#define FB_CALL_IN 2   /* fb_in_attn                      */

/* Attention kernels a plan may choose. */
#define FB_KERNEL_WARP_MMA 0 /* attn_kernel: warp-level MMA, groups of up to 64 rows (all head_dim 64)  */
#define FB_KERNEL_TC 1       /* tc_attn_kernel: tcgen05 with TMEM accumulators, one 128-row tile       */
#define FB_KERNEL_TC2 2      /* tc2_attn_kernel: tcgen05, two 128-row tiles of one head per CTA       */

/*
 * Launch plan of the attention kernel of one call.  A group is the rows of one
 * (sequence, kv-head): its block rows times the query heads sharing the kv-head,
 * cut into tiles of rows_per_tile.  Each tile's prefix keys are split over
 * `splits` CTAs of one cluster, whose partials are combined in distributed shared
 * memory (splits = 1: no cluster).
 */
typedef struct fb_plan_info {
  int32_t kernel;         /* FB_KERNEL_*                                          */
  int32_t rows_per_tile;  /* query rows (token x q-head of the group) per tile     */
  int32_t tiles;          /* tiles per group                                       */
  int32_t work_items;     /* (sequence, kv-head, tile) items (two-tile kernel: pairs) */
  int32_t splits;         /* CTAs per item over the prefix keys (cluster size)      */
  int32_t ctas;           /* grid size = work_items x splits                        */
  int32_t threads;        /* threads per CTA                                        */
  int32_t smem_bytes;     /* dynamic shared memory per CTA                          */
  int32_t keys_per_chunk; /* keys per pipeline stage (TMA box rows)                 */
  int32_t num_sms;        /* SM count the plan was made for                         */
  /* Lean reuse path of fb_step (blocks of at most 128 keys): a work item whose
   * q-heads all reuse the cache skips the streaming pipeline; its CTAs share its
   * rows and run the block attention and the merge with the cached partial from
   * one round of loads. */
  int32_t lean_reuse;      /* 1 when the call has the lean path                     */
  int32_t lean_smem_bytes; /* shared memory it uses per CTA at most (of smem_bytes) */
  int32_t lean_early;      /* 1 when its loads start before the reuse decision is known
                              (the grid is resident in one wave); see Ordering       */
} fb_plan_info;

/*
 * The launch plan `call` (FB_CALL_*) would use for this problem on the current
 * device (148 SMs when no device is visible).  Pure host computation: the
 * cu_seqlens pointers are not read.  FB_ERR_INVALID_ARG for a bad problem, an
 * unknown call or a NULL out.
 */
fb_status fb_plan_query(const fb_problem* problem, int32_t call, fb_plan_info* out);

/*
 * Bytes of workspace that fb_out_attn / fb_step need for this problem (a
 * completion counter and the per-head similarity scores; partials stay on chip).
 * Pure host computation.
 */
fb_status fb_workspace_size(const fb_problem* problem, size_t* bytes);

/* Zero a workspace (device) before its first use.  Calls leave it zeroed again. */
fb_status fb_workspace_init(void* workspace, size_t bytes, fb_stream_t stream);

/*
 * Out-of-block partial (FlashBlock, "Mecanismo Central": A_out over J_out with
 * L_out = log Z_out).  For every active row and every q-head h of sequence b
 * with head_mask[b*H_q+h] != 0 (head_mask NULL = all heads), attends over all
 * prefix tokens of b and writes (A_out, L_out) at the row's cache position:
 *   a_out[(cu_seqlens_kv_in[b] + q_rows[r]) * H_q + h][0..d)  fp32
 *   l_out[ same row * H_q + h ]                                fp32
 * Heads with mask 0 are not touched.  q [total_q, H_q, d] bf16; k_out, v_out
 * [total_kv_out, H_kv, d] bf16.  The prefix keys are split into key ranges whose
 * partials are combined with the same log-space rule.
 */
fb_status fb_out_attn(const fb_problem* problem, const fb_bf16* q, const fb_bf16* k_out,
                      const fb_bf16* v_out, const uint8_t* head_mask, float* a_out, float* l_out,
                      void* workspace, size_t workspace_bytes, fb_stream_t stream);

/*
 * In-block partial (FlashBlock, "Mecanismo Central": A_in over J_in, the block's
 * tokens, with no mask inside the block).  Locked tokens' K/V are part of J_in.
 * Outputs in packed row order: a_in [total_q, H_q, d] fp32, l_in [total_q, H_q] fp32.
 */
fb_status fb_in_attn(const fb_problem* problem, const fb_bf16* q, const fb_bf16* k_in,
                     const fb_bf16* v_in, float* a_in, float* l_in, fb_stream_t stream);

/*
 * Log-space merge of two partials (FlashBlock, "Mecanismo Central", the A_full
 * equation), element-wise over n (row, head) entries of width d:
 *   a_out, a_in [n, d] fp32;  l_out, l_in [n] fp32.
 * Writes a_full_f32 [n, d] fp32 and/or a_full_bf16 [n, d] bf16 (either may be
 * NULL, not both) and l_full [n] fp32 (may be NULL).  d any positive size.
 */
fb_status fb_merge(int64_t n, int32_t d, const float* a_out, const float* l_out, const float* a_in,
                   const float* l_in, float* a_full_f32, fb_bf16* a_full_bf16, float* l_full,
                   fb_stream_t stream);

/*
 * Per-head similarity of the FB_GATE_HEAD gate (FlashBlock, "Estrategias de
 * Reutilizacion Adaptativa", per-head selection).  cos_out[b*H_q+h] = cosine
 * between the active-row queries of (b, h), flattened rows x d, and q_ref at the
 * same block positions.  fp32, fixed reduction order.  A zero denominator gives 0.
 */
fb_status fb_head_similarity(const fb_problem* problem, const fb_bf16* q, const fb_bf16* q_ref,
                             float* cos_out, fb_stream_t stream);

/*
 * One denoise step of attention with the FlashBlock cache.
 * Per (b, h): recompute = FORCE_RECOMPUTE or !valid[b,h] or (not FORCE_REUSE and
 *   (head_reuse_in ? !head_reuse_in[b,h]
 *                  : !((!GATE_TAU or n_updated[b] < tau) and (!GATE_HEAD or cos_bh > gamma)))).
 * Heads that recompute get a fresh (A_out, L_out) over the prefix, stored in the
 * cache with valid = 1 (and q_ref = the current queries when q_ref is not NULL);
 * every head then attends over its block and merges with the cache:
 *   a_full [total_q, H_q, d] bf16,  l_full [total_q, H_q] fp32 (may be NULL).
 * n_updated [num_seqs] int32 (device; needed by FB_GATE_TAU).  head_reuse_in
 * [num_seqs, H_q] uint8 (device, 1 = reuse) replaces the gates when not NULL.
 * decision_out [num_seqs, H_q] uint8 (device, 1 = recomputed) may be NULL.
 * The workspace must come from fb_workspace_size and be zeroed once
 * (fb_workspace_init).  Calls on the same workspace must not overlap on the GPU.
 */
fb_status fb_step(const fb_problem* problem, const fb_params* params, const fb_cache* cache,
                  const fb_bf16* q, const fb_bf16* k_in, const fb_bf16* v_in, const fb_bf16* k_out,
                  const fb_bf16* v_out, const int32_t* n_updated, const uint8_t* head_reuse_in,
                  fb_bf16* a_full, float* l_full, uint8_t* decision_out, void* workspace,
                  size_t workspace_bytes, fb_stream_t stream);

/* Mark every cache entry of the problem's sequences empty (valid = 0): a new
 * block, a full refresh or a branch resync. */
fb_status fb_cache_invalidate(const fb_problem* problem, const fb_cache* cache, fb_stream_t stream);

/*
 * Branch hooks for multi-branch decoding (BlockBatch, gist.science/fr/paper/2605.29233,
 * "Methodologie : BlockBatch", items 2 and 3).  Both act on the FlashBlock cache only;
 * the caller moves K/V itself.
 *
 * fb_cache_copy_seq -- leader-based synchronisation: the lagging branch dst_seq takes
 *   the state of the leader src_seq.  For every q-head, the entries of block positions
 *   0..min(B_src, B_dst)-1 (a_out, l_out, and q_ref / m_acc when present) are copied
 *   from src_seq to dst_seq, and valid[dst_seq, :] = valid[src_seq, :]; when B_dst >
 *   B_src the positions without a source leave dst_seq's heads empty (valid = 0).
 *   src_seq == dst_seq is a no-op.  Errors: an index outside [0, num_seqs).
 * fb_cache_invalidate_seqs -- periodic full-sequence refresh of some branches:
 *   valid[b, :] = 0 (and m_acc[b, :] = 0 when present) for every b with
 *   seq_mask[b] != 0 (uint8 [num_seqs], device); seq_mask NULL = every sequence.
 * Asynchronous on `stream`; the problem's cu_seqlens_kv_in are read on the device.
 */
fb_status fb_cache_copy_seq(const fb_problem* problem, const fb_cache* cache, int32_t src_seq, int32_t dst_seq,
                            fb_stream_t stream);
fb_status fb_cache_invalidate_seqs(const fb_problem* problem, const fb_cache* cache, const uint8_t* seq_mask,
                                   fb_stream_t stream);

/*
 * Sparse-residual layout (FlashBlock, gist.science/es/paper/2602.05305, "Estrategias de
 * Reutilizacion Adaptativa", third bullet: the keys a sparse-attention pattern does not
 * select form the out-of-block set, whose contribution FlashBlock caches).  For every
 * sequence b the selected prefix keys join the block's keys and the rest form the
 * residual prefix:
 *   J_in'(b)  = block keys of b, then the selected prefix keys (increasing order)
 *   J_out'(b) = prefix keys of b that are not selected (order kept)
 * cu_sel [num_seqs+1] (device) offsets into sel_idx; sel_idx [total_sel] (device) holds,
 * per sequence, strictly increasing positions in [0, N_b) of the selected prefix keys;
 * total_sel (host) = cu_sel[num_seqs].  Outputs (device, caller-owned):
 *   k_ext, v_ext [total_kv_in + total_sel, H_kv, d] (THD bf16): J_in' of every sequence;
 *   kv_out_skip [ceil(total_kv_out / 32)] uint32: the bitmask of the selected prefix
 *     tokens (bit t of the global prefix row t); this call writes the bits of every
 *     sequence's prefix tokens (cleared, then the selected ones set) and leaves bits
 *     past total_kv_out as they are;
 *   cu_seqlens_kv_in_ext = cu_seqlens_kv_in + cu_sel ([num_seqs+1]; may be NULL).
 * The residual prefix is not copied: J_out' is the prefix (k_out, v_out,
 * cu_seqlens_kv_out unchanged) with kv_out_skip set in the problem, which every prefix
 * pass honours.  The block keeps positions 0..B_b-1 of J_in', so cu_seqlens_q and q_rows
 * stay valid: fb_step on that problem (cu_seqlens_kv_in_ext, kv_out_skip) with a cache of
 * total_kv_in + total_sel rows caches the residual and recomputes the selected keys every
 * step; with a fresh cache the result is full attention over prefix and block.  The
 * selection is fixed for a block (a new one changes the residual: refill the cache).
 * The pass moves the block rows and the selected rows only, in one kernel.  A selection
 * that is not increasing or out of range records FB_ERR_INVALID_ARG on the device
 * (fb_device_status); that sequence's skip bits are left cleared and its
 * cu_seqlens_kv_in_ext entry unwritten, and its J_in' rows are unspecified (the
 * selected rows next to a bad entry are not written).  A sequence whose offsets are
 * inconsistent is not touched at all.  At most 65535 sequences per call (FB_ERR_UNSUPPORTED beyond).
 */
fb_status fb_sparse_layout(const fb_problem* problem, const int32_t* cu_sel, const int32_t* sel_idx,
                           int32_t total_sel, const fb_bf16* k_out, const fb_bf16* v_out, const fb_bf16* k_in,
                           const fb_bf16* v_in, fb_bf16* k_ext, fb_bf16* v_ext, uint32_t* kv_out_skip,
                           int32_t* cu_seqlens_kv_in_ext, fb_stream_t stream);

/*
 * Block transition (FlashBlock, gist.science/es/paper/2602.05305, "Mecanismo Central": a
 * finished block stops being denoised and its tokens become context of the next block,
 * i.e. part of its out-of-block set J_out).  For every sequence b:
 *   J_out'(b) = J_out(b) followed by J_in(b) (block order),  cu_out'[b] = cu_out[b] + cu_in[b]
 * k_out, v_out [total_kv_out, H_kv, d] and k_in, v_in [total_kv_in, H_kv, d] (THD bf16,
 * device) are the prefix and the finished block's final K/V; the result goes to k_dst,
 * v_dst [total_kv_out + total_kv_in, H_kv, d] (device, caller-owned) and, when not NULL,
 * cu_seqlens_kv_out_dst [num_seqs+1] (device).
 *   - New buffers (k_dst != k_out): every prefix row and block row is copied; the source
 *     and destination must not overlap.
 *   - In place (k_dst == k_out and v_dst == v_out; one sequence only, the buffers must
 *     hold total_kv_out + total_kv_in rows): only the block rows are written, after the
 *     prefix.  FB_ERR_UNSUPPORTED for more sequences (later ones would have to move).
 * The next block brings new queries: call fb_cache_invalidate before its first fb_step
 * (every head then recomputes over the grown prefix).  Asynchronous on `stream`; index
 * arrays that disagree with the host totals record FB_ERR_INVALID_ARG on the device
 * (that sequence is skipped).  At most 65535 sequences per call.
 */
fb_status fb_prefix_append(const fb_problem* problem, const fb_bf16* k_out, const fb_bf16* v_out,
                           const fb_bf16* k_in, const fb_bf16* v_in, fb_bf16* k_dst, fb_bf16* v_dst,
                           int32_t* cu_seqlens_kv_out_dst, fb_stream_t stream);

/*
 * Self-test of the failure path of the bounded waits (no counterpart in the pages):
 * launches one CTA that waits on an mbarrier nothing will ever complete, with the same
 * bounded wait the attention kernels use (about two seconds), so the wait runs out,
 * FB_ERR_TIMEOUT is recorded in the device status word and the kernel returns; the
 * context stays usable.  Read the result with fb_device_status().
 */
fb_status fb_selftest_wait_timeout(fb_stream_t stream);

/* Release the host-side tensor-map cache (descriptors of K/V buffers seen so far). */
fb_status fb_release_cache(void);

/* Synchronise `stream`, then read and clear the device status word:
 * *code = FB_OK; FB_ERR_TIMEOUT if a bounded wait ran out since the last read;
 * FB_ERR_INVALID_ARG if a kernel found an index array (cu_seqlens, q_rows) that
 * disagrees with the host totals -- the affected work was skipped, not done out
 * of bounds. */
fb_status fb_device_status(int32_t* code, fb_stream_t stream);

/*
 * fb_step without a workspace argument, for callers that cannot allocate device
 * memory (a framework allocator owns all of it, a plugin must not allocate, or an
 * allocation inside the step loop is not acceptable).  The pages describe no such
 * call; it exists only for these integrations.
 *
 * Arguments and results are those of fb_step.  Instead of a caller workspace the
 * call uses a scratch array built into the library: 64 KiB of device memory that
 * every GPU loading the library holds until the process exits.  It covers every
 * problem whose fb_workspace_size is at most 64 KiB: num_seqs x num_heads_q up to
 * 16320, fewer for multi-head problems of 256+ rows per head (their workspace also
 * holds the two-tile work order).  Larger problems return FB_ERR_UNSUPPORTED
 * (message in fb_noalloc_last_error()) -- use fb_step with a workspace for them.
 * No call allocates: the first call on a device resolves the scratch address
 * (cudaGetSymbolAddress, with that device current), so make that first call before
 * capturing a stream.  If the device's context is re-created (cudaDeviceReset), the
 * next call resolves the address again, so that call too belongs before a capture.
 * Every call on a device shares the one array, which keeps the last call's
 * contents (the call clears the part that must start at zero): calls that could
 * overlap on the GPU race and must be ordered, e.g. issued on one stream.
 * Every failure is described by fb_noalloc_last_error().
 */
fb_status fb_step_noalloc(const fb_problem* problem, const fb_params* params, const fb_cache* cache,
                          const fb_bf16* q, const fb_bf16* k_in, const fb_bf16* v_in, const fb_bf16* k_out,
                          const fb_bf16* v_out, const int32_t* n_updated, const uint8_t* head_reuse_in,
                          fb_bf16* a_full, float* l_full, uint8_t* decision_out, fb_stream_t stream);

/* Message of the last fb_step_noalloc failure on this thread (every kind: argument
 * errors, a problem above the scratch limit, CUDA errors); empty after a call that
 * succeeded.  Argument errors are also reported through fb_last_error(). */
const char* fb_noalloc_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* FLASHBLOCK_H */
