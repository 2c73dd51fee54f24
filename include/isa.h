/*
 * isa.h -- C ABI of the In-context Sparse Attention (ISA) forward, sm_100a.
 *
 * Method: "Lightning Unified Video Editing via In-Context Sparse Attention"
 * (Shao et al., 2026), abstract.  The sequence of every (batch, head) holds
 * N_src source-video tokens followed by N_ctx context tokens.  ISA runs in
 * four stages, each a call (or part of a call) below:
 *   1. context pre-selection   (abstract, first insight: context tokens are
 *      less salient; redundant context is pruned)      -> isa_preselect_ctx
 *   2. query sharpness + dynamic query grouping (abstract, second insight:
 *      sharpness tracks approximation error)            -> isa_route_queries
 *   3. full attention for the routed (sharp) queries    -> isa_attn_fwd
 *   4. 0-th order Taylor sparse attention for the rest  -> isa_attn_fwd
 * The abstract gives only this outline; the formulas implemented are:
 *   blocks   per segment, `block` tokens each, the last one of each segment
 *            partial; cnt_b tokens in block b; Xbar_b = block mean of x.
 *   s        scale (1/sqrt(d) when shape->scale <= 0).
 *   saliency sal_c = sum_r cnt_r * softmax_c(s Qbar_r.Kbar_c + ln cnt_c) / N
 *            over all key blocks c; context blocks ranked by it; the top
 *            n_keep = ceil(keep*nCB - g(nCB)) are kept; source blocks always;
 *            g(n) = min(1e-6*n, 0.5) absorbs the float32 rounding of keep/rho.
 *   sharp_i  max_b softmax_b(s q_i.Kbar_b + ln cnt_b) over kept blocks.
 *   routing  the n_route = ceil(rho*N - g(N)) sharpest queries (ties: lower
 *            index first) -> full attention over every token of every kept
 *            block; the others -> sum_b cnt_b e^{s q.Kbar_b} Vbar_b /
 *            sum_b cnt_b e^{s q.Kbar_b} over kept blocks.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every tensor pointer is a DEVICE pointer owned by the caller, 16-byte
 *   aligned.  q, k, v, out are contiguous [B, H, N, d] bf16 (given here as
 *   uint16_t bit patterns), d innermost, N = N_src + N_ctx; rows 0..N_src-1
 *   of each head are source tokens, the rest context tokens.
 * - Index outputs are int32, ascending within each (b, h).
 * - The library allocates no memory and keeps no state between calls; all
 *   scratch lives in the caller's workspace `ws` of `ws_bytes` bytes
 *   (16-byte aligned), sized by isa_workspace_size().  The first 256 bytes
 *   of `ws` are a control block: an int32 device status word at offset 0
 *   (0 = no error) and an int32 fault-injection word at offset 4 (tests
 *   only; leave it 0).  Zero the control block once after allocating ws.
 * - Calls validate every argument before launching anything and return an
 *   isa_status; on an error nothing is launched.  Launches are asynchronous
 *   on `stream` (a cudaStream_t; NULL = legacy default stream).  A kernel
 *   that gives up on a bounded wait writes ISA_ERR_DEVICE_TIMEOUT into the
 *   status word and exits; read it with isa_read_device_status().  After a
 *   non-zero device status the outputs of the calls since the last reset
 *   are undefined (rows may be left unwritten).
 * - Supported: d in {64, 128}; block in {64, 128}; N_src >= 1; N_ctx >= 0;
 *   0 <= keep <= 1; 0 <= rho <= 1; ceil(N_ctx/block) <= 4096;
 *   B*H <= 65535.  Anything else returns ISA_ERR_UNSUPPORTED.
 */
#ifndef ISA_H_
#define ISA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ISA_OK = 0,
  ISA_ERR_INVALID_ARG = 1,    /* null pointer, misalignment, negative size */
  ISA_ERR_UNSUPPORTED = 2,    /* valid but outside the supported shapes */
  ISA_ERR_WORKSPACE = 3,      /* ws_bytes smaller than required */
  ISA_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed */
  ISA_ERR_DEVICE_TIMEOUT = 5  /* a kernel's bounded wait expired */
} isa_status;

/* Problem shape.  scale <= 0 selects 1/sqrt(d). */
typedef struct {
  int B, H, N_src, N_ctx, d, block;
  float keep, rho, scale;
} isa_shape;

/* Number of kept context blocks per (b, h): ceil(keep*nCB - g(nCB)), nCB =
 * ceil(N_ctx/block).  Returns -1 on an invalid shape. */
int isa_n_keep(const isa_shape* shape);

/* Number of routed queries per (b, h): ceil(rho*N - g(N)).  -1 if invalid. */
int isa_n_route(const isa_shape* shape);

/* Number of routed query blocks per (b, h) of the block-granular grouping
 * (isa_route_blocks_taylor_fwd): ceil(rho*nB - g(nB)), nB = nSB + nCB.
 * -1 if invalid. */
int isa_n_route_blocks(const isa_shape* shape);

/* Bytes of workspace needed by every ISA call on this shape (0 if invalid). */
size_t isa_workspace_size(const isa_shape* shape);

/* Stage 1, context pre-selection.
 * Computes the block means of q, k, v (kept in ws for the later calls), the
 * saliency of every context block and the n_keep most salient ones.
 *   kept_ctx_idx [B, H, n_keep] int32 out: context block numbers (0-based
 *                within the context segment), ascending.  May be NULL only
 *                when n_keep == 0.
 *   saliency     [B, H, nCB] float out, or NULL.
 * The block means written into ws are inputs of isa_route_queries and
 * isa_attn_fwd; call this first with the same ws.  The means of v are
 * pooled for the source blocks and for the context blocks this call keeps
 * only (the others are never read), so the later calls on this ws must be
 * given the kept set returned here: another one is reported as
 * ISA_ERR_INVALID_ARG in the device status word (outputs undefined). */
int isa_preselect_ctx(const isa_shape* shape, const uint16_t* q, const uint16_t* k,
                      const uint16_t* v, int32_t* kept_ctx_idx, float* saliency,
                      void* ws, size_t ws_bytes, void* stream);

/* Stage 2, query sharpness and dynamic grouping.
 * Uses the block means in ws (from isa_preselect_ctx) and the kept set.
 *   kept_ctx_idx [B, H, n_keep] int32 in (ascending, distinct, < nCB).
 *   routed_idx   [B, H, n_route] int32 out: the sharpest queries, ascending.
 *   taylor_idx   [B, H, N - n_route] int32 out: every other query, ascending.
 *   sharpness    [B, H, N] float out, or NULL.
 * routed_idx / taylor_idx may be NULL when their size is 0. */
int isa_route_queries(const isa_shape* shape, const uint16_t* q, const int32_t* kept_ctx_idx,
                      int32_t* routed_idx, int32_t* taylor_idx, float* sharpness,
                      void* ws, size_t ws_bytes, void* stream);

/* Stages 3 and 4: full attention for routed_idx rows, 0-th order Taylor
 * attention for taylor_idx rows; writes every row of out [B, H, N, d] bf16
 * exactly once when routed_idx and taylor_idx partition 0..N-1.  Uses the
 * block means in ws (from isa_preselect_ctx). */
int isa_attn_fwd(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                 const int32_t* kept_ctx_idx, const int32_t* routed_idx, const int32_t* taylor_idx,
                 uint16_t* out, void* ws, size_t ws_bytes, void* stream);

/* Stages 2 and 4 in one pass over q (the fast path of isa_forward): computes
 * the sharpness of every query and the 0-th order Taylor output of EVERY
 * row of out [B, H, N, d], then routes exactly as isa_route_queries.  Follow
 * it with isa_full_attn_fwd on the same out: that overwrites the routed rows
 * with full attention, leaving the Taylor rows as written here.  Arguments
 * as in isa_route_queries; sharpness may be NULL. */
int isa_route_taylor_fwd(const isa_shape* shape, const uint16_t* q, const int32_t* kept_ctx_idx,
                         int32_t* routed_idx, int32_t* taylor_idx, float* sharpness, uint16_t* out,
                         void* ws, size_t ws_bytes, void* stream);

/* Stage 3 alone: full attention for the routed_idx rows of out over every
 * token of every source block and of the kept context blocks (the part of
 * isa_attn_fwd that does not need the block means).  Independent of stage 4:
 * the two may run concurrently on different streams (disjoint rows of out). */
int isa_full_attn_fwd(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                      const int32_t* kept_ctx_idx, const int32_t* routed_idx, uint16_t* out,
                      void* ws, size_t ws_bytes, void* stream);

/* Stage 4 alone: 0-th order Taylor attention for the taylor_idx rows of out
 * over the kept block means (block means in ws from isa_preselect_ctx). */
int isa_taylor_attn_fwd(const isa_shape* shape, const uint16_t* q, const int32_t* kept_ctx_idx,
                        const int32_t* taylor_idx, uint16_t* out, void* ws, size_t ws_bytes,
                        void* stream);

/* Stage 3 for an explicit row list: full attention, over every token of
 * every source block and of the kept context blocks, for the n_rows entries
 * of row_idx [B, H, n_rows] int32 per (b, h).  An entry of -1 is padding:
 * it is computed on a zero query and never stored; any other entry outside
 * [0, N) is skipped and reported as ISA_ERR_INVALID_ARG in the device
 * status word.  Entries must not repeat within a (b, h).  With
 * row_idx = routed_idx and n_rows = n_route this is isa_full_attn_fwd. */
int isa_full_attn_rows_fwd(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const int32_t* kept_ctx_idx, const int32_t* row_idx, int n_rows, uint16_t* out,
                           void* ws, size_t ws_bytes, void* stream);

/* Stages 2 and 4 with the dynamic query grouping taken over whole query
 * blocks (a variant reading: the abstract does not fix the unit grouped).
 * Query blocks use the per-segment partition of the keys; block b scores
 * the mean sharpness of its cnt_b queries (fp32); the n_rb =
 * isa_n_route_blocks() best blocks (ties: lower block index) are routed.
 * Like isa_route_taylor_fwd, writes the 0-th order Taylor output of EVERY
 * row of out; follow it with isa_full_attn_rows_fwd(routed_rows,
 * n_rb * block) to overwrite the routed blocks' rows with full attention.
 *   routed_blk_idx [B, H, n_rb] int32 out: routed block numbers (source
 *                  blocks 0..nSB-1, then context blocks), ascending.
 *   routed_rows    [B, H, n_rb * block] int32 out: entry r*block + t is
 *                  row t of routed block r, or -1 past a partial block's
 *                  last row.
 *   block_score    [B, H, nB] float out (mean sharpness per block), or NULL.
 *   sharpness      [B, H, N] float out, or NULL.
 * Supported up to nB = 16384 query blocks per head (else
 * ISA_ERR_UNSUPPORTED).  routed_* may be NULL when n_rb == 0. */
int isa_route_blocks_taylor_fwd(const isa_shape* shape, const uint16_t* q, const int32_t* kept_ctx_idx,
                                int32_t* routed_blk_idx, int32_t* routed_rows, float* block_score,
                                float* sharpness, uint16_t* out, void* ws, size_t ws_bytes, void* stream);

/* The forward with block-granular grouping: isa_preselect_ctx,
 * isa_route_blocks_taylor_fwd, isa_full_attn_rows_fwd on one stream, with
 * every index set held inside ws.  out [B, H, N, d] bf16. */
int isa_forward_blocks(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                       uint16_t* out, void* ws, size_t ws_bytes, void* stream);

/* First-order Taylor variant of stage 4.  The abstract names its
 * approximation "0-th order"; the next order keeps the linear term of exp
 * around the block mean, exp(s q.k_j) ~= exp(s q.Kbar_b)(1 + s q.(k_j -
 * Kbar_b)) for j in kept block b, which gives
 *   o_i = [sum_b cnt_b e_ib Vbar_b + s sum_b e_ib C_b^T q_i] / sum_b cnt_b e_ib,
 *   e_ib = exp(s q_i.Kbar_b),  C_b = sum_{j in b} (k_j - Kbar_b) v_j^T (d x d).
 * Costs about d/2 times the 0-th order pass (one d x d product per query
 * and kept block) and is closer to full attention.
 *
 * isa_taylor1_workspace_size: bytes of the second workspace `cws` these
 * calls need: the correction matrices C_b of every kept block, bf16
 * [B, H, nSB + n_keep, d, d] row-major ([d_in][d_out]); 0 if invalid.
 *
 * isa_taylor1_attn_fwd: writes the first-order Taylor output of the
 * taylor_idx [B, H, N - n_route] rows of out (entries of -1 are padding),
 * from q, k, v, the kept set and the block means in ws (isa_preselect_ctx
 * first, same ws).  cws (16-byte aligned, >= isa_taylor1_workspace_size
 * bytes, else ISA_ERR_WORKSPACE) receives the C_b.
 *
 * isa_forward_taylor1: the forward with this variant: isa_preselect_ctx,
 * isa_route_taylor_fwd (its 0-th order rows are overwritten), full
 * attention for the routed rows, first-order Taylor for the others; index
 * sets held inside ws. */
size_t isa_taylor1_workspace_size(const isa_shape* shape);
int isa_taylor1_attn_fwd(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         const int32_t* kept_ctx_idx, const int32_t* taylor_idx, uint16_t* out,
                         void* ws, size_t ws_bytes, void* cws, size_t cws_bytes, void* stream);
int isa_forward_taylor1(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        uint16_t* out, void* ws, size_t ws_bytes, void* cws, size_t cws_bytes, void* stream);

/* All four stages in order on one stream (isa_preselect_ctx,
 * isa_route_taylor_fwd, isa_full_attn_fwd), with the kept set and the
 * routed and Taylor index sets held inside ws.  out [B, H, N, d] bf16. */
int isa_forward(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                uint16_t* out, void* ws, size_t ws_bytes, void* stream);

/* All four stages like isa_forward, for callers that cannot allocate device
 * memory: frameworks whose caching allocator owns every free byte of the
 * GPU, serving loops that must not allocate after start-up, or plugins that
 * are handed tensors but no way to obtain scratch.  (The ISA pages have no
 * counterpart; this is a packaging of the same path.)
 * The scratch is a fixed array of ISA_STATIC_SCRATCH_BYTES inside this
 * library; every GPU that loads the library holds it until the process
 * exits.  Shapes whose isa_workspace_size() exceeds it (e.g. 40 heads of
 * 75600 + 75600 tokens) return ISA_ERR_WORKSPACE without launching
 * anything; invalid shapes return what isa_forward returns.  The first call
 * on a device looks up the array's device address (cudaGetSymbolAddress,
 * with that device current); make that first call before any stream
 * capture.  Each call clears the scratch's control block and calls
 * isa_forward on it; nothing is allocated or freed.  All calls share the
 * one array, which keeps the last call's contents: calls that overlap on
 * the GPU (different streams, or different host threads on one device)
 * race and corrupt each other.  The device status word of these calls is
 * not readable by the caller, so a device-side timeout (which leaves rows of
 * out unwritten or stale) goes unseen here; use isa_forward with an own
 * workspace when device-side timeouts must be observed. */
#define ISA_STATIC_SCRATCH_BYTES (64u << 20)
int isa_forward_static(const isa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                       uint16_t* out, void* stream);

/* All four stages on HOST buffers, end to end: copies q, k, v in, runs the
 * forward and copies out back, for callers whose tensors live in host
 * memory.  (The ISA pages have no counterpart; this is a packaging of the
 * same path.)  Every (b, h) is independent, so the B*H heads are taken in
 * `groups` consecutive slices (groups <= 0: two heads a slice from 8 heads
 * on, else one slice); the copy-in of a slice on stream_in, the forward of
 * the one before on stream_compute (isa_forward on the slice) and the
 * copy-out of the one before that on stream_out run at once, so both PCIe
 * directions overlap the kernels.  Each (b, h) gets the same index sets as
 * under isa_forward; only the merge of the full-attention key-split tail
 * can round differently (it depends on how many heads share a launch).
 *   hq, hk, hv   [B, H, N, d] bf16 in (pinned host memory for asynchronous
 *                copies; pageable memory works, with synchronous copies).
 *   hout         [B, H, N, d] bf16 out (host memory).
 *   staging      device buffer of staging_bytes >= isa_host_staging_size(
 *                shape, groups) bytes, 16-byte aligned, owned by the caller:
 *                a workspace for one slice (its first 256 bytes are the
 *                control block; isa_read_device_status(staging, ...) reads
 *                its status word) and a ring of up to 3 slices of q, k, v,
 *                out.  Nothing else is allocated on the device.
 *   streams      stream_in / stream_out may be NULL (then stream_compute is
 *                used for the copies too, without overlap).
 * The call returns once everything is enqueued; the last copy-out is
 * ordered before any later work on stream_compute, so synchronising
 * stream_compute makes hout complete.  hq, hk, hv must not change and hout
 * must not be read before then.  Argument errors return before anything is
 * enqueued; an error from a slice's isa_forward is returned as it is, with
 * earlier slices already enqueued.  isa_host_staging_size returns 0 for an
 * invalid shape. */
size_t isa_host_staging_size(const isa_shape* shape, int groups);
int isa_forward_host(const isa_shape* shape, const uint16_t* hq, const uint16_t* hk, const uint16_t* hv,
                     uint16_t* hout, void* staging, size_t staging_bytes, int groups, void* stream_compute,
                     void* stream_in, void* stream_out);

/* In-house dense flash attention (the latency baseline; equals ISA at
 * keep = rho = 1): out = softmax(scale q k^T) v over all N keys, per (b, h),
 * non-causal.  scale <= 0 selects 1/sqrt(d).  ws: a zeroed buffer of
 * isa_dense_workspace_size(d) bytes (control block as above, then scratch
 * for the key-split tail; a smaller ws >= 256 bytes also works, without
 * the split).  isa_dense_workspace_size returns 0 for an unsupported d. */
size_t isa_dense_workspace_size(int d);
int isa_dense_attn_fwd(int B, int H, int N, int d, float scale, const uint16_t* q,
                       const uint16_t* k, const uint16_t* v, uint16_t* out,
                       void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream`, returns the device status word of ws (an
 * isa_status) and resets it to 0.  Returns ISA_ERR_CUDA if reading fails. */
int isa_read_device_status(void* ws, void* stream);

/* Static description of a status code. */
const char* isa_status_string(int status);

/* Description of the CUDA error behind the calling thread's most recent
 * ISA_ERR_CUDA (a static string owned by the CUDA runtime). */
const char* isa_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* ISA_H_ */
