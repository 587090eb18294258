/*
 * libnabla — NABLA adaptive block-sparse attention for 3D video token grids,
 * native to NVIDIA B200 (sm_100a).
 *
 * The library exports a plain C ABI: device pointers, sizes and a CUDA stream
 * (passed as an opaque pointer; cudaStream_t converts to it).  No call
 * allocates device memory; the caller owns every buffer, including the
 * workspace.  Every call is asynchronous on the given stream and returns
 * argument errors immediately.  Errors found on the device (a CSR capacity
 * overflow, a bad block index, a pipeline wait that ran out) are OR-ed into a
 * status word at the head of the workspace and reported by
 * nabla_query_status().
 *
 * Conventions shared by all calls
 *   Q, K, V, O : bf16, [B, H, S, d] row-major; 16-byte aligned base pointers.
 *   LSE        : fp32, [B, H, S]; natural log of sum_j exp(scale * q_i . k_j)
 *                over the keys row i attends to.
 *   Blocks     : 64 consecutive tokens.  nb = S / 64.  Tokens are ordered
 *                tile-major, so block r is the 4x4x4 token tile number r of a
 *                tile grid Tt x Th x Tw in (t, h, w) raster order.
 *   Block CSR  : row_ptr int32 [B*H*nb + 1], col_idx int32 [nnz]; global row
 *                g = (b*H + h)*nb + r lists the key blocks query block r of
 *                head (b, h) attends to.  Column indices are head-local
 *                (0 <= c < nb).
 *   Supported  : d in {64, 128}; S % 64 == 0; 1 <= nb <= 4096;
 *                B*H*nb*nb < 2^31.
 */
#ifndef NABLA_H_
#define NABLA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NABLA_API __attribute__((visibility("default")))
#else
#define NABLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t is `struct CUstream_st*`; this alias keeps the header free of
 * CUDA includes.  NULL is the legacy default stream. */
typedef struct CUstream_st* nabla_stream_t;

typedef enum {
    NABLA_OK = 0,
    NABLA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer */
    NABLA_ERR_UNSUPPORTED = 2,  /* shape outside the supported set above */
    NABLA_ERR_CAPACITY = 3,     /* the kept blocks did not fit col_capacity */
    NABLA_ERR_CUDA = 4,         /* a CUDA runtime call failed; see nabla_last_error() */
    NABLA_ERR_TIMEOUT = 5,      /* a device pipeline wait ran out; the kernel returned early */
    NABLA_ERR_BAD_INDEX = 6     /* a CSR column index outside [0, nb) was skipped */
} nabla_status;

typedef struct {
    int32_t B, H, S, d;   /* batch, heads, tokens, head dim */
    int32_t Tt, Th, Tw;   /* tile grid (4x4x4-token tiles); Tt*Th*Tw must equal S/64 */
    int32_t layout;       /* token order of Q, K, V, O, LSE along S: NABLA_LAYOUT_TILE_MAJOR
                             (0; block r = tokens 64r..64r+63) or NABLA_LAYOUT_RASTER (1;
                             token (t,h,w) at (t*H + h)*W + w of the 4Tt x 4Th x 4Tw grid,
                             block r = tile r of the grid, read in place: the reorder of the
                             NABLA review's Figure 4 fused into the loads and the O/LSE
                             stores).  RASTER needs the tile grid and is accepted by
                             nabla_build_mask, bsa_fwd and bsa_fwd_with_mask(_static); the
                             other calls return NABLA_ERR_UNSUPPORTED for it. */
} nabla_shape;

enum { NABLA_LAYOUT_TILE_MAJOR = 0, NABLA_LAYOUT_RASTER = 1 };

typedef struct {
    float thr;            /* keep the smallest sorted prefix with mass >= 1 - thr; thr in [0, 1] */
    int32_t use_sta;      /* nonzero: OR in the sliding-tile window below */
    int32_t wt, wh, ww;   /* STA half-window in tiles along t, h, w (>= 0) */
    int32_t topk;         /* > 0: keep the topk most probable blocks per row instead of the
                             mass rule (thr is then ignored); 0: mass rule */
} nabla_mask_params;

enum {
    NABLA_OP_BUILD_MASK = 0,     /* workspace for nabla_build_mask */
    NABLA_OP_FWD = 1,            /* workspace for bsa_fwd */
    NABLA_OP_FWD_WITH_MASK = 2,  /* workspace for bsa_fwd_with_mask */
    NABLA_OP_BWD = 3,            /* workspace for bsa_bwd */
    NABLA_OP_BUILD_XATTN = 4     /* workspace for nabla_build_mask_xattn */
};

/* Bytes of workspace the operation needs for this shape (0 on a bad shape).
 * The first 256 bytes are a header holding the device status word; zero them
 * once with nabla_workspace_init() before the first call. */
NABLA_API size_t nabla_workspace_size(const nabla_shape* shape, int op);

/* Zero the workspace header (status word) on `stream`. */
NABLA_API nabla_status nabla_workspace_init(void* workspace, nabla_stream_t stream);

/* Read and clear the device status word: synchronises `stream`, returns
 * NABLA_OK or the first device-side error recorded since the last query. */
NABLA_API nabla_status nabla_query_status(void* workspace, nabla_stream_t stream);

/*
 * NABLA mask builder (Algorithm 1 of "NABLA: Neighborhood Adaptive
 * Block-Level Attention"; its reading in the pith.science review, sections
 * "What carries the argument" and "Core claim", and referee minor comment 2).
 * Per head: mean-pool Q and K over each 64-token block, form the reduced map
 * Qbar Kbar^T / sqrt(d), softmax each row, order each row's blocks by
 * descending probability (ties: lower block index first) and keep the
 * smallest prefix whose mass reaches 1 - thr (thr == 0 keeps every block; the
 * top block is always kept).  With use_sta, OR in the sliding-tile window of
 * "Sliding Tile Attention" (clipped at the grid edge).  The result is written
 * as block CSR with ascending column indices per row.
 * With params->topk > 0 the row keeps instead its topk most probable blocks
 * (same order and ties), the fixed-budget baseline the NABLA paper's
 * Appendix C compares the mass rule with.
 *
 *   q, k          device bf16 [B,H,S,d]
 *   mask_u8       optional device uint8 [B,H,nb,nb] (1 = kept), or NULL
 *   row_ptr       device int32 [B*H*nb + 1]
 *   col_idx       device int32 [col_capacity]; B*H*nb*nb always suffices
 *   nnz_out       optional device int32 [1]: total kept blocks, or NULL
 *   workspace     device, nabla_workspace_size(shape, NABLA_OP_BUILD_MASK) bytes
 * If the kept blocks exceed col_capacity, col_idx is left partly written and
 * NABLA_ERR_CAPACITY is recorded in the status word; row_ptr is still exact.
 */
NABLA_API nabla_status nabla_build_mask(const nabla_shape* shape, const nabla_mask_params* params,
                              const void* q, const void* k, uint8_t* mask_u8, int32_t* row_ptr,
                              int32_t* col_idx, int64_t col_capacity, int32_t* nnz_out,
                              void* workspace, nabla_stream_t stream);

/*
 * Block-sparse attention forward (FlashAttention's tiled online softmax, as
 * in the FlashAttention abstract's block-sparse extension; NABLA feeds it the
 * mask above in place of FlexAttention).  For each query block r of head
 * (b, h) and each key block j listed in its CSR row, accumulate
 * softmax(scale * Q_r K_j^T) V_j exactly over the listed blocks.
 *
 *   q, k, v       device bf16 [B,H,S,d]
 *   row_ptr       device int32 [B*H*nb + 1], col_idx device int32 (head-local)
 *   scale         softmax scale; <= 0 selects 1/sqrt(d)
 *   o             device bf16 [B,H,S,d]
 *   lse           device fp32 [B,H,S] (may be NULL)
 *   workspace     device, nabla_workspace_size(shape, NABLA_OP_FWD) bytes: the
 *                 256-byte header for tile-major tokens; for raster token
 *                 order (256-byte aligned) also tile-major copies of K and V
 *                 (2 * B*H*S*d bf16), which the call fills with the token
 *                 reorder before the attention kernels, so that only Q, O and
 *                 LSE are addressed in raster order inside them
 * A query block with an empty list gets O = 0 and LSE = -inf.  Duplicate
 * column indices count once; indices outside [0, nb) are skipped and recorded
 * as NABLA_ERR_BAD_INDEX.
 * The call is one kernel launch.  Each query tile (two query blocks) takes,
 * per row, the max of the first key tile the row's block lists as the softmax
 * reference and keeps it; if a later tile's scores exceed that reference by
 * more than 16 in log2 units (a tile's partial row sum above 2^16), the query
 * tile is computed again with the reference raised as the scores grow.  Word
 * 1 of the workspace header is set when any tile of the call was recomputed,
 * and word 2 counts the calls that needed it (nabla_query_exact_passes); the
 * result does not depend on which pass produced it beyond rounding.  One
 * workspace must not serve two calls that may run at the same time.
 */
NABLA_API nabla_status bsa_fwd(const nabla_shape* shape, const void* q, const void* k, const void* v,
                     const int32_t* row_ptr, const int32_t* col_idx, float scale, void* o,
                     float* lse, void* workspace, nabla_stream_t stream);

/*
 * Block-sparse attention forward with a caller-supplied static block mask
 * (the calibrated per-(timestep, layer, head) masks of "Accelerating
 * Text-to-Video Generation with Calibrated Sparse Attention", section B
 * "Inference": precomputed binary masks, only the selected blocks computed).
 *
 *   mask_u8       device uint8 [B,H,nb,nb]; nonzero = attend to the block
 *   workspace     device, nabla_workspace_size(shape, NABLA_OP_FWD_WITH_MASK),
 *                 256-byte aligned (raster token order: with the K/V copies
 *                 at its end, as for bsa_fwd)
 * Other arguments as for bsa_fwd.  The mask is compacted to block CSR inside
 * the workspace, then bsa_fwd runs on it.
 */
NABLA_API nabla_status bsa_fwd_with_mask(const nabla_shape* shape, const void* q, const void* k,
                               const void* v, const uint8_t* mask_u8, float scale, void* o,
                               float* lse, void* workspace, nabla_stream_t stream);

/*
 * Static-mask attention forward that allocates nothing (no counterpart in the
 * paper; it exists for callers that cannot allocate device memory).
 *
 * Some callers cannot call cudaMalloc or hand over a workspace: a serving
 * runtime that owns all device memory through its own pool, code running
 * inside another framework's CUDA-graph capture, or an embedded host with a
 * fixed memory budget.  This call computes exactly what bsa_fwd_with_mask
 * computes, but keeps the block CSR it builds from the mask in a fixed
 * device array owned by the library (NABLA_STATIC_SCRATCH_BYTES, 32 MiB, held
 * on each device that has used it until the process exits).  It allocates
 * nothing and takes no workspace; with raster token order, K and V are read
 * in place by 5D boxes (no tile-major copies), which is slower.
 *
 *   q, k, v, mask_u8, scale, o, lse   as for bsa_fwd_with_mask
 *   status_out   optional device int32 [1], or NULL: receives the call's
 *                device status bits (0 = completed; 1 = a pipeline wait ran
 *                out) in stream order
 * Returns NABLA_ERR_UNSUPPORTED, with a message, when the shape's block CSR
 * does not fit the array (B*H*(S/64)^2 above roughly 8.3 million blocks).
 * Every call shares the one array: calls whose GPU work can overlap (other
 * streams without ordering) race; calls on one stream are safe.  The first
 * call on each device looks up the array's device address; make it before
 * any stream capture starts.
 */
#define NABLA_STATIC_SCRATCH_BYTES (32u * 1024u * 1024u)
NABLA_API nabla_status bsa_fwd_with_mask_static(const nabla_shape* shape, const void* q,
                                                const void* k, const void* v,
                                                const uint8_t* mask_u8, float scale, void* o,
                                                float* lse, int32_t* status_out,
                                                nabla_stream_t stream);

/*
 * One NABLA attention layer on host-resident tensors: per head, the mask of
 * nabla_build_mask (Algorithm 1 of the NABLA paper, optional STA union) and
 * then bsa_fwd over it, with Q, K, V read from and O, LSE written to host
 * memory.  The result equals nabla_build_mask + bsa_fwd (scale 1/sqrt(d)) on
 * device copies of the same tensors.
 *
 * Heads are independent, so the call moves them in chunks of at most
 * heads_per_chunk heads through two device slots: while chunk c computes,
 * chunk c+1's inputs go host-to-device and chunk c-1's outputs go
 * device-to-host on two streams the library owns, ordered with events.  The
 * slots compute on `stream` and on a third library stream, so consecutive
 * chunks' kernels may overlap on the GPU.  With
 * page-locked (pinned) host buffers the copies overlap the kernels; pageable
 * buffers give the same result without the overlap.  The chunks ramp up
 * (1, 2, 4, ... heads) and end on a chunk of heads_per_chunk/4 heads, so that
 * the first input copy and the last output copy, which overlap nothing, stay
 * short; nabla_layer_host_chunks gives the schedule.
 *
 *   q_host, k_host, v_host   host bf16 [B,H,S,d], tile-major tokens
 *   o_host                   host bf16 [B,H,S,d]
 *   lse_host                 host fp32 [B,H,S]
 *   heads_per_chunk          heads per pipeline chunk (> 0; 4 suits S = 76800)
 *   workspace    device, nabla_layer_host_workspace_size(shape, heads_per_chunk)
 *                bytes, 256-byte aligned; its first 256 bytes are the status
 *                header (nabla_workspace_init once, nabla_query_status after)
 * Returns once the work is queued.  All of it, the last output copy
 * included, is ordered before anything later queued on `stream`: synchronise
 * `stream` before reading o_host or lse_host.  Argument errors (the mask
 * parameters included) return before anything is queued; a CUDA error part
 * way through still orders every copy already queued before later work on
 * `stream`, so the host buffers are free once `stream` is synchronised.  The library's streams are
 * per device, so two calls in flight at once on one device (other host
 * threads, or other streams without ordering) are not supported.
 */
NABLA_API size_t nabla_layer_host_workspace_size(const nabla_shape* shape, int heads_per_chunk);
/* Chunk schedule of nabla_layer_host for `heads` = B*H heads: returns the
 * number of chunks (0 on a non-positive argument) and writes the first
 * min(count, capacity) chunk sizes, in order, to host `sizes` (may be NULL). */
NABLA_API int64_t nabla_layer_host_chunks(int64_t heads, int heads_per_chunk, int32_t* sizes,
                                          int64_t capacity);
NABLA_API nabla_status nabla_layer_host(const nabla_shape* shape, const nabla_mask_params* params,
                                        const void* q_host, const void* k_host,
                                        const void* v_host, void* o_host, float* lse_host,
                                        int heads_per_chunk, void* workspace,
                                        nabla_stream_t stream);

/*
 * Block mask from XAttention antidiagonal scores instead of the pooled map
 * ("XAttention: Block Sparse Attention with Antidiagonal Scoring" notes:
 * blocks scored along antidiagonals, selected by a threshold).  With stride St
 * (4, 8 or 16), strided rows i, j of a head score
 *     a_ij = (1/St) sum_{s<St} q_{i*St + St-1-s} . k_{j*St + s} / sqrt(d)
 * (the mean of the antidiagonal of the St x St sub-block of Q K^T), p_i =
 * softmax over all strided keys, and block (r, c) scores the mean over r's
 * 64/St strided rows of the mass p puts on c's strided keys; each row of
 * scores sums to 1.  The scores then go through nabla_build_mask's selection
 * (params: thr mass rule or topk, optional STA window; the tile grid is
 * needed only for the STA window), giving the same CSR outputs.
 *   scores   device fp32 [B,H,nb,nb] or NULL (then kept in the workspace)
 *   workspace  device, nabla_workspace_size(shape, NABLA_OP_BUILD_XATTN) bytes
 * Other arguments as for nabla_build_mask; tile-major tokens only.
 */
NABLA_API nabla_status nabla_build_mask_xattn(const nabla_shape* shape,
                                              const nabla_mask_params* params, int32_t stride,
                                              const void* q, const void* k, float* scores,
                                              uint8_t* mask_u8, int32_t* row_ptr,
                                              int32_t* col_idx, int64_t col_capacity,
                                              int32_t* nnz_out, void* workspace,
                                              nabla_stream_t stream);

/*
 * Block-sparse attention backward: the gradients of bsa_fwd's O with respect
 * to Q, K and V over the same block CSR (FlashAttention's backward, which
 * recomputes P from the saved LSE; NABLA trains through the same block mask,
 * "NABLA: Neighborhood Adaptive Block-Level Attention", review summary).  With
 * P = exp(scale Q K^T - LSE) on kept blocks (0 elsewhere) and
 * D_i = sum_k dO_ik O_ik:
 *     dV = P^T dO,  dS = P o (dO V^T - D),  dQ = scale dS K,  dK = scale dS^T Q
 *   q, k, v, o, dout   device bf16 [B,H,S,d], 16-byte aligned; o and lse are
 *                      bsa_fwd's outputs for the same q, k, v, CSR and scale
 *   lse                device fp32 [B,H,S], 16-byte aligned
 *   row_ptr, col_idx   the forward's block CSR (any column order; duplicates
 *                      count once; out-of-range indices are skipped and
 *                      reported as NABLA_ERR_BAD_INDEX)
 *   scale              <= 0 selects 1/sqrt(d)
 *   dq, dk, dv         device bf16 [B,H,S,d] outputs, written in full (rows
 *                      that no kept block reaches get 0)
 *   workspace          device, nabla_workspace_size(shape, NABLA_OP_BWD) bytes
 * Stream-ordered; deterministic (no atomics in the gradient sums).
 */
NABLA_API nabla_status bsa_bwd(const nabla_shape* shape, const void* q, const void* k,
                               const void* v, const void* o, const void* dout, const float* lse,
                               const int32_t* row_ptr, const int32_t* col_idx, float scale,
                               void* dq, void* dk, void* dv, void* workspace,
                               nabla_stream_t stream);

/*
 * Token reordering between raster and tile-major order (the neighbourhood
 * reorder of "NABLA: Neighborhood Adaptive Block-Level Attention", review
 * Figure 4, with 4x4x4 tiles: each 64-token attention block becomes one tile
 * of the T x H x W = 4Tt x 4Th x 4Tw token grid).
 *   raster      s_r = (t*H + h)*W + w
 *   tile-major  s_m = ((tt*Th + th)*Tw + tw)*64 + (ut*4 + uh)*4 + uw,
 *               t = 4tt + ut, h = 4th + uh, w = 4tw + uw
 * NABLA_TO_TILE_MAJOR moves token s_r of src to s_m of dst; NABLA_TO_RASTER is
 * the inverse (for O after attention).  src, dst: device [B,H,S,d] rows of d
 * 16-bit elements (bf16), 16-byte aligned, not aliasing; S = 64*Tt*Th*Tw;
 * d a multiple of 8.  Stream-ordered; no workspace.
 */
enum { NABLA_TO_TILE_MAJOR = 0, NABLA_TO_RASTER = 1 };
NABLA_API nabla_status nabla_reorder_tokens(const nabla_shape* shape, int direction,
                                            const void* src, void* dst, nabla_stream_t stream);

/*
 * Block attention energy: for every (query block r, key block c) pair listed
 * in the block CSR, the softmax mass the 64 queries of r place on the 64 keys
 * of c, averaged over the queries:
 *     E[r][c] = (1/64) sum_{i in r} sum_{j in c} exp(scale * q_i.k_j - lse_i)
 * This is the per-block "energy" that CalibAtt's offline calibration
 * thresholds ("Accelerating Text-to-Video Generation with Calibrated Sparse
 * Attention", section 2 "Methodologie: CalibAtt", A "Offline Kalibratie") and the true block mass of the fidelity check the NABLA
 * review asks for (major comment 1).  With lse from a dense bsa_fwd (every
 * block listed) each row of E sums to 1.
 *   q, k        device bf16 [B,H,S,d], 16-byte aligned (tile-major tokens)
 *   lse         device fp32 [B,H,S] natural-log LSE per query row; a row with
 *               lse = -inf (or any non-finite value) contributes nothing
 *   row_ptr, col_idx  block CSR as for bsa_fwd (the blocks to evaluate)
 *   scale       softmax scale; <= 0 selects 1/sqrt(d)
 *   energy      device fp32 [B,H,nb,nb], written in full: unlisted blocks 0
 *   block_mass  device fp32 [B,H,nb] or NULL: sum of the row's listed E
 *   workspace   device, nabla_workspace_size(shape, NABLA_OP_FWD) bytes
 * Device-side failures (timeouts, bad column indices) are recorded in the
 * workspace status word; a CTA that timed out leaves its two rows unwritten.
 */
NABLA_API nabla_status nabla_block_energy(const nabla_shape* shape, const void* q, const void* k,
                                          const float* lse, const int32_t* row_ptr,
                                          const int32_t* col_idx, float scale, float* energy,
                                          float* block_mass, void* workspace,
                                          nabla_stream_t stream);

/*
 * Calibrated static masks (CalibAtt, Methodology A: per (timestep, layer,
 * head) the minimal block set holding 1 - eps of each row's energy, averaged
 * over the calibration runs; blocks that are consistently missed are skipped).
 * nabla_calib_accumulate applies the minimal-prefix rule of nabla_build_mask
 * (thr = eps, ties to the lower block index, the largest block always kept,
 * eps = 0 keeps every block) to each row of energy normalised by its sum, and
 * adds 1 to votes[b,h,r,c] for each kept block; a row whose energy sums to 0
 * keeps nothing.  Call it once per calibration run (eps is the caller's eps(t)
 * for the timestep being calibrated), starting from votes = 0.
 * nabla_calib_finalize writes mask_u8 = (votes >= min_votes), the uint8
 * [B,H,nb,nb] mask that bsa_fwd_with_mask takes; min_votes = 1 skips exactly
 * the blocks no run selected.
 *   energy   device fp32 [B,H,nb,nb];  votes  device int32 [B,H,nb,nb]
 * Both calls are stream-ordered and need no workspace.
 */
NABLA_API nabla_status nabla_calib_accumulate(const nabla_shape* shape, const float* energy,
                                              float eps, int32_t* votes, nabla_stream_t stream);
NABLA_API nabla_status nabla_calib_finalize(const nabla_shape* shape, const int32_t* votes,
                                            int32_t min_votes, uint8_t* mask_u8,
                                            nabla_stream_t stream);

/* Message for the last error returned on the calling host thread. */
NABLA_API const char* nabla_last_error(void);

/* ABI version (major * 10000 + minor * 100 + patch). */
NABLA_API int nabla_version(void);

/*
 * Diagnostics and tuning (not part of the method).
 *
 * nabla_set_wait_limit_ns: time limit of every pipeline wait inside the
 * attention kernel, in nanoseconds (0 restores the default of 2 s).  A wait
 * that runs out makes the kernel drain its copies in flight, free its tensor
 * memory, record NABLA_ERR_TIMEOUT and return.  Tests set a tiny limit to
 * check that path without hanging anything.
 *
 * nabla_set_exact_reference: 1 makes every forward compute every query tile
 * with the exact reference only (the reference raised as each row's scores
 * grow); 0 (the default) restores the scheme described at bsa_fwd.
 * Process-wide; for tests and for reproducing the exact-reference numerics.
 *
 * nabla_set_pair_mode: which kernel runs a d = 128 tile-major forward's
 * fixed-reference pass.  0 (the default): one CTA per two query blocks.  1: CTA
 * pairs (each pair of CTAs walks the union of four query blocks' lists with
 * M = 256 products, each CTA loading half of every K and V tile) for block
 * lists from nabla_build_mask (bsa_fwd, nabla_layer_host), one CTA for caller
 * masks.  2: CTA pairs always.  Process-wide; the results agree within
 * rounding either way.  The pair kernel is slower on the layers measured here
 * (its cross-SM handshakes lie on every tile's critical path).
 *
 * nabla_query_exact_passes: synchronises the stream and returns word 2 of a
 * forward workspace's header: how many forwards on it needed the
 * exact-reference recomputation of a query tile since nabla_workspace_init
 * (-1 on a CUDA error).
 *
 * nabla_selftest_mma_pair: one product over a pair of CTAs (tcgen05
 * cta_group::2, M = 256), each CTA holding half of A and half of B:
 *   variant 0: C [256][256] = A B^T, a = A [256][128], b = B [256][128] (bf16)
 *   variant 1: C [256][128] = P V, a = P [256][256] (staged in tensor memory),
 *              b = V [256][128] (bf16, N-major halves)
 *   c: device fp32, row-major.
 *
 * nabla_build_mask_stage_ms: runs nabla_build_mask once (no uint8 mask) with
 * CUDA events between its kernels, synchronises the stream, and writes the
 * milliseconds of its four stages to ms_out[0..3]: pooling, the reduced map,
 * the selection, the CSR compaction.  Arguments as for nabla_build_mask.
 *
 * nabla_selftest_fp64_tflops: times independent fp64 fma chains on every SM
 * (a few milliseconds), synchronises the stream and writes the measured fp64
 * rate in TFLOP/s: the denominator of the reduced map's roofline.
 *
 * nabla_selftest_fp64_exp_rate: times independent chains of fp64 exp on every
 * SM (a few milliseconds), synchronises the stream and writes the measured
 * rate in 1e9 exponentials per second: the denominator of the selection's
 * arithmetic roofline (one fp64 exp per entry of the reduced map).
 *
 * nabla_selftest_ex2_rate: the same for the fp32 ex2.approx instruction (the
 * exponential unit), in 1e9 per second: the floor of the block-energy kernel,
 * which takes 4,096 exponentials per kept 64 x 64 block.
 * All three return NABLA_ERR_INVALID_ARG for a NULL output before any CUDA
 * call.
 *
 * nabla_selftest_mma: one 128 x N x 128 bf16 product through the same
 * tcgen05/TMA building blocks the attention kernel uses, for layout checks.
 *   variant 0: C[m][n] = sum_k A[m][k] B[n][k]   (both K-major, N = 128)
 *   variant 1: C[m][n] = sum_k A[m][k] B[k][n]   (B N-major, one N=128 MMA)
 *   variant 2: as 1 with two N=64 MMAs
 *   variant 3: as 1 with A staged in tensor memory
 *   a, b: device bf16 [128][128] row-major; c: device fp32 [128][128].
 */
NABLA_API void nabla_set_wait_limit_ns(uint64_t ns);
NABLA_API void nabla_set_exact_reference(int on);
NABLA_API void nabla_set_pair_mode(int mode);
NABLA_API int nabla_query_exact_passes(const void* workspace, nabla_stream_t stream);
NABLA_API nabla_status nabla_selftest_mma(int variant, const void* a, const void* b, float* c,
                                void* workspace, nabla_stream_t stream);
NABLA_API nabla_status nabla_build_mask_stage_ms(const nabla_shape* shape,
                                                 const nabla_mask_params* params, const void* q,
                                                 const void* k, int32_t* row_ptr, int32_t* col_idx,
                                                 int64_t col_capacity, int32_t* nnz_out,
                                                 void* workspace, nabla_stream_t stream,
                                                 float* ms_out);
NABLA_API nabla_status nabla_selftest_fp64_tflops(nabla_stream_t stream, double* tflops_out);
NABLA_API nabla_status nabla_selftest_fp64_exp_rate(nabla_stream_t stream, double* gexp_out);
NABLA_API nabla_status nabla_selftest_ex2_rate(nabla_stream_t stream, double* gexp_out);
NABLA_API nabla_status nabla_selftest_mma_pair(int variant, const void* a, const void* b, float* c,
                                               void* workspace, nabla_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* NABLA_H_ */
