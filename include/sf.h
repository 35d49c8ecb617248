/*
 * sf.h -- C ABI of the B200 sparse training step of Sparse-First fine-tuning.
 *
 * Source of the method: the Sparse-First fine-tuning page (tensorwirelabs.com,
 * paper-sparse-first). A training step touches active rows only and runs:
 *   sf_mask_update   section 2.1  per-row masks from the charge rule (conductor / row tracker)
 *   sf_masked_dw     section 2.2  dW = dX^T A, all-empty 32-row tiles skipped outright
 *   sf_embed_grad    sections 1, 2.2  embedding-row gradient of the active rows only
 *   sf_sparse_update sections 2.3-2.4  fused int8 + residual rebuild, coupled Adam step,
 *                                      requantisation and masked write-back of live weights
 *
 * Conventions shared by every call
 *   - Pointers are DEVICE pointers unless a comment says "host". The caller owns and allocates
 *     every buffer; the library allocates nothing and keeps no state between calls.
 *   - Every call only enqueues work on `stream` (a cudaStream_t; NULL is the legacy default
 *     stream) and returns. No call waits on the device or reads results back (section 2.6
 *     prepares step N only from what step N-1 left behind); conditions found on the device are
 *     OR-ed into the device word *dev_status (SF_STATUS_* bits), which the caller reads after
 *     the step. dev_status may be NULL.
 *   - The return value reports, synchronously and before any work is enqueued, argument, shape
 *     and alignment errors (SF_ERR_*), and launch errors (SF_ERR_CUDA). On an error nothing of
 *     the call has been enqueued, except for SF_ERR_CUDA from a later launch of a multi-launch
 *     call, which the message string names.
 *   - Results are deterministic: the same inputs give the same bits, run to run.
 *   - Hardware: NVIDIA B200 (sm_100a) only.
 *
 * Matrix layout. A weight matrix W has R rows (output features) and C columns (input
 * features), row-major. A row's mask bit, moments, gradient and Adam step count follow the row;
 * "tile" w is rows 32w .. 32w+31. R must be a multiple of 32 and C a multiple of 8.
 */
#ifndef SF_H
#define SF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes ---------------------------------------------------------------------- */
#define SF_OK               0
#define SF_ERR_ARG         -1   /* null pointer, bad size, inconsistent shapes */
#define SF_ERR_ALIGN       -2   /* a pointer or leading dimension breaks the 16-byte rule */
#define SF_ERR_UNSUPPORTED -3   /* a size beyond what this build handles (see each call) */
#define SF_ERR_CUDA        -4   /* a CUDA runtime call or launch failed */
#define SF_ERR_NO_DEVICE   -5   /* no sm_100 device is current */

/* ---- device status bits (OR-ed into *dev_status) --------------------------------------- */
#define SF_STATUS_SLOT_OVERFLOW  0x1u  /* an active row found no free moment slot; it is not updated */
#define SF_STATUS_NONFINITE      0x2u  /* a non-finite gradient, moment or weight was produced */
#define SF_STATUS_BAD_TOKEN      0x4u  /* a token or row id outside [0, R) was ignored */
#define SF_STATUS_WAIT_TIMEOUT   0x8u  /* a kernel gave up a bounded wait and skipped its work */
/* Test hook: with SF_TEST_DW_WITHHOLD=1 in the environment, sf_masked_dw's first launch withholds
 * one pipeline stage of CTA 0, so that a bounded wait runs out and WAIT_TIMEOUT is raised. */

typedef void *sf_stream;               /* cudaStream_t */

/*
 * Row-mask state of one matrix (an embedding table or a projection). All arrays are device
 * memory owned by the caller; sf_mask_init() puts them in their starting state.
 *   charge[R]        float   per-row charge q_r of the charge rule (section 2.1)
 *   accum[R]         uint32  per-window accumulator; the library keeps it zero between calls.
 *                            Token sources count hits in it, one uint32 per row; output sources
 *                            (SF_SRC_OUTPUT_BF16, sf_forward_tracked) keep the row magnitude as
 *                            bf16 in its first 2R bytes, and then need it 16-byte aligned
 *   words[R/32]      uint32  the mask: bit i of words[w] is row 32w+i
 *   active_rows[R]   int32   active rows, ascending; the first counts[0] are valid
 *   active_tiles[R/32] int32 tiles holding an active row, ascending; first counts[1] valid
 *   tile_rows[R/32]  int32   for the j-th active tile, the number of active rows in the tiles
 *                            before it (the position of its first row in active_rows)
 *   row_slot[R]      int32   moment/gradient slot of each row, -1 for none
 *   free_slots[slot_cap] int32  stack of free slots (the top counts[2] entries)
 *   slot_step[slot_cap]  int32  Adam step count of each slot; 0 marks fresh (zero) moments
 *   counts[8]        int32   [0] active rows, [1] active tiles, [2] free slots, [3] active rows
 *                            with no slot, [4] rows that took a fresh slot in the last call,
 *                            [5] used inside sf_mask_update (zero between calls), [6..7]
 *                            reserved (zero)
 * Moments exist only for active rows (section 2.3): a row that turns active takes a free slot
 * with fresh moments, a row that turns inactive returns its slot and its moments are dropped.
 * Slot numbers are an implementation detail; compare state by row.
 */
typedef struct sf_mask {
    int32_t   R;
    int32_t   slot_cap;
    float    *charge;
    uint32_t *accum;
    uint32_t *words;
    int32_t  *active_rows;
    int32_t  *active_tiles;
    int32_t  *tile_rows;
    int32_t  *row_slot;
    int32_t  *free_slots;
    int32_t  *slot_step;
    int32_t  *counts;
} sf_mask;

/* Reset a mask to its starting state: zero charge, no active row, every slot free.
 * Errors: SF_ERR_ARG for a null array, R not a positive multiple of 32, slot_cap < 0. */
int sf_mask_init(const sf_mask *mk /* host */, sf_stream stream);

/* ---- sf_mask_update: section 2.1, "Observing activity" ---------------------------------
 * Folds one observation window into each mask and rebuilds its lists and slots.
 * Per row r: share_r = h_r / max_r' h_r' (0 when every h is 0), an fp32 division;
 *            charge_r <- charge_r / 2 + share_r / 2;   row r active while charge_r >= threshold
 * (the pages use 0.01). The activity h_r of a window depends on the source:
 *   SF_SRC_TOKENS      ptr = int32 token ids [n]: h_r = occurrences of id r (the conductor).
 *                      Ids outside [0, R) are ignored and set SF_STATUS_BAD_TOKEN.
 *   SF_SRC_OUTPUT_BF16 ptr = bf16 forward outputs Y [n x ld] (n tokens, columns = rows of W):
 *                      h_r = max over tokens of |Y[t, r]| (the row tracker). ptr and ld*2
 *                      must be 16-byte aligned. A NaN output carries no magnitude (it is
 *                      skipped); an infinite output counts as the largest finite bf16
 *                      magnitude (3.3895e38), so charges stay finite. Either sets
 *                      SF_STATUS_NONFINITE.
 *   SF_SRC_HITS_U32    ptr = uint32 hit counts [R] counted by the caller (e.g. on the host).
 *   SF_SRC_WORDS       ptr = uint32 mask words [R/32]: the mask is set directly, the charge
 *                      is not touched (explicit masks).
 * Then: masks, ascending active row and tile lists, counts, and slots (released rows push their
 * slot, newly active rows pop one; a row that finds none sets SF_STATUS_SLOT_OVERFLOW and has
 * row_slot -1). `masks` and `srcs` are host arrays of n_masks entries; each entry is
 * independent. Errors: SF_ERR_ARG (shape / kind / null), SF_ERR_ALIGN, SF_ERR_UNSUPPORTED for
 * R > 262144 or slot_cap > R.
 * Launches, per batch of up to 240 masks: the accumulate pass (TOKENS and OUTPUT sources), then
 * the finalize: one launch (a CTA per mask), or three when a mask of the batch has
 * SF_MASK_SPLIT_ROWS rows or more (busiest row and charge rule over 2,048-row blocks of all the
 * batch's masks, then a CTA per mask for slots and lists), chained by programmatic dependent
 * launch. While the finalize runs, a mask's active_tiles and tile_rows hold intermediate bits.
 */
#define SF_MASK_SPLIT_ROWS 16384
#define SF_SRC_TOKENS       0
#define SF_SRC_OUTPUT_BF16  1
#define SF_SRC_HITS_U32     2
#define SF_SRC_WORDS        3

typedef struct sf_mask_src {
    int32_t     kind;
    int32_t     n;      /* TOKENS: ids in the window; OUTPUT: tokens (rows of Y); else unused */
    int64_t     ld;     /* OUTPUT: row stride of Y in elements (>= R, multiple of 8) */
    const void *ptr;
} sf_mask_src;

int sf_mask_update(const sf_mask *masks /* host [n_masks] */,
                   const sf_mask_src *srcs /* host [n_masks] */, int n_masks,
                   float threshold, uint32_t *dev_status, sf_stream stream);

/* ---- sf_masked_dw: section 2.2, "Masked backward pass" ----------------------------------
 * For every projection p: dW = dX^T A over T tokens, where dX [T x ld_dx] bf16 is the upstream
 * gradient of the projection's outputs (column r belongs to weight row r) and A [T x ld_a] bf16
 * its inputs. Masks are read one 32-row tile at a time: a tile whose mask word is zero is never
 * visited (nothing of it is loaded, multiplied or stored), and rows whose bit is clear inside
 * a live tile are discarded at the store. Active row r with slot k = row_slot[r] >= 0 gets
 *     dW[k * ld_dw + c] = sum_t dX[t, r] * A[t, c]      (fp32, accumulated in fp32 from bf16)
 * and nothing else of dW is written. Runs on the tensor cores (tcgen05, TMA) as persistent
 * launches over the work of all problems (as few launches as the kernel parameter space allows).
 * Consecutive problems that read the same A (same pointer, ld_a, C and T: the q, k, v projections
 * of a layer, or gate and up) are grouped: their rows share 128-row tensor-core tiles and A is
 * streamed once per group. With scratch `ws` (sf_masked_dw_ws_bytes() bytes, 16-byte aligned)
 * a group whose mask is scattered first gathers its active rows of dX into the scratch, so a
 * tile holds 128 active rows instead of four 32-row mask tiles; the choice is made on the device
 * from the live masks, per group, and does not change the result. With ws = NULL every group
 * runs on mask tiles. The launches of one call are chained with programmatic dependent launch:
 * they overlap one another, never the work enqueued before or after the call. Their pipeline
 * waits are bounded: a wait that runs out (2 s) sets SF_STATUS_WAIT_TIMEOUT and that CTA skips
 * the rest of its work (its dW rows are then not written). Requirements: T >= 0; C a multiple of
 * 8; when T > 0, ld_dx and ld_a multiples of 8 and dX, A 16-byte aligned; dW 16-byte aligned,
 * ld_dw a multiple of 4 and >= C. Errors: SF_ERR_ARG (also for ws smaller than needed),
 * SF_ERR_ALIGN, SF_ERR_UNSUPPORTED (slot_cap above 2^28).
 */
#define SF_DW_MAX_PER_LAUNCH 96   /* problems (and groups) per launch, at most */

typedef struct sf_dw_problem {
    const void *dX;     /* bf16 [T x ld_dx] */
    int64_t     ld_dx;
    const void *A;      /* bf16 [T x ld_a] */
    int64_t     ld_a;
    int32_t     T;
    int32_t     C;
    sf_mask     mask;   /* R = mask.R; reads words, active_tiles, counts, row_slot */
    float      *dW;     /* fp32 [mask.slot_cap x ld_dw], row = slot */
    int64_t     ld_dw;
} sf_dw_problem;

size_t sf_masked_dw_ws_bytes(const sf_dw_problem *probs /* host [n] */, int n);

/* Weight rows per tensor-core unit of this build (256: a CTA pair's cta_group::2 MMA; 128: one
 * CTA). A group runs in row mode when its active rows need fewer units than its mask tiles do
 * (UNIT / 32 tiles per unit). Host-side mirrors of that choice (e.g. for counting the work) ask
 * here. Needs no device. */
int sf_masked_dw_unit_rows(void);

int sf_masked_dw(const sf_dw_problem *probs /* host [n] */, int n, void *ws, size_t ws_bytes,
                 uint32_t *dev_status, sf_stream stream);

/* ---- sf_embed_grad: sections 1 and 2.2 (embedding rows) ---------------------------------
 * A row's gradient comes only from the batch positions holding its token, and only rows the
 * mask marks active are computed: for each active row r with slot k,
 *     G[k * ld_g + c] = sum over tokens t with tokens[t] == r of dY[t, c]
 * (fp32; an active row with no token gets zeros). dY is [n_tok x ld_dy] bf16, H columns.
 * Tokens of inactive rows are dropped. Deterministic: each row's tokens are summed in one fixed
 * order (ascending position, split over eight partial sums that are added in a fixed order).
 * Needs caller scratch `ws` of sf_embed_grad_ws_bytes() bytes (16-byte aligned).
 * Limits: n_tok <= 16384, slot_cap <= 49152 (SF_ERR_UNSUPPORTED beyond).
 * Requirements: H, ld_dy multiples of 8, ld_g multiple of 4 >= H, dY and G 16-byte aligned.
 */
size_t sf_embed_grad_ws_bytes(int n_tok, int slot_cap);

int sf_embed_grad(const int32_t *tokens, int n_tok, const void *dY, int H, int64_t ld_dy,
                  const sf_mask *mk /* host */, float *G, int64_t ld_g,
                  void *ws, size_t ws_bytes, uint32_t *dev_status, sf_stream stream);

/* ---- sf_embed_grad_noalloc: allocation-free variant of sf_embed_grad ------------------
 * No counterpart in the paper: an operational addition. Same inputs, result and guarantees as
 * sf_embed_grad, but without the caller's scratch buffer, for callers that must not allocate
 * device memory themselves (a plugin whose host framework owns every device allocation, or a
 * latency-critical loop that cannot afford cudaMalloc's implicit synchronisation). The scratch
 * is a fixed array of SF_EMBED_NOALLOC_SCRATCH_INTS int32 (256 KiB) in the library's own device
 * memory, present on every GPU that loads the library until the process exits; a call needs
 * 4 * slot_cap + 4 + n_tok of them and returns SF_ERR_UNSUPPORTED beyond that. The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress) and caches it for the
 * device's current context (a new context, e.g. after cudaDeviceReset, repeats the lookup); make
 * that first call before any stream capture. All calls on a GPU share the array: calls that can
 * overlap on the GPU (different streams or threads) race on it and must be ordered by the
 * caller. This entry point allocates nothing.
 */
#define SF_EMBED_NOALLOC_SCRATCH_INTS 65536

int sf_embed_grad_noalloc(const int32_t *tokens, int n_tok, const void *dY, int H, int64_t ld_dy,
                          const sf_mask *mk /* host */, float *G, int64_t ld_g,
                          uint32_t *dev_status, sf_stream stream);

/* ---- sf_sparse_update: sections 2.3 and 2.4 --------------------------------------------
 * Storage of a matrix (section 2.3): W = s*q + delta with q int8 [R x C], s fp32 [R] (one scale
 * per row), delta fp32 [R x C] the full-precision residual; moments m, v fp16 [slot_cap x C]
 * kept only for active rows; grad fp32 [slot_cap x C] (row = slot); live bf16 [R x C], the
 * weights the next forward pass reads (NULL: no write-back).
 * For each active row r of each matrix (rows without a slot are skipped), per column c:
 *   W   = fma(s, q, delta)                          rebuilt weight, held in registers only
 *   g_a = grad[slot(r)], g_b = partner grad[partner slot(r)] or 0 if the partner row is inactive
 *   g   = clamp(g, -clip, clip) for both when clip > 0
 *   gt  = fma(c_partner, g_b, c_self * g_a)         coupled pair mix (section 2.4); unpaired
 *                                                   matrices use c_self = 1, c_partner = 0
 *   m1  = fma(beta1, m, one_minus_b1 * gt),  v1 = fma(beta2, v, one_minus_b2 * gt * gt)
 *         (m = v = 0 when the slot is fresh)
 *   u   = (m1 * bc1[t]) / (sqrt(v1 * bc2[t]) + eps),   t = step count after this step
 *   W'  = fma(-lr, u, W), then W' = fma(-lr * wd, W, W') when wd != 0 (decoupled decay,
 *         wd = lambda * cos(alpha) in the pages' terms)
 *   m, v <- fp16(m1), fp16(v1)
 * then per row: s' = max|W'| / 127; q' = round-half-even(W' / s') in [-127, 127];
 * delta' = fma(-s', q', W') (s' = 0: q' = 0, delta' = W'); live = bf16(W').
 * Rows outside the mask are neither read nor written (section 2.3).
 * All matrices of a step go in one call: pairs (gate-up, query-output, key-value) name each
 * other through `partner`. A matrix reads its partner's gradient and row_slot only, so the
 * order inside the call does not matter. Non-finite results set SF_STATUS_NONFINITE.
 * bc1/bc2 are tables of 1/(1-beta^t) for t = 0..t_max (sf_adam_tables); a step count above
 * t_max uses entry t_max. Errors: SF_ERR_ARG, SF_ERR_ALIGN, SF_ERR_UNSUPPORTED for C > 32768.
 */
typedef struct sf_matrix {
    int32_t     C;
    int32_t     partner;     /* index into the mats array, -1 when unpaired */
    float       c_self;
    float       c_partner;
    sf_mask     mask;        /* R, active rows, row_slot, slot_step */
    int8_t     *q;
    float      *s;
    float      *delta;
    uint16_t   *m;           /* fp16 bits */
    uint16_t   *v;           /* fp16 bits */
    const float *grad;
    uint16_t   *live;        /* bf16 bits, may be NULL */
} sf_matrix;

typedef struct sf_adam {
    float lr, beta1, beta2, eps;
    float one_minus_b1, one_minus_b2;   /* fp32 (1 - beta), passed so every side agrees */
    float wd;                           /* decoupled weight decay, 0 = off */
    float clip;                         /* element clip, <= 0 = off */
    const float *bc1, *bc2;             /* device tables [t_max + 1] */
    int32_t t_max;
} sf_adam;

/* Fill bc[t] = (float)(1 / (1 - beta^t)) for t = 1..t_max (beta^t as t successive fp64
 * products of the fp32 beta), bc[0] = 1, for both betas. Device arrays of t_max + 1 floats. */
int sf_adam_tables(float beta1, float beta2, int t_max, float *bc1, float *bc2,
                   sf_stream stream);

int sf_sparse_update(const sf_matrix *mats /* host [n_mats] */, int n_mats,
                     const sf_adam *hp /* host */, uint32_t *dev_status, sf_stream stream);

/* ---- sf_checkpoint_save / sf_checkpoint_restore: section 2.6 --------------------------------
 * Only rows in the active set are saved, so a snapshot is as small as that set, and it is put
 * back when the loss rebounds (the policy that decides when is host logic). A checkpoint of one matrix is a snapshot, at save time, of each active row (ascending):
 *   rows[k] the row, q[k*C..] int8, s[k], delta[k*C..] fp32, m, v[k*C..] fp16 bits (zeros for a
 *   row without a slot), step[k] its Adam step count; *count the rows saved (device).
 * Buffers hold `cap` rows; a save with more active rows keeps the first cap and sets
 * SF_STATUS_SLOT_OVERFLOW. Restore writes q, s and delta of every saved row back and rebuilds its
 * live row (bf16 of fma(s, q, delta)); moments and step count go back only to rows that hold a
 * slot now (moments exist only for active rows). Rows not in the checkpoint are untouched.
 * Restore reads at most cap rows (a larger *count is clamped); a saved row id outside [0, R) is
 * skipped and sets SF_STATUS_BAD_TOKEN. `mats` and `ck` are host arrays of n entries (same order). Requirements: C a multiple of 16,
 * all row buffers 16-byte aligned. Errors: SF_ERR_ARG, SF_ERR_ALIGN.
 */
typedef struct sf_checkpoint {
    int32_t   cap;
    int32_t  *count;
    int32_t  *rows;
    int8_t   *q;
    float    *s;
    float    *delta;
    uint16_t *m;
    uint16_t *v;
    int32_t  *step;
} sf_checkpoint;

int sf_checkpoint_save(const sf_matrix *mats /* host [n] */, const sf_checkpoint *ck /* host [n] */,
                       int n, uint32_t *dev_status, sf_stream stream);
int sf_checkpoint_restore(const sf_matrix *mats /* host [n] */, const sf_checkpoint *ck /* host [n] */,
                          int n, uint32_t *dev_status, sf_stream stream);

/* ---- sf_forward_tracked: section 2.1, the forward pass that the row tracker observes ---------
 * A projection's activity for the charge rule is the magnitude of the outputs its forward pass
 * produced. This call computes that forward pass and keeps the statistic on the way:
 *     Y[t, r] = bf16_rn( sum_c A[t, c] * W[r, c] )     (fp32 accumulation, tensor cores)
 * for every problem, stores Y, and folds max over its tokens of |Y[t, r]| (of the stored bf16
 * values, with sf_mask_update's reading for non-finite outputs) into mask.accum[r] -- the same
 * numbers sf_mask_update's SF_SRC_OUTPUT_BF16 pass would find by reading Y again. The window is
 * then closed by sf_mask_update_phase(..., SF_PHASE_SECOND, ...) with an SF_SRC_OUTPUT_BF16
 * source naming the same Y. Several calls may fold into one window before it is closed.
 *   A  bf16 [T x ld_a]  the projection's inputs, token-major
 *   W  bf16 [R x ld_w]  its weights (the bf16 live copy sf_sparse_update writes), row-major
 *   Y  bf16 [T x ld_y]  its outputs (written)
 * Requirements: R = mask.R a multiple of 32; C a multiple of 8; when T > 0, ld_a and ld_w
 * multiples of 8 and >= C, ld_y a multiple of 8 and >= R, A, W, Y 16-byte aligned.
 * Errors: SF_ERR_ARG, SF_ERR_ALIGN, SF_ERR_CUDA.
 */
typedef struct sf_fwd_problem {
    const void *A;
    int64_t     ld_a;
    const void *W;
    int64_t     ld_w;
    void       *Y;
    int64_t     ld_y;
    int32_t     T;
    int32_t     C;
    sf_mask     mask;   /* R = mask.R; folds into mask.accum */
} sf_fwd_problem;

int sf_forward_tracked(const sf_fwd_problem *probs /* host [n] */, int n, uint32_t *dev_status,
                       sf_stream stream);

/* ---- sf_mask_update_phase / sf_masked_dw_phase: one pass of a two-pass call ------------------
 * No counterpart in the paper: a measurement aid. sf_mask_update and sf_masked_dw each run two
 * passes; these variants enqueue only the pass `phase` names, so that a caller can record CUDA
 * events between the passes and time each kernel on its own. SF_PHASE_FIRST then SF_PHASE_SECOND
 * on one stream, with the same arguments and nothing in between that touches their buffers,
 * does exactly what the full call (SF_PHASE_ALL) does.
 *   sf_mask_update: FIRST = the activity pass (token histogram / column absmax into accum);
 *                   SECOND = the finalize pass (charges, mask words, lists, slots).
 *   sf_masked_dw:   FIRST = the row gather of the groups that run in row mode (nothing when
 *                   ws is NULL); SECOND = the main tensor-core launches.
 * Errors: those of the full call, and SF_ERR_ARG for an unknown phase.
 */
#define SF_PHASE_ALL    0
#define SF_PHASE_FIRST  1
#define SF_PHASE_SECOND 2

int sf_mask_update_phase(const sf_mask *masks /* host [n_masks] */,
                         const sf_mask_src *srcs /* host [n_masks] */, int n_masks, float threshold,
                         int phase, uint32_t *dev_status, sf_stream stream);
int sf_masked_dw_phase(const sf_dw_problem *probs /* host [n] */, int n, void *ws, size_t ws_bytes,
                       int phase, uint32_t *dev_status, sf_stream stream);

/* ---- helpers (not on the hot path) ------------------------------------------------------ */

/* Quantise a full-precision matrix into the int8 + scale + residual storage of section 2.3
 * (same per-row rule as the update: s = max|W| / 127, q = round-half-even(W / s),
 * delta = fma(-s, q, W)); live (may be NULL) gets bf16(W). W [R x C] fp32 row-major. */
int sf_quantize_init(const float *W, int R, int C, int8_t *q, float *s, float *delta,
                     uint16_t *live, sf_stream stream);

/* Text for a return code. */
const char *sf_status_string(int code);

/* Library version: major * 10000 + minor * 100 + patch. */
int sf_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SF_H */
