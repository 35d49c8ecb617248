// sf_mask.cu -- row masks of the sparse step: conductor and row tracker.
//
// "Sparse-First Fine-Tuning" (tensorwirelabs.com), section 2.1 (Observing activity): each row
// of each weight matrix carries a charge q. When a window closes, q is replaced by
// q/2 + share/2, where share is the row's activity in that window relative to the most active
// row; the row counts as active while q >= 0.01. For the embedding (the conductor) activity is
// the token's hit count, for a projection (the row tracker) the size of its forward outputs.
// One mask per step serves all later stages. Section 2.3 keeps optimizer moments for active
// rows only; the slot lifecycle below is that rule.
//
// Four launches per call, each covering every mask of the call; the last three are chained by
// programmatic dependent launch:
//   mask_accum_kernel     the window's activity into accum[] -- token histogram (integer
//                         atomics), or the column absmax of Y (16-byte loads, packed u16 max,
//                         per CTA one bf16 max-reduction per column, eight columns per
//                         instruction). HBM-bound streaming pass.
//   mask_hmax_kernel      the busiest row of each mask: 2,048-row blocks, one atomicMax each.
//   mask_charge_kernel    the charge update and the new mask words, 2,048-row blocks, and per
//                         32-row tile the rows that release a slot or need one.
//   mask_finalize_kernel  one CTA per mask: slot release / allocation in ascending row order,
//                         ordered lists.
// The reductions are order-free (integer adds, max), so masks and lists are bit-exact. A large
// mask's per-row work is spread over many SMs by the middle two launches: one CTA reading and
// writing a 32,000-row mask's state is bound by one SM's memory throughput (~20 us).
#include "sf_common.cuh"
#include "sf_host.h"

namespace sf {
namespace {

constexpr int kAccumThreads = 256;
constexpr int kColsPerThread = 8;                            // one 16-byte load of bf16
constexpr int kColsPerCta = kAccumThreads * kColsPerThread;  // 2048
constexpr int kTokensPerSeg = 512;
constexpr int kMinTokensPerSeg = 32;
#ifndef SF_MASK_PREFETCH_ROWS
#define SF_MASK_PREFETCH_ROWS 8
#endif
constexpr int kPrefetchRows = SF_MASK_PREFETCH_ROWS;   // prefetch distance of the column-max pass
constexpr int kTokensPerTokCta = kAccumThreads * 8;          // histogram: 8 ids per thread
constexpr int kFinalizeThreads = 1024;
constexpr int kMaxRows = 262144;                             // three bit masks per tile fit in smem

struct MaskDesc {
    int32_t R, slot_cap, kind, n;
    int64_t ld;
    const void *src;
    float *charge;
    uint32_t *accum;
    uint32_t *words;
    int32_t *active_rows;
    int32_t *active_tiles;
    int32_t *tile_rows;
    int32_t *row_slot;
    int32_t *free_slots;
    int32_t *slot_step;
    int32_t *counts;
    int32_t cta_begin;    // first CTA of this mask in the accumulate launch
    int32_t blk_begin;    // first 2,048-row block of this mask in the hmax and charge launches
    int32_t col_blocks;   // OUTPUT: 2048-column blocks
    int32_t tok_segs;     // OUTPUT: token segments
};

constexpr int kMaxMasksPerLaunch = 240;

struct MaskBatch {
    int32_t n;
    int32_t total_ctas;
    int32_t total_blks;
    MaskDesc d[kMaxMasksPerLaunch];
};
static_assert(sizeof(MaskBatch) <= 32764, "kernel parameter space");

__device__ __forceinline__ int find_mask(const MaskBatch &b, int cta)
{
    int lo = 0, hi = b.n - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (b.d[mid].cta_begin <= cta) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ int find_mask_blk(const MaskBatch &b, int blk)
{
    int lo = 0, hi = b.n - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (b.d[mid].blk_begin <= blk) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// An output source keeps the window's row magnitudes as bf16, two bytes per row at the start of
// accum (16-byte aligned): the column-max pass reduces eight rows per instruction into it.
// Counts (tokens) stay one uint32 per row. Either is read back as the uint32 the charge rule
// takes: a count, or the magnitude widened to fp32 bits.
__device__ __forceinline__ uint16_t *accum_bf16(const MaskDesc &d) { return reinterpret_cast<uint16_t *>(d.accum); }

__device__ __forceinline__ uint32_t activity(const MaskDesc &d, int r)
{
    if (d.kind == SF_SRC_OUTPUT_BF16) return (uint32_t)accum_bf16(d)[r] << 16;
    return d.kind == SF_SRC_HITS_U32 ? static_cast<const uint32_t *>(d.src)[r] : d.accum[r];
}

__global__ void __launch_bounds__(kAccumThreads)
mask_accum_kernel(const __grid_constant__ MaskBatch b, uint32_t *status)
{
    const int i = find_mask(b, blockIdx.x);
    const MaskDesc &d = b.d[i];
    const int local = blockIdx.x - d.cta_begin;

    if (d.kind == SF_SRC_TOKENS) {
        const int32_t *tok = static_cast<const int32_t *>(d.src);
        const int base = local * kTokensPerTokCta;
        bool bad = false;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int t = base + j * kAccumThreads + threadIdx.x;
            if (t < d.n) {
                const int r = tok[t];
                if (r >= 0 && r < d.R) atomicAdd(&d.accum[r], 1u);
                else bad = true;
            }
        }
        if (bad) set_status(status, SF_STATUS_BAD_TOKEN);
        return;
    }

    // SF_SRC_OUTPUT_BF16: column absmax of Y[T x ld] over one token segment.
    const int cb = local % d.col_blocks;
    const int seg = local / d.col_blocks;
    const int c0 = cb * kColsPerCta + threadIdx.x * kColsPerThread;
    if (c0 >= d.R) return;
    const int seg_len = (d.n + d.tok_segs - 1) / d.tok_segs;
    const int t0 = seg * seg_len;
    const int t1 = min(d.n, t0 + seg_len);
    const uint16_t *Y = static_cast<const uint16_t *>(d.src);
    // |bf16| as an unsigned 16-bit pattern orders like the magnitude; keep two per word.
    uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
    int t = t0;
    for (; t + 8 <= t1; t += 8) {
        // token rows kPrefetchRows ahead of this batch, into L2 (one lane per 128-byte line): the
        // loads in flight per SM are register-limited, the prefetches are not
        if ((threadIdx.x & 7) == 0 && t + kPrefetchRows + 8 <= t1) {
#pragma unroll
            for (int j = 0; j < 8; ++j) prefetch_l2(Y + (size_t)(t + kPrefetchRows + j) * d.ld + c0);
        }
        uint4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            v[j] = __ldcs(reinterpret_cast<const uint4 *>(Y + (size_t)(t + j) * d.ld + c0));
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            m0 = __vmaxu2(m0, v[j].x & 0x7FFF7FFFu);
            m1 = __vmaxu2(m1, v[j].y & 0x7FFF7FFFu);
            m2 = __vmaxu2(m2, v[j].z & 0x7FFF7FFFu);
            m3 = __vmaxu2(m3, v[j].w & 0x7FFF7FFFu);
        }
    }
    for (; t < t1; ++t) {
        uint4 v = __ldcs(reinterpret_cast<const uint4 *>(Y + (size_t)t * d.ld + c0));
        m0 = __vmaxu2(m0, v.x & 0x7FFF7FFFu);
        m1 = __vmaxu2(m1, v.y & 0x7FFF7FFFu);
        m2 = __vmaxu2(m2, v.z & 0x7FFF7FFFu);
        m3 = __vmaxu2(m3, v.w & 0x7FFF7FFFu);
    }
    uint32_t mm[4] = {m0, m1, m2, m3};
    // |bf16| patterns above 0x7F80 are NaN, 0x7F80 is infinity. Reading for non-finite outputs:
    // a NaN carries no magnitude, an infinity counts as the largest finite bf16 magnitude
    // (0x7F7F). The packed max is at least 0x7F80 exactly when the segment held one, so only
    // then is the segment read again with each value mapped first (rare; nothing changes for
    // finite outputs).
    bool nonfinite = false;
#pragma unroll
    for (int j = 0; j < 4; ++j)
        nonfinite |= (mm[j] & 0xFFFFu) >= 0x7F80u || (mm[j] >> 16) >= 0x7F80u;
    if (nonfinite) {
#pragma unroll
        for (int j = 0; j < 4; ++j) mm[j] = 0u;
        for (int tt = t0; tt < t1; ++tt) {
            const uint4 v = __ldcs(reinterpret_cast<const uint4 *>(Y + (size_t)tt * d.ld + c0));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t a = w[j] & 0x7FFF7FFFu;
                a &= ~__vcmpgtu2(a, 0x7F807F80u);          // NaN -> 0
                a = __vminu2(a, 0x7F7F7F7Fu);              // infinity -> largest finite
                mm[j] = __vmaxu2(mm[j], a);
            }
        }
        set_status(status, SF_STATUS_NONFINITE);
    }
    // the segment's maxima of the thread's eight columns into the mask's bf16 accumulator, one
    // reduction for all eight (the packed pairs are in memory order)
    if (mm[0] | mm[1] | mm[2] | mm[3]) red_max_bf16x8(accum_bf16(d) + c0, mm[0], mm[1], mm[2], mm[3]);
}

// The busiest row, the charge rule and the new words run over 2,048-row blocks (256 threads: a
// warp per 32-row tile, lane = row, the loads of kBatch tiles issued before any is used); the
// finalize then runs one CTA per mask over the bit masks they leave: new words in words[],
// the rows that release a slot in active_tiles[] and those that need one in tile_rows[] (one
// uint32 per tile; both arrays are rewritten with the lists afterwards). The slot sweeps and the
// lists go over rounds of kRound words: a block scan of the per-word counts gives every tile its
// offsets, and a warp per tile writes its rows' entries, touching global memory only for rows
// that change state. The busiest row's value meets in counts[5] (reset by the finalize).
constexpr int kBlkThreads = 256;
constexpr int kBlkRows = 2048;
constexpr int kSplitRows = SF_MASK_SPLIT_ROWS;   // masks from this many rows on take the split finalize
constexpr int kBlkWords = kBlkRows / 32;
constexpr int kBatch = 4;
constexpr int kRound = 512;       // words per scan round; per-round sums stay below 2^15 per field

__global__ void __launch_bounds__(kBlkThreads)
mask_hmax_kernel(const __grid_constant__ MaskBatch b)
{
    griddep_launch_dependents();
    griddep_wait();                           // the window's activity
    __shared__ uint32_t max_scratch[33];
    const int i = find_mask_blk(b, blockIdx.x);
    const MaskDesc &d = b.d[i];
    if (d.kind == SF_SRC_WORDS) return;
    const uint32_t *vals = d.kind == SF_SRC_HITS_U32 ? static_cast<const uint32_t *>(d.src) : d.accum;
    const int r0 = (blockIdx.x - d.blk_begin) * kBlkRows;
    const int r1 = min(d.R, r0 + kBlkRows);
    uint32_t hmax = 0;
    if (d.kind == SF_SRC_OUTPUT_BF16) {       // bf16 magnitudes, eight rows per 16-byte load
        uint32_t m2 = 0;
#pragma unroll
        for (int u = 0; u < kBlkRows / (8 * kBlkThreads); ++u) {
            const int r = r0 + 8 * (u * kBlkThreads + (int)threadIdx.x);
            if (r < r1) {
                const uint4 v = *reinterpret_cast<const uint4 *>(accum_bf16(d) + r);
                m2 = __vmaxu2(m2, __vmaxu2(__vmaxu2(v.x, v.y), __vmaxu2(v.z, v.w)));
            }
        }
        hmax = max(m2 & 0xFFFFu, m2 >> 16) << 16;
    } else if ((reinterpret_cast<uintptr_t>(vals) & 15) == 0) {
        // rows come in whole 32-row tiles, so each thread's four-row groups stay in the block
#pragma unroll
        for (int u = 0; u < kBlkRows / (4 * kBlkThreads); ++u) {
            const int r = r0 + 4 * (u * kBlkThreads + (int)threadIdx.x);
            if (r < r1) {
                const uint4 v = *reinterpret_cast<const uint4 *>(vals + r);
                hmax = max(hmax, max(max(v.x, v.y), max(v.z, v.w)));
            }
        }
    } else {                                  // a caller's hit counts need only 4-byte alignment
        for (int r = r0 + (int)threadIdx.x; r < r1; r += kBlkThreads) hmax = max(hmax, vals[r]);
    }
    hmax = block_max_u32(hmax, max_scratch);
    if (threadIdx.x == 0 && hmax) atomicMax(reinterpret_cast<unsigned int *>(&d.counts[5]), hmax);
}

// The charge rule and the new mask words of tiles [w_begin, w_end) of one mask, a warp per tile
// (w = w_begin + warp, + nwarps, ...); per tile the new word and the rows that release a slot or
// need one go to new_w[w], rel_w[w], need_w[w] (shared memory, or the mask's own arrays).
__device__ __forceinline__ void charge_words(const MaskDesc &d, int w_begin, int w_end, int warp, int nwarps,
                                             float H, float thr, uint32_t *new_w, uint32_t *rel_w,
                                             uint32_t *need_w)
{
    const int lane = threadIdx.x & 31;
    const int kind = d.kind;
    const uint32_t *src_u32 = static_cast<const uint32_t *>(d.src);
    for (int w0 = w_begin + warp; w0 < w_end; w0 += nwarps * kBatch) {
        uint32_t hv[kBatch], ow[kBatch];
        float qv[kBatch];
        int sl[kBatch];
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const int w = w0 + k * nwarps;
            hv[k] = 0u;
            ow[k] = 0u;
            qv[k] = 0.0f;
            sl[k] = -1;
            if (w < w_end) {
                const int r = (w << 5) + lane;
                if (kind == SF_SRC_WORDS) {
                    hv[k] = src_u32[w];
                } else {
                    hv[k] = activity(d, r);
                    qv[k] = d.charge[r];
                }
                ow[k] = d.words[w];
                sl[k] = d.row_slot[r];
            }
        }
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const int w = w0 + k * nwarps;
            if (w >= w_end) break;                               // uniform across the warp
            const int r = (w << 5) + lane;
            bool act;
            if (kind == SF_SRC_WORDS) {
                act = (hv[k] >> lane) & 1u;
            } else {
                const float h = kind == SF_SRC_OUTPUT_BF16 ? __uint_as_float(hv[k]) : __uint2float_rn(hv[k]);
                const float share = (H == 0.0f) ? 0.0f : __fdiv_rn(h, H);
                const float q = __fadd_rn(__fmul_rn(0.5f, qv[k]), __fmul_rn(0.5f, share));
                d.charge[r] = q;
                if (kind == SF_SRC_OUTPUT_BF16) accum_bf16(d)[r] = 0;    // ready for the next window
                else if (kind == SF_SRC_TOKENS) d.accum[r] = 0u;
                act = q >= thr;
            }
            const bool was = (ow[k] >> lane) & 1u;
            const uint32_t nword = __ballot_sync(0xffffffffu, act);
            const uint32_t rel = __ballot_sync(0xffffffffu, was && !act && sl[k] >= 0);
            const uint32_t need = __ballot_sync(0xffffffffu, act && sl[k] < 0);
            if (lane == 0) {
                new_w[w] = nword;
                rel_w[w] = rel;
                need_w[w] = need;
            }
        }
    }
}

__device__ __forceinline__ float busiest_value(const MaskDesc &d, uint32_t hmax)
{
    return d.kind == SF_SRC_OUTPUT_BF16 ? __uint_as_float(hmax) : __uint2float_rn(hmax);
}

__global__ void __launch_bounds__(kBlkThreads)
mask_charge_kernel(const __grid_constant__ MaskBatch b, float thr)
{
    griddep_launch_dependents();
    griddep_wait();                           // the busiest row
    const int i = find_mask_blk(b, blockIdx.x);
    const MaskDesc &d = b.d[i];
    const int w_begin = (blockIdx.x - d.blk_begin) * kBlkWords;
    const int w_end = min(d.R >> 5, w_begin + kBlkWords);
    const float H = busiest_value(d, static_cast<uint32_t>(d.counts[5]));
    charge_words(d, w_begin, w_end, threadIdx.x >> 5, kBlkThreads / 32, H, thr, d.words,
                 reinterpret_cast<uint32_t *>(d.active_tiles), reinterpret_cast<uint32_t *>(d.tile_rows));
}

// fused = 1: the CTA also finds the busiest row and runs the charge rule itself (one launch; the
// masks of the call are small enough for one SM each); fused = 0: mask_hmax_kernel and
// mask_charge_kernel ran first and left the bit masks in the mask's arrays.
__global__ void __launch_bounds__(kFinalizeThreads, 2)   // two per SM: a call's masks fit one wave
mask_finalize_kernel(const __grid_constant__ MaskBatch b, float thr, int fused, uint32_t *status)
{
    griddep_launch_dependents();
    extern __shared__ uint32_t smem_words[];
    __shared__ int scan_scratch[33];
    __shared__ uint32_t max_scratch[33];
    __shared__ int s_off[kRound];
    __shared__ int s_toff[kRound];

    const MaskDesc &d = b.d[blockIdx.x];
    const int R = d.R, nw = R >> 5;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int nwarps = kFinalizeThreads / 32;
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t *new_w = smem_words;
    uint32_t *rel_w = smem_words + nw;
    uint32_t *need_w = smem_words + 2 * nw;
    griddep_wait();                           // the window's activity, or the charge pass's bit masks
    if (fused) {
        uint32_t hmax = 0;
        if (d.kind == SF_SRC_OUTPUT_BF16) {      // eight bf16 magnitudes per 16-byte load
            const uint4 *v8 = reinterpret_cast<const uint4 *>(accum_bf16(d));
            uint32_t m2 = 0;
#pragma unroll 4
            for (int k = tid; k < (R >> 3); k += kFinalizeThreads) {
                const uint4 v = v8[k];
                m2 = __vmaxu2(m2, __vmaxu2(__vmaxu2(v.x, v.y), __vmaxu2(v.z, v.w)));
            }
            hmax = max(m2 & 0xFFFFu, m2 >> 16) << 16;
        } else if (d.kind != SF_SRC_WORDS) {
            const uint32_t *vals = d.kind == SF_SRC_HITS_U32 ? static_cast<const uint32_t *>(d.src) : d.accum;
#pragma unroll 4
            for (int r = tid; r < R; r += kFinalizeThreads) hmax = max(hmax, vals[r]);
        }
        hmax = block_max_u32(hmax, max_scratch);
        charge_words(d, 0, nw, warp, nwarps, busiest_value(d, hmax), thr, new_w, rel_w, need_w);
    } else {
        for (int w = tid; w < nw; w += kFinalizeThreads) {
            new_w[w] = d.words[w];
            rel_w[w] = static_cast<uint32_t>(d.active_tiles[w]);
            need_w[w] = static_cast<uint32_t>(d.tile_rows[w]);
        }
    }
    __syncthreads();

    // (3) rows that turned inactive push their slots onto the free stack, ascending row order
    int top = d.counts[2];
    for (int base = 0; base < nw; base += kRound) {
        const int w = base + tid;
        const int c = (tid < kRound && w < nw) ? __popc(rel_w[w]) : 0;
        int total;
        const int off = block_exclusive_scan(c, scan_scratch, &total);
        if (tid < kRound) s_off[tid] = off;
        __syncthreads();
        if (total) {
            for (int j = warp; j < kRound && base + j < nw; j += nwarps) {
                const uint32_t rel = rel_w[base + j];
                if ((rel >> lane) & 1u) {
                    const int r = ((base + j) << 5) + lane;
                    d.free_slots[top + s_off[j] + __popc(rel & lt)] = d.row_slot[r];
                    d.row_slot[r] = -1;
                }
            }
        }
        top += total;
        __syncthreads();
    }

    // (4) rows that need a slot pop one from the top (ascending row order); lists and words
    const int top2 = top;
    int need_base = 0, rows_base = 0, tiles_base = 0, over = 0;
    for (int base = 0; base < nw; base += kRound) {
        const int w = base + tid;
        const bool mine = tid < kRound && w < nw;
        const uint32_t word = mine ? new_w[w] : 0u;
        const uint32_t nd = mine ? need_w[w] : 0u;
        int tot1, tot2;
        const int off1 = block_exclusive_scan((__popc(nd) << 16) | __popc(word), scan_scratch, &tot1);
        const int off2 = block_exclusive_scan(word != 0u, scan_scratch, &tot2);
        if (tid < kRound) {
            s_off[tid] = off1;
            s_toff[tid] = off2;
        }
        __syncthreads();
        for (int j = warp; j < kRound && base + j < nw; j += nwarps) {
            const int wj = base + j;
            const uint32_t wd = new_w[wj], ndw = need_w[wj];
            const int r = (wj << 5) + lane;
            const int roff = rows_base + (s_off[j] & 0xFFFF);
            if ((ndw >> lane) & 1u) {
                const int idx = need_base + (s_off[j] >> 16) + __popc(ndw & lt);
                if (idx < top2) {
                    const int sl = d.free_slots[top2 - 1 - idx];
                    d.row_slot[r] = sl;
                    d.slot_step[sl] = 0;                           // fresh moments
                } else {
                    ++over;
                }
            }
            if ((wd >> lane) & 1u) d.active_rows[roff + __popc(wd & lt)] = r;
            if (lane == 0) {
                d.words[wj] = wd;
                if (wd) {
                    const int t = tiles_base + s_toff[j];
                    d.active_tiles[t] = wj;
                    d.tile_rows[t] = roff;
                }
            }
        }
        need_base += tot1 >> 16;
        rows_base += tot1 & 0xFFFF;
        tiles_base += tot2;
        __syncthreads();
    }
    int total_over;
    block_exclusive_scan(over, scan_scratch, &total_over);
    if (tid == 0) {
        d.counts[0] = rows_base;
        d.counts[1] = tiles_base;
        d.counts[2] = max(top2 - need_base, 0);
        d.counts[3] = total_over;
        d.counts[4] = min(need_base, top2);
        d.counts[5] = 0;                      // the busiest row's meeting point, for the next window
        if (total_over) set_status(status, SF_STATUS_SLOT_OVERFLOW);
    }
}

__global__ void mask_init_kernel(sf_mask m)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < m.R) {
        m.charge[i] = 0.0f;
        m.accum[i] = 0u;
        m.active_rows[i] = 0;
        m.row_slot[i] = -1;
        if ((i & 31) == 0) {
            m.words[i >> 5] = 0u;
            m.active_tiles[i >> 5] = 0;
            m.tile_rows[i >> 5] = 0;
        }
    }
    if (i < m.slot_cap) {
        m.free_slots[i] = m.slot_cap - 1 - i;     // the first pops hand out 0, 1, 2, ...
        m.slot_step[i] = 0;
    }
    if (i == 0) {
        m.counts[0] = 0;
        m.counts[1] = 0;
        m.counts[2] = m.slot_cap;
        for (int k = 3; k < 8; ++k) m.counts[k] = 0;
    }
}

// CTAs of the accumulate pass resident per SM (set by its registers), looked up once
int accum_ctas_per_sm()
{
    static int n = 0;
    if (n <= 0) {
        int k = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&k, mask_accum_kernel, kAccumThreads, 0) != cudaSuccess || k <= 0)
            k = 6;
        n = k;
    }
    return n;
}

}  // namespace
}  // namespace sf

using namespace sf;

extern "C" int sf_mask_init(const sf_mask *mk, sf_stream stream)
{
    if (!mk) return SF_ERR_ARG;
    const int rc = check_mask(*mk);
    if (rc != SF_OK) return rc;
    const int n = mk->R > mk->slot_cap ? mk->R : mk->slot_cap;
    mask_init_kernel<<<(n + 255) / 256, 256, 0, as_stream(stream)>>>(*mk);
    return launch_status();
}

extern "C" int sf_mask_update_phase(const sf_mask *masks, const sf_mask_src *srcs, int n_masks,
                                    float threshold, int phase, uint32_t *dev_status, sf_stream stream)
{
    if (phase != SF_PHASE_ALL && phase != SF_PHASE_FIRST && phase != SF_PHASE_SECOND) return SF_ERR_ARG;
    if (n_masks < 0 || (n_masks > 0 && (!masks || !srcs))) return SF_ERR_ARG;
    if (!(threshold >= 0.0f)) return SF_ERR_ARG;
    // validate everything before the first launch
    int max_rows = 0;
    for (int i = 0; i < n_masks; ++i) {
        const sf_mask &m = masks[i];
        const sf_mask_src &s = srcs[i];
        int rc = check_mask(m);
        if (rc != SF_OK) return rc;
        if (m.R > kMaxRows) return SF_ERR_UNSUPPORTED;
        if (m.R > max_rows) max_rows = m.R;
        switch (s.kind) {
        case SF_SRC_TOKENS:
            if (s.n < 0 || (s.n > 0 && !s.ptr)) return SF_ERR_ARG;
            break;
        case SF_SRC_OUTPUT_BF16:
            if (s.n < 0 || (s.n > 0 && !s.ptr) || s.ld < m.R) return SF_ERR_ARG;
            if ((s.ld & 7) || !aligned16(s.ptr) || !aligned16(m.accum)) return SF_ERR_ALIGN;
            break;
        case SF_SRC_HITS_U32:
        case SF_SRC_WORDS:
            if (!s.ptr) return SF_ERR_ARG;
            break;
        default:
            return SF_ERR_ARG;
        }
    }
    if (n_masks == 0) return SF_OK;
    cudaStream_t st = as_stream(stream);
    const size_t fin_smem = (size_t)3 * (max_rows / 32) * sizeof(uint32_t);
    // opt-in beyond 48 KB of shared memory in all, static included (set from 40 KB dynamic on)
    if (fin_smem > 40 * 1024 &&
        cudaFuncSetAttribute(mask_finalize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)fin_smem) != cudaSuccess)
        return SF_ERR_CUDA;

    const int sms = sm_count();
    for (int first = 0; first < n_masks; first += kMaxMasksPerLaunch) {
        const int cnt = n_masks - first < kMaxMasksPerLaunch ? n_masks - first : kMaxMasksPerLaunch;
        // Token segment length of the column-absmax pass: 512 tokens, shortened (down to 32) when
        // the launch would otherwise give each SM fewer than ~2 CTAs, so that enough loads are in
        // flight to cover HBM latency (a lone projection has only R / 2048 column blocks). Each
        // segment ends in one max-reduction per column, so shorter segments cost atomics: for one 7B
        // layer at 4,096 tokens the pass measured fastest at ~2 CTAs per SM (4: +2 us, 8: +7 us,
        // 16: +35 us).
        int seg_tokens = kTokensPerSeg;
        {
            long base = 0;
            for (int j = 0; j < cnt; ++j) {
                const sf_mask_src &s = srcs[first + j];
                if (s.kind == SF_SRC_OUTPUT_BF16)
                    base += (long)((masks[first + j].R + kColsPerCta - 1) / kColsPerCta) *
                            ((s.n + kTokensPerSeg - 1) / kTokensPerSeg);
            }
            const long target = 2L * (sms > 0 ? sms : 148);
            while (base > 0 && seg_tokens > kMinTokensPerSeg && base * (kTokensPerSeg / seg_tokens) < target)
                seg_tokens >>= 1;
            // A large call gets shorter segments still, until it spans ~8 waves of resident CTAs:
            // the launch's last wave then idles fewer SMs (the 32-layer 7B step, 2,048 tokens:
            // 512 tokens 0.856 ms, 256 0.827, 128 0.813). Never below 128 tokens nor to more than
            // 16 segments of the longest source: each segment ends in a max-reduction per column
            // (64 tokens: 0.872 ms; one 7B layer at 4,096 tokens is fastest at 256).
            const long waves8 = 8L * accum_ctas_per_sm() * (sms > 0 ? sms : 148);
            int longest = 0;
            for (int j = 0; j < cnt; ++j)
                if (srcs[first + j].kind == SF_SRC_OUTPUT_BF16) longest = max(longest, srcs[first + j].n);
            const int floor_tokens = max(128, longest / 16);
            while (base > 0 && seg_tokens > floor_tokens && base * (kTokensPerSeg / seg_tokens) < waves8)
                seg_tokens >>= 1;
        }
        MaskBatch batch;
        batch.n = cnt;
        int ctas = 0, blks = 0;
        for (int j = 0; j < cnt; ++j) {
            const sf_mask &m = masks[first + j];
            const sf_mask_src &s = srcs[first + j];
            MaskDesc &d = batch.d[j];
            d.R = m.R;
            d.slot_cap = m.slot_cap;
            d.kind = s.kind;
            d.n = s.n;
            d.ld = s.ld;
            d.src = s.ptr;
            d.charge = m.charge;
            d.accum = m.accum;
            d.words = m.words;
            d.active_rows = m.active_rows;
            d.active_tiles = m.active_tiles;
            d.tile_rows = m.tile_rows;
            d.row_slot = m.row_slot;
            d.free_slots = m.free_slots;
            d.slot_step = m.slot_step;
            d.counts = m.counts;
            d.cta_begin = ctas;
            d.blk_begin = blks;
            blks += (m.R + kBlkRows - 1) / kBlkRows;
            d.col_blocks = (m.R + kColsPerCta - 1) / kColsPerCta;
            d.tok_segs = (s.n + seg_tokens - 1) / seg_tokens;
            if (s.kind == SF_SRC_TOKENS)
                ctas += (s.n + kTokensPerTokCta - 1) / kTokensPerTokCta;
            else if (s.kind == SF_SRC_OUTPUT_BF16)
                ctas += d.col_blocks * d.tok_segs;
        }
        batch.total_ctas = ctas;
        batch.total_blks = blks;
        if (ctas > 0 && phase != SF_PHASE_SECOND) {
            mask_accum_kernel<<<ctas, kAccumThreads, 0, st>>>(batch, dev_status);
            if (launch_status() != SF_OK) return SF_ERR_CUDA;
        }
        if (phase != SF_PHASE_FIRST) {
            // one launch when every mask of the batch is small enough for one SM; otherwise the
            // busiest row and the charge rule go over 2,048-row blocks first
            int batch_max_rows = 0;
            for (int j = 0; j < cnt; ++j) batch_max_rows = max(batch_max_rows, masks[first + j].R);
            const int fused = batch_max_rows < kSplitRows;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[0].val.programmaticStreamSerializationAllowed = 1;
            cudaLaunchConfig_t cfg = {};
            cfg.stream = st;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (!fused) {
                cfg.gridDim = dim3(blks);
                cfg.blockDim = dim3(kBlkThreads);
                if (cudaLaunchKernelEx(&cfg, mask_hmax_kernel, batch) != cudaSuccess) return SF_ERR_CUDA;
                if (cudaLaunchKernelEx(&cfg, mask_charge_kernel, batch, threshold) != cudaSuccess)
                    return SF_ERR_CUDA;
            }
            cfg.gridDim = dim3(cnt);
            cfg.blockDim = dim3(kFinalizeThreads);
            cfg.dynamicSmemBytes = fin_smem;
            if (cudaLaunchKernelEx(&cfg, mask_finalize_kernel, batch, threshold, fused, dev_status) != cudaSuccess)
                return SF_ERR_CUDA;
        }
    }
    return SF_OK;
}

extern "C" int sf_mask_update(const sf_mask *masks, const sf_mask_src *srcs, int n_masks,
                              float threshold, uint32_t *dev_status, sf_stream stream)
{
    return sf_mask_update_phase(masks, srcs, n_masks, threshold, SF_PHASE_ALL, dev_status, stream);
}
