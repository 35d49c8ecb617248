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
// Two launches per call, each covering every mask of the call:
//   mask_accum_kernel     the window's activity into accum[] -- token histogram (integer
//                         atomics), or the column absmax of Y (16-byte loads, packed u16 max,
//                         one atomicMax per column and CTA). HBM-bound streaming pass.
//   mask_finalize_kernel  one CTA per mask: busiest row, charge update, ballot into mask words,
//                         slot release / allocation in ascending row order, ordered lists.
// Both reductions are order-free (integer adds, max), so masks and lists are bit-exact.
#include "sf_common.cuh"
#include "sf_host.h"

namespace sf {
namespace {

constexpr int kAccumThreads = 256;
constexpr int kColsPerThread = 8;                            // one 16-byte load of bf16
constexpr int kColsPerCta = kAccumThreads * kColsPerThread;  // 2048
constexpr int kTokensPerSeg = 512;
constexpr int kTokensPerTokCta = kAccumThreads * 8;          // histogram: 8 ids per thread
constexpr int kFinalizeThreads = 1024;
constexpr int kMaxRows = 262144;                             // words of two masks fit in smem

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
    int32_t col_blocks;   // OUTPUT: 2048-column blocks
    int32_t tok_segs;     // OUTPUT: token segments
};

constexpr int kMaxMasksPerLaunch = 240;

struct MaskBatch {
    int32_t n;
    int32_t total_ctas;
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
    const uint32_t mm[4] = {m0, m1, m2, m3};
    bool nonfinite = false;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t half = (mm[j] >> (16 * h)) & 0xFFFFu;
            nonfinite |= half >= 0x7F80u;
            // widen bf16 magnitude to fp32 bits; non-negative floats order as unsigned ints
            if (half) atomicMax(&d.accum[c0 + 2 * j + h], half << 16);
        }
    }
    if (nonfinite) set_status(status, SF_STATUS_NONFINITE);
}

__global__ void __launch_bounds__(kFinalizeThreads)
mask_finalize_kernel(const __grid_constant__ MaskBatch b, float thr, uint32_t *status)
{
    extern __shared__ uint32_t smem_words[];
    __shared__ int scan_scratch[33];
    __shared__ uint32_t max_scratch[33];
    __shared__ int s_free_top, s_rows, s_tiles, s_fresh;

    const MaskDesc &d = b.d[blockIdx.x];
    const int R = d.R, nw = R >> 5;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwarps = blockDim.x >> 5;
    uint32_t *new_w = smem_words;
    uint32_t *old_w = smem_words + nw;

    // (1) busiest row of the window
    uint32_t hmax = 0;
    if (d.kind == SF_SRC_TOKENS || d.kind == SF_SRC_OUTPUT_BF16) {
        for (int r = tid; r < R; r += blockDim.x) hmax = max(hmax, d.accum[r]);
    } else if (d.kind == SF_SRC_HITS_U32) {
        const uint32_t *hits = static_cast<const uint32_t *>(d.src);
        for (int r = tid; r < R; r += blockDim.x) hmax = max(hmax, hits[r]);
    }
    hmax = block_max_u32(hmax, max_scratch);

    // (2) charge rule and new mask words: one warp per 32-row tile
    for (int w = warp; w < nw; w += nwarps) {
        const int r = (w << 5) + lane;
        bool act;
        if (d.kind == SF_SRC_WORDS) {
            act = (static_cast<const uint32_t *>(d.src)[w] >> lane) & 1u;
        } else {
            float h, H;
            if (d.kind == SF_SRC_TOKENS) {
                h = __uint2float_rn(d.accum[r]);
                H = __uint2float_rn(hmax);
                d.accum[r] = 0u;                       // ready for the next window
            } else if (d.kind == SF_SRC_OUTPUT_BF16) {
                h = __uint_as_float(d.accum[r]);
                H = __uint_as_float(hmax);
                d.accum[r] = 0u;
            } else {
                h = __uint2float_rn(static_cast<const uint32_t *>(d.src)[r]);
                H = __uint2float_rn(hmax);
            }
            const float share = (H == 0.0f) ? 0.0f : __fdiv_rn(h, H);
            const float q = __fadd_rn(__fmul_rn(0.5f, d.charge[r]), __fmul_rn(0.5f, share));
            d.charge[r] = q;
            act = q >= thr;
        }
        const uint32_t word = __ballot_sync(0xffffffffu, act);
        if (lane == 0) {
            new_w[w] = word;
            old_w[w] = d.words[w];
        }
    }
    if (tid == 0) {
        s_free_top = d.counts[2];
        s_rows = 0;
        s_tiles = 0;
        s_fresh = 0;
    }
    __syncthreads();

    // (3) rows that turned inactive return their slots, ascending row order
    for (int base = 0; base < nw; base += blockDim.x) {
        const int w = base + tid;
        const uint32_t gone = (w < nw) ? (old_w[w] & ~new_w[w]) : 0u;
        int mine = 0;
        for (uint32_t bits = gone; bits; bits &= bits - 1)
            mine += d.row_slot[(w << 5) + __ffs(bits) - 1] >= 0;
        int total;
        const int off = block_exclusive_scan(mine, scan_scratch, &total);
        const int top = s_free_top;
        int j = 0;
        for (uint32_t bits = gone; bits; bits &= bits - 1) {
            const int r = (w << 5) + __ffs(bits) - 1;
            const int s = d.row_slot[r];
            if (s >= 0) {
                d.free_slots[top + off + j] = s;
                ++j;
                d.row_slot[r] = -1;
            }
        }
        __syncthreads();
        if (tid == 0) s_free_top = top + total;
        __syncthreads();
    }

    // (4) active rows without a slot take one from the top of the stack, ascending row order
    int over = 0;
    for (int base = 0; base < nw; base += blockDim.x) {
        const int w = base + tid;
        const uint32_t act = (w < nw) ? new_w[w] : 0u;
        int mine = 0;
        for (uint32_t bits = act; bits; bits &= bits - 1)
            mine += d.row_slot[(w << 5) + __ffs(bits) - 1] < 0;
        int total;
        const int off = block_exclusive_scan(mine, scan_scratch, &total);
        const int top = s_free_top;
        int j = 0;
        for (uint32_t bits = act; bits; bits &= bits - 1) {
            const int r = (w << 5) + __ffs(bits) - 1;
            if (d.row_slot[r] >= 0) continue;
            const int idx = off + j;
            ++j;
            if (idx < top) {
                const int s = d.free_slots[top - 1 - idx];
                d.row_slot[r] = s;
                d.slot_step[s] = 0;                    // fresh moments
            } else {
                ++over;
            }
        }
        __syncthreads();
        if (tid == 0) {
            s_fresh += min(total, top);
            s_free_top = max(top - total, 0);
        }
        __syncthreads();
    }

    // (5) ascending active-row and active-tile lists, new mask words
    for (int base = 0; base < nw; base += blockDim.x) {
        const int w = base + tid;
        const uint32_t word = (w < nw) ? new_w[w] : 0u;
        int nrows, ntiles;
        const int roff = block_exclusive_scan(__popc(word), scan_scratch, &nrows);
        const int toff = block_exclusive_scan(word != 0u, scan_scratch, &ntiles);
        const int rb = s_rows + roff;
        int j = 0;
        for (uint32_t bits = word; bits; bits &= bits - 1)
            d.active_rows[rb + j++] = (w << 5) + __ffs(bits) - 1;
        if (word) {
            d.active_tiles[s_tiles + toff] = w;
            d.tile_rows[s_tiles + toff] = rb;
        }
        if (w < nw) d.words[w] = word;
        __syncthreads();
        if (tid == 0) {
            s_rows += nrows;
            s_tiles += ntiles;
        }
        __syncthreads();
    }
    int total_over;
    block_exclusive_scan(over, scan_scratch, &total_over);
    if (tid == 0) {
        d.counts[0] = s_rows;
        d.counts[1] = s_tiles;
        d.counts[2] = s_free_top;
        d.counts[3] = total_over;
        d.counts[4] = s_fresh;
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

extern "C" int sf_mask_update(const sf_mask *masks, const sf_mask_src *srcs, int n_masks,
                              float threshold, uint32_t *dev_status, sf_stream stream)
{
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
            if ((s.ld & 7) || !aligned16(s.ptr)) return SF_ERR_ALIGN;
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
    const size_t fin_smem = (size_t)2 * (max_rows / 32) * sizeof(uint32_t);
    if (fin_smem > 48 * 1024 &&
        cudaFuncSetAttribute(mask_finalize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)fin_smem) != cudaSuccess)
        return SF_ERR_CUDA;

    for (int first = 0; first < n_masks; first += kMaxMasksPerLaunch) {
        const int cnt = n_masks - first < kMaxMasksPerLaunch ? n_masks - first : kMaxMasksPerLaunch;
        MaskBatch batch;
        batch.n = cnt;
        int ctas = 0;
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
            d.col_blocks = (m.R + kColsPerCta - 1) / kColsPerCta;
            d.tok_segs = (s.n + kTokensPerSeg - 1) / kTokensPerSeg;
            if (s.kind == SF_SRC_TOKENS)
                ctas += (s.n + kTokensPerTokCta - 1) / kTokensPerTokCta;
            else if (s.kind == SF_SRC_OUTPUT_BF16)
                ctas += d.col_blocks * d.tok_segs;
        }
        batch.total_ctas = ctas;
        if (ctas > 0) {
            mask_accum_kernel<<<ctas, kAccumThreads, 0, st>>>(batch, dev_status);
            if (launch_status() != SF_OK) return SF_ERR_CUDA;
        }
        mask_finalize_kernel<<<cnt, kFinalizeThreads, fin_smem, st>>>(batch, threshold, dev_status);
        if (launch_status() != SF_OK) return SF_ERR_CUDA;
    }
    return SF_OK;
}
