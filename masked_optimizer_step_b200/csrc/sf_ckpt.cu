// sf_ckpt.cu -- checkpoint and rewind of the active rows.
//
// "Sparse-First Fine-Tuning" (tensorwirelabs.com), section 2.6: only rows in the active set are
// saved, so a snapshot is as small as that set;
// when the loss rebounds past a threshold the checkpoint is restored. A checkpoint here is a
// snapshot, at save time, of every active row's q, s, delta, moments and Adam step count, in
// ascending row order. Restoring writes q, s and delta back, rebuilds the row's bf16 live
// weights from them, and gives the moments back only to rows that hold a slot now (moments
// exist only for active rows, section 2.3).
//
// Both directions are one persistent launch over all matrices of the call; a 256-thread CTA
// copies one row at a time with 16-byte vector accesses. Bandwidth-bound: per row 9*C + 12 bytes
// each way (q 1, delta 4, m 2, v 2 per column; s and the step count per row).
#include "sf_common.cuh"
#include "sf_host.h"

namespace sf {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxMats = 160;

struct CkDesc {
    int32_t R, C, cap;
    const int32_t *active_rows;
    const int32_t *counts;
    const int32_t *row_slot;
    int32_t *slot_step;
    int8_t *q;
    float *s;
    float *delta;
    uint16_t *m;
    uint16_t *v;
    uint16_t *live;
    int32_t *c_count;
    int32_t *c_rows;
    int8_t *c_q;
    float *c_s;
    float *c_delta;
    uint16_t *c_m;
    uint16_t *c_v;
    int32_t *c_step;
};

struct CkBatch {
    int32_t n;
    int32_t restore;
    CkDesc d[kMaxMats];
};
static_assert(sizeof(CkBatch) <= 32764, "kernel parameter space");

// Copy nbytes (a multiple of 16; rows are 16-byte aligned since C % 16 == 0) as 16-byte vectors,
// four loads in flight per thread before their stores.
__device__ __forceinline__ void copy_row(void *dst, const void *src, int nbytes)
{
    uint4 *d = static_cast<uint4 *>(dst);
    const uint4 *s = static_cast<const uint4 *>(src);
    const int n = nbytes >> 4;
    int i = threadIdx.x;
    for (; i + 3 * kThreads < n; i += 4 * kThreads) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = s[i + u * kThreads];
#pragma unroll
        for (int u = 0; u < 4; ++u) d[i + u * kThreads] = v[u];
    }
    for (; i < n; i += kThreads) d[i] = s[i];
}

__global__ void __launch_bounds__(kThreads)
ckpt_kernel(const __grid_constant__ CkBatch b, uint32_t *status)
{
    __shared__ int s_prefix[kMaxMats + 1];
    __shared__ int scan_scratch[33];
    const int tid = threadIdx.x;
    {
        int c = 0;
        if (tid < b.n) {
            const CkDesc &d = b.d[tid];
            if (b.restore) {
                c = max(0, min(*d.c_count, d.cap));   // a count the buffers cannot hold is clamped
            } else {
                c = min(d.counts[0], d.cap);
                if (blockIdx.x == 0) {
                    *d.c_count = c;
                    if (d.counts[0] > d.cap) set_status(status, SF_STATUS_SLOT_OVERFLOW);
                }
            }
        }
        int total;
        const int off = block_exclusive_scan(c, scan_scratch, &total);
        if (tid < b.n) s_prefix[tid] = off;
        if (tid == 0) s_prefix[b.n] = total;
        __syncthreads();
    }
    const int total = s_prefix[b.n];
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        int lo = 0, hi = b.n - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_prefix[mid] <= item) lo = mid; else hi = mid - 1;
        }
        const CkDesc &d = b.d[lo];
        const int k = item - s_prefix[lo];
        const int C = d.C;
        const size_t kc = (size_t)k * C;
        if (!b.restore) {
            const int r = d.active_rows[k];
            const int slot = d.row_slot[r];
            const size_t rc = (size_t)r * C;
            copy_row(d.c_q + kc, d.q + rc, C);
            copy_row(d.c_delta + kc, d.delta + rc, 4 * C);
            if (slot >= 0) {
                copy_row(d.c_m + kc, d.m + (size_t)slot * C, 2 * C);
                copy_row(d.c_v + kc, d.v + (size_t)slot * C, 2 * C);
            } else {
                uint4 *zm = reinterpret_cast<uint4 *>(d.c_m + kc), *zv = reinterpret_cast<uint4 *>(d.c_v + kc);
                for (int i = tid; i < (2 * C) >> 4; i += kThreads) zm[i] = zv[i] = make_uint4(0, 0, 0, 0);
            }
            if (tid == 0) {
                d.c_rows[k] = r;
                d.c_s[k] = d.s[r];
                d.c_step[k] = slot >= 0 ? d.slot_step[slot] : 0;
            }
        } else {
            const int r = d.c_rows[k];
            if (r < 0 || r >= d.R) {                 // not a row of this matrix: skip it, say so
                if (tid == 0) set_status(status, SF_STATUS_BAD_TOKEN);
                continue;
            }
            const int slot = d.row_slot[r];
            const size_t rc = (size_t)r * C;
            const float sc = d.c_s[k];
            copy_row(d.q + rc, d.c_q + kc, C);
            copy_row(d.delta + rc, d.c_delta + kc, 4 * C);
            if (d.live) {
                for (int c0 = tid * 8; c0 < C; c0 += kThreads * 8) {
                    const uint2 qv = *reinterpret_cast<const uint2 *>(d.c_q + kc + c0);
                    const float4 d0 = *reinterpret_cast<const float4 *>(d.c_delta + kc + c0);
                    const float4 d1 = *reinterpret_cast<const float4 *>(d.c_delta + kc + c0 + 4);
                    const float dl[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
                    uint32_t lw[4];
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        float w[2];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int e = 2 * e2 + h;
                            const int8_t qe = static_cast<int8_t>(((e < 4 ? qv.x : qv.y) >> (8 * (e & 3))) & 0xFF);
                            w[h] = __fmaf_rn(sc, (float)qe, dl[e]);
                        }
                        const __nv_bfloat162 l = __floats2bfloat162_rn(w[0], w[1]);
                        lw[e2] = *reinterpret_cast<const uint32_t *>(&l);
                    }
                    *reinterpret_cast<uint4 *>(d.live + rc + c0) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                }
            }
            if (slot >= 0) {
                copy_row(d.m + (size_t)slot * C, d.c_m + kc, 2 * C);
                copy_row(d.v + (size_t)slot * C, d.c_v + kc, 2 * C);
            }
            if (tid == 0) {
                d.s[r] = sc;
                if (slot >= 0) d.slot_step[slot] = d.c_step[k];
            }
        }
        __syncthreads();
    }
}

int run(const sf_matrix *mats, const sf_checkpoint *ck, int n, int restore, uint32_t *status,
        sf_stream stream)
{
    if (n < 0 || (n > 0 && (!mats || !ck))) return SF_ERR_ARG;
    for (int i = 0; i < n; ++i) {
        const sf_matrix &a = mats[i];
        const sf_checkpoint &c = ck[i];
        int rc = check_mask(a.mask);
        if (rc != SF_OK) return rc;
        if (a.C <= 0 || (a.C & 15)) return SF_ERR_ARG;
        if (!a.q || !a.s || !a.delta || !a.m || !a.v) return SF_ERR_ARG;
        if (c.cap < 0 || !c.count || (c.cap > 0 && (!c.rows || !c.q || !c.s || !c.delta || !c.m || !c.v || !c.step)))
            return SF_ERR_ARG;
        const void *ptrs[] = {a.q, a.delta, a.m, a.v, c.q, c.delta, c.m, c.v};
        for (const void *p : ptrs)
            if (p && !aligned16(p)) return SF_ERR_ALIGN;
        if (a.live && !aligned16(a.live)) return SF_ERR_ALIGN;
    }
    if (n == 0) return SF_OK;
    const int sms = sm_count();
    if (sms <= 0) return SF_ERR_NO_DEVICE;
    cudaStream_t st = as_stream(stream);
    for (int first = 0; first < n; first += kMaxMats) {
        const int cnt = n - first < kMaxMats ? n - first : kMaxMats;
        CkBatch b;
        b.n = cnt;
        b.restore = restore;
        for (int j = 0; j < cnt; ++j) {
            const sf_matrix &a = mats[first + j];
            const sf_checkpoint &c = ck[first + j];
            CkDesc &d = b.d[j];
            d.R = a.mask.R;
            d.C = a.C;
            d.cap = c.cap;
            d.active_rows = a.mask.active_rows;
            d.counts = a.mask.counts;
            d.row_slot = a.mask.row_slot;
            d.slot_step = a.mask.slot_step;
            d.q = a.q;
            d.s = a.s;
            d.delta = a.delta;
            d.m = a.m;
            d.v = a.v;
            d.live = a.live;
            d.c_count = c.count;
            d.c_rows = c.rows;
            d.c_q = c.q;
            d.c_s = c.s;
            d.c_delta = c.delta;
            d.c_m = c.m;
            d.c_v = c.v;
            d.c_step = c.step;
        }
        ckpt_kernel<<<sms * 8, kThreads, 0, st>>>(b, status);
        if (launch_status() != SF_OK) return SF_ERR_CUDA;
    }
    return SF_OK;
}

}  // namespace
}  // namespace sf

extern "C" int sf_checkpoint_save(const sf_matrix *mats, const sf_checkpoint *ck, int n,
                                  uint32_t *dev_status, sf_stream stream)
{
    return sf::run(mats, ck, n, 0, dev_status, stream);
}

extern "C" int sf_checkpoint_restore(const sf_matrix *mats, const sf_checkpoint *ck, int n,
                                     uint32_t *dev_status, sf_stream stream)
{
    return sf::run(mats, ck, n, 1, dev_status, stream);
}
