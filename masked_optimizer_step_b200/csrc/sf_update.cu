// sf_update.cu -- fused sparse update of the active rows (int8 + residual storage, coupled
// Adam step, requantisation, masked write-back of live weights).
//
// "Sparse-First Fine-Tuning" (tensorwirelabs.com):
//   section 2.3: weights live as int8 codes q, one fp32 scale s per row and an fp32 residual
//     delta; for an active row the kernel turns (q, s, delta) back into fp32 weights that never
//     leave registers, steps them, and stores fresh q, s and delta; rows outside the mask are
//     not touched at all, and the bf16 copy the forward pass reads is refreshed for the updated
//     rows only;
//   section 2.4: gate/up, query/output and key/value are coupled in pairs, each matrix's
//     gradient feeding its partner's moments; the mixed gradient then goes through ordinary
//     bias-corrected Adam, with a decoupled weight decay whose strength carries a cos(alpha).
//
// Design: one persistent launch covers every active row of every matrix of the step. A CTA of
// 256 threads owns one row at a time: it streams the row's q, delta, gradient(s) and fp16
// moments in with 8- and 16-byte vector loads (all coalesced), parks the new weight in shared
// memory, finds the new row absmax with a block reduction, then requantises and streams q,
// delta and the bf16 live row out. Four CTAs per SM keep ~100 KB of loads in flight per SM. HBM-bound: per active
// element it reads 1 + 4 + 4 + 2 + 2 bytes and writes 1 + 4 + 2 + 2 + 2 bytes.
// Every floating-point step is an explicitly rounded intrinsic, in a fixed order, so results
// are bit-reproducible and independent of the compiler's contraction choices.
#include "sf_common.cuh"
#include "sf_host.h"

namespace sf {
namespace {

#ifndef SF_UPDATE_THREADS
#define SF_UPDATE_THREADS 256
#endif
constexpr int kThreads = SF_UPDATE_THREADS;     // threads per CTA (one row at a time)
constexpr int kMaxMatsPerLaunch = 256;
constexpr int kMaxC = 32768;

struct UpdDesc {
    int32_t R, C;
    float c_self, c_partner;
    const int32_t *active_rows;
    const int32_t *counts;
    const int32_t *row_slot;
    int32_t *slot_step;
    int8_t *q;
    float *s;
    float *delta;
    uint16_t *m;
    uint16_t *v;
    const float *grad;
    uint16_t *live;
    const float *pgrad;          // partner gradient, or null
    const int32_t *prow_slot;    // partner row -> slot, or null
};

struct UpdBatch {
    int32_t n;
    float lr, beta1, beta2, eps, omb1, omb2, wd, clip;
    const float *bc1;
    const float *bc2;
    int32_t t_max;
    UpdDesc d[kMaxMatsPerLaunch];
};
static_assert(sizeof(UpdBatch) <= 32764, "kernel parameter space");

// q' = clamp(rint(W / s), -127, 127) with W / s the correctly rounded quotient. The quotient
// matters only through its rounding to an integer, so it is first formed as W * rcp(s): that
// product is within 1.6e-5 of W / s and the rounded quotient within 7.6e-6 (|W / s| <= 127.5),
// so the two differ by less than 2.3e-5 and can only round differently when the product lies
// that close to a half-integer. The exact division is taken whenever the product lies within
// 2^-14 (about 6.1e-5) of a half-integer, i.e. farther than 0.5 - 2^-14 from the nearest
// integer: a band chosen wider than the 2.3e-5 bound on purpose (about 1 element in 8,000 takes
// it). y - rint(y) is exact for these magnitudes.
__device__ __forceinline__ float quant_code(float w, float sp, float rcp, bool fast)
{
    float qf;
    const float y = __fmul_rn(w, rcp);
    const float r = rintf(y);
    if (fast && fabsf(y - r) <= 0.5f - 0x1p-14f) qf = r;
    else qf = rintf(__fdiv_rn(w, sp));
    return fminf(fmaxf(qf, -127.0f), 127.0f);
}

// Pass 1 of one 8-column chunk: rebuild, mix, Adam. Returns the new weights; stores moments.
struct Chunk {
    uint2 q;
    float4 d0, d1, g0, g1, p0, p1;
    uint4 m, v;
};

__device__ __forceinline__ void load_chunk(Chunk &k, const int8_t *qrow, const float *drow, const float *grow,
                                           const float *prow, const uint16_t *mrow, const uint16_t *vrow,
                                           int c0, bool partner, bool moments)
{
    k.q = __ldcs(reinterpret_cast<const uint2 *>(qrow + c0));
    k.d0 = __ldcs(reinterpret_cast<const float4 *>(drow + c0));
    k.d1 = __ldcs(reinterpret_cast<const float4 *>(drow + c0 + 4));
    k.g0 = __ldcs(reinterpret_cast<const float4 *>(grow + c0));
    k.g1 = __ldcs(reinterpret_cast<const float4 *>(grow + c0 + 4));
    if (partner) {
        k.p0 = __ldg(reinterpret_cast<const float4 *>(prow + c0));
        k.p1 = __ldg(reinterpret_cast<const float4 *>(prow + c0 + 4));
    } else {
        k.p0 = k.p1 = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (moments) {
        k.m = __ldcs(reinterpret_cast<const uint4 *>(mrow + c0));
        k.v = __ldcs(reinterpret_cast<const uint4 *>(vrow + c0));
    } else {
        k.m = k.v = make_uint4(0u, 0u, 0u, 0u);
    }
}

struct AdamRow {
    float sc, c_self, c_partner, beta1, beta2, omb1, omb2, bc1, bc2, eps, nlr, nlrwd, clip, wd;
};

// nan_sum stays exactly 0 while every new weight is finite (w * 0 is 0 for finite w, NaN for
// inf or NaN, and a NaN survives every later addition); big tracks the largest moment, which
// must stay below 65520 to be representable in fp16.
__device__ __forceinline__ void adam_chunk(const Chunk &k, const AdamRow &a, float (&wn)[8], uint4 &mo,
                                           uint4 &vo, float &amax, float &nan_sum, float &big)
{
    const float dl[8] = {k.d0.x, k.d0.y, k.d0.z, k.d0.w, k.d1.x, k.d1.y, k.d1.z, k.d1.w};
    const float ga_[8] = {k.g0.x, k.g0.y, k.g0.z, k.g0.w, k.g1.x, k.g1.y, k.g1.z, k.g1.w};
    const float gb_[8] = {k.p0.x, k.p0.y, k.p0.z, k.p0.w, k.p1.x, k.p1.y, k.p1.z, k.p1.w};
    const uint32_t mw[4] = {k.m.x, k.m.y, k.m.z, k.m.w};
    const uint32_t vw[4] = {k.v.x, k.v.y, k.v.z, k.v.w};
    uint32_t mout[4], vout[4];
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) {
        const float2 mo2 = __half22float2(*reinterpret_cast<const __half2 *>(&mw[e2]));
        const float2 vo2 = __half22float2(*reinterpret_cast<const __half2 *>(&vw[e2]));
        float m1[2], v1[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = 2 * e2 + h;
            const int8_t qe = static_cast<int8_t>(((e < 4 ? k.q.x : k.q.y) >> (8 * (e & 3))) & 0xFF);
            const float W = __fmaf_rn(a.sc, (float)qe, dl[e]);
            float ga = ga_[e], gb = gb_[e];
            if (a.clip > 0.0f) {
                ga = fminf(fmaxf(ga, -a.clip), a.clip);
                gb = fminf(fmaxf(gb, -a.clip), a.clip);
            }
            const float gt = __fmaf_rn(a.c_partner, gb, __fmul_rn(a.c_self, ga));
            const float mold = h ? mo2.y : mo2.x;
            const float vold = h ? vo2.y : vo2.x;
            m1[h] = __fmaf_rn(a.beta1, mold, __fmul_rn(a.omb1, gt));
            v1[h] = __fmaf_rn(a.beta2, vold, __fmul_rn(a.omb2, __fmul_rn(gt, gt)));
            const float u = __fdiv_rn(__fmul_rn(m1[h], a.bc1),
                                      __fadd_rn(__fsqrt_rn(__fmul_rn(v1[h], a.bc2)), a.eps));
            float Wn = __fmaf_rn(a.nlr, u, W);
            if (a.wd != 0.0f) Wn = __fmaf_rn(a.nlrwd, W, Wn);
            wn[e] = Wn;
            amax = fmaxf(amax, fabsf(Wn));
            nan_sum = __fmaf_rn(Wn, 0.0f, nan_sum);
            big = fmaxf(big, fmaxf(fabsf(m1[h]), v1[h]));
        }
        const __half2 mh = __floats2half2_rn(m1[0], m1[1]);
        const __half2 vh = __floats2half2_rn(v1[0], v1[1]);
        mout[e2] = *reinterpret_cast<const uint32_t *>(&mh);
        vout[e2] = *reinterpret_cast<const uint32_t *>(&vh);
    }
    mo = make_uint4(mout[0], mout[1], mout[2], mout[3]);
    vo = make_uint4(vout[0], vout[1], vout[2], vout[3]);
}

// One CTA owns one row at a time. Pass 1 streams the row's q, delta, gradient(s) and moments
// through registers, UNROLL chunks of 8 columns per thread in flight, stores the new moments at
// once and parks the new fp32 weight in shared memory (4*C bytes), so a thread needs few
// registers and several CTAs share an SM; pass 2 requantises from shared memory.
template <int UNROLL>
__global__ void __launch_bounds__(kThreads, (UNROLL == 1 ? 1024 : 768) / kThreads)
update_kernel(const __grid_constant__ UpdBatch b, uint32_t *status)
{
    extern __shared__ float4 wrow4[];                 // new weights of the current row
    __shared__ int s_prefix[kMaxMatsPerLaunch + 1];
    __shared__ int scan_scratch[33];
    __shared__ uint32_t max_scratch[33];
    __shared__ int s_meta[5];
    __shared__ float s_metaf[3];

    const int tid = threadIdx.x;
    for (int base = 0; base < b.n; base += kThreads) {   // prefix of active-row counts
        const int i = base + tid;
        const int c = i < b.n ? b.d[i].counts[0] : 0;
        int tot;
        const int off = block_exclusive_scan(c, scan_scratch, &tot);
        const int run = base == 0 ? 0 : s_prefix[base];
        __syncthreads();
        if (i < b.n) s_prefix[i] = run + off;
        if (tid == 0) s_prefix[min(base + kThreads, b.n)] = run + tot;
        __syncthreads();
    }
    const int total = s_prefix[b.n];
    float nan_sum = 0.0f, big = 0.0f;

    // Per-row metadata is a chain of dependent loads (row id -> slot -> step count -> bias
    // corrections). Thread 0 walks the chain of the CTA's next row one link per phase of the
    // current row, so its latency hides behind the current row's traffic, and publishes the
    // result in shared memory for the next iteration.
    auto locate = [&](int item) {
        int lo = 0, hi = b.n - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_prefix[mid] <= item) lo = mid; else hi = mid - 1;
        }
        return lo;
    };
    int n_lo = 0, n_r = 0, n_slot = -1, n_pslot = -1, n_t = 0;
    float n_sc = 0.0f;
    auto publish = [&]() {
        const int ti = n_t + 1 < b.t_max ? n_t + 1 : b.t_max;
        s_meta[0] = n_lo;
        s_meta[1] = n_r;
        s_meta[2] = n_slot;
        s_meta[3] = n_pslot;
        s_meta[4] = n_t;
        s_metaf[0] = n_sc;
        s_metaf[1] = b.bc1[ti];
        s_metaf[2] = b.bc2[ti];
    };
    auto link_slot = [&]() {                        // needs n_r
        const UpdDesc &dn = b.d[n_lo];
        n_slot = dn.row_slot[n_r];
        n_pslot = dn.prow_slot ? dn.prow_slot[n_r] : -1;
        n_sc = dn.s[n_r];
    };
    auto link_step = [&]() {                        // needs n_slot
        n_t = n_slot >= 0 ? b.d[n_lo].slot_step[n_slot] : 0;
    };
    if (tid == 0 && (int)blockIdx.x < total) {
        n_lo = locate(blockIdx.x);
        n_r = b.d[n_lo].active_rows[blockIdx.x - s_prefix[n_lo]];
        link_slot();
        link_step();
        publish();
    }

    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        __syncthreads();                 // this row's metadata is published; the shared row is free
        const UpdDesc &d = b.d[s_meta[0]];
        const int r = s_meta[1], slot = s_meta[2], pslot = s_meta[3], t_old = s_meta[4];
        const float sc = s_metaf[0], bc1 = s_metaf[1], bc2 = s_metaf[2];
        const int nxt = item + gridDim.x;
        const bool chain = tid == 0 && nxt < total;
        if (chain) {                                 // link 1: the next row's id
            n_lo = locate(nxt);
            n_r = b.d[n_lo].active_rows[nxt - s_prefix[n_lo]];
        }
        if (slot < 0) {                              // no moments for this row (overflow)
            if (chain) {
                link_slot();
                link_step();
            }
            __syncthreads();                         // every thread has read this row's metadata
            if (chain) publish();
            continue;
        }
        const int t = t_old + 1;
        AdamRow a;
        a.sc = sc;
        a.c_self = d.c_self;
        a.c_partner = d.c_partner;
        a.beta1 = b.beta1;
        a.beta2 = b.beta2;
        a.omb1 = b.omb1;
        a.omb2 = b.omb2;
        a.bc1 = bc1;
        a.bc2 = bc2;
        a.eps = b.eps;
        a.nlr = -b.lr;
        a.nlrwd = __fmul_rn(-b.lr, b.wd);
        a.clip = b.clip;
        a.wd = b.wd;
        const int C = d.C, nchunks = C >> 3;
        const int8_t *qrow = d.q + (size_t)r * C;
        const float *drow = d.delta + (size_t)r * C;
        const float *grow = d.grad + (size_t)slot * C;
        const float *prow = d.pgrad + (size_t)(pslot < 0 ? 0 : pslot) * C;
        uint16_t *mrow = d.m + (size_t)slot * C;
        uint16_t *vrow = d.v + (size_t)slot * C;
        const bool partner = pslot >= 0, moments = t_old > 0;

        // ---- pass 1: rebuild, mix, Adam; moments out, new weight to shared memory ----
        float amax = 0.0f;
        for (int j0 = tid; j0 < nchunks; j0 += kThreads * UNROLL) {
            {   // the thread's next chunk: into L2 now, so its loads next iteration hit L2. One lane in
                // each group that shares a 128-byte line asks for it.
                const int jn = j0 + kThreads * UNROLL;
                if (jn < nchunks) {
                    const int cn = jn << 3;
                    if ((tid & 3) == 0) {
                        prefetch_l2(drow + cn);
                        prefetch_l2(grow + cn);
                        if (partner) prefetch_l2(prow + cn);
                    }
                    if ((tid & 7) == 0 && moments) {
                        prefetch_l2(mrow + cn);
                        prefetch_l2(vrow + cn);
                    }
                    if ((tid & 15) == 0) prefetch_l2(qrow + cn);
                }
            }
            Chunk k[UNROLL];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int j = j0 + u * kThreads;
                if (j < nchunks) load_chunk(k[u], qrow, drow, grow, prow, mrow, vrow, j << 3, partner, moments);
            }
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int j = j0 + u * kThreads;
                if (j >= nchunks) break;
                float wn[8];
                uint4 mo, vo;
                adam_chunk(k[u], a, wn, mo, vo, amax, nan_sum, big);
                __stcs(reinterpret_cast<uint4 *>(mrow + (j << 3)), mo);
                __stcs(reinterpret_cast<uint4 *>(vrow + (j << 3)), vo);
                wrow4[2 * j] = make_float4(wn[0], wn[1], wn[2], wn[3]);
                wrow4[2 * j + 1] = make_float4(wn[4], wn[5], wn[6], wn[7]);
            }
        }
        if (chain) link_slot();                      // link 2: the next row's slot and scale

        // new per-row scale from the row absmax (non-negative floats order as unsigned ints);
        // the reduction's barriers also publish the shared-memory row to every thread
        const float rmax = __uint_as_float(block_max_u32(__float_as_uint(amax), max_scratch));
        const float sp = __fdiv_rn(rmax, 127.0f);
        const float rcp = __frcp_rn(sp);
        const bool fast = sp != 0.0f && isfinite(rcp);
        if (chain) link_step();                      // link 3: the next row's step count

        // ---- pass 2: requantise from shared memory, write q, delta and the live row ----
        int8_t *qout = d.q + (size_t)r * C;
        float *dout = d.delta + (size_t)r * C;
        uint16_t *lout = d.live ? d.live + (size_t)r * C : nullptr;
        for (int j = tid; j < nchunks; j += kThreads) {
            const int c0 = j << 3;
            const float4 w0 = wrow4[2 * j], w1 = wrow4[2 * j + 1];
            const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            uint32_t qo[2] = {0u, 0u};
            float dn[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float qf = 0.0f, de = wv[e];
                if (sp != 0.0f) {
                    qf = quant_code(wv[e], sp, rcp, fast);
                    de = __fmaf_rn(-sp, qf, wv[e]);
                }
                qo[e >> 2] |= ((uint32_t)(int)qf & 0xFFu) << (8 * (e & 3));
                dn[e] = de;
            }
            __stcs(reinterpret_cast<uint2 *>(qout + c0), make_uint2(qo[0], qo[1]));
            __stcs(reinterpret_cast<float4 *>(dout + c0), make_float4(dn[0], dn[1], dn[2], dn[3]));
            __stcs(reinterpret_cast<float4 *>(dout + c0 + 4), make_float4(dn[4], dn[5], dn[6], dn[7]));
            if (lout) {
                const __nv_bfloat162 l0 = __floats2bfloat162_rn(wv[0], wv[1]);
                const __nv_bfloat162 l1 = __floats2bfloat162_rn(wv[2], wv[3]);
                const __nv_bfloat162 l2 = __floats2bfloat162_rn(wv[4], wv[5]);
                const __nv_bfloat162 l3 = __floats2bfloat162_rn(wv[6], wv[7]);
                __stcs(reinterpret_cast<uint4 *>(lout + c0),
                       make_uint4(*reinterpret_cast<const uint32_t *>(&l0), *reinterpret_cast<const uint32_t *>(&l1),
                                  *reinterpret_cast<const uint32_t *>(&l2), *reinterpret_cast<const uint32_t *>(&l3)));
            }
        }
        if (tid == 0) {
            d.s[r] = sp;
            d.slot_step[slot] = t;
        }
        if (chain) publish();                        // link 4: bias corrections; ready for the next row
    }
    if (nan_sum != 0.0f || !(big < 65520.0f)) set_status(status, SF_STATUS_NONFINITE);
}

// 1/(1 - beta^t) for t = 0..t_max; beta^t as t successive fp64 products of the fp32 beta.
__global__ void adam_tables_kernel(float beta1, float beta2, int t_max, float *bc1, float *bc2)
{
    const float beta = threadIdx.x == 0 ? beta1 : beta2;
    float *bc = threadIdx.x == 0 ? bc1 : bc2;
    double p = 1.0;
    bc[0] = 1.0f;
    for (int t = 1; t <= t_max; ++t) {
        p = __dmul_rn(p, (double)beta);
        bc[t] = __double2float_rn(__ddiv_rn(1.0, __dsub_rn(1.0, p)));
    }
}

// Initial quantisation, one CTA per row: s = max|W| / 127, q = rint(W / s), delta = fma(-s, q, W).
__global__ void __launch_bounds__(256)
quantize_kernel(const float *W, int C, int8_t *q, float *s, float *delta, uint16_t *live)
{
    __shared__ uint32_t max_scratch[33];
    const size_t row = (size_t)blockIdx.x * C;
    float amax = 0.0f;
    for (int c = threadIdx.x; c < C; c += blockDim.x) amax = fmaxf(amax, fabsf(W[row + c]));
    const float sp = __fdiv_rn(__uint_as_float(block_max_u32(__float_as_uint(amax), max_scratch)), 127.0f);
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
        const float x = W[row + c];
        float qf = 0.0f, de = x;
        if (sp != 0.0f) {
            qf = fminf(fmaxf(rintf(__fdiv_rn(x, sp)), -127.0f), 127.0f);
            de = __fmaf_rn(-sp, qf, x);
        }
        q[row + c] = (int8_t)(int)qf;
        delta[row + c] = de;
        if (live) live[row + c] = __bfloat16_as_ushort(__float2bfloat16_rn(x));
    }
    if (threadIdx.x == 0) s[blockIdx.x] = sp;
}

}  // namespace
}  // namespace sf

using namespace sf;

extern "C" int sf_adam_tables(float beta1, float beta2, int t_max, float *bc1, float *bc2,
                              sf_stream stream)
{
    if (t_max < 1 || !bc1 || !bc2) return SF_ERR_ARG;
    if (!(beta1 >= 0.0f && beta1 < 1.0f && beta2 >= 0.0f && beta2 < 1.0f)) return SF_ERR_ARG;
    adam_tables_kernel<<<1, 2, 0, as_stream(stream)>>>(beta1, beta2, t_max, bc1, bc2);
    return launch_status();
}

extern "C" int sf_quantize_init(const float *W, int R, int C, int8_t *q, float *s, float *delta,
                                uint16_t *live, sf_stream stream)
{
    if (!W || !q || !s || !delta || R < 0 || C < 0) return SF_ERR_ARG;
    if (R == 0 || C == 0) return SF_OK;
    quantize_kernel<<<R, 256, 0, as_stream(stream)>>>(W, C, q, s, delta, live);
    return launch_status();
}

extern "C" int sf_sparse_update(const sf_matrix *mats, int n_mats, const sf_adam *hp,
                                uint32_t *dev_status, sf_stream stream)
{
    if (n_mats < 0 || (n_mats > 0 && !mats) || !hp) return SF_ERR_ARG;
    if (!hp->bc1 || !hp->bc2 || hp->t_max < 1) return SF_ERR_ARG;
    int maxC = 8;
    for (int i = 0; i < n_mats; ++i) {
        const sf_matrix &a = mats[i];
        int rc = check_mask(a.mask);
        if (rc != SF_OK) return rc;
        if (a.C <= 0 || (a.C & 7)) return SF_ERR_ARG;
        if (a.C > kMaxC) return SF_ERR_UNSUPPORTED;
        if (!a.q || !a.s || !a.delta || !a.m || !a.v || !a.grad) return SF_ERR_ARG;
        if (!aligned16(a.delta) || !aligned16(a.m) || !aligned16(a.v) || !aligned16(a.grad) ||
            ((uintptr_t)a.q & 7) || (a.live && !aligned16(a.live)))
            return SF_ERR_ALIGN;
        if (a.partner >= n_mats || a.partner < -1 || a.partner == i) return SF_ERR_ARG;
        if (a.partner >= 0) {
            const sf_matrix &p = mats[a.partner];
            if (p.mask.R != a.mask.R || p.C != a.C) return SF_ERR_ARG;
        }
        if (a.C > maxC) maxC = a.C;
    }
    if (n_mats == 0) return SF_OK;
    const int sms = sm_count();
    if (sms <= 0) return SF_ERR_NO_DEVICE;
    const size_t smem = (size_t)maxC * sizeof(float);
#ifndef SF_UPDATE_UNROLL
#define SF_UPDATE_UNROLL 1
#endif
    const int unroll = SF_UPDATE_UNROLL;
    const void *fn = unroll == 2 ? (const void *)update_kernel<2> : (const void *)update_kernel<1>;
    // opt-in beyond 48 KB of shared memory in all, static included (set from 40 KB dynamic on)
    if (smem > 40 * 1024 &&
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return SF_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, smem) != cudaSuccess ||
        per_sm <= 0)
        return SF_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    for (int first = 0; first < n_mats; first += kMaxMatsPerLaunch) {
        const int cnt = n_mats - first < kMaxMatsPerLaunch ? n_mats - first : kMaxMatsPerLaunch;
        UpdBatch b;
        b.n = cnt;
        b.lr = hp->lr;
        b.beta1 = hp->beta1;
        b.beta2 = hp->beta2;
        b.eps = hp->eps;
        b.omb1 = hp->one_minus_b1;
        b.omb2 = hp->one_minus_b2;
        b.wd = hp->wd;
        b.clip = hp->clip;
        b.bc1 = hp->bc1;
        b.bc2 = hp->bc2;
        b.t_max = hp->t_max;
        for (int j = 0; j < cnt; ++j) {
            const sf_matrix &a = mats[first + j];
            UpdDesc &d = b.d[j];
            d.R = a.mask.R;
            d.C = a.C;
            d.c_self = a.c_self;
            d.c_partner = a.c_partner;
            d.active_rows = a.mask.active_rows;
            d.counts = a.mask.counts;
            d.row_slot = a.mask.row_slot;
            d.slot_step = a.mask.slot_step;
            d.q = a.q;
            d.s = a.s;
            d.delta = a.delta;
            d.m = a.m;
            d.v = a.v;
            d.grad = a.grad;
            d.live = a.live;
            d.pgrad = a.partner >= 0 ? mats[a.partner].grad : nullptr;
            d.prow_slot = a.partner >= 0 ? mats[a.partner].mask.row_slot : nullptr;
        }
        // A plain launch: the kernel reads the masks' lists and slots from its first instruction,
        // and the call may directly follow the masks' finalize, which releases its successor
        // early (programmatic dependent launch) for its own chained launches.
        if (unroll == 2)
            update_kernel<2><<<sms * per_sm, kThreads, smem, st>>>(b, dev_status);
        else
            update_kernel<1><<<sms * per_sm, kThreads, smem, st>>>(b, dev_status);
        if (launch_status() != SF_OK) return SF_ERR_CUDA;
    }
    return SF_OK;
}
