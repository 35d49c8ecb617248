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
// 512 threads owns one row at a time: it streams the row's q, delta, gradient(s) and fp16
// moments in with 8- and 16-byte vector loads (all coalesced), keeps the new weight in
// registers, finds the new row absmax with a block reduction, then requantises from the
// registers and streams q, delta, moments and the bf16 live row out. HBM-bound: per active
// element it reads 1 + 4 + 4 + 2 + 2 bytes and writes 1 + 4 + 2 + 2 + 2 bytes.
// Every floating-point step is an explicitly rounded intrinsic, in a fixed order, so results
// are bit-reproducible and independent of the compiler's contraction choices.
#include "sf_common.cuh"
#include "sf_host.h"

namespace sf {
namespace {

constexpr int kThreads = 512;
constexpr int kMaxMatsPerLaunch = 200;
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
static_assert(sizeof(UpdBatch) < 32000, "kernel parameter space");

template <int CPT>   // 8-column chunks per thread; one chunk per thread fits two CTAs per SM
__global__ void __launch_bounds__(kThreads, CPT == 1 ? 2 : 1)
update_kernel(const __grid_constant__ UpdBatch b, uint32_t *status)
{
    __shared__ int s_prefix[kMaxMatsPerLaunch + 1];
    __shared__ int scan_scratch[33];
    __shared__ uint32_t max_scratch[33];

    const int tid = threadIdx.x;
    {   // prefix of active-row counts over the matrices of this launch
        const int c = tid < b.n ? b.d[tid].counts[0] : 0;
        int total;
        const int off = block_exclusive_scan(c, scan_scratch, &total);
        if (tid < b.n) s_prefix[tid] = off;
        if (tid == 0) s_prefix[b.n] = total;
        __syncthreads();
    }
    const int total = s_prefix[b.n];
    const float nlr = -b.lr;
    const float nlrwd = __fmul_rn(-b.lr, b.wd);
    bool nonfinite = false;

    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        int lo = 0, hi = b.n - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_prefix[mid] <= item) lo = mid; else hi = mid - 1;
        }
        const UpdDesc &d = b.d[lo];
        const int r = d.active_rows[item - s_prefix[lo]];
        const int slot = d.row_slot[r];
        if (slot < 0) continue;                       // no moments for this row (overflow)
        const int pslot = d.prow_slot ? d.prow_slot[r] : -1;
        const int t_old = d.slot_step[slot];
        const int t = t_old + 1;
        const int ti = t < b.t_max ? t : b.t_max;
        const float bc1 = b.bc1[ti], bc2 = b.bc2[ti];
        const float sc = d.s[r];
        const int C = d.C, nchunks = C >> 3;
        const size_t wrow = (size_t)r * C;
        const size_t grow = (size_t)slot * C;
        const size_t prow = (size_t)pslot * C;

        // Phase A: issue every load of this thread's chunks before any arithmetic, so that
        // CPT x ~100 bytes per thread are in flight at once.
        uint2 qv[CPT];
        float4 dv[CPT][2], gv[CPT][2], pv[CPT][2];
        uint4 mv[CPT], vv[CPT];
#pragma unroll
        for (int k = 0; k < CPT; ++k) {
            const int j = tid + k * kThreads;
            if (j < nchunks) {
                const int c0 = j << 3;
                qv[k] = __ldcs(reinterpret_cast<const uint2 *>(d.q + wrow + c0));
                dv[k][0] = __ldcs(reinterpret_cast<const float4 *>(d.delta + wrow + c0));
                dv[k][1] = __ldcs(reinterpret_cast<const float4 *>(d.delta + wrow + c0 + 4));
                gv[k][0] = __ldcs(reinterpret_cast<const float4 *>(d.grad + grow + c0));
                gv[k][1] = __ldcs(reinterpret_cast<const float4 *>(d.grad + grow + c0 + 4));
                if (pslot >= 0) {
                    pv[k][0] = __ldg(reinterpret_cast<const float4 *>(d.pgrad + prow + c0));
                    pv[k][1] = __ldg(reinterpret_cast<const float4 *>(d.pgrad + prow + c0 + 4));
                } else {
                    pv[k][0] = pv[k][1] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
                if (t_old > 0) {
                    mv[k] = __ldcs(reinterpret_cast<const uint4 *>(d.m + grow + c0));
                    vv[k] = __ldcs(reinterpret_cast<const uint4 *>(d.v + grow + c0));
                } else {
                    mv[k] = vv[k] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
        }

        // Phase B: rebuild, mix, Adam; moments go out at once, the new weight stays in registers.
        float w[CPT][8];
        float amax = 0.0f;
#pragma unroll
        for (int k = 0; k < CPT; ++k) {
            const int j = tid + k * kThreads;
            if (j >= nchunks) continue;
            const int c0 = j << 3;
            const float dl[8] = {dv[k][0].x, dv[k][0].y, dv[k][0].z, dv[k][0].w,
                                 dv[k][1].x, dv[k][1].y, dv[k][1].z, dv[k][1].w};
            const float ga_[8] = {gv[k][0].x, gv[k][0].y, gv[k][0].z, gv[k][0].w,
                                  gv[k][1].x, gv[k][1].y, gv[k][1].z, gv[k][1].w};
            const float gb_[8] = {pv[k][0].x, pv[k][0].y, pv[k][0].z, pv[k][0].w,
                                  pv[k][1].x, pv[k][1].y, pv[k][1].z, pv[k][1].w};
            const uint32_t mw[4] = {mv[k].x, mv[k].y, mv[k].z, mv[k].w};
            const uint32_t vw[4] = {vv[k].x, vv[k].y, vv[k].z, vv[k].w};
            uint32_t mout[4], vout[4];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int8_t qe = static_cast<int8_t>(((e < 4 ? qv[k].x : qv[k].y) >> (8 * (e & 3))) & 0xFF);
                const float W = __fmaf_rn(sc, (float)qe, dl[e]);
                float ga = ga_[e], gb = gb_[e];
                if (b.clip > 0.0f) {
                    ga = fminf(fmaxf(ga, -b.clip), b.clip);
                    gb = fminf(fmaxf(gb, -b.clip), b.clip);
                }
                const float gt = __fmaf_rn(d.c_partner, gb, __fmul_rn(d.c_self, ga));
                const uint16_t mh = (uint16_t)(mw[e >> 1] >> (16 * (e & 1)));
                const uint16_t vh = (uint16_t)(vw[e >> 1] >> (16 * (e & 1)));
                const float m_old = __half2float(__ushort_as_half(mh));
                const float v_old = __half2float(__ushort_as_half(vh));
                const float m1 = __fmaf_rn(b.beta1, m_old, __fmul_rn(b.omb1, gt));
                const float v1 = __fmaf_rn(b.beta2, v_old, __fmul_rn(b.omb2, __fmul_rn(gt, gt)));
                const float u = __fdiv_rn(__fmul_rn(m1, bc1),
                                          __fadd_rn(__fsqrt_rn(__fmul_rn(v1, bc2)), b.eps));
                float Wn = __fmaf_rn(nlr, u, W);
                if (b.wd != 0.0f) Wn = __fmaf_rn(nlrwd, W, Wn);
                const uint16_t m16 = __half_as_ushort(__float2half_rn(m1));
                const uint16_t v16 = __half_as_ushort(__float2half_rn(v1));
                nonfinite |= !isfinite(Wn) || (v16 & 0x7C00u) == 0x7C00u || (m16 & 0x7C00u) == 0x7C00u;
                if (e & 1) {
                    mout[e >> 1] |= (uint32_t)m16 << 16;
                    vout[e >> 1] |= (uint32_t)v16 << 16;
                } else {
                    mout[e >> 1] = m16;
                    vout[e >> 1] = v16;
                }
                w[k][e] = Wn;
                amax = fmaxf(amax, fabsf(Wn));
            }
            __stcs(reinterpret_cast<uint4 *>(d.m + grow + c0), make_uint4(mout[0], mout[1], mout[2], mout[3]));
            __stcs(reinterpret_cast<uint4 *>(d.v + grow + c0), make_uint4(vout[0], vout[1], vout[2], vout[3]));
        }

        // new per-row scale from the row absmax (non-negative floats order as unsigned ints)
        const float rmax = __uint_as_float(block_max_u32(__float_as_uint(amax), max_scratch));
        const float sp = __fdiv_rn(rmax, 127.0f);

#pragma unroll
        for (int k = 0; k < CPT; ++k) {
            const int j = tid + k * kThreads;
            if (j >= nchunks) continue;
            const int c0 = j << 3;
            uint32_t qo[2] = {0u, 0u};
            float dn[8];
            uint32_t lo16[4];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float Wn = w[k][e];
                float qf = 0.0f, de = Wn;
                if (sp != 0.0f) {
                    qf = rintf(__fdiv_rn(Wn, sp));
                    qf = fminf(fmaxf(qf, -127.0f), 127.0f);
                    de = __fmaf_rn(-sp, qf, Wn);
                }
                const int qi = (int)qf;
                qo[e >> 2] |= ((uint32_t)qi & 0xFFu) << (8 * (e & 3));
                dn[e] = de;
                const uint16_t lb = __bfloat16_as_ushort(__float2bfloat16_rn(Wn));
                if (e & 1) lo16[e >> 1] |= (uint32_t)lb << 16; else lo16[e >> 1] = lb;
            }
            __stcs(reinterpret_cast<uint2 *>(d.q + wrow + c0), make_uint2(qo[0], qo[1]));
            __stcs(reinterpret_cast<float4 *>(d.delta + wrow + c0), make_float4(dn[0], dn[1], dn[2], dn[3]));
            __stcs(reinterpret_cast<float4 *>(d.delta + wrow + c0 + 4), make_float4(dn[4], dn[5], dn[6], dn[7]));
            if (d.live)
                __stcs(reinterpret_cast<uint4 *>(d.live + wrow + c0), make_uint4(lo16[0], lo16[1], lo16[2], lo16[3]));
        }
        if (tid == 0) {
            d.s[r] = sp;
            d.slot_step[slot] = t;
        }
    }
    if (nonfinite) set_status(status, SF_STATUS_NONFINITE);
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

template <int CPT>
int launch_update(const UpdBatch &b, int grid, uint32_t *status, cudaStream_t st)
{
    update_kernel<CPT><<<grid, kThreads, 0, st>>>(b, status);
    return launch_status();
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
    const int cpt_needed = (maxC / 8 + kThreads - 1) / kThreads;
    const int sms = sm_count();
    if (sms <= 0) return SF_ERR_NO_DEVICE;
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
        const int grid = sms * 2;
        int rc;
        switch (cpt_needed) {
        case 1: rc = launch_update<1>(b, grid, dev_status, st); break;
        case 2: rc = launch_update<2>(b, grid, dev_status, st); break;
        case 3: rc = launch_update<3>(b, grid, dev_status, st); break;
        case 4: rc = launch_update<4>(b, grid, dev_status, st); break;
        case 5: case 6: rc = launch_update<6>(b, grid, dev_status, st); break;
        default: rc = launch_update<8>(b, grid, dev_status, st); break;
        }
        if (rc != SF_OK) return rc;
    }
    return SF_OK;
}
