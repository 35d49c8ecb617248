// sf_fwd.cu -- the forward projection with the row tracker folded into its epilogue.
//
// "Sparse-First Fine-Tuning" (tensorwirelabs.com), section 2.1 (Observing activity): a
// projection's row activity for the charge rule comes from the magnitudes of the outputs its
// forward pass produced. Read on its own, that pass is a second trip through every output
// (T x R bf16 per projection, the largest stream of the sparse step). Here the forward product
// itself keeps the statistic: the kernel computes Y = A W^T, rounds it to bf16, stores it, and
// folds max over its tokens of |Y[t, r]| (of the stored bf16 values) into the mask's
// accumulator -- exactly what the column-max pass of sf_mask_update would have found, so
// sf_mask_update_phase(SF_PHASE_SECOND) can finalize the masks at once.
//
// Shapes: A is T x C (token-major layer inputs), W is R x C (the live weights, row-major), Y is
// T x R. In GEMM terms M = tokens, N = weight rows, K = C, and both operands are K-major.
//
// CTA (1 per SM, 320 threads, persistent over the (problem, 128-token, 256-row) units):
//   warp 0      TMA producer: per 64-column stage, a {64, 128} box of A and a {64, 256} box of
//               W, both with the 128-byte swizzle, into a 4-deep ring;
//   warp 1      allocates 512 TMEM columns; one thread issues tcgen05.mma kind::f16 (M=128,
//               N=256, K=16) chunk by chunk into two 256-column buffers (each chunk of 1024
//               columns of C starts from zero);
//   warps 2-9   epilogue: two warps per TMEM lane quarter, one per 128-row half of the unit;
//               each adds the finished chunks into fp32 registers (round to nearest), rounds the
//               sums to bf16, stores its token's 128 outputs, takes the column magnitudes' max
//               over the warp's 32 tokens (redux.sync), combines the four warps of its half in
//               shared memory and issues one atomicMax per weight row and unit.
// Non-finite outputs follow sf_mask_update's reading: a NaN adds no magnitude, an infinity
// counts as the largest finite bf16 magnitude; either sets SF_STATUS_NONFINITE.
// Every mbarrier wait is bounded (2 s), as in the masked dW kernel.
#include <string.h>

#include "sf_common.cuh"
#include "sf_host.h"

namespace sf {
namespace {

#ifndef SF_FWD_PAIR
#define SF_FWD_PAIR 1
#endif
// CTAs sharing a unit: with 2, a cluster pair runs one tcgen05.mma with cta_group::2 (M = 256
// tokens): each CTA loads its own 128 tokens of A and its own 128 of the unit's 256 weight rows
// (completing on the even CTA's barriers), so each SM loads 32 KB per stage instead of 48 KB.
// Measured on B200 (parity green in both builds), one 7B layer at 2,048 tokens: 1,248 vs 1,222
// TFLOP/s; 32 layers: 1,020 vs 1,114. One CTA per unit is the default.
constexpr int FPAIR = SF_FWD_PAIR;
static_assert(FPAIR == 1 || FPAIR == 2, "one CTA or a CTA pair per unit");
constexpr int FM = 128;                 // tokens per CTA (TMEM lanes)
constexpr int FUM = FM * FPAIR;         // tokens per unit
constexpr int FN = 256;                 // weight rows per unit
constexpr int FNC = FN / FPAIR;         // weight rows each CTA loads
constexpr int FK = 64;                  // columns of C per stage (128 bytes of bf16)
constexpr int F_UMMA_K = 16;
constexpr int F_STAGES = FPAIR == 2 ? 6 : 4;
constexpr int F_A_BYTES = FM * FK * 2;              // 16 KB
constexpr int F_W_BYTES = FNC * FK * 2;             // 32 KB (16 KB per CTA of a pair)
constexpr int F_STAGE_BYTES = F_A_BYTES + F_W_BYTES;
constexpr int F_CHUNK_STAGES = 1024 / FK;           // accumulation chunk: 1024 columns of C
constexpr int F_NBUF = 2;
constexpr int F_TMEM_COLS = F_NBUF * FN;
constexpr int F_EPI_WARPS = 8;
constexpr int F_EPI_COLS = FN / 2;
constexpr int F_THREADS = 64 + 32 * F_EPI_WARPS;
constexpr size_t F_SMEM_BYTES = (size_t)F_STAGES * F_STAGE_BYTES + 1024;
constexpr int F_MAX_PROBS = 96;

// kind::f16 instruction descriptor: fp32 accumulator, bf16 A and B, both K-major, N, M.
constexpr uint32_t kFwdIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(FN >> 3) << 17) |
                               ((uint32_t)(FUM >> 4) << 24);
constexpr uint32_t kSW128 = 2;

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t addr)
{
    // K-major, 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart (SBO); the
    // leading offset is unused for this layout (1, as the canonical form has it).
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
           (1ull << 46) | ((uint64_t)kSW128 << 61);
}

struct alignas(64) FwdProb {
    CUtensorMap tm_a;            // A: dims {C, T}, box {64, 128}, 128-byte swizzle
    CUtensorMap tm_w;            // W: dims {C, R}, box {64, 256 / pair}, 128-byte swizzle
    uint16_t *Y;
    int64_t ld_y;
    uint32_t *accum;
    int32_t T, C, R, n_mt, n_nt, unit_begin;
};

struct FwdBatch {
    int32_t n_prob, total_units;
    alignas(64) FwdProb p[F_MAX_PROBS];
};
static_assert(sizeof(FwdBatch) <= 32764, "kernel parameter space");

struct FUnit {
    int p, mt, nt;
};

__device__ __forceinline__ FUnit fdecode(const FwdBatch &b, int u)
{
    int lo = 0, hi = b.n_prob - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (b.p[mid].unit_begin <= u) lo = mid; else hi = mid - 1;
    }
    const int local = u - b.p[lo].unit_begin;
    FUnit x;
    x.p = lo;
    x.nt = local / b.p[lo].n_mt;                      // consecutive units share the W tile
    x.mt = local - x.nt * b.p[lo].n_mt;
    return x;
}

// |bf16| bits with the tracker's reading of non-finite values (NaN -> 0, infinity -> 0x7F7F).
__device__ __forceinline__ uint32_t tracked_magnitude(uint32_t bits, bool &nonfinite)
{
    uint32_t a = bits & 0x7FFFu;
    if (a >= 0x7F80u) {
        nonfinite = true;
        a = a == 0x7F80u ? 0x7F7Fu : 0u;
    }
    return a;
}

__global__ void __launch_bounds__(F_THREADS, 1)
forward_tracked_kernel(const __grid_constant__ FwdBatch b, uint32_t *status)
{
    const uint32_t crank = FPAIR == 2 ? cluster_ctarank() : 0u;
    const bool leader = crank == 0;
    const int unit0 = blockIdx.x / FPAIR, ustep = gridDim.x / FPAIR;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full_bar[F_STAGES], empty_bar[F_STAGES], tfull_bar[F_NBUF], tempty_bar[F_NBUF], drain_bar;
    __shared__ uint32_t tmem_base_s;
    __shared__ volatile int abort_flag;
    __shared__ uint32_t colmax[2][4][F_EPI_COLS];

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int total_units = b.total_units;

    if (tid == 0) {
        abort_flag = 0;
        for (int s = 0; s < F_STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < F_NBUF; ++a) {
            mbar_init(&tfull_bar[a], 1);
            mbar_init(&tempty_bar[a], F_EPI_WARPS * FPAIR);     // the leader's counts both CTAs
        }
        mbar_init(&drain_bar, 1);
        fence_mbarrier_init();
    }
    if (warp == 1) {
        if (FPAIR == 2) tmem_alloc_pair(&tmem_base_s, F_TMEM_COLS);
        else tmem_alloc(&tmem_base_s, F_TMEM_COLS);
    }
    tc_fence_before();
    __syncthreads();
    if (FPAIR == 2) cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_s;

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            for (int i = 0; i < b.n_prob; ++i) {
                prefetch_tmap(&b.p[i].tm_a);
                prefetch_tmap(&b.p[i].tm_w);
            }
            int stage = 0;
            uint32_t phase = 0;
            bool issued[F_STAGES] = {};
            uint32_t issued_parity[F_STAGES] = {};
            bool ok = true;
            for (int u = unit0; u < total_units && ok; u += ustep) {
                const FUnit x = fdecode(b, u);
                const FwdProb &p = b.p[x.p];
                const int nk = (p.C + FK - 1) / FK;
                const int t0 = x.mt * FUM + (int)crank * FM, r0 = x.nt * FN + (int)crank * FNC;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag)) { ok = false; break; }
                    uint8_t *sa = smem + stage * F_STAGE_BYTES;
                    if (leader) mbar_arrive_expect_tx(&full_bar[stage], FPAIR * F_STAGE_BYTES);
                    if (FPAIR == 2) {
                        tma_load_2d_pair(sa, &p.tm_a, &full_bar[stage], kb * FK, t0);
                        tma_load_2d_pair(sa + F_A_BYTES, &p.tm_w, &full_bar[stage], kb * FK, r0);
                    } else {
                        tma_load_2d(sa, &p.tm_a, &full_bar[stage], kb * FK, t0);
                        tma_load_2d(sa + F_A_BYTES, &p.tm_w, &full_bar[stage], kb * FK, r0);
                    }
                    issued[stage] = true;
                    issued_parity[stage] = phase;
                    if (++stage == F_STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            {   // the MMA issuer commits drain_bar once it has finished or given up
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&drain_bar, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {}
            }
            if ((!ok || abort_flag) && leader) {
                for (int s = 0; s < F_STAGES; ++s) {
                    if (!issued[s]) continue;
                    const uint64_t t0 = globaltimer_ns();
                    while (!mbar_try_wait(&full_bar[s], issued_parity[s]) && globaltimer_ns() - t0 < kWaitLimitNs) {}
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t buf_phase = 0;
            bool ok = true;
            for (int u = unit0; u < total_units && ok; u += ustep) {
                const FUnit x = fdecode(b, u);
                const int nk = (b.p[x.p].C + FK - 1) / FK;
                for (int kb = 0; kb < nk; ++kb) {
                    const int in_chunk = kb % F_CHUNK_STAGES;
                    if (in_chunk == 0) {
                        if (!mbar_wait(&tempty_bar[buf], buf_phase ^ 1u, &abort_flag)) { ok = false; break; }
                        tc_fence_after();
                    }
                    if (!mbar_wait(&full_bar[stage], phase, &abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * F_STAGE_BYTES);
                    const uint32_t sw = sa + F_A_BYTES;
                    const uint32_t d_tmem = tmem_base + (uint32_t)(buf * FN);
#pragma unroll
                    for (int k = 0; k < FK / F_UMMA_K; ++k) {     // 16 columns of C = 32 bytes
                        if (FPAIR == 2)
                            mma_bf16_pair(d_tmem, kmajor_desc(sa + k * 32), kmajor_desc(sw + k * 32), kFwdIdesc,
                                          (in_chunk | k) != 0);
                        else
                            mma_bf16(d_tmem, kmajor_desc(sa + k * 32), kmajor_desc(sw + k * 32), kFwdIdesc,
                                     (in_chunk | k) != 0);
                    }
                    if (FPAIR == 2) mma_commit_pair(&empty_bar[stage], 3);
                    else mma_commit(&empty_bar[stage]);
                    if (++stage == F_STAGES) { stage = 0; phase ^= 1u; }
                    if (in_chunk == F_CHUNK_STAGES - 1 || kb == nk - 1) {
                        if (FPAIR == 2) mma_commit_pair(&tfull_bar[buf], 3);
                        else mma_commit(&tfull_bar[buf]);
                        if (++buf == F_NBUF) { buf = 0; buf_phase ^= 1u; }
                    }
                }
            }
            if (FPAIR == 2) mma_commit_pair(&drain_bar, 3);
            else mma_commit(&drain_bar);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&drain_bar, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {}
        }
    } else {
        // --------------------------- epilogue (warps 2..9) ---------------------------
        const int quad = warp & 3;              // TMEM lanes (tokens) 32*quad .. 32*quad+31
        const int half = (warp - 2) >> 2;       // weight rows half*128 .. +127 of the unit
        const int bar_id = 1 + half;            // named barrier of the half's four warps
        int buf = 0;
        uint32_t buf_phase = 0;
        bool nonfinite = false;
        for (int u = unit0; u < total_units; u += ustep) {
            const FUnit x = fdecode(b, u);
            const FwdProb &p = b.p[x.p];
            const int nk = (p.C + FK - 1) / FK;
            const int t = x.mt * FUM + (int)crank * FM + quad * 32 + lane;   // this lane's token
            const int r0 = x.nt * FN + half * F_EPI_COLS;           // first weight row of the half
            float acc[F_EPI_COLS];
#pragma unroll
            for (int j = 0; j < F_EPI_COLS; ++j) acc[j] = 0.0f;
            bool ready = true;
            const int nchunks = (nk + F_CHUNK_STAGES - 1) / F_CHUNK_STAGES;
            for (int ch = 0; ch < nchunks; ++ch) {
                ready = __all_sync(0xffffffffu, mbar_wait(&tfull_bar[buf], buf_phase, &abort_flag));
                if (!ready) break;
                tc_fence_after();
                const uint32_t t_row = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * FN + half * F_EPI_COLS);
#pragma unroll
                for (int cc = 0; cc < F_EPI_COLS / 32; ++cc) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(t_row + cc * 32, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) acc[cc * 32 + j] = __fadd_rn(acc[cc * 32 + j], __uint_as_float(v[j]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (FPAIR == 2 && !leader) mbar_arrive_remote(&tempty_bar[buf], 0);
                    else mbar_arrive(&tempty_bar[buf]);
                }
                if (++buf == F_NBUF) { buf = 0; buf_phase ^= 1u; }
            }
            if (!ready) break;
            // round to bf16, store this token's outputs, and the warp's column maxima
            const bool t_ok = t < p.T;
            uint16_t *yrow = p.Y + (size_t)(t_ok ? t : 0) * p.ld_y;
#pragma unroll
            for (int g = 0; g < F_EPI_COLS / 8; ++g) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __nv_bfloat162 h = __floats2bfloat162_rn(acc[8 * g + 2 * e], acc[8 * g + 2 * e + 1]);
                    w[e] = *reinterpret_cast<const uint32_t *>(&h);
                }
                const int r = r0 + 8 * g;
                if (t_ok && r < p.R)
                    *reinterpret_cast<uint4 *>(yrow + r) = make_uint4(w[0], w[1], w[2], w[3]);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t bits = (w[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
                    const uint32_t m = __reduce_max_sync(0xffffffffu, t_ok ? tracked_magnitude(bits, nonfinite) : 0u);
                    if (lane == ((8 * g + e) & 31)) colmax[half][quad][8 * g + e] = m;
                }
            }
            asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(128) : "memory");
            {   // one thread per weight row of the half: the largest of the four warps' maxima, into
                // the mask's bf16 accumulator two rows at a time (the even lane of each pair)
                const int c = (warp & 3) * 32 + lane;           // 0..127 over the half's 4 warps
                const uint32_t m = max(max(colmax[half][0][c], colmax[half][1][c]),
                                       max(colmax[half][2][c], colmax[half][3][c]));
                const uint32_t m_next = __shfl_down_sync(0xffffffffu, m, 1);
                if ((lane & 1) == 0 && (m | m_next) && r0 + c < p.R)
                    red_max_bf16x2(reinterpret_cast<uint16_t *>(p.accum) + r0 + c, (uint16_t)m, (uint16_t)m_next);
            }
            asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(128) : "memory");
        }
        if (nonfinite) set_status(status, SF_STATUS_NONFINITE);
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (FPAIR == 2) cluster_sync();            // neither CTA leaves while the pair's MMAs may run
    if (abort_flag && tid == 0) set_status(status, SF_STATUS_WAIT_TIMEOUT);
    if (warp == 1) {
        tc_fence_after();
        if (FPAIR == 2) tmem_dealloc_pair(tmem_base, F_TMEM_COLS);
        else tmem_dealloc(tmem_base, F_TMEM_COLS);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn fwd_encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// bf16 K-major map over a row-major [rows x ld] matrix with `cols` valid columns, box {64, box_rows}.
bool encode_kmajor(CUtensorMap *m, const void *base, int cols, int rows, int64_t ld, int box_rows)
{
    EncodeTiledFn fn = fwd_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    const cuuint32_t box[2] = {(cuuint32_t)FK, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace sf

using namespace sf;

extern "C" int sf_forward_tracked(const sf_fwd_problem *probs, int n, uint32_t *dev_status, sf_stream stream)
{
    if (n < 0 || (n > 0 && !probs)) return SF_ERR_ARG;
    for (int i = 0; i < n; ++i) {
        const sf_fwd_problem &p = probs[i];
        const int R = p.mask.R;
        if (R <= 0 || (R & 31) || !p.mask.accum || p.T < 0 || p.C <= 0 || (p.C & 7)) return SF_ERR_ARG;
        if (!aligned16(p.mask.accum)) return SF_ERR_ALIGN;     // the bf16 accumulator takes 16-byte reductions
        if (p.T > 0) {
            if (!p.A || !p.W || !p.Y || p.ld_a < p.C || p.ld_w < p.C || p.ld_y < R) return SF_ERR_ARG;
            if ((p.ld_a & 7) || (p.ld_w & 7) || (p.ld_y & 7) || !aligned16(p.A) || !aligned16(p.W) || !aligned16(p.Y))
                return SF_ERR_ALIGN;
        }
    }
    if (n == 0) return SF_OK;
    const int sms = sm_count();
    if (sms <= 0) return SF_ERR_NO_DEVICE;
    if (cudaFuncSetAttribute(forward_tracked_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)F_SMEM_BYTES) != cudaSuccess)
        return SF_ERR_CUDA;
    int pair_slots = 0;                       // CTA pairs that can be resident at once
    if (FPAIR == 2) {
        cudaLaunchConfig_t qcfg = {};
        cudaLaunchAttribute qattr;
        qattr.id = cudaLaunchAttributeClusterDimension;
        qattr.val.clusterDim.x = 2;
        qattr.val.clusterDim.y = 1;
        qattr.val.clusterDim.z = 1;
        qcfg.gridDim = dim3(2 * sms);
        qcfg.blockDim = dim3(F_THREADS);
        qcfg.dynamicSmemBytes = F_SMEM_BYTES;
        qcfg.attrs = &qattr;
        qcfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&pair_slots, forward_tracked_kernel, &qcfg) != cudaSuccess || pair_slots <= 0)
            return SF_ERR_CUDA;
    }
    cudaStream_t st = as_stream(stream);
    FwdBatch *batch = new FwdBatch;
    int rc = SF_OK;
    for (int first = 0; first < n && rc == SF_OK; first += F_MAX_PROBS) {
        const int cnt = n - first < F_MAX_PROBS ? n - first : F_MAX_PROBS;
        memset(batch, 0, sizeof(*batch));
        int units = 0;
        for (int j = 0; j < cnt; ++j) {
            const sf_fwd_problem &p = probs[first + j];
            FwdProb &d = batch->p[batch->n_prob];
            if (p.T == 0) continue;                       // no tokens: nothing to compute or fold
            if (!encode_kmajor(&d.tm_a, p.A, p.C, p.T, p.ld_a, FM) ||
                !encode_kmajor(&d.tm_w, p.W, p.C, p.mask.R, p.ld_w, FNC)) {
                rc = SF_ERR_CUDA;
                break;
            }
            d.Y = static_cast<uint16_t *>(p.Y);
            d.ld_y = p.ld_y;
            d.accum = p.mask.accum;
            d.T = p.T;
            d.C = p.C;
            d.R = p.mask.R;
            d.n_mt = (p.T + FUM - 1) / FUM;
            d.n_nt = (p.mask.R + FN - 1) / FN;
            d.unit_begin = units;
            units += d.n_mt * d.n_nt;
            ++batch->n_prob;
        }
        if (rc != SF_OK || batch->n_prob == 0) continue;
        batch->total_units = units;
        const int slots = FPAIR == 2 ? pair_slots : sms;
        const int grid = FPAIR * (units < slots ? units : slots);
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 2;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(F_THREADS);
        cfg.dynamicSmemBytes = F_SMEM_BYTES;
        cfg.stream = st;
        cfg.attrs = &attr;
        cfg.numAttrs = FPAIR == 2 ? 1 : 0;
        if (cudaLaunchKernelEx(&cfg, forward_tracked_kernel, *batch, dev_status) != cudaSuccess ||
            launch_status() != SF_OK)
            rc = SF_ERR_CUDA;
    }
    delete batch;
    return rc;
}
