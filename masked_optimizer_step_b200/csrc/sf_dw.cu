// sf_dw.cu -- row-masked weight gradient dW = dX^T A on the tcgen05 tensor cores.
//
// "Sparse-First Fine-Tuning" (tensorwirelabs.com), section 2.2 (Masked backward pass): a
// projection's weight gradient is dW = dX^T A. Rows are grouped in 32-row tiles; a tile whose
// mask word is zero costs nothing (it is never loaded, multiplied or stored), and rows whose
// bit is clear inside a live tile are dropped when the result is written out.
//
// Shapes: dX is T x R (token-major; column r is weight row r), A is T x C (token-major). In
// GEMM terms M = weight rows, N = columns, K = tokens, and BOTH operands are M/N-contiguous
// ("MN-major"): tcgen05 reads them that way directly, so nothing is transposed in memory.
//
// Work: the mask's ascending active-tile list is cut into M-tiles of four 32-row tiles (128
// rows, gathered from anywhere in the matrix); each M-tile x 256-column N-tile is one unit.
// All-empty tiles never appear in the list, so they cost nothing at all. One persistent launch
// walks the units of every projection of the call (problem-major, so a projection's A stays in
// L2 while its units run).
//
// CTA (1 per SM, 192 threads, warp-specialised):
//   warp 0      TMA producer: per 64-token stage, four 32-row boxes of dX (SWIZZLE_64B) and
//               four 64-column boxes of A (SWIZZLE_128B) into a 4-deep shared-memory ring;
//   warp 1      allocates 512 TMEM columns, one thread issues tcgen05.mma kind::f16
//               (M=128, N=256, K=16, bf16 in, fp32 accumulate) into one of two 256-column
//               accumulators, and commits stage releases / accumulator-ready to mbarriers;
//   warps 2-5   epilogue: tcgen05.ld 32 lanes x 32 columns at a time (warp w reads TMEM lanes
//               32*(w%4)..), tests each row's mask bit and slot, stores fp32 rows of dW.
// The two accumulators let the epilogue of one unit overlap the main loop of the next.
// Every mbarrier wait is bounded (2 s): on expiry the CTA raises SF_STATUS_WAIT_TIMEOUT, drains
// its own TMA loads, frees its TMEM and exits.
#include "sf_common.cuh"
#include "sf_host.h"

namespace sf {
namespace {

constexpr int BM = 128;                 // rows per unit: four 32-row mask tiles
constexpr int BN = 256;                 // columns per unit
constexpr int BK = 64;                  // tokens per pipeline stage
constexpr int UMMA_K = 16;              // K of one tcgen05.mma kind::f16
constexpr int STAGES = 4;
constexpr int A_TILE_BYTES = 32 * BK * 2;          // one 32-row tile x 64 tokens (64 B rows)
constexpr int A_STAGE_BYTES = 4 * A_TILE_BYTES;    // 16 KB
constexpr int B_BOX_BYTES = 64 * BK * 2;           // 64 columns x 64 tokens (128 B rows)
constexpr int B_STAGE_BYTES = (BN / 64) * B_BOX_BYTES;   // 32 KB
constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr int TMEM_COLS = 2 * BN;       // two accumulators
constexpr int kThreads = 192;
constexpr int kMaxProblems = SF_DW_MAX_PER_LAUNCH;
constexpr size_t kSmemBytes = (size_t)STAGES * STAGE_BYTES + 1024;   // + alignment slack

struct alignas(64) DwDesc {
    CUtensorMap tm_dx;           // dims {R, T}, box {32, 64}, 64-byte swizzle
    CUtensorMap tm_a;            // dims {C, T}, box {64, 64}, 128-byte swizzle
    const uint32_t *words;
    const int32_t *active_tiles;
    const int32_t *counts;
    const int32_t *row_slot;
    float *dW;
    int64_t ld_dw;
    int32_t R, C, T, n_ntiles;
};

struct DwBatch {
    int32_t n;
    DwDesc d[kMaxProblems];
};
static_assert(sizeof(DwBatch) < 32000, "kernel parameter space");

// Shared-memory matrix descriptor (tcgen05 "matrix descriptor"): start address, leading and
// stride byte offsets (16-byte units), version 1, swizzle mode in bits 61..63.
//   MN-major + swizzle: LBO = distance between successive swizzle-width chunks along M/N,
//                       SBO = distance between successive groups of 8 rows along K.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout)
{
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}
constexpr uint32_t kLayoutSW128 = 2;
constexpr uint32_t kLayoutSW64 = 4;

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both MN-major, N, M.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                            ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

struct Unit {
    int p, mt, nt;
};

__device__ __forceinline__ Unit decode(int u, const int *prefix, int n, const DwBatch &b)
{
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= u) lo = mid; else hi = mid - 1;
    }
    const int local = u - prefix[lo];
    Unit x;
    x.p = lo;
    x.mt = local / b.d[lo].n_ntiles;
    x.nt = local - x.mt * b.d[lo].n_ntiles;
    return x;
}

__global__ void __launch_bounds__(kThreads, 1)
masked_dw_kernel(const __grid_constant__ DwBatch b, uint32_t *status)
{
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full_bar[STAGES], empty_bar[STAGES], tfull_bar[2], tempty_bar[2], drain_bar;
    __shared__ uint32_t tmem_base_s;
    __shared__ int prefix[kMaxProblems + 1];
    __shared__ int scan_scratch[33];
    __shared__ volatile int abort_flag;

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    {   // units per problem: ceil(active tiles / 4) M-tiles x N-tiles
        int units = 0;
        if (tid < b.n) units = ((b.d[tid].counts[1] + 3) >> 2) * b.d[tid].n_ntiles;
        int total;
        const int off = block_exclusive_scan(units, scan_scratch, &total);
        if (tid < b.n) prefix[tid] = off;
        if (tid == 0) prefix[b.n] = total;
    }
    if (tid == 0) {
        abort_flag = 0;
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull_bar[a], 1);
            mbar_init(&tempty_bar[a], 4);
        }
        mbar_init(&drain_bar, 1);
        fence_mbarrier_init();
    }
    if (warp == 1) tmem_alloc(&tmem_base_s, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_s;
    const int total_units = prefix[b.n];

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            for (int i = 0; i < b.n; ++i) {
                prefetch_tmap(&b.d[i].tm_dx);
                prefetch_tmap(&b.d[i].tm_a);
            }
            int stage = 0;
            uint32_t phase = 0;
            bool issued[STAGES] = {false, false, false, false};
            uint32_t issued_parity[STAGES] = {0, 0, 0, 0};
            bool ok = true;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
                const Unit x = decode(u, prefix, b.n, b);
                const DwDesc &d = b.d[x.p];
                const int nk = (d.T + BK - 1) / BK;
                const int n_tiles = d.counts[1];
                int tile[4];
                int nvalid = 0;
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const int idx = x.mt * 4 + s;
                    tile[s] = idx < n_tiles ? d.active_tiles[idx] : -1;
                    nvalid += tile[s] >= 0;
                }
                const uint32_t bytes = nvalid * A_TILE_BYTES + B_STAGE_BYTES;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag)) { ok = false; break; }
                    uint8_t *sa = smem + stage * STAGE_BYTES;
                    uint8_t *sb = sa + A_STAGE_BYTES;
                    mbar_arrive_expect_tx(&full_bar[stage], bytes);
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        if (tile[s] >= 0)
                            tma_load_2d(sa + s * A_TILE_BYTES, &d.tm_dx, &full_bar[stage], tile[s] * 32, kb * BK);
#pragma unroll
                    for (int j = 0; j < BN / 64; ++j)
                        tma_load_2d(sb + j * B_BOX_BYTES, &d.tm_a, &full_bar[stage], x.nt * BN + j * 64, kb * BK);
                    issued[stage] = true;
                    issued_parity[stage] = phase;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok || abort_flag) {
                // drain this CTA's own loads before the shared memory goes away
                for (int s = 0; s < STAGES; ++s) {
                    if (!issued[s]) continue;
                    const uint64_t t0 = globaltimer_ns();
                    while (!mbar_try_wait(&full_bar[s], issued_parity[s]) &&
                           globaltimer_ns() - t0 < kWaitLimitNs) {}
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
                const Unit x = decode(u, prefix, b.n, b);
                const int nk = (b.d[x.p].T + BK - 1) / BK;
                if (nk == 0) continue;
                if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, &abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&full_bar[stage], phase, &abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_STAGE_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        // 16 tokens = 16 rows of 64 B (A) or 128 B (B)
                        const uint64_t da = smem_desc(sa + k * UMMA_K * 64, A_TILE_BYTES, 8 * 64, kLayoutSW64);
                        const uint64_t db = smem_desc(sb + k * UMMA_K * 128, B_BOX_BYTES, 8 * 128, kLayoutSW128);
                        mma_bf16(d_tmem, da, db, kIdesc, (kb | k) != 0);
                    }
                    mma_commit(&empty_bar[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma_commit(&tfull_bar[acc]);
                if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
            }
            // every MMA this thread issued has finished before TMEM is released
            mma_commit(&drain_bar);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&drain_bar, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {}
        }
    } else {
        // ------------------------------ epilogue (warps 2..5) ------------------------------
        const int quad = warp & 3;              // TMEM lanes 32*quad .. 32*quad+31
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
            const Unit x = decode(u, prefix, b.n, b);
            const DwDesc &d = b.d[x.p];
            const int nk = (d.T + BK - 1) / BK;
            const int idx = x.mt * 4 + quad;
            int slot = -1;
            if (idx < d.counts[1]) {
                const int tile = d.active_tiles[idx];
                if ((d.words[tile] >> lane) & 1u) slot = d.row_slot[tile * 32 + lane];
            }
            const int col_base = x.nt * BN;
            float *out = slot >= 0 ? d.dW + (size_t)slot * d.ld_dw : nullptr;
            if (nk == 0) {                      // no tokens: the gradient is zero
                if (out)
                    for (int c = col_base; c < min(d.C, col_base + BN); c += 4)
                        *reinterpret_cast<float4 *>(out + c) = make_float4(0.f, 0.f, 0.f, 0.f);
                continue;
            }
            // every lane waits; the outcome is made warp-uniform before the aligned TMEM loads
            const bool ready = __all_sync(0xffffffffu, mbar_wait(&tfull_bar[acc], acc_phase, &abort_flag));
            if (!ready) break;
            tc_fence_after();
            const uint32_t t_row = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(t_row + cc * 32, v);
                tmem_ld_wait();
                const int c0 = col_base + cc * 32;
                if (out && c0 < d.C) {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (c0 + 4 * j < d.C)
                            *reinterpret_cast<float4 *>(out + c0 + 4 * j) =
                                make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                            __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty_bar[acc]);
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
    }

    __syncwarp();                       // lanes 1..31 of the producer and MMA warps rejoin lane 0
    tc_fence_before();
    __syncthreads();
    if (abort_flag && tid == 0) set_status(status, SF_STATUS_WAIT_TIMEOUT);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ------------------------------------ host side ------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
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

// bf16 2-D map over a token-major matrix [rows_T x ld], `width` valid columns, box {bx, 64}.
bool encode_bf16(CUtensorMap *m, const void *base, int width, int T, int64_t ld, int bx,
                 CUtensorMapSwizzle sw)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)width, (cuuint64_t)(T > 0 ? T : 1)};
    const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    const cuuint32_t box[2] = {(cuuint32_t)bx, (cuuint32_t)BK};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace sf

using namespace sf;

extern "C" int sf_masked_dw(const sf_dw_problem *probs, int n, uint32_t *dev_status, sf_stream stream)
{
    if (n < 0 || (n > 0 && !probs)) return SF_ERR_ARG;
    for (int i = 0; i < n; ++i) {
        const sf_dw_problem &p = probs[i];
        int rc = check_mask(p.mask);
        if (rc != SF_OK) return rc;
        if (p.T < 0 || p.C <= 0 || (p.C & 7) || !p.dW) return SF_ERR_ARG;
        if (p.ld_dw < p.C) return SF_ERR_ARG;
        if ((p.ld_dw & 3) || !aligned16(p.dW)) return SF_ERR_ALIGN;
        if (p.T > 0) {                       // dX and A are read only when there are tokens
            if (!p.dX || !p.A || p.ld_dx < p.mask.R || p.ld_a < p.C) return SF_ERR_ARG;
            if ((p.ld_dx & 7) || (p.ld_a & 7) || !aligned16(p.dX) || !aligned16(p.A)) return SF_ERR_ALIGN;
        }
    }
    if (n == 0) return SF_OK;
    const int sms = sm_count();
    if (sms <= 0) return SF_ERR_NO_DEVICE;
    cudaStream_t st = as_stream(stream);
    if (cudaFuncSetAttribute(masked_dw_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes) != cudaSuccess)
        return SF_ERR_CUDA;
    for (int first = 0; first < n; first += kMaxProblems) {
        const int cnt = n - first < kMaxProblems ? n - first : kMaxProblems;
        DwBatch batch;
        memset(&batch, 0, sizeof(batch));
        batch.n = cnt;
        long long max_units = 0;
        for (int j = 0; j < cnt; ++j) {
            const sf_dw_problem &p = probs[first + j];
            DwDesc &d = batch.d[j];
            const void *dx = p.T > 0 ? p.dX : p.dW;     // any valid address when there are no tokens
            const void *a = p.T > 0 ? p.A : p.dW;
            if (!encode_bf16(&d.tm_dx, dx, p.mask.R, p.T, p.T > 0 ? p.ld_dx : p.mask.R, 32,
                             CU_TENSOR_MAP_SWIZZLE_64B) ||
                !encode_bf16(&d.tm_a, a, p.C, p.T, p.T > 0 ? p.ld_a : p.C, 64,
                             CU_TENSOR_MAP_SWIZZLE_128B))
                return SF_ERR_CUDA;
            d.words = p.mask.words;
            d.active_tiles = p.mask.active_tiles;
            d.counts = p.mask.counts;
            d.row_slot = p.mask.row_slot;
            d.dW = p.dW;
            d.ld_dw = p.ld_dw;
            d.R = p.mask.R;
            d.C = p.C;
            d.T = p.T;
            d.n_ntiles = (p.C + BN - 1) / BN;
            max_units += (long long)((p.mask.R / 32 + 3) / 4) * d.n_ntiles;
        }
        const int grid = (int)(max_units < sms ? max_units : sms);
        masked_dw_kernel<<<grid, kThreads, kSmemBytes, st>>>(batch, dev_status);
        if (launch_status() != SF_OK) return SF_ERR_CUDA;
    }
    return SF_OK;
}
