// sf_dw.cu -- row-masked weight gradient dW = dX^T A on the tcgen05 tensor cores.
//
// "Sparse-First Fine-Tuning" (tensorwirelabs.com), section 2.2 (Masked backward pass): a
// projection's weight gradient is dW = dX^T A. Rows are grouped in 32-row tiles; a tile whose
// mask word is zero costs nothing (it is never loaded, multiplied or stored), and rows whose
// bit is clear inside a live tile are dropped when the result is written out.
//
// Shapes: dX is T x R (token-major; column r is weight row r), A is T x C (token-major). In
// GEMM terms M = weight rows, N = columns, K = tokens. A (the B operand) is read in place,
// N-contiguous ("MN-major"); tile mode reads dX's tiles in place too (M-contiguous), while row
// mode's gather stores each gathered row's tokens contiguously (K-major). tcgen05 reads both
// layouts directly, so nothing else is transposed.
//
// Groups. Consecutive problems of a call that read the same A (same pointer, stride, C and T --
// e.g. the q, k and v projections of a layer, or gate and up) form a group: their rows share
// M-tiles and A is streamed once per group. Each group runs in one of two modes, chosen on the
// device from the live masks (no host readback):
//   tile mode  the pages' design: the ascending list of active 32-row tiles of each problem is
//              cut into 128-row M-tiles of four tiles, gathered straight from dX by TMA; rows of
//              a live tile that are inactive are computed and dropped at the store.
//   row mode   a gather kernel first copies just the active rows of every problem of the group
//              into a dense buffer (caller scratch; each row's tokens contiguous), so an M-tile
//              holds 128 active rows instead of four tiles. Same result; far fewer tensor-core FLOPs when rows are
//              scattered (at 1% scattered rows, a live tile holds ~1.2 active rows).
// Row mode is used when the group's active rows fit the scratch and it needs fewer M-tiles.
//
// CTA (1 per SM, 320 threads, warp-specialised, persistent over the units of the launch):
//   warp 0      TMA producer: per 64-token stage, the A-operand -- four 32-row boxes of dX
//               (tile mode, SWIZZLE_64B) or up to four {64 tokens, 32 rows} boxes of the
//               gathered rows, only those holding rows (row mode, SWIZZLE_128B) -- and the
//               stage's four 64-column chunks of A in one 3-D box (SWIZZLE_128B), into a 4-deep
//               ring;
//   warp 1      allocates 512 TMEM columns, one thread issues tcgen05.mma kind::f16
//               (M=128, N=256, K=16, bf16 in, fp32 accumulate). Each chunk of 1024 tokens goes
//               into one of two 256-column TMEM buffers, starting from zero; the thread commits
//               stage releases and chunk-ready signals to mbarriers;
//   warps 2-9   epilogue: two warps per TMEM lane quarter (warp w reads lanes 32*(w%4)..), one
//               per 128-column half; each adds every finished chunk into fp32 registers
//               (round to nearest), then maps each lane to its weight row and slot and stores
//               the row of dW once per unit.
// Every mbarrier wait is bounded (2 s): on expiry the CTA raises SF_STATUS_WAIT_TIMEOUT, drains
// its own TMA loads, frees its TMEM and exits.
#include <stdlib.h>
#include <string.h>

#include "sf_common.cuh"
#include "sf_host.h"

namespace sf {
namespace {

constexpr int BM = 128;                 // rows per CTA of a unit (TMEM lanes)
constexpr int BN = 256;                 // columns per unit (one tcgen05.mma N)
#ifndef SF_DW_PAIR
#define SF_DW_PAIR 1
#endif
// CTAs sharing a unit: with 2, a cluster pair runs one tcgen05.mma with cta_group::2 (M = 256):
// each CTA loads its own 128 rows and its own half of the unit's columns (completing on the
// even CTA's barriers), so the shared-memory traffic per FLOP is two thirds of a single CTA's.
// Measured on B200 (parity green in both builds): no faster on dense masks (50% of rows:
// 186 vs 182 us for one 11008 x 4096 projection at 4,096 tokens) and 24% slower on the 7B step's
// scattered 1% masks (0.82 vs 0.66 ms), so one CTA per unit is the default.
constexpr int PAIR = SF_DW_PAIR;
static_assert(PAIR == 1 || PAIR == 2, "one CTA or a CTA pair per unit");
constexpr int UM = BM * PAIR;           // rows per unit
constexpr int UNIT_TILES = UM / 32;     // 32-row mask tiles per unit (tile mode)
constexpr int B_COLS = BN / PAIR;       // columns of the unit each CTA loads
#ifndef SF_DW_BK
#define SF_DW_BK 64
#endif
constexpr int BK = SF_DW_BK;            // tokens per pipeline stage
constexpr int UMMA_K = 16;              // K of one tcgen05.mma kind::f16
static_assert(BK % UMMA_K == 0 && BK <= 256, "stage depth");
#ifndef SF_DW_STAGES
#define SF_DW_STAGES (PAIR == 2 ? 6 : 4)
#endif
constexpr int STAGES = SF_DW_STAGES;
constexpr int A_TILE_BYTES = 32 * BK * 2;          // 32 rows x 64 tokens (64 B rows)
constexpr int A_STAGE_BYTES = 4 * A_TILE_BYTES;    // 16 KB
constexpr int B_BOX_BYTES = 64 * BK * 2;           // 64 columns x 64 tokens (128 B rows)
constexpr int B_STAGE_BYTES = (B_COLS / 64) * B_BOX_BYTES;   // 16 KB (pair) or 32 KB
constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
// Accumulation in chunks. The tensor core adds each product block into its fp32 accumulator
// with truncation, so over a long token sum the rounding errors share one sign and grow faster
// than the sum (measured: ~T^1.5, a shrink toward zero). Each chunk of CHUNK tokens is therefore
// summed by the MMAs into a TMEM buffer that starts from zero, and the epilogue adds the
// finished chunks into fp32 registers with round-to-nearest. Two buffers let the MMAs fill one
// while the epilogue drains the other.
#ifndef SF_DW_CHUNK
#define SF_DW_CHUNK 1024
#endif
constexpr int CHUNK_STAGES = SF_DW_CHUNK / BK;     // pipeline stages per accumulation chunk
static_assert(SF_DW_CHUNK % BK == 0 && CHUNK_STAGES >= 1, "chunk of whole stages");
constexpr int NBUF = 2;                 // TMEM chunk buffers
constexpr int TMEM_COLS = NBUF * BN;    // 512: all of the SM's tensor memory (1 CTA per SM)
constexpr int kEpiWarps = 8;            // two per TMEM lane quarter, one per 128-column half
constexpr int kEpiCols = BN / 2;        // running sums per epilogue thread
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr size_t kSmemBytes = (size_t)STAGES * STAGE_BYTES + 1024;   // + alignment slack
constexpr int kMaxPerGroup = 8;
constexpr int kGatherTokens = 32;       // tokens per gather CTA
constexpr int kGatherThreads = 256;

struct alignas(64) DwProb {
    CUtensorMap tm_dx;           // dX: dims {R, T}, box {32, 64}, 64-byte swizzle (tile mode)
    const int32_t *active_tiles;
    const int32_t *counts;
    const int32_t *row_slot;
    float *dW;
    int64_t ld_dw;
};

struct alignas(64) DwGroup {
    // A: when C is a multiple of 64, 3-D {64 columns, T, C / 64 chunks} with box {64, 64,
    // B_COLS / 64}: one load brings the CTA's column chunks of a stage, chunk after chunk (the
    // layout the four 2-D boxes give); otherwise 2-D {C, T}, box {64, 64}. 128-byte swizzle.
    CUtensorMap tm_a;
    // gathered rows, stored row by row (each row's tokens contiguous, stride tp): 2-D {T, mcap},
    // box {64 tokens, 32 rows}, 128-byte swizzle -- a K-major operand, as the tensor cores read
    // fastest; tokens from T to tp are outside the map and read as zeros. A stage loads only the
    // 32-row boxes that hold gathered rows of the CTA's M-tile
    CUtensorMap tm_g;
    const int32_t *info;         // device: [0] mode (1 = rows), [1] gathered rows (null: tiles only)
    const int32_t *rowmap;       // device: per gathered row, (slot << 3) | problem, or -1
    int32_t first, count, C, T, n_ntiles, mcap, a3d;
};

struct DwBatch {
    int32_t n_prob, n_group;
    int32_t withhold_test;       // test hook: CTA 0 arms its first stage but issues no loads
    // variable-length payload: n_group DwGroup then n_prob DwProb
    alignas(64) unsigned char payload[32640];
};
static_assert(sizeof(DwBatch) <= 32764, "kernel parameter space");

// The gather pass has its own, lean parameters (no tensor maps), so one launch covers a call.
struct GatherProb {
    const uint16_t *dx;
    const int32_t *active_rows;
    const int32_t *counts;
    const int32_t *row_slot;
    int64_t ld_dx;
    int32_t R;
};

struct GatherGroup {
    uint16_t *dxg;               // [mcap x tp]: gathered row k holds dX[t, r_k] at dxg[k * tp + t]
    int32_t *info;
    int32_t *rowmap;
    int32_t first, count, T, mcap, tp;
};

constexpr int kMaxGatherGroups = 192;
constexpr int kMaxGatherProbs = 384;

struct GatherBatch {
    int32_t n_group, n_prob;
    GatherGroup g[kMaxGatherGroups];
    GatherProb p[kMaxGatherProbs];
};
static_assert(sizeof(GatherBatch) <= 32764, "kernel parameter space");

__device__ __forceinline__ const DwGroup &grp(const DwBatch &b, int g)
{
    return reinterpret_cast<const DwGroup *>(b.payload)[g];
}
__device__ __forceinline__ const DwProb &prb(const DwBatch &b, int p)
{
    return reinterpret_cast<const DwProb *>(b.payload + (size_t)b.n_group * sizeof(DwGroup))[p];
}

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

// Instruction descriptors, kind::f16: fp32 accumulator, bf16 A and B, N, M. Tile mode reads dX
// in place, so both operands are MN-major (bits 15, 16); row mode's gathered rows are K-major.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                            ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(UM >> 4) << 24);
constexpr uint32_t kIdescRows = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(UM >> 4) << 24);

// K-major, 128-byte swizzle: rows of 128 bytes (64 tokens), 8-row groups 1024 bytes apart; the
// leading offset is unused for this layout.
__device__ __forceinline__ uint64_t kmajor_sw128_desc(uint32_t addr)
{
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
           (1ull << 46) | ((uint64_t)2u << 61);
}

// Row mode when the group's active rows fit the scratch and need fewer units than the mask
// tiles do. Every reader computes the same answer from the same counts.
__device__ __forceinline__ bool choose_rows(int rows, int tiles_mt, int mcap)
{
    return mcap > 0 && rows <= mcap && (rows + UM - 1) / UM < tiles_mt;
}

// ------------------------------------ gather kernel ------------------------------------
// Row mode: dxg[k, t] = dX_p[t, r] for the group's k-th active row r (problems in call order,
// rows ascending; each gathered row's tokens contiguous), and rowmap[k] = (slot(r) << 3) | p. One CTA per (group, 32 tokens); a thread
// takes a gathered row and issues its 32 token loads back to back. The reads are single
// elements spread over dX: each one costs the DRAM fetch of the line around it, so in a group
// with fewer than one active row in 16 the loads ask L2 for 64-byte fetches instead of the
// default 128 bytes (measured on the 7B step's layout at 1%: ~57 instead of ~99 DRAM bytes per
// gathered element, the pass ~30% faster); denser groups use whole lines, which they need
// anyway (64-byte fetches measured ~3x slower at 50%). Many small independent loads per thread
// keep enough requests in flight.
// A thread writes its row's 32 tokens as 64 contiguous bytes. The first CTA of a group records
// the mode and the row map, which the main kernel (next on the stream) reads.
__global__ void __launch_bounds__(kGatherThreads)
dw_gather_kernel(const __grid_constant__ GatherBatch b, int blocks_per_group)
{
    const int gi = blockIdx.x / blocks_per_group;
    const int tb = blockIdx.x - gi * blocks_per_group;
    const GatherGroup &g = b.g[gi];
    __shared__ int row_pre[kMaxPerGroup + 1];
    __shared__ int s_rows_mode, s_sparse;
    if (threadIdx.x == 0) {
        int rows = 0, tiles_mt = 0;
        long long all_rows = 0;
        for (int k = 0; k < g.count; ++k) {
            const GatherProb &p = b.p[g.first + k];
            row_pre[k] = rows;
            rows += p.counts[0];
            tiles_mt += (p.counts[1] + UNIT_TILES - 1) / UNIT_TILES;
            all_rows += p.R;
        }
        row_pre[g.count] = rows;
        s_rows_mode = choose_rows(rows, tiles_mt, g.mcap);
        s_sparse = 16LL * rows < all_rows;             // fewer than 1 row in 16 active
        if (tb == 0) {
            g.info[0] = s_rows_mode;
            g.info[1] = rows;
        }
    }
    __syncthreads();
    if (!s_rows_mode) return;
    const int t0 = tb * kGatherTokens;
    const int nt = min(g.T - t0, kGatherTokens);
    const int rows = row_pre[g.count];
    for (int k = threadIdx.x; k < rows; k += kGatherThreads) {
        int q = 0;
        while (q + 1 < g.count && row_pre[q + 1] <= k) ++q;
        const GatherProb &p = b.p[g.first + q];
        const int r = p.active_rows[k - row_pre[q]];
        if (tb == 0) {
            const int slot = p.row_slot[r];
            g.rowmap[k] = slot >= 0 ? (slot << 3) | q : -1;
        }
        if (nt <= 0) continue;
        const uint16_t *src = p.dx + (size_t)t0 * p.ld_dx + r;
        uint16_t *dst = g.dxg + (size_t)k * g.tp + t0;
        uint16_t v[kGatherTokens];
        if (s_sparse) {
#pragma unroll
            for (int t = 0; t < kGatherTokens; ++t)
                if (t < nt) v[t] = ld_nc_l2_64b_u16(src + (size_t)t * p.ld_dx);
        } else {
#pragma unroll
            for (int t = 0; t < kGatherTokens; ++t)
                if (t < nt) v[t] = __ldcs(src + (size_t)t * p.ld_dx);
        }
        if (nt == kGatherTokens) {            // t0 is a multiple of 32 and tp of 8: 16-byte aligned
#pragma unroll
            for (int q4 = 0; q4 < kGatherTokens / 8; ++q4) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) w[e] = (uint32_t)v[8 * q4 + 2 * e] | ((uint32_t)v[8 * q4 + 2 * e + 1] << 16);
                *reinterpret_cast<uint4 *>(dst + 8 * q4) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        } else {
#pragma unroll
            for (int t = 0; t < kGatherTokens; ++t)
                if (t < nt) dst[t] = v[t];
        }
    }
}

// ------------------------------------ unit decoding ------------------------------------

struct Unit {
    int g;          // group
    int mt;         // M-tile within the group (row mode) or within problem p (tile mode)
    int nt;         // N-tile
    int p;          // problem (tile mode), -1 in row mode
    int rows_mode;
};

struct SmemPlan {
    int unit_prefix[SF_DW_MAX_PER_LAUNCH + 1];     // per group
    int rows_mode[SF_DW_MAX_PER_LAUNCH];
    int mt_prefix[SF_DW_MAX_PER_LAUNCH + 1];       // per problem: M-tiles before it in its group
};

__device__ __forceinline__ Unit decode(int u, const SmemPlan &sp, const DwBatch &b)
{
    int lo = 0, hi = b.n_group - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sp.unit_prefix[mid] <= u) lo = mid; else hi = mid - 1;
    }
    const DwGroup &g = grp(b, lo);
    const int local = u - sp.unit_prefix[lo];
    Unit x;
    x.g = lo;
    x.rows_mode = sp.rows_mode[lo];
    const int mt = local / g.n_ntiles;
    x.nt = local - mt * g.n_ntiles;
    if (x.rows_mode) {
        x.mt = mt;
        x.p = -1;
    } else {
        int p = g.first;
        while (p + 1 < g.first + g.count && sp.mt_prefix[p + 1] <= mt) ++p;
        x.p = p;
        x.mt = mt - sp.mt_prefix[p];
    }
    return x;
}

// ------------------------------------ main kernel ------------------------------------

__global__ void __launch_bounds__(kThreads, 1)
masked_dw_kernel(const __grid_constant__ DwBatch b, uint32_t *status)
{
    // CTA pairs: the even CTA of a cluster (the leader) issues the MMAs of both and owns the
    // stage barriers; the odd one loads its halves (completing on the leader's barriers) and
    // drains its own TMEM lanes.
    const uint32_t crank = PAIR == 2 ? cluster_ctarank() : 0u;
    const bool leader = crank == 0;
    const int unit0 = blockIdx.x / PAIR, ustep = gridDim.x / PAIR;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full_bar[STAGES], empty_bar[STAGES], tfull_bar[NBUF], tempty_bar[NBUF], drain_bar;
    __shared__ uint32_t tmem_base_s;
    __shared__ SmemPlan sp;
    __shared__ int scan_scratch[33];
    __shared__ volatile int abort_flag;

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // The launches of one call write disjoint problems, so the next one may take SMs as soon as
    // this one's CTAs drain (its CTAs cannot share an SM with these: shared memory). Every launch
    // reads only what the gather pass and the masks left, which were complete before the first
    // launch of the call started.
    griddep_launch_dependents();

    {   // per group: mode and units; per problem: M-tiles before it inside its group
        int units = 0;
        if (tid < b.n_group) {
            const DwGroup &g = grp(b, tid);
            int acc = 0;
            for (int k = 0; k < g.count; ++k) {
                sp.mt_prefix[g.first + k] = acc;
                acc += (prb(b, g.first + k).counts[1] + UNIT_TILES - 1) / UNIT_TILES;
            }
            const int rows_mode = g.info != nullptr && g.info[0] != 0;
            sp.rows_mode[tid] = rows_mode;
            units = (rows_mode ? (g.info[1] + UM - 1) / UM : acc) * g.n_ntiles;
        }
        int total;
        const int off = block_exclusive_scan(units, scan_scratch, &total);
        if (tid < b.n_group) sp.unit_prefix[tid] = off;
        if (tid == 0) sp.unit_prefix[b.n_group] = total;
    }
    if (tid == 0) {
        abort_flag = 0;
        for (int s = 0; s < STAGES; ++s) {
            // in a pair only the leader's full barriers are used: both CTAs' loads complete on them
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < NBUF; ++a) {
            mbar_init(&tfull_bar[a], 1);
            mbar_init(&tempty_bar[a], kEpiWarps * PAIR);    // the leader's counts both CTAs' warps
        }
        mbar_init(&drain_bar, 1);
        fence_mbarrier_init();
    }
    if (warp == 1) {
        if (PAIR == 2) tmem_alloc_pair(&tmem_base_s, TMEM_COLS);
        else tmem_alloc(&tmem_base_s, TMEM_COLS);
    }
    tc_fence_before();
    __syncthreads();
    if (PAIR == 2) cluster_sync();            // both CTAs' barriers exist before either uses them
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_s;
    const int total_units = sp.unit_prefix[b.n_group];

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            for (int i = 0; i < b.n_group; ++i) {
                prefetch_tmap(&grp(b, i).tm_a);
                if (sp.rows_mode[i]) prefetch_tmap(&grp(b, i).tm_g);
            }
            int stage = 0;
            uint32_t phase = 0;
            bool issued[STAGES] = {};
            uint32_t issued_parity[STAGES] = {};
            bool ok = true;
            for (int u = unit0; u < total_units && ok; u += ustep) {
                const Unit x = decode(u, sp, b);
                const DwGroup &g = grp(b, x.g);
                const int nk = (g.T + BK - 1) / BK;
                const CUtensorMap *tm_rows;
                int coord[4];
                int nvalid = 0;
                if (x.rows_mode) {
                    // K-major 32-row boxes of the CTA's gathered rows, as many as hold rows: the
                    // MMA also reads the rest of the 128-row operand (whatever an earlier stage
                    // left), which only feeds accumulator rows the epilogue discards
                    tm_rows = &g.tm_g;
                    const int r0 = x.mt * UM + (int)crank * BM;
                    const int n_here = min(BM, max(0, g.info[1] - r0));
#pragma unroll
                    for (int s = 0; s < 4; ++s) coord[s] = 32 * s < n_here ? r0 + 32 * s : -1;
                    nvalid = (n_here + 31) / 32;
                } else {
                    const DwProb &p = prb(b, x.p);
                    tm_rows = &p.tm_dx;
                    const int n_tiles = p.counts[1];
#pragma unroll
                    for (int s = 0; s < 4; ++s) {
                        const int idx = x.mt * UNIT_TILES + (int)crank * 4 + s;
                        coord[s] = idx < n_tiles ? p.active_tiles[idx] * 32 : -1;
                        nvalid += coord[s] >= 0;
                    }
                }
                // the leader's barrier counts both CTAs' bytes: the peer's boxes are the next four
                // tiles (or gathered rows) of the unit
                int nvalid_peer = 0;
                if (PAIR == 2 && leader) {
#pragma unroll
                    for (int s = 0; s < 4; ++s) {
                        if (x.rows_mode) nvalid_peer += x.mt * UM + BM + 32 * s < g.info[1];
                        else nvalid_peer += x.mt * UNIT_TILES + 4 + s < prb(b, x.p).counts[1];
                    }
                }
                const uint32_t bytes = (nvalid + nvalid_peer) * A_TILE_BYTES + PAIR * B_STAGE_BYTES;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag)) { ok = false; break; }
                    uint8_t *sa = smem + stage * STAGE_BYTES;
                    uint8_t *sb = sa + A_STAGE_BYTES;
                    if (leader) mbar_arrive_expect_tx(&full_bar[stage], PAIR == 2 ? bytes : nvalid * A_TILE_BYTES + B_STAGE_BYTES);
                    // test hook (failure detection): the stage's bytes never arrive, so the MMA
                    // issuer's bounded wait runs out and the CTA unwinds with WAIT_TIMEOUT
                    const bool withhold = b.withhold_test && blockIdx.x == 0 && u == unit0 && kb == 0;
                    if (!withhold) {
                        if (x.rows_mode) {
#pragma unroll
                            for (int s = 0; s < 4; ++s)
                                if (coord[s] >= 0) {
                                    if (PAIR == 2) tma_load_2d_pair(sa + s * A_TILE_BYTES, tm_rows, &full_bar[stage], kb * BK, coord[s]);
                                    else tma_load_2d(sa + s * A_TILE_BYTES, tm_rows, &full_bar[stage], kb * BK, coord[s]);
                                }
                        } else {
#pragma unroll
                            for (int s = 0; s < 4; ++s)
                                if (coord[s] >= 0) {
                                    if (PAIR == 2) tma_load_2d_pair(sa + s * A_TILE_BYTES, tm_rows, &full_bar[stage], coord[s], kb * BK);
                                    else tma_load_2d(sa + s * A_TILE_BYTES, tm_rows, &full_bar[stage], coord[s], kb * BK);
                                }
                        }
                        if (g.a3d) {                      // the CTA's column chunks in one load
                            const int chunk = (x.nt * BN + (int)crank * B_COLS) / 64;
                            if (PAIR == 2) tma_load_3d_pair(sb, &g.tm_a, &full_bar[stage], 0, kb * BK, chunk);
                            else tma_load_3d(sb, &g.tm_a, &full_bar[stage], 0, kb * BK, chunk);
                        } else {
#pragma unroll
                            for (int j = 0; j < B_COLS / 64; ++j) {
                                const int col = x.nt * BN + (int)crank * B_COLS + j * 64;
                                if (PAIR == 2) tma_load_2d_pair(sb + j * B_BOX_BYTES, &g.tm_a, &full_bar[stage], col, kb * BK);
                                else tma_load_2d(sb + j * B_BOX_BYTES, &g.tm_a, &full_bar[stage], col, kb * BK);
                            }
                        }
                    }
                    issued[stage] = true;
                    issued_parity[stage] = phase;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            {   // the MMA issuer commits drain_bar once it has finished or given up; only then is
                // abort_flag final for this CTA
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&drain_bar, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {}
            }
            if ((!ok || abort_flag) && leader) {
                // drain the loads armed on this CTA's barriers before the shared memory goes away
                // (in a pair both CTAs' loads complete on the leader's barriers)
                for (int s = 0; s < STAGES; ++s) {
                    if (!issued[s]) continue;
                    const uint64_t t0 = globaltimer_ns();
                    while (!mbar_try_wait(&full_bar[s], issued_parity[s]) &&
                           globaltimer_ns() - t0 < kWaitLimitNs) {}
                }
            }
        }
    } else if (warp == 1 && PAIR == 2 && !leader) {
        // the odd CTA of a pair issues no MMAs: the leader's thread issues them for both
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t buf_phase = 0;
            bool ok = true;
            for (int u = unit0; u < total_units && ok; u += ustep) {
                const Unit x = decode(u, sp, b);
                const int nk = (grp(b, x.g).T + BK - 1) / BK;
                const uint32_t idesc = x.rows_mode ? kIdescRows : kIdesc;
                for (int kb = 0; kb < nk; ++kb) {
                    const int in_chunk = kb % CHUNK_STAGES;
                    if (in_chunk == 0) {             // a fresh chunk: wait until its buffer is drained
                        if (!mbar_wait(&tempty_bar[buf], buf_phase ^ 1u, &abort_flag)) { ok = false; break; }
                        tc_fence_after();
                    }
                    if (!mbar_wait(&full_bar[stage], phase, &abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_STAGE_BYTES;
                    const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        // 16 tokens: 32 bytes into each K-major row (row mode), or 16 rows of 64 B
                        // (tile mode's A-operand) and of 128 B (the B-operand)
                        const uint64_t da = x.rows_mode
                            ? kmajor_sw128_desc(sa + k * UMMA_K * 2)
                            : smem_desc(sa + k * UMMA_K * 64, A_TILE_BYTES, 8 * 64, kLayoutSW64);
                        const uint64_t db = smem_desc(sb + k * UMMA_K * 128, B_BOX_BYTES, 8 * 128, kLayoutSW128);
                        if (PAIR == 2) mma_bf16_pair(d_tmem, da, db, idesc, (in_chunk | k) != 0);
                        else mma_bf16(d_tmem, da, db, idesc, (in_chunk | k) != 0);
                    }
                    if (PAIR == 2) mma_commit_pair(&empty_bar[stage], 3);   // both CTAs' stages free
                    else mma_commit(&empty_bar[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                    if (in_chunk == CHUNK_STAGES - 1 || kb == nk - 1) {   // chunk complete
                        if (PAIR == 2) mma_commit_pair(&tfull_bar[buf], 3);
                        else mma_commit(&tfull_bar[buf]);
                        if (++buf == NBUF) { buf = 0; buf_phase ^= 1u; }
                    }
                }
            }
            // every MMA this thread issued has finished before TMEM is released
            if (PAIR == 2) mma_commit_pair(&drain_bar, 3);
            else mma_commit(&drain_bar);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&drain_bar, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {}
        }
    } else {
        // --------------------------- epilogue (warps 2..2+kEpiWarps-1) ---------------------------
        // A warp may only read the TMEM lane quarter warp_id % 4; two warps share each quarter,
        // one per 128-column half of the unit.
        const int quad = warp & 3;              // TMEM lanes 32*quad .. 32*quad+31
        const int half = (warp - 2) >> 2;       // columns half*128 .. half*128+127 of the unit
        int buf = 0;
        uint32_t buf_phase = 0;
        for (int u = unit0; u < total_units; u += ustep) {
            const Unit x = decode(u, sp, b);
            const DwGroup &g = grp(b, x.g);
            const int nk = (g.T + BK - 1) / BK;
            // the weight row of this lane's accumulator row, its slot and its output
            int slot = -1;
            const DwProb *p = nullptr;
            if (x.rows_mode) {
                const int k = x.mt * UM + (int)crank * BM + quad * 32 + lane;
                if (k < g.info[1]) {
                    const int e = g.rowmap[k];
                    if (e >= 0) {
                        p = &prb(b, g.first + (e & 7));
                        slot = e >> 3;
                    }
                }
            } else {
                p = &prb(b, x.p);
                const int idx = x.mt * UNIT_TILES + (int)crank * 4 + quad;
                if (idx < p->counts[1]) slot = p->row_slot[p->active_tiles[idx] * 32 + lane];
            }
            const int col_base = x.nt * BN + half * kEpiCols;
            float *out = slot >= 0 ? p->dW + (size_t)slot * p->ld_dw : nullptr;
            float acc[kEpiCols];
#pragma unroll
            for (int j = 0; j < kEpiCols; ++j) acc[j] = 0.0f;
            bool ready = true;
            const int nchunks = (nk + CHUNK_STAGES - 1) / CHUNK_STAGES;
            for (int ch = 0; ch < nchunks; ++ch) {
                // every lane waits; the outcome is made warp-uniform before the aligned TMEM loads
                ready = __all_sync(0xffffffffu, mbar_wait(&tfull_bar[buf], buf_phase, &abort_flag));
                if (!ready) break;
                tc_fence_after();
                const uint32_t t_row = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * BN + half * kEpiCols);
#pragma unroll
                for (int cc = 0; cc < kEpiCols / 32; ++cc) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(t_row + cc * 32, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) acc[cc * 32 + j] = __fadd_rn(acc[cc * 32 + j], __uint_as_float(v[j]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {                 // the leader's MMAs may refill the buffer
                    if (PAIR == 2 && !leader) mbar_arrive_remote(&tempty_bar[buf], 0);
                    else mbar_arrive(&tempty_bar[buf]);
                }
                if (++buf == NBUF) { buf = 0; buf_phase ^= 1u; }
            }
            if (!ready) break;
            if (out) {                          // no tokens: the sums stay zero, the gradient is zero
#pragma unroll
                for (int j = 0; j < kEpiCols / 4; ++j)
                    if (col_base + 4 * j < g.C)
                        *reinterpret_cast<float4 *>(out + col_base + 4 * j) =
                            make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
            }
        }
    }

    __syncwarp();                       // lanes 1..31 of the producer and MMA warps rejoin lane 0
    tc_fence_before();
    __syncthreads();
    if (PAIR == 2) cluster_sync();            // neither CTA leaves while the pair's MMAs may run
    if (abort_flag && tid == 0) set_status(status, SF_STATUS_WAIT_TIMEOUT);
    if (warp == 1) {
        tc_fence_after();
        if (PAIR == 2) tmem_dealloc_pair(tmem_base, TMEM_COLS);
        else tmem_dealloc(tmem_base, TMEM_COLS);
    }
    // Complete only after the launch before this one has: whatever the stream runs next then
    // sees every launch of the call finished.
    griddep_wait();
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

// bf16 2-D map over a token-major matrix [T x ld], `width` valid columns, box {bx, 64}.
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

// bf16 3-D map over a token-major matrix [T x ld] seen as {inner, T, chunks}: element
// (i, t, k) is base[t * ld + k * inner + i]; box {inner, 64, box_chunks}.
bool encode_bf16_chunks(CUtensorMap *m, const void *base, int inner, int T, int chunks, int64_t ld,
                        int box_chunks, CUtensorMapSwizzle sw)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)(T > 0 ? T : 1), (cuuint64_t)chunks};
    const cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)inner * 2};
    const cuuint32_t box[3] = {(cuuint32_t)inner, (cuuint32_t)BK, (cuuint32_t)box_chunks};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 2-D map over the gathered rows [mcap x tp] (row k's tokens contiguous), valid tokens T:
// box {64 tokens, 128 rows}, 128-byte swizzle (a K-major operand tile).
bool encode_rows_kmajor(CUtensorMap *m, const void *base, int T, int mcap, int64_t tp)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)T, (cuuint64_t)mcap};
    const cuuint64_t strides[1] = {(cuuint64_t)tp * 2};
    const cuuint32_t box[2] = {(cuuint32_t)BK, 32u};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Groups of a call: runs of consecutive problems with the same A, stride, C and T.
struct HostGroup {
    int first, count;
    int mcap;                    // gathered-row capacity (multiple of 32)
    size_t ws_off;               // byte offset of the group's scratch: info, row map, rows
};

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr size_t kInfoBytes = 256;

size_t rowmap_bytes(int mcap) { return round_up((size_t)mcap * sizeof(int32_t), 256); }

int plan_groups(const sf_dw_problem *probs, int n, HostGroup *out, size_t *ws_total)
{
    int ng = 0;
    size_t off = 0;
    for (int i = 0; i < n;) {
        int j = i + 1;
        while (j < n && j - i < kMaxPerGroup && probs[j].A == probs[i].A && probs[j].ld_a == probs[i].ld_a &&
               probs[j].C == probs[i].C && probs[j].T == probs[i].T)
            ++j;
        HostGroup &g = out[ng++];
        g.first = i;
        g.count = j - i;
        size_t cap = 0;
        for (int k = i; k < j; ++k) cap += (size_t)probs[k].mask.slot_cap;
        g.mcap = (int)round_up(cap, 32);
        g.ws_off = off;
        off += kInfoBytes + rowmap_bytes(g.mcap) +
               round_up((size_t)round_up(probs[i].T > 0 ? probs[i].T : 0, 8) * g.mcap * 2, 256);
        i = j;
    }
    *ws_total = off;
    return ng;
}

size_t launch_bytes(const HostGroup &g) { return sizeof(DwGroup) + (size_t)g.count * sizeof(DwProb); }

}  // namespace
}  // namespace sf

using namespace sf;

extern "C" int sf_masked_dw_unit_rows(void) { return UM; }

extern "C" size_t sf_masked_dw_ws_bytes(const sf_dw_problem *probs, int n)
{
    if (n <= 0 || !probs) return 0;
    HostGroup *groups = new HostGroup[n];
    size_t total = 0;
    plan_groups(probs, n, groups, &total);
    delete[] groups;
    return total;
}

extern "C" int sf_masked_dw_phase(const sf_dw_problem *probs, int n, void *ws, size_t ws_bytes, int phase,
                                  uint32_t *dev_status, sf_stream stream)
{
    if (phase != SF_PHASE_ALL && phase != SF_PHASE_FIRST && phase != SF_PHASE_SECOND) return SF_ERR_ARG;
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
        if ((long long)p.mask.slot_cap * 8 > INT32_MAX) return SF_ERR_UNSUPPORTED;   // row map packing
    }
    if (n == 0) return SF_OK;
    // Test hook for the bounded-wait path: with SF_TEST_DW_WITHHOLD set in the environment, the
    // first main launch's CTA 0 withholds one stage of loads (see the producer).
    const char *withhold_env = getenv("SF_TEST_DW_WITHHOLD");
    const int withhold = withhold_env && withhold_env[0] && withhold_env[0] != '0';
    HostGroup *groups = new HostGroup[n];
    size_t need = 0;
    const int ng = plan_groups(probs, n, groups, &need);
    const bool use_ws = ws != nullptr;
    int rc = SF_OK;
    if (use_ws && ws_bytes < need) rc = SF_ERR_ARG;
    else if (use_ws && !aligned16(ws)) rc = SF_ERR_ALIGN;
    const int sms = rc == SF_OK ? sm_count() : 0;
    if (rc == SF_OK && sms <= 0) rc = SF_ERR_NO_DEVICE;
    if (rc == SF_OK && cudaFuncSetAttribute(masked_dw_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            (int)kSmemBytes) != cudaSuccess)
        rc = SF_ERR_CUDA;
    int pair_slots = 0;                       // CTA pairs that can be resident at once
    if (rc == SF_OK && PAIR == 2 && phase != SF_PHASE_FIRST) {
        cudaLaunchConfig_t qcfg = {};
        cudaLaunchAttribute qattr;
        qattr.id = cudaLaunchAttributeClusterDimension;
        qattr.val.clusterDim.x = 2;
        qattr.val.clusterDim.y = 1;
        qattr.val.clusterDim.z = 1;
        qcfg.gridDim = dim3(2 * sms);
        qcfg.blockDim = dim3(kThreads);
        qcfg.dynamicSmemBytes = kSmemBytes;
        qcfg.attrs = &qattr;
        qcfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&pair_slots, masked_dw_kernel, &qcfg) != cudaSuccess || pair_slots <= 0)
            rc = SF_ERR_CUDA;
    }
    cudaStream_t st = as_stream(stream);
    auto scratch = [&](const HostGroup &hg) { return static_cast<uint8_t *>(ws) + hg.ws_off; };
    auto row_ok = [&](const HostGroup &hg) { return use_ws && probs[hg.first].T > 0 && hg.mcap > 0; };

    // ---- gather pass: every group of the call, in as few launches as the parameters allow ----
    GatherBatch *gb = (rc == SF_OK && use_ws && phase != SF_PHASE_SECOND) ? new GatherBatch : nullptr;
    for (int gi = 0; gb && rc == SF_OK && gi < ng;) {
        memset(gb, 0, sizeof(*gb));
        int tok_blocks = 1;
        while (gi < ng && gb->n_group < kMaxGatherGroups && gb->n_prob + groups[gi].count <= kMaxGatherProbs) {
            const HostGroup &hg = groups[gi++];
            if (!row_ok(hg)) continue;
            GatherGroup &g = gb->g[gb->n_group++];
            uint8_t *base = scratch(hg);
            g.info = reinterpret_cast<int32_t *>(base);
            g.rowmap = reinterpret_cast<int32_t *>(base + kInfoBytes);
            g.dxg = reinterpret_cast<uint16_t *>(base + kInfoBytes + rowmap_bytes(hg.mcap));
            g.first = gb->n_prob;
            g.count = hg.count;
            g.T = probs[hg.first].T;
            g.mcap = hg.mcap;
            g.tp = (int)round_up((size_t)g.T, 8);
            tok_blocks = max(tok_blocks, (g.T + kGatherTokens - 1) / kGatherTokens);
            for (int q = 0; q < hg.count; ++q) {
                const sf_dw_problem &p = probs[hg.first + q];
                GatherProb &d = gb->p[gb->n_prob++];
                d.dx = static_cast<const uint16_t *>(p.dX);
                d.active_rows = p.mask.active_rows;
                d.counts = p.mask.counts;
                d.row_slot = p.mask.row_slot;
                d.ld_dx = p.ld_dx;
                d.R = p.mask.R;
            }
        }
        if (gb->n_group > 0) {
            dw_gather_kernel<<<gb->n_group * tok_blocks, kGatherThreads, 0, st>>>(*gb, tok_blocks);
            if (launch_status() != SF_OK) rc = SF_ERR_CUDA;
        }
    }
    delete gb;

    // ---- main pass: groups split over launches so that each launch's parameters fit ----
    const size_t payload = sizeof(DwBatch::payload);
    size_t all = 0;
    for (int k = 0; k < ng; ++k) all += launch_bytes(groups[k]);
    int n_launch = (int)((all + payload - 1) / payload);
    DwBatch *batch = (rc == SF_OK && phase != SF_PHASE_FIRST) ? new DwBatch : nullptr;
    int gi = 0;
    int n_main_launches = 0;
    for (int li = 0; batch && rc == SF_OK && gi < ng; ++li) {
        size_t left = 0;
        for (int k = gi; k < ng; ++k) left += launch_bytes(groups[k]);
        const int launches_left = n_launch - li > 1 ? n_launch - li : 1;
        const size_t target = (left + launches_left - 1) / launches_left;
        int g_end = gi, np = 0;
        size_t used = 0;
        while (g_end < ng) {
            const size_t add = launch_bytes(groups[g_end]);
            if (g_end > gi && (used + add > payload || used >= target)) break;
            if (g_end - gi + 1 > SF_DW_MAX_PER_LAUNCH || np + groups[g_end].count > SF_DW_MAX_PER_LAUNCH) break;
            used += add;
            np += groups[g_end].count;
            ++g_end;
        }
        if (g_end == gi) { rc = SF_ERR_UNSUPPORTED; break; }
        if (g_end < ng && li + 1 >= n_launch) ++n_launch;     // an uneven split needs one more
        memset(batch, 0, sizeof(*batch));
        batch->n_group = g_end - gi;
        batch->withhold_test = withhold && n_main_launches == 0;
        batch->n_prob = np;
        DwGroup *gd = reinterpret_cast<DwGroup *>(batch->payload);
        DwProb *pd = reinterpret_cast<DwProb *>(batch->payload + (size_t)batch->n_group * sizeof(DwGroup));
        long long max_units = 0;
        int pi = 0;
        for (int k = gi; k < g_end && rc == SF_OK; ++k) {
            const HostGroup &hg = groups[k];
            const sf_dw_problem &p0 = probs[hg.first];
            DwGroup &g = gd[k - gi];
            const void *a = p0.T > 0 ? p0.A : p0.dW;     // any valid address when there are no tokens
            const int64_t lda = p0.T > 0 ? p0.ld_a : p0.C;
            g.a3d = p0.C % 64 == 0 &&
                    encode_bf16_chunks(&g.tm_a, a, 64, p0.T, p0.C / 64, lda, B_COLS / 64, CU_TENSOR_MAP_SWIZZLE_128B);
            if (!g.a3d && !encode_bf16(&g.tm_a, a, p0.C, p0.T, lda, 64, CU_TENSOR_MAP_SWIZZLE_128B))
                rc = SF_ERR_CUDA;
            g.first = pi;
            g.count = hg.count;
            g.C = p0.C;
            g.T = p0.T;
            g.n_ntiles = (p0.C + BN - 1) / BN;
            g.mcap = hg.mcap;
            if (row_ok(hg)) {
                uint8_t *base = scratch(hg);
                g.info = reinterpret_cast<const int32_t *>(base);
                g.rowmap = reinterpret_cast<const int32_t *>(base + kInfoBytes);
                const void *dxg = base + kInfoBytes + rowmap_bytes(hg.mcap);
                if (!encode_rows_kmajor(&g.tm_g, dxg, p0.T, hg.mcap, (int64_t)round_up((size_t)p0.T, 8)))
                    rc = SF_ERR_CUDA;
            }
            long long tiles_mt = 0;
            for (int q = 0; q < hg.count; ++q, ++pi) {
                const sf_dw_problem &p = probs[hg.first + q];
                DwProb &d = pd[pi];
                const void *dx = p.T > 0 ? p.dX : p.dW;
                if (!encode_bf16(&d.tm_dx, dx, p.mask.R, p.T, p.T > 0 ? p.ld_dx : p.mask.R, 32,
                                 CU_TENSOR_MAP_SWIZZLE_64B))
                    rc = SF_ERR_CUDA;
                d.active_tiles = p.mask.active_tiles;
                d.counts = p.mask.counts;
                d.row_slot = p.mask.row_slot;
                d.dW = p.dW;
                d.ld_dw = p.ld_dw;
                tiles_mt += (p.mask.R / 32 + UNIT_TILES - 1) / UNIT_TILES;
            }
            max_units += tiles_mt * g.n_ntiles;
        }
        if (rc != SF_OK) break;
        const long long slots = PAIR == 2 ? (long long)pair_slots : (long long)sms;
        const int grid = PAIR * (int)(max_units < slots ? max_units : slots);
        if (grid > 0) {
            // launches after the first of the call overlap their predecessor's last wave
            cudaLaunchAttribute attr[2];
            int na = 0;
            if (PAIR == 2) {
                attr[na].id = cudaLaunchAttributeClusterDimension;
                attr[na].val.clusterDim.x = 2;
                attr[na].val.clusterDim.y = 1;
                attr[na].val.clusterDim.z = 1;
                ++na;
            }
            if (n_main_launches > 0) {
                attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
                attr[na].val.programmaticStreamSerializationAllowed = 1;
                ++na;
            }
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(grid);
            cfg.blockDim = dim3(kThreads);
            cfg.dynamicSmemBytes = kSmemBytes;
            cfg.stream = st;
            cfg.attrs = attr;
            cfg.numAttrs = na;
            if (cudaLaunchKernelEx(&cfg, masked_dw_kernel, *batch, dev_status) != cudaSuccess ||
                launch_status() != SF_OK) {
                rc = SF_ERR_CUDA;
                break;
            }
            ++n_main_launches;
        }
        gi = g_end;
    }
    delete batch;
    delete[] groups;
    return rc;
}

extern "C" int sf_masked_dw(const sf_dw_problem *probs, int n, void *ws, size_t ws_bytes,
                            uint32_t *dev_status, sf_stream stream)
{
    return sf_masked_dw_phase(probs, n, ws, ws_bytes, SF_PHASE_ALL, dev_status, stream);
}
