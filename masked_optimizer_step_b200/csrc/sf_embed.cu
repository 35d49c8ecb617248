// sf_embed.cu -- embedding-row gradient restricted to active rows.
//
// "Sparse-First Fine-Tuning" (tensorwirelabs.com), sections 1 and 2.2: an embedding row can
// have a nonzero gradient only if its token occurs in the batch, so with a large vocabulary
// the mask cuts nearly all of the table's gradient work. Row r gets G[r] = the sum of the
// upstream gradients dY[t] over the batch positions t holding token r, and only rows the
// conductor marks active are computed and stored.
//
// Three launches, each of the last two a programmatic dependent of the one before:
//   embed_index_kernel  one CTA: for every token whose row is active, its slot (the loads of four
//                       tokens per thread in flight together, the slots kept in shared memory);
//                       per-slot counts (shared-memory atomics, exact), an exclusive scan into
//                       segment offsets, a table of (slot, segment) per active row, and a scatter
//                       of the token positions into their slot's segment.
//   embed_sort_kernel   one warp per segment over the whole grid: the segment's positions sorted
//                       ascending through a bitmap of positions, so the sum order is fixed.
//   embed_sum_kernel    persistent: one item = (table entry, 256-column chunk). 8 warps each sum
//                       every 8th token of the row's sorted segment with 16-byte loads (up to
//                       eight in flight per lane) and the partial sums are added in warp order.
//                       Active rows without tokens get zeros.
// Traffic: dY rows of the tokens of active rows are read once per column chunk (8 KB per token
// at H = 4096); 16 KB per active row is written.
#include <atomic>
#include <mutex>

#include <climits>

#include "sf_common.cuh"
#include "sf_host.h"

namespace sf {
namespace {

constexpr int kIndexThreads = 1024;
constexpr int kSumThreads = 256;
constexpr int kSumWarps = kSumThreads / 32;
constexpr int kChunkCols = 256;             // 32 lanes x 8 bf16
constexpr int kMaxTokens = 16384;
constexpr int kMaxSlots = 49152;

// Scratch layout (int32 words): tbl[4 * slot_cap] | n_tbl[4] | perm[n_tok]
//   tbl[j] = {slot, first, end, 0} of the j-th active row that holds a slot (active-row order);
//   perm[first .. end) are that row's token positions, ascending.
constexpr size_t scratch_ints(int n_tok, int slot_cap)
{
    return 4 * (size_t)slot_cap + 4 + (size_t)n_tok;
}

constexpr int kBatch = 4;                   // tokens per thread whose loads are in flight together
constexpr size_t kSmemLimit = 200 * 1024;   // dynamic shared memory of the index kernel, at most
constexpr int kIndexWarps = kIndexThreads / 32;

// The index kernel keeps the counts cnt[slot_cap] and, when they fit, each token's slot
// s_slot[n_tok] in shared memory (otherwise the slots are looked up again for the scatter).
constexpr size_t index_smem_ints(int n_tok, int slot_cap, bool keep_slots)
{
    return (size_t)slot_cap + (keep_slots ? (size_t)n_tok : 0);
}

constexpr int kSortThreads = 256;           // 8 warps, one segment at a time each

// The slot of token id r, or -1 (bad id, inactive row, or a row without a slot). The mask word
// and the slot are loaded together: both depend only on r.
__device__ __forceinline__ int slot_of(int r, uint32_t word, int slot)
{
    return ((word >> (r & 31)) & 1u) ? slot : -1;
}

__device__ __forceinline__ int active_slot(const int32_t *tok, int t, const sf_mask &mk)
{
    const int r = tok[t];
    if (r < 0 || r >= mk.R) return -1;
    return slot_of(r, mk.words[r >> 5], mk.row_slot[r]);
}

// One warp sorts the m >= 2 positions src[0 .. m) (a segment, in any order) into dst[0 .. m),
// ascending (dst may be src): each position sets its bit in the warp's n_tok-bit map, and the set
// bits are read back in order. Lane l owns the map words [l * wpl, (l + 1) * wpl): it alone
// clears them and reads them back (a warp scan of the lanes' bit counts places its positions),
// so only the bit setting needs the warp's barriers, and a next segment may start at once.
__device__ __forceinline__ void sort_segment(const int32_t *src, int32_t *dst, int m, uint32_t *bm, int words,
                                             int lane)
{
    const int wpl = (words + 31) >> 5;                       // bitmap words per lane
    const int q0 = min(words, lane * wpl), q1 = min(words, q0 + wpl);
    for (int q = q0; q < q1; ++q) bm[q] = 0u;
    __syncwarp();
    for (int i0 = 0; i0 < m; i0 += 32 * kBatch * 2) {        // loads in flight, then the bits
        int p[kBatch * 2];
#pragma unroll
        for (int u = 0; u < kBatch * 2; ++u) {
            const int i = i0 + u * 32 + lane;
            p[u] = i < m ? src[i] : -1;
        }
#pragma unroll
        for (int u = 0; u < kBatch * 2; ++u)
            if (p[u] >= 0) atomicOr(&bm[p[u] >> 5], 1u << (p[u] & 31));
    }
    __syncwarp();
    int c = 0;
    for (int q = q0; q < q1; ++q) c += __popc(bm[q]);
    int out = warp_inclusive_scan(c) - c;
    for (int q = q0; q < q1; ++q) {
        uint32_t bits = bm[q];
        while (bits) {
            dst[out++] = q * 32 + __ffs(bits) - 1;
            bits &= bits - 1u;
        }
    }
}

__global__ void __launch_bounds__(kIndexThreads)
embed_index_kernel(const int32_t *tok, int n_tok, sf_mask mk, int4 *tbl, int32_t *n_tbl, int32_t *perm,
                   int keep_slots, uint32_t *status)
{
    extern __shared__ int smem_i[];
    const int cap = mk.slot_cap;
    int *cnt = smem_i;
    int *s_slot = smem_i + cap;
    __shared__ int scan_scratch[33];
    __shared__ int s_total;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    griddep_launch_dependents();                 // the sort kernel may start; it waits for this grid
    for (int s = tid; s < cap; s += blockDim.x) cnt[s] = 0;
    // the first blockDim active rows and their slots, for the table: loaded beside the first
    // tokens' loads (row ids and count with the token ids, slots with the mask words)
    const int n_act = mk.counts[0];
    const int act_row0 = tid < mk.R ? mk.active_rows[tid] : -1;
    int act_slot0 = -1;
    __syncthreads();
    // 1. the slot of each token, kBatch tokens per thread at a time so that their loads overlap
    //    (id, then mask word and slot together); exact counts
    bool bad = false;
    for (int base = 0; base < n_tok; base += kBatch * blockDim.x) {
        int r[kBatch], sl[kBatch];
        uint32_t w[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int t = base + u * (int)blockDim.x + tid;
            r[u] = t < n_tok ? tok[t] : -1;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int t = base + u * (int)blockDim.x + tid;
            const bool valid = r[u] >= 0 && r[u] < mk.R;
            if (t < n_tok && !valid) bad = true;
            w[u] = valid ? mk.words[r[u] >> 5] : 0u;
            sl[u] = valid ? mk.row_slot[r[u]] : -1;
        }
        if (base == 0 && tid < n_act) act_slot0 = mk.row_slot[act_row0];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int t = base + u * (int)blockDim.x + tid;
            sl[u] = r[u] >= 0 && r[u] < mk.R ? slot_of(r[u], w[u], sl[u]) : -1;
            if (sl[u] >= 0) atomicAdd(&cnt[sl[u]], 1);
            if (keep_slots && t < n_tok) s_slot[t] = sl[u];
        }
    }
    if (n_tok == 0 && tid < n_act) act_slot0 = mk.row_slot[act_row0];
    if (bad) set_status(status, SF_STATUS_BAD_TOKEN);
    __syncthreads();
    // 2. exclusive scan of the counts in slot order: warp w owns a contiguous run of slots, read
    //    32 consecutive slots at a time (no bank conflicts); one scan over the warps' totals, then
    //    each warp scans its run with a carry. cnt[s] becomes segment s's start (its fill cursor)
    {
        const int per_w = ((cap + kIndexWarps - 1) / kIndexWarps + 31) & ~31;
        const int w0 = min(cap, warp * per_w), w1 = min(cap, w0 + per_w);
        int local = 0;
        for (int s = w0 + lane; s < w1; s += 32) local += cnt[s];
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) local += __shfl_xor_sync(0xffffffffu, local, d);
        if (lane == 0) scan_scratch[warp] = local;
        __syncthreads();
        if (warp == 0) {
            const int v = lane < kIndexWarps ? scan_scratch[lane] : 0;
            const int inc = warp_inclusive_scan(v);
            if (lane < kIndexWarps) scan_scratch[lane] = inc - v;
            if (lane == 31) s_total = inc;
        }
        __syncthreads();
        int carry = scan_scratch[warp];
        for (int s0 = w0; s0 < w1; s0 += 32) {
            const int s = s0 + lane;
            const int c = s < w1 ? cnt[s] : 0;
            const int inc = warp_inclusive_scan(c);
            if (s < w1) cnt[s] = carry + inc - c;
            carry += __shfl_sync(0xffffffffu, inc, 31);
        }
    }
    __syncthreads();
    // 3. the table of active rows that hold a slot, in active-row order; a segment ends where
    //    the next slot's begins
    {
        const int total = s_total;
        int base_j = 0;
        for (int base = 0; base < n_act; base += blockDim.x) {
            const int k = base + tid;
            const int sl = base == 0 ? act_slot0 : (k < n_act ? mk.row_slot[mk.active_rows[k]] : -1);
            int tot;
            const int j = block_exclusive_scan(sl >= 0, scan_scratch, &tot);
            if (sl >= 0) tbl[base_j + j] = make_int4(sl, cnt[sl], sl + 1 < cap ? cnt[sl + 1] : total, 0);
            base_j += tot;
        }
        if (tid == 0) n_tbl[0] = base_j;
    }
    __syncthreads();
    // 4. every token of an active row into its slot's segment (in no particular order: the
    //    sort kernel orders each segment)
    for (int base = 0; base < n_tok; base += blockDim.x) {
        const int t = base + tid;
        const int s = t < n_tok ? (keep_slots ? s_slot[t] : active_slot(tok, t, mk)) : -1;
        if (s >= 0) perm[atomicAdd(&cnt[s], 1)] = t;
    }
}

// Each segment of the table sorted ascending in place, one warp per segment over the whole
// grid, so the order the sums take below is fixed whatever order the scatter's atomics gave.
__global__ void __launch_bounds__(kSortThreads)
embed_sort_kernel(const int4 *tbl, const int32_t *n_tbl, int32_t *perm, int n_tok)
{
    extern __shared__ uint32_t sort_bm[];        // one n_tok-bit map per warp
    griddep_launch_dependents();                 // the sum kernel may start; it waits for this grid
    griddep_wait();                              // the index kernel's table and scatter
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int words = (n_tok + 31) >> 5;
    uint32_t *bm = sort_bm + (size_t)warp * words;
    const int n_seg = n_tbl[0];
    const int nw = (int)(gridDim.x * (blockDim.x >> 5));
    for (int j = (int)blockIdx.x * (int)(blockDim.x >> 5) + warp; j < n_seg; j += nw) {
        const int4 e = tbl[j];
        const int m = e.z - e.y;
        if (m >= 2) sort_segment(perm + e.y, perm + e.y, m, bm, words, lane);
    }
}

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4 &v)
{
    const uint32_t ww[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        acc[2 * e] = __fadd_rn(acc[2 * e], __uint_as_float(ww[e] << 16));
        acc[2 * e + 1] = __fadd_rn(acc[2 * e + 1], __uint_as_float(ww[e] & 0xFFFF0000u));
    }
}

// Adds the bf16 rows held by lanes j0 .. j0 + U - 1 of `mine` (token positions) into acc, in
// that order, U loads in flight.
template <int U>
__device__ __forceinline__ void sum_batch(float (&acc)[8], const uint16_t *dY, long long ld_dy, int c0,
                                          bool col_ok, int mine, int j0)
{
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int p = __shfl_sync(0xffffffffu, mine, j0 + u);
        if (col_ok) v[u] = __ldg(reinterpret_cast<const uint4 *>(dY + (size_t)p * ld_dy + c0));
    }
    if (col_ok) {
#pragma unroll
        for (int u = 0; u < U; ++u) add_bf16x8(acc, v[u]);
    }
}

__global__ void __launch_bounds__(kSumThreads, 2)
embed_sum_kernel(const uint16_t *dY, int H, long long ld_dy, float *G, long long ld_g, const int4 *tbl,
                 const int32_t *n_tbl, const int32_t *perm)
{
    __shared__ float part[2][kSumWarps][kChunkCols];     // two items' partial sums, alternately
    griddep_wait();                             // the table and the sorted positions
    const int nchunks = (H + kChunkCols - 1) / kChunkCols;
    const int total = n_tbl[0] * nchunks;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // The next item's table entry is loaded while the current item runs, and its first batch of
    // positions once the current item's loads are issued, so an item starts with its dY loads.
    int4 e_next = make_int4(0, 0, 0, 0);
    int mine_next = 0;
    if ((int)blockIdx.x < total) {
        e_next = tbl[blockIdx.x / nchunks];
        const int idx = warp + kSumWarps * lane;
        mine_next = idx < e_next.z - e_next.y ? __ldg(perm + e_next.y + idx) : 0;
    }
    int buf = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x, buf ^= 1) {
        const int j = item / nchunks;
        const int chunk = item - j * nchunks;
        const int4 e = e_next;                  // slot, first, end
        const int mine_first = mine_next;
        const int nxt = item + (int)gridDim.x;
        if (nxt < total) e_next = tbl[nxt / nchunks];
        const int slot = e.x, b0 = e.y, n = e.z - e.y;
        const int c0 = chunk * kChunkCols + lane * 8;
        const bool col_ok = c0 < H;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        // warp w sums positions w, w + 8, w + 16, ... of the sorted segment, in that order; a
        // batch holds the warp's next 32 positions, one per lane, handed out by shuffles and
        // loaded 8, 4, 2, 1 at a time (the count is the same for the whole warp)
        for (int base = warp; base < n; base += kSumWarps * 32) {
            const int idx = base + kSumWarps * lane;
            const int mine = base == warp ? mine_first : (idx < n ? __ldg(perm + b0 + idx) : 0);
            const int cnt = min(32, (n - base + kSumWarps - 1) / kSumWarps);
            int j0 = 0;
            for (; j0 + 8 <= cnt; j0 += 8) sum_batch<8>(acc, dY, ld_dy, c0, col_ok, mine, j0);
            if (cnt - j0 >= 4) { sum_batch<4>(acc, dY, ld_dy, c0, col_ok, mine, j0); j0 += 4; }
            if (cnt - j0 >= 2) { sum_batch<2>(acc, dY, ld_dy, c0, col_ok, mine, j0); j0 += 2; }
            if (cnt - j0 >= 1) sum_batch<1>(acc, dY, ld_dy, c0, col_ok, mine, j0);
        }
        if (nxt < total) {
            const int idx = warp + kSumWarps * lane;
            mine_next = idx < e_next.z - e_next.y ? __ldg(perm + e_next.y + idx) : 0;
        }
        // fixed-order combination of the 8 warps' partial sums; the buffers alternate, so the
        // next item may write its partial sums while this item's are still being read
#pragma unroll
        for (int q = 0; q < 8; ++q) part[buf][warp][lane * 8 + q] = acc[q];
        __syncthreads();
        const int col = chunk * kChunkCols + tid;
        if (col < H) {
            float sum = part[buf][0][tid];
#pragma unroll
            for (int w = 1; w < kSumWarps; ++w) sum = __fadd_rn(sum, part[buf][w][tid]);
            G[(size_t)slot * ld_g + col] = sum;
        }
    }
}

// The three launches of one embedding-row gradient, on scratch of scratch_ints(n_tok, slot_cap)
// words (16-byte aligned).
int launch_embed(const int32_t *tokens, int n_tok, const void *dY, int H, int64_t ld_dy, const sf_mask &mk,
                 float *G, int64_t ld_g, int32_t *scratch, uint32_t *dev_status, cudaStream_t st)
{
    int4 *tbl = reinterpret_cast<int4 *>(scratch);
    int32_t *n_tbl = scratch + 4 * (size_t)mk.slot_cap;
    int32_t *perm = n_tbl + 4;
    const int keep_slots = index_smem_ints(n_tok, mk.slot_cap, true) * sizeof(int) <= kSmemLimit;
    const size_t smem = index_smem_ints(n_tok, mk.slot_cap, keep_slots) * sizeof(int);
    if (smem > kSmemLimit) return SF_ERR_UNSUPPORTED;
    // above 48 KB of shared memory in all, static included, the launch needs the opt-in
    // attribute; it is set from 40 KB of dynamic memory on (the static part is far below 8 KB)
    if (smem > 40 * 1024 &&
        cudaFuncSetAttribute(embed_index_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return SF_ERR_CUDA;
    const int sms = sm_count();
    if (sms <= 0) return SF_ERR_NO_DEVICE;
    embed_index_kernel<<<1, kIndexThreads, smem, st>>>(tokens, n_tok, mk, tbl, n_tbl, perm, keep_slots, dev_status);
    if (launch_status() != SF_OK) return SF_ERR_CUDA;
    // the sort and sum kernels are programmatic dependents of the kernel before them: their CTAs
    // are placed while it runs and wait for its completion before reading what it wrote
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(kSortThreads);
    cfg.dynamicSmemBytes = (size_t)(kSortThreads / 32) * (((size_t)n_tok + 31) / 32) * sizeof(uint32_t);
    if (cudaLaunchKernelEx(&cfg, embed_sort_kernel, static_cast<const int4 *>(tbl),
                           static_cast<const int32_t *>(n_tbl), perm, n_tok) != cudaSuccess)
        return SF_ERR_CUDA;
    cfg.gridDim = dim3(sms * 4);
    cfg.blockDim = dim3(kSumThreads);
    cfg.dynamicSmemBytes = 0;
    if (cudaLaunchKernelEx(&cfg, embed_sum_kernel, static_cast<const uint16_t *>(dY), H, (long long)ld_dy, G,
                           (long long)ld_g, static_cast<const int4 *>(tbl), static_cast<const int32_t *>(n_tbl),
                           static_cast<const int32_t *>(perm)) != cudaSuccess)
        return SF_ERR_CUDA;
    return launch_status();
}

}  // namespace
}  // namespace sf

using namespace sf;

extern "C" size_t sf_embed_grad_ws_bytes(int n_tok, int slot_cap)
{
    if (n_tok < 0 || slot_cap < 0) return 0;
    const size_t b = scratch_ints(n_tok, slot_cap) * sizeof(int32_t);
    return (b + 255) & ~(size_t)255;
}

extern "C" int sf_embed_grad(const int32_t *tokens, int n_tok, const void *dY, int H,
                             int64_t ld_dy, const sf_mask *mk, float *G, int64_t ld_g, void *ws,
                             size_t ws_bytes, uint32_t *dev_status, sf_stream stream)
{
    if (!mk || !G || H <= 0 || n_tok < 0 || (n_tok > 0 && (!tokens || !dY))) return SF_ERR_ARG;
    int rc = check_mask(*mk);
    if (rc != SF_OK) return rc;
    if (n_tok > kMaxTokens || mk->slot_cap > kMaxSlots) return SF_ERR_UNSUPPORTED;
    if ((H & 7) || ld_dy < H || (ld_dy & 7) || ld_g < H || (ld_g & 3)) return SF_ERR_ARG;
    if ((n_tok > 0 && !aligned16(dY)) || !aligned16(G) || !aligned16(ws)) return SF_ERR_ALIGN;
    if (!ws || ws_bytes < sf_embed_grad_ws_bytes(n_tok, mk->slot_cap)) return SF_ERR_ARG;
    if (mk->slot_cap == 0) return SF_OK;
    return launch_embed(tokens, n_tok, dY, H, ld_dy, *mk, G, ld_g, static_cast<int32_t *>(ws), dev_status,
                        as_stream(stream));
}

// ---------------------------------------------------------------------------------------------
// Allocation-free variant of sf_embed_grad.
//
// Some callers cannot hand the library a scratch buffer: they run inside a host program that
// owns every device allocation (a plugin of a framework with its own memory pool, where a
// foreign cudaMalloc would bypass the pool's accounting), or inside a latency-critical loop
// where cudaMalloc's implicit device synchronisation is not acceptable. For them the scratch
// of the embedding-row gradient lives in a fixed array in the library's own device memory.
// The array exists once per GPU that loads the library and stays allocated until the process
// exits; every call on that GPU uses it, so calls that overlap on the GPU (other streams, other
// threads) race on it and must be serialised by the caller. Nothing in it has to start at zero:
// each call writes the parts it later reads.
// ---------------------------------------------------------------------------------------------
namespace sf {
namespace {

constexpr int kNoAllocScratchInts = SF_EMBED_NOALLOC_SCRATCH_INTS;
static __device__ __align__(256) int32_t g_embed_scratch[kNoAllocScratchInts];

constexpr int kMaxDevices = 64;

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

// The driver's cuCtxGetCurrent, looked up once through the runtime (the library links no
// driver library directly).
CtxGetCurrentFn ctx_get_current()
{
    static std::atomic<CtxGetCurrentFn> fn{nullptr};
    CtxGetCurrentFn f = fn.load(std::memory_order_acquire);
    if (f) return f;
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !p)
        return nullptr;
    f = reinterpret_cast<CtxGetCurrentFn>(p);
    fn.store(f, std::memory_order_release);
    return f;
}

struct ScratchAddr {
    CUcontext ctx;               // the context the address belongs to
    int32_t *addr;
};
ScratchAddr g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of g_embed_scratch in the current context (the array's name in host code is
// only a stand-in for the symbol, not a device pointer). It is looked up with
// cudaGetSymbolAddress the first time a device is used and again whenever the device's current
// context is not the one the cached address came from (after cudaDeviceReset, or under another
// driver-API context), so a stale address is never handed to a kernel.
int32_t *noalloc_scratch()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    CtxGetCurrentFn get = ctx_get_current();
    CUcontext ctx = nullptr;
    if (!get || get(&ctx) != CUDA_SUCCESS) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchAddr &e = g_scratch_addr[dev];
    if (ctx && e.addr && e.ctx == ctx) return e.addr;
    void *addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_embed_scratch) != cudaSuccess || !addr) return nullptr;
    if (get(&ctx) != CUDA_SUCCESS || !ctx) return nullptr;     // current once the runtime has bound it
    e.ctx = ctx;
    e.addr = static_cast<int32_t *>(addr);
    return e.addr;
}

}  // namespace
}  // namespace sf

extern "C" int sf_embed_grad_noalloc(const int32_t *tokens, int n_tok, const void *dY, int H,
                                     int64_t ld_dy, const sf_mask *mk, float *G, int64_t ld_g,
                                     uint32_t *dev_status, sf_stream stream)
{
    if (!mk || !G || H <= 0 || n_tok < 0 || (n_tok > 0 && (!tokens || !dY))) return SF_ERR_ARG;
    int rc = check_mask(*mk);
    if (rc != SF_OK) return rc;
    if (n_tok > kMaxTokens || mk->slot_cap > kMaxSlots) return SF_ERR_UNSUPPORTED;
    if (scratch_ints(n_tok, mk->slot_cap) > (size_t)kNoAllocScratchInts) return SF_ERR_UNSUPPORTED;
    if ((H & 7) || ld_dy < H || (ld_dy & 7) || ld_g < H || (ld_g & 3)) return SF_ERR_ARG;
    if ((n_tok > 0 && !aligned16(dY)) || !aligned16(G)) return SF_ERR_ALIGN;
    if (mk->slot_cap == 0) return SF_OK;
    int32_t *scratch = noalloc_scratch();
    if (!scratch) return SF_ERR_CUDA;
    return launch_embed(tokens, n_tok, dY, H, ld_dy, *mk, G, ld_g, scratch, dev_status, as_stream(stream));
}
