// sf_embed.cu -- embedding-row gradient restricted to active rows.
//
// "Sparse-First Fine-Tuning" (tensorwirelabs.com), sections 1 and 2.2: an embedding row can
// have a nonzero gradient only if its token occurs in the batch, so with a large vocabulary
// the mask cuts nearly all of the table's gradient work. Row r gets G[r] = the sum of the
// upstream gradients dY[t] over the batch positions t holding token r, and only rows the
// conductor marks active are computed and stored.
//
// Two launches:
//   embed_index_kernel  one CTA: for every token whose row is active, its slot; per-slot counts
//                       (shared-memory atomics, exact), an exclusive scan into segment offsets,
//                       and a stable scatter of token positions into their slot's segment of ws
//                       (ascending within a segment, so the sum order is fixed).
//   embed_sum_kernel    persistent: one item = (active row, 256-column chunk). 8 warps each
//                       sum every 8th token of the row's sorted segment with 16-byte loads (eight
//                       in flight per lane) and the partial sums are added in warp order. Active
//                       rows without tokens get zeros.
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
constexpr int kSumUnroll = 8;               // token loads in flight per lane

// ws layout: seg_off[slot_cap + 1] int32 | perm[n_tok] int32
__global__ void __launch_bounds__(kIndexThreads)
embed_index_kernel(const int32_t *tok, int n_tok, sf_mask mk, int32_t *seg_off, int32_t *perm,
                   uint32_t *status)
{
    extern __shared__ int cnt[];            // [slot_cap]
    __shared__ int scan_scratch[33];
    __shared__ int s_run;
    const int cap = mk.slot_cap;
    for (int s = threadIdx.x; s < cap; s += blockDim.x) cnt[s] = 0;
    if (threadIdx.x == 0) s_run = 0;
    __syncthreads();
    bool bad = false;
    for (int t = threadIdx.x; t < n_tok; t += blockDim.x) {
        const int r = tok[t];
        if (r < 0 || r >= mk.R) { bad = true; continue; }
        if (!((mk.words[r >> 5] >> (r & 31)) & 1u)) continue;   // inactive row: dropped
        const int s = mk.row_slot[r];
        if (s >= 0) atomicAdd(&cnt[s], 1);
    }
    if (bad) set_status(status, SF_STATUS_BAD_TOKEN);
    __syncthreads();
    // exclusive scan of the counts, in slot order, chunk by chunk
    for (int base = 0; base < cap; base += blockDim.x) {
        const int s = base + threadIdx.x;
        const int c = s < cap ? cnt[s] : 0;
        int total;
        const int off = block_exclusive_scan(c, scan_scratch, &total);
        const int run = s_run;
        if (s < cap) {
            seg_off[s] = run + off;
            cnt[s] = 0;                     // becomes the fill cursor
        }
        __syncthreads();
        if (threadIdx.x == 0) s_run = run + total;
        __syncthreads();
    }
    if (threadIdx.x == 0) seg_off[cap] = s_run;
    __syncthreads();
    // Stable scatter: a slot's positions land in ascending order. Tokens go in rounds of
    // blockDim (one per thread, in order); inside a warp, lanes holding the same slot rank
    // themselves by lane; across warps, each warp's group leaders claim their slots' next places
    // in warp order, one warp per barrier step. So the sum order below never depends on timing.
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    for (int base = 0; base < n_tok; base += blockDim.x) {
        const int t = base + threadIdx.x;
        int s = -1;
        if (t < n_tok) {
            const int r = tok[t];
            if (r >= 0 && r < mk.R && ((mk.words[r >> 5] >> (r & 31)) & 1u)) s = mk.row_slot[r];
        }
        const uint32_t peers = __match_any_sync(0xffffffffu, s);
        const int leader = __ffs(peers) - 1;
        int place = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            if (warp == w && s >= 0 && lane == leader) {
                place = cnt[s];
                cnt[s] = place + __popc(peers);
            }
            __syncthreads();
        }
        place = __shfl_sync(0xffffffffu, place, leader);
        if (s >= 0) perm[seg_off[s] + place + __popc(peers & lt)] = t;
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

__global__ void __launch_bounds__(kSumThreads)
embed_sum_kernel(const uint16_t *dY, int H, long long ld_dy, sf_mask mk, float *G, long long ld_g,
                 const int32_t *seg_off, const int32_t *perm)
{
    __shared__ float part[kSumWarps][kChunkCols];
    const int n_act = mk.counts[0];
    const int nchunks = (H + kChunkCols - 1) / kChunkCols;
    const int total = n_act * nchunks;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        const int k = item / nchunks;
        const int chunk = item - k * nchunks;
        const int r = mk.active_rows[k];
        const int slot = mk.row_slot[r];
        if (slot < 0) continue;
        const int b0 = seg_off[slot], n = seg_off[slot + 1] - b0;
        const int c0 = chunk * kChunkCols + lane * 8;
        const bool col_ok = c0 < H;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        // warp w sums positions w, w + 8, w + 16, ... of the sorted segment, in that order; a
        // batch holds the warp's next 32 positions, one per lane, handed out by shuffles
        for (int base = warp; base < n; base += kSumWarps * 32) {
            const int idx = base + kSumWarps * lane;
            const int mine = idx < n ? __ldg(perm + b0 + idx) : 0;
            const int cnt = min(32, (n - base + kSumWarps - 1) / kSumWarps);
            for (int j0 = 0; j0 < cnt; j0 += kSumUnroll) {
                uint4 v[kSumUnroll];
#pragma unroll
                for (int u = 0; u < kSumUnroll; ++u) {
                    const int p = __shfl_sync(0xffffffffu, mine, (j0 + u) & 31);
                    if (j0 + u < cnt && col_ok)
                        v[u] = __ldg(reinterpret_cast<const uint4 *>(dY + (size_t)p * ld_dy + c0));
                }
#pragma unroll
                for (int u = 0; u < kSumUnroll; ++u)
                    if (j0 + u < cnt && col_ok) add_bf16x8(acc, v[u]);
            }
        }
        // fixed-order combination of the 8 warps' partial sums
#pragma unroll
        for (int e = 0; e < 8; ++e) part[warp][lane * 8 + e] = acc[e];
        __syncthreads();
        const int col = chunk * kChunkCols + tid;
        if (col < H) {
            float s = part[0][tid];
#pragma unroll
            for (int w = 1; w < kSumWarps; ++w) s = __fadd_rn(s, part[w][tid]);
            G[(size_t)slot * ld_g + col] = s;
        }
        __syncthreads();
    }
}

// The two launches of one embedding-row gradient, on scratch seg_off[slot_cap + 1] | perm[n_tok].
int launch_embed(const int32_t *tokens, int n_tok, const void *dY, int H, int64_t ld_dy, const sf_mask &mk,
                 float *G, int64_t ld_g, int32_t *scratch, uint32_t *dev_status, cudaStream_t st)
{
    int32_t *seg_off = scratch;
    int32_t *perm = seg_off + mk.slot_cap + 1;
    const size_t smem = (size_t)mk.slot_cap * sizeof(int);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(embed_index_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return SF_ERR_CUDA;
    const int sms = sm_count();
    if (sms <= 0) return SF_ERR_NO_DEVICE;
    embed_index_kernel<<<1, kIndexThreads, smem, st>>>(tokens, n_tok, mk, seg_off, perm, dev_status);
    if (launch_status() != SF_OK) return SF_ERR_CUDA;
    embed_sum_kernel<<<sms * 4, kSumThreads, 0, st>>>(static_cast<const uint16_t *>(dY), H, ld_dy,
                                                      mk, G, ld_g, seg_off, perm);
    return launch_status();
}

}  // namespace
}  // namespace sf

using namespace sf;

extern "C" size_t sf_embed_grad_ws_bytes(int n_tok, int slot_cap)
{
    if (n_tok < 0 || slot_cap < 0) return 0;
    const size_t b = ((size_t)slot_cap + 1 + (size_t)n_tok) * sizeof(int32_t);
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
    if ((long long)mk->slot_cap + 1 + n_tok > kNoAllocScratchInts) return SF_ERR_UNSUPPORTED;
    if ((H & 7) || ld_dy < H || (ld_dy & 7) || ld_g < H || (ld_g & 3)) return SF_ERR_ARG;
    if ((n_tok > 0 && !aligned16(dY)) || !aligned16(G)) return SF_ERR_ALIGN;
    if (mk->slot_cap == 0) return SF_OK;
    int32_t *scratch = noalloc_scratch();
    if (!scratch) return SF_ERR_CUDA;
    return launch_embed(tokens, n_tok, dY, H, ld_dy, *mk, G, ld_g, scratch, dev_status, as_stream(stream));
}
