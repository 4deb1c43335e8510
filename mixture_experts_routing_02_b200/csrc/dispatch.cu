// Dispatch kernels: expert counts, segment tables (plain, capacity, balanced plan or overflow
// re-routing), the stable rank of every (token, k) pair inside its expert, and the copies that
// write each token row straight into its k final expert-contiguous slots.
//
// The permutation is a counting sort on the expert id with one digit pass: the rank of a pair
// inside its expert is (pairs of that expert before its block) + (earlier pairs of the same
// block).  Three ways to get the first term:
//   * dispatch_count_kernel (plain / capacity up to kCountMaxPairs pairs, balanced plan up to
//     kCountMaxPairsPlan): every CTA counts all ids itself (and computes the plan from the
//     totals), so no CTA waits for another and one launch does counts, tables, ranks and copies;
//   * dispatch_fused_kernel (plain / capacity, any size) and rank_kernel (balanced plan, or
//     tables given): an exclusive prefix over tiles found with a decoupled look-back (Merrill &
//     Garland, "Single-pass Parallel Prefix Scan with Decoupled Look-back", 2016): each tile
//     publishes its own per-expert counts at once and its inclusive prefix as soon as it knows
//     it, so a tile only waits for tiles already running.  Tiles are taken in order from an
//     atomic ticket, which guarantees that every tile a CTA waits for is held by a CTA that is
//     running;
//   * reroute_grid_kernel (overflow re-routing): a cooperative grid runs the capacity rounds, the
//     CTAs exchanging per-expert counts through a bounded grid barrier.
// Every wait is bounded.
//
// Sources: "Sparsely-Gated MoE 구현 관점에서 살펴보기", section "순전파 과정 ..."
// (permute tokens into expert order) and "로드 밸런싱 손실(load-balancing loss)과 용량(capacity)은
// 별개" (capacity; overflow dropped or sent to another candidate); "5.3 Expert Parallelism",
// section "2. 디스패처 엔지니어링" (bincount per destination); the MoonEP page, sections
// "이 기술은 무엇인가" (rows written to their final slot, no separate sort and copy; static
// shapes, no host sync) and "설치 및 통합" (tokens_per_expert, cu_seqlens).
#include "common.cuh"
#include "kernels.h"
#include "vec.cuh"
#include "plan.cuh"
#include "route.cuh"

namespace moe {

namespace {

constexpr uint32_t kFlagAggregate = 1u << 30;
constexpr uint32_t kFlagPrefix = 2u << 30;
constexpr uint32_t kValueMask = (1u << 30) - 1;
constexpr int kPermuteWarps = kPermuteThreads / 32;
constexpr int kCopyUnroll = 8;
constexpr int kLookbackWindow = 128;  // earlier tiles read per look-back round trip (when E allows)
constexpr int kLookbackUnroll = 32;   // most look-back words one thread reads per round trip
constexpr int kCountThreads = 1024;
constexpr int kCountWarps = kCountThreads / 32;
constexpr int kCountBatch = 8;   // expert ids per thread loaded together in the counting pass (scalar loads)
constexpr int kCountBatch4 = 4;  // 16-byte loads (4 ids each) per thread in flight together

// Exclusive scan over the 256 threads of a block; *total receives the sum.
__device__ __forceinline__ int block_exclusive_scan_256(int v, int* warp_sums, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += t;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < 8 ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += t;
        }
        if (lane < 8) warp_sums[lane] = w;  // inclusive
    }
    __syncthreads();
    const int before = warp > 0 ? warp_sums[warp - 1] : 0;
    if (total != nullptr) *total = warp_sums[7];
    __syncthreads();
    return before + x - v;
}

// ------------------------------------------------------------------------------ histogram

__global__ void __launch_bounds__(256) histogram_kernel(const int32_t* __restrict__ ids, int n, int E,
                                                        int32_t* __restrict__ counts) {
    __shared__ int h[kMaxExperts];
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const int e = __ldg(ids + i);
        if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) atomicAdd(&h[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        if (h[e] != 0) atomicAdd(counts + e, h[e]);
}

// Per-CTA histograms written to partials[cta][E] (every entry, zeros included), so nothing needs
// clearing first and no global atomics are used; the segment / plan kernel sums them.  The same
// launch clears the permutation's look-back words (zero_ptr), which the permutation reads next.
__global__ void __launch_bounds__(256) histogram_partial_kernel(const int32_t* __restrict__ ids, int n, int E,
                                                                int32_t* __restrict__ partials,
                                                                uint32_t* __restrict__ zero_ptr, size_t zero_words) {
    __shared__ int h[kMaxExperts];
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    // warp-aggregated: one shared atomic per distinct expert in a warp
    const int lane = threadIdx.x & 31;
    const int stride = gridDim.x * blockDim.x;
    for (int base = blockIdx.x * blockDim.x; base < n; base += stride) {
        const int i = base + threadIdx.x;
        int e = i < n ? __ldg(ids + i) : -1;
        if (static_cast<unsigned>(e) >= static_cast<unsigned>(E)) e = -1;
        const unsigned same = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && lane == __ffs(same) - 1) atomicAdd(&h[e], __popc(same));
    }
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < zero_words;
         i += static_cast<size_t>(gridDim.x) * blockDim.x)
        zero_ptr[i] = 0u;
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) partials[blockIdx.x * E + e] = h[e];
}

// counts[e] from the per-CTA partials (and written out), or read from counts when partials is null
__device__ __forceinline__ int expert_count(const int32_t* counts_in, const int32_t* partials, int n_partials, int E,
                                            int e, int32_t* counts_out) {
    if (partials == nullptr) return counts_in[e];
    int c = 0;
    for (int g = 0; g < n_partials; ++g) c += partials[g * E + e];
    counts_out[e] = c;
    return c;
}

// ------------------------------------------------------------------------------ plain segments

__global__ void __launch_bounds__(256) segments_kernel(int32_t* counts, const int32_t* partials, int n_partials,
                                                       int E, int capacity, int32_t* seg_expert, int32_t* seg_offsets,
                                                       int32_t* seg_first_rank) {
    __shared__ int warp_sums[8];
    const int e = threadIdx.x;
    int v = 0;
    if (e < E) {
        const int c = expert_count(counts, partials, n_partials, E, e, counts);
        v = (capacity > 0 && c > capacity) ? capacity : c;
    }
    int total;
    const int excl = block_exclusive_scan_256(v, warp_sums, &total);
    if (e < E) {
        seg_expert[e] = e;
        seg_offsets[e] = excl;
        seg_first_rank[e] = 0;
    }
    if (e == 0) seg_offsets[E] = total;
}

// ------------------------------------------------------------------------------ balanced plan

__global__ void __launch_bounds__(256) plan_kernel(int32_t* counts, const int32_t* partials, int n_partials, int E,
                                                   int R, int S, int k, int B, int32_t* seg_expert,
                                                   int32_t* seg_offsets, int32_t* seg_first_rank, int32_t* status) {
    __shared__ PlanSmem sm;
    for (int e = threadIdx.x; e < E; e += blockDim.x) sm.c[e] = expert_count(counts, partials, n_partials, E, e, counts);
    __syncthreads();
    compute_plan(sm, E, R, S, k, B, seg_expert, seg_offsets, seg_first_rank, status, true);
}

// ------------------------------------------------------------------------------ stable rank + permute

// Threads per expert in the look-back: a power of two, at most a warp, G * E <= kPermuteThreads.
__device__ __forceinline__ int lookback_group(int E) {
    int g = 32;
    while (g > 1 && g * E > kPermuteThreads) g >>= 1;
    return g;
}

struct TileSmem {
    int wcnt[kPermuteWarps][kMaxExperts];  // per-warp counts of each expert in the tile
    int h[kMaxExperts];                    // tile counts
    int excl[kMaxExperts];                 // pairs of each expert in earlier tiles
    int abort;
};

// Stable rank of the pairs of one tile.  Called by the whole CTA with sm.wcnt zeroed; ends
// with a barrier.  *e = expert of this thread's pair (-1: none or out of range), *r = the
// pair's rank among all pairs of that expert in q order.  A look-back wait that runs out
// reports MOE_DEV_ERR_TIMEOUT, sets sm.abort and publishes nothing further for this tile.
__device__ __forceinline__ void rank_tile(const PermuteArgs& a, int tile, TileSmem& sm, int* e_out, int* r_out) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = a.E, k = a.k;
    const int t0 = tile * a.tokens_per_tile;
    const int t1 = min(a.T, t0 + a.tokens_per_tile);
    const int q0 = t0 * k;
    const int nq = (t1 - t0) * k;

    // 1. expert of this thread's pair and its rank among equal experts of the same warp
    int e = -1;
    if (tid < nq) {
        e = __ldg(a.ids + q0 + tid);
        if (static_cast<unsigned>(e) >= static_cast<unsigned>(E)) e = -1;
    }
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int wrank = __popc(same & ((1u << lane) - 1u));
    if (e >= 0 && wrank == 0) sm.wcnt[warp][e] = __popc(same);
    __syncthreads();

    // 2. tile histogram, published at once (tile 0: as its inclusive prefix)
    if (tid < E) {
        int h = 0;
#pragma unroll
        for (int w = 0; w < kPermuteWarps; ++w) h += sm.wcnt[w][tid];
        sm.h[tid] = h;
        st_relaxed_u32(a.tile_state + static_cast<size_t>(tile) * E + tid,
                       (tile == 0 ? kFlagPrefix : kFlagAggregate) | static_cast<uint32_t>(h));
        if (tile == 0) sm.excl[tid] = 0;
    }
    __syncthreads();
    // 3. look back over a window of W = G * U earlier tiles per round trip: thread g of the
    //    expert's group reads the U words of tiles hi - g*U - u (u < U), all loads in flight
    //    together; the group adds the aggregates up to the nearest inclusive prefix and moves
    //    the window back only when it holds no prefix.  Tiles tend to start together, so few
    //    prefixes exist early; a wide window keeps the walk to a few round trips.  Every
    //    decision is uniform inside a group.
    const int G = lookback_group(E);
    const int U = kLookbackWindow / G < kLookbackUnroll ? kLookbackWindow / G : kLookbackUnroll;
    if (tile > 0 && tid < E * G) {
        const int ge = tid / G, g = tid % G;
        const int base = lane & ~(G - 1);
        const unsigned gmask = (G == 32 ? 0xffffffffu : ((1u << G) - 1u)) << base;
        int excl = 0;
        int hi = tile - 1;
        uint64_t t_start = 0;
        uint32_t spins = 0;
        bool gave_up = false;
        while (hi >= 0) {
            uint32_t w[kLookbackUnroll];
#pragma unroll
            for (int u = 0; u < kLookbackUnroll; ++u) {
                const int j = hi - g * U - u;
                w[u] = (u < U && j >= 0) ? ld_relaxed_u32(a.tile_state + static_cast<size_t>(j) * E + ge)
                                         : kFlagPrefix;  // before tile 0: an inclusive prefix of 0
            }
            int first = kLookbackUnroll;  // nearest prefix among this thread's words
#pragma unroll
            for (int u = kLookbackUnroll - 1; u >= 0; --u)
                if (u < U && (w[u] & ~kValueMask) == kFlagPrefix) first = u;
            const unsigned has = __ballot_sync(gmask, first < kLookbackUnroll) & gmask;
            const int gp = has ? __ffs(has >> base) - 1 : G;  // thread holding the nearest prefix
            // words needed: all of threads g < gp, and u <= first of thread gp
            const int need_u = g < gp ? U : (g == gp ? first + 1 : 0);
            bool miss = false;
            int v = 0;
#pragma unroll
            for (int u = 0; u < kLookbackUnroll; ++u) {
                if (u < need_u) {
                    if ((w[u] & ~kValueMask) == 0) miss = true;
                    v += static_cast<int>(w[u] & kValueMask);
                }
            }
            if (__ballot_sync(gmask, miss) & gmask) {
                int out = 0;
                if (g == 0 && (++spins & 63u) == 0) {
                    const uint64_t now = globaltimer_ns();
                    if (t_start == 0) t_start = now;
                    else if (now - t_start > kWaitLimitNs) out = 1;
                }
                if (__shfl_sync(gmask, out, base)) {
                    if (g == 0) {
                        report(a.status, MOE_DEV_ERR_TIMEOUT);
                        sm.abort = 1;
                    }
                    gave_up = true;
                    break;
                }
                continue;
            }
            for (int o = G >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(gmask, v, o);
            excl += v;
            if (has) break;
            hi -= G * U;
        }
        // a tile that gave up publishes no prefix, so the tiles after it give up too
        if (g == 0) {
            if (!gave_up)
                st_relaxed_u32(a.tile_state + static_cast<size_t>(tile) * E + ge,
                               kFlagPrefix | static_cast<uint32_t>(excl + sm.h[ge]));
            sm.excl[ge] = excl;
        }
    }
    __syncthreads();
    int r = -1;
    if (e >= 0) {
        r = sm.excl[e] + wrank;
        for (int w = 0; w < warp; ++w) r += sm.wcnt[w][e];
    }
    *e_out = e;
    *r_out = r;
}

__global__ void __launch_bounds__(kPermuteThreads) rank_kernel(const PermuteArgs a) {
    __shared__ TileSmem sm;
    __shared__ int s_excl[kMaxExperts];
    __shared__ int s_cbeg[kMaxExperts + 1];
    __shared__ int s_cseg[kMaxSegments];
    __shared__ int warp_sums[8];
    __shared__ int s_tile;

    const int tid = threadIdx.x;
    const int E = a.E, k = a.k;

    // segments of each expert (CSR in shared memory); order inside an expert does not matter
    if (tid < E) s_excl[tid] = 0;
    if (tid == 0) sm.abort = 0;
    __syncthreads();
    for (int s = tid; s < a.n_seg; s += blockDim.x) {
        const int ex = __ldg(a.seg_expert + s);
        if (static_cast<unsigned>(ex) < static_cast<unsigned>(E) &&
            __ldg(a.seg_offsets + s + 1) > __ldg(a.seg_offsets + s))
            atomicAdd(&s_excl[ex], 1);
    }
    __syncthreads();
    {
        int total;
        const int excl = block_exclusive_scan_256(tid < E ? s_excl[tid] : 0, warp_sums, &total);
        if (tid < E) { s_cbeg[tid] = excl; s_excl[tid] = excl; }
        if (tid == 0) s_cbeg[E] = total;
    }
    __syncthreads();
    for (int s = tid; s < a.n_seg; s += blockDim.x) {
        const int ex = __ldg(a.seg_expert + s);
        if (static_cast<unsigned>(ex) < static_cast<unsigned>(E) &&
            __ldg(a.seg_offsets + s + 1) > __ldg(a.seg_offsets + s))
            s_cseg[atomicAdd(&s_excl[ex], 1)] = s;
    }
    __syncthreads();

    for (;;) {
        if (tid == 0) s_tile = static_cast<int>(atomicAdd(a.ticket, 1u)) + a.first_tile;
        for (int i = tid; i < kPermuteWarps * kMaxExperts; i += blockDim.x) (&sm.wcnt[0][0])[i] = 0;
        __syncthreads();
        const int tile = s_tile;
        if (tile >= a.n_tiles || sm.abort) break;
        int e, r;
        rank_tile(a, tile, sm, &e, &r);
        if (sm.abort) break;

        // 3. final slot of each pair: its expert's segment that holds rank r
        const int q0 = tile * a.tokens_per_tile * k;
        const int nq = (min(a.T, (tile + 1) * a.tokens_per_tile) - tile * a.tokens_per_tile) * k;
        if (tid < nq) {
            int dst = -1;
            if (e >= 0) {
                for (int p = s_cbeg[e]; p < s_cbeg[e + 1]; ++p) {
                    const int s = s_cseg[p];
                    const int fr = __ldg(a.seg_first_rank + s);
                    const int off = __ldg(a.seg_offsets + s);
                    const int len = __ldg(a.seg_offsets + s + 1) - off;
                    if (r >= fr && r < fr + len) { dst = off + (r - fr); break; }
                }
            }
            a.dest[q0 + tid] = dst;
            if (dst >= 0) a.src[dst] = q0 + tid;
        }
        __syncthreads();
    }
}

// Copy the row of token t of X to its final slots dj[0..k) with 16-byte vectors, kCopyUnroll in
// flight per lane (one warp; for X or Xp not 32-byte aligned).
__device__ __forceinline__ void copy_row_v4(const __nv_bfloat16* __restrict__ x, int t, const int* dj, int k, int d,
                                         int rows, __nv_bfloat16* __restrict__ xp, int lane) {
    const int vec_per_row = d / 8;
    const uint4* xs = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d);
    for (int v = lane; v < vec_per_row; v += 32 * kCopyUnroll) {
        uint4 val[kCopyUnroll];
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u)
            if (v + 32 * u < vec_per_row) val[u] = __ldg(xs + v + 32 * u);
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            if (j < k && dj[j] >= 0 && dj[j] < rows) {
                uint4* dst = reinterpret_cast<uint4*>(xp + static_cast<size_t>(dj[j]) * d);
#pragma unroll
                for (int u = 0; u < kCopyUnroll; ++u)
                    if (v + 32 * u < vec_per_row) dst[v + 32 * u] = val[u];
            }
        }
    }
}

// Copy the row of token t of X to its final slots dj[0..k) (one warp).  Slots outside [0, rows)
// are skipped.  V8 (X and Xp 32-byte aligned; rows are multiples of 128 bytes): each lane moves
// 32-byte vectors, kCopyUnroll / 2 in flight, half the memory instructions of 16-byte vectors.
// The kernels that copy rows are instantiated for both and launched by the alignment.
template <bool V8>
__device__ __forceinline__ void copy_row(const __nv_bfloat16* __restrict__ x, int t, const int* dj, int k, int d,
                                         int rows, __nv_bfloat16* __restrict__ xp, int lane) {
    // a token whose pairs were all dropped is not read at all (dj is the same in every lane)
    bool any = false;
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) any |= (j < k && dj[j] >= 0 && dj[j] < rows);
    if (!any) return;
    if (!V8) {
        copy_row_v4(x, t, dj, k, d, rows, xp, lane);
        return;
    }
    constexpr int U = kCopyUnroll / 2;
    const int vec_per_row = d / 16;
    const uint8_t* xs = reinterpret_cast<const uint8_t*>(x + static_cast<size_t>(t) * d);
    for (int v = lane; v < vec_per_row; v += 32 * U) {
        Vec32 val[U];
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (v + 32 * u < vec_per_row) val[u] = ld_nc_v8(xs + static_cast<size_t>(v + 32 * u) * 32);
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            if (j < k && dj[j] >= 0 && dj[j] < rows) {
                uint8_t* dst = reinterpret_cast<uint8_t*>(xp + static_cast<size_t>(dj[j]) * d);
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (v + 32 * u < vec_per_row) st_v8(dst + static_cast<size_t>(v + 32 * u) * 32, val[u]);
            }
        }
    }
}

// The whole dispatch of the plain (or capacity) layout in one launch, in two phases.
//  1. Tiles from the ticket, as in rank_kernel: each pair's stable rank inside its expert,
//     kept in dest for now.  The tile that holds the last ticket knows every expert's total
//     (its inclusive prefix), so it writes counts and the segment tables and raises "ready".
//  2. Every CTA (those that got no tile too) waits for "ready" and for all tiles to be
//     ranked, then, one warp per token, turns ranks into final slots (capacity applied),
//     writes dest and src, and copies the token's row to its slots.
// A CTA only ever waits on tiles that running CTAs hold (tickets are taken in order), so no
// CTA needs to be resident at the same time as another; every wait is bounded.  While
// waiting, each warp prefetches the rows of X it will copy into L2, so the copy overlaps
// the ranking.
template <bool V8>
__global__ void __launch_bounds__(kPermuteThreads, 4) dispatch_fused_kernel(const PermuteArgs a) {
    __shared__ TileSmem sm;
    __shared__ int warp_sums[8];
    __shared__ int s_tile;
    __shared__ int s_off[kMaxExperts];
    __shared__ int s_go;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = a.E, k = a.k;
    const int warps_total = gridDim.x * kPermuteWarps;
    const int my_warp = blockIdx.x * kPermuteWarps + warp;
    if (tid == 0) sm.abort = 0;

    // phase 1
    for (;;) {
        if (tid == 0) s_tile = static_cast<int>(atomicAdd(a.ticket, 1u)) + a.first_tile;
        for (int i = tid; i < kPermuteWarps * kMaxExperts; i += blockDim.x) (&sm.wcnt[0][0])[i] = 0;
        __syncthreads();
        const int tile = s_tile;
        if (tile >= a.n_tiles || sm.abort) break;
        int e, r;
        rank_tile(a, tile, sm, &e, &r);
        if (sm.abort) break;
        const int q0 = tile * a.tokens_per_tile * k;
        const int nq = (min(a.T, (tile + 1) * a.tokens_per_tile) - tile * a.tokens_per_tile) * k;
        if (tid < nq) a.dest[q0 + tid] = r;  // rank for now (-1: no expert)
        if (tile == a.n_tiles - 1) {
            const int total_e = tid < E ? sm.excl[tid] + sm.h[tid] : 0;
            const int v = (a.capacity > 0 && total_e > a.capacity) ? a.capacity : total_e;
            int total;
            const int off = block_exclusive_scan_256(tid < E ? v : 0, warp_sums, &total);
            if (tid < E) {
                a.counts[tid] = total_e;
                a.seg_expert_out[tid] = tid;
                a.seg_offsets_out[tid] = off;
                a.seg_first_rank_out[tid] = 0;
            }
            if (tid == 0) a.seg_offsets_out[E] = total;
        }
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            red_release_add_u32(a.sync + 0, 1u);
            if (tile == a.n_tiles - 1) st_release_u32(a.sync + 1, 1u);
        }
    }
    if (sm.abort) {
        if (tid == 0) st_relaxed_u32(a.sync + 2, 1u);
        return;
    }

    // rows of X this warp copies in phase 2: into L2 while the last tiles are ranked
    if (a.prefetch_x && lane == 0)
        for (int t = my_warp; t < a.T; t += warps_total)
            prefetch_l2_bulk(a.x + static_cast<size_t>(t) * a.d, static_cast<uint32_t>(a.d) * 2u);

    // phase 2
    if (tid == 0) {
        int go = 1;
        const uint64_t t0 = globaltimer_ns();
        uint32_t spins = 0;
        while (!(ld_acquire_u32(a.sync + 1) == 1u &&
                 ld_acquire_u32(a.sync + 0) == static_cast<uint32_t>(a.n_tiles))) {
            if (ld_relaxed_u32(a.sync + 2) != 0u) { go = 0; break; }
            if ((++spins & 63u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) {
                report(a.status, MOE_DEV_ERR_TIMEOUT);
                st_relaxed_u32(a.sync + 2, 1u);
                go = 0;
                break;
            }
        }
        s_go = go;
    }
    __syncthreads();
    if (!s_go) return;
    for (int e = tid; e < E; e += blockDim.x) s_off[e] = __ldcg(a.seg_offsets_out + e);
    __syncthreads();

    for (int t = my_warp; t < a.T; t += warps_total) {
        int mine = -1;
        if (lane < k) {
            const int q = t * k + lane;
            const int e = __ldg(a.ids + q);
            const int r = __ldcg(a.dest + q);
            if (static_cast<unsigned>(e) < static_cast<unsigned>(E) && r >= 0 &&
                (a.capacity == 0 || r < a.capacity)) {
                mine = s_off[e] + r;
                if (mine >= a.rows) mine = -1;
            }
            a.dest[q] = mine;
            if (mine >= 0) a.src[mine] = q;
        }
        int dj[kMaxTopK];
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) dj[j] = __shfl_sync(0xffffffffu, mine, j);
        copy_row<V8>(a.x, t, dj, k, a.d, a.rows, a.xp, lane);
    }
}

// Dispatch of the plain (or capacity) layout in one launch with no communication between CTAs,
// for inputs of up to kCountMaxPairs pairs.  The tokens form 2G blocks for G CTAs; CTA b owns
// block b and block 2G-1-b (one from the front, one from the back: with a capacity, later
// tokens lose more pairs, so the pairing evens out the rows each CTA copies).  Each CTA
//  1. counts the expert ids of ALL pairs in shared memory (one shared atomic per id), split
//     into the pairs before its first block, the pairs between its blocks and the rest: the
//     totals give the segment offsets and the partial sums give each block's exclusive prefix
//     per expert, so neither a look-back nor a second launch is needed (the counting is
//     repeated by every CTA; it reads T*k ids from L2, which is why it is limited to small T*k);
//  2. ranks the pairs of its blocks in q order (match_any inside a warp, per-warp counts across
//     warps), applies the capacity, writes dest and src (CTA 0 also writes counts and tables);
//  3. copies each of its tokens' rows to the token's slots, one warp per token, the two blocks
//     forming one list over all warps (a token whose pairs were all dropped is not read).
// Dynamic shared memory of the count dispatch with a balanced plan: the plan, its segment tables
// and each expert's segments (CSR by expert).
struct CountPlanSmem {
    PlanSmem plan;
    int seg_e[kMaxSegments], seg_fr[kMaxSegments], seg_off[kMaxSegments + 1];
    int cbeg[kMaxExperts + 1], cfill[kMaxExperts], cseg[kMaxSegments];
};

template <bool PLAN, bool V8>
__global__ void __launch_bounds__(kCountThreads, 1) dispatch_count_kernel(const PermuteArgs a) {
    extern __shared__ __align__(16) uint8_t count_dsmem[];
    __shared__ int s_a[kMaxExperts];    // pairs of each expert before the first block
    __shared__ int s_m[kMaxExperts];    // ... from the first block up to the second
    __shared__ int s_tot[kMaxExperts];  // ... from the second block on; then: all pairs
    __shared__ int s_off[kMaxExperts];  // segment offsets
    __shared__ int s_run[kMaxExperts];  // pairs of each expert before the current chunk
    __shared__ int s_wcnt[kCountWarps][kMaxExperts];
    __shared__ int warp_sums[kCountWarps];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = a.E, k = a.k;
    const unsigned lanemask_lt = (1u << lane) - 1u;
    const int n = a.T * k;
    const int G = gridDim.x;
    const int tb = (a.T + 2 * G - 1) / (2 * G);
    int tb_[2], te_[2];
    {
        const int blk[2] = {static_cast<int>(blockIdx.x), 2 * G - 1 - static_cast<int>(blockIdx.x)};
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            tb_[r] = min(a.T, blk[r] * tb);
            te_[r] = min(a.T, tb_[r] + tb);
        }
    }
    const int q1 = tb_[0] * k, q2 = tb_[1] * k;  // q1 <= q2

    for (int i = tid; i < E; i += blockDim.x) { s_a[i] = 0; s_m[i] = 0; s_tot[i] = 0; }
    for (int i = tid; i < kCountWarps * kMaxExperts; i += blockDim.x) (&s_wcnt[0][0])[i] = 0;
    __syncthreads();

    // 1. counts of all pairs, split at the starts of the two blocks: 16-byte loads of 4 ids,
    // kCountBatch4 of them in flight per thread (scalar loads if the ids are not 16-byte aligned)
    auto count_one = [&](int e, int i) {
        if (static_cast<unsigned>(e) < static_cast<unsigned>(E))
            atomicAdd(i < q1 ? &s_a[e] : (i < q2 ? &s_m[e] : &s_tot[e]), 1);
    };
    int scalar_from = 0;
    if ((reinterpret_cast<uintptr_t>(a.ids) & 15u) == 0) {
        const int n4 = n >> 2;
        const int4* ids4 = reinterpret_cast<const int4*>(a.ids);
        for (int base = 0; base < n4; base += blockDim.x * kCountBatch4) {
            int4 ev[kCountBatch4];
#pragma unroll
            for (int u = 0; u < kCountBatch4; ++u) {
                const int i = base + u * blockDim.x + tid;
                ev[u] = i < n4 ? __ldg(ids4 + i) : make_int4(-1, -1, -1, -1);
            }
#pragma unroll
            for (int u = 0; u < kCountBatch4; ++u) {
                const int i = 4 * (base + u * blockDim.x + tid);
                count_one(ev[u].x, i);
                count_one(ev[u].y, i + 1);
                count_one(ev[u].z, i + 2);
                count_one(ev[u].w, i + 3);
            }
        }
        scalar_from = n4 << 2;
    }
    for (int base = scalar_from; base < n; base += blockDim.x * kCountBatch) {
        int ev[kCountBatch];
#pragma unroll
        for (int u = 0; u < kCountBatch; ++u) {
            const int i = base + u * blockDim.x + tid;
            ev[u] = i < n ? __ldg(a.ids + i) : -1;
        }
#pragma unroll
        for (int u = 0; u < kCountBatch; ++u) count_one(ev[u], base + u * blockDim.x + tid);
    }
    __syncthreads();

    CountPlanSmem& ps = *reinterpret_cast<CountPlanSmem*>(count_dsmem);
    if (PLAN) {
        // 2a. the balanced plan from the totals, computed by every CTA alike; CTA 0 publishes
        // counts and the tables; each CTA keeps the segments of every expert (CSR)
        for (int e = tid; e < E; e += blockDim.x) ps.plan.c[e] = s_a[e] + s_m[e] + s_tot[e];
        __syncthreads();
        compute_plan(ps.plan, E, a.R, a.S, k, a.B, ps.seg_e, ps.seg_off, ps.seg_fr, a.status, blockIdx.x == 0);
        if (blockIdx.x == 0) {
            for (int e = tid; e < E; e += blockDim.x) a.counts[e] = ps.plan.c[e];
            for (int sg = tid; sg < a.n_seg; sg += blockDim.x) {
                a.seg_expert_out[sg] = ps.seg_e[sg];
                a.seg_offsets_out[sg] = ps.seg_off[sg];
                a.seg_first_rank_out[sg] = ps.seg_fr[sg];
            }
            if (tid == 0) a.seg_offsets_out[a.n_seg] = ps.seg_off[a.n_seg];
        }
        for (int e = tid; e < E; e += blockDim.x) ps.cfill[e] = 0;
        __syncthreads();
        for (int sg = tid; sg < a.n_seg; sg += blockDim.x) {
            const int ex = ps.seg_e[sg];
            if (static_cast<unsigned>(ex) < static_cast<unsigned>(E) && ps.seg_off[sg + 1] > ps.seg_off[sg])
                atomicAdd(&ps.cfill[ex], 1);
        }
        __syncthreads();
        if (warp == 0) {
            int carry = 0;
            for (int e0 = 0; e0 < E; e0 += 32) {
                const int e = e0 + lane;
                const int v = e < E ? ps.cfill[e] : 0;
                int x = v;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, x, o);
                    if (lane >= o) x += t;
                }
                if (e < E) { ps.cbeg[e] = carry + x - v; ps.cfill[e] = carry + x - v; }
                carry += __shfl_sync(0xffffffffu, x, 31);
            }
            if (lane == 0) ps.cbeg[E] = carry;
        }
        __syncthreads();
        // segments in ascending index inside each expert (the order does not matter: ranges are disjoint)
        for (int sg = tid; sg < a.n_seg; sg += blockDim.x) {
            const int ex = ps.seg_e[sg];
            if (static_cast<unsigned>(ex) < static_cast<unsigned>(E) && ps.seg_off[sg + 1] > ps.seg_off[sg])
                ps.cseg[atomicAdd(&ps.cfill[ex], 1)] = sg;
        }
        __syncthreads();
    } else {
    // 2a. segment offsets (capacity applied); CTA 0 publishes counts and the tables
    {
        const int tot = tid < E ? s_a[tid] + s_m[tid] + s_tot[tid] : 0;
        const int v = (a.capacity > 0 && tot > a.capacity) ? a.capacity : tot;
        // exclusive scan over the CTA (E <= 256 <= blockDim.x)
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += t;
        }
        if (lane == 31) warp_sums[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int w = warp_sums[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += t;
            }
            warp_sums[lane] = w;  // inclusive over warps
        }
        __syncthreads();
        const int off = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
        if (tid < E) {
            s_off[tid] = off;
            if (blockIdx.x == 0) {
                a.counts[tid] = tot;
                a.seg_expert_out[tid] = tid;
                a.seg_offsets_out[tid] = off;
                a.seg_first_rank_out[tid] = 0;
            }
        }
        if (blockIdx.x == 0 && tid == 0) a.seg_offsets_out[E] = warp_sums[kCountWarps - 1];
    }
    }

    // 2b. stable ranks of the pairs of each block, in chunks of blockDim.x pairs
#pragma unroll 1
    for (int r = 0; r < 2; ++r) {
        if (r == 1 && tb_[1] == tb_[0]) break;  // one block only (2G > T at the end)
        for (int x = tid; x < E; x += blockDim.x) s_run[x] = r == 0 ? s_a[x] : s_a[x] + s_m[x];
        __syncthreads();
        const int qb = tb_[r] * k, qe = te_[r] * k;
        for (int q0 = qb; q0 < qe; q0 += blockDim.x) {
            const int q = q0 + tid;
            int e = -1;
            if (q < qe) {
                e = __ldg(a.ids + q);
                if (static_cast<unsigned>(e) >= static_cast<unsigned>(E)) e = -1;
            }
            const unsigned same = __match_any_sync(0xffffffffu, e);
            const int wrank = __popc(same & lanemask_lt);
            if (e >= 0 && wrank == 0) s_wcnt[warp][e] = __popc(same);
            __syncthreads();
            if (q < qe) {
                int dst = -1;
                if (e >= 0) {
                    int rk = s_run[e] + wrank;
                    for (int w = 0; w < warp; ++w) rk += s_wcnt[w][e];
                    if (PLAN) {
                        // the expert's segment holding rank rk (home rows, then replica pieces)
                        for (int p = ps.cbeg[e]; p < ps.cbeg[e + 1]; ++p) {
                            const int sg = ps.cseg[p];
                            const int fr = ps.seg_fr[sg], off = ps.seg_off[sg], len = ps.seg_off[sg + 1] - off;
                            if (rk >= fr && rk < fr + len) { dst = off + (rk - fr); break; }
                        }
                        if (dst >= a.rows) dst = -1;
                    } else if (a.capacity == 0 || rk < a.capacity) {
                        dst = s_off[e] + rk;
                        if (dst >= a.rows) dst = -1;
                    }
                }
                a.dest[q] = dst;
                if (dst >= 0) a.src[dst] = q;
            }
            __syncthreads();
            for (int x = tid; x < E; x += blockDim.x) {
                int c = 0;
                for (int w = 0; w < kCountWarps; ++w) { c += s_wcnt[w][x]; s_wcnt[w][x] = 0; }
                s_run[x] += c;
            }
            __syncthreads();
        }
    }

    // 3. rows of this CTA's tokens to their slots: both blocks form one list over all warps
    {
        const int n0 = te_[0] - tb_[0];
        const int n1 = tb_[1] == tb_[0] ? 0 : te_[1] - tb_[1];
        for (int i = warp; i < n0 + n1; i += kCountWarps) {
            const int t = i < n0 ? tb_[0] + i : tb_[1] + (i - n0);
            const int mine = lane < k ? a.dest[static_cast<size_t>(t) * k + lane] : -1;
            int dj[kMaxTopK];
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j) dj[j] = __shfl_sync(0xffffffffu, mine, j);
            copy_row<V8>(a.x, t, dj, k, a.d, a.rows, a.xp, lane);
        }
    }
}

// ------------------------------------------------------------------------------ overflow re-routing

// Stable ranks inside one CTA of kRerouteThreads threads, for a list of n entries whose keys
// (experts, -1 = none) come from key(i): warp w owns the contiguous range [w*L, (w+1)*L) of the
// list, counts its keys per expert (cnt[w][e]), the counts become exclusive prefixes across warps
// (plus base[e]), and each warp walks its range again handing out ranks in list order.  Two
// block barriers in all.  rank_out(i, e, r) receives every entry with a key; totals[e] (if not
// null) the number of entries per expert.
template <typename KeyF, typename OutF>
__device__ __forceinline__ void warp_range_ranks(int n, int E, int (*cnt)[kMaxExperts], const int* base,
                                                 int* totals, KeyF key, OutF rank_out) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int kWarps = kRerouteThreads / 32;
    const unsigned lanemask_lt = (1u << lane) - 1u;
    const int L = (n + kWarps - 1) / kWarps;
    const int b0 = min(n, warp * L), b1 = min(n, b0 + L);
    for (int e = lane; e < E; e += 32) cnt[warp][e] = 0;
    __syncwarp();
    for (int i0 = b0; i0 < b1; i0 += 32) {
        const int i = i0 + lane;
        const int e = i < b1 ? key(i) : -1;
        const unsigned same = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && (same & lanemask_lt) == 0) cnt[warp][e] += __popc(same);
        __syncwarp();
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = base ? base[e] : 0;
        for (int w = 0; w < kWarps; ++w) {
            const int c = cnt[w][e];
            cnt[w][e] = run;
            run += c;
        }
        if (totals) totals[e] = run - (base ? base[e] : 0);
    }
    __syncthreads();
    for (int i0 = b0; i0 < b1; i0 += 32) {
        const int i = i0 + lane;
        const int e = i < b1 ? key(i) : -1;
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const int r = e >= 0 ? cnt[warp][e] + __popc(same & lanemask_lt) : -1;
        __syncwarp();
        if (e >= 0 && (same & lanemask_lt) == 0) cnt[warp][e] += __popc(same);
        __syncwarp();
        if (e >= 0) rank_out(i, e, r);
    }
    __syncthreads();
}

// Order-preserving compaction inside one CTA: entries i < n with keep(i) are written, in order,
// through put(position, i); returns the number kept.  Same warp ranges; two barriers.
template <typename KeepF, typename PutF>
__device__ __forceinline__ int warp_range_compact(int n, int* warp_cnt /*[33]*/, KeepF keep, PutF put) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int kWarps = kRerouteThreads / 32;
    const int L = (n + kWarps - 1) / kWarps;
    const int b0 = min(n, warp * L), b1 = min(n, b0 + L);
    int c = 0;
    for (int i0 = b0; i0 < b1; i0 += 32) {
        const int i = i0 + lane;
        c += __popc(__ballot_sync(0xffffffffu, i < b1 && keep(i)));
    }
    if (lane == 0) warp_cnt[warp] = c;
    __syncthreads();
    if (warp == 0) {
        const int v = warp_cnt[lane];
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += t;
        }
        warp_cnt[lane] = x - v;
        if (lane == 31) warp_cnt[32] = x;
    }
    __syncthreads();
    int pos = warp_cnt[warp];
    for (int i0 = b0; i0 < b1; i0 += 32) {
        const int i = i0 + lane;
        const bool k = i < b1 && keep(i);
        const unsigned b = __ballot_sync(0xffffffffu, k);
        if (k) put(pos + __popc(b & ((1u << lane) - 1u)), i);
        pos += __popc(b);
    }
    const int total = warp_cnt[32];
    __syncthreads();
    return total;
}

// Each token's experts in candidate order (logit descending, equal logits: the lower id), one
// warp per token over the whole GPU: every lane ranks its U experts against all E by shuffles
// and writes them to their positions.  A token's first k candidates are its top-k.
template <int U>
__global__ void __launch_bounds__(256) candidate_order_kernel(const float* __restrict__ logits, int T, int E,
                                                              int stride, uint8_t* __restrict__ cand) {
    const int lane = threadIdx.x & 31;
    const int warps_total = gridDim.x * (blockDim.x >> 5);
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps_total) {
        const float* lt = logits + static_cast<size_t>(t) * E;
        float v[U];
        int rank[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            v[u] = (lane + 32 * u < E) ? __ldg(lt + lane + 32 * u) : -INFINITY;
            rank[u] = 0;
        }
#pragma unroll
        for (int u2 = 0; u2 < U; ++u2) {
            for (int src = 0; src < 32; ++src) {
                const float o = __shfl_sync(0xffffffffu, v[u2], src);
                const int oe = 32 * u2 + src;
                if (oe >= E) break;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int e = lane + 32 * u;
                    rank[u] += (o > v[u] || (o == v[u] && oe < e)) ? 1 : 0;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = lane + 32 * u;
            if (e < E) cand[static_cast<size_t>(t) * stride + rank[u]] = static_cast<uint8_t>(e);
        }
    }
}

// Capacity with re-routing of the overflow ("로드 밸런싱 손실 ... 용량(capacity)은 별개": a pair
// over its expert's capacity may go to another candidate):
//  round 0  each expert keeps its first C pairs in q order (stable ranks over the pair list);
//  round r  every unplaced pair proposes to its token's next candidate in logit order (the
//           token's experts are sorted once; its cursor starts after its top-k) among the experts
//           that had room when the round began; a token's unplaced pairs take consecutive
//           candidates in j order; each expert accepts the proposals in q order while it has room;
//           a pair without a candidate is dropped.
// Segment e holds expert e's rows: round 0 first, then round 1, ...; q order inside a round.
// Writes counts (the plain histogram), the tables, dest and src; X rows are then copied by
// scatter_rows_kernel.  At most E + 1 rounds: each round either places every proposal or fills
// an expert (with a skewed router, about one expert fills per round).

// Bounded grid-wide barrier of a cooperative launch: bar[0] counts the CTAs that arrived, bar[1]
// is the generation.  Thread 0 of each CTA arrives; the last one clears the count and advances the
// generation; the others wait for it (bounded: a wait that runs out reports MOE_DEV_ERR_TIMEOUT and
// sets *abort, and an aborted CTA no longer arrives, so the others run out too and every CTA ends).
// The fences before the arrival and after the wait order each CTA's global writes before the
// other CTAs' reads that follow the barrier.
__device__ __forceinline__ bool grid_barrier(uint32_t* bar, int32_t* status, volatile int* abort) {
    __syncthreads();
    if (threadIdx.x == 0 && !*abort) {
        const uint32_t gen = ld_acquire_u32(bar + 1);
        __threadfence();
        if (atomicAdd(bar, 1u) == gridDim.x - 1) {
            st_relaxed_u32(bar, 0u);
            __threadfence();
            st_release_u32(bar + 1, gen + 1u);
        } else {
            const uint64_t t0 = globaltimer_ns();
            while (ld_acquire_u32(bar + 1) == gen) {
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    report(status, MOE_DEV_ERR_TIMEOUT);
                    *abort = 1;
                    break;
                }
                sleep_ns(64);
            }
        }
        __threadfence();
    }
    __syncthreads();
    return *abort == 0;
}

// The rounds above over the whole GPU: a cooperative launch of G CTAs (one per SM at most), every
// CTA taking the same decisions from the same exchanged counts.  CTA c owns a fixed slice of whole
// tokens (pairs [c*L, (c+1)*L), L a multiple of k, at most kRerouteSliceMax pairs) and keeps all of
// the slice's state in shared memory: its unplaced pairs in q order, their proposals, each pair's
// final expert and rank, each token's candidate cursor.  CTA order is q order and one thread walks
// a token's unplaced pairs in j order, so a round needs one exchange through global memory: the
// CTAs' per-expert counts of their proposals (round 0: of their pairs), through a bounded grid
// barrier.  From the exchanged [G, E] counts each CTA takes the counts of the CTAs before it as the
// base of its stable ranks (the same q-ordered ranks as one CTA over the whole list) and the
// totals, from which every CTA derives the experts' new row counts and the number of pairs still
// unplaced.  Exchanged counts are read through L2 (ld.global.cg).
constexpr int kRerouteSliceMax = 4096 + kMaxTopK;  // pairs of one CTA's slice (shared memory: 6 ints each)

size_t reroute_smem_bytes() { return size_t(6) * kRerouteSliceMax * sizeof(int); }

__global__ void __launch_bounds__(kRerouteThreads, 1) reroute_grid_kernel(RerouteArgs a) {
    extern __shared__ __align__(16) int rr_dsmem[];
    int* s_pend = rr_dsmem;                     // unplaced pairs (offsets in the slice), q order
    int* s_next = s_pend + kRerouteSliceMax;    // the same after a round
    int* s_prop = s_next + kRerouteSliceMax;    // each unplaced pair's proposal (-1: no candidate left)
    int* s_fexp = s_prop + kRerouteSliceMax;    // each pair's final expert (-1: none yet)
    int* s_fslot = s_fexp + kRerouteSliceMax;   // and its rank in that expert's rows
    int* s_cur = s_fslot + kRerouteSliceMax;    // each token's next candidate position
    __shared__ int s_cnt[kRerouteThreads / 32][kMaxExperts];
    __shared__ int s_loc[kMaxExperts];       // this CTA's counts, then: all CTAs' totals
    __shared__ int s_base[kMaxExperts];      // counts of the CTAs before this one
    __shared__ int s_assigned[kMaxExperts];
    __shared__ int s_room[kMaxExperts];
    __shared__ int s_wc[33];
    __shared__ int s_sum, s_any_open;
    __shared__ volatile int s_abort;

    const int tid = threadIdx.x, G = gridDim.x, cta = blockIdx.x;
    const int E = a.E, k = a.k, C = a.capacity;
    const int n = a.T * k;
    const int tokens_per_cta = (a.T + G - 1) / G;
    const int b0 = min(n, cta * tokens_per_cta * k), e0 = min(n, b0 + tokens_per_cta * k);
    const int nl = e0 - b0;  // <= kRerouteSliceMax (checked by the launcher)
    // testing only (moe_testing_reroute_stalled): CTA 0 starts aborted, so it never arrives at the
    // first grid barrier and every other CTA's bounded wait there runs out
    if (tid == 0) s_abort = (a.test_skip_arrival != 0 && cta == 0) ? 1 : 0;
    int xbuf = 0;

    // this CTA's counts s_loc[0..E) exchanged with every CTA's: s_base = the sum over the CTAs before
    // this one, s_loc = the sum over all.  Two buffers in turn: a CTA writes a buffer again only after
    // the barrier of the next exchange, which every CTA passes only after reading it.
    auto exchange = [&]() -> bool {
        int32_t* buf = a.xchg + static_cast<size_t>(xbuf) * kRerouteMaxCtas * kMaxExperts;
        xbuf ^= 1;
        for (int x = tid; x < E; x += blockDim.x) __stcg(buf + static_cast<size_t>(cta) * kMaxExperts + x, s_loc[x]);
        if (!grid_barrier(a.bar, a.status, &s_abort)) return false;
        for (int x = tid; x < E; x += blockDim.x) {
            int before = 0, all = 0;
            for (int c0 = 0; c0 < G; c0 += 16) {  // 16 CTAs' counts in flight together
                int v[16];
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    v[u] = c0 + u < G ? __ldcg(buf + static_cast<size_t>(c0 + u) * kMaxExperts + x) : 0;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    all += v[u];
                    if (c0 + u < cta) before += v[u];
                }
            }
            s_base[x] = before;
            s_loc[x] = all;
        }
        __syncthreads();
        return true;
    };
    auto id_of = [&](int i) -> int {  // expert of pair b0 + i (-1: outside [0, E))
        const int e = __ldg(a.ids + b0 + i);
        return static_cast<unsigned>(e) < static_cast<unsigned>(E) ? e : -1;
    };
    // a block-wide sum over the experts of per_expert(e)
    auto sum_over = [&](auto per_expert) -> int {
        if (tid == 0) s_sum = 0;
        __syncthreads();
        int v = 0;
        for (int x = tid; x < E; x += blockDim.x) v += per_expert(x);
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if ((tid & 31) == 0 && v) atomicAdd(&s_sum, v);
        __syncthreads();
        return s_sum;
    };

    // ---- round 0: stable ranks of the slice's pairs; keep the first C of each expert
    for (int t = tid; t < nl / k; t += blockDim.x) s_cur[t] = k;
    for (int x = tid; x < E; x += blockDim.x) s_loc[x] = 0;
    __syncthreads();
    for (int i = tid; i < nl; i += blockDim.x) {
        s_fexp[i] = -1;
        s_fslot[i] = -1;
        const int e = id_of(i);
        if (e >= 0) atomicAdd(&s_loc[e], 1);
    }
    __syncthreads();
    if (!exchange()) return;
    if (cta == 0)
        for (int x = tid; x < E; x += blockDim.x) a.counts[x] = s_loc[x];
    warp_range_ranks(nl, E, s_cnt, s_base, nullptr, [&](int i) { return id_of(i); },
                     [&](int i, int e, int r) {
                         if (r < C) { s_fexp[i] = e; s_fslot[i] = r; }
                     });
    for (int x = tid; x < E; x += blockDim.x) s_assigned[x] = min(s_loc[x], C);
    int n_pend = sum_over([&](int x) { return max(0, s_loc[x] - C); });  // over all CTAs
    int* pend = s_pend;
    int* next = s_next;
    int n_local = warp_range_compact(nl, s_wc, [&](int i) { return id_of(i) >= 0 && s_fexp[i] < 0; },
                                     [&](int pos, int i) { pend[pos] = i; });

    for (int round = 1; round <= E + 1 && n_pend > 0; ++round) {
        if (tid == 0) s_any_open = 0;
        __syncthreads();
        for (int x = tid; x < E; x += blockDim.x) {
            s_room[x] = C - s_assigned[x];
            if (s_room[x] > 0) s_any_open = 1;
        }
        __syncthreads();
        if (!s_any_open) break;  // the same on every CTA
        // proposals: the thread at a token's first unplaced pair walks that token's pairs in j order
        for (int i = tid; i < n_local; i += blockDim.x) {
            const int tl = pend[i] / k;  // token within the slice (b0 is a multiple of k)
            if (i > 0 && pend[i - 1] / k == tl) continue;
            const uint8_t* ct = a.cand + static_cast<size_t>(b0 / k + tl) * a.cand_stride;
            int pos = s_cur[tl];
            for (int j = i; j < n_local && pend[j] / k == tl; ++j) {
                while (pos < E) {
                    const int base = pos & ~15;
                    const uint4 c4 = __ldg(reinterpret_cast<const uint4*>(ct + base));
                    const uint32_t words[4] = {c4.x, c4.y, c4.z, c4.w};
                    bool found = false;
                    for (; pos < base + 16 && pos < E; ++pos) {
                        const int ex = (words[(pos - base) >> 2] >> (8 * ((pos - base) & 3))) & 0xffu;
                        if (s_room[ex] > 0) { found = true; break; }
                    }
                    if (found) break;
                }
                s_prop[j] = pos < E ? static_cast<int>(ct[pos]) : -1;
                pos = pos < E ? pos + 1 : E;
            }
            s_cur[tl] = pos;
        }
        // acceptance in q order: ranks of the proposals over all CTAs
        for (int x = tid; x < E; x += blockDim.x) s_loc[x] = 0;
        __syncthreads();
        for (int i = tid; i < n_local; i += blockDim.x) {
            const int e = s_prop[i];
            if (e >= 0) atomicAdd(&s_loc[e], 1);
        }
        __syncthreads();
        if (!exchange()) return;
        warp_range_ranks(n_local, E, s_cnt, s_base, nullptr, [&](int i) { return s_prop[i]; },
                         [&](int i, int e, int r) {
                             if (r < s_room[e]) {
                                 s_fexp[pend[i]] = e;
                                 s_fslot[pend[i]] = s_assigned[e] + r;
                             }
                         });
        n_pend = sum_over([&](int x) { return max(0, s_loc[x] - s_room[x]); });  // rejected stay unplaced
        for (int x = tid; x < E; x += blockDim.x) s_assigned[x] += min(s_loc[x], s_room[x]);
        // still unplaced: a proposal that was not accepted (a pair without a candidate is dropped)
        n_local = warp_range_compact(n_local, s_wc, [&](int i) { return s_prop[i] >= 0 && s_fexp[pend[i]] < 0; },
                                     [&](int pos, int i) { next[pos] = pend[i]; });
        int* tmp = pend; pend = next; next = tmp;
    }

    // tables (CTA 0) and the positions of this CTA's pairs: segment e starts at the scan of the rows
    __syncthreads();
    if (tid < 32) {
        int carry = 0;
        for (int x0 = 0; x0 < E; x0 += 32) {
            const int e = x0 + tid;
            const int v = e < E ? s_assigned[e] : 0;
            int x = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, x, o);
                if (tid >= o) x += t;
            }
            if (e < E) {
                s_room[e] = carry + x - v;
                if (cta == 0) {
                    a.seg_expert[e] = e;
                    a.seg_offsets[e] = carry + x - v;
                    a.seg_first_rank[e] = 0;
                }
            }
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
        if (tid == 0 && cta == 0) a.seg_offsets[E] = carry;
    }
    __syncthreads();
    for (int i = tid; i < nl; i += blockDim.x) {
        const int e = s_fexp[i];
        int dst = -1;
        if (e >= 0) {
            dst = s_room[e] + s_fslot[i];
            if (dst >= a.rows) dst = -1;
        }
        a.dest[b0 + i] = dst;
        if (dst >= 0) a.src[dst] = b0 + i;
    }
}

// ------------------------------------------------------------------------------ row scatter

// One warp per token: read the token's row of X once (16-byte vectors, 8 in flight per lane)
// and write it to each of its k final slots.  Pure streaming: no shared memory, no barriers.
template <bool V8>
__global__ void __launch_bounds__(256) scatter_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                           const int32_t* __restrict__ dest, int T, int k, int d,
                                                           int rows, __nv_bfloat16* __restrict__ xp) {
    const int lane = threadIdx.x & 31;
    const int warps_total = gridDim.x * (blockDim.x >> 5);
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps_total) {
        const int mine = lane < k ? __ldg(dest + static_cast<size_t>(t) * k + lane) : -1;
        int dj[kMaxTopK];
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) dj[j] = __shfl_sync(0xffffffffu, mine, j);
        copy_row<V8>(x, t, dj, k, d, rows, xp, lane);
    }
}

// ------------------------------------------------------------------------------ top-k from given logits

// Routing from fp32 logits, one warp per token (lanes over experts).  The logits of token t are
// sum_s part[s * split_stride + t * ldp + e] over the n_split parts in order (+ bias[e]): one
// part is the logits themselves (moe_route_from_logits); several are the partial sums of a
// router projection whose reduction was split over more CTAs.  Writes the logits (optional),
// then either the top-k ids and weights or, for expert-choice routing (scores_t non-null), the
// softmax over all E experts stored expert-major.
template <int U, int KMAX>
__global__ void __launch_bounds__(256) route_logits_kernel(const float* __restrict__ part, int n_split, int ldp,
                                                           size_t split_stride, const float* __restrict__ bias, int T,
                                                           int E, int k, int route_flags, float* __restrict__ logits,
                                                           int32_t* __restrict__ ids, float* __restrict__ w,
                                                           float* __restrict__ scores_t) {
    const int lane = threadIdx.x & 31;
    const int warps_total = gridDim.x * (blockDim.x >> 5);
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps_total)
        route_token<U, KMAX>(part, n_split, ldp, split_stride, bias, T, E, k, route_flags, logits, ids, w, scores_t, t,
                             lane);
}

}  // namespace

int permute_tokens_per_tile(int T, int k) {
    // as many whole tokens as fit in kPermutePairs pairs (one pair per thread)
    (void)T;
    const int t = kPermutePairs / k;
    return t < 1 ? 1 : t;
}

int permute_n_tiles(int T, int k) {
    const int tpt = permute_tokens_per_tile(T, k);
    return (T + tpt - 1) / tpt;
}

size_t permute_scratch_bytes(int T, int k, int E) {
    return 256 + static_cast<size_t>(permute_n_tiles(T, k)) * static_cast<size_t>(E) * sizeof(uint32_t);
}

size_t permute_ws_bytes(int T, int k, int E) {
    return permute_scratch_bytes(T, k, E) +
           static_cast<size_t>(kMaxHistogramPartials) * static_cast<size_t>(E) * sizeof(int32_t);
}

cudaError_t launch_histogram(const int32_t* ids, int n_pairs, int E, int32_t* counts, int num_sms,
                             cudaStream_t stream) {
    cudaError_t err = cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, stream);
    if (err != cudaSuccess) return err;
    if (n_pairs == 0) return cudaSuccess;
    int grid = (n_pairs + 2047) / 2048;
    if (grid > 2 * num_sms) grid = 2 * num_sms;
    histogram_kernel<<<grid, 256, 0, stream>>>(ids, n_pairs, E, counts);
    return cudaGetLastError();
}

int histogram_partial_ctas(int n_pairs) {
    int g = (n_pairs + 1023) / 1024;
    if (g > kMaxHistogramPartials) g = kMaxHistogramPartials;
    return g < 1 ? 1 : g;
}

cudaError_t launch_histogram_partials(const int32_t* ids, int n_pairs, int E, int32_t* partials, uint32_t* zero_ptr,
                                      size_t zero_bytes, cudaStream_t stream) {
    histogram_partial_kernel<<<histogram_partial_ctas(n_pairs), 256, 0, stream>>>(ids, n_pairs, E, partials, zero_ptr,
                                                                                   zero_bytes / 4);
    return cudaGetLastError();
}

cudaError_t launch_segments(int32_t* counts, const int32_t* partials, int n_partials, int E, int capacity,
                            int32_t* seg_expert, int32_t* seg_offsets, int32_t* seg_first_rank, cudaStream_t stream) {
    segments_kernel<<<1, 256, 0, stream>>>(counts, partials, n_partials, E, capacity, seg_expert, seg_offsets,
                                           seg_first_rank);
    return cudaGetLastError();
}

cudaError_t launch_plan(int32_t* counts, const int32_t* partials, int n_partials, int E, int R, int S, int k, int B,
                        int32_t* seg_expert, int32_t* seg_offsets, int32_t* seg_first_rank, int32_t* status,
                        cudaStream_t stream) {
    plan_kernel<<<1, 256, 0, stream>>>(counts, partials, n_partials, E, R, S, k, B, seg_expert, seg_offsets,
                                       seg_first_rank, status);
    return cudaGetLastError();
}

// rows move in 32-byte vectors when X and Xp allow it
static bool rows_v8(const void* x, const void* xp) {
    return ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(xp)) & 31u) == 0;
}

cudaError_t launch_permute(const PermuteArgs& a, bool ws_cleared, int num_sms, cudaStream_t stream) {
    if (!ws_cleared) {
        cudaError_t err = cudaMemsetAsync(a.ticket, 0, permute_scratch_bytes(a.T, a.k, a.E), stream);
        if (err != cudaSuccess) return err;
    }
    if (a.n_tiles == 0) return cudaSuccess;
    int grid = a.n_tiles < 8 * num_sms ? a.n_tiles : 8 * num_sms;
    rank_kernel<<<grid, kPermuteThreads, 0, stream>>>(a);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    int sgrid = (a.T + 7) / 8;
    if (sgrid > 16 * num_sms) sgrid = 16 * num_sms;
    if (rows_v8(a.x, a.xp)) scatter_rows_kernel<true><<<sgrid, 256, 0, stream>>>(a.x, a.dest, a.T, a.k, a.d, a.rows, a.xp);
    else scatter_rows_kernel<false><<<sgrid, 256, 0, stream>>>(a.x, a.dest, a.T, a.k, a.d, a.rows, a.xp);
    return cudaGetLastError();
}

cudaError_t launch_dispatch_fused(const PermuteArgs& a, int num_sms, cudaStream_t stream) {
    cudaError_t err = cudaMemsetAsync(a.ticket, 0, permute_scratch_bytes(a.T, a.k, a.E), stream);
    if (err != cudaSuccess) return err;
    if (a.n_tiles == 0) return cudaSuccess;
    int grid = (a.T + kPermuteWarps - 1) / kPermuteWarps;  // one warp per token in the copy phase
    if (grid > 4 * num_sms) grid = 4 * num_sms;
    if (grid < 1) grid = 1;
    if (rows_v8(a.x, a.xp)) dispatch_fused_kernel<true><<<grid, kPermuteThreads, 0, stream>>>(a);
    else dispatch_fused_kernel<false><<<grid, kPermuteThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_dispatch_count(const PermuteArgs& a, int num_sms, cudaStream_t stream) {
    if (a.T == 0) return cudaSuccess;
    int grid = num_sms;
    if (grid > a.T) grid = a.T;
    const bool v8 = rows_v8(a.x, a.xp);
    if (a.R > 0) {
        const int smem = static_cast<int>(sizeof(CountPlanSmem));
        auto kern = v8 ? dispatch_count_kernel<true, true> : dispatch_count_kernel<true, false>;
        const cudaError_t err = set_max_dynamic_smem(kern, smem);
        if (err != cudaSuccess) return err;
        kern<<<grid, kCountThreads, smem, stream>>>(a);
    } else {
        auto kern = v8 ? dispatch_count_kernel<false, true> : dispatch_count_kernel<false, false>;
        kern<<<grid, kCountThreads, 0, stream>>>(a);
    }
    return cudaGetLastError();
}

size_t reroute_ws_bytes(int T, int k) {
    auto up = [](size_t b) { return (b + 255) & ~size_t(255); };
    const size_t tk = static_cast<size_t>(T) * k;
    (void)tk;
    return 256 + up(static_cast<size_t>(T) * kMaxExperts) + up(size_t(2) * kRerouteMaxCtas * kMaxExperts * sizeof(int32_t));
}

cudaError_t launch_reroute(const RerouteArgs& a0, void* ws, const __nv_bfloat16* x, __nv_bfloat16* xp, int d,
                           int num_sms, cudaStream_t stream) {
    if (a0.T == 0) return cudaSuccess;
    RerouteArgs a = a0;
    const size_t tk = static_cast<size_t>(a.T) * a.k;
    uint8_t* p = static_cast<uint8_t*>(ws) + 256;
    auto take = [&](size_t bytes) { uint8_t* r = p; p += (bytes + 255) & ~size_t(255); return r; };
    a.cand_stride = (a.E + 15) & ~15;  // <= kMaxExperts bytes per token, as reroute_ws_bytes reserves
    a.cand = take(static_cast<size_t>(a.T) * a.cand_stride);
    {
        int grid = (a.T + 7) / 8;
        if (grid > 8 * num_sms) grid = 8 * num_sms;
        const int st = a.cand_stride;
        if (a.E <= 32) candidate_order_kernel<1><<<grid, 256, 0, stream>>>(a.logits, a.T, a.E, st, a.cand);
        else if (a.E <= 64) candidate_order_kernel<2><<<grid, 256, 0, stream>>>(a.logits, a.T, a.E, st, a.cand);
        else if (a.E <= 128) candidate_order_kernel<4><<<grid, 256, 0, stream>>>(a.logits, a.T, a.E, st, a.cand);
        else candidate_order_kernel<8><<<grid, 256, 0, stream>>>(a.logits, a.T, a.E, st, a.cand);
        const cudaError_t e0 = cudaGetLastError();
        if (e0 != cudaSuccess) return e0;
    }
    a.xchg = reinterpret_cast<int32_t*>(take(size_t(2) * kRerouteMaxCtas * kMaxExperts * sizeof(int32_t)));
    a.bar = static_cast<uint32_t*>(ws);  // the first 8 bytes of the workspace header
    // the rounds over about one CTA per SM (fewer for few pairs), co-resident by a cooperative launch
    const int smem = static_cast<int>(reroute_smem_bytes());
    cudaError_t err = set_max_dynamic_smem(reroute_grid_kernel, smem);
    if (err != cudaSuccess) return err;
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, reroute_grid_kernel, kRerouteThreads, smem);
    if (err != cudaSuccess) return err;
    int G = (static_cast<int>(tk) + kRerouteThreads - 1) / kRerouteThreads;
    if (G > a.T) G = a.T;  // every CTA owns whole tokens
    const int resident = num_sms * (per_sm > 1 ? per_sm : 1);
    if (G > resident) G = resident;
    if (G > kRerouteMaxCtas) G = kRerouteMaxCtas;
    if (G < 1) G = 1;
    // every CTA's slice fits its shared memory (with T*k <= kRerouteMaxPairs and one CTA on each of
    // at least 128 SMs, a slice holds at most 4096 + k pairs)
    if (static_cast<int64_t>((a.T + G - 1) / G) * a.k > kRerouteSliceMax) return cudaErrorInvalidValue;
    err = cudaMemsetAsync(a.bar, 0, 2 * sizeof(uint32_t), stream);
    if (err != cudaSuccess) return err;
    void* kargs[] = {&a};
    err = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(reroute_grid_kernel), dim3(G),
                                      dim3(kRerouteThreads), kargs, static_cast<size_t>(smem), stream);
    if (err != cudaSuccess) return err;
    int sgrid = (a.T + 7) / 8;
    if (sgrid > 16 * num_sms) sgrid = 16 * num_sms;
    if (rows_v8(x, xp)) scatter_rows_kernel<true><<<sgrid, 256, 0, stream>>>(x, a.dest, a.T, a.k, d, a.rows, xp);
    else scatter_rows_kernel<false><<<sgrid, 256, 0, stream>>>(x, a.dest, a.T, a.k, d, a.rows, xp);
    return cudaGetLastError();
}

cudaError_t launch_route_from_logits(const float* logits, int T, int E, int k, int route_flags, int32_t* ids,
                                     float* w, int num_sms, cudaStream_t stream) {
    return launch_route_logits(logits, 1, E, 0, nullptr, T, E, k, route_flags, nullptr, ids, w, nullptr, num_sms,
                               stream);
}

cudaError_t launch_route_logits(const float* part, int n_split, int ldp, size_t split_stride, const float* bias, int T,
                                int E, int k, int route_flags, float* logits, int32_t* ids, float* w, float* scores_t,
                                int num_sms, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    // one warp per token, grid-stride; at most four 256-thread CTAs per SM, so one wave
    int grid = (T + 7) / 8;
    if (grid > 4 * num_sms) grid = 4 * num_sms;
    using Kern = void (*)(const float*, int, int, size_t, const float*, int, int, int, int, float*, int32_t*, float*,
                          float*);
    // the loops bounded by E rounded up to 32, 64, 128 or 256 experts and by k rounded up to 2, 4 or 8
    static const Kern table[4][3] = {
        {route_logits_kernel<1, 2>, route_logits_kernel<1, 4>, route_logits_kernel<1, 8>},
        {route_logits_kernel<2, 2>, route_logits_kernel<2, 4>, route_logits_kernel<2, 8>},
        {route_logits_kernel<4, 2>, route_logits_kernel<4, 4>, route_logits_kernel<4, 8>},
        {route_logits_kernel<8, 2>, route_logits_kernel<8, 4>, route_logits_kernel<8, 8>}};
    const int ui = E <= 32 ? 0 : (E <= 64 ? 1 : (E <= 128 ? 2 : 3));
    const int ki = k <= 2 ? 0 : (k <= 4 ? 1 : 2);
    table[ui][ki]<<<grid, 256, 0, stream>>>(part, n_split, ldp, split_stride, bias, T, E, k, route_flags, logits, ids,
                                            w, scores_t);
    return cudaGetLastError();
}

}  // namespace moe
