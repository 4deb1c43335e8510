// Dispatch kernels: histogram, segment tables (plain or balanced plan), the stable
// rank of every (token, k) pair inside its expert, and the scatter that writes each
// token row straight into its k final expert-contiguous slots.
//
// The permutation is a counting sort on the expert id with one digit pass: the
// global histogram is known beforehand (histogram_kernel), and the rank of a
// pair inside its expert is (pairs of that expert in earlier tiles) + (earlier
// pairs of the same tile).  The first term is an exclusive prefix over tiles,
// found with a decoupled look-back (Merrill & Garland, "Single-pass Parallel
// Prefix Scan with Decoupled Look-back", 2016): each tile publishes its own
// per-expert counts at once and its inclusive prefix as soon as it knows it,
// so a tile only waits for tiles already running.  Tiles are taken in order
// from an atomic ticket, which guarantees that every tile a CTA waits for is
// held by a CTA that is running.  Every wait is bounded.
//
// Sources: "Sparsely-Gated MoE 구현 관점에서 살펴보기", section "순전파 과정 ..."
// (permute tokens into expert order); "5.3 Expert Parallelism", section
// "2. 디스패처 엔지니어링" (bincount per destination); the MoonEP page, sections
// "이 기술은 무엇인가" (rows written to their final slot, no separate sort and
// copy; static shapes, no host sync) and "설치 및 통합" (tokens_per_expert,
// cu_seqlens).
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr uint32_t kFlagAggregate = 1u << 30;
constexpr uint32_t kFlagPrefix = 2u << 30;
constexpr uint32_t kValueMask = (1u << 30) - 1;
constexpr int kPermuteWarps = kPermuteThreads / 32;
constexpr int kCopyUnroll = 8;

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

constexpr int kMaxGroups = 256;

__global__ void __launch_bounds__(256) plan_kernel(int32_t* counts, const int32_t* partials, int n_partials, int E,
                                                   int R, int S, int k, int B, int32_t* seg_expert,
                                                   int32_t* seg_offsets, int32_t* seg_first_rank, int32_t* status) {
    __shared__ int c[kMaxExperts];
    __shared__ int order[kMaxExperts];  // experts of each group by (count desc, id asc)
    __shared__ int given[kMaxExperts];  // rows an expert hands to other groups
    __shared__ int next_rank[kMaxExperts];
    __shared__ int qe[kMaxExperts], qn[kMaxExperts];  // the donor queue
    __shared__ int load[kMaxGroups];
    __shared__ int n_slots[kMaxGroups];
    __shared__ int slot_e[kMaxSegments], slot_n[kMaxSegments], slot_r[kMaxSegments];
    __shared__ int seg_len[kMaxSegments];
    __shared__ int warp_sums[8];
    __shared__ int infeasible;

    const int tid = threadIdx.x;
    const int epg = E / R;
    const int per_group = epg + B;
    const int n_seg = R * per_group;
    const int cap = S * k;

    for (int e = tid; e < E; e += blockDim.x) {
        c[e] = expert_count(counts, partials, n_partials, E, e, counts);
        given[e] = 0;
    }
    __syncthreads();
    for (int g = tid; g < R; g += blockDim.x) {
        int s = 0;
        for (int e = g * epg; e < (g + 1) * epg; ++e) s += c[e];
        load[g] = s;
    }
    for (int e = tid; e < E; e += blockDim.x) {
        const int g = e / epg;
        int rank = 0;
        for (int o = g * epg; o < (g + 1) * epg; ++o) rank += (c[o] > c[e]) || (c[o] == c[e] && o < e);
        order[g * epg + rank] = e;
    }
    __syncthreads();

    if (tid == 0) {
        // the queue of excess rows, groups ascending, experts by (count desc, id asc)
        int nq = 0, total = 0;
        for (int g = 0; g < R; ++g) total += load[g];
        int bad = (total != R * cap);
        for (int g = 0; g < R; ++g) {
            int excess = load[g] - cap;
            for (int i = 0; i < epg && excess > 0; ++i) {
                const int e = order[g * epg + i];
                const int take = c[e] < excess ? c[e] : excess;
                if (take > 0) { given[e] = take; qe[nq] = e; qn[nq] = take; ++nq; excess -= take; }
            }
        }
        // groups below the cap, ascending, take from the front of the queue
        int head = 0;
        for (int g = 0; g < R; ++g) {
            int deficit = cap - load[g];
            int ns = 0;
            while (deficit > 0 && head < nq) {
                const int take = qn[head] < deficit ? qn[head] : deficit;
                if (ns < B) { slot_e[g * B + ns] = qe[head]; slot_n[g * B + ns] = take; }
                ++ns;
                qn[head] -= take;
                deficit -= take;
                if (qn[head] == 0) ++head;
            }
            if (ns > B || deficit > 0) bad = 1;
            n_slots[g] = ns < B ? ns : B;
        }
        // within-expert rank at which each piece starts: after the home rows, in creation order
        for (int e = 0; e < E; ++e) next_rank[e] = c[e] - given[e];
        for (int g = 0; g < R; ++g)
            for (int i = 0; i < n_slots[g]; ++i) {
                const int idx = g * B + i;
                slot_r[idx] = next_rank[slot_e[idx]];
                next_rank[slot_e[idx]] += slot_n[idx];
            }
        infeasible = bad;
        if (bad) report(status, MOE_DEV_ERR_PLAN);
    }
    __syncthreads();

    const bool bad = infeasible != 0;
    for (int s = tid; s < n_seg; s += blockDim.x) {
        const int g = s / per_group, i = s - g * per_group;
        int ex = -1, len = 0, fr = 0;
        if (!bad) {
            if (i < epg) {
                ex = g * epg + i;
                len = c[ex] - given[ex];
            } else if (i - epg < n_slots[g]) {
                const int idx = g * B + (i - epg);
                ex = slot_e[idx];
                len = slot_n[idx];
                fr = slot_r[idx];
            }
        }
        seg_expert[s] = ex;
        seg_first_rank[s] = fr;
        seg_len[s] = len;
    }
    __syncthreads();
    // offsets: exclusive scan of the lengths, each thread owning a contiguous chunk
    const int chunk = (n_seg + blockDim.x - 1) / blockDim.x;
    const int a = tid * chunk;
    int local = 0;
    for (int s = a; s < a + chunk && s < n_seg; ++s) local += seg_len[s];
    int total;
    int run = block_exclusive_scan_256(local, warp_sums, &total);
    for (int s = a; s < a + chunk && s < n_seg; ++s) {
        seg_offsets[s] = run;
        run += seg_len[s];
    }
    if (tid == 0) seg_offsets[n_seg] = total;
}

// ------------------------------------------------------------------------------ stable rank + permute

__global__ void __launch_bounds__(kPermuteThreads) rank_kernel(const PermuteArgs a) {
    __shared__ int s_wcnt[kPermuteWarps][kMaxExperts];
    __shared__ int s_excl[kMaxExperts];
    __shared__ int s_cbeg[kMaxExperts + 1];
    __shared__ int s_cseg[kMaxSegments];
    __shared__ int warp_sums[8];
    __shared__ int s_tile;
    __shared__ int s_abort;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = a.E, k = a.k;

    // segments of each expert (CSR in shared memory); order inside an expert does not matter
    if (tid < E) s_excl[tid] = 0;
    if (tid == 0) s_abort = 0;
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

    const unsigned lanemask_lt = (1u << lane) - 1u;

    for (;;) {
        if (tid == 0) s_tile = static_cast<int>(atomicAdd(a.ticket, 1u)) + a.first_tile;
        for (int i = tid; i < kPermuteWarps * kMaxExperts; i += blockDim.x) (&s_wcnt[0][0])[i] = 0;
        __syncthreads();
        const int tile = s_tile;
        if (tile >= a.n_tiles || s_abort) break;

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
        const int wrank = __popc(same & lanemask_lt);
        if (e >= 0 && wrank == 0) s_wcnt[warp][e] = __popc(same);
        __syncthreads();

        // 2. tile histogram, publish, look back, publish the inclusive prefix
        if (tid < E) {
            int h = 0;
#pragma unroll
            for (int w = 0; w < kPermuteWarps; ++w) h += s_wcnt[w][tid];
            uint32_t* mine = a.tile_state + static_cast<size_t>(tile) * E + tid;
            int excl = 0;
            if (tile == 0) {
                st_relaxed_u32(mine, kFlagPrefix | static_cast<uint32_t>(h));
            } else {
                st_relaxed_u32(mine, kFlagAggregate | static_cast<uint32_t>(h));
                int j = tile - 1;
                uint64_t t_start = 0;
                uint32_t spins = 0;
                bool gave_up = false;
                while (j >= 0) {
                    const uint32_t w = ld_relaxed_u32(a.tile_state + static_cast<size_t>(j) * E + tid);
                    const uint32_t flag = w & ~kValueMask;
                    if (flag == 0) {
                        if ((++spins & 63u) == 0) {
                            const uint64_t now = globaltimer_ns();
                            if (t_start == 0) t_start = now;
                            else if (now - t_start > kWaitLimitNs) {
                                report(a.status, MOE_DEV_ERR_TIMEOUT);
                                s_abort = 1;
                                gave_up = true;
                                break;
                            }
                        }
                        continue;
                    }
                    excl += static_cast<int>(w & kValueMask);
                    if (flag == kFlagPrefix) break;
                    --j;
                }
                // a tile that gave up publishes no prefix, so the tiles after it give up too
                if (!gave_up) st_relaxed_u32(mine, kFlagPrefix | static_cast<uint32_t>(excl + h));
            }
            s_excl[tid] = excl;
        }
        __syncthreads();
        if (s_abort) break;

        // 3. final slot of each pair
        if (tid < nq) {
            int dst = -1;
            if (e >= 0) {
                int r = s_excl[e] + wrank;
                for (int w = 0; w < warp; ++w) r += s_wcnt[w][e];
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

        __syncthreads();
    }
}

// ------------------------------------------------------------------------------ row scatter

// One warp per token: read the token's row of X once (16-byte vectors, 8 in flight per lane)
// and write it to each of its k final slots.  Pure streaming: no shared memory, no barriers.
__global__ void __launch_bounds__(256) scatter_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                           const int32_t* __restrict__ dest, int T, int k, int d,
                                                           int rows, __nv_bfloat16* __restrict__ xp) {
    const int lane = threadIdx.x & 31;
    const int warps_total = gridDim.x * (blockDim.x >> 5);
    const int vec_per_row = d / 8;
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps_total) {
        const int mine = lane < k ? __ldg(dest + static_cast<size_t>(t) * k + lane) : -1;
        int dj[kMaxTopK];
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) dj[j] = __shfl_sync(0xffffffffu, mine, j);
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
}

// ------------------------------------------------------------------------------ top-k from given logits

__global__ void __launch_bounds__(256) route_from_logits_kernel(const float* __restrict__ logits, int T, int E,
                                                                int k, int route_flags, int32_t* __restrict__ ids,
                                                                float* __restrict__ w) {
    const int lane = threadIdx.x & 31;
    const int warps_total = gridDim.x * (blockDim.x >> 5);
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps_total) {
        float v[kMaxExperts / 32];
        unsigned taken = 0;
#pragma unroll
        for (int u = 0; u < kMaxExperts / 32; ++u) {
            const int e = lane + 32 * u;
            v[u] = e < E ? __ldg(logits + static_cast<size_t>(t) * E + e) : -INFINITY;
            if (e >= E) taken |= 1u << u;
        }
        float sv[kMaxTopK];
        int si[kMaxTopK];
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            sv[j] = 0.f;
            si[j] = 0;
            if (j < k) {
                float bv = -INFINITY;
                int bi = 0x7fffffff;
#pragma unroll
                for (int u = 0; u < kMaxExperts / 32; ++u) {
                    const int e = lane + 32 * u;
                    if (!((taken >> u) & 1u) && (v[u] > bv || (v[u] == bv && e < bi))) { bv = v[u]; bi = e; }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                    if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
                }
                if (bi < E && (bi & 31) == lane) taken |= 1u << (bi >> 5);
                sv[j] = bv;
                si[j] = bi;
            }
        }
        // denominator over all E logits (softmax-all mode), shifted by the largest (sv[0])
        float all = 0.f;
        if (route_flags & MOE_ROUTE_SOFTMAX_ALL) {
#pragma unroll
            for (int u = 0; u < kMaxExperts / 32; ++u)
                if (lane + 32 * u < E) all += expf(v[u] - sv[0]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) all += __shfl_xor_sync(0xffffffffu, all, o);
        }
        if (lane == 0) {
            float ex[kMaxTopK], sum = 0.f;
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j) {
                ex[j] = j < k ? expf(sv[j] - sv[0]) : 0.f;
                sum += ex[j];
            }
            const float inv = 1.0f / ((route_flags & MOE_ROUTE_SOFTMAX_ALL) ? all : sum);
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j)
                if (j < k) {
                    ids[static_cast<size_t>(t) * k + j] = si[j];
                    w[static_cast<size_t>(t) * k + j] = ex[j] * inv;
                }
        }
    }
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
    scatter_rows_kernel<<<sgrid, 256, 0, stream>>>(a.x, a.dest, a.T, a.k, a.d, a.rows, a.xp);
    return cudaGetLastError();
}

cudaError_t launch_route_from_logits(const float* logits, int T, int E, int k, int route_flags, int32_t* ids,
                                     float* w, int num_sms, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    int grid = (T + 7) / 8;
    if (grid > 8 * num_sms) grid = 8 * num_sms;
    route_from_logits_kernel<<<grid, 256, 0, stream>>>(logits, T, E, k, route_flags, ids, w);
    return cudaGetLastError();
}

}  // namespace moe
