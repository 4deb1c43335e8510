// Expert parallelism over R ranks (one GPU each): the balanced plan's R groups become R ranks.
//
// Rank g holds the E/R experts homed in group g plus B replica weight slots ([E/R + B, F, d]
// per weight matrix), and receives exactly S*k dispatched rows (its group's rows of the
// single-GPU balanced layout).  A step of the layer on rank g:
//   1. route its S tokens and count their experts (the single-GPU calls);
//   2. exchange the counts: counts_all [R, E] (a collective of the caller's choosing);
//   3. ep_plan_kernel: the same deterministic plan on every rank, from counts_all; rank g keeps
//      its group's segment tables;
//   4. ep_prefetch_kernel: the weights of the experts its replica slots serve are copied from
//      their home ranks (peer loads) into its replica slots;
//   5. ep_dispatch_kernel: every pair's final slot on its owning rank, and the token's row
//      stored straight into that slot (peer stores);
//   6. after a barrier, the grouped GEMMs on the rank's own S*k rows and own weight slots;
//   7. after a barrier, ep_combine_kernel: each token's k output rows read back from their
//      owners (peer loads) and summed with the router weights.
// The destination of every row is the one of the single-GPU balanced plan over the R*S tokens
// in rank order, so R ranks reproduce that layout exactly (the owner's rows are rows
// [g*S*k, (g+1)*S*k) of the single-GPU Xp).
//
// No kernel here waits for another rank: the barriers are stream-ordered collectives between
// launches.  With fewer GPUs than ranks, one launch can serve several source ranks (n_src > 1),
// with the "peer" buffers all in local memory.  No TMA and no multicast: peer memory is only
// touched by plain 16-byte loads and stores.
//
// Sources: the MoonEP page ("가장 바쁜 랭크가 속도를 정합니다: MoonEP의 계획 코드를 직접
// 돌려봤습니다"), sections "이 기술은 무엇인가" (each row written to its final position on the
// receiving rank, static S x K shapes, no host sync), "설치 및 통합" (Buffer.dispatch /
// prefetch_weight / combine; replica weight slots [E, E+B)) and "실제 실험 결과" (the memory each
// rank holds); "5.3 Expert Parallelism", section "2. 디스패처 엔지니어링" (exchange the counts,
// then the tokens).
#include "common.cuh"
#include "kernels.h"
#include "vec.cuh"
#include "plan.cuh"

namespace moe {

namespace {

constexpr int kEpThreads = 1024;
constexpr int kEpWarps = kEpThreads / 32;
constexpr int kEpCountBatch = 8;
constexpr int kEpCopyUnroll = 8;

// Dynamic shared memory of the dispatch: the plan over all groups, its segment tables, each
// expert's segments (CSR) and the pairs of each expert on the source ranks before this one.
struct EpSmem {
    PlanSmem plan;
    int seg_e[kMaxSegments], seg_fr[kMaxSegments], seg_off[kMaxSegments + 1];
    int cbeg[kMaxExperts + 1], cfill[kMaxExperts], cseg[kMaxSegments];
    int pre[kMaxExperts];
};

// Dynamic shared memory of the plan kernel.
struct EpPlanSmem {
    PlanSmem plan;
    int seg_e[kMaxSegments], seg_fr[kMaxSegments], seg_off[kMaxSegments + 1];
};

// plan.c[e] = total pairs of expert e over the R ranks; pre[e] (if non-null) = those of the
// ranks before `rank`.
__device__ __forceinline__ void ep_totals(const int32_t* counts_all, int R, int E, int rank, int* c, int* pre) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int tot = 0, before = 0;
        for (int r = 0; r < R; ++r) {
            const int v = __ldg(counts_all + static_cast<size_t>(r) * E + e);
            tot += v;
            if (r < rank) before += v;
        }
        c[e] = tot;
        if (pre) pre[e] = before;
    }
}

// ------------------------------------------------------------------------------ plan of one rank

__global__ void __launch_bounds__(256) ep_plan_kernel(const int32_t* __restrict__ counts_all, int R, int S, int k,
                                                      int E, int B, int rank, int32_t* counts, int32_t* seg_expert,
                                                      int32_t* seg_slot, int32_t* seg_offsets, int32_t* status) {
    extern __shared__ __align__(16) uint8_t ep_plan_dsmem[];
    EpPlanSmem& ps = *reinterpret_cast<EpPlanSmem*>(ep_plan_dsmem);
    ep_totals(counts_all, R, E, rank, ps.plan.c, nullptr);
    __syncthreads();
    compute_plan(ps.plan, E, R, S, k, B, ps.seg_e, ps.seg_off, ps.seg_fr, status, true);
    const int per_group = E / R + B;
    const int s0 = rank * per_group;
    const int row0 = ps.seg_off[s0];
    for (int i = threadIdx.x; i < per_group; i += blockDim.x) {
        const int ex = ps.seg_e[s0 + i];
        const bool live = ex >= 0 && ps.seg_off[s0 + i + 1] > ps.seg_off[s0 + i];
        seg_expert[i] = ex;
        seg_slot[i] = live ? i : -1;
        seg_offsets[i] = ps.seg_off[s0 + i] - row0;
    }
    if (threadIdx.x == 0) seg_offsets[per_group] = ps.seg_off[s0 + per_group] - row0;
    if (counts)
        for (int e = threadIdx.x; e < E; e += blockDim.x) counts[e] = ps.plan.c[e];
}

// ------------------------------------------------------------------------------ replica weights

// The copies of this rank's replica slots as one flat list of work items (used slot u, matrix m,
// chunk c of kPrefetchChunkBytes), taken by the CTAs in turn.  Each CTA first lists the slots in
// use (a segment with rows) and their experts in shared memory, so an item starts its copy with no
// dependent load.  An item copies its chunk of expert e's matrix m from slot e - h*E/R of e's home
// rank h into this rank's slot E/R + j.  So however few slots are in use, every CTA of the grid
// streams their bytes: 32-byte vectors (16-byte ones when a weight buffer is not 32-byte aligned),
// four per thread in flight.
constexpr int kPrefetchChunkBytes = 32768;

template <bool V8>
__global__ void __launch_bounds__(256) ep_prefetch_kernel(const __grid_constant__ EpPrefetchArgs a) {
    __shared__ int s_slot[kMaxSegments];    // replica slots in use, in slot order
    __shared__ int s_expert[kMaxSegments];  // and their experts
    __shared__ int s_n;
    const int epg = a.E / a.R;
    if (threadIdx.x < 32) {
        int n = 0;
        for (int j0 = 0; j0 < a.B; j0 += 32) {
            const int j = j0 + static_cast<int>(threadIdx.x);
            int e = -1;
            if (j < a.B) {
                const int sg = epg + j;
                e = __ldg(a.seg_expert + sg);
                if (e >= a.E || __ldg(a.seg_offsets + sg + 1) <= __ldg(a.seg_offsets + sg)) e = -1;
            }
            const unsigned b = __ballot_sync(0xffffffffu, e >= 0);
            if (e >= 0) {
                const int pos = n + __popc(b & ((1u << threadIdx.x) - 1u));
                s_slot[pos] = j;
                s_expert[pos] = e;
            }
            n += __popc(b);
        }
        if (threadIdx.x == 0) s_n = n;
    }
    __syncthreads();
    constexpr int VB = V8 ? 32 : 16;                    // bytes per vector
    constexpr int kChunk = kPrefetchChunkBytes / VB;    // vectors per work item
    const size_t mat = static_cast<size_t>(a.F) * a.d;  // elements of one expert's matrix
    const size_t nvec = mat * 2 / VB;                   // F*d is a multiple of 4096
    const int chunks = static_cast<int>((nvec + kChunk - 1) / kChunk);
    const int64_t items = static_cast<int64_t>(s_n) * 3 * chunks;
    for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
        const int c = static_cast<int>(it % chunks);
        const int m = static_cast<int>((it / chunks) % 3);
        const int u = static_cast<int>(it / (3 * static_cast<int64_t>(chunks)));
        const int sg = epg + s_slot[u];
        const int e = s_expert[u];
        const int h = e / epg;
        const uint8_t* src = reinterpret_cast<const uint8_t*>(a.w[m][h] + static_cast<size_t>(e - h * epg) * mat);
        uint8_t* dst = reinterpret_cast<uint8_t*>(a.w[m][a.rank] + static_cast<size_t>(sg) * mat);
        const size_t v0 = static_cast<size_t>(c) * kChunk;
        const size_t v1 = v0 + kChunk < nvec ? v0 + kChunk : nvec;
        size_t v = v0 + threadIdx.x;
        if constexpr (V8) {
            for (; v + 3 * 256 < v1; v += 4 * 256) {
                const Vec32 a0 = ld_nc_v8(src + v * 32), a1 = ld_nc_v8(src + (v + 256) * 32);
                const Vec32 a2 = ld_nc_v8(src + (v + 512) * 32), a3 = ld_nc_v8(src + (v + 768) * 32);
                st_v8(dst + v * 32, a0);
                st_v8(dst + (v + 256) * 32, a1);
                st_v8(dst + (v + 512) * 32, a2);
                st_v8(dst + (v + 768) * 32, a3);
            }
            for (; v < v1; v += 256) st_v8(dst + v * 32, ld_nc_v8(src + v * 32));
        } else {
            const uint4* s4 = reinterpret_cast<const uint4*>(src);
            uint4* d4 = reinterpret_cast<uint4*>(dst);
            for (; v + 3 * 256 < v1; v += 4 * 256) {
                const uint4 a0 = __ldg(s4 + v), a1 = __ldg(s4 + v + 256);
                const uint4 a2 = __ldg(s4 + v + 512), a3 = __ldg(s4 + v + 768);
                d4[v] = a0;
                d4[v + 256] = a1;
                d4[v + 512] = a2;
                d4[v + 768] = a3;
            }
            for (; v < v1; v += 256) d4[v] = __ldg(s4 + v);
        }
    }
}

// ------------------------------------------------------------------------------ dispatch

// Copy token row xs (d bf16) to the k destinations dst[0..k) (null: none), one warp: V8 (every
// row 32-byte aligned) 32-byte vectors, kEpCopyUnroll / 2 in flight per lane, else 16-byte
// vectors, kEpCopyUnroll in flight.
template <bool V8>
__device__ __forceinline__ void ep_copy_row(const __nv_bfloat16* __restrict__ xs, __nv_bfloat16* const* dst, int k,
                                            int d, int lane) {
    bool any = false;
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) any |= (j < k && dst[j] != nullptr);
    if (!any) return;
    if constexpr (V8) {
        constexpr int U = kEpCopyUnroll / 2;
        const int vec_per_row = d / 16;
        const uint8_t* s = reinterpret_cast<const uint8_t*>(xs);
        for (int v = lane; v < vec_per_row; v += 32 * U) {
            Vec32 val[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (v + 32 * u < vec_per_row) val[u] = ld_nc_v8(s + static_cast<size_t>(v + 32 * u) * 32);
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j) {
                if (j < k && dst[j] != nullptr) {
                    uint8_t* o = reinterpret_cast<uint8_t*>(dst[j]);
#pragma unroll
                    for (int u = 0; u < U; ++u)
                        if (v + 32 * u < vec_per_row) st_v8(o + static_cast<size_t>(v + 32 * u) * 32, val[u]);
                }
            }
        }
    } else {
        const int vec_per_row = d / 8;
        const uint4* s = reinterpret_cast<const uint4*>(xs);
        for (int v = lane; v < vec_per_row; v += 32 * kEpCopyUnroll) {
            uint4 val[kEpCopyUnroll];
#pragma unroll
            for (int u = 0; u < kEpCopyUnroll; ++u)
                if (v + 32 * u < vec_per_row) val[u] = __ldg(s + v + 32 * u);
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j) {
                if (j < k && dst[j] != nullptr) {
                    uint4* o = reinterpret_cast<uint4*>(dst[j]);
#pragma unroll
                    for (int u = 0; u < kEpCopyUnroll; ++u)
                        if (v + 32 * u < vec_per_row) o[v + 32 * u] = val[u];
                }
            }
        }
    }
}

// One launch serves n_src source ranks with ctas_per_src CTAs each.  A CTA of source rank r owns
// two blocks of r's tokens (one from the front, one from the back) and
//  1. counts r's expert ids in shared memory, split at the starts of its two blocks;
//  2. computes the plan over all ranks from counts_all (every CTA of every rank alike) and the
//     pairs of each expert on the ranks before r;
//  3. gives each pair of its blocks its rank among all pairs of its expert in global order
//     (rank-major, then q = t*k + j), finds the segment that holds that rank and so the pair's
//     owner and row there; writes dest (owner * S*k + row) and the owner's src (global pair
//     index, a peer store);
//  4. stores each token's row into its k slots on their owners (peer stores).
template <bool V8>
__global__ void __launch_bounds__(kEpThreads, 1) ep_dispatch_kernel(const __grid_constant__ EpDispatchArgs a) {
    extern __shared__ __align__(16) uint8_t ep_dsmem[];
    EpSmem& ps = *reinterpret_cast<EpSmem*>(ep_dsmem);
    __shared__ int s_a[kMaxExperts];    // pairs of each expert before the first block
    __shared__ int s_m[kMaxExperts];    // ... from the first block up to the second
    __shared__ int s_tot[kMaxExperts];  // ... from the second block on
    __shared__ int s_run[kMaxExperts];  // pairs of each expert before the current chunk
    __shared__ int s_wcnt[kEpWarps][kMaxExperts];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int i_src = blockIdx.x / a.ctas_per_src;
    const int G = a.ctas_per_src;
    const int b = blockIdx.x - i_src * G;
    const int rank = a.src0 + i_src;
    const int E = a.E, k = a.k, T = a.S;
    const int cap = a.S * k;
    const int total_rows = a.R * cap;
    const int32_t* __restrict__ ids = a.ids[i_src];
    const unsigned lanemask_lt = (1u << lane) - 1u;
    const int n = T * k;
    const int tb = (T + 2 * G - 1) / (2 * G);
    int tb_[2], te_[2];
    {
        const int blk[2] = {b, 2 * G - 1 - b};
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            tb_[r] = min(T, blk[r] * tb);
            te_[r] = min(T, tb_[r] + tb);
        }
    }
    const int q1 = tb_[0] * k, q2 = tb_[1] * k;

    for (int i = tid; i < E; i += blockDim.x) { s_a[i] = 0; s_m[i] = 0; s_tot[i] = 0; }
    for (int i = tid; i < kEpWarps * kMaxExperts; i += blockDim.x) (&s_wcnt[0][0])[i] = 0;
    ep_totals(a.counts_all, a.R, E, rank, ps.plan.c, ps.pre);
    __syncthreads();

    // 1. this source rank's pairs, split at the starts of the two blocks
    for (int base = 0; base < n; base += blockDim.x * kEpCountBatch) {
        int ev[kEpCountBatch];
#pragma unroll
        for (int u = 0; u < kEpCountBatch; ++u) {
            const int i = base + u * blockDim.x + tid;
            ev[u] = i < n ? __ldg(ids + i) : -1;
        }
#pragma unroll
        for (int u = 0; u < kEpCountBatch; ++u) {
            const int i = base + u * blockDim.x + tid;
            const int e = ev[u];
            if (static_cast<unsigned>(e) < static_cast<unsigned>(E))
                atomicAdd(i < q1 ? &s_a[e] : (i < q2 ? &s_m[e] : &s_tot[e]), 1);
        }
    }

    // 2. the plan over all ranks (the first CTA of the launch reports an infeasible plan)
    compute_plan(ps.plan, E, a.R, a.S, k, a.B, ps.seg_e, ps.seg_off, ps.seg_fr, a.status, blockIdx.x == 0);
    if (blockIdx.x == 0 && a.seg_offsets_out != nullptr) {
        for (int e = tid; e < E; e += blockDim.x) a.counts_out[e] = ps.plan.c[e];
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
    for (int sg = tid; sg < a.n_seg; sg += blockDim.x) {
        const int ex = ps.seg_e[sg];
        if (static_cast<unsigned>(ex) < static_cast<unsigned>(E) && ps.seg_off[sg + 1] > ps.seg_off[sg])
            ps.cseg[atomicAdd(&ps.cfill[ex], 1)] = sg;
    }
    __syncthreads();

    // 3. global ranks of the pairs of each block, their owners and rows
    int32_t* __restrict__ dest = a.dest[i_src];
    const int q_base = rank * n;  // global index of this rank's first pair
#pragma unroll 1
    for (int r = 0; r < 2; ++r) {
        if (r == 1 && tb_[1] == tb_[0]) break;
        for (int x = tid; x < E; x += blockDim.x) s_run[x] = ps.pre[x] + (r == 0 ? s_a[x] : s_a[x] + s_m[x]);
        __syncthreads();
        const int qb = tb_[r] * k, qe = te_[r] * k;
        for (int q0 = qb; q0 < qe; q0 += blockDim.x) {
            const int q = q0 + tid;
            int e = -1;
            if (q < qe) {
                e = __ldg(ids + q);
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
                    for (int p = ps.cbeg[e]; p < ps.cbeg[e + 1]; ++p) {
                        const int sg = ps.cseg[p];
                        const int fr = ps.seg_fr[sg], off = ps.seg_off[sg], len = ps.seg_off[sg + 1] - off;
                        if (rk >= fr && rk < fr + len) { dst = off + (rk - fr); break; }
                    }
                    if (dst >= total_rows) dst = -1;
                }
                dest[q] = dst;
                if (dst >= 0) {
                    const int owner = dst / cap;
                    a.src[owner][dst - owner * cap] = q_base + q;
                }
            }
            __syncthreads();
            for (int x = tid; x < E; x += blockDim.x) {
                int c = 0;
                for (int w = 0; w < kEpWarps; ++w) { c += s_wcnt[w][x]; s_wcnt[w][x] = 0; }
                s_run[x] += c;
            }
            __syncthreads();
        }
    }

    // 4. rows of this CTA's tokens into their owners' slots: both blocks form one list over all warps
    {
        const __nv_bfloat16* __restrict__ x = a.x[i_src];
        const int n0 = te_[0] - tb_[0];
        const int n1 = tb_[1] == tb_[0] ? 0 : te_[1] - tb_[1];
        for (int i = warp; i < n0 + n1; i += kEpWarps) {
            const int t = i < n0 ? tb_[0] + i : tb_[1] + (i - n0);
            __nv_bfloat16* mine = nullptr;
            if (lane < k) {
                const int dr = dest[static_cast<size_t>(t) * k + lane];
                if (dr >= 0 && dr < total_rows) {
                    const int owner = dr / cap;
                    mine = a.xp[owner] + static_cast<size_t>(dr - owner * cap) * a.d;
                }
            }
            __nv_bfloat16* dj[kMaxTopK];
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j)
                dj[j] = reinterpret_cast<__nv_bfloat16*>(
                    __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(mine), j));
            ep_copy_row<V8>(x + static_cast<size_t>(t) * a.d, dj, k, a.d, lane);
        }
    }
    // the stores above may go to other GPUs: make them visible system-wide before the kernel ends,
    // so that whatever synchronisation follows the kernel on this stream also follows them
    __threadfence_system();
}

// Pairs of each expert in each token group: the CTAs of group g (blockIdx.x / per_group) each
// count a slice of the group's S*k ids in shared memory (16-byte loads when aligned) and add their
// nonzero counts to counts_all[g][e], which the launcher clears first.
__global__ void __launch_bounds__(kEpThreads) group_histogram_kernel(const int32_t* __restrict__ ids, int S, int k,
                                                                     int E, int per_group,
                                                                     int32_t* __restrict__ counts_all) {
    __shared__ int h[kMaxExperts];
    const int g = blockIdx.x / per_group, c = blockIdx.x - g * per_group;
    const int n = S * k;
    const int32_t* gi = ids + static_cast<size_t>(g) * n;
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    auto one = [&](int e) {
        if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) atomicAdd(&h[e], 1);
    };
    int from = 0;
    if ((reinterpret_cast<uintptr_t>(gi) & 15u) == 0) {
        const int n4 = n >> 2;
        const int4* g4 = reinterpret_cast<const int4*>(gi);
        for (int i = c * blockDim.x + threadIdx.x; i < n4; i += per_group * blockDim.x) {
            const int4 v = __ldg(g4 + i);
            one(v.x); one(v.y); one(v.z); one(v.w);
        }
        from = n4 << 2;
    }
    for (int i = from + c * blockDim.x + threadIdx.x; i < n; i += per_group * blockDim.x) one(__ldg(gi + i));
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        if (h[e] != 0) atomicAdd(counts_all + static_cast<size_t>(g) * E + e, h[e]);
}

// ------------------------------------------------------------------------------ combine

// out_i[t] = sum over j with dest_i[t*k+j] >= 0 of w_i[t, j] * Yp_owner[row], accumulated in
// fp32 in ascending j, for the n_src source ranks i; one warp per (source, token), each lane
// owning 16-byte vectors of the row with the k gathers of a vector in flight together.
template <int KMAX, int UNROLL, typename OutT>
__global__ void __launch_bounds__(256) ep_combine_kernel(const __grid_constant__ EpCombineArgs a) {
    const int lane = threadIdx.x & 31;
    const int warps_total = gridDim.x * (blockDim.x >> 5);
    const int vec_per_row = a.d / 4;
    const int cap = a.S * a.k;
    const int total_rows = a.R * cap;
    const int n_tok = a.n_src * a.S;
    for (int gt = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); gt < n_tok; gt += warps_total) {
        const int i = gt / a.S, t = gt - i * a.S;
        const float* mine = nullptr;
        float mine_w = 0.f;
        if (lane < a.k) {
            const int dr = __ldg(a.dest[i] + static_cast<size_t>(t) * a.k + lane);
            mine_w = __ldg(a.w[i] + static_cast<size_t>(t) * a.k + lane);
            if (dr >= 0 && dr < total_rows) {
                const int owner = dr / cap;
                mine = a.yp[owner] + static_cast<size_t>(dr - owner * cap) * a.d;
            }
        }
        const float* yr[KMAX];
        float wr[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            yr[j] = reinterpret_cast<const float*>(
                __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(mine), j));
            wr[j] = __shfl_sync(0xffffffffu, mine_w, j);
            if (j >= a.k) yr[j] = nullptr;
        }
        OutT* orow = static_cast<OutT*>(a.out[i]) + static_cast<size_t>(t) * a.d;
        for (int v0 = lane; v0 < vec_per_row; v0 += 32 * UNROLL) {
            float4 val[UNROLL][KMAX];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int v = v0 + 32 * u;
#pragma unroll
                for (int j = 0; j < KMAX; ++j)
                    if (yr[j] != nullptr && v < vec_per_row) val[u][j] = __ldg(reinterpret_cast<const float4*>(yr[j]) + v);
            }
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int v = v0 + 32 * u;
                if (v >= vec_per_row) break;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    if (yr[j] != nullptr) {
                        acc.x = fmaf(wr[j], val[u][j].x, acc.x);
                        acc.y = fmaf(wr[j], val[u][j].y, acc.y);
                        acc.z = fmaf(wr[j], val[u][j].z, acc.z);
                        acc.w = fmaf(wr[j], val[u][j].w, acc.w);
                    }
                }
                store_out4(orow, v, acc);
            }
        }
    }
}

template <typename OutT>
void launch_ep_combine_t(const EpCombineArgs& a, int grid, cudaStream_t stream) {
    if (a.k <= 2)
        ep_combine_kernel<2, 4, OutT><<<grid, 256, 0, stream>>>(a);
    else if (a.k <= 4)
        ep_combine_kernel<4, 2, OutT><<<grid, 256, 0, stream>>>(a);
    else
        ep_combine_kernel<kMaxTopK, 2, OutT><<<grid, 256, 0, stream>>>(a);
}

}  // namespace

cudaError_t launch_ep_plan(const int32_t* counts_all, int R, int S, int k, int E, int B, int rank, int32_t* counts,
                           int32_t* seg_expert, int32_t* seg_slot, int32_t* seg_offsets, int32_t* status,
                           cudaStream_t stream) {
    const int smem = static_cast<int>(sizeof(EpPlanSmem));
    const cudaError_t err = set_max_dynamic_smem(ep_plan_kernel, smem);
    if (err != cudaSuccess) return err;
    ep_plan_kernel<<<1, 256, smem, stream>>>(counts_all, R, S, k, E, B, rank, counts, seg_expert, seg_slot,
                                             seg_offsets, status);
    return cudaGetLastError();
}

cudaError_t launch_ep_prefetch(const EpPrefetchArgs& a, int num_sms, cudaStream_t stream) {
    if (a.B == 0) return cudaSuccess;
    bool v8 = true;
    for (int m = 0; m < 3; ++m)
        for (int r = 0; r < a.R; ++r) v8 = v8 && (reinterpret_cast<uintptr_t>(a.w[m][r]) & 31u) == 0;
    // four 256-thread CTAs per SM
    if (v8) ep_prefetch_kernel<true><<<4 * num_sms, 256, 0, stream>>>(a);
    else ep_prefetch_kernel<false><<<4 * num_sms, 256, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_ep_dispatch(const EpDispatchArgs& a0, int num_sms, cudaStream_t stream) {
    if (a0.S == 0 || a0.n_src == 0) return cudaSuccess;
    EpDispatchArgs a = a0;
    // one CTA per SM (1024 threads, ~113 KB of shared memory), all in one wave
    int per = num_sms / a.n_src;
    if (per > a.S) per = a.S;
    if (per < 1) per = 1;
    a.ctas_per_src = per;
    // 32-byte row copies when every source's X and every owner's Xp is 32-byte aligned
    uintptr_t al = 0;
    for (int i = 0; i < a.n_src; ++i) al |= reinterpret_cast<uintptr_t>(a.x[i]);
    for (int r = 0; r < a.R; ++r) al |= reinterpret_cast<uintptr_t>(a.xp[r]);
    auto kern = (al & 31u) == 0 ? ep_dispatch_kernel<true> : ep_dispatch_kernel<false>;
    const int smem = static_cast<int>(sizeof(EpSmem));
    cudaError_t err = set_max_dynamic_smem(kern, smem);
    if (err != cudaSuccess) return err;
    kern<<<per * a.n_src, kEpThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_group_histogram(const int32_t* ids, int R, int S, int k, int E, int32_t* counts_all,
                                   int num_sms, cudaStream_t stream) {
    if (R == 0) return cudaSuccess;
    cudaError_t err = cudaMemsetAsync(counts_all, 0, static_cast<size_t>(R) * E * sizeof(int32_t), stream);
    if (err != cudaSuccess) return err;
    int per_group = num_sms / R;
    const int per_needed = (S * k + 4 * kEpThreads - 1) / (4 * kEpThreads);  // ~4 ids per thread at least
    if (per_group > per_needed) per_group = per_needed;
    if (per_group < 1) per_group = 1;
    group_histogram_kernel<<<R * per_group, kEpThreads, 0, stream>>>(ids, S, k, E, per_group, counts_all);
    return cudaGetLastError();
}

cudaError_t launch_ep_combine(const EpCombineArgs& a, bool out_bf16, int num_sms, cudaStream_t stream) {
    const int n_tok = a.n_src * a.S;
    if (n_tok == 0) return cudaSuccess;
    int grid = (n_tok + 7) / 8;
    if (grid > 8 * num_sms) grid = 8 * num_sms;
    if (out_bf16)
        launch_ep_combine_t<__nv_bfloat16>(a, grid, stream);
    else
        launch_ep_combine_t<float>(a, grid, stream);
    return cudaGetLastError();
}

}  // namespace moe
