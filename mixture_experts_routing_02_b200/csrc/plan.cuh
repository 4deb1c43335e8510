// The greedy balanced plan (shared by the single-GPU dispatch and the expert-parallel kernels):
// every one of R groups receives exactly S*k rows; overloaded groups hand rows of their most
// loaded experts to replica slots of underloaded groups.
//
// Source: the MoonEP page ("가장 바쁜 랭크가 속도를 정합니다: MoonEP의 계획 코드를 직접
// 돌려봤습니다"), sections "개요", "이 기술은 무엇인가", "설치 및 통합" and "실제 실험 결과": exactly
// S x K rows per rank, replicas of overloaded experts in the spare slots [E, E+B), an error when
// the allocation exceeds the capacity.  The page does not give the algorithm; the greedy below is
// the reading this library uses (groups above S*k queue their excess, count descending / id
// ascending; groups below take their deficit from the front of the queue, one replica slot per
// (expert, group) piece; an expert's rows fill its home segment first, then its pieces).
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kMaxGroups = 256;

// Exclusive scan over the threads of a block (any multiple of 32 up to 1024); *total = the sum.
// warp_sums: 33 ints.  Ends with a barrier.
__device__ __forceinline__ int block_exclusive_scan_any(int v, int* warp_sums, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += t;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        const int w0 = lane < nwarps ? warp_sums[lane] : 0;
        int w = w0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += t;
        }
        __syncwarp();
        if (lane < nwarps) warp_sums[lane] = w - w0;
        if (lane == 31) warp_sums[32] = w;
    }
    __syncthreads();
    const int r = warp_sums[warp] + x - v;
    if (total != nullptr) *total = warp_sums[32];
    __syncthreads();
    return r;
}

// Shared memory of the balanced plan.
struct PlanSmem {
    int c[kMaxExperts];          // rows of each expert (filled by the caller)
    int order[kMaxExperts];      // experts of each group by (count desc, id asc)
    int given[kMaxExperts];      // rows an expert hands to other groups
    int next_rank[kMaxExperts];
    int qe[kMaxExperts], qn[kMaxExperts];  // the donor queue
    int load[kMaxGroups];
    int n_slots[kMaxGroups];
    int slot_e[kMaxSegments], slot_n[kMaxSegments], slot_r[kMaxSegments];
    int seg_len[kMaxSegments];
    int warp_sums[33];
    int infeasible;
};

// The greedy balanced plan from sm.c (written by the caller before a barrier) into the segment
// tables (any memory).  Called by the whole block; the greedy itself runs on one thread.  An
// infeasible plan (a group needs more than B replica slots) writes every segment empty and, if
// report_status, sets MOE_DEV_ERR_PLAN.
__device__ void compute_plan(PlanSmem& sm, int E, int R, int S, int k, int B, int* seg_expert, int* seg_offsets,
                             int* seg_first_rank, int32_t* status, bool report_status) {
    const int tid = threadIdx.x;
    const int epg = E / R;
    const int per_group = epg + B;
    const int n_seg = R * per_group;
    const int cap = S * k;

    for (int e = tid; e < E; e += blockDim.x) sm.given[e] = 0;
    for (int g = tid; g < R; g += blockDim.x) {
        int s = 0;
        for (int e = g * epg; e < (g + 1) * epg; ++e) s += sm.c[e];
        sm.load[g] = s;
    }
    for (int e = tid; e < E; e += blockDim.x) {
        const int g = e / epg;
        int rank = 0;
        for (int o = g * epg; o < (g + 1) * epg; ++o) rank += (sm.c[o] > sm.c[e]) || (sm.c[o] == sm.c[e] && o < e);
        sm.order[g * epg + rank] = e;
    }
    __syncthreads();

    if (tid == 0) {
        // the queue of excess rows, groups ascending, experts by (count desc, id asc)
        int nq = 0, total = 0;
        for (int g = 0; g < R; ++g) total += sm.load[g];
        int bad = (total != R * cap);
        for (int g = 0; g < R; ++g) {
            int excess = sm.load[g] - cap;
            for (int i = 0; i < epg && excess > 0; ++i) {
                const int e = sm.order[g * epg + i];
                const int take = sm.c[e] < excess ? sm.c[e] : excess;
                if (take > 0) { sm.given[e] = take; sm.qe[nq] = e; sm.qn[nq] = take; ++nq; excess -= take; }
            }
        }
        // groups below the cap, ascending, take from the front of the queue
        int head = 0;
        for (int g = 0; g < R; ++g) {
            int deficit = cap - sm.load[g];
            int ns = 0;
            while (deficit > 0 && head < nq) {
                const int take = sm.qn[head] < deficit ? sm.qn[head] : deficit;
                if (ns < B) { sm.slot_e[g * B + ns] = sm.qe[head]; sm.slot_n[g * B + ns] = take; }
                ++ns;
                sm.qn[head] -= take;
                deficit -= take;
                if (sm.qn[head] == 0) ++head;
            }
            if (ns > B || deficit > 0) bad = 1;
            sm.n_slots[g] = ns < B ? ns : B;
        }
        // within-expert rank at which each piece starts: after the home rows, in creation order
        for (int e = 0; e < E; ++e) sm.next_rank[e] = sm.c[e] - sm.given[e];
        for (int g = 0; g < R; ++g)
            for (int i = 0; i < sm.n_slots[g]; ++i) {
                const int idx = g * B + i;
                sm.slot_r[idx] = sm.next_rank[sm.slot_e[idx]];
                sm.next_rank[sm.slot_e[idx]] += sm.slot_n[idx];
            }
        sm.infeasible = bad;
        if (bad && report_status) report(status, MOE_DEV_ERR_PLAN);
    }
    __syncthreads();

    const bool bad = sm.infeasible != 0;
    for (int s = tid; s < n_seg; s += blockDim.x) {
        const int g = s / per_group, i = s - g * per_group;
        int ex = -1, len = 0, fr = 0;
        if (!bad) {
            if (i < epg) {
                ex = g * epg + i;
                len = sm.c[ex] - sm.given[ex];
            } else if (i - epg < sm.n_slots[g]) {
                const int idx = g * B + (i - epg);
                ex = sm.slot_e[idx];
                len = sm.slot_n[idx];
                fr = sm.slot_r[idx];
            }
        }
        seg_expert[s] = ex;
        seg_first_rank[s] = fr;
        sm.seg_len[s] = len;
    }
    __syncthreads();
    // offsets: exclusive scan of the lengths, each thread owning a contiguous chunk
    const int chunk = (n_seg + blockDim.x - 1) / blockDim.x;
    const int a = tid * chunk;
    int local = 0;
    for (int s = a; s < a + chunk && s < n_seg; ++s) local += sm.seg_len[s];
    int total;
    int run = block_exclusive_scan_any(local, sm.warp_sums, &total);
    for (int s = a; s < a + chunk && s < n_seg; ++s) {
        seg_offsets[s] = run;
        run += sm.seg_len[s];
    }
    if (tid == 0) seg_offsets[n_seg] = total;
    __syncthreads();
}

}  // namespace
}  // namespace moe
