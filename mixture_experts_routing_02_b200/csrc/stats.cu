// Routing statistics of one dispatch, for monitoring the routing distribution
// ("Expert를 똑같이 나눴는데도 GPU가 대기하는 이유", section "라우팅 분포와 학습 안정성":
// watch per-expert token counts and dropped tokens) and the balanced plan's
// figures (MoonEP page, "실제 실험 결과": the busiest group's load against the
// mean, the share of migrated tokens, the replica slots in use).
//
// One CTA reads the raw counts [E] and the segment tables [n_seg] / [n_seg+1]
// (a few KB) and writes MOE_STAT_COUNT int32 values; the layout of the values
// is given in include/moe_routing.h.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

__global__ void __launch_bounds__(256) routing_stats_kernel(const int32_t* __restrict__ counts,
                                                            const int32_t* __restrict__ seg_expert,
                                                            const int32_t* __restrict__ seg_offsets, int E,
                                                            int n_seg, int R, int B, int pairs,
                                                            int32_t* __restrict__ stats) {
    __shared__ int s_max_load, s_active, s_max_seg, s_max_group_load, s_max_group_rows, s_migrated, s_replicas;
    const int tid = threadIdx.x;
    if (tid == 0) {
        s_max_load = 0; s_active = 0; s_max_seg = 0; s_max_group_load = 0; s_max_group_rows = 0;
        s_migrated = 0; s_replicas = 0;
    }
    __syncthreads();
    if (counts != nullptr) {
        for (int e = tid; e < E; e += blockDim.x) {
            const int c = counts[e];
            atomicMax(&s_max_load, c);
            if (c > 0) atomicAdd(&s_active, 1);
        }
    }
    // with a plan, group g owns segments [g * per, (g + 1) * per): its E/R home experts, then its
    // B replica slots; a slot in use names an expert and holds rows
    const int home = R > 0 ? E / R : 1;
    const int per = R > 0 ? home + B : 1;
    for (int s = tid; s < n_seg; s += blockDim.x) {
        const int len = seg_offsets[s + 1] - seg_offsets[s];
        atomicMax(&s_max_seg, len);
        if (R > 0 && s % per >= home && seg_expert[s] >= 0 && len > 0) {
            atomicAdd(&s_migrated, len);
            atomicAdd(&s_replicas, 1);
        }
    }
    for (int g = tid; g < R; g += blockDim.x) {
        if (counts != nullptr) {
            int load = 0;
            for (int e = g * home; e < (g + 1) * home; ++e) load += counts[e];
            atomicMax(&s_max_group_load, load);
        }
        atomicMax(&s_max_group_rows, seg_offsets[(g + 1) * per] - seg_offsets[g * per]);
    }
    __syncthreads();
    if (tid == 0) {
        const int rows = seg_offsets[n_seg];
        const bool have = counts != nullptr;
        stats[MOE_STAT_PAIRS] = pairs;
        stats[MOE_STAT_ROWS] = rows;
        stats[MOE_STAT_DROPPED] = pairs - rows;
        stats[MOE_STAT_MAX_EXPERT_LOAD] = have ? s_max_load : -1;
        stats[MOE_STAT_ACTIVE_EXPERTS] = have ? s_active : -1;
        stats[MOE_STAT_MAX_SEGMENT_ROWS] = s_max_seg;
        // without a plan every expert is its own group
        stats[MOE_STAT_MAX_GROUP_LOAD] = have ? (R > 0 ? s_max_group_load : s_max_load) : -1;
        stats[MOE_STAT_MAX_GROUP_ROWS] = R > 0 ? s_max_group_rows : s_max_seg;
        stats[MOE_STAT_MIGRATED_ROWS] = s_migrated;
        stats[MOE_STAT_REPLICAS_USED] = s_replicas;
    }
}

}  // namespace

cudaError_t launch_routing_stats(const int32_t* counts, const int32_t* seg_expert, const int32_t* seg_offsets,
                                 int E, int n_seg, int R, int B, int pairs, int32_t* stats, cudaStream_t st) {
    routing_stats_kernel<<<1, 256, 0, st>>>(counts, seg_expert, seg_offsets, E, n_seg, R, B, pairs, stats);
    return cudaGetLastError();
}

}  // namespace moe
