// Routing of one token from its router logits, by one warp: the logits are the sum of n_split
// partial slices (in slice order, so the result does not depend on timing) plus the bias; then
// either the top-k ids in descending order (equal logits: the lower id) with their weights (softmax
// over the selected logits, or over all E with MOE_ROUTE_SOFTMAX_ALL), or, for expert-choice
// routing (scores_t non-null), the softmax over all E stored expert-major.  Used by
// route_logits_kernel, one warp per token.
//
// Sources: "Sparsely-Gated MoE 구현 관점에서 살펴보기", sections "Top-2 라우팅의 수치 예시" and
// "pure Python으로 Top-k Router 확인하기"; "Expert를 똑같이 나눴는데도 GPU가 대기하는 이유", section
// "라우팅 분포와 학습 안정성" (expert choice).
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

// U: experts per lane (E <= 32U); KMAX: the largest k.  Both bound the unrolled loops only: the
// arithmetic and its order do not depend on them.
template <int U, int KMAX>
__device__ __forceinline__ void route_token(const float* __restrict__ part, int n_split, int ldp, size_t split_stride,
                                            const float* __restrict__ bias, int T, int E, int k, int route_flags,
                                            float* __restrict__ logits, int32_t* __restrict__ ids,
                                            float* __restrict__ w, float* __restrict__ scores_t, int t, int lane) {
    float v[U];
    unsigned taken = 0;
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int e = lane + 32 * u;
        v[u] = -INFINITY;
        if (e < E) {
            const float* p = part + static_cast<size_t>(t) * ldp + e;
            float acc = __ldg(p);
            for (int sp = 1; sp < n_split; ++sp) acc += __ldg(p + sp * split_stride);
            if (bias != nullptr) acc += __ldg(bias + e);
            v[u] = acc;
            if (logits != nullptr) logits[static_cast<size_t>(t) * E + e] = acc;
        } else {
            taken |= 1u << u;
        }
    }
    if (scores_t != nullptr) {
        float m = -INFINITY;
#pragma unroll
        for (int u = 0; u < U; ++u) m = fmaxf(m, v[u]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float sum = 0.f;
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (lane + 32 * u < E) sum += expf(v[u] - m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float inv = 1.0f / sum;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = lane + 32 * u;
            if (e < E) scores_t[static_cast<size_t>(e) * T + t] = expf(v[u] - m) * inv;
        }
        return;
    }
    float sv[KMAX];
    int si[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        sv[j] = 0.f;
        si[j] = 0;
        if (j < k) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int u = 0; u < U; ++u) {
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
        for (int u = 0; u < U; ++u)
            if (lane + 32 * u < E) all += expf(v[u] - sv[0]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) all += __shfl_xor_sync(0xffffffffu, all, o);
    }
    if (lane == 0) {
        float ex[KMAX], sum = 0.f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            ex[j] = j < k ? expf(sv[j] - sv[0]) : 0.f;
            sum += ex[j];
        }
        const float inv = 1.0f / ((route_flags & MOE_ROUTE_SOFTMAX_ALL) ? all : sum);
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            if (j < k) {
                ids[static_cast<size_t>(t) * k + j] = si[j];
                w[static_cast<size_t>(t) * k + j] = ex[j] * inv;
            }
    }
}

}  // namespace
}  // namespace moe
