// Router for small expert counts (E <= 32): logits = X W_r^T (+ b), top-k and the softmax over the
// selected logits, on the CUDA cores.
//
// With few experts the projection is a thin GEMV-like pass over X (2*d*E flops per 2*d bytes of X),
// bound by reading X, and a 128-row tensor-core tile would leave most SMs idle (T/128 CTAs).  Here a
// warp takes two tokens at a time: each lane reads 16-byte vectors of both rows and the matching
// vectors of every expert's router row (W_r stays in L1/L2: E*d*2 bytes), accumulates in fp32, and
// the warp reduces the per-lane partial logits with shuffles.  The selection rule is the same as in
// the tensor-core router: descending logit, strict '>' while scanning experts in ascending id, so
// equal logits keep the lower id.
//
// Sources: "Sparsely-Gated MoE 구현 관점에서 살펴보기", sections "순전파 과정(forward pass)은 디스패치와
// 결합(combine)을 포함" (X @ W_r.T), "Top-2 라우팅의 수치 예시" and "pure Python으로 Top-k Router
// 확인하기" (softmax over the selected logits, shifted by their maximum).
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kTokensPerWarp = 2;

template <int EMAX>
__global__ void __launch_bounds__(256) route_simt_kernel(const __nv_bfloat16* __restrict__ x,
                                                         const __nv_bfloat16* __restrict__ w_router,
                                                         const float* __restrict__ bias, int T, int d, int E, int k,
                                                         float* __restrict__ logits, int32_t* __restrict__ ids,
                                                         float* __restrict__ w) {
    const int lane = threadIdx.x & 31;
    const int warps_total = gridDim.x * (blockDim.x >> 5);
    const int vec_per_row = d / 8;
    for (int t0 = (blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * kTokensPerWarp; t0 < T;
         t0 += warps_total * kTokensPerWarp) {
        float acc[kTokensPerWarp][EMAX];
#pragma unroll
        for (int u = 0; u < kTokensPerWarp; ++u)
#pragma unroll
            for (int e = 0; e < EMAX; ++e) acc[u][e] = 0.f;
        const int nt = min(kTokensPerWarp, T - t0);
        for (int v = lane; v < vec_per_row; v += 32) {
            float xf[kTokensPerWarp][8];
#pragma unroll
            for (int u = 0; u < kTokensPerWarp; ++u) {
                uint4 xv = make_uint4(0, 0, 0, 0);
                if (u < nt) xv = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(t0 + u) * d) + v);
                const uint32_t p[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    xf[u][2 * i] = bf16_lo(p[i]);
                    xf[u][2 * i + 1] = bf16_hi(p[i]);
                }
            }
#pragma unroll
            for (int e = 0; e < EMAX; ++e) {
                if (e < E) {
                    const uint4 wv = __ldg(reinterpret_cast<const uint4*>(w_router + static_cast<size_t>(e) * d) + v);
                    const uint32_t p[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float w0 = bf16_lo(p[i]), w1 = bf16_hi(p[i]);
#pragma unroll
                        for (int u = 0; u < kTokensPerWarp; ++u) {
                            acc[u][e] = fmaf(xf[u][2 * i], w0, acc[u][e]);
                            acc[u][e] = fmaf(xf[u][2 * i + 1], w1, acc[u][e]);
                        }
                    }
                }
            }
        }
        // warp reduction of every partial logit; every lane ends with the full sums
#pragma unroll
        for (int u = 0; u < kTokensPerWarp; ++u)
#pragma unroll
            for (int e = 0; e < EMAX; ++e)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc[u][e] += __shfl_xor_sync(0xffffffffu, acc[u][e], o);

        // lane u finishes token t0 + u
#pragma unroll
        for (int u = 0; u < kTokensPerWarp; ++u) {
            if (lane == u && u < nt) {
                const int t = t0 + u;
                float tv[kMaxTopK];
                int ti[kMaxTopK];
#pragma unroll
                for (int j = 0; j < kMaxTopK; ++j) { tv[j] = -INFINITY; ti[j] = 0x7fffffff; }
#pragma unroll
                for (int e = 0; e < EMAX; ++e) {
                    if (e < E) {
                        float lv = acc[u][e];
                        if (bias != nullptr) lv += __ldg(bias + e);
                        if (logits != nullptr) logits[static_cast<size_t>(t) * E + e] = lv;
                        float cv = lv;
                        int ci = e;
#pragma unroll
                        for (int j = 0; j < kMaxTopK; ++j) {
                            const bool gt = cv > tv[j];
                            const float ov = tv[j];
                            const int oi = ti[j];
                            tv[j] = gt ? cv : ov;
                            ti[j] = gt ? ci : oi;
                            cv = gt ? ov : cv;
                            ci = gt ? oi : ci;
                        }
                    }
                }
                float ex[kMaxTopK], sum = 0.f;
#pragma unroll
                for (int j = 0; j < kMaxTopK; ++j) {
                    ex[j] = (j < k) ? expf(tv[j] - tv[0]) : 0.f;
                    sum += ex[j];
                }
                const float inv = 1.0f / sum;
#pragma unroll
                for (int j = 0; j < kMaxTopK; ++j)
                    if (j < k) {
                        ids[static_cast<size_t>(t) * k + j] = ti[j];
                        w[static_cast<size_t>(t) * k + j] = ex[j] * inv;
                    }
            }
        }
    }
}

}  // namespace

cudaError_t launch_route_simt(const __nv_bfloat16* x, const __nv_bfloat16* w_router, const float* bias, int T, int d,
                              int E, int k, float* logits, int32_t* ids, float* w, int num_sms, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    const int warps = (T + kTokensPerWarp - 1) / kTokensPerWarp;
    int grid = (warps + 7) / 8;
    if (grid > 8 * num_sms) grid = 8 * num_sms;
    if (E <= 8)
        route_simt_kernel<8><<<grid, 256, 0, stream>>>(x, w_router, bias, T, d, E, k, logits, ids, w);
    else if (E <= 16)
        route_simt_kernel<16><<<grid, 256, 0, stream>>>(x, w_router, bias, T, d, E, k, logits, ids, w);
    else
        route_simt_kernel<kRouteSimtMaxExperts><<<grid, 256, 0, stream>>>(x, w_router, bias, T, d, E, k, logits, ids,
                                                                          w);
    return cudaGetLastError();
}

}  // namespace moe
