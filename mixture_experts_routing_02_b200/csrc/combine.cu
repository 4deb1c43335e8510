// Combine: out[t] = base[t] + sum_j w[t, j] * Yp[dest[t*k + j]] over the kept pairs,
// accumulated in fp32 in ascending j; Yp and base (optional, e.g. the shared expert's
// output) are fp32; out is stored in fp32, or rounded once to bf16.
//
// Sources: "Sparsely-Gated MoE 구현 관점에서 살펴보기", section "순전파 과정 ..."
// (un-permute the expert outputs and combine them with the router weights);
// the MoonEP page, section "설치 및 통합" (combine returns the tokens in their
// original order).
//
// One warp per token: each lane owns 16-byte vectors (4 floats) of the row,
// issues the k gathers of a vector before using any of them, and writes the
// result with one 16-byte store.  The kernel is HBM-bound: it reads k rows and
// writes one row per token.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

// KMAX: the largest k this instance handles (registers scale with KMAX * UNROLL);
// UNROLL: row vectors per lane whose gathers are all in flight together; OutT: float or bf16.
template <int KMAX, int UNROLL, typename OutT>
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ yp, const int32_t* __restrict__ dest,
                                                      const float* __restrict__ w, const float* __restrict__ base,
                                                      int T, int k, int d, int rows, OutT* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int warps_total = gridDim.x * (blockDim.x >> 5);
    const int vec_per_row = d / 4;  // float4 vectors
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps_total) {
        int mine_d = -1;
        float mine_w = 0.f;
        if (lane < k) {
            mine_d = __ldg(dest + static_cast<size_t>(t) * k + lane);
            mine_w = __ldg(w + static_cast<size_t>(t) * k + lane);
        }
        int dr[KMAX];
        float wr[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            dr[j] = __shfl_sync(0xffffffffu, mine_d, j);
            wr[j] = __shfl_sync(0xffffffffu, mine_w, j);
            if (j >= k || dr[j] >= rows) dr[j] = -1;  // dropped, or outside Yp: contributes nothing
        }
        OutT* orow = out + static_cast<size_t>(t) * d;
        const float4* brow = base ? reinterpret_cast<const float4*>(base + static_cast<size_t>(t) * d) : nullptr;
        for (int v0 = lane; v0 < vec_per_row; v0 += 32 * UNROLL) {
            // all gathers of UNROLL vectors issued before any is used
            float4 val[UNROLL][KMAX];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int v = v0 + 32 * u;
#pragma unroll
                for (int j = 0; j < KMAX; ++j)
                    if (dr[j] >= 0 && v < vec_per_row)
                        val[u][j] = __ldg(reinterpret_cast<const float4*>(yp + static_cast<size_t>(dr[j]) * d) + v);
            }
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int v = v0 + 32 * u;
                if (v >= vec_per_row) break;
                float4 acc = brow ? __ldg(brow + v) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    if (dr[j] >= 0) {
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

}  // namespace

template <typename OutT>
static cudaError_t launch_combine_t(const float* yp, const int32_t* dest, const float* w, const float* base, int T, int k,
                             int d, int rows, OutT* out, int grid, cudaStream_t stream) {
    auto kern = k <= 2 ? combine_kernel<2, 4, OutT>
                       : (k <= 4 ? combine_kernel<4, 2, OutT> : combine_kernel<kMaxTopK, 2, OutT>);
    kern<<<grid, 256, 0, stream>>>(yp, dest, w, base, T, k, d, rows, out);
    return cudaGetLastError();
}

cudaError_t launch_combine(const float* yp, const int32_t* dest, const float* w, const float* base, int T, int k,
                           int d, int rows, void* out, bool out_bf16, int num_sms, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    int grid = (T + 7) / 8;
    if (grid > 8 * num_sms) grid = 8 * num_sms;
    const cudaError_t err =
        out_bf16 ? launch_combine_t(yp, dest, w, base, T, k, d, rows, static_cast<__nv_bfloat16*>(out), grid, stream)
                 : launch_combine_t(yp, dest, w, base, T, k, d, rows, static_cast<float*>(out), grid, stream);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

}  // namespace moe
