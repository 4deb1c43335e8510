// Combine: out[t] = base[t] + sum_j w[t, j] * Yp[dest[t*k + j]] over the kept pairs,
// accumulated in fp32 in ascending j; Yp and base (optional, e.g. the shared expert's
// output) are fp32; out is stored in fp32, or rounded once to bf16.
//
// Sources: "Sparsely-Gated MoE 구현 관점에서 살펴보기", section "순전파 과정 ..."
// (un-permute the expert outputs and combine them with the router weights);
// the MoonEP page, section "설치 및 통합" (combine returns the tokens in their
// original order).
//
// One warp per token: each lane owns 32-byte vectors (8 floats) of the row (16-byte
// vectors where the buffers are only 16-byte aligned), issues the k gathers of a vector
// before using any of them, and writes the result with one store.  The kernel is HBM-bound: it reads k rows and
// writes one row per token.
#include "common.cuh"
#include "kernels.h"
#include "vec.cuh"

namespace moe {

namespace {

// VW floats of a row moved by one instruction: 4 (16-byte vectors) or 8 (32-byte vectors, when
// Yp, base and an fp32 out are 32-byte aligned: half the memory instructions).
template <int VW>
struct FVec {
    float f[VW];
};

template <int VW>
__device__ __forceinline__ FVec<VW> ld_fvec(const float* p) {
    FVec<VW> r;
    if constexpr (VW == 8) {
        const Vec32 v = ld_nc_v8(p);
#pragma unroll
        for (int i = 0; i < 8; ++i) r.f[i] = __uint_as_float(v.w[i]);
    } else {
        const float4 v = __ldg(reinterpret_cast<const float4*>(p));
        r.f[0] = v.x; r.f[1] = v.y; r.f[2] = v.z; r.f[3] = v.w;
    }
    return r;
}

template <int VW>
__device__ __forceinline__ void st_fvec(float* p, const FVec<VW>& a) {
    if constexpr (VW == 8) {
        Vec32 v;
#pragma unroll
        for (int i = 0; i < 8; ++i) v.w[i] = __float_as_uint(a.f[i]);
        st_v8(p, v);
    } else {
        *reinterpret_cast<float4*>(p) = make_float4(a.f[0], a.f[1], a.f[2], a.f[3]);
    }
}

// rounded once to bf16 (round to nearest even): 16- or 8-byte stores
template <int VW>
__device__ __forceinline__ void st_fvec(__nv_bfloat16* p, const FVec<VW>& a) {
    if constexpr (VW == 8) {
        *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(a.f[0], a.f[1]), pack_bf16x2(a.f[2], a.f[3]),
                                                  pack_bf16x2(a.f[4], a.f[5]), pack_bf16x2(a.f[6], a.f[7]));
    } else {
        *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(a.f[0], a.f[1]), pack_bf16x2(a.f[2], a.f[3]));
    }
}

// KMAX: the largest k this instance handles (registers scale with KMAX * UNROLL * VW);
// UNROLL: row vectors per lane whose gathers are all in flight together; OutT: float or bf16.
template <int KMAX, int UNROLL, int VW, typename OutT>
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ yp, const int32_t* __restrict__ dest,
                                                      const float* __restrict__ w, const float* __restrict__ base,
                                                      int T, int k, int d, int rows, OutT* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int warps_total = gridDim.x * (blockDim.x >> 5);
    const int vec_per_row = d / VW;
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
        const float* brow = base ? base + static_cast<size_t>(t) * d : nullptr;
        for (int v0 = lane; v0 < vec_per_row; v0 += 32 * UNROLL) {
            // all gathers of UNROLL vectors issued before any is used
            FVec<VW> val[UNROLL][KMAX];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int v = v0 + 32 * u;
#pragma unroll
                for (int j = 0; j < KMAX; ++j)
                    if (dr[j] >= 0 && v < vec_per_row)
                        val[u][j] = ld_fvec<VW>(yp + static_cast<size_t>(dr[j]) * d + static_cast<size_t>(v) * VW);
            }
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int v = v0 + 32 * u;
                if (v >= vec_per_row) break;
                FVec<VW> acc;
                if (brow) {
                    acc = ld_fvec<VW>(brow + static_cast<size_t>(v) * VW);
                } else {
#pragma unroll
                    for (int i = 0; i < VW; ++i) acc.f[i] = 0.f;
                }
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    if (dr[j] >= 0) {
#pragma unroll
                        for (int i = 0; i < VW; ++i) acc.f[i] = fmaf(wr[j], val[u][j].f[i], acc.f[i]);
                    }
                }
                st_fvec<VW>(orow + static_cast<size_t>(v) * VW, acc);
            }
        }
    }
}

}  // namespace

template <typename OutT>
static cudaError_t launch_combine_t(const float* yp, const int32_t* dest, const float* w, const float* base, int T, int k,
                             int d, int rows, OutT* out, int grid, cudaStream_t stream) {
    // 32-byte vectors need Yp, base and an fp32 out 32-byte aligned (a bf16 out gets 16-byte stores)
    const uintptr_t al = reinterpret_cast<uintptr_t>(yp) | reinterpret_cast<uintptr_t>(base) |
                         (sizeof(OutT) == 4 ? reinterpret_cast<uintptr_t>(out) : 0);
    auto kern = (al & 31u) == 0
                    ? (k <= 2 ? combine_kernel<2, 2, 8, OutT>
                              : (k <= 4 ? combine_kernel<4, 1, 8, OutT> : combine_kernel<kMaxTopK, 1, 8, OutT>))
                    : (k <= 2 ? combine_kernel<2, 4, 4, OutT>
                              : (k <= 4 ? combine_kernel<4, 2, 4, OutT> : combine_kernel<kMaxTopK, 2, 4, OutT>));
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
