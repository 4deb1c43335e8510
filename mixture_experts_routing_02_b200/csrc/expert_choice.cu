// Expert-choice routing: experts choose tokens instead of tokens choosing experts
// ("Expert를 똑같이 나눴는데도 GPU가 대기하는 이유: MoE의 토큰 쏠림", section "라우팅 분포와
// 학습 안정성").  The router scores S[t, e] (softmax over the experts of token t) arrive
// expert-major from the route GEMM's epilogue; here
//   * ec_select_kernel: one CTA per expert finds the C'-th largest score of its column by a
//     three-pass radix select (11 + 11 + 10 bits of an order-preserving key) and then
//     compacts the kept tokens in ascending token order: the row of a kept token is the
//     number of kept tokens before it, from one block-wide scan per 1024 tokens.  Equal
//     scores at the threshold go to the lower token ids.  It also writes the segment table
//     (segment e = expert e, C' rows) and the [T, E] map from (token, expert) to row.
//   * ec_gather_kernel: Xp[r] = X[src[r]], one warp per row, 32-byte vectors (16-byte ones for
//     buffers that are only 16-byte aligned).
//   * ec_combine_kernel: out[t] = base[t] + sum of row_w[r] * Yp[r] over the rows r of
//     token t in ascending expert order, one warp per (token, column part); out in fp32 or bf16.
// The gather and the combine are HBM-bound; the selection reads the E x T scores four
// times, from L2.
#include "common.cuh"
#include "kernels.h"
#include "vec.cuh"

namespace moe {

namespace {

constexpr int kSelectWarps = kSelectThreads / 32;
constexpr int kSelectSmemKeys = 48 * 1024;  // 192 KB of keys: up to 49152 tokens per expert column
static_assert(kSelectWarps == 32, "the warp-total scan below uses one lane per warp");

// Order-preserving map of fp32 bits to uint32: larger float -> larger key.
__device__ __forceinline__ uint32_t order_key(uint32_t u) { return (u & 0x80000000u) ? ~u : (u | 0x80000000u); }

// Exclusive prefix sum of v over the CTA's threads in index order; *total = the CTA's sum.
// Ends with a barrier, so `warp_sums` ([kSelectWarps + 1]) may be reused right after.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_sums, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
    }
    if (lane == 31) warp_sums[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const uint32_t w = warp_sums[lane];
        uint32_t wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += t;
        }
        __syncwarp();
        warp_sums[lane] = wi - w;
        if (lane == 31) warp_sums[kSelectWarps] = wi;
    }
    __syncthreads();
    const uint32_t r = warp_sums[warp] + inc - v;
    *total = warp_sums[kSelectWarps];
    __syncthreads();
    return r;
}

// Inverse of order_key.
__device__ __forceinline__ uint32_t key_bits(uint32_t k) { return (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k; }

// SMEM: the expert's T keys are loaded once into dynamic shared memory (T <= kSelectSmemKeys)
// and every pass reads them there; otherwise every pass reads the scores from global memory.
template <bool SMEM>
__global__ void __launch_bounds__(kSelectThreads, 1)
    ec_select_kernel(const float* __restrict__ scores_t, int T, int E, int cp, int32_t* __restrict__ seg_expert,
                     int32_t* __restrict__ seg_offsets, int32_t* __restrict__ src, float* __restrict__ row_w,
                     int32_t* __restrict__ emap) {
    __shared__ uint32_t hist[2048];
    __shared__ uint32_t warp_sums[kSelectWarps + 1];
    __shared__ uint32_t sel[2];
    extern __shared__ uint32_t skeys[];
    const int e = blockIdx.x;
    const int tid = threadIdx.x;
    if (tid == 0) { sel[0] = 0; sel[1] = 1; }
    const uint32_t* col = reinterpret_cast<const uint32_t*>(scores_t) + static_cast<size_t>(e) * T;
    if (SMEM) {
        for (int t = tid; t < T; t += kSelectThreads) skeys[t] = order_key(__ldg(col + t));
        __syncthreads();
    }
    auto key_at = [&](int t) -> uint32_t { return SMEM ? skeys[t] : order_key(__ldg(col + t)); };
    if (tid == 0) {
        seg_expert[e] = e;
        seg_offsets[e] = e * cp;
        if (e == E - 1) seg_offsets[E] = E * cp;
    }

    // ---- radix select of the cp-th largest key, most significant digit first
    uint32_t prefix = 0, mask = 0, need = static_cast<uint32_t>(cp);  // need: rank (from the top) inside the class
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nb = pass == 2 ? 1024 : 2048;
        for (int i = tid; i < nb; i += kSelectThreads) hist[i] = 0;
        __syncthreads();
        for (int t = tid; t < T; t += kSelectThreads) {
            const uint32_t k = key_at(t);
            if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & static_cast<uint32_t>(nb - 1)], 1u);
        }
        __syncthreads();
        // thread i owns `per` bins counted down from the top digit; `above` = keys in higher bins
        const int per = nb / kSelectThreads;
        uint32_t mine = 0;
        for (int j = 0; j < per; ++j) mine += hist[nb - 1 - (tid * per + j)];
        uint32_t tot;
        const uint32_t above = block_exclusive_scan(mine, warp_sums, &tot);
        if (above < need && above + mine >= need) {
            uint32_t a = above;
            for (int j = 0; j < per; ++j) {
                const int b = nb - 1 - (tid * per + j);
                const uint32_t h = hist[b];
                if (a + h >= need) {
                    sel[0] = static_cast<uint32_t>(b);
                    sel[1] = need - a;
                    break;
                }
                a += h;
            }
        }
        __syncthreads();
        prefix |= sel[0] << shift;
        mask |= static_cast<uint32_t>(nb - 1) << shift;
        need = sel[1];
        __syncthreads();
    }
    // prefix = the threshold key; `need` keys equal to it are kept (the lowest token ids),
    // together with every key above it: cp - need of them

    // ---- compaction in ascending token order
    uint32_t run_gt = 0, run_eq = 0;
    const int base_row = e * cp;
#pragma unroll 1
    for (int t0 = 0; t0 < T; t0 += kSelectThreads) {
        const int t = t0 + tid;
        uint32_t raw = 0;
        bool gt = false, eq = false;
        if (t < T) {
            const uint32_t k = key_at(t);
            raw = key_bits(k);
            gt = k > prefix;
            eq = k == prefix;
        }
        uint32_t tot;
        const uint32_t ex = block_exclusive_scan((gt ? 1u : 0u) | (eq ? 0x10000u : 0u), warp_sums, &tot);
        const uint32_t gt_before = run_gt + (ex & 0xffffu), eq_before = run_eq + (ex >> 16);
        if (t < T) {
            int32_t row = -1;
            const uint32_t pos = gt_before + min(eq_before, need);
            if ((gt || (eq && eq_before < need)) && pos < static_cast<uint32_t>(cp)) {  // pos < cp always holds
                row = base_row + static_cast<int32_t>(pos);
                src[row] = t;
                row_w[row] = __uint_as_float(raw);
            }
            emap[static_cast<size_t>(t) * E + e] = row;
        }
        run_gt += tot & 0xffffu;
        run_eq += tot >> 16;
    }
}

constexpr int kGatherUnroll = 8;

// V8 (X and Xp 32-byte aligned): 32-byte vectors, kGatherUnroll / 2 in flight per lane; else
// 16-byte vectors, kGatherUnroll in flight.
template <bool V8>
__global__ void __launch_bounds__(256) ec_gather_kernel(const __nv_bfloat16* __restrict__ x,
                                                        const int32_t* __restrict__ src, int rows, int T, int d,
                                                        __nv_bfloat16* __restrict__ xp) {
    const int lane = threadIdx.x & 31;
    const int warps_total = gridDim.x * (blockDim.x >> 5);
    for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps_total) {
        const int t = __ldg(src + r);
        if (t < 0 || t >= T) continue;
        if constexpr (V8) {
            constexpr int U = kGatherUnroll / 2;
            const int vec_per_row = d / 16;
            const uint8_t* xs = reinterpret_cast<const uint8_t*>(x + static_cast<size_t>(t) * d);
            uint8_t* dst = reinterpret_cast<uint8_t*>(xp + static_cast<size_t>(r) * d);
            for (int v = lane; v < vec_per_row; v += 32 * U) {
                Vec32 val[U];
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (v + 32 * u < vec_per_row) val[u] = ld_nc_v8(xs + static_cast<size_t>(v + 32 * u) * 32);
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (v + 32 * u < vec_per_row) st_v8(dst + static_cast<size_t>(v + 32 * u) * 32, val[u]);
            }
        } else {
            const int vec_per_row = d / 8;
            const uint4* xs = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d);
            uint4* dst = reinterpret_cast<uint4*>(xp + static_cast<size_t>(r) * d);
            for (int v = lane; v < vec_per_row; v += 32 * kGatherUnroll) {
                uint4 val[kGatherUnroll];
#pragma unroll
                for (int u = 0; u < kGatherUnroll; ++u)
                    if (v + 32 * u < vec_per_row) val[u] = __ldg(xs + v + 32 * u);
#pragma unroll
                for (int u = 0; u < kGatherUnroll; ++u)
                    if (v + 32 * u < vec_per_row) dst[v + 32 * u] = val[u];
            }
        }
    }
}

constexpr int kCombineWarps = 8;
constexpr int kCombineUnroll = 2;   // row vectors per lane whose gathers are in flight together
constexpr int kCombineMaxParts = 4; // column parts per token (work items: token x part)

// VW floats per vector: 8 (32-byte loads and stores; Yp, base and an fp32 out 32-byte aligned) or 4.
template <int VW>
struct EcVec {
    float f[VW];
};

template <int VW>
__device__ __forceinline__ EcVec<VW> ec_ld(const float* p) {
    EcVec<VW> r;
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
__device__ __forceinline__ void ec_st(float* p, const EcVec<VW>& a) {
    if constexpr (VW == 8) {
        Vec32 v;
#pragma unroll
        for (int i = 0; i < 8; ++i) v.w[i] = __float_as_uint(a.f[i]);
        st_v8(p, v);
    } else {
        *reinterpret_cast<float4*>(p) = make_float4(a.f[0], a.f[1], a.f[2], a.f[3]);
    }
}

template <int VW>
__device__ __forceinline__ void ec_st(__nv_bfloat16* p, const EcVec<VW>& a) {
    if constexpr (VW == 8) {
        *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(a.f[0], a.f[1]), pack_bf16x2(a.f[2], a.f[3]),
                                                  pack_bf16x2(a.f[4], a.f[5]), pack_bf16x2(a.f[6], a.f[7]));
    } else {
        *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(a.f[0], a.f[1]), pack_bf16x2(a.f[2], a.f[3]));
    }
}

// One warp per work item (token t, column part p of `parts`): the token's (row, weight) pairs
// in ascending expert order go to shared memory, then the part's vectors are accumulated two
// rows at a time with all their gathers in flight.  Cutting each row into parts gives the warps
// several small items each, so the last wave is short.
template <int VW, typename OutT>
__global__ void __launch_bounds__(kCombineWarps * 32)
    ec_combine_kernel(const float* __restrict__ yp, const int32_t* __restrict__ emap, const float* __restrict__ row_w,
                      const float* __restrict__ base, int T, int E, int d, int rows, int parts,
                      OutT* __restrict__ out) {
    __shared__ int2 picks[kCombineWarps][kMaxExperts];  // (row, weight bits) of the current token
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int warps_total = gridDim.x * kCombineWarps;
    const int vec_per_row = d / VW;
    const int vec_per_part = (vec_per_row + parts - 1) / parts;
    int2* my = picks[warp];
    const int64_t items = static_cast<int64_t>(T) * parts;
    for (int64_t item = static_cast<int64_t>(blockIdx.x) * kCombineWarps + warp; item < items; item += warps_total) {
        const int t = static_cast<int>(item / parts), part = static_cast<int>(item % parts);
        int n = 0;
        for (int c = 0; c < E; c += 32) {
            const int e = c + lane;
            const int r = e < E ? __ldg(emap + static_cast<size_t>(t) * E + e) : -1;
            const bool ok = r >= 0 && r < rows;
            const unsigned ball = __ballot_sync(0xffffffffu, ok);
            if (ok) {
                const int pos = n + __popc(ball & ((1u << lane) - 1u));
                my[pos] = make_int2(r, __float_as_int(__ldg(row_w + r)));
            }
            n += __popc(ball);
        }
        __syncwarp();
        OutT* orow = out + static_cast<size_t>(t) * d;
        const float* brow = base ? base + static_cast<size_t>(t) * d : nullptr;
        const int vb = part * vec_per_part;
        const int ve = min(vec_per_row, vb + vec_per_part);
        for (int v0 = vb + lane; v0 < ve; v0 += 32 * kCombineUnroll) {
            EcVec<VW> acc[kCombineUnroll];
#pragma unroll
            for (int u = 0; u < kCombineUnroll; ++u) {
                const int v = v0 + 32 * u;
                if (brow && v < ve) {
                    acc[u] = ec_ld<VW>(brow + static_cast<size_t>(v) * VW);
                } else {
#pragma unroll
                    for (int i = 0; i < VW; ++i) acc[u].f[i] = 0.f;
                }
            }
            int p = 0;
            // two rows at a time: all 2 x kCombineUnroll gathers in flight before any is used
            for (; p + 1 < n; p += 2) {
                const int2 a = my[p], b = my[p + 1];
                EcVec<VW> ya[kCombineUnroll], yb[kCombineUnroll];
#pragma unroll
                for (int u = 0; u < kCombineUnroll; ++u) {
                    const int v = v0 + 32 * u;
                    if (v < ve) {
                        ya[u] = ec_ld<VW>(yp + static_cast<size_t>(a.x) * d + static_cast<size_t>(v) * VW);
                        yb[u] = ec_ld<VW>(yp + static_cast<size_t>(b.x) * d + static_cast<size_t>(v) * VW);
                    }
                }
#pragma unroll
                for (int u = 0; u < kCombineUnroll; ++u) {
                    if (v0 + 32 * u < ve) {
#pragma unroll
                        for (int i = 0; i < VW; ++i) acc[u].f[i] = fmaf(__int_as_float(a.y), ya[u].f[i], acc[u].f[i]);
#pragma unroll
                        for (int i = 0; i < VW; ++i) acc[u].f[i] = fmaf(__int_as_float(b.y), yb[u].f[i], acc[u].f[i]);
                    }
                }
            }
            if (p < n) {
                const int2 a = my[p];
#pragma unroll
                for (int u = 0; u < kCombineUnroll; ++u) {
                    const int v = v0 + 32 * u;
                    if (v < ve) {
                        const EcVec<VW> y = ec_ld<VW>(yp + static_cast<size_t>(a.x) * d + static_cast<size_t>(v) * VW);
#pragma unroll
                        for (int i = 0; i < VW; ++i) acc[u].f[i] = fmaf(__int_as_float(a.y), y.f[i], acc[u].f[i]);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < kCombineUnroll; ++u)
                if (v0 + 32 * u < ve) ec_st<VW>(orow + static_cast<size_t>(v0 + 32 * u) * VW, acc[u]);
        }
        __syncwarp();
    }
}

}  // namespace

cudaError_t launch_ec_select(const float* scores_t, int T, int E, int cp, int32_t* seg_expert, int32_t* seg_offsets,
                             int32_t* src, float* row_w, int32_t* emap, cudaStream_t stream) {
    if (T == 0 || E == 0) return cudaSuccess;
    if (T <= kSelectSmemKeys) {
        const size_t smem = static_cast<size_t>(T) * sizeof(uint32_t);
        if (smem > 48 * 1024) {
            const cudaError_t err = set_max_dynamic_smem(ec_select_kernel<true>, static_cast<int>(kSelectSmemKeys * sizeof(uint32_t)));
            if (err != cudaSuccess) return err;
        }
        ec_select_kernel<true><<<E, kSelectThreads, smem, stream>>>(scores_t, T, E, cp, seg_expert, seg_offsets, src,
                                                                    row_w, emap);
    } else {
        ec_select_kernel<false><<<E, kSelectThreads, 0, stream>>>(scores_t, T, E, cp, seg_expert, seg_offsets, src,
                                                                  row_w, emap);
    }
    return cudaGetLastError();
}

cudaError_t launch_ec_gather(const __nv_bfloat16* x, const int32_t* src, int rows, int T, int d, __nv_bfloat16* xp,
                             int num_sms, cudaStream_t stream) {
    if (rows == 0) return cudaSuccess;
    int grid = (rows + 7) / 8;
    if (grid > 8 * num_sms) grid = 8 * num_sms;
    if (((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(xp)) & 31u) == 0)
        ec_gather_kernel<true><<<grid, 256, 0, stream>>>(x, src, rows, T, d, xp);
    else
        ec_gather_kernel<false><<<grid, 256, 0, stream>>>(x, src, rows, T, d, xp);
    return cudaGetLastError();
}

cudaError_t launch_ec_combine(const float* yp, const int32_t* emap, const float* row_w, const float* base, int T,
                              int E, int d, int rows, void* out, bool out_bf16, int num_sms, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    // 32-byte vectors need Yp, base and an fp32 out 32-byte aligned (a bf16 out gets 16-byte stores)
    const uintptr_t al = reinterpret_cast<uintptr_t>(yp) | reinterpret_cast<uintptr_t>(base) |
                         (out_bf16 ? 0 : reinterpret_cast<uintptr_t>(out));
    const bool v8 = (al & 31u) == 0;
    // parts of at least one full pass of the warp (32 lanes x kCombineUnroll vectors)
    const int vw = v8 ? 8 : 4;
    int parts = d / (32 * kCombineUnroll * vw);
    if (parts > kCombineMaxParts) parts = kCombineMaxParts;
    if (parts < 1) parts = 1;
    const int64_t items = static_cast<int64_t>(T) * parts;
    int grid = static_cast<int>((items + kCombineWarps - 1) / kCombineWarps);
    if (grid > 8 * num_sms) grid = 8 * num_sms;
    const dim3 block(kCombineWarps * 32);
    if (out_bf16) {
        auto* o = static_cast<__nv_bfloat16*>(out);
        if (v8) ec_combine_kernel<8, __nv_bfloat16><<<grid, block, 0, stream>>>(yp, emap, row_w, base, T, E, d, rows, parts, o);
        else ec_combine_kernel<4, __nv_bfloat16><<<grid, block, 0, stream>>>(yp, emap, row_w, base, T, E, d, rows, parts, o);
    } else {
        auto* o = static_cast<float*>(out);
        if (v8) ec_combine_kernel<8, float><<<grid, block, 0, stream>>>(yp, emap, row_w, base, T, E, d, rows, parts, o);
        else ec_combine_kernel<4, float><<<grid, block, 0, stream>>>(yp, emap, row_w, base, T, E, d, rows, parts, o);
    }
    return cudaGetLastError();
}

}  // namespace moe
