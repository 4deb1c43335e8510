// Grouped GEMM on the 5th-generation tensor cores (tcgen05 / TMEM / TMA).
//
// One persistent kernel template serves three contractions of the layer:
//   * the router projection logits = X W_r^T, with top-k and the softmax over
//     the selected logits fused into the epilogue ("Sparsely-Gated MoE 구현
//     관점에서 살펴보기", sections "순전파 과정 ..." and "Top-2 라우팅의 수치 예시"),
//     or, for expert-choice routing, with the softmax over all E logits stored
//     expert-major ("Expert를 똑같이 나눴는데도 GPU가 대기하는 이유", section
//     "라우팅 분포와 학습 안정성");
//   * the gate and up projections of every expert in one launch, with SwiGLU
//     fused into the epilogue ("5.3 Expert Parallelism", section "3. 고도화된
//     최적화: 오버래핑(Overlapping) 및 GroupGEMM"; MoonEP page "설치 및 통합":
//     the grouped GEMM selects each expert's rows through cu_seqlens);
//   * the down projection of every expert.
//
// Rows come in segments (rows [off[s], off[s+1]) use expert seg_expert[s]);
// the segment table is read on the device, so token counts never go back to
// the host.  The work unit is a 128-row x BN-column output tile; tiles are
// ordered segment-major, then by column tile, then by row tile, so the CTAs
// running at the same moment share the same expert weight tile through L2
// and each expert's weights cross HBM about once.
//
// CTA layout (192 threads, one CTA per SM):
//   warp 0      TMA producer: A tile [128 x 64] and B tile [N x 64] per stage
//   warp 1      allocates 512 TMEM columns; one lane issues tcgen05.mma
//               (M=128, N=mma_n, K=16, bf16 x bf16 -> fp32) and commits
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (one row per thread),
//               fused math, a shared-memory transpose, then row-contiguous 16-byte
//               stores of the valid rows
// Two accumulator buffers (columns [0,256) and [256,512)) let the epilogue of
// one tile overlap the main loop of the next.  In the down projection with
// d_ff <= 4096 a segment's last tile of at most 32 rows swaps the operand roles
// (see swapped_cols): the warps keep their jobs, the MMA warp issues two narrow
// MMAs per K step and the epilogue stores columns instead of rows.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kUmmaK = 16;
constexpr int kMaxStages = 8;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccStride = 256;
constexpr uint32_t kABytes = kBM * kBK * 2;
constexpr int kStageWords = 32 * 33;  // one epilogue warp's transpose buffer (32 rows x 33 words)

struct TileCoord {
    int seg, m, n, row0, row_end, expert;
};

__device__ __forceinline__ TileCoord decode_tile(int tile, const int* prefix, int n_seg, int n_tiles_n,
                                                 const GemmArgs& g, int bm = kBM) {
    const int key = tile / n_tiles_n;
    int lo = 0, hi = n_seg;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= key) lo = mid; else hi = mid;
    }
    TileCoord c;
    c.seg = lo;
    const int mt = prefix[lo + 1] - prefix[lo];
    const int local = tile - prefix[lo] * n_tiles_n;
    c.n = local / mt;
    c.m = local - c.n * mt;
    const int start = g.seg_offsets ? __ldg(g.seg_offsets + lo) : 0;
    c.row_end = g.seg_offsets ? __ldg(g.seg_offsets + lo + 1) : g.M;
    c.row0 = start + c.m * bm;
    c.expert = g.seg_expert ? __ldg(g.seg_expert + lo) : 0;
    return c;
}

// One warp: cumulative count of bm-row tiles over the segments (empty / unused segments have none).
__device__ __forceinline__ void build_tile_prefix(int* prefix, const GemmArgs& g, int bm, int lane) {
    int carry = 0;
    for (int b = 0; b < g.n_seg; b += 32) {
        const int s = b + lane;
        int mt = 0;
        if (s < g.n_seg) {
            const int a = g.seg_offsets ? __ldg(g.seg_offsets + s) : 0;
            const int e = g.seg_offsets ? __ldg(g.seg_offsets + s + 1) : g.M;
            const bool live = (g.seg_expert == nullptr) || __ldg(g.seg_expert + s) >= 0;
            mt = (live && e > a) ? (e - a + bm - 1) / bm : 0;
        }
        int v = mt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += t;
        }
        if (s < g.n_seg) prefix[s] = carry + v - mt;
        carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) prefix[g.n_seg] = carry;
}

// Epilogue of one warp's 32 accumulator rows (rows row_base.. of the output, columns n0..n0+BN)
// for the SwiGLU (bf16 Hp) and plain (fp32 Yp) contractions.  Each thread owns one row of the
// accumulator; the rows go through a per-warp shared-memory transpose so that the global stores
// are row-contiguous (whole 128-byte lines per group of lanes), with rows >= row_end masked.
template <int EPI>
__device__ __forceinline__ void epilogue_rows(const GemmArgs& g, uint32_t t_row, int row_base, int row_end, int n0,
                                              int lane, uint32_t* stg, size_t out_off = 0) {
    if (EPI == kEpiSwiglu) {
        for (int cc = 0; cc < g.BN; cc += 32) {
            uint32_t gr[32], ur[32];
            tmem_ld32(t_row + cc, gr);
            tmem_ld32(t_row + g.BN + cc, ur);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float g0 = __uint_as_float(gr[2 * i]), g1 = __uint_as_float(gr[2 * i + 1]);
                const float u0 = __uint_as_float(ur[2 * i]), u1 = __uint_as_float(ur[2 * i + 1]);
                const float h0 = g0 / (1.0f + __expf(-g0)) * u0;
                const float h1 = g1 / (1.0f + __expf(-g1)) * u1;
                stg[lane * 17 + i] = pack_bf16x2(h0, h1);
            }
            __syncwarp();
            if (n0 + cc < g.N) {
                // 32 rows x 64 bytes: 4 lanes per row, 8 rows per pass
                const int rr = lane >> 2, q = lane & 3;
#pragma unroll
                for (int pass = 0; pass < 4; ++pass) {
                    const int rl = pass * 8 + rr;
                    const int grow = row_base + rl;
                    if (grow < row_end) {
                        const uint32_t* src = stg + rl * 17 + q * 4;
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) +
                                                              static_cast<size_t>(grow) * g.ldo + n0 + cc + q * 8);
                        *dst = make_uint4(src[0], src[1], src[2], src[3]);
                    }
                }
            }
            __syncwarp();
        }
    } else {
        for (int cc = 0; cc < g.BN; cc += 32) {
            uint32_t r[32];
            tmem_ld32(t_row + cc, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) stg[lane * 33 + i] = r[i];
            __syncwarp();
            if (n0 + cc < g.N) {
                // 32 rows x 128 bytes: 8 lanes per row, 4 rows per pass
                const int rr = lane >> 3, q = lane & 7;
#pragma unroll
                for (int pass = 0; pass < 8; ++pass) {
                    const int rl = pass * 4 + rr;
                    const int grow = row_base + rl;
                    if (grow < row_end) {
                        const uint32_t* src = stg + rl * 33 + q * 4;
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(g.out) + out_off +
                                                              static_cast<size_t>(grow) * g.ldo + n0 + cc + q * 4);
                        *dst = make_uint4(src[0], src[1], src[2], src[3]);
                    }
                }
            }
            __syncwarp();
        }
    }
}

// A segment's last row tile holds r = row_end - row0 rows (1..128), and a 128-row MMA spends the
// same time on its 128 - r padding rows as on real ones.  In the down projection (256-row weight
// tiles, plain fp32 epilogue) a last tile with r <= g.swap_tail rows is computed with the operands
// swapped: the 256 weight rows of the B stage become two 128-row A operands, the tile's rows the
// N = ceil16(r) operand, and the accumulators hold [output column][row] at column offsets 0 and
// 128 of the buffer.  Measured on B200 (same box, each kernel alone): segments of 128 + 16 and
// 128 + 32 rows over 256 experts (d = 7168, d_ff = 2048) ran the down projection in 1.73 / 1.82 ms
// instead of 2.18 / 2.16 ms; tails of 64 or 96 rows gained nothing (2.11 vs 2.03 ms, 1.95 vs
// 1.92 ms), and the gate/up projection, whose swapped tiles issue four MMAs per 64-column stage
// with two weight matrices, got slower at every tail size (3.82-4.53 vs 3.41-3.43 ms).  With a long
// reduction the swapped tile gains nothing either: on Mixtral-like segments (d_ff = 14336) the down
// projection took 1.4-1.7 % longer with it, so the host turns it on only for d_ff <= 4096.  Returns
// N, or 0 for a tile computed the usual way.
__device__ __forceinline__ int swapped_cols(const TileCoord& c, const GemmArgs& g) {
    const int r = c.row_end - c.row0;
    return (g.swap_tail > 0 && r <= g.swap_tail) ? (r + 15) & ~15 : 0;
}

// Epilogue of a swapped down-projection tile: TMEM lane = output column (f for the accumulator at
// column offset 0, f + 128 for the one at 128), TMEM column = the tile's row.  Each store
// instruction writes one row's 32 consecutive fp32 columns (128 contiguous bytes per warp).
__device__ __forceinline__ void epilogue_swapped(const GemmArgs& g, uint32_t t_row, int row0, int r, int nt, int f) {
    float* out = static_cast<float*>(g.out);
    for (int h = 0; h < 2; ++h) {
        const int fh = f + 128 * h;
        for (int cc = 0; cc < nt; cc += 32) {
            uint32_t v[32];
            tmem_ld32(t_row + 128 * h + cc, v);
            tmem_ld_wait();
            if (fh < g.N) {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (cc + i < r) out[static_cast<size_t>(row0 + cc + i) * g.ldo + fh] = __uint_as_float(v[i]);
            }
        }
    }
}

// SPLITK: the reduction is cut into g.k_splits equal parts, each a work unit of its own, and
// part s of a tile is stored (plain fp32 epilogue) at out + s * split_stride; the caller sums
// the parts.  Used for the router projection, whose T/128 row tiles are too few for the SMs.
template <int EPI, bool SPLITK>
__global__ void __launch_bounds__(kThreads, 1)
    umma_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                     const __grid_constant__ CUtensorMap tmB1, const GemmArgs g) {
    __shared__ __align__(8) uint64_t full_bar[kMaxStages];
    __shared__ __align__(8) uint64_t empty_bar[kMaxStages];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    __shared__ int tile_prefix[kMaxSegments + 1];
    // swapped width of each tile, by the CTA's tile sequence number mod 16: written by the producer
    // before the tile's first stage is armed, read by the MMA issuer after that stage's full barrier
    // (the producer runs at most `stages` <= 8 stages, hence tiles, ahead)
    __shared__ int tile_swap[16];
    extern __shared__ uint8_t dsmem[];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int stages = g.stages;
    const uint32_t b_stage_bytes = static_cast<uint32_t>(g.mma_n) * 128u;

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + stages * kABytes;
    uint32_t* epi_stage = reinterpret_cast<uint32_t*>(sB + stages * b_stage_bytes);

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull_bar[b], 1);
            mbar_init(&tempty_bar[b], 4);
        }
        mbar_init(&drain_bar, 1);
        abort_sh = 0;
        mbar_fence_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB0);
        if (EPI == kEpiSwiglu) tma_prefetch_desc(&tmB1);
    }
    if (warp == 1) tmem_alloc(&tmem_base_sh, kTmemCols);
    if (warp == 2) build_tile_prefix(tile_prefix, g, kBM, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem_base = tmem_base_sh;
    static_assert(!SPLITK || EPI == kEpiStore, "split reductions use the plain fp32 epilogue");
    const int n_split = SPLITK ? g.k_splits : 1;
    const int total = tile_prefix[g.n_seg] * g.n_tiles_n * n_split;
    const int nkb = g.K / kBK;

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            const uint32_t tx = kABytes + (EPI == kEpiRoute ? static_cast<uint32_t>(g.N) * 128u : b_stage_bytes);
            // testing only (moe_testing_gemm_stalled): CTA 0's first stage is never filled, so the
            // MMA warp's bounded wait on it runs out and every role takes the abort path
            const bool skip_first = g.test_skip_first_load != 0 && blockIdx.x == 0;
            bool ok = true;
            int seq = 0;
            for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++seq) {
                const int split = SPLITK ? tile % n_split : 0;
                const TileCoord c = decode_tile(SPLITK ? tile / n_split : tile, tile_prefix, g.n_seg, g.n_tiles_n, g);
                const int n0 = c.n * g.BN;
                if (EPI == kEpiStore && !SPLITK) tile_swap[seq & 15] = swapped_cols(c, g);
                const int kb0 = SPLITK ? split * nkb / n_split : 0;
                const int kb1 = SPLITK ? (split + 1) * nkb / n_split : nkb;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_sh, g.status)) { ok = false; break; }
                    if (!(skip_first && issued == 0)) {
                        mbar_arrive_expect_tx(&full_bar[stage], tx);
                        uint8_t* a_dst = sA + stage * kABytes;
                        uint8_t* b_dst = sB + stage * b_stage_bytes;
                        tma_load_2d(a_dst, &tmA, kb * kBK, c.row0, &full_bar[stage]);
                        if (EPI == kEpiRoute) {
                            tma_load_2d(b_dst, &tmB0, kb * kBK, 0, &full_bar[stage]);
                        } else if (EPI == kEpiSwiglu) {
                            tma_load_3d(b_dst, &tmB0, kb * kBK, n0, c.expert, &full_bar[stage]);
                            tma_load_3d(b_dst + g.BN * 128, &tmB1, kb * kBK, n0, c.expert, &full_bar[stage]);
                        } else {
                            tma_load_3d(b_dst, &tmB0, kb * kBK, n0, c.expert, &full_bar[stage]);
                        }
                    }
                    ++issued;
                    if (++stage == stages) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                // give every copy still in flight a bounded chance to land before the CTA exits
                const int first = issued > stages ? issued - stages : 0;
                for (int i = first; i < issued; ++i) {
                    if (skip_first && i == 0) continue;  // never issued
                    mbar_wait(&full_bar[i % stages], static_cast<uint32_t>((i / stages) & 1), nullptr, nullptr);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            const uint32_t idesc = umma_idesc_bf16(kBM, g.mma_n);
            // stage s's descriptors are stage 0's plus s stages (the address field counts 16-byte units)
            const uint64_t adesc_0 = umma_desc_sw128(smem_u32(sA));
            const uint64_t bdesc_0 = umma_desc_sw128(smem_u32(sB));
            bool ok = true;
            int seq = 0;
            for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++seq) {
                if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, &abort_sh, g.status)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc) * kAccStride;
                const int split = SPLITK ? tile % n_split : 0;
                const int kb0 = SPLITK ? split * nkb / n_split : 0;
                const int kb1 = SPLITK ? (split + 1) * nkb / n_split : nkb;
                int nt = 0;
                if (EPI == kEpiStore && !SPLITK) {
                    // the tile's swapped width, published by the producer before it armed the tile's
                    // first stage (the usual loop below waits on that stage again at no cost)
                    if (!mbar_wait(&full_bar[stage], phase, &abort_sh, g.status)) { ok = false; break; }
                    nt = tile_swap[seq & 15];
                } else if (EPI == kEpiSwiglu) {
                    // the same wait for the first stage ahead of the loop: same-box timings of the gate/up
                    // projection on Mixtral-like shapes were 1.3-1.7 % shorter with it (no change on
                    // DeepSeek-like ones); the loop itself is unchanged
                    if (!mbar_wait(&full_bar[stage], phase, &abort_sh, g.status)) { ok = false; break; }
                }
                if (nt > 0) {
                    // swapped: weight rows [0,128) and [128,256) of the B stage against the tile's rows
                    const uint32_t idesc_sw = umma_idesc_bf16(kBM, nt);
                    for (int kb = kb0; kb < kb1; ++kb) {
                        if (!mbar_wait(&full_bar[stage], phase, &abort_sh, g.status)) { ok = false; break; }
                        tc_fence_after();
                        const uint64_t adesc = adesc_0 + static_cast<uint64_t>(stage) * (kABytes >> 4);
                        const uint64_t wdesc0 = bdesc_0 + static_cast<uint64_t>(stage) * (b_stage_bytes >> 4);
                        const uint64_t wdesc1 = wdesc0 + ((128u * 128u) >> 4);  // weight rows [128, 256)
#pragma unroll
                        for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
                            const uint32_t accum = (kb != kb0 || kk != 0) ? 1u : 0u;
                            umma_bf16(d_tmem, wdesc0 + 2 * kk, adesc + 2 * kk, idesc_sw, accum);
                            umma_bf16(d_tmem + 128, wdesc1 + 2 * kk, adesc + 2 * kk, idesc_sw, accum);
                        }
                        umma_commit(&empty_bar[stage]);
                        if (++stage == stages) { stage = 0; phase ^= 1u; }
                    }
                } else {
                    for (int kb = kb0; kb < kb1; ++kb) {
                        if (!mbar_wait(&full_bar[stage], phase, &abort_sh, g.status)) { ok = false; break; }
                        tc_fence_after();
                        const uint64_t adesc = adesc_0 + static_cast<uint64_t>(stage) * (kABytes >> 4);
                        const uint64_t bdesc = bdesc_0 + static_cast<uint64_t>(stage) * (b_stage_bytes >> 4);
#pragma unroll
                        for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
                            // +32 bytes per K=16 step inside the 128-byte swizzle atom (encoded >> 4)
                            umma_bf16(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
                        }
                        umma_commit(&empty_bar[stage]);
                        if (++stage == stages) { stage = 0; phase ^= 1u; }
                    }
                }
                if (!ok) break;
                umma_commit(&tfull_bar[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            // every MMA issued by this thread completes before tensor memory is released
            umma_commit(&drain_bar);
            mbar_wait(&drain_bar, 0, nullptr, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ epilogue
        const int quarter = warp & 3;  // a warp may only touch TMEM lanes [32*(warp%4), +32)
        const int r_in_tile = quarter * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const TileCoord c = decode_tile(SPLITK ? tile / n_split : tile, tile_prefix, g.n_seg, g.n_tiles_n, g);
            const size_t out_off = SPLITK ? static_cast<size_t>(tile % n_split) * g.split_stride : 0;
            const bool got = mbar_wait(&tfull_bar[acc], acc_phase, &abort_sh, g.status);
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(acc) * kAccStride;
            const int row = c.row0 + r_in_tile;
            const bool valid = row < c.row_end;
            const int n0 = c.n * g.BN;

            if (EPI == kEpiSwiglu || EPI == kEpiStore) {
                const int nt = (EPI == kEpiStore && !SPLITK) ? swapped_cols(c, g) : 0;
                if (nt > 0)
                    epilogue_swapped(g, t_row, c.row0, c.row_end - c.row0, nt, n0 + r_in_tile);
                else
                    epilogue_rows<EPI>(g, t_row, c.row0 + quarter * 32, c.row_end, n0, lane,
                                       epi_stage + (warp - 2) * kStageWords, out_off);
            } else if (g.scores_t != nullptr) {
                // expert choice: softmax over the E logits of this row, stored expert-major so
                // that the 32 lanes (consecutive rows) of a warp write 128 contiguous bytes
                float run_max = -INFINITY, run_sum = 0.f;
                for (int cc = 0; cc < g.N; cc += 32) {
                    uint32_t r[32];
                    tmem_ld32(t_row + cc, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int e = cc + i;
                        if (e < g.N) {
                            float v = __uint_as_float(r[i]);
                            if (g.bias != nullptr) v += __ldg(g.bias + e);
                            if (valid && g.logits != nullptr) g.logits[static_cast<size_t>(row) * g.N + e] = v;
                            if (v > run_max) {
                                run_sum = run_sum * expf(run_max - v) + 1.0f;
                                run_max = v;
                            } else {
                                run_sum += expf(v - run_max);
                            }
                        }
                    }
                }
                const float inv = 1.0f / run_sum;
                for (int cc = 0; cc < g.N; cc += 32) {
                    uint32_t r[32];
                    tmem_ld32(t_row + cc, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int e = cc + i;
                        if (e < g.N && valid) {
                            float v = __uint_as_float(r[i]);
                            if (g.bias != nullptr) v += __ldg(g.bias + e);
                            g.scores_t[static_cast<size_t>(e) * g.M + row] = expf(v - run_max) * inv;
                        }
                    }
                }
            } else {
                // router: top-k over the E logits of this row, softmax over the selected ones
                float tv[kMaxTopK];
                int ti[kMaxTopK];
#pragma unroll
                for (int j = 0; j < kMaxTopK; ++j) { tv[j] = -INFINITY; ti[j] = 0x7fffffff; }
                const bool softmax_all = (g.route_flags & MOE_ROUTE_SOFTMAX_ALL) != 0;
                float run_max = -INFINITY, run_sum = 0.f;  // online softmax denominator over all logits
                for (int cc = 0; cc < g.N; cc += 32) {
                    uint32_t r[32];
                    tmem_ld32(t_row + cc, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int e = cc + i;
                        if (e < g.N) {
                            float v = __uint_as_float(r[i]);
                            if (g.bias != nullptr) v += __ldg(g.bias + e);
                            if (valid && g.logits != nullptr) g.logits[static_cast<size_t>(row) * g.N + e] = v;
                            if (softmax_all) {
                                if (v > run_max) {
                                    run_sum = run_sum * expf(run_max - v) + 1.0f;
                                    run_max = v;
                                } else {
                                    run_sum += expf(v - run_max);
                                }
                            }
                            // insertion into the sorted list; strict '>' keeps the lower id on ties
                            float cv = v;
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
                }
                if (valid) {
                    float ex[kMaxTopK];
                    float sum = 0.f;
#pragma unroll
                    for (int j = 0; j < kMaxTopK; ++j) {
                        ex[j] = (j < g.k) ? expf(tv[j] - tv[0]) : 0.f;
                        sum += ex[j];
                    }
                    // run_max == tv[0]: the largest logit is the first selected one
                    const float inv = 1.0f / (softmax_all ? run_sum : sum);
#pragma unroll
                    for (int j = 0; j < kMaxTopK; ++j) {
                        if (j < g.k) {
                            g.topk_ids[static_cast<size_t>(row) * g.k + j] = ti[j];
                            g.topk_w[static_cast<size_t>(row) * g.k + j] = ex[j] * inv;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty_bar[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}


}  // namespace

size_t gemm_smem_bytes(int stages, int mma_n) {
    return 1024 + static_cast<size_t>(stages) * (kABytes + static_cast<size_t>(mma_n) * 128u) +
           4 * kStageWords * sizeof(uint32_t);
}

int gemm_pick_stages(int mma_n) {
    const size_t per = kABytes + static_cast<size_t>(mma_n) * 128u;
    int s = static_cast<int>((kGemmSmemBudget - 1024) / per);
    if (s > kMaxStages) s = kMaxStages;
    return s;
}

template <int EPI, bool SPLITK>
static cudaError_t launch_one(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const GemmArgs& g,
                              int grid, cudaStream_t stream) {
    auto kern = umma_gemm_kernel<EPI, SPLITK>;
    size_t smem = gemm_smem_bytes(g.stages, g.mma_n);
    if (smem < kGemmSmemMin) smem = kGemmSmemMin;  // keeps one CTA per SM (all TMEM columns are taken)
    cudaError_t err = set_max_dynamic_smem(kern, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    kern<<<grid, kThreads, smem, stream>>>(a, b0, b1, g);
    return cudaGetLastError();
}

cudaError_t launch_umma_gemm(int epi, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                             const GemmArgs& g, int grid, cudaStream_t stream) {
    switch (epi) {
        case kEpiRoute: return launch_one<kEpiRoute, false>(a, b0, b1, g, grid, stream);
        case kEpiSwiglu: return launch_one<kEpiSwiglu, false>(a, b0, b1, g, grid, stream);
        default:
            return g.k_splits > 1 ? launch_one<kEpiStore, true>(a, b0, b1, g, grid, stream)
                                  : launch_one<kEpiStore, false>(a, b0, b1, g, grid, stream);
    }
}

}  // namespace moe
