// C ABI of the library: argument validation, TMA descriptor encoding and the
// launch sequence of every call.  Nothing here allocates device memory,
// synchronises the host, or keeps per-call state; the only process-wide state
// is the driver entry point of cuTensorMapEncodeTiled and a per-device cache
// of the SM count.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

using namespace moe;

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool have_encoder() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode != nullptr;
}

int sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (dev >= 0 && dev < 64) cache[dev] = n;
    return n;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Dims {
    int T, d, E, k, F, C, R, B, S, flags;
    bool out_bf16;  // the layer output [T, d] is stored in bf16 (else fp32)
    bool ec() const { return (flags & MOE_ROUTE_EXPERT_CHOICE) != 0; }
    bool rr() const { return (flags & MOE_ROUTE_REROUTE) != 0; }
    int cp() const { return ec() ? std::min(C, T) : 0; }  // expert choice: rows per expert
    int n_seg;
    int rows;  // rows_alloc
};

moe_status_t check_shape(const moe_shape_t* s, Dims* out) {
    if (s == nullptr) return MOE_ERR_INVALID_ARG;
    Dims v;
    v.T = s->T; v.d = s->d_model; v.E = s->n_experts; v.k = s->top_k; v.F = s->d_ff;
    v.C = s->capacity; v.R = s->n_groups; v.B = s->replica_slots; v.flags = s->route_flags;
    if (s->out_dtype != MOE_DTYPE_F32 && s->out_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    v.out_bf16 = s->out_dtype == MOE_DTYPE_BF16;
    if (v.flags & ~(MOE_ROUTE_SOFTMAX_ALL | MOE_ROUTE_EXPERT_CHOICE | MOE_ROUTE_REROUTE)) return MOE_ERR_INVALID_ARG;
    const bool ec = (v.flags & MOE_ROUTE_EXPERT_CHOICE) != 0;
    if (ec && ((v.flags & MOE_ROUTE_SOFTMAX_ALL) || s->capacity < 1 || s->n_groups != 0)) return MOE_ERR_INVALID_ARG;
    const bool rr = (v.flags & MOE_ROUTE_REROUTE) != 0;
    if (rr && (ec || s->capacity < 1 || s->n_groups != 0)) return MOE_ERR_INVALID_ARG;
    if (v.T < 0 || v.d < 1 || v.E < 1 || v.k < 1 || v.k > v.E || v.F < 1 || v.C < 0 || v.R < 0 || v.B < 0)
        return MOE_ERR_INVALID_ARG;
    if (v.R > 0 && (v.E % v.R != 0 || v.T % v.R != 0 || v.C > 0)) return MOE_ERR_INVALID_ARG;
    if (v.E > kMaxExperts || v.k > kMaxTopK || v.d % 64 != 0 || v.F % 64 != 0) return MOE_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(v.T) * v.k >= (int64_t(1) << 30)) return MOE_ERR_UNSUPPORTED;
    const int64_t n_seg = v.R > 0 ? static_cast<int64_t>(v.R) * (v.E / v.R + v.B) : v.E;
    if (n_seg > kMaxSegments) return MOE_ERR_UNSUPPORTED;
    v.n_seg = static_cast<int>(n_seg);
    v.S = v.R > 0 ? v.T / v.R : v.T;
    int64_t rows = static_cast<int64_t>(v.T) * v.k;
    if (v.C > 0) rows = std::min<int64_t>(rows, static_cast<int64_t>(v.C) * v.E);
    if (rr && static_cast<int64_t>(v.T) * v.k > kRerouteMaxPairs) return MOE_ERR_UNSUPPORTED;
    if (ec) {
        // segment e holds expert e's C' = min(C, T) chosen tokens
        rows = static_cast<int64_t>(std::min(v.C, v.T)) * v.E;
        if (rows >= (int64_t(1) << 30)) return MOE_ERR_UNSUPPORTED;
    }
    v.rows = static_cast<int>(rows);
    if (out) *out = v;
    return MOE_OK;
}

bool encode(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box) {
    const cuuint32_t es[3] = {1, 1, 1};
    return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, K] row-major bf16, tiles of 128 rows x 64 columns
bool tmap_rows(CUtensorMap* m, const void* p, int rows, int K) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t box[2] = {64, 128};
    return encode(m, p, 2, dims, strides, box);
}

// [E, N, K] row-major bf16 (one [N, K] weight per expert), tiles of box_n rows x 64 columns of one expert
bool tmap_experts(CUtensorMap* m, const void* p, int E, int N, int K, int box_n) {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(E)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * 2, static_cast<cuuint64_t>(K) * N * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_n), 1};
    return encode(m, p, 3, dims, strides, box);
}

inline moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// ------------------------------------------------------------------------------ implementations

moe_status_t route_impl(const Dims& v, const moe_bf16_t* x, const moe_bf16_t* w_router, const float* bias,
                        float* logits, int32_t* ids, float* w, int32_t* status, cudaStream_t st) {
    if (!x || !w_router || !ids || !w) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_router)) return MOE_ERR_INVALID_ARG;
    if (v.T == 0) return MOE_OK;
    if (!have_encoder()) return MOE_ERR_CUDA;
    const int epad = std::max(16, (v.E + 15) / 16 * 16);
    CUtensorMap ta, tb;
    if (!tmap_rows(&ta, x, v.T, v.d)) return MOE_ERR_CUDA;
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(v.d), static_cast<cuuint64_t>(v.E)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(v.d) * 2};
        const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(v.E)};
        if (!encode(&tb, w_router, 2, dims, strides, box)) return MOE_ERR_CUDA;
    }
    GemmArgs g{};
    g.seg_offsets = nullptr; g.seg_expert = nullptr; g.n_seg = 1; g.M = v.T; g.K = v.d; g.N = v.E;
    g.BN = epad; g.n_tiles_n = 1; g.mma_n = epad; g.stages = gemm_pick_stages(epad);
    g.bias = bias; g.logits = logits; g.topk_ids = ids; g.topk_w = w; g.k = v.k; g.status = status;
    g.route_flags = v.flags;
    const int grid = std::min(sm_count(), (v.T + 127) / 128);
    return cuda_status(launch_umma_gemm(kEpiRoute, ta, tb, tb, g, grid, st));
}

// The router projection has only ceil(T/128) row tiles.  When they are fewer than the SMs, its
// reduction over d is cut into S parts (each at least 4 k-blocks of 64), the S*ceil(T/128) work
// units write fp32 partial logits [S][T][ldp] to a workspace, and a warp-per-token kernel sums
// the parts in order (so the result does not depend on timing), adds the bias and routes.  (Routing
// the rows inside the GEMM's clusters instead, after a cluster barrier, measured slower: it routes
// with one warp per 8 tokens instead of one warp per token over the whole GPU.)
constexpr int kMaxRouteSplits = 8;

int route_splits(const Dims& v) {
    const int m_tiles = (v.T + 127) / 128;
    int s = sm_count() / std::max(1, m_tiles);
    s = std::min(s, kMaxRouteSplits);
    s = std::min(s, (v.d / 64) / 4);
    return std::max(s, 1);
}

int route_ldp(const Dims& v) {
    const int epad = std::max(16, (v.E + 15) / 16 * 16);
    return (epad + 31) / 32 * 32;
}

size_t route_ws_bytes(const Dims& v) {
    const int S = route_splits(v);
    if (S < 2) return 0;
    return align256(static_cast<size_t>(S) * v.T * route_ldp(v) * sizeof(float));
}

// Split router projection + routing; false when it does not apply (one part, or no workspace).
bool route_split_impl(const Dims& v, const moe_bf16_t* x, const moe_bf16_t* w_router, const float* bias,
                      float* logits, int32_t* ids, float* w, float* scores, int32_t* status, void* ws,
                      size_t ws_bytes, cudaStream_t st, moe_status_t* result) {
    const size_t need = route_ws_bytes(v);
    if (need == 0 || ws == nullptr || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return false;
    if (!have_encoder()) { *result = MOE_ERR_CUDA; return true; }
    const int S = route_splits(v);
    const int epad = std::max(16, (v.E + 15) / 16 * 16);
    const int ldp = route_ldp(v);
    CUtensorMap ta, tb;
    if (!tmap_rows(&ta, x, v.T, v.d) || !tmap_experts(&tb, w_router, 1, v.E, v.d, epad)) {
        *result = MOE_ERR_CUDA;
        return true;
    }
    GemmArgs g{};
    g.seg_offsets = nullptr; g.seg_expert = nullptr; g.n_seg = 1; g.M = v.T; g.K = v.d; g.N = v.E;
    g.BN = epad; g.n_tiles_n = 1; g.mma_n = epad; g.stages = gemm_pick_stages(epad);
    g.out = ws; g.ldo = ldp; g.status = status;
    g.k_splits = S; g.split_stride = static_cast<size_t>(v.T) * ldp;
    const int grid = std::min(sm_count(), (v.T + 127) / 128 * S);
    moe_status_t r = cuda_status(launch_umma_gemm(kEpiStore, ta, tb, tb, g, grid, st));
    if (r == MOE_OK)
        r = cuda_status(launch_route_logits(static_cast<const float*>(ws), S, ldp, g.split_stride, bias, v.T, v.E, v.k,
                                            v.flags & ~MOE_ROUTE_EXPERT_CHOICE, logits, ids, w, scores, sm_count(), st));
    *result = r;
    return true;
}

// Expert-choice scores: the router projection with the softmax over all E logits in the
// epilogue, written expert-major ([E, T]).
moe_status_t route_scores_impl(const Dims& v, const moe_bf16_t* x, const moe_bf16_t* w_router, const float* bias,
                               float* scores, int32_t* status, cudaStream_t st) {
    if (!x || !w_router || !scores) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_router)) return MOE_ERR_INVALID_ARG;
    if (v.T == 0) return MOE_OK;
    if (!have_encoder()) return MOE_ERR_CUDA;
    const int epad = std::max(16, (v.E + 15) / 16 * 16);
    CUtensorMap ta, tb;
    if (!tmap_rows(&ta, x, v.T, v.d)) return MOE_ERR_CUDA;
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(v.d), static_cast<cuuint64_t>(v.E)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(v.d) * 2};
        const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(v.E)};
        if (!encode(&tb, w_router, 2, dims, strides, box)) return MOE_ERR_CUDA;
    }
    GemmArgs g{};
    g.seg_offsets = nullptr; g.seg_expert = nullptr; g.n_seg = 1; g.M = v.T; g.K = v.d; g.N = v.E;
    g.BN = epad; g.n_tiles_n = 1; g.mma_n = epad; g.stages = gemm_pick_stages(epad);
    g.bias = bias; g.scores_t = scores; g.k = v.k; g.status = status;
    const int grid = std::min(sm_count(), (v.T + 127) / 128);
    return cuda_status(launch_umma_gemm(kEpiRoute, ta, tb, tb, g, grid, st));
}

moe_status_t choose_impl(const Dims& v, const float* scores, const moe_bf16_t* x, int32_t* seg_expert,
                         int32_t* seg_offsets, int32_t* src, float* row_w, int32_t* emap, moe_bf16_t* xp,
                         cudaStream_t st) {
    if (!scores || !x || !seg_expert || !seg_offsets || !src || !row_w || !emap || !xp) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(xp)) return MOE_ERR_INVALID_ARG;
    if (v.T == 0) return MOE_OK;
    moe_status_t s = cuda_status(launch_ec_select(scores, v.T, v.E, v.cp(), seg_expert, seg_offsets, src, row_w,
                                                  emap, st));
    if (s != MOE_OK) return s;
    return cuda_status(launch_ec_gather(reinterpret_cast<const __nv_bfloat16*>(x), src, v.rows, v.T, v.d,
                                        reinterpret_cast<__nv_bfloat16*>(xp), sm_count(), st));
}

moe_status_t gate_up_impl(const Dims& v, const moe_bf16_t* xp, const int32_t* seg_expert, const int32_t* seg_offsets,
                          const moe_bf16_t* wg, const moe_bf16_t* wu, moe_bf16_t* hp, int32_t* status,
                          cudaStream_t st, bool test_stall = false) {
    if (!xp || !seg_expert || !seg_offsets || !wg || !wu || !hp) return MOE_ERR_INVALID_ARG;
    if (!aligned16(xp) || !aligned16(wg) || !aligned16(wu) || !aligned16(hp)) return MOE_ERR_INVALID_ARG;
    if (v.T == 0 || v.rows == 0) return MOE_OK;
    if (!have_encoder()) return MOE_ERR_CUDA;
    const int bn = v.F >= 128 ? 128 : v.F;
    CUtensorMap ta, tg, tu;
    if (!tmap_rows(&ta, xp, v.rows, v.d) || !tmap_experts(&tg, wg, v.E, v.F, v.d, bn) ||
        !tmap_experts(&tu, wu, v.E, v.F, v.d, bn))
        return MOE_ERR_CUDA;
    GemmArgs g{};
    g.seg_offsets = seg_offsets; g.seg_expert = seg_expert; g.n_seg = v.n_seg; g.M = v.rows; g.K = v.d; g.N = v.F;
    g.BN = bn; g.n_tiles_n = (v.F + bn - 1) / bn; g.mma_n = 2 * bn;
    g.out = hp; g.ldo = v.F; g.k = v.k; g.status = status;
    g.test_skip_first_load = test_stall ? 1 : 0;
    g.stages = gemm_pick_stages(2 * bn);
    const int64_t max_tiles = (static_cast<int64_t>(v.rows) / 128 + v.n_seg) * g.n_tiles_n;
    const int grid = static_cast<int>(std::min<int64_t>(sm_count(), max_tiles));
    return cuda_status(launch_umma_gemm(kEpiSwiglu, ta, tg, tu, g, grid, st));
}

moe_status_t down_impl(const Dims& v, const moe_bf16_t* hp, const int32_t* seg_expert, const int32_t* seg_offsets,
                       const moe_bf16_t* wd, float* yp, int32_t* status, cudaStream_t st) {
    if (!hp || !seg_expert || !seg_offsets || !wd || !yp) return MOE_ERR_INVALID_ARG;
    if (!aligned16(hp) || !aligned16(wd) || !aligned16(yp)) return MOE_ERR_INVALID_ARG;
    if (v.T == 0 || v.rows == 0) return MOE_OK;
    if (!have_encoder()) return MOE_ERR_CUDA;
    const int bn = v.d >= 256 ? 256 : v.d;
    CUtensorMap ta, tb;
    if (!tmap_rows(&ta, hp, v.rows, v.F) || !tmap_experts(&tb, wd, v.E, v.d, v.F, bn)) return MOE_ERR_CUDA;
    GemmArgs g{};
    g.seg_offsets = seg_offsets; g.seg_expert = seg_expert; g.n_seg = v.n_seg; g.M = v.rows; g.K = v.F; g.N = v.d;
    g.BN = bn; g.n_tiles_n = (v.d + bn - 1) / bn; g.mma_n = bn;
    g.out = yp; g.ldo = v.d; g.k = v.k; g.status = status;
    g.swap_tail = (bn == 256 && v.F <= kSwapTailMaxK) ? kSwapTailRows : 0;
    g.stages = gemm_pick_stages(bn);
    const int64_t max_tiles = (static_cast<int64_t>(v.rows) / 128 + v.n_seg) * g.n_tiles_n;
    const int grid = static_cast<int>(std::min<int64_t>(sm_count(), max_tiles));
    return cuda_status(launch_umma_gemm(kEpiStore, ta, tb, tb, g, grid, st));
}

moe_status_t segments_or_plan(const Dims& v, int32_t* counts, const int32_t* partials, int n_partials,
                              int32_t* seg_expert, int32_t* seg_offsets, int32_t* seg_first_rank, int32_t* status,
                              cudaStream_t st) {
    if (v.R > 0)
        return cuda_status(launch_plan(counts, partials, n_partials, v.E, v.R, v.S, v.k, v.B, seg_expert, seg_offsets,
                                       seg_first_rank, status, st));
    return cuda_status(
        launch_segments(counts, partials, n_partials, v.E, v.C, seg_expert, seg_offsets, seg_first_rank, st));
}

moe_status_t reroute_impl(const Dims& v, const moe_bf16_t* x, const int32_t* ids, const float* logits,
                          int32_t* counts, int32_t* seg_expert, int32_t* seg_offsets, int32_t* seg_first_rank,
                          int32_t* dest, int32_t* src, moe_bf16_t* xp, int32_t* status, void* ws, size_t ws_bytes,
                          cudaStream_t st, bool test_stall = false) {
    if (!x || !ids || !logits || !counts || !seg_expert || !seg_offsets || !seg_first_rank || !dest || !src || !xp)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(xp)) return MOE_ERR_INVALID_ARG;
    if (ws == nullptr || ws_bytes < reroute_ws_bytes(v.T, v.k) || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return MOE_ERR_WORKSPACE;
    RerouteArgs a{};
    a.ids = ids; a.logits = logits;
    a.T = v.T; a.k = v.k; a.E = v.E; a.capacity = v.C; a.rows = v.rows;
    a.counts = counts; a.seg_expert = seg_expert; a.seg_offsets = seg_offsets; a.seg_first_rank = seg_first_rank;
    a.dest = dest; a.src = src; a.status = status;
    a.test_skip_arrival = test_stall ? 1 : 0;
    return cuda_status(launch_reroute(a, ws, reinterpret_cast<const __nv_bfloat16*>(x),
                                      reinterpret_cast<__nv_bfloat16*>(xp), v.d, sm_count(), st));
}

moe_status_t dispatch_impl(const Dims& v, const moe_bf16_t* x, const int32_t* ids, int32_t plan_ready,
                           int32_t* counts, int32_t* seg_expert, int32_t* seg_offsets, int32_t* seg_first_rank,
                           int32_t* dest, int32_t* src, moe_bf16_t* xp, int32_t* status, void* ws,
                           size_t ws_bytes, cudaStream_t st, int first_tile = 0) {
    if (!x || !ids || !counts || !seg_expert || !seg_offsets || !seg_first_rank || !dest || !src || !xp)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(xp)) return MOE_ERR_INVALID_ARG;
    const size_t need = permute_ws_bytes(v.T, v.k, v.E);
    if (ws == nullptr || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_WORKSPACE;
    const size_t scratch = permute_scratch_bytes(v.T, v.k, v.E);
    PermuteArgs a{};
    a.ids = ids; a.x = reinterpret_cast<const __nv_bfloat16*>(x); a.xp = reinterpret_cast<__nv_bfloat16*>(xp);
    a.seg_expert = seg_expert; a.seg_offsets = seg_offsets; a.seg_first_rank = seg_first_rank;
    a.dest = dest; a.src = src;
    a.ticket = static_cast<uint32_t*>(ws);
    a.sync = static_cast<uint32_t*>(ws) + 1;
    a.tile_state = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + 256);
    a.status = status;
    a.T = v.T; a.k = v.k; a.E = v.E; a.d = v.d; a.n_seg = v.n_seg;
    a.tokens_per_tile = permute_tokens_per_tile(v.T, v.k);
    a.rows = v.rows;
    a.first_tile = first_tile;
    a.n_tiles = permute_n_tiles(v.T, v.k);
    const int64_t pairs = static_cast<int64_t>(v.T) * v.k;
    if (!plan_ready && a.n_tiles > 0 && v.R > 0 && v.R <= kEpMaxRanks && first_tile == 0 &&
        static_cast<int64_t>(v.S) * v.k <= kCountMaxPairsPlan) {
        // The balanced plan's R token groups run as R sources of the expert-parallel dispatch, all
        // buffers local: each CTA counts only its own group's ids (the per-group counts come from
        // one small launch), and the layout is the same.  Counts per group go to the partials area.
        int32_t* counts_all = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + scratch);
        moe_status_t s = cuda_status(launch_group_histogram(ids, v.R, v.S, v.k, v.E, counts_all, sm_count(), st));
        if (s != MOE_OK) return s;
        EpDispatchArgs e{};
        const int cap = v.S * v.k;
        for (int g = 0; g < v.R; ++g) {
            e.x[g] = a.x + static_cast<size_t>(g) * v.S * v.d;
            e.ids[g] = ids + static_cast<size_t>(g) * cap;
            e.dest[g] = dest + static_cast<size_t>(g) * cap;
            e.xp[g] = a.xp + static_cast<size_t>(g) * cap * v.d;
            e.src[g] = src + static_cast<size_t>(g) * cap;
        }
        e.counts_all = counts_all; e.status = status;
        e.R = v.R; e.S = v.S; e.k = v.k; e.E = v.E; e.d = v.d; e.B = v.B; e.n_seg = v.n_seg;
        e.src0 = 0; e.n_src = v.R;
        e.counts_out = counts; e.seg_expert_out = seg_expert; e.seg_offsets_out = seg_offsets;
        e.seg_first_rank_out = seg_first_rank;
        return cuda_status(launch_ep_dispatch(e, sm_count(), st));
    }
    if (!plan_ready && a.n_tiles > 0 &&
        (v.R == 0 || (pairs <= kCountMaxPairsPlan && first_tile == 0))) {
        // counts, tables, ranks and row copies in one launch
        a.capacity = v.C;
        a.counts = counts; a.seg_expert_out = seg_expert; a.seg_offsets_out = seg_offsets;
        a.seg_first_rank_out = seg_first_rank;
        a.prefetch_x = static_cast<size_t>(v.T) * v.d * 2 <= (size_t(48) << 20);
        a.R = v.R; a.S = v.S; a.B = v.B;
        if (v.R > 0 || (pairs <= kCountMaxPairs && first_tile == 0))
            return cuda_status(launch_dispatch_count(a, sm_count(), st));
        return cuda_status(launch_dispatch_fused(a, sm_count(), st));
    }
    if (!plan_ready) {
        // histogram partials + clearing of the look-back scratch in one launch, then the tables
        int32_t* partials = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + scratch);
        moe_status_t s = cuda_status(launch_histogram_partials(ids, v.T * v.k, v.E, partials,
                                                               static_cast<uint32_t*>(ws), scratch, st));
        if (s != MOE_OK) return s;
        s = segments_or_plan(v, counts, partials, histogram_partial_ctas(v.T * v.k), seg_expert, seg_offsets,
                             seg_first_rank, status, st);
        if (s != MOE_OK) return s;
    }
    return cuda_status(launch_permute(a, !plan_ready, sm_count(), st));
}

// Scratch of moe_dispatch_static: one array in the library's device image.  Host code
// may not use the symbol itself as a device address; its address is looked up once
// per device with cudaGetSymbolAddress (with that device current) and cached.
constexpr size_t kStaticScratchBytes = size_t(4) << 20;  // 4 MiB
static __device__ __align__(256) unsigned char g_dispatch_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (nullptr on failure).
void* static_scratch_address() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess || p == nullptr) return nullptr;
        g_scratch_addr[dev] = p;
    }
    return g_scratch_addr[dev];
}

struct LayerLayout {
    size_t ids, w, counts, seg_expert, seg_offsets, seg_first_rank, dest, src, dispatch_ws, xp, hp, yp, scores, emap,
        row_w, route_ws, logits, total;
    size_t dispatch_ws_bytes;
};

LayerLayout layer_layout(const Dims& v) {
    LayerLayout L{};
    size_t o = 0;
    // expert choice keeps no per-pair arrays and no dispatch workspace
    const size_t tk = v.ec() ? 0 : static_cast<size_t>(v.T) * v.k;
    const size_t te = v.ec() ? static_cast<size_t>(v.T) * v.E : 0;
    L.ids = o; o = align256(o + tk * 4);
    L.w = o; o = align256(o + tk * 4);
    L.counts = o; o = align256(o + static_cast<size_t>(v.E) * 4);
    L.seg_expert = o; o = align256(o + static_cast<size_t>(v.n_seg) * 4);
    L.seg_offsets = o; o = align256(o + static_cast<size_t>(v.n_seg + 1) * 4);
    L.seg_first_rank = o; o = align256(o + static_cast<size_t>(v.n_seg) * 4);
    L.dest = o; o = align256(o + tk * 4);
    L.src = o; o = align256(o + static_cast<size_t>(v.rows) * 4);
    L.dispatch_ws_bytes = v.ec() ? 0 : (v.rr() ? reroute_ws_bytes(v.T, v.k) : permute_ws_bytes(v.T, v.k, v.E));
    L.dispatch_ws = o; o = align256(o + L.dispatch_ws_bytes);
    L.xp = o; o = align256(o + static_cast<size_t>(v.rows) * v.d * 2);
    L.hp = o; o = align256(o + static_cast<size_t>(v.rows) * v.F * 2);
    L.yp = o; o = align256(o + static_cast<size_t>(v.rows) * v.d * 4);
    L.scores = o; o = align256(o + te * 4);
    L.emap = o; o = align256(o + te * 4);
    L.row_w = o; o = align256(o + (v.ec() ? static_cast<size_t>(v.rows) * 4 : 0));
    L.route_ws = o; o = align256(o + route_ws_bytes(v));
    L.logits = o; o = align256(o + (v.rr() ? static_cast<size_t>(v.T) * v.E * 4 : 0));
    L.total = o;
    return L;
}

// Expert-parallel shapes: the balanced plan's R groups are R ranks of S = T / R tokens each.
moe_status_t check_ep_shape(const moe_shape_t* shape, Dims* v) {
    const moe_status_t s = check_shape(shape, v);
    if (s != MOE_OK) return s;
    if (v->R < 1 || v->ec() || v->rr()) return MOE_ERR_INVALID_ARG;
    if (v->R > kEpMaxRanks) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

// The shape of one rank's grouped GEMMs: S*k rows in E/R + B segments over E/R + B weight slots.
Dims ep_local_dims(const Dims& v) {
    Dims l = v;
    l.E = v.E / v.R + v.B;
    l.n_seg = l.E;
    l.T = v.S;
    l.rows = v.S * v.k;
    l.R = 0;
    return l;
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status_t s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: size outside the supported range";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing, misaligned or too small";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA: CUDA runtime or launch failure";
    }
    return "unknown moe_status_t";
}

moe_status_t moe_layout(const moe_shape_t* shape, int32_t* n_segments, int32_t* rows_alloc) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (n_segments) *n_segments = v.n_seg;
    if (rows_alloc) *rows_alloc = v.rows;
    return MOE_OK;
}

moe_status_t moe_workspace_size(const moe_shape_t* shape, size_t* dispatch_bytes, size_t* layer_bytes) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (dispatch_bytes)
        *dispatch_bytes = v.ec() ? 0 : (v.rr() ? reroute_ws_bytes(v.T, v.k) : permute_ws_bytes(v.T, v.k, v.E));
    if (layer_bytes) *layer_bytes = layer_layout(v).total;
    return MOE_OK;
}

moe_status_t moe_route(const moe_shape_t* shape, const moe_bf16_t* x, const moe_bf16_t* w_router, const float* bias,
                       float* logits, int32_t* topk_ids, float* topk_w, int32_t* status, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (v.ec()) return MOE_ERR_INVALID_ARG;  // expert choice has its own calls
    return route_impl(v, x, w_router, bias, logits, topk_ids, topk_w, status, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_route_workspace_size(const moe_shape_t* shape, size_t* bytes) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (bytes) *bytes = route_ws_bytes(v);
    return MOE_OK;
}

moe_status_t moe_route_ws(const moe_shape_t* shape, const moe_bf16_t* x, const moe_bf16_t* w_router,
                          const float* bias, float* logits, int32_t* topk_ids, float* topk_w, int32_t* status,
                          void* ws, size_t ws_bytes, moe_stream_t stream) {
    Dims v;
    moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (v.ec()) return MOE_ERR_INVALID_ARG;  // expert choice has its own calls
    if (!x || !w_router || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_router)) return MOE_ERR_INVALID_ARG;
    if (v.T == 0) return MOE_OK;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (route_split_impl(v, x, w_router, bias, logits, topk_ids, topk_w, nullptr, status, ws, ws_bytes, st, &s)) return s;
    return route_impl(v, x, w_router, bias, logits, topk_ids, topk_w, status, st);
}

moe_status_t moe_route_scores_ws(const moe_shape_t* shape, const moe_bf16_t* x, const moe_bf16_t* w_router,
                                 const float* bias, float* scores, int32_t* status, void* ws, size_t ws_bytes,
                                 moe_stream_t stream) {
    Dims v;
    moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (!v.ec()) return MOE_ERR_INVALID_ARG;
    if (!x || !w_router || !scores) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_router)) return MOE_ERR_INVALID_ARG;
    if (v.T == 0) return MOE_OK;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (route_split_impl(v, x, w_router, bias, nullptr, nullptr, nullptr, scores, status, ws, ws_bytes, st, &s)) return s;
    return route_scores_impl(v, x, w_router, bias, scores, status, st);
}

moe_status_t moe_route_from_logits(const moe_shape_t* shape, const float* logits, int32_t* topk_ids, float* topk_w,
                                   moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (v.ec()) return MOE_ERR_INVALID_ARG;  // expert choice has its own calls
    if (!logits || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_route_from_logits(logits, v.T, v.E, v.k, v.flags, topk_ids, topk_w, sm_count(),
                                                static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_histogram(const moe_shape_t* shape, const int32_t* topk_ids, int32_t* counts, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (v.ec()) return MOE_ERR_INVALID_ARG;  // expert choice has its own calls
    if (!topk_ids || !counts) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_histogram(topk_ids, v.T * v.k, v.E, counts, sm_count(), static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_segments(const moe_shape_t* shape, const int32_t* counts, int32_t* seg_expert, int32_t* seg_offsets,
                          int32_t* seg_first_rank, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (v.ec()) return MOE_ERR_INVALID_ARG;  // expert choice has its own calls
    if (v.rr()) return MOE_ERR_INVALID_ARG;  // re-routing has its own dispatch call
    if (v.R > 0 || !counts || !seg_expert || !seg_offsets || !seg_first_rank) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_segments(const_cast<int32_t*>(counts), nullptr, 0, v.E, v.C, seg_expert, seg_offsets,
                                       seg_first_rank, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_plan_balanced(const moe_shape_t* shape, const int32_t* counts, int32_t* seg_expert,
                               int32_t* seg_offsets, int32_t* seg_first_rank, int32_t* status, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (v.ec()) return MOE_ERR_INVALID_ARG;  // expert choice has its own calls
    if (v.rr()) return MOE_ERR_INVALID_ARG;  // re-routing has its own dispatch call
    if (v.R == 0 || !counts || !seg_expert || !seg_offsets || !seg_first_rank) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_plan(const_cast<int32_t*>(counts), nullptr, 0, v.E, v.R, v.S, v.k, v.B, seg_expert,
                                   seg_offsets, seg_first_rank, status, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_dispatch(const moe_shape_t* shape, const moe_bf16_t* x, const int32_t* topk_ids, int32_t plan_ready,
                          int32_t* counts, int32_t* seg_expert, int32_t* seg_offsets, int32_t* seg_first_rank,
                          int32_t* dest, int32_t* src, moe_bf16_t* xp, int32_t* status, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (v.ec()) return MOE_ERR_INVALID_ARG;  // expert choice has its own calls
    if (v.rr()) return MOE_ERR_INVALID_ARG;  // re-routing has its own dispatch call
    return dispatch_impl(v, x, topk_ids, plan_ready, counts, seg_expert, seg_offsets, seg_first_rank, dest, src, xp,
                         status, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_dispatch_static(const moe_shape_t* shape, const moe_bf16_t* x, const int32_t* topk_ids,
                                 int32_t plan_ready, int32_t* counts, int32_t* seg_expert, int32_t* seg_offsets,
                                 int32_t* seg_first_rank, int32_t* dest, int32_t* src, moe_bf16_t* xp,
                                 int32_t* status, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (v.ec()) return MOE_ERR_INVALID_ARG;  // expert choice has its own calls
    if (v.rr()) return MOE_ERR_INVALID_ARG;  // re-routing has its own dispatch call
    if (permute_ws_bytes(v.T, v.k, v.E) > kStaticScratchBytes) return MOE_ERR_UNSUPPORTED;
    void* scratch = static_scratch_address();
    if (scratch == nullptr) return MOE_ERR_CUDA;
    return dispatch_impl(v, x, topk_ids, plan_ready, counts, seg_expert, seg_offsets, seg_first_rank, dest, src, xp,
                         status, scratch, kStaticScratchBytes, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_dispatch_reroute(const moe_shape_t* shape, const moe_bf16_t* x, const int32_t* topk_ids,
                                  const float* logits, int32_t* counts, int32_t* seg_expert, int32_t* seg_offsets,
                                  int32_t* seg_first_rank, int32_t* dest, int32_t* src, moe_bf16_t* xp,
                                  int32_t* status, void* ws, size_t ws_bytes, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (!v.rr()) return MOE_ERR_INVALID_ARG;
    return reroute_impl(v, x, topk_ids, logits, counts, seg_expert, seg_offsets, seg_first_rank, dest, src, xp, status,
                        ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_expert_gate_up(const moe_shape_t* shape, const moe_bf16_t* xp, const int32_t* seg_expert,
                                const int32_t* seg_offsets, const moe_bf16_t* w_gate, const moe_bf16_t* w_up,
                                moe_bf16_t* hp, int32_t* status, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    return gate_up_impl(v, xp, seg_expert, seg_offsets, w_gate, w_up, hp, status, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_expert_down(const moe_shape_t* shape, const moe_bf16_t* hp, const int32_t* seg_expert,
                             const int32_t* seg_offsets, const moe_bf16_t* w_down, float* yp, int32_t* status,
                             moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    return down_impl(v, hp, seg_expert, seg_offsets, w_down, yp, status, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_expert_ffn(const moe_shape_t* shape, const moe_bf16_t* xp, const int32_t* seg_expert,
                            const int32_t* seg_offsets, const moe_bf16_t* w_gate, const moe_bf16_t* w_up,
                            const moe_bf16_t* w_down, moe_bf16_t* hp, float* yp, int32_t* status,
                            moe_stream_t stream) {
    Dims v;
    moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    s = gate_up_impl(v, xp, seg_expert, seg_offsets, w_gate, w_up, hp, status, st);
    if (s != MOE_OK) return s;
    return down_impl(v, hp, seg_expert, seg_offsets, w_down, yp, status, st);
}

moe_status_t moe_combine(const moe_shape_t* shape, const float* yp, const int32_t* dest, const float* topk_w,
                         void* out, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (v.ec()) return MOE_ERR_INVALID_ARG;  // expert choice has its own calls
    if (!yp || !dest || !topk_w || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(yp) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_combine(yp, dest, topk_w, nullptr, v.T, v.k, v.d, v.rows, out, v.out_bf16, sm_count(),
                                      static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_testing_dispatch_stalled(const moe_shape_t* shape, const moe_bf16_t* x, const int32_t* topk_ids,
                                          int32_t* counts, int32_t* seg_expert, int32_t* seg_offsets,
                                          int32_t* seg_first_rank, int32_t* dest, int32_t* src, moe_bf16_t* xp,
                                          int32_t* status, void* ws, size_t ws_bytes, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (v.ec()) return MOE_ERR_INVALID_ARG;  // expert choice has its own calls
    if (v.rr()) return MOE_ERR_INVALID_ARG;  // re-routing has its own dispatch call
    if (permute_n_tiles(v.T, v.k) < 2) return MOE_ERR_INVALID_ARG;  // needs a tile that waits on tile 0
    return dispatch_impl(v, x, topk_ids, 0, counts, seg_expert, seg_offsets, seg_first_rank, dest, src, xp, status,
                         ws, ws_bytes, static_cast<cudaStream_t>(stream), 1);
}

moe_status_t moe_testing_reroute_stalled(const moe_shape_t* shape, const moe_bf16_t* x, const int32_t* topk_ids,
                                         const float* logits, int32_t* counts, int32_t* seg_expert,
                                         int32_t* seg_offsets, int32_t* seg_first_rank, int32_t* dest, int32_t* src,
                                         moe_bf16_t* xp, int32_t* status, void* ws, size_t ws_bytes,
                                         moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (!v.rr()) return MOE_ERR_INVALID_ARG;
    if (static_cast<int64_t>(v.T) * v.k <= kRerouteThreads || v.T < 2) return MOE_ERR_INVALID_ARG;  // needs 2+ CTAs
    return reroute_impl(v, x, topk_ids, logits, counts, seg_expert, seg_offsets, seg_first_rank, dest, src, xp, status,
                        ws, ws_bytes, static_cast<cudaStream_t>(stream), true);
}

moe_status_t moe_testing_gemm_stalled(const moe_shape_t* shape, const moe_bf16_t* xp, const int32_t* seg_expert,
                                      const int32_t* seg_offsets, const moe_bf16_t* w_gate, const moe_bf16_t* w_up,
                                      moe_bf16_t* hp, int32_t* status, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (v.T == 0 || v.rows == 0) return MOE_ERR_INVALID_ARG;  // needs a tile whose wait can run out
    return gate_up_impl(v, xp, seg_expert, seg_offsets, w_gate, w_up, hp, status, static_cast<cudaStream_t>(stream),
                        true);
}

moe_status_t moe_combine_add(const moe_shape_t* shape, const float* yp, const int32_t* dest, const float* topk_w,
                             const float* base, void* out, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (v.ec()) return MOE_ERR_INVALID_ARG;  // expert choice has its own calls
    if (!yp || !dest || !topk_w || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(yp) || !aligned16(out) || (base && !aligned16(base))) return MOE_ERR_INVALID_ARG;
    if (v.out_bf16 && base != nullptr && static_cast<const void*>(base) == out) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_combine(yp, dest, topk_w, base, v.T, v.k, v.d, v.rows, out, v.out_bf16, sm_count(),
                                      static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_shared_expert(const moe_shape_t* shape, int32_t d_ff_shared, const moe_bf16_t* x,
                               const moe_bf16_t* w_gate_s, const moe_bf16_t* w_up_s, const moe_bf16_t* w_down_s,
                               moe_bf16_t* h_s, float* y_s, int32_t* status, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    const int Fs = d_ff_shared;
    if (Fs < 1) return MOE_ERR_INVALID_ARG;
    if (Fs % 64 != 0) return MOE_ERR_UNSUPPORTED;
    if (!x || !w_gate_s || !w_up_s || !w_down_s || !h_s || !y_s) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_gate_s) || !aligned16(w_up_s) || !aligned16(w_down_s) || !aligned16(h_s) ||
        !aligned16(y_s))
        return MOE_ERR_INVALID_ARG;
    if (v.T == 0) return MOE_OK;
    if (!have_encoder()) return MOE_ERR_CUDA;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    // one segment of all T rows and a single "expert": the same kernels as the routed FFN
    {
        const int bn = Fs >= 128 ? 128 : Fs;
        CUtensorMap ta, tg, tu;
        if (!tmap_rows(&ta, x, v.T, v.d) || !tmap_experts(&tg, w_gate_s, 1, Fs, v.d, bn) ||
            !tmap_experts(&tu, w_up_s, 1, Fs, v.d, bn))
            return MOE_ERR_CUDA;
        GemmArgs g{};
        g.seg_offsets = nullptr; g.seg_expert = nullptr; g.n_seg = 1; g.M = v.T; g.K = v.d; g.N = Fs;
        g.BN = bn; g.n_tiles_n = (Fs + bn - 1) / bn; g.mma_n = 2 * bn; g.stages = gemm_pick_stages(2 * bn);
        g.out = h_s; g.ldo = Fs; g.status = status;
        const int64_t tiles = static_cast<int64_t>((v.T + 127) / 128) * g.n_tiles_n;
        const int grid = static_cast<int>(std::min<int64_t>(sm_count(), tiles));
        const moe_status_t r = cuda_status(launch_umma_gemm(kEpiSwiglu, ta, tg, tu, g, grid, st));
        if (r != MOE_OK) return r;
    }
    {
        const int bn = v.d >= 256 ? 256 : v.d;
        CUtensorMap ta, tb;
        if (!tmap_rows(&ta, h_s, v.T, Fs) || !tmap_experts(&tb, w_down_s, 1, v.d, Fs, bn)) return MOE_ERR_CUDA;
        GemmArgs g{};
        g.seg_offsets = nullptr; g.seg_expert = nullptr; g.n_seg = 1; g.M = v.T; g.K = Fs; g.N = v.d;
        g.BN = bn; g.n_tiles_n = (v.d + bn - 1) / bn; g.mma_n = bn; g.stages = gemm_pick_stages(bn);
        g.out = y_s; g.ldo = v.d; g.status = status;
        g.swap_tail = (bn == 256 && Fs <= kSwapTailMaxK) ? kSwapTailRows : 0;
        const int64_t tiles = static_cast<int64_t>((v.T + 127) / 128) * g.n_tiles_n;
        const int grid = static_cast<int>(std::min<int64_t>(sm_count(), tiles));
        return cuda_status(launch_umma_gemm(kEpiStore, ta, tb, tb, g, grid, st));
    }
}

moe_status_t moe_route_scores(const moe_shape_t* shape, const moe_bf16_t* x, const moe_bf16_t* w_router,
                              const float* bias, float* scores, int32_t* status, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (!v.ec()) return MOE_ERR_INVALID_ARG;
    return route_scores_impl(v, x, w_router, bias, scores, status, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_expert_choose(const moe_shape_t* shape, const float* scores, const moe_bf16_t* x,
                               int32_t* seg_expert, int32_t* seg_offsets, int32_t* src, float* row_w, int32_t* emap,
                               moe_bf16_t* xp, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (!v.ec()) return MOE_ERR_INVALID_ARG;
    return choose_impl(v, scores, x, seg_expert, seg_offsets, src, row_w, emap, xp, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_combine_expert_choice(const moe_shape_t* shape, const float* yp, const int32_t* emap,
                                       const float* row_w, const float* base, void* out, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (!v.ec()) return MOE_ERR_INVALID_ARG;
    if (!yp || !emap || !row_w || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(yp) || !aligned16(out) || (base && !aligned16(base))) return MOE_ERR_INVALID_ARG;
    if (v.out_bf16 && base != nullptr && static_cast<const void*>(base) == out) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_ec_combine(yp, emap, row_w, base, v.T, v.E, v.d, v.rows, out, v.out_bf16, sm_count(),
                                         static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_routing_stats(const moe_shape_t* shape, const int32_t* counts, const int32_t* seg_expert,
                               const int32_t* seg_offsets, int32_t* stats, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (v.ec()) return MOE_ERR_INVALID_ARG;  // expert choice keeps no per-pair counts
    if (!seg_expert || !seg_offsets || !stats) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_routing_stats(counts, seg_expert, seg_offsets, v.E, v.n_seg, v.R, v.B, v.T * v.k,
                                            stats, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_layer_views(const moe_shape_t* shape, void* ws, moe_layer_views_t* views) {
    Dims v;
    const moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (!ws || !views) return MOE_ERR_INVALID_ARG;
    const LayerLayout L = layer_layout(v);
    uint8_t* b = static_cast<uint8_t*>(ws);
    views->topk_ids = reinterpret_cast<int32_t*>(b + L.ids);
    views->topk_w = reinterpret_cast<float*>(b + L.w);
    views->counts = reinterpret_cast<int32_t*>(b + L.counts);
    views->seg_expert = reinterpret_cast<int32_t*>(b + L.seg_expert);
    views->seg_offsets = reinterpret_cast<int32_t*>(b + L.seg_offsets);
    views->seg_first_rank = reinterpret_cast<int32_t*>(b + L.seg_first_rank);
    views->dest = reinterpret_cast<int32_t*>(b + L.dest);
    views->src = reinterpret_cast<int32_t*>(b + L.src);
    views->xp = reinterpret_cast<moe_bf16_t*>(b + L.xp);
    views->hp = reinterpret_cast<moe_bf16_t*>(b + L.hp);
    views->yp = reinterpret_cast<float*>(b + L.yp);
    views->dispatch_ws = b + L.dispatch_ws;
    views->dispatch_ws_bytes = L.dispatch_ws_bytes;
    views->scores = v.ec() ? reinterpret_cast<float*>(b + L.scores) : nullptr;
    views->emap = v.ec() ? reinterpret_cast<int32_t*>(b + L.emap) : nullptr;
    views->row_w = v.ec() ? reinterpret_cast<float*>(b + L.row_w) : nullptr;
    views->logits = v.rr() ? reinterpret_cast<float*>(b + L.logits) : nullptr;
    return MOE_OK;
}

moe_status_t moe_layer_fwd(const moe_shape_t* shape, const moe_bf16_t* x, const moe_bf16_t* w_router,
                           const float* bias, const moe_bf16_t* w_gate, const moe_bf16_t* w_up,
                           const moe_bf16_t* w_down, void* out, int32_t* status, void* ws, size_t ws_bytes,
                           moe_stream_t stream) {
    Dims v;
    moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (!out || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    const LayerLayout L = layer_layout(v);
    if (ws == nullptr || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_WORKSPACE;
    if (v.T == 0) return MOE_OK;
    moe_layer_views_t w;
    moe_layer_views(shape, ws, &w);
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* route_ws = static_cast<uint8_t*>(ws) + L.route_ws;
    const size_t route_ws_len = route_ws_bytes(v);
    if (v.ec()) {
        if (!route_split_impl(v, x, w_router, bias, nullptr, nullptr, nullptr, w.scores, status, route_ws,
                              route_ws_len, st, &s))
            s = route_scores_impl(v, x, w_router, bias, w.scores, status, st);
        if (s != MOE_OK) return s;
        s = choose_impl(v, w.scores, x, w.seg_expert, w.seg_offsets, w.src, w.row_w, w.emap, w.xp, st);
        if (s != MOE_OK) return s;
        s = gate_up_impl(v, w.xp, w.seg_expert, w.seg_offsets, w_gate, w_up, w.hp, status, st);
        if (s != MOE_OK) return s;
        s = down_impl(v, w.hp, w.seg_expert, w.seg_offsets, w_down, w.yp, status, st);
        if (s != MOE_OK) return s;
        return cuda_status(launch_ec_combine(w.yp, w.emap, w.row_w, nullptr, v.T, v.E, v.d, v.rows, out, v.out_bf16,
                                             sm_count(), st));
    }
    if (!route_split_impl(v, x, w_router, bias, w.logits, w.topk_ids, w.topk_w, nullptr, status, route_ws,
                          route_ws_len, st, &s))
        s = route_impl(v, x, w_router, bias, w.logits, w.topk_ids, w.topk_w, status, st);
    if (s != MOE_OK) return s;
    if (v.rr()) {
        s = reroute_impl(v, x, w.topk_ids, w.logits, w.counts, w.seg_expert, w.seg_offsets, w.seg_first_rank, w.dest,
                         w.src, w.xp, status, w.dispatch_ws, w.dispatch_ws_bytes, st);
        if (s != MOE_OK) return s;
        s = gate_up_impl(v, w.xp, w.seg_expert, w.seg_offsets, w_gate, w_up, w.hp, status, st);
        if (s != MOE_OK) return s;
        s = down_impl(v, w.hp, w.seg_expert, w.seg_offsets, w_down, w.yp, status, st);
        if (s != MOE_OK) return s;
        return cuda_status(
            launch_combine(w.yp, w.dest, w.topk_w, nullptr, v.T, v.k, v.d, v.rows, out, v.out_bf16, sm_count(), st));
    }
    s = dispatch_impl(v, x, w.topk_ids, 0, w.counts, w.seg_expert, w.seg_offsets, w.seg_first_rank, w.dest, w.src,
                      w.xp, status, w.dispatch_ws, w.dispatch_ws_bytes, st);
    if (s != MOE_OK) return s;
    s = gate_up_impl(v, w.xp, w.seg_expert, w.seg_offsets, w_gate, w_up, w.hp, status, st);
    if (s != MOE_OK) return s;
    s = down_impl(v, w.hp, w.seg_expert, w.seg_offsets, w_down, w.yp, status, st);
    if (s != MOE_OK) return s;
    return cuda_status(
        launch_combine(w.yp, w.dest, w.topk_w, nullptr, v.T, v.k, v.d, v.rows, out, v.out_bf16, sm_count(), st));
}

moe_status_t moe_layer_fwd_aux(const moe_shape_t* shape, const moe_bf16_t* x, const moe_bf16_t* w_router,
                               const float* bias, const moe_bf16_t* w_gate, const moe_bf16_t* w_up,
                               const moe_bf16_t* w_down, void* out, const moe_aux_t* aux, int32_t* status, void* ws,
                               size_t ws_bytes, moe_stream_t stream) {
    Dims v;
    moe_status_t s = check_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (aux && v.ec() && (aux->topk_ids || aux->topk_w || aux->dest || aux->counts || aux->stats))
        return MOE_ERR_INVALID_ARG;  // expert choice keeps no per-pair results
    s = moe_layer_fwd(shape, x, w_router, bias, w_gate, w_up, w_down, out, status, ws, ws_bytes, stream);
    if (s != MOE_OK || aux == nullptr || v.T == 0) return s;
    moe_layer_views_t w;
    moe_layer_views(shape, ws, &w);
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t tk = static_cast<size_t>(v.T) * v.k;
    auto copy = [&](void* dst, const void* src, size_t bytes) -> moe_status_t {
        if (dst == nullptr || bytes == 0) return MOE_OK;
        return cuda_status(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st));
    };
    if ((s = copy(aux->topk_ids, w.topk_ids, tk * 4)) != MOE_OK) return s;
    if ((s = copy(aux->topk_w, w.topk_w, tk * 4)) != MOE_OK) return s;
    if ((s = copy(aux->counts, w.counts, static_cast<size_t>(v.E) * 4)) != MOE_OK) return s;
    if ((s = copy(aux->seg_offsets, w.seg_offsets, static_cast<size_t>(v.n_seg + 1) * 4)) != MOE_OK) return s;
    if ((s = copy(aux->dest, w.dest, tk * 4)) != MOE_OK) return s;
    if (aux->stats)
        return cuda_status(launch_routing_stats(w.counts, w.seg_expert, w.seg_offsets, v.E, v.n_seg, v.R, v.B,
                                                v.T * v.k, aux->stats, st));
    return MOE_OK;
}

moe_status_t moe_ep_sizes(const moe_shape_t* shape, size_t* xp_bytes, size_t* replica_weight_bytes,
                          int32_t* n_local_segments) {
    Dims v;
    const moe_status_t s = check_ep_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (xp_bytes) *xp_bytes = static_cast<size_t>(v.S) * v.k * v.d * 2;
    if (replica_weight_bytes) *replica_weight_bytes = static_cast<size_t>(v.B) * 3 * v.d * v.F * 2;
    if (n_local_segments) *n_local_segments = v.E / v.R + v.B;
    return MOE_OK;
}

moe_status_t moe_ep_plan(const moe_shape_t* shape, int32_t rank, const int32_t* counts_all, int32_t* counts,
                         int32_t* seg_expert, int32_t* seg_slot, int32_t* seg_offsets, int32_t* status,
                         moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_ep_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (rank < 0 || rank >= v.R || !counts_all || !seg_expert || !seg_slot || !seg_offsets) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_ep_plan(counts_all, v.R, v.S, v.k, v.E, v.B, rank, counts, seg_expert, seg_slot,
                                      seg_offsets, status, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_ep_prefetch_weights(const moe_shape_t* shape, int32_t rank, const int32_t* seg_expert,
                                     const int32_t* seg_offsets, moe_bf16_t* const* w_gate, moe_bf16_t* const* w_up,
                                     moe_bf16_t* const* w_down, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_ep_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (rank < 0 || rank >= v.R || !seg_expert || !seg_offsets || !w_gate || !w_up || !w_down)
        return MOE_ERR_INVALID_ARG;
    EpPrefetchArgs a{};
    moe_bf16_t* const* tabs[3] = {w_gate, w_up, w_down};
    for (int m = 0; m < 3; ++m)
        for (int r = 0; r < v.R; ++r) {
            if (tabs[m][r] == nullptr || !aligned16(tabs[m][r])) return MOE_ERR_INVALID_ARG;
            a.w[m][r] = reinterpret_cast<__nv_bfloat16*>(tabs[m][r]);
        }
    a.seg_expert = seg_expert; a.seg_offsets = seg_offsets;
    a.R = v.R; a.E = v.E; a.B = v.B; a.F = v.F; a.d = v.d; a.rank = rank;
    return cuda_status(launch_ep_prefetch(a, sm_count(), static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_ep_dispatch(const moe_shape_t* shape, int32_t src_rank, int32_t n_src, const moe_bf16_t* const* x,
                             const int32_t* const* topk_ids, const int32_t* counts_all, int32_t* const* dest,
                             moe_bf16_t* const* xp, int32_t* const* src, int32_t* status, moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_ep_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (v.S * static_cast<int64_t>(v.k) > kCountMaxPairsPlan) return MOE_ERR_UNSUPPORTED;
    if (n_src < 1 || src_rank < 0 || src_rank + n_src > v.R) return MOE_ERR_INVALID_ARG;
    if (!x || !topk_ids || !counts_all || !dest || !xp || !src) return MOE_ERR_INVALID_ARG;
    EpDispatchArgs a{};
    for (int i = 0; i < n_src; ++i) {
        if (!x[i] || !topk_ids[i] || !dest[i] || !aligned16(x[i])) return MOE_ERR_INVALID_ARG;
        a.x[i] = reinterpret_cast<const __nv_bfloat16*>(x[i]);
        a.ids[i] = topk_ids[i];
        a.dest[i] = dest[i];
    }
    for (int r = 0; r < v.R; ++r) {
        if (!xp[r] || !src[r] || !aligned16(xp[r])) return MOE_ERR_INVALID_ARG;
        a.xp[r] = reinterpret_cast<__nv_bfloat16*>(xp[r]);
        a.src[r] = src[r];
    }
    a.counts_all = counts_all; a.status = status;
    a.R = v.R; a.S = v.S; a.k = v.k; a.E = v.E; a.d = v.d; a.B = v.B; a.n_seg = v.n_seg;
    a.src0 = src_rank; a.n_src = n_src;
    return cuda_status(launch_ep_dispatch(a, sm_count(), static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_ep_expert_ffn(const moe_shape_t* shape, const moe_bf16_t* xp, const int32_t* seg_slot,
                               const int32_t* seg_offsets, const moe_bf16_t* w_gate, const moe_bf16_t* w_up,
                               const moe_bf16_t* w_down, moe_bf16_t* hp, float* yp, int32_t* status,
                               moe_stream_t stream) {
    Dims v;
    moe_status_t s = check_ep_shape(shape, &v);
    if (s != MOE_OK) return s;
    const Dims l = ep_local_dims(v);
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    s = gate_up_impl(l, xp, seg_slot, seg_offsets, w_gate, w_up, hp, status, st);
    if (s != MOE_OK) return s;
    return down_impl(l, hp, seg_slot, seg_offsets, w_down, yp, status, st);
}

moe_status_t moe_ep_combine(const moe_shape_t* shape, int32_t src_rank, int32_t n_src, const float* const* yp,
                            const int32_t* const* dest, const float* const* topk_w, void* const* out,
                            moe_stream_t stream) {
    Dims v;
    const moe_status_t s = check_ep_shape(shape, &v);
    if (s != MOE_OK) return s;
    if (n_src < 1 || src_rank < 0 || src_rank + n_src > v.R) return MOE_ERR_INVALID_ARG;
    if (!yp || !dest || !topk_w || !out) return MOE_ERR_INVALID_ARG;
    EpCombineArgs a{};
    for (int r = 0; r < v.R; ++r) {
        if (!yp[r] || !aligned16(yp[r])) return MOE_ERR_INVALID_ARG;
        a.yp[r] = yp[r];
    }
    for (int i = 0; i < n_src; ++i) {
        if (!dest[i] || !topk_w[i] || !out[i] || !aligned16(out[i])) return MOE_ERR_INVALID_ARG;
        a.dest[i] = dest[i];
        a.w[i] = topk_w[i];
        a.out[i] = out[i];
    }
    a.R = v.R; a.S = v.S; a.k = v.k; a.d = v.d; a.n_src = n_src;
    (void)src_rank;  // the source rank only matters for the dispatch's global pair order
    return cuda_status(launch_ep_combine(a, v.out_bf16, sm_count(), static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
