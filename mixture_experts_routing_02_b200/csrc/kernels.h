// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 8;
constexpr int kMaxSegments = 2048;
constexpr size_t kGemmSmemBudget = 200 * 1024;  // operand stages of the GEMM
constexpr size_t kGemmSmemMin = 120 * 1024;     // > half an SM's shared memory: one CTA per SM
constexpr int kSwapTailRows = 32;                // down projection: largest segment tail computed
                                                 // with swapped operands
constexpr int kSwapTailMaxK = 4096;              // ... when its reduction (d_ff) is at most this long

enum EpiKind : int { kEpiRoute = 0, kEpiSwiglu = 1, kEpiStore = 2 };

struct GemmArgs {
    const int32_t* seg_offsets;  // [n_seg+1] or nullptr: a single segment of M rows
    const int32_t* seg_expert;   // [n_seg] or nullptr: expert 0
    int n_seg;
    int M;          // rows when seg_offsets == nullptr
    int K;          // reduction length, multiple of 64
    int N;          // valid output columns (route: E)
    int BN;         // output columns per tile
    int n_tiles_n;  // column tiles
    int mma_n;      // UMMA N
    int stages;     // smem pipeline depth
    void* out;      // bf16 Hp (SwiGLU epilogue) or fp32 Yp (store epilogue)
    int ldo;
    const float* bias;
    float* logits;
    int32_t* topk_ids;
    float* topk_w;
    int k;
    int route_flags;  // MOE_ROUTE_SOFTMAX_ALL: weights from a softmax over all N logits
    float* scores_t;  // route only: non-null = write softmax scores [N, M] (expert-major) instead of top-k
    int k_splits;          // plain fp32 epilogue only: > 1 cuts the reduction into this many parts
    size_t split_stride;   // elements between the outputs of consecutive parts
    int32_t* status;
    int test_skip_first_load;  // testing only: CTA 0 never issues its first stage's copy (its waits time out)
    int swap_tail;  // plain epilogue with 256-row B stages: a segment's last row tile holding at most
                    // this many rows is computed with the operands swapped (0: never)
};

size_t gemm_smem_bytes(int stages, int mma_n);
int gemm_pick_stages(int mma_n);
cudaError_t launch_umma_gemm(int epi, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                             const GemmArgs& g, int grid, cudaStream_t stream);

// dispatch.cu
constexpr int kPermuteThreads = 256;
constexpr int kPermutePairs = 256;          // most (t, j) pairs per look-back tile (one per thread)

struct PermuteArgs {
    const int32_t* ids;
    const __nv_bfloat16* x;
    __nv_bfloat16* xp;
    const int32_t* seg_expert;
    const int32_t* seg_offsets;
    const int32_t* seg_first_rank;
    int32_t* dest;
    int32_t* src;
    uint32_t* tile_state;  // [n_tiles * E], zero on entry
    uint32_t* ticket;      // zero on entry
    int32_t* status;
    int T, k, E, d, n_seg, tokens_per_tile, n_tiles;
    int rows;        // rows of xp: dest values outside [0, rows) are never written through
    int first_tile;  // 0; 1 only in moe_testing_dispatch_stalled (tile 0 is never taken)
    // single-launch dispatch (no plan, tables not given): it writes the tables itself
    int capacity;              // 0 = none
    int32_t* counts;           // [E] out
    int32_t* seg_expert_out;   // [E] out
    int32_t* seg_offsets_out;  // [E + 1] out
    int32_t* seg_first_rank_out;
    uint32_t* sync;            // [3] zero on entry: tiles ranked, tables ready, abort
    int prefetch_x;            // 1: prefetch the rows of X into L2 while the ranks are found
    int R, S, B;               // balanced plan (count dispatch only): groups, tokens per group, slots
};

constexpr int kMaxHistogramPartials = 64;   // CTAs of the fused histogram (one partial count row each)

int permute_tokens_per_tile(int T, int k);
int permute_n_tiles(int T, int k);
// Dispatch workspace: [ticket, 256 B][look-back words, n_tiles * E * 4 B] = the permutation's
// scratch, then [histogram partials, kMaxHistogramPartials * E * 4 B].
size_t permute_scratch_bytes(int T, int k, int E);
size_t permute_ws_bytes(int T, int k, int E);
int histogram_partial_ctas(int n_pairs);

cudaError_t launch_histogram(const int32_t* ids, int n_pairs, int E, int32_t* counts, int num_sms,
                             cudaStream_t stream);
// partial histograms (partials[histogram_partial_ctas(n)][E]) + clearing zero_bytes at zero_ptr
cudaError_t launch_histogram_partials(const int32_t* ids, int n_pairs, int E, int32_t* partials, uint32_t* zero_ptr,
                                      size_t zero_bytes, cudaStream_t stream);
// partials == nullptr: counts is the input; else counts is written as the sum of the partials
cudaError_t launch_segments(int32_t* counts, const int32_t* partials, int n_partials, int E, int capacity,
                            int32_t* seg_expert, int32_t* seg_offsets, int32_t* seg_first_rank, cudaStream_t stream);
cudaError_t launch_plan(int32_t* counts, const int32_t* partials, int n_partials, int E, int R, int S, int k, int B,
                        int32_t* seg_expert, int32_t* seg_offsets, int32_t* seg_first_rank, int32_t* status,
                        cudaStream_t stream);
// ws_cleared: the ticket and look-back words are already zero (cleared by the fused histogram)
cudaError_t launch_permute(const PermuteArgs& a, bool ws_cleared, int num_sms, cudaStream_t stream);
// Histogram, segment tables, stable rank and row copies in one launch (plain or capacity layout):
// with a look-back across tiles (any size), or with every CTA recounting all ids (up to
// kCountMaxPairs pairs; no communication between CTAs, no workspace).
cudaError_t launch_dispatch_fused(const PermuteArgs& a, int num_sms, cudaStream_t stream);
cudaError_t launch_dispatch_count(const PermuteArgs& a, int num_sms, cudaStream_t stream);
constexpr int kCountMaxPairs = 1 << 16;
constexpr int kCountMaxPairsPlan = 1 << 20;  // with a balanced plan the copies dwarf the recounting
constexpr int kRerouteMaxPairs = 1 << 19;    // re-routing: one CTA per SM holds 4096 pairs at most

// Overflow re-routing (the capacity rounds on a cooperative grid; T*k <= kRerouteMaxPairs), then the
// row copies.
constexpr int kRerouteThreads = 1024;
struct RerouteArgs {
    const int32_t* ids;
    const float* logits;  // [T, E] fp32: the candidate order of each token
    int T, k, E, capacity, rows;
    int32_t* counts;
    int32_t* seg_expert;
    int32_t* seg_offsets;
    int32_t* seg_first_rank;
    int32_t* dest;
    int32_t* src;
    // scratch, set by launch_reroute from the workspace
    uint8_t* cand;   // [T, cand_stride] each token's experts in candidate order (first E bytes of a row)
    int cand_stride; // E rounded up to 16: every row starts on a 16-byte boundary
    uint32_t* bar;   // [2] grid barrier (arrivals, generation); arrivals zero on entry
    int32_t* xchg;   // [2][kRerouteMaxCtas][kMaxExperts] per-CTA counts, two buffers used in turn
    int32_t* status; // MOE_DEV_ERR_TIMEOUT if a grid barrier wait runs out (nullable)
    int test_skip_arrival;  // testing only: CTA 0 never arrives at the first grid barrier
};
constexpr int kRerouteMaxCtas = 256;  // CTAs of the grid-wide rounds (one per SM at most)
size_t reroute_ws_bytes(int T, int k);
cudaError_t launch_reroute(const RerouteArgs& a, void* ws, const __nv_bfloat16* x, __nv_bfloat16* xp, int d,
                           int num_sms, cudaStream_t stream);
cudaError_t launch_route_from_logits(const float* logits, int T, int E, int k, int route_flags, int32_t* ids,
                                     float* w, int num_sms, cudaStream_t stream);
// Routing from n_split partial logit slices (summed in order, + bias): top-k ids and weights, or
// expert-choice scores (scores_t [E, T]) when scores_t is non-null; logits optional.
cudaError_t launch_route_logits(const float* part, int n_split, int ldp, size_t split_stride, const float* bias, int T,
                                int E, int k, int route_flags, float* logits, int32_t* ids, float* w, float* scores_t,
                                int num_sms, cudaStream_t stream);

// combine.cu
// out: [T, d] fp32, or bf16 when out_bf16
cudaError_t launch_combine(const float* yp, const int32_t* dest, const float* w, const float* base, int T, int k,
                           int d, int rows, void* out, bool out_bf16, int num_sms, cudaStream_t stream);

// expert_choice.cu
constexpr int kSelectThreads = 1024;  // one CTA per expert
cudaError_t launch_ec_select(const float* scores_t, int T, int E, int cp, int32_t* seg_expert, int32_t* seg_offsets,
                             int32_t* src, float* row_w, int32_t* emap, cudaStream_t stream);
cudaError_t launch_ec_gather(const __nv_bfloat16* x, const int32_t* src, int rows, int T, int d, __nv_bfloat16* xp,
                             int num_sms, cudaStream_t stream);
cudaError_t launch_ec_combine(const float* yp, const int32_t* emap, const float* row_w, const float* base, int T,
                              int E, int d, int rows, void* out, bool out_bf16, int num_sms, cudaStream_t stream);

// ep.cu: expert parallelism over R ranks (pointer tables hold each rank's buffer; on one GPU the
// "ranks" are local buffers)
constexpr int kEpMaxRanks = 16;
struct EpDispatchArgs {
    const __nv_bfloat16* x[kEpMaxRanks];  // [n_src] source ranks' X [S, d]
    const int32_t* ids[kEpMaxRanks];      // [n_src] [S * k]
    int32_t* dest[kEpMaxRanks];           // [n_src] [S * k] out: owner * S*k + row
    __nv_bfloat16* xp[kEpMaxRanks];       // [R] each owner's Xp [S*k, d]
    int32_t* src[kEpMaxRanks];            // [R] each owner's src [S*k]: global pair index
    const int32_t* counts_all;            // [R, E]
    int32_t* status;
    int R, S, k, E, d, B, n_seg, src0, n_src, ctas_per_src;
    // optional (nullable): the totals and the tables of all R groups, written by CTA 0 (the
    // single-GPU balanced dispatch, where the R groups are token groups of one GPU)
    int32_t* counts_out;          // [E]
    int32_t* seg_expert_out;      // [n_seg]
    int32_t* seg_offsets_out;     // [n_seg + 1]
    int32_t* seg_first_rank_out;  // [n_seg]
};
struct EpCombineArgs {
    const float* yp[kEpMaxRanks];        // [R] each owner's Yp [S*k, d]
    const int32_t* dest[kEpMaxRanks];    // [n_src]
    const float* w[kEpMaxRanks];         // [n_src] router weights [S, k]
    void* out[kEpMaxRanks];              // [n_src] [S, d] fp32 or bf16
    int R, S, k, d, n_src;
};
struct EpPrefetchArgs {
    __nv_bfloat16* w[3][kEpMaxRanks];  // gate, up, down: each rank's [E/R + B, F, d] (down: [.., d, F])
    const int32_t* seg_expert;         // [E/R + B] of this rank (global expert ids)
    const int32_t* seg_offsets;        // [E/R + B + 1]
    int R, E, B, F, d, rank;
};
cudaError_t launch_ep_plan(const int32_t* counts_all, int R, int S, int k, int E, int B, int rank, int32_t* counts,
                           int32_t* seg_expert, int32_t* seg_slot, int32_t* seg_offsets, int32_t* status,
                           cudaStream_t stream);
cudaError_t launch_ep_prefetch(const EpPrefetchArgs& a, int num_sms, cudaStream_t stream);
cudaError_t launch_ep_dispatch(const EpDispatchArgs& a, int num_sms, cudaStream_t stream);
// counts_all[g, e] = pairs of expert e among the S*k pairs of token group g (cleared, then counted
// by about num_sms CTAs)
cudaError_t launch_group_histogram(const int32_t* ids, int R, int S, int k, int E, int32_t* counts_all,
                                   int num_sms, cudaStream_t stream);
cudaError_t launch_ep_combine(const EpCombineArgs& a, bool out_bf16, int num_sms, cudaStream_t stream);

// stats.cu: MOE_STAT_COUNT values from the counts (nullable) and segment tables of one dispatch
cudaError_t launch_routing_stats(const int32_t* counts, const int32_t* seg_expert, const int32_t* seg_offsets,
                                 int E, int n_seg, int R, int B, int pairs, int32_t* stats, cudaStream_t stream);

}  // namespace moe
