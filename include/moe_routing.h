/*
 * moe_routing.h -- C ABI of the single-GPU top-k Mixture-of-Experts FFN
 * layer forward for NVIDIA B200 (sm_100a).
 *
 * The layer (forward pipeline of "Sparsely-Gated MoE 구현 관점에서 살펴보기:
 * Router, Top-k, 부하 분산", section "순전파 과정(forward pass)은 디스패치와
 * 결합(combine)을 포함"):
 *
 *   logits = X W_r^T (+ b)                        moe_route
 *   ids, w = top-k of logits, softmax over them     moe_route / moe_route_from_logits
 *   counts = per-expert histogram of ids            moe_histogram
 *   segments (expert-contiguous layout), either
 *     one per expert, capped at C rows            moe_segments
 *     or the balanced plan over R groups          moe_plan_balanced
 *   Xp = rows of X written to their final slots     moe_dispatch
 *   Hp = silu(Xp W_g^T) * (Xp W_u^T)  per segment  moe_expert_gate_up
 *   Yp = Hp W_d^T                     per segment  moe_expert_down
 *   out[t] = sum_j w[t,j] Yp[dest[t*k+j]]           moe_combine
 *   all of the above in one call                    moe_layer_fwd
 *
 * Conventions for every call:
 *  - Tensor arguments are DEVICE pointers owned by the caller; the library
 *    allocates and frees nothing, keeps no per-call state and never
 *    synchronises the host.  All work is enqueued on `stream` (a
 *    cudaStream_t; NULL is the legacy default stream) and is asynchronous.
 *  - bf16 tensors are passed as `moe_bf16_t` (raw IEEE bfloat16 bits).
 *  - All matrices are row-major and dense.  Weights use the nn.Linear
 *    [out, in] layout: W_r [E, d], W_g and W_u [E, F, d], W_d [E, d, F].
 *  - The return value reports errors that the host can see before anything
 *    is enqueued (bad arguments, unsupported sizes, launch failures).  In
 *    that case nothing, or only a prefix of a composite call, was enqueued.
 *  - Errors only the device can see (an infeasible balanced plan, a bounded
 *    wait that ran out) are OR-ed into the caller's `int32_t *status` device
 *    word (MOE_DEV_ERR_* bits; 0 = fine).  The caller clears it and reads it
 *    whenever it next synchronises.  `status` may be NULL to ignore them.
 *  - Every wait inside a kernel is bounded (about two seconds); a wait that
 *    runs out sets MOE_DEV_ERR_TIMEOUT and the kernel returns.
 *
 * Supported sizes: 0 <= T, T*k < 2^30; 1 <= E <= 256; 1 <= k <= min(E, 8);
 * d_model and d_ff multiples of 64 (>= 64); at most 2048 segments.
 */
#ifndef MOE_ROUTING_H
#define MOE_ROUTING_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef uint16_t moe_bf16_t;
typedef void *moe_stream_t; /* cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* null pointer, negative size, k > E, bad group split */
    MOE_ERR_UNSUPPORTED = 2, /* sizes outside the supported range above */
    MOE_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required */
    MOE_ERR_CUDA = 4         /* a CUDA runtime call or launch failed */
} moe_status_t;

/* bits of the device status word */
#define MOE_DEV_ERR_PLAN 0x1    /* balanced plan needs more than B replica slots */
#define MOE_DEV_ERR_TIMEOUT 0x2 /* a bounded wait inside a kernel ran out */

/*
 * Layer shape.
 *   T              tokens (rows of X)
 *   d_model        hidden size d
 *   n_experts      E
 *   top_k          k
 *   d_ff           expert FFN inner size F
 *   capacity       0 = no limit; else C, the most rows one expert keeps.
 *                  A (t, j) pair whose stable rank inside its expert (pairs
 *                  ordered by q = t*k + j) is >= C is dropped: dest = -1, it
 *                  contributes nothing, and the kept weights of that token
 *                  are not renormalised.  ("로드 밸런싱 손실(load-balancing
 *                  loss)과 용량(capacity)은 별개": overflow skips the expert
 *                  and leaves only the residual path.)  The caller computes C,
 *                  e.g. ceil(cf * T * k / E).
 *   n_groups       R; 0 = no balanced plan.  With R > 0 the E experts are
 *                  homed in R contiguous groups of E/R, the T tokens form R
 *                  groups of S = T/R, and every group receives exactly S*k
 *                  rows ("가장 바쁜 랭크가 속도를 정합니다: MoonEP의 계획 코드를 직접
 *                  돌려봤습니다", sections "개요" and "이 기술은 무엇인가").
 *                  Requires E % R == 0, T % R == 0 and capacity == 0.
 *   replica_slots  B, replica slots per group (the page's [E, E+B) slots).
 *   route_flags    0: weights = softmax over the k selected logits (default);
 *                  MOE_ROUTE_SOFTMAX_ALL: weights = softmax over all E logits,
 *                  taken at the k selected experts and not renormalised (they
 *                  sum to less than 1).  "Sparsely-Gated MoE 구현 관점에서
 *                  살펴보기", section "Top-2 라우팅의 수치 예시": whether the
 *                  softmax comes before or after the top-k differs between
 *                  implementations; with renormalisation both orders agree.
 *                  MOE_ROUTE_EXPERT_CHOICE: experts choose tokens instead of
 *                  tokens choosing experts ("Expert를 똑같이 나눴는데도 GPU가
 *                  대기하는 이유: MoE의 토큰 쏠림", section "라우팅 분포와 학습
 *                  안정성").  Scores S[t, e] = softmax over the E logits of
 *                  token t; expert e keeps the C tokens with the largest
 *                  S[t, e] (equal scores: the lower token id), laid out in
 *                  ascending token order in segment e, which holds
 *                  C' = min(C, T) rows; token t's output is the sum of
 *                  S[t, e] * FFN_e(x_t) over the experts that kept it (0 if
 *                  none did).  Requires capacity >= 1 (the C above) and
 *                  n_groups == 0; excludes MOE_ROUTE_SOFTMAX_ALL; top_k is
 *                  not used by the selection (only validated).  n_seg = E,
 *                  rows_alloc = E * C'.  Takes moe_route_scores,
 *                  moe_expert_choose and moe_combine_expert_choice in place of
 *                  moe_route, moe_dispatch and moe_combine, which reject it.
 *                  MOE_ROUTE_REROUTE: with a capacity, a pair over its expert's
 *                  capacity goes to another candidate instead of being dropped
 *                  ("Sparsely-Gated MoE 구현 관점에서 살펴보기", section "로드 밸런싱
 *                  손실(load-balancing loss)과 용량(capacity)은 별개").  Round 0 is
 *                  the capacity rule; in round r >= 1 every unplaced pair
 *                  proposes to its token's next candidate in logit order (below
 *                  its top-k; equal logits: lower id) among the experts that had
 *                  room when the round began, a token's unplaced pairs taking
 *                  consecutive candidates in j order; each expert accepts the
 *                  round's proposals in q order while it has room; a pair with
 *                  no candidate left is dropped.  A moved pair keeps its routing
 *                  weight.  Segment e holds its rows round by round, q order
 *                  inside a round.  Requires capacity >= 1, n_groups == 0 and
 *                  T * k <= 524288 (2^19); excludes MOE_ROUTE_EXPERT_CHOICE.  Takes
 *                  moe_dispatch_reroute (which needs the router's fp32 logits) in
 *                  place of moe_dispatch, which rejects it.
 */
#define MOE_ROUTE_SOFTMAX_ALL 0x1
#define MOE_ROUTE_EXPERT_CHOICE 0x2
#define MOE_ROUTE_REROUTE 0x4

/*
 *   out_dtype      element type of the layer output out [T, d] written by
 *                  moe_combine, moe_combine_add, moe_combine_expert_choice and
 *                  moe_layer_fwd: MOE_DTYPE_F32 (0, the value of a
 *                  zero-initialised shape) stores the fp32 accumulator;
 *                  MOE_DTYPE_BF16 rounds it once to bf16 (round to nearest
 *                  even), half the bytes written and read back by the caller.
 *                  Yp stays fp32 either way.
 */
#define MOE_DTYPE_F32 0
#define MOE_DTYPE_BF16 1

typedef struct {
    int32_t T;
    int32_t d_model;
    int32_t n_experts;
    int32_t top_k;
    int32_t d_ff;
    int32_t capacity;
    int32_t n_groups;
    int32_t replica_slots;
    int32_t route_flags;
    int32_t out_dtype;
} moe_shape_t;

/*
 * Segment tables.  The dispatched rows Xp / Hp / Yp are laid out as n_seg
 * consecutive segments; segment s holds rows [seg_offsets[s],
 * seg_offsets[s+1]) of expert seg_expert[s] (-1 = unused slot, 0 rows), and
 * its first row is the pair of within-expert rank seg_first_rank[s].  This is
 * the device-side cu_seqlens of the MoonEP page ("설치 및 통합").
 *   no plan:  n_seg = E, segment e = expert e, min(count_e, C) rows.
 *   plan:     n_seg = R * (E/R + B); group g owns segments
 *             [g*(E/R+B), (g+1)*(E/R+B)): its E/R home experts in ascending
 *             id, then its B replica slots in creation order; it spans rows
 *             [g*S*k, (g+1)*S*k).
 */

/* Human-readable name of a moe_status_t. */
MOE_API const char *moe_status_string(moe_status_t s);

/*
 * Sizes implied by a shape: *n_segments (as above) and *rows_alloc, the rows
 * Xp, Hp and Yp must have: T*k without capacity, min(T*k, C*E) with it.
 * Host only; enqueues nothing.  Either output pointer may be NULL.
 */
MOE_API moe_status_t moe_layout(const moe_shape_t *shape, int32_t *n_segments, int32_t *rows_alloc);

/*
 * Workspace bytes for moe_dispatch (*dispatch_bytes) and for moe_layer_fwd
 * (*layer_bytes, which also holds every intermediate of the layer).  Host
 * only.  Either output pointer may be NULL.
 */
MOE_API moe_status_t moe_workspace_size(const moe_shape_t *shape, size_t *dispatch_bytes, size_t *layer_bytes);

/*
 * Router projection fused with top-k and the renormalised softmax
 * ("Sparsely-Gated MoE 구현 관점에서 살펴보기", sections "Router를 텐서 형태에서
 * 추적하기", "Top-2 라우팅의 수치 예시", "pure Python으로 Top-k Router 확인하기").
 *   x        [T, d] bf16            w_router [E, d] bf16
 *   bias     [E] fp32 or NULL; added to the logits before selection
 *   logits   [T, E] fp32 out, or NULL to skip writing it
 *   topk_ids [T, k] int32 out: the k largest logits, descending; equal
 *            values go to the lower expert id
 *   topk_w   [T, k] fp32 out: w_j = exp(l_j - l_max) / sum_sel exp(l - l_max)
 *            (with MOE_ROUTE_SOFTMAX_ALL the sum runs over all E logits)
 * The projection runs on the tensor cores (bf16 in, fp32 accumulate); the
 * selection is made on the fp32 logits.
 */
MOE_API moe_status_t moe_route(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *w_router,
                       const float *bias, float *logits, int32_t *topk_ids, float *topk_w,
                       int32_t *status, moe_stream_t stream);

/* Top-k selection and weights alone, on given fp32 logits [T, E] (same selection and weights as moe_route). */
MOE_API moe_status_t moe_route_from_logits(const moe_shape_t *shape, const float *logits, int32_t *topk_ids,
                                   float *topk_w, moe_stream_t stream);

/*
 * Histogram: counts[e] = number of (t, j) with topk_ids[t, j] == e, raw (before any
 * capacity).  ("5.3 Expert Parallelism", section "2. 디스패처 엔지니어링":
 * the per-destination bincount; MoonEP page "설치 및 통합": tokens_per_expert.)
 *   topk_ids [T, k] int32 in, values in [0, E)     counts [E] int32 out
 */
MOE_API moe_status_t moe_histogram(const moe_shape_t *shape, const int32_t *topk_ids, int32_t *counts,
                           moe_stream_t stream);

/*
 * Plain segment layout: one segment per expert holding min(counts[e], C)
 * rows (all of them when capacity == 0); seg_offsets is the exclusive scan.
 *   counts [E] in; seg_expert [E], seg_offsets [E+1], seg_first_rank [E] out.
 * Requires n_groups == 0.
 */
MOE_API moe_status_t moe_segments(const moe_shape_t *shape, const int32_t *counts, int32_t *seg_expert,
                          int32_t *seg_offsets, int32_t *seg_first_rank, moe_stream_t stream);

/*
 * Balanced plan (MoonEP page, sections "개요", "이 기술은 무엇인가",
 * "설치 및 통합", "실제 실험 결과").  Every one of the R groups receives
 * exactly S*k rows; overloaded groups give rows of their most loaded experts
 * (descending count, ties to the lower id) to underloaded groups, which hold
 * them in replica slots.  Deterministic; the algorithm, which the page does
 * not give, is: groups above S*k in ascending order queue their excess as
 * (expert, rows) chunks; groups below S*k in ascending order take their
 * deficit from the front of that queue, one replica slot per (expert, group)
 * piece; an expert's rows in stable order fill its home segment first, then
 * its pieces in creation order.
 *   counts [E] in (Σ counts must be T*k); seg tables [n_seg] / [n_seg+1] out.
 * If some group would need more than B slots the plan is infeasible (the
 * page's `alloc.sum(dim=0) > CAP` error): MOE_DEV_ERR_PLAN is set in *status
 * and every segment is written empty, so later calls move and compute nothing.
 */
MOE_API moe_status_t moe_plan_balanced(const moe_shape_t *shape, const int32_t *counts, int32_t *seg_expert,
                               int32_t *seg_offsets, int32_t *seg_first_rank, int32_t *status,
                               moe_stream_t stream);

/*
 * Dispatch.  When plan_ready == 0 this computes counts
 * and the segment tables first (as moe_histogram, then moe_plan_balanced if
 * n_groups > 0 else moe_segments), writing them to the given buffers; when
 * plan_ready != 0 they are inputs from earlier calls.  Each pair gets its
 * stable rank r inside its expert (pairs in q = t*k + j order) and its final
 * row
 *   dest[t*k+j] = seg_offsets[s] + r - seg_first_rank[s]
 * for the segment s of that expert covering rank r (-1 if none: dropped), and
 * the token's row is copied straight to that slot ("MoonEP", section "이 기술은
 * 무엇인가": writing each row to its final position makes the separate sort
 * and copy disappear):
 *   Xp[dest[t*k+j]] = X[t],  src[dest[q]] = q.
 *   x [T, d] bf16 in; dest [T*k] int32 out; src [rows_alloc] int32 out;
 *   xp [rows_alloc, d] bf16 out (rows past seg_offsets[n_seg] untouched).
 *   ws, ws_bytes: at least moe_workspace_size()'s dispatch_bytes of device
 *   memory; its contents need not be initialised and are clobbered.
 * Kernels: with plan_ready == 0, one launch (no plan and T*k <= 65536, or a
 * plan and T*k <= 2^20: every CTA counts all ids itself and computes the
 * tables; no plan and larger: a memset and one launch with a decoupled
 * look-back over tiles of pairs); otherwise the histogram, the plan, the
 * look-back ranks and the row copies as separate launches.
 */
MOE_API moe_status_t moe_dispatch(const moe_shape_t *shape, const moe_bf16_t *x, const int32_t *topk_ids,
                          int32_t plan_ready, int32_t *counts, int32_t *seg_expert,
                          int32_t *seg_offsets, int32_t *seg_first_rank, int32_t *dest,
                          int32_t *src, moe_bf16_t *xp, int32_t *status, void *ws, size_t ws_bytes,
                          moe_stream_t stream);

/*
 * moe_dispatch without a workspace argument, for callers that cannot allocate
 * device memory: code that runs while a stream is being captured into a CUDA
 * graph (where cudaMalloc is not allowed), plug-in hooks of runtimes that hand
 * over only input and output buffers, and processes whose device memory is
 * already fully reserved by a pool they do not own.  The pages have no
 * counterpart of this call; it is a convenience of this library.
 *
 * Arguments and results are those of moe_dispatch.  The look-back scratch
 * (ticket + per-tile words) is taken from one 4 MiB array in the library's
 * device image instead of `ws`; every GPU on which the library is loaded holds
 * those 4 MiB until the process exits.  Shapes whose scratch would exceed
 * 4 MiB (256 + n_tiles * E * 4 + 64 * E * 4 bytes, n_tiles = ceil(T /
 * max(1, 256 / k))) are rejected with MOE_ERR_UNSUPPORTED before anything is
 * enqueued.  No call allocates: the first call on each device looks up the
 * array's device address (cudaGetSymbolAddress, with that device current) and
 * caches it, so make that first call before any stream capture begins.
 *
 * All calls share the one array.  Each call clears the part it needs on
 * `stream` before using it, but two calls whose work can overlap on the same
 * GPU (different streams without ordering between them, or different host
 * threads) race on the array and give wrong results: order them.
 */
MOE_API moe_status_t moe_dispatch_static(const moe_shape_t *shape, const moe_bf16_t *x,
                                 const int32_t *topk_ids, int32_t plan_ready, int32_t *counts,
                                 int32_t *seg_expert, int32_t *seg_offsets,
                                 int32_t *seg_first_rank, int32_t *dest, int32_t *src,
                                 moe_bf16_t *xp, int32_t *status, moe_stream_t stream);

/*
 * Grouped GEMM of the gate and up projections fused with SwiGLU
 * ("5.3 Expert Parallelism", section "3. 고도화된 최적화: 오버래핑(Overlapping) 및
 * GroupGEMM": all experts' GEMMs in one launch):
 *   Hp[r, :] = silu(Xp[r] W_g[e]^T) * (Xp[r] W_u[e]^T),  e = expert of r's segment,
 * silu(z) = z / (1 + exp(-z)); fp32 accumulation in tensor memory, Hp
 * rounded to bf16.  Segment sizes are read on the device (no host sync).
 *   xp [rows_alloc, d]; w_gate, w_up [E, F, d]; hp [rows_alloc, F] out.
 */
MOE_API moe_status_t moe_expert_gate_up(const moe_shape_t *shape, const moe_bf16_t *xp,
                                const int32_t *seg_expert, const int32_t *seg_offsets,
                                const moe_bf16_t *w_gate, const moe_bf16_t *w_up, moe_bf16_t *hp,
                                int32_t *status, moe_stream_t stream);

/*
 * Grouped down projection Yp[r, :] = Hp[r] W_d[e]^T, accumulated in fp32 and
 * stored in fp32 (Yp is only read by the combine; keeping it in fp32 leaves
 * one rounding, the bf16 Hp operand, between the expert and the output).
 *   hp [rows_alloc, F] bf16; w_down [E, d, F] bf16; yp [rows_alloc, d] fp32 out.
 * Tiles of 128 rows x 256 columns, one CTA each; with d_ff <= 4096 a segment's
 * last tile of at most 32 rows is computed with the weight tile as the 128-row
 * MMA operand and its rows as the narrow one (same results within fp32
 * accumulation order).
 */
MOE_API moe_status_t moe_expert_down(const moe_shape_t *shape, const moe_bf16_t *hp,
                             const int32_t *seg_expert, const int32_t *seg_offsets,
                             const moe_bf16_t *w_down, float *yp, int32_t *status,
                             moe_stream_t stream);

/* moe_expert_gate_up then moe_expert_down. */
MOE_API moe_status_t moe_expert_ffn(const moe_shape_t *shape, const moe_bf16_t *xp, const int32_t *seg_expert,
                            const int32_t *seg_offsets, const moe_bf16_t *w_gate,
                            const moe_bf16_t *w_up, const moe_bf16_t *w_down, moe_bf16_t *hp,
                            float *yp, int32_t *status, moe_stream_t stream);

/*
 * Combine ("Sparsely-Gated MoE 구현 관점에서 살펴보기", section "순전파 과정
 * ...", last step: un-permute and weight by the router; MoonEP page
 * "설치 및 통합": combine):
 *   out[t] = sum over j with dest[t*k+j] >= 0 of topk_w[t, j] * Yp[dest[t*k+j]]
 * accumulated in fp32 in ascending j and stored in shape->out_dtype: the fp32
 * accumulator, or that value rounded once to bf16.  A token whose pairs were all
 * dropped gets 0.
 *   yp [rows_alloc, d] fp32; dest [T*k]; topk_w [T, k];
 *   out [T, d] fp32 or bf16 (16-byte aligned).
 */
MOE_API moe_status_t moe_combine(const moe_shape_t *shape, const float *yp, const int32_t *dest,
                         const float *topk_w, void *out, moe_stream_t stream);

/*
 * Combine with a base term: out[t] = base[t] + the combine above (base [T, d]
 * fp32, nullable: then identical to moe_combine), stored in shape->out_dtype.
 * With base = the shared expert's output (moe_shared_expert) this finishes a
 * layer with a shared expert.  out may alias base when out is fp32; with a bf16
 * out an aliasing base is rejected (MOE_ERR_INVALID_ARG).
 */
MOE_API moe_status_t moe_combine_add(const moe_shape_t *shape, const float *yp, const int32_t *dest,
                             const float *topk_w, const float *base, void *out,
                             moe_stream_t stream);

/*
 * Shared expert: a dense SwiGLU FFN applied to every token, y_s = silu(X W_gs^T) *
 * (X W_us^T) W_ds^T ("5.3 Expert Parallelism", section "3. 고도화된 최적화:
 * 오버래핑(Overlapping) 및 GroupGEMM", first optimisation: the shared expert is
 * local to every device, so its GEMMs can run on a second stream while the
 * routed tokens are being routed and dispatched).  Same tensor-core kernels as
 * the routed experts, as one segment of T rows.
 *   d_ff_shared  F_s, multiple of 64
 *   x [T, d] bf16; w_gate_s, w_up_s [F_s, d] bf16; w_down_s [d, F_s] bf16
 *   h_s [T, F_s] bf16 (scratch, written); y_s [T, d] fp32 out.
 * Enqueued on `stream`; to overlap, use a stream other than the routed path's
 * and make moe_combine_add wait for it.
 */
MOE_API moe_status_t moe_shared_expert(const moe_shape_t *shape, int32_t d_ff_shared, const moe_bf16_t *x,
                               const moe_bf16_t *w_gate_s, const moe_bf16_t *w_up_s,
                               const moe_bf16_t *w_down_s, moe_bf16_t *h_s, float *y_s,
                               int32_t *status, moe_stream_t stream);

/*
 * The whole layer: moe_route_ws (logits not stored) -> moe_dispatch ->
 * moe_expert_gate_up -> moe_expert_down -> moe_combine, all on `stream`.
 * With MOE_ROUTE_EXPERT_CHOICE: moe_route_scores_ws -> moe_expert_choose ->
 * moe_expert_gate_up -> moe_expert_down -> moe_combine_expert_choice; the
 * views topk_ids, topk_w, dest, seg_first_rank and dispatch_ws are then unused.
 * With MOE_ROUTE_REROUTE the dispatch is moe_dispatch_reroute (the logits are
 * then kept in the workspace).
 * out [T, d] in shape->out_dtype (fp32, or bf16 as the pages' layer returns
 * it).  The intermediates live in `ws` (moe_workspace_size()'s layer_bytes);
 * their addresses are given by moe_layer_views.
 */
MOE_API moe_status_t moe_layer_fwd(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *w_router,
                           const float *bias, const moe_bf16_t *w_gate, const moe_bf16_t *w_up,
                           const moe_bf16_t *w_down, void *out, int32_t *status, void *ws,
                           size_t ws_bytes, moe_stream_t stream);

/*
 * Testing only: moe_dispatch (plan_ready = 0) with tile 0 of the stable-rank pass
 * never taken, so every other tile's look-back waits on a flag that nothing sets.
 * Each such wait gives up after its bound (about 2 s), sets MOE_DEV_ERR_TIMEOUT in
 * *status and returns; dest / src / xp are then incomplete (pairs whose dest was
 * not written keep the caller's values; values outside [0, rows_alloc) are never
 * written through).  It shows that a wait that cannot end returns an error
 * instead of hanging, and that the context stays usable.  Needs T large enough
 * for at least two tiles (T * k > 256).
 */
MOE_API moe_status_t moe_testing_dispatch_stalled(const moe_shape_t *shape, const moe_bf16_t *x,
                                          const int32_t *topk_ids, int32_t *counts,
                                          int32_t *seg_expert, int32_t *seg_offsets,
                                          int32_t *seg_first_rank, int32_t *dest, int32_t *src,
                                          moe_bf16_t *xp, int32_t *status, void *ws, size_t ws_bytes,
                                          moe_stream_t stream);

/*
 * Testing only: moe_dispatch_reroute in which CTA 0 of the re-routing rounds'
 * cooperative grid never arrives at the first grid barrier, so every other CTA's
 * wait there can never end.  Each wait gives up after its bound (about 2 s), sets
 * MOE_DEV_ERR_TIMEOUT in *status and its CTA returns; counts, the tables, dest,
 * src and xp are then incomplete (values outside [0, rows_alloc) are never written
 * through).  It shows that the grid barrier returns an error instead of hanging and
 * leaves the context usable.  Needs MOE_ROUTE_REROUTE and T * k > 1024 (two CTAs).
 */
MOE_API moe_status_t moe_testing_reroute_stalled(const moe_shape_t *shape, const moe_bf16_t *x,
                                         const int32_t *topk_ids, const float *logits, int32_t *counts,
                                         int32_t *seg_expert, int32_t *seg_offsets, int32_t *seg_first_rank,
                                         int32_t *dest, int32_t *src, moe_bf16_t *xp, int32_t *status,
                                         void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Testing only: moe_expert_gate_up in which CTA 0 never issues the copy of its
 * first pipeline stage, so the tensor-core issuer's wait on that stage can never
 * end.  The wait gives up after its bound (about 2 s), sets MOE_DEV_ERR_TIMEOUT
 * in *status and raises the CTA's abort flag; the copy issuer and the epilogue
 * warps see it and stop, the copies already in flight are waited for (bounded),
 * and the CTA frees its tensor memory before it exits.  The tiles of CTA 0 are
 * not written; the other CTAs' tiles are.  It shows that the GEMM's abort path
 * returns an error instead of hanging and leaves the context (and the SMs'
 * tensor memory) usable.  Needs at least one row (rows_alloc > 0 and T > 0).
 */
MOE_API moe_status_t moe_testing_gemm_stalled(const moe_shape_t *shape, const moe_bf16_t *xp,
                                      const int32_t *seg_expert, const int32_t *seg_offsets,
                                      const moe_bf16_t *w_gate, const moe_bf16_t *w_up, moe_bf16_t *hp,
                                      int32_t *status, moe_stream_t stream);

/*
 * The router projection on more CTAs.  Its ceil(T/128) row tiles can be fewer than the SMs;
 * with a workspace the reduction over d is split into S parts (S chosen from T, d and the SM
 * count; each part at least 256 columns of d), the parts' fp32 partial logits go to the
 * workspace, and a second kernel sums them in a fixed order, adds the bias and routes.  The
 * results equal those of moe_route / moe_route_scores up to fp32 rounding of the logits.
 *   moe_route_workspace_size: bytes needed (0 when the split does not pay: then the calls
 *                             below run the single-pass kernel and ignore ws)
 *   ws: device, 256-byte aligned, at least that size; contents need no initialisation.
 */
MOE_API moe_status_t moe_route_workspace_size(const moe_shape_t *shape, size_t *bytes);
MOE_API moe_status_t moe_route_ws(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *w_router,
                          const float *bias, float *logits, int32_t *topk_ids, float *topk_w, int32_t *status,
                          void *ws, size_t ws_bytes, moe_stream_t stream);
MOE_API moe_status_t moe_route_scores_ws(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *w_router,
                                 const float *bias, float *scores, int32_t *status, void *ws, size_t ws_bytes,
                                 moe_stream_t stream);

/*
 * Expert-choice routing (shape.route_flags = MOE_ROUTE_EXPERT_CHOICE; see
 * moe_shape_t).  Router scores, transposed so that each expert's column is
 * contiguous:
 *   x        [T, d] bf16            w_router [E, d] bf16
 *   bias     [E] fp32 or NULL; added to the logits
 *   scores   [E, T] fp32 out: scores[e * T + t] = exp(l_te - max_e' l_te') /
 *            sum_e' exp(l_te' - max_e' l_te')
 * The projection runs on the tensor cores (bf16 in, fp32 accumulate) with
 * the softmax in its epilogue.  Rejects shapes without the flag.
 */
MOE_API moe_status_t moe_route_scores(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *w_router,
                              const float *bias, float *scores, int32_t *status, moe_stream_t stream);

/*
 * Expert-choice selection and dispatch: each expert keeps its C' = min(C, T)
 * highest-scoring tokens (compared as fp32; equal scores go to the lower
 * token id), and their rows of X are copied into segment e of Xp in
 * ascending token order.
 *   scores      [E, T] fp32 (moe_route_scores)
 *   x           [T, d] bf16
 *   seg_expert  [E] int32 out: e;  seg_offsets [E + 1] int32 out: e * C'
 *   src         [E * C'] int32 out: token of each row
 *   row_w       [E * C'] fp32 out: the score S[src, e] of each row
 *   emap        [T, E] int32 out: row of (t, e), or -1 if e did not keep t
 *   xp          [E * C', d] bf16 out
 * Scores must be finite.  Two launches (selection: one CTA per expert;
 * row copy).  Rejects shapes without the flag.
 */
MOE_API moe_status_t moe_expert_choose(const moe_shape_t *shape, const float *scores, const moe_bf16_t *x,
                               int32_t *seg_expert, int32_t *seg_offsets, int32_t *src, float *row_w,
                               int32_t *emap, moe_bf16_t *xp, moe_stream_t stream);

/*
 * Expert-choice combine: out[t] = base[t] + sum over e ascending with
 * emap[t, e] >= 0 of row_w[r] * yp[r], r = emap[t, e], accumulated in fp32.
 *   yp [E * C', d] fp32;  emap [T, E] int32;  row_w [E * C'] fp32
 *   base [T, d] fp32 or NULL;  out [T, d] in shape->out_dtype (an fp32 out may
 *   alias base; a bf16 out may not)
 * Rows outside [0, E * C') contribute nothing.  Rejects shapes without the flag.
 */
MOE_API moe_status_t moe_combine_expert_choice(const moe_shape_t *shape, const float *yp, const int32_t *emap,
                                       const float *row_w, const float *base, void *out,
                                       moe_stream_t stream);

/*
 * Dispatch with overflow re-routing (shape.route_flags has MOE_ROUTE_REROUTE):
 * as moe_dispatch (plan_ready = 0), plus
 *   logits [T, E] fp32: the router logits that chose topk_ids (moe_route's
 *          logits output); they order each token's further candidates
 * counts receives the plain histogram of topk_ids; seg_offsets the rows each
 * expert ends with (at most C).  ws: moe_workspace_size's dispatch_bytes for
 * this shape (device, 256-byte aligned; no initialisation needed).  Launches:
 * each token's candidate order, the rounds (a cooperative grid of up to one CTA
 * per SM exchanging per-expert counts through a bounded grid barrier; a wait
 * that runs out sets MOE_DEV_ERR_TIMEOUT in *status) and the row copies.
 */
MOE_API moe_status_t moe_dispatch_reroute(const moe_shape_t *shape, const moe_bf16_t *x, const int32_t *topk_ids,
                                  const float *logits, int32_t *counts, int32_t *seg_expert,
                                  int32_t *seg_offsets, int32_t *seg_first_rank, int32_t *dest, int32_t *src,
                                  moe_bf16_t *xp, int32_t *status, void *ws, size_t ws_bytes,
                                  moe_stream_t stream);

/* Device addresses of the intermediates moe_layer_fwd keeps in its workspace. */
typedef struct {
    int32_t *topk_ids;       /* [T, k] */
    float *topk_w;           /* [T, k] */
    int32_t *counts;         /* [E] */
    int32_t *seg_expert;     /* [n_seg] */
    int32_t *seg_offsets;    /* [n_seg + 1] */
    int32_t *seg_first_rank; /* [n_seg] */
    int32_t *dest;           /* [T * k] */
    int32_t *src;            /* [rows_alloc] */
    moe_bf16_t *xp;          /* [rows_alloc, d] */
    moe_bf16_t *hp;          /* [rows_alloc, F] */
    float *yp;               /* [rows_alloc, d] fp32 */
    void *dispatch_ws;       /* moe_dispatch's own workspace */
    size_t dispatch_ws_bytes;
    float *scores;           /* [E, T] expert-choice scores (NULL without the flag) */
    int32_t *emap;           /* [T, E] expert-choice row map (NULL without the flag) */
    float *row_w;            /* [rows_alloc] expert-choice row weights (NULL without the flag) */
    float *logits;           /* [T, E] router logits (MOE_ROUTE_REROUTE only, else NULL) */
} moe_layer_views_t;

/*
 * Routing statistics of one dispatch (top-k modes), for monitoring the routing
 * distribution ("Expert를 똑같이 나눴는데도 GPU가 대기하는 이유", section "라우팅 분포와
 * 학습 안정성": per-expert token counts, dropped tokens) and the balanced plan
 * (MoonEP page, "실제 실험 결과": busiest group against the mean, migrated tokens,
 * replica slots in use).  One small kernel; nothing returns to the host.
 *   counts [E]: the raw per-expert counts the dispatch wrote (nullable: the
 *   values that need them are then -1); seg_expert [n_seg], seg_offsets
 *   [n_seg + 1]: its segment tables (e.g. the moe_layer_views of a layer run).
 *   stats [MOE_STAT_COUNT] int32 out (device):
 *     MOE_STAT_PAIRS             T * k
 *     MOE_STAT_ROWS              rows placed (seg_offsets[n_seg])
 *     MOE_STAT_DROPPED           pairs not placed (capacity, re-routing with no room)
 *     MOE_STAT_MAX_EXPERT_LOAD   max over experts of counts[e]
 *     MOE_STAT_ACTIVE_EXPERTS    experts with counts[e] > 0
 *     MOE_STAT_MAX_SEGMENT_ROWS  rows of the longest segment (the longest GEMM)
 *     MOE_STAT_MAX_GROUP_LOAD    with a plan: max over groups of the counts of its home
 *                                experts (before the plan; the mean is T*k/R); else as
 *                                MOE_STAT_MAX_EXPERT_LOAD
 *     MOE_STAT_MAX_GROUP_ROWS    with a plan: max over groups of the rows it computes
 *                                (S*k for a feasible plan); else as MOE_STAT_MAX_SEGMENT_ROWS
 *     MOE_STAT_MIGRATED_ROWS     rows in replica segments (computed outside the home group)
 *     MOE_STAT_REPLICAS_USED     replica segments holding rows
 * MOE_ERR_INVALID_ARG for expert-choice shapes and null tables.
 */
#define MOE_STAT_PAIRS 0
#define MOE_STAT_ROWS 1
#define MOE_STAT_DROPPED 2
#define MOE_STAT_MAX_EXPERT_LOAD 3
#define MOE_STAT_ACTIVE_EXPERTS 4
#define MOE_STAT_MAX_SEGMENT_ROWS 5
#define MOE_STAT_MAX_GROUP_LOAD 6
#define MOE_STAT_MAX_GROUP_ROWS 7
#define MOE_STAT_MIGRATED_ROWS 8
#define MOE_STAT_REPLICAS_USED 9
#define MOE_STAT_COUNT 10
MOE_API moe_status_t moe_routing_stats(const moe_shape_t *shape, const int32_t *counts,
                               const int32_t *seg_expert, const int32_t *seg_offsets,
                               int32_t *stats, moe_stream_t stream);

/*
 * Expert parallelism across R ranks, one GPU each ("가장 바쁜 랭크가 속도를
 * 정합니다: MoonEP의 계획 코드를 직접 돌려봤습니다", sections "이 기술은 무엇인가"
 * and "설치 및 통합"; "5.3 Expert Parallelism", section "2. 디스패처 엔지니어링").
 * The balanced plan's R groups are R ranks: rank g owns the E/R experts homed
 * in group g (experts [g*E/R, (g+1)*E/R)) plus B replica weight slots, holds
 * S = T/R tokens, and computes exactly S*k rows.  A step on rank g:
 *   route its S tokens (moe_route / moe_route_ws with T = S) and count them
 *   (moe_histogram); gather every rank's counts into counts_all [R, E] (a
 *   collective of the caller's); moe_ep_plan; moe_ep_prefetch_weights;
 *   moe_ep_dispatch; a barrier; moe_ep_expert_ffn; a barrier; moe_ep_combine.
 * The layout equals the single-GPU balanced plan over the R*S tokens in rank
 * order: rank g's dispatched rows are rows [g*S*k, (g+1)*S*k) of that layout.
 * Peer buffers are passed as HOST arrays of device pointers, one per rank
 * (entry r = rank r's buffer, a peer-mapped address on a multi-GPU node); the
 * kernels touch them with plain loads and stores only and never wait for
 * another rank, so the barriers are the caller's stream-ordered collectives.
 * With fewer GPUs than ranks, one call can serve several source ranks (n_src >
 * 1) whose buffers all live on the calling GPU.
 *
 * Shape of every moe_ep_* call: T = R*S (all ranks' tokens), n_groups = R
 * (1 <= R <= MOE_EP_MAX_RANKS), replica_slots = B, capacity = 0, no expert
 * choice or re-routing; S*k <= 2^20.  Per rank:
 *   weights   w_gate, w_up [E/R + B, F, d], w_down [E/R + B, d, F]: slot i < E/R
 *             holds home expert g*E/R + i, slot E/R + j replica slot j
 *   rows      xp [S*k, d] bf16, src [S*k] int32, hp [S*k, F] bf16, yp [S*k, d] fp32
 *   tables    seg_expert / seg_slot [E/R + B], seg_offsets [E/R + B + 1]
 */
#define MOE_EP_MAX_RANKS 16

/*
 * Per-rank sizes (host only; outputs nullable): *xp_bytes = S*k*d*2, the
 * dispatch buffer a rank receives into; *replica_weight_bytes = B*3*d*F*2, the
 * replica weight slots (the MoonEP page's "실제 실험 결과" memory table: 0.44 GiB
 * and 0.33 GiB at S = 4096, d = 7168, k = 8, F = 2048, B = 4);
 * *n_local_segments = E/R + B.
 */
MOE_API moe_status_t moe_ep_sizes(const moe_shape_t *shape, size_t *xp_bytes, size_t *replica_weight_bytes,
                          int32_t *n_local_segments);

/*
 * The balanced plan over all ranks from counts_all [R, E] (row r = rank r's
 * raw counts), identical on every rank, reduced to rank `rank`'s segments:
 *   counts      [E] out (nullable): total pairs of each expert
 *   seg_expert  [E/R + B] out: global expert of each local segment (-1 unused)
 *   seg_slot    [E/R + B] out: local weight slot of each segment (its index),
 *               -1 for a segment without rows
 *   seg_offsets [E/R + B + 1] out: rows of each segment inside the rank's S*k
 * An infeasible plan sets MOE_DEV_ERR_PLAN and writes empty segments.  One CTA.
 */
MOE_API moe_status_t moe_ep_plan(const moe_shape_t *shape, int32_t rank, const int32_t *counts_all,
                         int32_t *counts, int32_t *seg_expert, int32_t *seg_slot, int32_t *seg_offsets,
                         int32_t *status, moe_stream_t stream);

/*
 * Replica weights (MoonEP page, "설치 및 통합": prefetch_weight fills the
 * slots [E, E+B) from the plan).  For each replica slot j of rank `rank` whose
 * segment has rows, the gate, up and down matrices of its expert e are copied
 * from slot e - h*E/R of e's home rank h into slot E/R + j of this rank.
 *   seg_expert, seg_offsets: this rank's tables (moe_ep_plan)
 *   w_gate, w_up, w_down: host arrays of R device pointers, each rank's
 *   [E/R + B, ...] weight tensor (this rank's entry is written).
 */
MOE_API moe_status_t moe_ep_prefetch_weights(const moe_shape_t *shape, int32_t rank, const int32_t *seg_expert,
                                     const int32_t *seg_offsets, moe_bf16_t *const *w_gate,
                                     moe_bf16_t *const *w_up, moe_bf16_t *const *w_down,
                                     moe_stream_t stream);

/*
 * Dispatch of the source ranks [src_rank, src_rank + n_src) (MoonEP page,
 * "이 기술은 무엇인가": each row is written straight to its final slot on the
 * receiving rank).  Pair (t, j) of rank r has global index q = r*S*k + t*k + j;
 * its stable rank among all pairs of its expert (q order) selects the plan's
 * segment that holds it, hence its owner g and row; then
 *   dest_r[t*k + j] = g*S*k + row,  src_g[row] = q,  xp_g[row] = x_r[t].
 *   x, topk_ids, dest: host arrays of n_src device pointers ([S, d] bf16,
 *                      [S, k] int32, [S*k] int32 out)
 *   counts_all: [R, E] as for moe_ep_plan
 *   xp, src: host arrays of R device pointers (each owner's receive buffers)
 * One launch; every CTA recomputes the plan from counts_all.  The kernel ends
 * with a system-scope fence, so a collective that follows it on the stream
 * also follows its stores to other GPUs.
 */
MOE_API moe_status_t moe_ep_dispatch(const moe_shape_t *shape, int32_t src_rank, int32_t n_src,
                             const moe_bf16_t *const *x, const int32_t *const *topk_ids,
                             const int32_t *counts_all, int32_t *const *dest, moe_bf16_t *const *xp,
                             int32_t *const *src, int32_t *status, moe_stream_t stream);

/*
 * One rank's grouped GEMMs (moe_expert_gate_up then moe_expert_down) on its S*k
 * rows, its E/R + B segments (seg_slot as the segment's weight slot) and its own
 * weight slots.  All pointers are this rank's device memory.
 */
MOE_API moe_status_t moe_ep_expert_ffn(const moe_shape_t *shape, const moe_bf16_t *xp, const int32_t *seg_slot,
                               const int32_t *seg_offsets, const moe_bf16_t *w_gate, const moe_bf16_t *w_up,
                               const moe_bf16_t *w_down, moe_bf16_t *hp, float *yp, int32_t *status,
                               moe_stream_t stream);

/*
 * Combine of the source ranks [src_rank, src_rank + n_src): out_r[t] = sum over
 * j of w_r[t, j] * yp_g[row], with (g, row) from dest_r[t*k + j] = g*S*k + row
 * (fp32, ascending j), stored in shape->out_dtype.
 *   yp: host array of R device pointers (each owner's [S*k, d] fp32)
 *   dest, topk_w, out: host arrays of n_src device pointers
 */
MOE_API moe_status_t moe_ep_combine(const moe_shape_t *shape, int32_t src_rank, int32_t n_src,
                            const float *const *yp, const int32_t *const *dest, const float *const *topk_w,
                            void *const *out, moe_stream_t stream);

/*
 * Routing results of a layer call, copied into the caller's own device buffers
 * (every pointer nullable: NULL = not wanted).
 */
typedef struct {
    int32_t *topk_ids;    /* [T, k] */
    float *topk_w;        /* [T, k] */
    int32_t *counts;      /* [E] raw per-expert counts */
    int32_t *seg_offsets; /* [n_seg + 1] */
    int32_t *dest;        /* [T * k] row of each pair, -1 = dropped */
    int32_t *stats;       /* [MOE_STAT_COUNT], as moe_routing_stats writes them */
} moe_aux_t;

/*
 * moe_layer_fwd, then the requested routing results copied out of the workspace
 * (device-to-device copies on `stream`) and, with aux->stats, moe_routing_stats.
 * aux may be NULL (then identical to moe_layer_fwd).  Expert-choice shapes have
 * no per-pair results: requesting topk_ids, topk_w, dest, counts or stats for them
 * is MOE_ERR_INVALID_ARG (seg_offsets is allowed).
 */
MOE_API moe_status_t moe_layer_fwd_aux(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *w_router,
                               const float *bias, const moe_bf16_t *w_gate, const moe_bf16_t *w_up,
                               const moe_bf16_t *w_down, void *out, const moe_aux_t *aux, int32_t *status,
                               void *ws, size_t ws_bytes, moe_stream_t stream);

/* Fill *views with the addresses inside a layer workspace `ws`. Host only. */
MOE_API moe_status_t moe_layer_views(const moe_shape_t *shape, void *ws, moe_layer_views_t *views);

#ifdef __cplusplus
}
#endif

#endif /* MOE_ROUTING_H */
