/*
 * moe_rt.h — C ABI of libmoert.so: MoE token dispatch and combine on one
 * B200 (sm_100a), expert-parallel ranks simulated as contiguous partitions
 * of the send buffer.
 *
 * Sources (page titles; sections named inline below):
 *   [Megatron MORI]  "Add MORI as a Token Dispatcher" (ROCm/Megatron-LM PR #135)
 *   [UltraEP]        "Integrate UltraEP Runtime for MoE EP Load Balancing" (InternLM/xtuner PR #2050)
 *   [Megatron MoE]   "Megatron MoE 实现" (MoELayer.forward: route, dispatch, experts, combine)
 *   [mscclpp HT]     mscclpp python/ page, high-throughput dispatch/combine summary
 *   [DeepSpeed EP]   deepspeed/moe/ep_tp_dispatch.py (route-full / partition-dispatch helpers)
 *
 * Conventions shared by every call
 * --------------------------------
 * Memory.  Every pointer argument is DEVICE memory owned by the caller, except
 *   `problem` and `layout`, which are host structs read during the call only.
 *   The library allocates nothing and keeps no state between calls. Tensors
 *   are dense row-major; bf16 tensors are passed as uint16_t bit patterns.
 *   hidden / send / expert-output / gradient buffers must be 16-byte aligned.
 * Streams.  `stream` is a cudaStream_t (NULL = the legacy default stream).
 *   Every call only enqueues work on it: no host synchronisation, no host
 *   read of device data ([Megatron MORI]: sync-free counts and padded buffers).
 * Sizes.  Buffers have fixed upper-bound sizes ([Megatron MORI]: work on the
 *   full [max_tokens, ...] padded buffers and mask the tail). rows_max =
 *   E*ceil(capacity/T) when capacity > 0, else (N*k + E*(T-1))/T + E*(row_align - 1)
 *   (N*k without alignment or TP folding, T = tp_size). N*k and rows_max must be < 2^31.
 * Returns.  MOE_OK or a negative host-detected error; on MOE_ERR_INVALID,
 *   MOE_ERR_UNSUPPORTED or MOE_ERR_SCRATCH_LIMIT nothing is enqueued (every
 *   check comes before the first launch). MOE_ERR_CUDA means a launch failed;
 *   a call that enqueues two kernels may then have enqueued the first.
 *   Device-detected problems are OR-ed into *layout->status as MOE_DEV_* bits;
 *   read them when convenient (no call waits for them).
 * Concurrency.  A layout / workspace pair backs one dispatch at a time
 *   ([Megatron MORI] review thread: one staging region per op means two calls
 *   of the same op must not be in flight together). Reusing the layout for
 *   combine and both backward calls is intended ([mscclpp HT]: cached
 *   dispatch via previous_handle).
 */
#ifndef MOE_RT_H
#define MOE_RT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_RT_ABI_VERSION 6

/* Every entry point is exported; everything else in the library is hidden. */
#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

/* Host-detected return codes (nothing was enqueued). */
#define MOE_OK 0
#define MOE_ERR_INVALID (-1)     /* bad size, NULL required pointer, misaligned buffer, inconsistent problem */
#define MOE_ERR_UNSUPPORTED (-2) /* valid but beyond the kernels' limits (see each call) */
#define MOE_ERR_CUDA (-3)        /* a CUDA runtime call or launch failed */
#define MOE_ERR_SCRATCH_LIMIT (-4) /* moe_dispatch_layout_noalloc: E_log above MOE_NOALLOC_MAX_E_LOG */

/* Device-detected status bits, OR-ed into *layout->status. */
#define MOE_DEV_EXPERT_RANGE 0x1u /* a topk id outside [-1, E_log): the entry was skipped as if -1 */
#define MOE_DEV_TIMEOUT 0x2u      /* a bounded device wait ran out; outputs of that call are invalid */
#define MOE_DEV_ROW_RANGE 0x4u    /* a dest_row outside [-1, rows_max): that row was skipped */

/* moe_problem_t.flags */
#define MOE_FLAG_NONE 0u
/* Test hook: in the dispatch layout the first block of the scan never publishes
 * its counts, so the next block's look-back waits for a word that never comes,
 * with a ~10 ms limit; the timeout path runs without hanging anything. */
#define MOE_FLAG_TEST_WAIT_TIMEOUT 0x80000000u
/* moe_dispatch only: stage each token row through shared memory with bulk (TMA)
 * copies, one bulk load per row and one bulk store per kept destination row,
 * instead of 16-byte vector loads and stores. Same results bit for bit; on B200
 * slower for this one-read / k-write scatter, so it is not the default. */
#define MOE_FLAG_DISPATCH_BULK_COPY 0x1u

/* The problem statement ([DeepSpeed EP] RoutedAssignmentPayload; it follows the
 * pages' shapes: hidden [N,H] bf16, topk ids [N,k] int32, probs [N,k] fp32). */
typedef struct {
    int64_t N;            /* tokens (>= 0) */
    int32_t H;            /* hidden size, a positive multiple of 8 (16-byte rows) */
    int32_t k;            /* top-k, 1..32 */
    int32_t E_log;        /* logical experts (router width), 1..2048, divisible by R */
    int32_t num_replicas; /* UltraEP replica slots in total (0 = no reroute), divisible by R, <= E_log */
    int32_t R;            /* simulated EP ranks, >= 1 */
    int32_t capacity;     /* per-expert capacity C (0 = unlimited) */
    uint32_t flags;       /* MOE_FLAG_* */
    int32_t row_align;    /* 0 or 1 = none; A > 1: each expert's rows are padded up to a multiple of A
                             ([Megatron MORI]: router padding for FP8 grouped GEMMs). With a capacity,
                             ceil(C / tp_size) must be a multiple of A. */
    int32_t tp_size;      /* TP folding ([DeepSpeed EP] partition_assignments): T peers share the
                             assignments; 0 or 1 = none, at most MOE_MAX_TP */
    int32_t tp_rank;      /* this peer, 0 <= tp_rank < T. The layout then keeps only the active
                             assignments whose stable per-expert ordinal o satisfies o % T == tp_rank,
                             at local ordinal o / T; capacity drops stay global. */
} moe_problem_t;

#define MOE_MAX_TP 8

/*
 * Outputs of moe_dispatch_layout, all device buffers of the sizes shown
 * (E = E_log + num_replicas physical experts, E_loc = E / R per rank).
 * Physical numbering: rank r owns experts [r*E_loc, (r+1)*E_loc); with replicas
 * the first E_log/R of them are the masters of logical experts
 * r*E_log/R + i, the rest are replica slots.
 */
typedef struct {
    /* per assignment a = t*k + j, [N*k] */
    int32_t *phys_idx;  /* physical expert, -1 for a -1 (or skipped) id */
    int32_t *ordinal;   /* stable rank among earlier assignments to the same physical expert, -1 as above */
    int32_t *dest_row;  /* send-buffer row, -1 if the id is -1 or the assignment was dropped */
    uint8_t *drop_mask; /* 1 = over capacity */
    /* per logical expert, [E_log] */
    int32_t *counts_logical; /* router histogram before reroute */
    int32_t *placement;      /* physical replica slot of a hot expert, else -1 */
    /* per physical expert */
    int32_t *counts_raw;        /* [E] assignments before capacity */
    int32_t *tokens_per_expert; /* [E] rows filled: min(counts_raw, C), or counts_raw when C = 0 */
    int32_t *expert_offsets;    /* [E+1] first row of each expert (e*C when C > 0); an expert owns
                                   C rows, or tokens_per_expert rounded up to a multiple of row_align */
    /* per rank */
    int32_t *input_splits;  /* [R] rows destined to rank r (pad rows included when C > 0) */
    int32_t *output_splits; /* [R] equal to input_splits on one GPU */
    int32_t *rank_offsets;  /* [R+1] first row of each rank */
    /* scalars */
    int32_t *counters; /* [8] assignments_total (valid ids), kept (rows in this buffer; [DeepSpeed EP]
                          assignments_local), dropped, padded, split_sum_in, split_sum_out, num_rows, error */
    int32_t *num_rows; /* [1] expert_offsets[E] */
    uint32_t *status;  /* [1] MOE_DEV_* bits; the caller zeroes it, calls only OR into it */
    /* per send-buffer row, [rows_max] */
    int32_t *row_token;        /* source token, -1 in pad / tail rows */
    int32_t *row_slot;         /* top-k slot j, -1 in pad / tail rows */
    int32_t *row_local_expert; /* expert id local to the row's rank, -1 in pad / tail rows */
    float *row_prob;           /* receiver-side prob p[t,j], 0 in pad / tail rows */
    uint8_t *pad_mask;         /* 1 = the row holds no assignment (capacity or alignment pad, or tail) */
    /* optional DeepEP-contract view, [R*N*k] or NULL */
    int32_t *local_topk; /* [r][t][j]: local id if (t,j) is kept on rank r, else -1 */
} moe_layout_t;

/* ABI version of the loaded library (MOE_RT_ABI_VERSION it was built with). */
MOE_API int moe_abi_version(void);

/* Static text for a return code or a single MOE_DEV_* bit. Never NULL. */
MOE_API const char *moe_status_string(int code);

/*
 * Number of send-buffer rows (the first dimension of send / expert_out /
 * row_* buffers), see "Sizes" above. Host only.
 * Returns a negative MOE_ERR_* if the problem is invalid.
 */
MOE_API int64_t moe_rows_max(const moe_problem_t *problem);

/*
 * Bytes of device scratch moe_dispatch_layout needs (a ticket word and the
 * per-block look-back words of the scan). Host only. The scratch must be
 * zero-filled once before its first use; afterwards every call leaves it ready
 * for the next one, also a call that reported MOE_DEV_TIMEOUT (each look-back
 * word carries the epoch of the launch that wrote it).
 * Returns MOE_OK and sets *bytes, or a negative MOE_ERR_*.
 */
MOE_API int moe_layout_workspace_bytes(const moe_problem_t *problem, size_t *bytes);

/*
 * Router: softmax over E fp32 logits and top-k
 * ([Megatron MoE] MoELayer.router_and_preprocess; [Megatron MORI] router.py:
 * padding tokens do not take part in routing).
 *   logits      [N, E] fp32, device
 *   token_mask  [N] uint8 or NULL; a token with mask != 0 gets ids -1, probs 0
 *   topk_idx    [N, k] int32 out: the k largest logits, descending; equal
 *               logits to the lower expert id
 *   topk_probs  [N, k] fp32 out: exp(l - max) / sum_e exp(l - max) over all E
 *               (no renormalisation over the k chosen), CUDA expf
 * Limits: 1 <= k <= min(E, 32), E <= 1024 (MOE_ERR_UNSUPPORTED beyond).
 */
MOE_API int moe_route_topk(const float *logits, const uint8_t *token_mask, int64_t N, int32_t E, int32_t k,
                   int32_t *topk_idx, float *topk_probs, void *stream);

/*
 * Dispatch layout: optional UltraEP reroute, histogram, stable ordinals,
 * capacity drop / pad, exclusive scan, rank splits, row maps and the local
 * view, in two launches: a count pass whose blocks, ordered by an atomic
 * ticket, scan the per-expert counts with a decoupled look-back (each block
 * waits only for blocks that started before it, so any number of layouts may
 * run at once on any streams), and a fill pass for the row maps.
 *   [UltraEP]: hot-expert replicas from the layer's actual load, tokens
 *     rerouted logical -> physical; router semantics stay logical.
 *   [DeepSpeed EP] assignment_ordinals_by_expert: stable ordinals per expert;
 *     RoutedAssignmentPayload capacity_slots / drop_mask / pad_mask;
 *     _recompute_input_splits / partition_assignments: splits and counters.
 *   [Megatron MORI]: local ids with -1 sentinels, receiver-side probs, tails
 *     masked 0 / -1 / 0, fixed-size scatter instead of bincount (no host sync).
 * Readings where the pages are silent: ordinals follow the flattened [N,k]
 * order; drops are first-come; hot experts = the num_replicas largest
 * logical counts (ties to the lower id), placed greedily on the least-loaded
 * other rank with a free replica slot (own rank only if no other is free);
 * a hot expert's logical ordinal o goes to the master if o is even, to the
 * replica if odd (physical ordinal o/2).
 *   topk_idx    [N, k] int32, ids in [-1, E_log); others are skipped (MOE_DEV_EXPERT_RANGE)
 *   topk_probs  [N, k] fp32 or NULL (row_prob then 0)
 *   layout      every pointer except local_topk must be non-NULL
 *   workspace   moe_layout_workspace_bytes() bytes, zero-filled before first use
 * Limits: E_log <= 2048, k <= 32, R <= 64 when num_replicas > 0.
 * The only device-side wait (a block for its predecessors' look-back words) is
 * bounded by ~1 s; if it runs out, MOE_DEV_TIMEOUT is set and that call's
 * outputs are invalid (destination rows stay inside [-1, rows_max)).
 */
MOE_API int moe_dispatch_layout(const moe_problem_t *problem, const int32_t *topk_idx, const float *topk_probs,
                        const moe_layout_t *layout, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Dispatch layout and permute in one call ([Megatron MORI]: the permute is
 * fused into the dispatch node; [Megatron MoE] dispatch_postprocess: permuted
 * tokens and tokens_per_expert). Computes exactly the outputs of
 * moe_dispatch_layout followed by moe_permute (layout and send buffer, bit for
 * bit) in two launches: the layout's count pass, then one kernel that finishes
 * the layout and copies every kept token row to its send-buffer rows, zeroing
 * pad and tail rows. Each token row is read once and can be read while the
 * count pass runs; nothing passes through an intermediate row map in memory.
 *   topk_idx, topk_probs, layout, workspace  as for moe_dispatch_layout
 *   hidden [N, H] bf16; send [rows_max, H] bf16 (16-byte aligned, no overlap)
 * Same limits as moe_dispatch_layout.
 */
MOE_API int moe_dispatch(const moe_problem_t *problem, const int32_t *topk_idx, const float *topk_probs,
                         const moe_layout_t *layout, void *workspace, size_t workspace_bytes, const uint16_t *hidden,
                         uint16_t *send, void *stream);

/*
 * Dispatch layout for callers that cannot allocate device memory. The pages
 * have no counterpart of this entry point; it exists for the library's users.
 *
 * Some callers have no way to obtain device scratch: a C or Fortran host
 * program without an allocator of its own, a plugin running inside a host
 * application that owns every allocation, or a hot loop that must not touch
 * cudaMalloc (it can synchronise the device and fail under memory pressure).
 * This call computes exactly what moe_dispatch_layout computes, with the same
 * arguments except the workspace: its scratch is a fixed array inside the
 * library, MOE_NOALLOC_SCRATCH_BYTES bytes that every GPU which loads the
 * library keeps until the process exits. It calls no allocator.
 *
 * Limits and rules:
 *  - E_log <= MOE_NOALLOC_MAX_E_LOG, else MOE_ERR_SCRATCH_LIMIT and nothing is enqueued;
 *    every other argument rule of moe_dispatch_layout applies.
 *  - The current device must be the device that owns `stream` (the array used is
 *    that device's); a stream of another device gives MOE_ERR_INVALID.
 *  - The first call on a device looks up the array's device address (once per
 *    device, with that device current). Make that first call before any stream
 *    capture begins.
 *  - All calls share the one array and it keeps what the last call left there.
 *    Nothing in it has to start at zero after the first use: the scan's words
 *    carry the epoch of the launch that wrote them and the ticket word is rolled
 *    over by every launch, so a call that ran out of time (MOE_DEV_TIMEOUT) does
 *    not affect the next and the call enqueues nothing but its two kernels.
 *    Calls whose executions overlap on the GPU (for example on two streams)
 *    race on the array and give wrong results: order them on one stream.
 */
#define MOE_NOALLOC_MAX_E_LOG 512
#define MOE_NOALLOC_SCRATCH_BYTES (256 + 128 * MOE_NOALLOC_MAX_E_LOG * 8)
MOE_API int moe_dispatch_layout_noalloc(const moe_problem_t *problem, const int32_t *topk_idx,
                                        const float *topk_probs, const moe_layout_t *layout, void *stream);

/*
 * Permute ([Megatron MoE] dispatch_postprocess; [Megatron MORI] permute fused
 * into the dispatch node): send[dest_row[t,j]] = hidden[t] for every kept
 * (t,j); rows with pad_mask = 1 are zero-filled. Byte copy, bit-exact.
 * Reads layout->dest_row and layout->pad_mask.
 *   hidden [N, H] bf16; send [rows_max, H] bf16 (must not overlap hidden)
 */
MOE_API int moe_permute(const moe_problem_t *problem, const moe_layout_t *layout, const uint16_t *hidden, uint16_t *send,
                void *stream);

/*
 * Combine ([DeepSpeed EP] restore_combined: weighted rows added back one
 * top-k slot at a time in ascending slot order; [Megatron MoE] combine):
 *   out[t,h] = bf16_rn( fp32 chain acc = fmaf(p[t,j], y[dest_row[t,j], h], acc)
 *                       over ascending j with dest_row >= 0, from acc = +0 )
 * Deterministic, no atomics, bit-exact with the CPU definition, except for the
 * bit pattern of a NaN: a NaN element (from a NaN input or an inf - inf sum) is
 * a NaN exactly where the definition's is, but it is the canonical bf16 NaN that
 * the hardware conversion produces, not the sign and payload the CPU definition
 * keeps. Infinities and signed zeros follow IEEE fp32 and are bit-exact.
 *   expert_out [rows_max, H] bf16; topk_probs [N, k] fp32 or NULL (unit
 *   weights); out [N, H] bf16. Reads layout->dest_row.
 */
MOE_API int moe_combine(const moe_problem_t *problem, const moe_layout_t *layout, const uint16_t *expert_out,
                const float *topk_probs, uint16_t *out, void *stream);

/*
 * Restore after TP folding ([DeepSpeed EP] restore_combined: the peers' weighted
 * rows are gathered and added back per token one top-k slot at a time in
 * ascending slot order). On one GPU the gather is the set of peer buffers:
 * peer q's layout (from moe_dispatch_layout with tp_rank = q) and its expert
 * output. out[t,h] = bf16_rn( fp32 fmaf chain over ascending j of
 * p[t,j] * y_q[dest_row_q[t,j], h], q the one peer with dest_row_q[t,j] >= 0 ),
 * which equals moe_combine of the unfolded layout bit for bit.
 *   problem          the per-peer problem; tp_size = T peers (tp_rank is ignored)
 *   peer_layouts     host array of T layouts; reads dest_row and status of each
 *   peer_expert_out  host array of T device pointers, peer q's [rows_max, H] bf16
 *   topk_probs       [N, k] fp32 or NULL (unit weights); out [N, H] bf16
 * Device status bits go to peer 0's status word.
 */
MOE_API int moe_restore_combined(const moe_problem_t *problem, const moe_layout_t *peer_layouts,
                                 const uint16_t *const *peer_expert_out, const float *topk_probs, uint16_t *out,
                                 void *stream);

/*
 * DeepEP-style token-dedup view ([Megatron MORI]: the MORI dispatcher follows
 * the DeepEP contract: each token goes once to each rank that owns one of its
 * kept slots; the receiver gets local top-k ids with -1 sentinels and
 * receiver-side weights, and _indices_to_multihot turns them into a
 * [tokens, local experts] routing map with probs). One receive row per
 * (token, rank) pair, rank-major and token-ascending within a rank;
 * recv_max = N * min(k, R) rows, the rows past num_recv are tail rows
 * (token -1, ids -1, weights / map / probs 0, pad 1). R <= MOE_MAX_DEDUP_RANKS.
 * When E_loc is a multiple of 4, recv_probs must be 16-byte and
 * recv_routing_map 4-byte aligned (their rows are written four entries at a time).
 */
#define MOE_MAX_DEDUP_RANKS 32

typedef struct {
    int32_t *num_tokens_per_rank; /* [R] tokens each rank receives */
    int32_t *recv_rank_offsets;   /* [R+1] first receive row of each rank */
    int32_t *num_recv;            /* [1] recv_rank_offsets[R] */
    uint8_t *is_token_in_rank;    /* [N, R] */
    int32_t *token_rank_row;      /* [N, R] receive row of (t, r), -1 if t is not sent to r */
    int32_t *recv_src_token;      /* [recv_max] source token, -1 in the tail */
    int32_t *recv_topk_idx;       /* [recv_max, k] rank-local expert id of slot j, -1 if not on this rank */
    float *recv_topk_weights;     /* [recv_max, k] receiver-side prob, 0 where the id is -1 */
    uint8_t *recv_routing_map;    /* [recv_max, E_loc] multihot over the rank's experts */
    float *recv_probs;            /* [recv_max, E_loc] the prob at each set bit, else 0 */
    uint8_t *recv_pad_mask;       /* [recv_max] 1 in the tail */
    uint32_t *status;             /* [1] MOE_DEV_* bits, OR-ed */
} moe_dedup_t;

/* recv_max = N * min(k, R), or a negative MOE_ERR_* for an invalid problem. Host only. */
MOE_API int64_t moe_dedup_rows_max(const moe_problem_t *problem);

/* Scratch bytes of moe_dedup_layout (zero-filled once before first use, as for the layout;
 * it then stays ready for every later call). Host only. */
MOE_API int moe_dedup_workspace_bytes(const moe_problem_t *problem, size_t *bytes);

/*
 * Build the dedup view from a dispatch layout (reads layout->phys_idx and
 * layout->dest_row: a slot counts where dest_row >= 0): a count pass whose
 * blocks, in atomic-ticket order, rank the (token, rank) pairs with a decoupled
 * look-back over their per-rank counts (no block waits for one that started
 * after it), then a fill pass writes the receive rows and their data.
 * topk_probs [N, k] fp32 or NULL (weights 0). Limits: R <= MOE_MAX_DEDUP_RANKS,
 * N <= 262144.
 */
MOE_API int moe_dedup_layout(const moe_problem_t *problem, const moe_layout_t *layout, const float *topk_probs,
                             const moe_dedup_t *dedup, void *workspace, size_t workspace_bytes, void *stream);

/* Dispatch each token once per receiving rank: recv_x[token_rank_row[t,r]] = hidden[t]; tail rows zero.
 *   hidden [N, H] bf16; recv_x [recv_max, H] bf16 */
MOE_API int moe_dedup_dispatch(const moe_problem_t *problem, const moe_dedup_t *dedup, const uint16_t *hidden,
                               uint16_t *recv_x, void *stream);

/*
 * Receiver side of the DeepEP-style combine: for receive row w of token t on
 * rank r, partial[w] = bf16_rn( fp32 fmaf chain over ascending j of
 * p[t,j] * y[dest_row[t,j]] for the kept slots whose row lies in rank r's range
 * [rank_offsets[r], rank_offsets[r+1]) of the layout ); tail rows 0.
 * Reads dedup->token_rank_row and dedup->num_recv (of moe_dedup_layout on the
 * same layout); every kept slot row is read once per token.
 *   expert_out [rows_max, H] bf16 (the layout's send-buffer order);
 *   topk_probs [N, k] fp32 or NULL (unit weights); partial [recv_max, H] bf16
 */
MOE_API int moe_dedup_combine_local(const moe_problem_t *problem, const moe_layout_t *layout,
                                    const moe_dedup_t *dedup, const uint16_t *expert_out, const float *topk_probs,
                                    uint16_t *partial, void *stream);

/* Sender side: out[t] = bf16_rn( fp32 sum over ascending r of partial[token_rank_row[t,r]] ).
 *   partial [recv_max, H] bf16; out [N, H] bf16 */
MOE_API int moe_dedup_combine(const moe_problem_t *problem, const moe_dedup_t *dedup, const uint16_t *partial,
                              uint16_t *out, void *stream);

/*
 * Expert-parallel exchange between R ranks ([Megatron MoE] all-to-all token
 * dispatcher: every rank's permuted rows go to the rank owning their expert,
 * which orders what it received by local expert; [Megatron MORI]: dispatch
 * writes into the receivers' buffers with the permute fused in, and combine
 * reads the expert outputs back). Every rank runs moe_dispatch_layout on its own
 * tokens with the same problem (tp_size 1); the ranks' receive buffers are given
 * as device arrays of R device pointers, which may point into other GPUs' memory
 * mapped into this process (peer access) or, on one GPU, to separate buffers.
 * Receive layout of rank r: its experts ascending; within an expert the source
 * ranks ascending; each source's rows for that expert in its own send-buffer
 * order, its padding rows (capacity / alignment) included as zeros. Rows past a
 * rank's num_recv are left untouched. The caller orders the steps across ranks:
 * every rank's plan before its dispatch, every dispatch into a buffer before that
 * buffer's experts run, the experts before the combines that read them.
 * Pinned reading: the receive order above is the plainest one the pages' all-to-all
 * plus sort-by-local-expert gives (sources ascending within an expert).
 */
#define MOE_MAX_EP_RANKS 64

/* Rows of one rank's receive buffer: R x (rows one source can send to one rank:
 * E_loc*ceil(C/T) with a capacity, else N*k + E_loc*(row_align-1), at most rows_max).
 * Negative MOE_ERR_* for an invalid problem, MOE_ERR_UNSUPPORTED for tp_size > 1
 * or R > MOE_MAX_EP_RANKS. Host only. */
MOE_API int64_t moe_ep_recv_rows_max(const moe_problem_t *problem);

/*
 * Plan of the exchange for source rank src_rank, one small launch:
 *   offsets_all          [R][E+1] int32: every rank's layout expert_offsets (the
 *                        caller gathers them, e.g. with an all-gather)
 *   base                 [E] int32 out: the receive row on expert q's owner where
 *                        this rank's rows for q start
 *   recv_expert_offsets  [E_loc+1] int32 out: this rank's receive layout by local expert
 *   num_recv             [1] int32 out: rows this rank receives
 *   status               [1] MOE_DEV_* bits (MOE_DEV_ROW_RANGE if a receive buffer
 *                        of moe_ep_recv_rows_max rows cannot hold the exchange)
 * Limit: E <= 4096 physical experts.
 */
MOE_API int moe_ep_plan(const moe_problem_t *problem, const int32_t *offsets_all, int32_t src_rank, int32_t *base,
                        int32_t *recv_expert_offsets, int32_t *num_recv, uint32_t *status, void *stream);

/*
 * The all-gather of expert_offsets that the exchange needs, over peer memory
 * (the only collective of the exchange): writes this rank's layout
 * expert_offsets [E+1] into row src_rank of every rank's [R][E+1] offsets
 * table. peer_offsets_tables: device array of R device pointers (this rank's
 * own table included; the others mapped from their processes, see
 * moe_ipc_open, or other buffers on this GPU). Every rank's tables are
 * complete once every rank's call has run; the caller orders that (for
 * example an interprocess event per rank and a host barrier) before
 * moe_ep_plan reads them.
 */
MOE_API int moe_ep_publish_offsets(const moe_problem_t *problem, const int32_t *expert_offsets, int32_t src_rank,
                                   int32_t *const *peer_offsets_tables, void *stream);

/*
 * Dispatch with the exchange fused in: for every kept slot (t, j) of expert q,
 * peer_recv[q / E_loc][base[q] + dest_row[t,j] - expert_offsets[q]] = hidden[t];
 * this rank's padding rows of every expert are zeroed there.
 *   layout     this rank's layout (phys_idx, dest_row, expert_offsets, tokens_per_expert, status)
 *   base       [E] from moe_ep_plan for this rank
 *   hidden     [N, H] bf16; peer_recv: device array of R device pointers, each a
 *              [moe_ep_recv_rows_max, H] bf16 receive buffer
 */
MOE_API int moe_ep_dispatch(const moe_problem_t *problem, const moe_layout_t *layout, const int32_t *base,
                            const uint16_t *hidden, uint16_t *const *peer_recv, void *stream);

/*
 * Combine with the exchange fused in: out[t] = bf16_rn( fp32 fmaf chain over
 * ascending kept j of p[t,j] * y_r[base[q] + dest_row[t,j] - expert_offsets[q]] ),
 * q = phys_idx[t,j], r = q / E_loc: the same result as moe_combine over this
 * rank's own send-buffer order, bit for bit.
 *   peer_expert_out  device array of R device pointers, rank r's expert output
 *                    in its receive-buffer order
 *   topk_probs [N, k] fp32 or NULL (unit weights); out [N, H] bf16
 */
MOE_API int moe_ep_combine(const moe_problem_t *problem, const moe_layout_t *layout, const int32_t *base,
                           const uint16_t *const *peer_expert_out, const float *topk_probs, uint16_t *out,
                           void *stream);

/*
 * Backward of moe_ep_combine ([Megatron MORI]: combine backward with
 * receiver-side probs): for every kept slot (t, j) of expert q, at row
 * w = base[q] + dest_row[t,j] - expert_offsets[q] of owner r = q / E_loc:
 *   peer_grad_expert_out[r][w] = bf16_rn( fp32(p[t,j] * grad_out[t]) ),
 *   grad_probs[t,j] = fp32 dot( grad_out[t], peer_expert_out[r][w] ) (0 for a dropped slot),
 * with the same arithmetic as moe_combine_backward; this rank's padding rows in the
 * owners' gradient buffers are zeroed. The backward of moe_ep_dispatch is
 * moe_ep_combine with unit weights (topk_probs NULL) over the gradient buffers.
 *   peer_expert_out, peer_grad_expert_out: device arrays of R device pointers
 *   grad_out [N, H] bf16; topk_probs [N, k] fp32; grad_probs [N, k] fp32 out
 */
MOE_API int moe_ep_combine_backward(const moe_problem_t *problem, const moe_layout_t *layout, const int32_t *base,
                                    const uint16_t *grad_out, const uint16_t *const *peer_expert_out,
                                    const float *topk_probs, uint16_t *const *peer_grad_expert_out,
                                    float *grad_probs, void *stream);

/*
 * Sharing buffers between the processes of the exchange (one process per rank).
 * The owner exports a device buffer: the handle of the allocation that holds it
 * (cudaIpcGetMemHandle), the buffer's byte offset inside that allocation (so
 * that buffers carved out of a larger allocation, as caching allocators do,
 * can be shared) and its size. The handle is plain bytes: send it to the
 * other processes by any means. A peer process maps it with moe_ipc_open
 * (cudaIpcOpenMemHandle with lazy peer access: the buffer may be on this GPU or
 * on another one reachable by peer access) and gets the buffer's address and
 * the mapping, which moe_ipc_close releases. A process cannot open its own
 * handles. The owner keeps the buffer allocated until every peer has closed it.
 * Host calls; nothing is enqueued on a stream.
 */
typedef struct {
    unsigned char handle[64]; /* cudaIpcMemHandle_t of the allocation */
    uint64_t offset;          /* the buffer's byte offset inside that allocation */
    uint64_t bytes;           /* the buffer's size */
    int32_t device;           /* the owner's device ordinal (in the owner's process) */
    int32_t reserved;
} moe_ipc_buffer_t;

/* Export [ptr, ptr + bytes) of this process's device memory. MOE_ERR_INVALID if
 * the range is not inside one allocation of this process. */
MOE_API int moe_ipc_export(const void *ptr, size_t bytes, moe_ipc_buffer_t *out);

/* Map a buffer another process exported: *ptr = its address here, *mapping = the
 * mapping to pass to moe_ipc_close. */
MOE_API int moe_ipc_open(const moe_ipc_buffer_t *buf, void **ptr, void **mapping);

/* Release a mapping made by moe_ipc_open. */
MOE_API int moe_ipc_close(void *mapping);

/*
 * Backward of permute ([Megatron MORI]: dispatch backward sums the row
 * gradients back per token with receiver-side indices): combine with unit
 * weights, grad_hidden[t] = bf16_rn( fp32 sum over ascending kept j of
 * grad_send[dest_row[t,j]] ).
 *   grad_send [rows_max, H] bf16; grad_hidden [N, H] bf16
 */
MOE_API int moe_permute_backward(const moe_problem_t *problem, const moe_layout_t *layout, const uint16_t *grad_send,
                         uint16_t *grad_hidden, void *stream);

/*
 * Backward of combine ([Megatron MORI]: combine backward with receiver-side
 * probs):
 *   grad_expert_out[dest_row[t,j]] = bf16_rn( fp32(p[t,j] * grad_out[t]) ); pad rows 0
 *   grad_probs[t,j] = fp32 sum_h grad_out[t,h] * expert_out[dest_row[t,j],h]; 0 if no row
 * grad_probs is a deterministic fp32 tree reduction (not bit-equal to a
 * sequential sum; within the fp32 summation error bound).
 *   grad_out [N,H] bf16; expert_out [rows_max,H] bf16; topk_probs [N,k] fp32;
 *   grad_expert_out [rows_max,H] bf16; grad_probs [N,k] fp32.
 *   Reads layout->dest_row and layout->pad_mask.
 */
MOE_API int moe_combine_backward(const moe_problem_t *problem, const moe_layout_t *layout, const uint16_t *grad_out,
                         const uint16_t *expert_out, const float *topk_probs, uint16_t *grad_expert_out,
                         float *grad_probs, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_RT_H */
