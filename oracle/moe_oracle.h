/*
 * moe_oracle.h — plain, slow CPU oracle for MoE token dispatch / combine.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg load this library. The product path (the CUDA
 * library and its Python binding) never calls it and shares no code with it.
 *
 * Every function is the plain definition of one step, single-threaded, with
 * no blocking, fusion or reordering beyond what the definition states.
 * Citations name the page and the passage each step follows:
 *   [Megatron MORI]  "Add MORI as a Token Dispatcher" (ROCm/Megatron-LM PR #135)
 *   [UltraEP]        "Integrate UltraEP Runtime for MoE EP Load Balancing" (InternLM/xtuner PR #2050)
 *   [Megatron MoE]   "Megatron MoE 实现" (MoELayer.forward and its four steps)
 *   [mscclpp HT]     mscclpp python/ page: high-throughput dispatch/combine summary
 *   [DeepSpeed EP]   deepspeed/moe/ep_tp_dispatch.py (route-full / partition-dispatch helpers)
 *
 * Sizes: N*k and every row count must fit in int32.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int64_t N;            /* tokens */
    int32_t k;            /* top-k */
    int32_t E_log;        /* logical experts (router width) */
    int32_t num_replicas; /* replica slots in total; 0 = no reroute */
    int32_t R;            /* simulated expert-parallel ranks */
    int32_t C;            /* per-expert capacity; 0 = unlimited */
    int32_t align;        /* rows per expert rounded up to a multiple of align; 0 or 1 = none */
    int32_t tp_size;      /* TP folding: peers sharing the assignments; 0 or 1 = none */
    int32_t tp_rank;      /* this peer, 0 <= tp_rank < tp_size */
} oracle_problem;

/* Every output of the dispatch layout. Arrays are caller-allocated:
 *   per assignment [N*k]: phys_idx, ordinal, logical_ordinal, drop_mask, dest_row
 *   [E_log]: counts_logical, placement
 *   [E]: counts_raw, tokens_per_expert;   [E+1]: expert_offsets
 *   [R]: input_splits, output_splits;     [R+1]: rank_offsets
 *   [8]: counters;  [1]: num_rows
 *   per send-buffer row [rows_max]: row_token, row_slot, row_local_expert, row_prob, pad_mask
 *   [R*N*k]: local_topk (may be NULL)
 */
typedef struct {
    int32_t *phys_idx, *ordinal, *logical_ordinal, *dest_row;
    uint8_t *drop_mask;
    int32_t *counts_logical, *placement;
    int32_t *counts_raw, *tokens_per_expert, *expert_offsets;
    int32_t *input_splits, *output_splits, *rank_offsets;
    int32_t *counters, *num_rows;
    int32_t *row_token, *row_slot, *row_local_expert;
    float *row_prob;
    uint8_t *pad_mask;
    int32_t *local_topk;
} oracle_layout_out;

/* counters[] slots */
enum {
    ORC_ASSIGNMENTS_TOTAL = 0, /* assignments with a valid expert id */
    ORC_KEPT = 1,              /* assignments that own a send-buffer row */
    ORC_DROPPED = 2,           /* assignments over capacity */
    ORC_PADDED = 3,            /* send-buffer rows that hold no assignment */
    ORC_SPLIT_SUM_IN = 4,
    ORC_SPLIT_SUM_OUT = 5,
    ORC_NUM_ROWS = 6,
    ORC_ERROR = 7              /* 1 if an expert id was outside [-1, E_log) */
};

int oracle_problem_valid(const oracle_problem *p);
int32_t oracle_num_experts(const oracle_problem *p);
int64_t oracle_rows_max(const oracle_problem *p);

void oracle_route_topk(const float *logits, const uint8_t *token_mask, int64_t N, int32_t E, int32_t k,
                       int32_t *topk_idx, float *topk_probs);

int oracle_layout(const oracle_problem *p, const int32_t *topk_idx, const float *topk_probs,
                  const oracle_layout_out *o);

void oracle_permute(const oracle_problem *p, int32_t H, const int32_t *dest_row, int64_t rows_max,
                    const uint16_t *hidden, uint16_t *send);

void oracle_combine(const oracle_problem *p, int32_t H, const int32_t *dest_row, const uint16_t *expert_out,
                    const float *topk_probs, uint16_t *out);

void oracle_restore_combined(const oracle_problem *p, int32_t H, int32_t tp_size, const int32_t *const *dest_rows,
                             const uint16_t *const *expert_outs, const float *topk_probs, uint16_t *out);

void oracle_permute_backward(const oracle_problem *p, int32_t H, const int32_t *dest_row,
                             const uint16_t *grad_send, uint16_t *grad_hidden);

void oracle_combine_backward(const oracle_problem *p, int32_t H, int64_t rows_max, const int32_t *dest_row,
                             const int32_t *row_token, const float *row_prob, const uint16_t *grad_out,
                             const uint16_t *expert_out, uint16_t *grad_expert_out, float *grad_probs);

/* DeepEP-style token-dedup view (one row per (token, rank) with any kept slot on the rank). */
typedef struct {
    int32_t *num_tokens_per_rank; /* [R] */
    int32_t *recv_rank_offsets;   /* [R+1] */
    int32_t *num_recv;            /* [1] */
    uint8_t *is_token_in_rank;    /* [N*R] */
    int32_t *token_rank_row;      /* [N*R] */
    int32_t *recv_src_token;      /* [recv_max] */
    int32_t *recv_topk_idx;       /* [recv_max*k] */
    float *recv_topk_weights;     /* [recv_max*k] */
    uint8_t *recv_routing_map;    /* [recv_max*E_loc] */
    float *recv_probs;            /* [recv_max*E_loc] */
    uint8_t *recv_pad_mask;       /* [recv_max] */
} oracle_dedup_out;

int64_t oracle_dedup_rows_max(const oracle_problem *p);
int oracle_dedup_layout(const oracle_problem *p, const int32_t *phys_idx, const int32_t *dest_row,
                        const float *topk_probs, const oracle_dedup_out *o);
void oracle_dedup_combine_local(const oracle_problem *p, int32_t H, int64_t recv_max, const int32_t *dest_row,
                                const int32_t *rank_offsets, const int32_t *recv_src_token,
                                const int32_t *recv_rank_offsets, const uint16_t *expert_out,
                                const float *topk_probs, uint16_t *partial);

uint16_t oracle_bf16_from_f32(float x);
float oracle_f32_from_bf16(uint16_t b);

#ifdef __cplusplus
}
#endif
#endif
