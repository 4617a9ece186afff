/*
 * moe_oracle.c — plain, slow CPU oracle for MoE token dispatch / combine.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by the tests, the smoke check and the
 * benchmark's CPU-baseline leg, never by the product path. It shares no code,
 * header, table or helper with the CUDA library.
 *
 * Build: cc -O2 -std=c11 -ffp-contract=off -fPIC -shared (no fast-math), so
 * that every floating-point operation is exactly the one written here; the
 * one fused multiply-add of the combine is spelled fmaf().
 *
 * Page abbreviations are listed in moe_oracle.h.
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- bf16 ---- */

/* bf16 is the upper half of an IEEE binary32. Rounding keeps the upper 16
 * bits after adding half an ulp, ties to even; NaN stays a quiet NaN with its
 * sign. Widening is exact. */
uint16_t oracle_bf16_from_f32(float x)
{
    uint32_t b;
    memcpy(&b, &x, sizeof b);
    if ((b & 0x7F800000u) == 0x7F800000u && (b & 0x007FFFFFu) != 0)
        return (uint16_t)((b >> 16) | 0x0040u);
    uint32_t lsb = (b >> 16) & 1u;
    return (uint16_t)((b + 0x7FFFu + lsb) >> 16);
}

float oracle_f32_from_bf16(uint16_t h)
{
    uint32_t b = (uint32_t)h << 16;
    float x;
    memcpy(&x, &b, sizeof x);
    return x;
}

/* ------------------------------------------------------------- problem ---- */

int32_t oracle_num_experts(const oracle_problem *p) { return p->E_log + p->num_replicas; }

static int32_t oracle_align(const oracle_problem *p) { return p->align > 1 ? p->align : 1; }
static int32_t oracle_tp(const oracle_problem *p) { return p->tp_size > 1 ? p->tp_size : 1; }

/* Capacity slots per expert in one TP peer's buffer: ceil(C / tp_size). */
static int32_t oracle_local_capacity(const oracle_problem *p)
{
    int32_t T = oracle_tp(p);
    return p->C > 0 ? (p->C + T - 1) / T : 0;
}

int64_t oracle_rows_max(const oracle_problem *p)
{
    /* Sync-free padded buffers ([Megatron MORI], the commit that drops the
     * recv_num_token host sync): the send buffer always has its upper-bound
     * size. With a capacity it is E*C slots, otherwise one row per assignment
     * plus, with row alignment, at most align-1 pad rows per expert. A TP peer
     * holds at most ceil(c_e / tp_size) of each expert's c_e assignments. */
    const int64_t E = oracle_num_experts(p), T = oracle_tp(p);
    if (p->C > 0)
        return E * oracle_local_capacity(p);
    return (p->N * p->k + E * (T - 1)) / T + E * (oracle_align(p) - 1);
}

int oracle_problem_valid(const oracle_problem *p)
{
    if (p->N < 0 || p->k < 1 || p->E_log < 1 || p->R < 1 || p->C < 0 || p->num_replicas < 0 || p->align < 0)
        return 0;
    if (p->tp_size < 0 || p->tp_rank < 0 || p->tp_rank >= oracle_tp(p))
        return 0;
    if (p->C > 0 && oracle_local_capacity(p) % oracle_align(p) != 0)
        return 0;
    if (p->E_log % p->R != 0 || p->num_replicas % p->R != 0 || p->num_replicas > p->E_log)
        return 0;
    if (p->N * (int64_t)p->k > 0x7FFFFFFF || oracle_rows_max(p) > 0x7FFFFFFF)
        return 0;
    return 1;
}

/* --------------------------------------------------------------- route ---- */

/*
 * [Megatron MoE] MoELayer.router_and_preprocess: the router turns each token's
 * hidden state into routing probabilities and a top-k routing map.
 * [Megatron MORI] router.py: padding tokens take no part in routing.
 *
 * Definition used (softmax over all E experts, no renormalisation over the k
 * chosen ones):  p[t,e] = exp(l[t,e] - m) / sum_e' exp(l[t,e'] - m),  m = max_e l[t,e],
 * evaluated in double and rounded once to float. The k chosen experts are the
 * k largest logits (softmax is strictly increasing in the logit), listed in
 * descending order, equal logits broken towards the lower expert id. A masked
 * token gets ids -1 and probs 0.
 */
void oracle_route_topk(const float *logits, const uint8_t *token_mask, int64_t N, int32_t E, int32_t k,
                       int32_t *topk_idx, float *topk_probs)
{
    unsigned char *chosen = (unsigned char *)malloc((size_t)(E > 0 ? E : 1));
    for (int64_t t = 0; t < N; ++t) {
        const float *l = logits + t * E;
        int32_t *idx = topk_idx + t * k;
        float *pr = topk_probs + t * k;
        if (token_mask && token_mask[t]) {
            for (int32_t j = 0; j < k; ++j) {
                idx[j] = -1;
                pr[j] = 0.0f;
            }
            continue;
        }
        double m = (double)l[0];
        for (int32_t e = 1; e < E; ++e)
            if ((double)l[e] > m)
                m = (double)l[e];
        double s = 0.0;
        for (int32_t e = 0; e < E; ++e)
            s += exp((double)l[e] - m);
        memset(chosen, 0, (size_t)E);
        for (int32_t j = 0; j < k; ++j) {
            int32_t best = -1;
            for (int32_t e = 0; e < E; ++e) {
                if (chosen[e])
                    continue;
                if (best < 0 || l[e] > l[best]) /* strict: an equal logit keeps the lower id */
                    best = e;
            }
            chosen[best] = 1;
            idx[j] = best;
            pr[j] = (float)(exp((double)l[best] - m) / s);
        }
    }
    free(chosen);
}

/* -------------------------------------------------------------- layout ---- */

/*
 * Dispatch layout: every step of the dispatch side except the row copy.
 *
 * Notation: an assignment a = t*k + j is slot j of token t in the flattened,
 * row-major [N, k] order. Experts are numbered physically: rank r owns the
 * contiguous block [r*E_loc, (r+1)*E_loc) with E_loc = E/R. Without replicas
 * physical = logical. With replicas, rank r holds the masters of logical
 * experts r*M .. r*M+M-1 (M = E_log/R) at physical r*E_loc + i, followed by
 * S = num_replicas/R replica slots.
 *
 * Steps, in the pages' order:
 *  1. logical histogram and logical ordinals
 *       ([DeepSpeed EP] assignment_ordinals_by_expert: stable ordinals of the
 *        flattened assignments within each expert);
 *  2. hot-expert placement and logical->physical reroute ([UltraEP]: replicas
 *     of the experts that the current layer actually loads most, part of their
 *     tokens rerouted to the replica slot; router semantics stay logical);
 *  3. physical ordinals and counts;
 *  4. capacity: drop_mask, tokens_per_expert, pad rows ([DeepSpeed EP]
 *     RoutedAssignmentPayload.capacity_slots / drop_mask / pad_mask), then
 *     the optional TP folding of the active assignments ([DeepSpeed EP]
 *     partition_assignments);
 *  5. exclusive scan into expert_offsets, per-rank input_splits / rank_offsets,
 *     output_splits = input_splits ([DeepSpeed EP] _recompute_input_splits,
 *     partition_assignments);
 *  6. row maps: dest_row per assignment and, per send-buffer row, the token,
 *     top-k slot, receiver-side prob and rank-local expert id, -1 / 0 in pad
 *     and tail rows ([Megatron MORI]: local ids with -1 sentinels, receiver-side
 *     dispatched_probs, tails masked 0 / -1 / 0);
 *  7. the per-rank DeepEP-contract view local_topk and dispatch_counters
 *     ([DeepSpeed EP] dispatch_counters).
 *
 * Readings where the pages are silent (taken here, not from the pages): first-come drop
 * in flattened order; hot set = the num_replicas largest logical counts,
 * equal counts to the lower id; greedy placement onto the least-loaded other
 * rank with a free slot; a hot expert's logical ordinal o goes to the master
 * when o is even and to the replica when o is odd.
 *
 * Returns 0 on success, -1 for an invalid problem. An expert id outside
 * [-1, E_log) is skipped as if it were -1 and sets counters[ORC_ERROR].
 */
int oracle_layout(const oracle_problem *p, const int32_t *topk_idx, const float *topk_probs,
                  const oracle_layout_out *o)
{
    if (!oracle_problem_valid(p))
        return -1;
    const int64_t NK = p->N * p->k;
    const int32_t E_log = p->E_log, R = p->R, C = p->C, k = p->k;
    const int32_t E = oracle_num_experts(p);
    const int32_t E_loc = E / R;
    const int32_t M = E_log / R;
    const int32_t S = p->num_replicas / R;
    const int64_t rows_max = oracle_rows_max(p);
    int32_t error = 0;

    int32_t *seen = (int32_t *)calloc((size_t)(E > E_log ? E : E_log) + 1, sizeof(int32_t));

    /* 1. logical histogram and logical ordinals (running count of earlier
     *    assignments to the same logical expert, in flattened order). */
    for (int32_t e = 0; e < E_log; ++e)
        o->counts_logical[e] = 0;
    for (int64_t a = 0; a < NK; ++a) {
        int32_t e = topk_idx[a];
        if (e < -1 || e >= E_log) {
            error = 1;
            e = -1;
        }
        if (e < 0) {
            o->logical_ordinal[a] = -1;
            continue;
        }
        o->logical_ordinal[a] = seen[e]++;
        o->counts_logical[e] += 1;
    }

    /* 2. hot set and greedy placement. */
    for (int32_t e = 0; e < E_log; ++e)
        o->placement[e] = -1;
    if (p->num_replicas > 0) {
        unsigned char *is_hot = (unsigned char *)calloc((size_t)E_log, 1);
        int64_t *load = (int64_t *)calloc((size_t)R, sizeof(int64_t));
        int32_t *free_slots = (int32_t *)malloc((size_t)R * sizeof(int32_t));
        for (int32_t r = 0; r < R; ++r) {
            free_slots[r] = S;
            for (int32_t i = 0; i < M; ++i)
                load[r] += o->counts_logical[r * M + i];
        }
        for (int32_t h = 0; h < p->num_replicas; ++h) {
            /* next hottest: largest count, equal counts -> lower id */
            int32_t e = -1;
            for (int32_t c = 0; c < E_log; ++c)
                if (!is_hot[c] && (e < 0 || o->counts_logical[c] > o->counts_logical[e]))
                    e = c;
            is_hot[e] = 1;
            int32_t home = e / M;
            int32_t best = -1;
            for (int32_t r = 0; r < R; ++r)
                if (r != home && free_slots[r] > 0 && (best < 0 || load[r] < load[best]))
                    best = r;
            if (best < 0) /* only the master's own rank has a free slot left */
                best = home;
            int32_t slot = S - free_slots[best];
            free_slots[best] -= 1;
            o->placement[e] = best * E_loc + M + slot;
            int64_t moved = o->counts_logical[e] / 2;
            load[home] -= moved;
            load[best] += moved;
        }
        free(is_hot);
        free(load);
        free(free_slots);
    }

    /* 3. physical ids, physical ordinals (running count per physical expert),
     *    physical counts. */
    for (int32_t e = 0; e < E; ++e) {
        seen[e] = 0;
        o->counts_raw[e] = 0;
    }
    for (int64_t a = 0; a < NK; ++a) {
        int32_t lo = o->logical_ordinal[a];
        if (lo < 0) {
            o->phys_idx[a] = -1;
            o->ordinal[a] = -1;
            continue;
        }
        int32_t e = topk_idx[a];
        int32_t master = (e / M) * E_loc + (e % M);
        int32_t q = (o->placement[e] >= 0 && (lo % 2) == 1) ? o->placement[e] : master;
        o->phys_idx[a] = q;
        o->ordinal[a] = seen[q]++;
        o->counts_raw[q] += 1;
    }

    /* 4. capacity: an assignment whose physical ordinal reaches C is dropped. */
    int64_t valid = 0, dropped = 0;
    for (int64_t a = 0; a < NK; ++a) {
        o->drop_mask[a] = 0;
        if (o->phys_idx[a] < 0)
            continue;
        ++valid;
        if (C > 0 && o->ordinal[a] >= C) {
            o->drop_mask[a] = 1;
            ++dropped;
        }
    }

    /* 4b. TP folding ([DeepSpeed EP] partition_assignments): this peer keeps the
     *     active (valid, not dropped) assignments whose stable per-expert ordinal
     *     is congruent to tp_rank modulo tp_size; its local ordinal is the running
     *     count of earlier kept assignments to the same expert. Without folding
     *     every active assignment is kept at its own ordinal. */
    const int32_t T = oracle_tp(p);
    int32_t *local_ordinal = (int32_t *)malloc((size_t)(NK > 0 ? NK : 1) * sizeof(int32_t));
    for (int32_t e = 0; e < E; ++e) {
        o->tokens_per_expert[e] = 0;
        seen[e] = 0;
    }
    int64_t kept = 0;
    for (int64_t a = 0; a < NK; ++a) {
        int32_t q = o->phys_idx[a];
        local_ordinal[a] = -1;
        if (q < 0 || o->drop_mask[a] || o->ordinal[a] % T != p->tp_rank)
            continue;
        local_ordinal[a] = seen[q]++;
        o->tokens_per_expert[q] += 1;
        ++kept;
    }

    /* 5. exclusive scan and splits. With a capacity every expert owns C rows
     *    (ceil(C / tp_size) in a TP peer's buffer); otherwise its token count,
     *    rounded up to a multiple of the row alignment ([Megatron MORI]: router
     *    padding for FP8 grouped GEMMs). */
    const int32_t A = oracle_align(p);
    o->expert_offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e) {
        int32_t rows = C > 0 ? oracle_local_capacity(p) : o->tokens_per_expert[e];
        while (rows % A != 0)
            ++rows;
        o->expert_offsets[e + 1] = o->expert_offsets[e] + rows;
    }
    *o->num_rows = o->expert_offsets[E];
    int64_t split_sum = 0;
    for (int32_t r = 0; r < R; ++r) {
        o->rank_offsets[r] = o->expert_offsets[r * E_loc];
        o->input_splits[r] = o->expert_offsets[(r + 1) * E_loc] - o->expert_offsets[r * E_loc];
        o->output_splits[r] = o->input_splits[r];
        split_sum += o->input_splits[r];
    }
    o->rank_offsets[R] = o->expert_offsets[E];

    /* 6. row maps. Every row starts as a pad row, then each kept assignment
     *    claims row expert_offsets[e] + ordinal. */
    for (int64_t row = 0; row < rows_max; ++row) {
        o->row_token[row] = -1;
        o->row_slot[row] = -1;
        o->row_local_expert[row] = -1;
        o->row_prob[row] = 0.0f;
        o->pad_mask[row] = 1;
    }
    for (int64_t a = 0; a < NK; ++a) {
        int32_t q = o->phys_idx[a];
        if (local_ordinal[a] < 0) {
            o->dest_row[a] = -1;
            continue;
        }
        int32_t row = o->expert_offsets[q] + local_ordinal[a];
        o->dest_row[a] = row;
        o->row_token[row] = (int32_t)(a / k);
        o->row_slot[row] = (int32_t)(a % k);
        o->row_local_expert[row] = q - (q / E_loc) * E_loc;
        o->row_prob[row] = topk_probs ? topk_probs[a] : 0.0f;
        o->pad_mask[row] = 0;
    }

    /* 7. per-rank local view and counters. */
    if (o->local_topk) {
        for (int32_t r = 0; r < R; ++r)
            for (int64_t a = 0; a < NK; ++a) {
                int32_t q = o->phys_idx[a];
                int keep = local_ordinal[a] >= 0 && q / E_loc == r;
                o->local_topk[(int64_t)r * NK + a] = keep ? q - r * E_loc : -1;
            }
    }
    o->counters[ORC_ASSIGNMENTS_TOTAL] = (int32_t)valid;
    o->counters[ORC_KEPT] = (int32_t)kept;
    o->counters[ORC_DROPPED] = (int32_t)dropped;
    o->counters[ORC_PADDED] = (int32_t)(rows_max - kept);
    o->counters[ORC_SPLIT_SUM_IN] = (int32_t)split_sum;
    o->counters[ORC_SPLIT_SUM_OUT] = (int32_t)split_sum;
    o->counters[ORC_NUM_ROWS] = *o->num_rows;
    o->counters[ORC_ERROR] = error;

    free(local_ordinal);
    free(seen);
    return 0;
}

/* --------------------------------------------------------------- dedup ---- */

/*
 * DeepEP-style dispatch layout ([Megatron MORI]: the DeepEP contract the MORI
 * dispatcher follows; the receiver gets each token once, its local top-k ids
 * with -1 sentinels and receiver-side weights, and _indices_to_multihot turns
 * those into a [tokens, local experts] routing map with probs).
 * Rank r receives token t iff some kept slot j of t (dest_row >= 0) has a
 * physical expert on r. Rows are rank-major and token-ascending within a rank:
 *   token_rank_row[t,r] = recv_rank_offsets[r] + #{t' < t received by r}.
 * At most min(k, R) rows per token: recv_max = N * min(k, R).
 */
int64_t oracle_dedup_rows_max(const oracle_problem *p)
{
    int64_t m = p->k < p->R ? p->k : p->R;
    return p->N * m;
}

int oracle_dedup_layout(const oracle_problem *p, const int32_t *phys_idx, const int32_t *dest_row,
                        const float *topk_probs, const oracle_dedup_out *o)
{
    if (!oracle_problem_valid(p))
        return -1;
    const int64_t N = p->N;
    const int32_t k = p->k, R = p->R;
    const int32_t E_loc = oracle_num_experts(p) / R;
    const int64_t recv_max = oracle_dedup_rows_max(p);
    /* is_token_in_rank and the per-rank token counts */
    for (int32_t r = 0; r < R; ++r)
        o->num_tokens_per_rank[r] = 0;
    for (int64_t t = 0; t < N; ++t)
        for (int32_t r = 0; r < R; ++r) {
            uint8_t in = 0;
            for (int32_t j = 0; j < k; ++j)
                if (dest_row[t * k + j] >= 0 && phys_idx[t * k + j] / E_loc == r)
                    in = 1;
            o->is_token_in_rank[t * R + r] = in;
            o->num_tokens_per_rank[r] += in;
        }
    o->recv_rank_offsets[0] = 0;
    for (int32_t r = 0; r < R; ++r)
        o->recv_rank_offsets[r + 1] = o->recv_rank_offsets[r] + o->num_tokens_per_rank[r];
    *o->num_recv = o->recv_rank_offsets[R];
    /* every receive row starts as a tail row: token -1, ids -1, weights / map / probs 0 */
    for (int64_t row = 0; row < recv_max; ++row) {
        o->recv_src_token[row] = -1;
        o->recv_pad_mask[row] = 1;
        for (int32_t j = 0; j < k; ++j) {
            o->recv_topk_idx[row * k + j] = -1;
            o->recv_topk_weights[row * k + j] = 0.0f;
        }
        for (int32_t e = 0; e < E_loc; ++e) {
            o->recv_routing_map[row * E_loc + e] = 0;
            o->recv_probs[row * E_loc + e] = 0.0f;
        }
    }
    /* rank-major rows, tokens in ascending order within a rank */
    for (int32_t r = 0; r < R; ++r) {
        int32_t next = o->recv_rank_offsets[r];
        for (int64_t t = 0; t < N; ++t) {
            if (!o->is_token_in_rank[t * R + r]) {
                o->token_rank_row[t * R + r] = -1;
                continue;
            }
            int32_t row = next++;
            o->token_rank_row[t * R + r] = row;
            o->recv_src_token[row] = (int32_t)t;
            o->recv_pad_mask[row] = 0;
            for (int32_t j = 0; j < k; ++j) {
                int32_t q = phys_idx[t * k + j];
                if (dest_row[t * k + j] < 0 || q / E_loc != r)
                    continue;
                int32_t local = q - r * E_loc;
                float w = topk_probs ? topk_probs[t * k + j] : 0.0f;
                o->recv_topk_idx[(int64_t)row * k + j] = local;
                o->recv_topk_weights[(int64_t)row * k + j] = w;
                /* _indices_to_multihot: a set bit per local expert, its prob beside it */
                o->recv_routing_map[(int64_t)row * E_loc + local] = 1;
                o->recv_probs[(int64_t)row * E_loc + local] = w;
            }
        }
    }
    return 0;
}

/*
 * Receiver side of the DeepEP-style combine: each rank reduces, per received
 * token, the weighted outputs of the token's kept slots whose row lies in that
 * rank's part of the send buffer, in ascending slot order, fp32 fused
 * multiply-add from +0, rounded once to bf16. Tail rows are 0. The sender then
 * sums the partials over ranks (the unit-weight combine over token_rank_row).
 */
void oracle_dedup_combine_local(const oracle_problem *p, int32_t H, int64_t recv_max, const int32_t *dest_row,
                                const int32_t *rank_offsets, const int32_t *recv_src_token,
                                const int32_t *recv_rank_offsets, const uint16_t *expert_out,
                                const float *topk_probs, uint16_t *partial)
{
    for (int64_t row = 0; row < recv_max; ++row) {
        int32_t t = recv_src_token[row];
        int32_t r = -1;
        for (int32_t q = 0; q < p->R; ++q)
            if (row >= recv_rank_offsets[q] && row < recv_rank_offsets[q + 1])
                r = q;
        for (int32_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            if (t >= 0 && r >= 0)
                for (int32_t j = 0; j < p->k; ++j) {
                    int32_t d = dest_row[(int64_t)t * p->k + j];
                    if (d < rank_offsets[r] || d >= rank_offsets[r + 1])
                        continue;
                    float w = topk_probs ? topk_probs[(int64_t)t * p->k + j] : 1.0f;
                    acc = fmaf(w, oracle_f32_from_bf16(expert_out[(int64_t)d * H + h]), acc);
                }
            partial[row * H + h] = oracle_bf16_from_f32(acc);
        }
    }
}

/* ------------------------------------------------------------- permute ---- */

/*
 * [Megatron MoE] dispatch_postprocess gives the permuted tokens per expert;
 * [Megatron MORI] fuses this permute into the dispatch node and masks padded
 * tails with 0. send[dest_row[t,j]] = hidden[t] for every kept assignment; all
 * other rows are zero.
 */
void oracle_permute(const oracle_problem *p, int32_t H, const int32_t *dest_row, int64_t rows_max,
                    const uint16_t *hidden, uint16_t *send)
{
    memset(send, 0, (size_t)rows_max * (size_t)H * sizeof(uint16_t));
    for (int64_t t = 0; t < p->N; ++t)
        for (int32_t j = 0; j < p->k; ++j) {
            int32_t row = dest_row[t * p->k + j];
            if (row >= 0)
                memcpy(send + (int64_t)row * H, hidden + t * H, (size_t)H * sizeof(uint16_t));
        }
}

/* ------------------------------------------------------------- combine ---- */

/*
 * [DeepSpeed EP] restore_combined: weighted expert outputs are added back
 * into [num_tokens, H] one top-k slot at a time, in ascending slot order, so
 * the accumulation order per token is fixed. [Megatron MoE] combine.
 *
 * Precision (a reading; the page itself accumulates in the activation dtype):
 * fp32 accumulator starting at +0, one fused multiply-add per kept slot in
 * ascending j, one rounding to bf16 at the end.
 *   out[t,h] = bf16( fma(p[t,k-1], y[.,h], ... fma(p[t,0], y[.,h], +0) ... ) )
 * A NULL prob array means unit weights.
 */
void oracle_combine(const oracle_problem *p, int32_t H, const int32_t *dest_row, const uint16_t *expert_out,
                    const float *topk_probs, uint16_t *out)
{
    for (int64_t t = 0; t < p->N; ++t)
        for (int32_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int32_t j = 0; j < p->k; ++j) {
                int32_t row = dest_row[t * p->k + j];
                if (row < 0)
                    continue;
                float w = topk_probs ? topk_probs[t * p->k + j] : 1.0f;
                acc = fmaf(w, oracle_f32_from_bf16(expert_out[(int64_t)row * H + h]), acc);
            }
            out[t * H + h] = oracle_bf16_from_f32(acc);
        }
}

/*
 * [DeepSpeed EP] restore_combined: the TP peers' weighted outputs are gathered
 * and added back per token one top-k slot at a time in ascending slot order.
 * On one GPU the gather is the set of peer buffers: dest_rows[q] and
 * expert_outs[q] are peer q's row map and expert output; each assignment has a
 * row in at most one peer. Same fp32 fused multiply-add chain as the combine.
 */
void oracle_restore_combined(const oracle_problem *p, int32_t H, int32_t tp_size, const int32_t *const *dest_rows,
                             const uint16_t *const *expert_outs, const float *topk_probs, uint16_t *out)
{
    for (int64_t t = 0; t < p->N; ++t)
        for (int32_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int32_t j = 0; j < p->k; ++j)
                for (int32_t q = 0; q < tp_size; ++q) {
                    int32_t row = dest_rows[q][t * p->k + j];
                    if (row < 0)
                        continue;
                    float w = topk_probs ? topk_probs[t * p->k + j] : 1.0f;
                    acc = fmaf(w, oracle_f32_from_bf16(expert_outs[q][(int64_t)row * H + h]), acc);
                }
            out[t * H + h] = oracle_bf16_from_f32(acc);
        }
}

/* ------------------------------------------------------------ backward ---- */

/*
 * [Megatron MORI] backward of dispatch: the gradient of the copied rows is
 * summed back per token using receiver-side indices. Definition: fp32 sum of
 * grad_send[dest_row[t,j]] over ascending j (kept slots only), rounded once to bf16.
 */
void oracle_permute_backward(const oracle_problem *p, int32_t H, const int32_t *dest_row,
                             const uint16_t *grad_send, uint16_t *grad_hidden)
{
    for (int64_t t = 0; t < p->N; ++t)
        for (int32_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int32_t j = 0; j < p->k; ++j) {
                int32_t row = dest_row[t * p->k + j];
                if (row >= 0)
                    acc = acc + oracle_f32_from_bf16(grad_send[(int64_t)row * H + h]);
            }
            grad_hidden[t * H + h] = oracle_bf16_from_f32(acc);
        }
}

/*
 * [Megatron MORI] backward of combine with receiver-side probs
 * (dispatched_probs [total_recv, topk], not the sender's [N, topk]).
 * For out[t] = sum_j p[t,j] * y[dest_row[t,j]]:
 *   grad_expert_out[row] = bf16( fp32( row_prob[row] * g[row_token[row]] ) ), 0 in pad rows;
 *   grad_probs[t,j]     = fp32( sum_h g[t,h] * y[dest_row[t,j], h] )  summed in double,
 *                         ascending h; 0 where the slot has no row.
 */
void oracle_combine_backward(const oracle_problem *p, int32_t H, int64_t rows_max, const int32_t *dest_row,
                             const int32_t *row_token, const float *row_prob, const uint16_t *grad_out,
                             const uint16_t *expert_out, uint16_t *grad_expert_out, float *grad_probs)
{
    for (int64_t row = 0; row < rows_max; ++row) {
        int32_t t = row_token[row];
        for (int32_t h = 0; h < H; ++h) {
            uint16_t v = 0;
            if (t >= 0) {
                float prod = row_prob[row] * oracle_f32_from_bf16(grad_out[(int64_t)t * H + h]);
                v = oracle_bf16_from_f32(prod);
            }
            grad_expert_out[row * H + h] = v;
        }
    }
    for (int64_t t = 0; t < p->N; ++t)
        for (int32_t j = 0; j < p->k; ++j) {
            int32_t row = dest_row[t * p->k + j];
            double s = 0.0;
            if (row >= 0)
                for (int32_t h = 0; h < H; ++h)
                    s += (double)oracle_f32_from_bf16(grad_out[t * H + h]) *
                         (double)oracle_f32_from_bf16(expert_out[(int64_t)row * H + h]);
            grad_probs[t * p->k + j] = (float)s;
        }
}
