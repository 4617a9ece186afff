/*
 * moe_oracle_omp.c — the oracle's token-independent steps on every host core.
 *
 * TEST INFRASTRUCTURE ONLY (and a timed CPU reference): the benchmark times it as the all-cores
 * CPU baseline beside the single-threaded oracle; the tests check it against
 * that oracle. It is built into a library of its own (libmoe_oracle_omp.so,
 * gcc -fopenmp) from this file and moe_oracle.c; the single-threaded library
 * and its pins are untouched.
 *
 * Nothing here computes anything itself: each OpenMP thread calls the
 * unchanged single-threaded oracle function on a contiguous chunk of tokens.
 * Router top-k, permute and combine treat every token on its own, so the
 * results are the oracle's bit for bit. The dispatch layout is not here: its
 * stable ordinals run over all assignments in order, so it stays serial.
 */
#include <omp.h>
#include <stddef.h>
#include <string.h>

#include "moe_oracle.h"

int oracle_omp_threads(void) { return omp_get_max_threads(); }

/* This thread's contiguous share [*first, *first + *count) of n items. */
static void oracle_omp_share(int64_t n, int64_t *first, int64_t *count)
{
    const int64_t T = omp_get_num_threads(), i = omp_get_thread_num();
    const int64_t per = (n + T - 1) / T;
    int64_t f = per * i;
    if (f > n)
        f = n;
    *first = f;
    *count = (n - f < per) ? n - f : per;
}

void oracle_omp_route_topk(const float *logits, const uint8_t *token_mask, int64_t N, int32_t E, int32_t k,
                           int32_t *topk_idx, float *topk_probs)
{
#pragma omp parallel
    {
        int64_t t0, n;
        oracle_omp_share(N, &t0, &n);
        if (n > 0)
            oracle_route_topk(logits + t0 * E, token_mask ? token_mask + t0 : NULL, n, E, k, topk_idx + t0 * k,
                              topk_probs + t0 * k);
    }
}

/* The oracle's permute: every row zero, then each kept assignment's row copied.
 * The zero fill is split by rows; the copies by tokens (rows_max = 0 tells the
 * oracle's own call that the rows are already zero). */
void oracle_omp_permute(const oracle_problem *p, int32_t H, const int32_t *dest_row, int64_t rows_max,
                        const uint16_t *hidden, uint16_t *send)
{
#pragma omp parallel
    {
        int64_t r0, nr;
        oracle_omp_share(rows_max, &r0, &nr);
        if (nr > 0)
            memset(send + r0 * H, 0, (size_t)nr * (size_t)H * sizeof(uint16_t));
    }
#pragma omp parallel
    {
        int64_t t0, n;
        oracle_omp_share(p->N, &t0, &n);
        if (n > 0) {
            oracle_problem q = *p;
            q.N = n;
            oracle_permute(&q, H, dest_row + t0 * p->k, 0, hidden + t0 * H, send);
        }
    }
}

void oracle_omp_combine(const oracle_problem *p, int32_t H, const int32_t *dest_row, const uint16_t *expert_out,
                        const float *topk_probs, uint16_t *out)
{
#pragma omp parallel
    {
        int64_t t0, n;
        oracle_omp_share(p->N, &t0, &n);
        if (n > 0) {
            oracle_problem q = *p;
            q.N = n;
            oracle_combine(&q, H, dest_row + t0 * p->k, expert_out, topk_probs ? topk_probs + t0 * p->k : NULL,
                           out + t0 * H);
        }
    }
}
