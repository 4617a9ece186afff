// ep.cuh — the plan of the expert-parallel exchange.
//
// Megatron MoE page, the all-to-all token dispatcher: each rank's permuted rows
// go to the rank that owns their expert, and the receiver orders what it got by
// local expert. Megatron MORI page: dispatch writes into the receivers' buffers
// (the permute fused in), combine reads the expert outputs back.
//
// Receive layout of rank r: its experts q ascending; within q, the source ranks
// s ascending; each source's rows for q in its own send-buffer order (padding
// rows included). With rows[s][q] = expert_offsets_s[q+1] - expert_offsets_s[q]:
//   start[q] = sum of rows[s'][q'] over all sources s' and over the experts q'
//              of q's owner below q
//   base_s[q] = start[q] + sum of rows[s'][q] over sources s' < s
// ep_plan_kernel computes, from every rank's expert_offsets (gathered by the
// caller), base_s for this source s and this rank's own receive layout.
#pragma once

#include <cstdint>

#include "moe_rt.h"
#include "ptx.cuh"

namespace moert {

constexpr int EP_PLAN_THREADS = 1024;
constexpr int EP_PLAN_PER = 4; // experts per thread in the scan: E <= 4096

struct EpPlanArgs {
    const int32_t *offsets_all; // [R][E + 1]
    int32_t R, E, E_loc, src;
    int64_t recv_max;
    int32_t *base;                // [E]
    int32_t *recv_expert_offsets; // [E_loc + 1] of this rank
    int32_t *num_recv;            // [1]
    uint32_t *status;             // [1]
};

__global__ void __launch_bounds__(EP_PLAN_THREADS) ep_plan_kernel(EpPlanArgs a)
{
    extern __shared__ int32_t ep_smem[];
    int32_t *s_col = ep_smem;         // [E + 1] rows of expert q over all sources, then their exclusive scan
    int32_t *s_pre = s_col + a.E + 1; // [E] rows of expert q over sources before src
    __shared__ int32_t s_wsum[EP_PLAN_THREADS / 32];
    pdl_trigger();
    pdl_wait();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = a.E;
    uint32_t err = 0;
    for (int q = tid; q < E; q += EP_PLAN_THREADS) {
        int32_t col = 0, pre = 0;
        for (int s = 0; s < a.R; ++s) {
            const int32_t *o = a.offsets_all + static_cast<int64_t>(s) * (E + 1);
            const int32_t rows = __ldg(o + q + 1) - __ldg(o + q);
            if (rows < 0)
                err = MOE_DEV_ROW_RANGE;
            col += rows;
            pre += s < a.src ? rows : 0;
        }
        s_col[q] = col;
        s_pre[q] = pre;
    }
    __syncthreads();
    // exclusive scan of s_col over all experts (EP_PLAN_PER consecutive per thread)
    const int q0 = tid * EP_PLAN_PER;
    int32_t v[EP_PLAN_PER];
    int32_t sum = 0;
#pragma unroll
    for (int u = 0; u < EP_PLAN_PER; ++u) {
        v[u] = q0 + u < E ? s_col[q0 + u] : 0;
        sum += v[u];
    }
    int32_t inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o)
            inc += n;
    }
    if (lane == 31)
        s_wsum[warp] = inc;
    __syncthreads();
    int32_t wpre = 0;
    for (int w = 0; w < warp; ++w)
        wpre += s_wsum[w];
    __syncthreads(); // every thread has read s_col; it now takes the exclusive prefixes
    int32_t run = wpre + inc - sum;
#pragma unroll
    for (int u = 0; u < EP_PLAN_PER; ++u) {
        if (q0 + u < E)
            s_col[q0 + u] = run;
        run += v[u];
    }
    if (tid == EP_PLAN_THREADS - 1) // E <= EP_PLAN_THREADS * EP_PLAN_PER: the last thread's run is the total
        s_col[E] = run;
    __syncthreads();
    // s_col[q] = exclusive prefix over all experts; relative to the owner's first expert
    for (int q = tid; q < E; q += EP_PLAN_THREADS) {
        const int owner_first = (q / a.E_loc) * a.E_loc;
        const int64_t b = static_cast<int64_t>(s_col[q]) - s_col[owner_first] + s_pre[q];
        const int64_t mine = static_cast<int64_t>(__ldg(a.offsets_all + static_cast<int64_t>(a.src) * (E + 1) + q + 1)) -
                             __ldg(a.offsets_all + static_cast<int64_t>(a.src) * (E + 1) + q);
        if (b + mine > a.recv_max)
            err = MOE_DEV_ROW_RANGE; // the receive buffers are too small for this exchange
        a.base[q] = static_cast<int32_t>(b);
    }
    // this rank's own receive layout: where each local expert's rows start
    const int first = a.src * a.E_loc;
    for (int l = tid; l <= a.E_loc; l += EP_PLAN_THREADS)
        a.recv_expert_offsets[l] = s_col[first + l] - s_col[first];
    if (tid == 0)
        *a.num_recv = s_col[first + a.E_loc] - s_col[first];
    if (err)
        atomicOr(a.status, err);
}


// The all-gather of the ranks' expert_offsets over peer memory: this rank's
// [E+1] offsets go to row `src` of every rank's [R][E+1] table (peer_tables:
// R device pointers, own rank's table included). One thread per (rank, entry).
struct EpPublishArgs {
    const int32_t *offsets;      // [E + 1] this rank's layout expert_offsets
    int32_t *const *peer_tables; // [R] each a [R][E + 1] table
    int32_t R, E, src;
};

__global__ void __launch_bounds__(256) ep_publish_offsets_kernel(EpPublishArgs a)
{
    pdl_trigger();
    pdl_wait(); // the offsets come from the layout just before
    const int64_t n = static_cast<int64_t>(a.R) * (a.E + 1);
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int q = static_cast<int>(i / (a.E + 1));
        const int j = static_cast<int>(i - static_cast<int64_t>(q) * (a.E + 1));
        a.peer_tables[q][static_cast<int64_t>(a.src) * (a.E + 1) + j] = __ldg(a.offsets + j);
    }
}

} // namespace moert
