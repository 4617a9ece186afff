// dedup.cuh — the DeepEP-style token-dedup view and the receiver-side combine.
//
// Megatron MORI page: the MORI dispatcher follows the DeepEP contract — each
// token is sent once to every rank that owns one of its experts; the receiver
// gets rank-local top-k ids with -1 sentinels and receiver-side weights, and
// _indices_to_multihot turns those into a [tokens, local experts] routing map
// with probs. The combine comes back in two levels: every rank reduces its
// local slots per received token, the sender sums the partials over ranks.
//
// dedup_layout_kernel (one cooperative launch, bounded grid barrier):
//   phase 1  each lane builds, for its tokens, the bit set of ranks holding a
//            kept slot (register-resident); per warp and rank the tokens are
//            counted with __ballot_sync; the block publishes per-rank totals;
//   phase 2  every block reads all block totals (one batch of loads), scans
//            them into rank offsets, and places each (token, rank) pair at
//            offset + earlier blocks + earlier warps + earlier lanes of the
//            same rank (so rows are rank-major and token-ascending).
// dedup_fill_kernel then writes the receive-side ids, weights, multihot map
// and probs row by row over the whole GPU (they are a function of the row).
#pragma once

#include <cstdint>

#include "moe_rt.h"
#include "combine.cuh"
#include "grid_barrier.cuh"
#include "ptx.cuh"

namespace moert {

constexpr int DEDUP_THREADS = 256;
constexpr int DEDUP_WARPS = DEDUP_THREADS / 32;
constexpr int DEDUP_MAX_BLOCKS = 128;
constexpr int DEDUP_MAX_TPL = 8; // tokens per lane kept in registers

struct DedupArgs {
    const int32_t *phys_idx; // [N, k]
    const int32_t *dest_row; // [N, k]
    const float *probs;      // [N, k] or null
    int64_t N;
    int64_t recv_max;
    int32_t k, R, E_loc;
    int32_t G;
    int32_t *ws_counts;   // [G][R]
    uint32_t *ws_barrier; // [3] as in the layout: ticket word, unused, error bits
    uint64_t barrier_limit_ns;
    moe_dedup_t out;
};

__device__ __forceinline__ uint32_t dedup_lanemask_lt()
{
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

template <int TPL> // tokens per lane; a warp owns 32 * TPL consecutive tokens
__global__ void __launch_bounds__(DEDUP_THREADS) dedup_layout_kernel(DedupArgs a)
{
    __shared__ uint32_t s_wcnt[DEDUP_WARPS][MOE_MAX_DEDUP_RANKS]; // per-warp counts, then exclusive prefixes
    __shared__ int32_t s_part[2][DEDUP_THREADS];
    __shared__ int32_t s_pre[MOE_MAX_DEDUP_RANKS];
    __shared__ int32_t s_off[MOE_MAX_DEDUP_RANKS + 1];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x;
    const int R = a.R, k = a.k;
    const uint32_t lt = dedup_lanemask_lt();

    for (int i = tid; i < DEDUP_WARPS * MOE_MAX_DEDUP_RANKS; i += DEDUP_THREADS)
        (&s_wcnt[0][0])[i] = 0;
    __syncthreads();
    pdl_trigger();
    pdl_wait();

    const int64_t base = (static_cast<int64_t>(b) * DEDUP_WARPS + warp) * (32 * TPL);

    // ---- phase 1: rank sets of this lane's tokens, per-warp per-rank counts
    uint32_t mask[TPL];
#pragma unroll
    for (int u = 0; u < TPL; ++u) {
        const int64_t t = base + u * 32 + lane;
        uint32_t m = 0;
        if (t < a.N) {
            for (int j = 0; j < k; ++j) {
                const int32_t d = __ldg(a.dest_row + t * k + j);
                const int32_t q = __ldg(a.phys_idx + t * k + j);
                if (d >= 0 && q >= 0)
                    m |= 1u << (q / a.E_loc);
            }
        }
        mask[u] = m;
    }
#pragma unroll
    for (int u = 0; u < TPL; ++u)
        for (int r = 0; r < R; ++r) {
            const uint32_t bal = __ballot_sync(0xffffffffu, (mask[u] >> r) & 1u);
            if (lane == 0)
                s_wcnt[warp][r] += __popc(bal);
        }
    __syncthreads();
    if (tid < R) {
        uint32_t run = 0;
#pragma unroll
        for (int w = 0; w < DEDUP_WARPS; ++w) {
            const uint32_t c = s_wcnt[w][tid];
            s_wcnt[w][tid] = run;
            run += c;
        }
        a.ws_counts[static_cast<int64_t>(b) * R + tid] = static_cast<int32_t>(run);
    }

    if (!grid_barrier_ticket(a.ws_barrier, static_cast<uint32_t>(a.G), 0u, a.barrier_limit_ns)) {
        if (tid == 0)
            atomicOr(a.out.status, MOE_DEV_TIMEOUT);
        return;
    }

    // ---- phase 2a: earlier-block prefix and total per rank (P threads per rank)
    const int P = DEDUP_THREADS / R;
    if (tid < P * R) {
        const int r = tid % R, part = tid / R;
        int32_t pre = 0, tot = 0;
        for (int bb0 = part; bb0 < a.G; bb0 += 16 * P) {
            int32_t c[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int bb = bb0 + u * P;
                c[u] = bb < a.G ? __ldcg(a.ws_counts + static_cast<int64_t>(bb) * R + r) : 0;
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                tot += c[u];
                pre += (bb0 + u * P < b) ? c[u] : 0;
            }
        }
        s_part[0][tid] = pre;
        s_part[1][tid] = tot;
    }
    __syncthreads();
    if (warp == 0) {
        int32_t pre = 0, tot = 0;
        if (lane < R)
            for (int part = 0; part < P; ++part) {
                pre += s_part[0][part * R + lane];
                tot += s_part[1][part * R + lane];
            }
        int32_t inc = tot; // exclusive scan of the rank totals over the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t n = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o)
                inc += n;
        }
        if (lane < R) {
            s_pre[lane] = pre;
            s_off[lane] = inc - tot;
        }
        if (lane == R - 1)
            s_off[R] = inc;
        if (b == 0 && lane < R) {
            a.out.num_tokens_per_rank[lane] = tot;
            a.out.recv_rank_offsets[lane] = inc - tot;
            if (lane == R - 1) {
                a.out.recv_rank_offsets[R] = inc;
                *a.out.num_recv = inc;
            }
        }
    }
    __syncthreads();

    // ---- phase 2b: the row of each of this lane's (token, rank) pairs; the
    // per-row receive data is written row by row by dedup_fill_kernel
    const moe_dedup_t &o = a.out;
#pragma unroll
    for (int u = 0; u < TPL; ++u) {
        const int64_t t = base + u * 32 + lane;
        for (int r = 0; r < R; ++r) {
            const bool in = (mask[u] >> r) & 1u;
            const uint32_t bal = __ballot_sync(0xffffffffu, in);
            const int32_t row = in ? s_off[r] + s_pre[r] + static_cast<int32_t>(s_wcnt[warp][r]) + __popc(bal & lt)
                                   : -1;
            __syncwarp();
            if (lane == 0)
                s_wcnt[warp][r] += __popc(bal);
            __syncwarp();
            if (t >= a.N)
                continue;
            o.token_rank_row[t * R + r] = row;
            o.is_token_in_rank[t * R + r] = in ? 1 : 0;
            if (!in)
                continue;
            if (row >= a.recv_max) { // cannot happen for consistent inputs; never write out of bounds
                atomicOr(o.status, MOE_DEV_ROW_RANGE);
                continue;
            }
            o.recv_src_token[row] = static_cast<int32_t>(t);
        }
    }
}

// Per receive row (one thread each): rank from recv_rank_offsets, then the
// rank-local top-k ids and weights of the source token, the multihot map and
// its probs; tail rows get -1 / 0 and pad 1. Rows past num_recv are tail rows;
// recv_src_token of those rows is written here too.
struct DedupFillArgs {
    const int32_t *phys_idx; // [N, k]
    const int32_t *dest_row; // [N, k]
    const float *probs;      // [N, k] or null
    int64_t recv_max;
    int32_t k, R, E_loc;
    moe_dedup_t out;
};

__global__ void __launch_bounds__(256) dedup_fill_kernel(DedupFillArgs a)
{
    __shared__ int32_t s_roff[MOE_MAX_DEDUP_RANKS + 1];
    pdl_trigger();
    pdl_wait();
    const moe_dedup_t &o = a.out;
    if (threadIdx.x <= a.R)
        s_roff[threadIdx.x] = __ldg(o.recv_rank_offsets + threadIdx.x);
    __syncthreads();
    const int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (w >= a.recv_max)
        return;
    const int32_t num_recv = s_roff[a.R];
    const int k = a.k, E_loc = a.E_loc;
    int32_t t = -1, r = -1;
    if (w < num_recv) {
        t = __ldg(o.recv_src_token + w);
        r = 0;
        while (r + 1 < a.R && s_roff[r + 1] <= w)
            ++r;
    } else {
        o.recv_src_token[w] = -1;
    }
    o.recv_pad_mask[w] = t < 0 ? 1 : 0;
    uint8_t *map_row = o.recv_routing_map + w * E_loc;
    float *prob_row = o.recv_probs + w * E_loc;
    // the token's slots, eight at a time, all loads of a batch in flight together
    // (the first batch before the row is zeroed, so that nothing waits in between)
    constexpr int B = 8;
    int32_t dj[B], qj[B];
    float wj[B];
    auto load_batch = [&](int j0) {
#pragma unroll
        for (int u = 0; u < B; ++u) {
            const int j = j0 + u;
            dj[u] = -1;
            qj[u] = -1;
            wj[u] = 0.0f;
            if (t >= 0 && j < k) {
                const int64_t s = static_cast<int64_t>(t) * k + j;
                dj[u] = __ldg(a.dest_row + s);
                qj[u] = __ldg(a.phys_idx + s);
                if (a.probs != nullptr)
                    wj[u] = __ldg(a.probs + s);
            }
        }
    };
    load_batch(0);
    if ((E_loc & 15) == 0) {
        for (int c = 0; c < E_loc; c += 16)
            *reinterpret_cast<uint4 *>(map_row + c) = make_uint4(0, 0, 0, 0);
        for (int c = 0; c < E_loc; c += 4)
            *reinterpret_cast<float4 *>(prob_row + c) = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
        for (int c = 0; c < E_loc; ++c) {
            map_row[c] = 0;
            prob_row[c] = 0.0f;
        }
    }
    for (int j0 = 0; j0 < k; j0 += B) {
        if (j0 > 0)
            load_batch(j0);
#pragma unroll
        for (int u = 0; u < B; ++u) {
            const int j = j0 + u;
            if (j >= k)
                break;
            int32_t local = -1;
            float wt = 0.0f;
            if (dj[u] >= 0 && qj[u] >= 0 && qj[u] / E_loc == r) {
                local = qj[u] - r * E_loc;
                wt = wj[u];
                map_row[local] = 1;
                prob_row[local] = wt;
            }
            o.recv_topk_idx[w * k + j] = local;
            o.recv_topk_weights[w * k + j] = wt;
        }
    }
}

// Receiver-side partials, token-major: one thread per 16-byte column chunk of
// one token. Lane j holds slot j's row, prob and owning rank (from the layout's
// rank offsets). The kept slots are put in (rank, slot) order with a few warp
// ballots; the chunks are loaded in that order, all in flight at once, and
// folded with one accumulator that is stored as rank r's partial and reset
// whenever the rank changes, so each rank's slots accumulate in ascending slot
// order from +0 and every multiply-add is issued once. Every kept row is read
// once and every partial written once. The trailing `zero_blocks` CTAs zero
// the receive rows past num_recv.
struct DedupCombineArgs {
    const uint4 *y;                // [rows_max, V] expert outputs in send-buffer order
    const int32_t *dest_row;       // [N, k]
    const float *probs;            // [N, k] or null (unit weights)
    const int32_t *rank_offsets;   // [R+1] of the layout
    const int32_t *token_rank_row; // [N, R]
    const int32_t *num_recv;       // [1]
    uint4 *partial;                // [recv_max, V]
    uint32_t *status;
    int64_t N;
    int64_t recv_max;
    int64_t rows_max;
    int32_t k, R, V, nchunks;
    int64_t token_blocks; // N * nchunks; the blocks after them zero the tail
};

__device__ __forceinline__ void dedup_zero_tail(const DedupCombineArgs &a, int64_t worker, int64_t nworkers)
{
    const int64_t first = __ldg(a.num_recv);
    const uint4 z = make_uint4(0, 0, 0, 0);
    const int64_t total = (a.recv_max - first) * a.V;
    for (int64_t i = worker; i < total; i += nworkers)
        st_u4(a.partial + first * a.V + i, z);
}

// Lane j < k: position of kept slot j in (rank, slot) order, from one ballot per
// rank; dropped slots (rank R) come last. Returns the number of kept slots.
__device__ __forceinline__ int dedup_slot_order(int32_t rank, int k, int R, int lane, int32_t &pos)
{
    const uint32_t lt = (1u << lane) - 1u;
    int before = 0; // kept slots of lower ranks
    pos = 0;
    for (int r = 0; r < R; ++r) {
        const uint32_t m = __ballot_sync(0xffffffffu, lane < k && rank == r);
        if (rank == r)
            pos = before + __popc(m & lt);
        before += __popc(m);
    }
    return before;
}

template <int K> // top-k at compile time (1..8); 0 = runtime k <= 32, slots taken eight at a time
__global__ void __launch_bounds__(256, 4) dedup_combine_local_kernel(DedupCombineArgs a)
{
    pdl_trigger();
    pdl_wait();
    if (blockIdx.x >= a.token_blocks) {
        dedup_zero_tail(a, (blockIdx.x - a.token_blocks) * blockDim.x + threadIdx.x,
                        (gridDim.x - a.token_blocks) * blockDim.x);
        return;
    }
    // tokens last first: the send rows the permute wrote last are still in L2
    const int64_t tb = blockIdx.x / a.nchunks;
    const int c = static_cast<int>(blockIdx.x - tb * a.nchunks);
    const int64_t t = a.N - 1 - tb;
    const int v = c * blockDim.x + threadIdx.x;
    const int lane = threadIdx.x & 31;
    const int k = K > 0 ? K : a.k;
    const int R = a.R;
    // slot metadata: row, prob and owning rank (R for a dropped slot)
    int32_t d = -1;
    float p = 0.0f;
    if (lane < k) {
        d = __ldg(a.dest_row + t * k + lane);
        p = a.probs != nullptr ? __ldg(a.probs + t * k + lane) : 1.0f;
        if (d < -1 || d >= a.rows_max) {
            atomicOr(a.status, MOE_DEV_ROW_RANGE);
            d = -1;
        }
    }
    const int32_t rank_end = lane < R ? __ldg(a.rank_offsets + lane + 1) : INT32_MAX;
    const int32_t my_row = lane < R ? __ldg(a.token_rank_row + t * R + lane) : -1;
    int32_t rank = 0; // ranks whose rows end at or before this slot's row
    for (int r = 0; r < R; ++r)
        rank += (d >= __shfl_sync(0xffffffffu, rank_end, r)) ? 1 : 0;
    if (d < 0)
        rank = R;
    int32_t pos;
    const int kept = dedup_slot_order(rank, k, R, lane, pos);
    // lane i < kept takes the row, prob and rank of the slot at position i
    int32_t at = 0;
    for (int j = 0; j < k; ++j) {
        const int32_t pj = __shfl_sync(0xffffffffu, pos, j);
        const bool keptj = __shfl_sync(0xffffffffu, rank, j) < R;
        at = (keptj && pj == lane) ? j : at;
    }
    const int32_t d_at = __shfl_sync(0xffffffffu, d, at);
    const float p_at = __shfl_sync(0xffffffffu, p, at);
    const int32_t r_at = __shfl_sync(0xffffffffu, rank, at);
    // bit i: position i ends a rank's run (the last kept slot, or the next one has another rank)
    const int32_t r_next = __shfl_down_sync(0xffffffffu, r_at, 1);
    const uint32_t ends = __ballot_sync(0xffffffffu, lane < kept && (lane == kept - 1 || r_next != r_at));
    const bool active = v < a.V;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
        acc[e] = 0.0f;
    constexpr int STEP = K > 0 ? K : 8;
    for (int i0 = 0; i0 < kept; i0 += STEP) {
        uint4 yi[STEP];
#pragma unroll
        for (int u = 0; u < STEP; ++u) {
            const int32_t di = __shfl_sync(0xffffffffu, d_at, (i0 + u) & 31);
            if (i0 + u < kept && active)
                yi[u] = ld_stream_u4(a.y + static_cast<int64_t>(di) * a.V + v);
        }
#pragma unroll
        for (int u = 0; u < STEP; ++u) {
            const int i = i0 + u;
            if (i >= kept)
                break; // uniform over the warp
            const float pi = __shfl_sync(0xffffffffu, p_at, i);
            if (active)
                fma8(acc, pi, yi[u]);
            if ((ends >> i) & 1u) { // store rank r's partial and start the next rank from +0
                const int32_t r = __shfl_sync(0xffffffffu, r_at, i);
                const int32_t row = __shfl_sync(0xffffffffu, my_row, r);
                if (active) {
                    if (row < 0 || row >= a.recv_max) // a view of another layout
                        atomicOr(a.status, MOE_DEV_ROW_RANGE);
                    else
                        st_u4(a.partial + static_cast<int64_t>(row) * a.V + v, pack8(acc));
                }
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    acc[e] = 0.0f;
            }
        }
    }
}

} // namespace moert
