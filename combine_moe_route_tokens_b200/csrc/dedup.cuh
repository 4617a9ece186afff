// dedup.cuh — the DeepEP-style token-dedup view and the receiver-side combine.
//
// Megatron MORI page: the MORI dispatcher follows the DeepEP contract — each
// token is sent once to every rank that owns one of its experts; the receiver
// gets rank-local top-k ids with -1 sentinels and receiver-side weights, and
// _indices_to_multihot turns those into a [tokens, local experts] routing map
// with probs. The combine comes back in two levels: every rank reduces its
// local slots per received token, the sender sums the partials over ranks.
//
// dedup_count_kernel (blocks in ticket order, any grid size): each (token,
//            rank) pair's position among the tokens rank r receives, from
//            per-warp ballots and a decoupled look-back over the blocks' per-rank
//            counts (rows are rank-major and token-ascending);
// dedup_fill_kernel (one thread per pair and per receive row): the rank
//            offsets from the per-rank totals, the receive rows and their data
//            (ids, weights, multihot map, probs), the tail rows.
#pragma once

#include <cstdint>

#include "moe_rt.h"
#include "combine.cuh"
#include "lookback.cuh"
#include "ptx.cuh"

namespace moert {

constexpr int DEDUP_THREADS = 256;
constexpr int DEDUP_WARPS = DEDUP_THREADS / 32;
constexpr int DEDUP_MAX_BLOCKS = 128;
constexpr int DEDUP_MAX_TPL = 8; // tokens per lane kept in registers
constexpr int LB_CHUNK_DEDUP = 16; // predecessors one thread reads per look-back round

struct DedupArgs {
    const int32_t *phys_idx; // [N, k]
    const int32_t *dest_row; // [N, k]
    const float *probs;      // [N, k] or null
    int64_t N;
    int64_t recv_max;
    int32_t k, R, E_loc;
    int32_t G;                     // count blocks
    unsigned long long *ws_ticket; // ticket word (lookback.cuh)
    unsigned long long *ws_flags;  // [G][R] look-back words
    uint64_t wait_limit_ns;
    moe_dedup_t out;
};

__device__ __forceinline__ uint32_t dedup_lanemask_lt()
{
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// The count pass: blocks in ticket order (lookback.cuh). Each lane builds, for
// its tokens, the bit set of ranks holding a kept slot; per warp and rank the
// tokens are counted with __ballot_sync; per rank the block publishes its count
// and looks back over its predecessors (the same decoupled look-back as the
// dispatch layout, R columns). Every (token, rank) pair gets its position among
// rank r's tokens (earlier blocks + earlier warps + earlier lanes), written into
// token_rank_row as a rank-relative row; dedup_fill_kernel adds the rank's offset.
template <int TPL> // tokens per lane; a warp owns 32 * TPL consecutive tokens
__global__ void __launch_bounds__(DEDUP_THREADS) dedup_count_kernel(DedupArgs a)
{
    constexpr int W = LB_CHUNK_DEDUP;
    __shared__ uint32_t s_wcnt[DEDUP_WARPS][MOE_MAX_DEDUP_RANKS]; // per-warp counts, then exclusive prefixes
    __shared__ uint32_t s_agg[MOE_MAX_DEDUP_RANKS], s_excl[MOE_MAX_DEDUP_RANKS], s_state[MOE_MAX_DEDUP_RANKS];
    __shared__ uint32_t s_psum[DEDUP_THREADS], s_pflag[DEDUP_THREADS];
    __shared__ uint32_t s_vb, s_epoch, s_timeout;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int R = a.R, k = a.k;
    const int P = DEDUP_THREADS / R > 32 ? 32 : DEDUP_THREADS / R; // look-back parts per rank
    const uint32_t lt = dedup_lanemask_lt();

    for (int i = tid; i < DEDUP_WARPS * MOE_MAX_DEDUP_RANKS; i += DEDUP_THREADS)
        (&s_wcnt[0][0])[i] = 0;
    if (tid == 0) { // drawn before the wait, as in the dispatch layout's count pass
        uint32_t vb, epoch;
        lb_take_ticket(a.ws_ticket, static_cast<uint32_t>(a.G), &vb, &epoch);
        s_vb = vb;
        s_epoch = epoch;
        s_timeout = 0;
    }
    pdl_wait();
    __syncthreads();
    pdl_trigger();
    const uint32_t vb = s_vb, epoch = s_epoch;
    if (vb >= static_cast<uint32_t>(a.G)) { // two calls shared the workspace at once: stay inside it
        if (tid == 0)
            atomicOr(a.out.status, MOE_DEV_TIMEOUT);
        return;
    }
    const int64_t base = (static_cast<int64_t>(vb) * DEDUP_WARPS + warp) * (32 * TPL);

    // ---- rank sets of this lane's tokens, per-warp per-rank counts
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
    unsigned long long *my_words = a.ws_flags + static_cast<int64_t>(vb) * R;
    if (tid < R) {
        uint32_t run = 0;
#pragma unroll
        for (int w = 0; w < DEDUP_WARPS; ++w) {
            const uint32_t c = s_wcnt[w][tid];
            s_wcnt[w][tid] = run;
            run += c;
        }
        s_agg[tid] = run;
        s_excl[tid] = 0;
        s_state[tid] = 0;
        st_relaxed_u64(my_words + tid, lb_word(epoch, vb == 0 ? LB_INCL : LB_AGG, run, false));
    }
    __syncthreads();

    // ---- decoupled look-back over the R rank columns
    if (vb > 0) {
        int32_t hi = static_cast<int32_t>(vb) - 1;
        for (;;) {
            if (tid < P * R) {
                const int r = tid % R, part = tid / R;
                if (!(s_state[r] & 1u)) {
                    const LbChunk c = lb_scan_chunk<W>(a.ws_flags, R, r, hi - part * W, epoch, a.wait_limit_ns);
                    s_psum[tid] = c.sum;
                    s_pflag[tid] = c.closed ? 1u : 0u;
                    if (c.timeout)
                        s_timeout = 1;
                }
            }
            __syncthreads();
            int more = 0;
            if (tid < R && !(s_state[tid] & 1u)) {
                uint32_t sum = s_excl[tid];
                for (int part = 0; part < P; ++part) {
                    sum += s_psum[part * R + tid];
                    if (s_pflag[part * R + tid]) {
                        s_state[tid] = 1u;
                        break;
                    }
                }
                s_excl[tid] = sum;
                if (s_state[tid] & 1u)
                    st_relaxed_u64(my_words + tid, lb_word(epoch, LB_INCL, sum + s_agg[tid], false));
                else
                    more = 1;
            }
            hi -= P * W;
            if (!__syncthreads_or(more))
                break;
        }
        if (tid == 0 && s_timeout)
            atomicOr(a.out.status, MOE_DEV_TIMEOUT);
    }

    // ---- each (token, rank) pair's position among rank r's tokens
    const moe_dedup_t &o = a.out;
#pragma unroll
    for (int u = 0; u < TPL; ++u) {
        const int64_t t = base + u * 32 + lane;
        for (int r = 0; r < R; ++r) {
            const bool in = (mask[u] >> r) & 1u;
            const uint32_t bal = __ballot_sync(0xffffffffu, in);
            const int32_t rel = in ? static_cast<int32_t>(s_excl[r] + s_wcnt[warp][r] + __popc(bal & lt)) : -1;
            __syncwarp();
            if (lane == 0)
                s_wcnt[warp][r] += __popc(bal);
            __syncwarp();
            if (t >= a.N)
                continue;
            o.token_rank_row[t * R + r] = rel;
            o.is_token_in_rank[t * R + r] = in ? 1 : 0;
        }
    }
}

// The fill pass: a group of DEDUP_FILL_LANES threads per (rank, token) pair
// (pairs rank-major, so neighbouring groups write neighbouring rows) and per
// receive row. Every CTA turns the last count block's inclusive words (the
// per-rank token totals) into rank offsets; CTA 0 writes them out. A pair that
// sends its token to rank r turns its rank-relative row into the receive row w
// and writes that row's data: the source token, the rank-local top-k ids and
// weights, the multihot map with its probs (Megatron MORI page:
// _indices_to_multihot), pad 0. Each lane of the group holds some of the
// token's slots; the map and prob rows are split among the lanes, each lane
// builds its part from the slots (shuffled within the group) and stores it
// once. Rows past num_recv are tail rows: token -1, ids -1, weights / map /
// probs 0, pad 1.
constexpr int DEDUP_FILL_LANES = 8;
constexpr int DEDUP_FILL_THREADS = 256;

struct DedupFillArgs {
    const int32_t *phys_idx; // [N, k]
    const int32_t *dest_row; // [N, k]
    const float *probs;      // [N, k] or null
    int64_t N;
    int64_t recv_max;
    int32_t k, R, E_loc, G;
    const unsigned long long *ws_ticket;
    const unsigned long long *ws_flags;
    moe_dedup_t out;
};

// Row w's ids, weights, map and probs from the (local id, weight) of the token's
// slots held by the group's lanes (slot j on lane j % LANES, register j / LANES);
// local -1 marks a slot that is not on this rank (or a tail row).
__device__ __forceinline__ void dedup_write_row(const DedupFillArgs &a, int64_t w, const int32_t (&loc)[4],
                                                const float (&wt)[4], int gl, uint32_t gmask)
{
    const moe_dedup_t &o = a.out;
    const int k = a.k, E_loc = a.E_loc;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int j = u * DEDUP_FILL_LANES + gl;
        if (j < k) {
            o.recv_topk_idx[w * k + j] = loc[u];
            o.recv_topk_weights[w * k + j] = wt[u];
        }
    }
    uint8_t *map_row = o.recv_routing_map + w * E_loc;
    float *prob_row = o.recv_probs + w * E_loc;
    const int nu = (k + DEDUP_FILL_LANES - 1) / DEDUP_FILL_LANES;
    // every lane of the group runs the same iterations (the shuffles need all of them)
    if ((E_loc & 3) == 0) { // four entries at a time: one 16-byte prob store and one 4-byte map store
        for (int c0 = 0; c0 < E_loc; c0 += DEDUP_FILL_LANES * 4) {
            const int c = c0 + gl * 4;
            float4 pv = make_float4(0.f, 0.f, 0.f, 0.f);
            uint32_t mv = 0;
            for (int u = 0; u < nu; ++u)
                for (int sl = 0; sl < DEDUP_FILL_LANES; ++sl) {
                    const int32_t x = __shfl_sync(gmask, loc[u], sl, DEDUP_FILL_LANES);
                    const float y = __shfl_sync(gmask, wt[u], sl, DEDUP_FILL_LANES);
                    const int off = x - c;
                    if (x >= 0 && off >= 0 && off < 4) {
                        mv |= 1u << (8 * off);
                        if (off == 0)
                            pv.x = y;
                        else if (off == 1)
                            pv.y = y;
                        else if (off == 2)
                            pv.z = y;
                        else
                            pv.w = y;
                    }
                }
            if (c < E_loc) {
                *reinterpret_cast<float4 *>(prob_row + c) = pv;
                *reinterpret_cast<uint32_t *>(map_row + c) = mv;
            }
        }
    } else {
        for (int c0 = 0; c0 < E_loc; c0 += DEDUP_FILL_LANES) {
            const int c = c0 + gl;
            float pv = 0.0f;
            uint8_t mv = 0;
            for (int u = 0; u < nu; ++u)
                for (int sl = 0; sl < DEDUP_FILL_LANES; ++sl) {
                    const int32_t x = __shfl_sync(gmask, loc[u], sl, DEDUP_FILL_LANES);
                    const float y = __shfl_sync(gmask, wt[u], sl, DEDUP_FILL_LANES);
                    if (x == c) {
                        mv = 1;
                        pv = y;
                    }
                }
            if (c < E_loc) {
                prob_row[c] = pv;
                map_row[c] = mv;
            }
        }
    }
}

__global__ void __launch_bounds__(DEDUP_FILL_THREADS) dedup_fill_kernel(DedupFillArgs a)
{
    __shared__ int32_t s_roff[MOE_MAX_DEDUP_RANKS + 1];
    pdl_trigger();
    pdl_wait(); // the count pass is complete
    const moe_dedup_t &o = a.out;
    const int tid = threadIdx.x, R = a.R, k = a.k;
    if (tid < 32) { // rank totals from the last block's inclusive words, then their exclusive scan
        const uint32_t epoch = static_cast<uint32_t>(__ldcg(a.ws_ticket) >> 32) - 1u;
        int32_t tot = 0;
        bool ok = true;
        if (tid < R) {
            const uint64_t w = __ldcg(a.ws_flags + static_cast<int64_t>(a.G - 1) * R + tid);
            ok = lb_ready(w, epoch) && lb_incl(w);
            tot = ok ? static_cast<int32_t>(lb_value(w)) : 0;
        }
        if (__any_sync(0xffffffffu, !ok) && tid == 0 && blockIdx.x == 0)
            atomicOr(o.status, MOE_DEV_TIMEOUT);
        int32_t inc = tot;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int32_t n = __shfl_up_sync(0xffffffffu, inc, d);
            if (tid >= d)
                inc += n;
        }
        if (tid < R)
            s_roff[tid] = inc - tot;
        if (tid == R - 1)
            s_roff[R] = inc;
        if (blockIdx.x == 0 && tid < R) {
            o.num_tokens_per_rank[tid] = tot;
            o.recv_rank_offsets[tid] = inc - tot;
            if (tid == R - 1) {
                o.recv_rank_offsets[R] = inc;
                *o.num_recv = inc;
            }
        }
    }
    __syncthreads();
    const int gl = tid % DEDUP_FILL_LANES; // lane within the group
    const uint32_t gmask = 0xFFu << ((tid & 31) & ~(DEDUP_FILL_LANES - 1));
    const int64_t g = (static_cast<int64_t>(blockIdx.x) * DEDUP_FILL_THREADS + tid) / DEDUP_FILL_LANES;
    const int32_t num_recv = s_roff[R];
    int32_t loc[4];
    float wt[4];
    if (g < a.recv_max && g >= num_recv) { // a tail row
        if (gl == 0) {
            o.recv_src_token[g] = -1;
            o.recv_pad_mask[g] = 1;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            loc[u] = -1;
            wt[u] = 0.0f;
        }
        dedup_write_row(a, g, loc, wt, gl, gmask);
    }
    if (g >= a.N * R) // uniform over the group
        return;
    // pairs rank-major: neighbouring groups take neighbouring tokens of one rank, whose
    // rows are neighbours too
    const int r = static_cast<int>(g / a.N);
    const int64_t t = g - static_cast<int64_t>(r) * a.N;
    const int64_t pair = t * R + r;
    const int32_t rel = __ldcg(o.token_rank_row + pair);
    if (rel < 0)
        return;
    const int64_t w = static_cast<int64_t>(s_roff[r]) + rel;
    if (w >= a.recv_max || w >= s_roff[r + 1]) { // cannot happen for consistent counts; never write out of bounds
        if (gl == 0) {
            atomicOr(o.status, MOE_DEV_ROW_RANGE);
            o.token_rank_row[pair] = -1;
        }
        return;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) { // this lane's slots of the token: local id on rank r and weight
        const int j = u * DEDUP_FILL_LANES + gl;
        loc[u] = -1;
        wt[u] = 0.0f;
        if (j < k) {
            const int64_t sidx = t * k + j;
            const int32_t d = __ldg(a.dest_row + sidx);
            const int32_t q = __ldg(a.phys_idx + sidx);
            if (d >= 0 && q >= 0 && q / a.E_loc == r) {
                loc[u] = q - r * a.E_loc;
                wt[u] = a.probs != nullptr ? __ldg(a.probs + sidx) : 0.0f;
            }
        }
    }
    if (gl == 0) {
        o.token_rank_row[pair] = static_cast<int32_t>(w);
        o.recv_src_token[w] = static_cast<int32_t>(t);
        o.recv_pad_mask[w] = 0;
    }
    dedup_write_row(a, w, loc, wt, gl, gmask);
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
