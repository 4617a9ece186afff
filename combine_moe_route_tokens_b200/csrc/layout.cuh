// layout.cuh — the dispatch layout in one cooperative launch.
//
// Steps (page citations in moe_rt.h, moe_dispatch_layout):
//   phase 1  per-warp histograms of the logical ids of a contiguous slice of
//            the flattened [N,k] assignments (warp-aggregated with
//            __match_any_sync, one shared-memory add per distinct expert),
//            turned into per-warp exclusive prefixes and a per-block total
//            published to the workspace;
//   barrier  bounded grid barrier (co-residency guaranteed by the
//            cooperative launch);
//   phase 2  every block reads all block totals and so knows, per logical
//            expert, the total count and the count in earlier blocks; it
//            derives the hot-expert placement, physical counts, capacity,
//            the exclusive scan and the rank splits (block 0 publishes them),
//            then re-walks its slice: the stable logical ordinal of an
//            assignment is  earlier blocks + earlier warps + earlier
//            iterations of its warp + earlier lanes with the same id, and the
//            physical ordinal, drop flag and destination row follow in closed
//            form. Finally the pad / tail rows of the row maps are filled.
//
// Closed forms used by phase 2 (equal to counting physical ordinals
// directly, as the CPU definition does): a hot expert's assignment with
// logical ordinal o goes to the master if o is even, else to the replica, at
// physical ordinal o/2; so the master holds ceil(c/2) and the replica
// floor(c/2) of the expert's c assignments.
#pragma once

#include <cstdint>

#include "moe_rt.h"
#include "ptx.cuh"

namespace moert {

constexpr int LAYOUT_THREADS = 512;
constexpr int LAYOUT_WARPS = LAYOUT_THREADS / 32;
constexpr int LAYOUT_MAX_BLOCKS = 128;
constexpr int LAYOUT_MAX_E_LOG = 2048;
constexpr int LAYOUT_ITEMS_PER_BLOCK = 1024; // target slice per block before the block cap

struct LayoutArgs {
    const int32_t *topk_idx;
    const float *topk_probs;
    int64_t NK;
    int64_t rows_max;
    int32_t k, E_log, E, R, E_loc, M, S, num_replicas, C;
    int32_t sub; // assignments per warp slice, a multiple of 32
    int32_t G;   // blocks
    int32_t *ws_counts;   // [G][E_log + 1]: per-block logical totals, last column = error bits
    uint32_t *ws_barrier; // [2]: arrival count, generation
    uint64_t barrier_limit_ns;
    uint32_t barrier_extra; // test hook: extra arrivals the barrier waits for
    moe_layout_t out;
};

// Dynamic shared memory layout, in 32-bit words.
__host__ __device__ inline size_t layout_smem_words(int E_log, int E)
{
    return static_cast<size_t>(LAYOUT_WARPS) * E_log // per-warp counters
           + 3 * static_cast<size_t>(E_log)          // block prefix, totals, placement
           + 2 * static_cast<size_t>(E) + 1;         // physical counts, offsets
}

constexpr int LAYOUT_MAX_PLACEMENT_RANKS = 64;

// Bounded grid barrier with a generation counter; the state words are left
// ready for the next launch (count back to 0) unless the wait ran out.
__device__ __forceinline__ bool layout_grid_barrier(uint32_t *bar, uint32_t target, uint64_t limit_ns)
{
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        volatile uint32_t *vgen = bar + 1;
        const uint32_t gen = *vgen;
        __threadfence();
        const uint32_t arrived = atomicAdd(bar, 1u);
        int ok = 1;
        if (arrived == target - 1) {
            atomicExch(bar, 0u);
            __threadfence();
            atomicAdd(bar + 1, 1u);
        } else {
            const uint64_t t0 = global_timer_ns();
            while (*vgen == gen) {
                __nanosleep(100);
                if (global_timer_ns() - t0 > limit_ns) {
                    ok = 0;
                    break;
                }
            }
        }
        __threadfence();
        s_ok = ok;
    }
    __syncthreads();
    return s_ok != 0;
}

__device__ __forceinline__ uint32_t lanemask_lt()
{
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Hot set and greedy placement for the reroute, computed identically by every
// block from the logical totals. Warp 0 ranks the experts by (count desc, id
// asc) with num_replicas rounds of a warp arg-max; lane 0 then places them.
__device__ void layout_placement(const LayoutArgs &a, const int32_t *s_cnt, int32_t *s_repl, int64_t *s_load,
                                 int32_t *s_free, int32_t *s_hot)
{
    const int lane = threadIdx.x & 31;
    if (threadIdx.x >= 32)
        return;
    for (int r = lane; r < a.R; r += 32) {
        int64_t l = 0;
        for (int i = 0; i < a.M; ++i)
            l += s_cnt[r * a.M + i];
        s_load[r] = l;
        s_free[r] = a.S;
    }
    uint64_t taken = 0; // bit u: expert lane + 32u already chosen (E_log <= 2048)
    for (int h = 0; h < a.num_replicas; ++h) {
        uint64_t best = 0;
        for (int u = 0, e = lane; e < a.E_log; ++u, e += 32) {
            if ((taken >> u) & 1ull)
                continue;
            const uint64_t key =
                (static_cast<uint64_t>(static_cast<uint32_t>(s_cnt[e])) << 32) | static_cast<uint32_t>(~e);
            best = key > best ? key : best;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const uint64_t other = __shfl_xor_sync(0xffffffffu, best, o);
            best = other > best ? other : best;
        }
        const int e = static_cast<int>(~static_cast<uint32_t>(best));
        if ((e & 31) == lane)
            taken |= 1ull << (e >> 5);
        if (lane == 0)
            s_hot[h] = e;
    }
    __syncwarp();
    if (lane == 0) {
        for (int h = 0; h < a.num_replicas; ++h) {
            const int e = s_hot[h];
            const int home = e / a.M;
            int best = -1;
            for (int r = 0; r < a.R; ++r)
                if (r != home && s_free[r] > 0 && (best < 0 || s_load[r] < s_load[best]))
                    best = r;
            if (best < 0)
                best = home;
            const int slot = a.S - s_free[best];
            s_free[best] -= 1;
            s_repl[e] = best * a.E_loc + a.M + slot;
            const int64_t moved = s_cnt[e] / 2;
            s_load[home] -= moved;
            s_load[best] += moved;
        }
    }
}

// Sum of one int32 per thread over the block (all threads must call it).
__device__ __forceinline__ int32_t layout_block_sum(int32_t v, int32_t *s_scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0)
        s_scratch[warp] = v;
    __syncthreads();
    int32_t total = 0;
#pragma unroll
    for (int w = 0; w < LAYOUT_WARPS; ++w)
        total += s_scratch[w];
    return total;
}

__global__ void __launch_bounds__(LAYOUT_THREADS) layout_kernel(LayoutArgs a)
{
    extern __shared__ __align__(16) uint32_t layout_smem[];
    const int E_log = a.E_log, E = a.E;
    uint32_t *wcnt = layout_smem;                                            // [WARPS][E_log]
    int32_t *s_pre = reinterpret_cast<int32_t *>(wcnt + LAYOUT_WARPS * E_log); // [E_log]
    int32_t *s_cnt = s_pre + E_log;                                   // [E_log]
    int32_t *s_repl = s_cnt + E_log;                                  // [E_log]
    int32_t *s_raw = s_repl + E_log;                                  // [E]
    int32_t *s_off = s_raw + E;                                       // [E+1]
    __shared__ int64_t s_load[LAYOUT_MAX_PLACEMENT_RANKS];
    __shared__ int32_t s_free[LAYOUT_MAX_PLACEMENT_RANKS];
    __shared__ int32_t s_hot[LAYOUT_MAX_E_LOG];
    __shared__ int32_t s_scratch[LAYOUT_WARPS];
    __shared__ uint32_t s_err;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x;

    for (int i = tid; i < LAYOUT_WARPS * E_log; i += LAYOUT_THREADS)
        wcnt[i] = 0;
    if (tid == 0)
        s_err = 0;
    __syncthreads();

    const int64_t base = (static_cast<int64_t>(b) * LAYOUT_WARPS + warp) * a.sub;

    // ---- phase 1: per-warp histograms
    uint32_t err = 0;
    for (int it = 0; it < a.sub; it += 32) {
        const int64_t i = base + it + lane;
        int e = -1;
        if (i < a.NK) {
            e = __ldg(a.topk_idx + i);
            if (e < -1 || e >= E_log) {
                err |= MOE_DEV_EXPERT_RANGE;
                e = -1;
            }
        }
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && lane == __ffs(peers) - 1)
            wcnt[warp * E_log + e] += __popc(peers);
        __syncwarp(); // the next update of this counter may come from another lane
    }
    err = __reduce_or_sync(0xffffffffu, err);
    if (lane == 0 && err)
        atomicOr(&s_err, err);
    __syncthreads();
    for (int e = tid; e < E_log; e += LAYOUT_THREADS) {
        uint32_t run = 0;
#pragma unroll
        for (int w = 0; w < LAYOUT_WARPS; ++w) {
            const uint32_t c = wcnt[w * E_log + e];
            wcnt[w * E_log + e] = run;
            run += c;
        }
        a.ws_counts[static_cast<int64_t>(b) * (E_log + 1) + e] = static_cast<int32_t>(run);
    }
    if (tid == 0)
        a.ws_counts[static_cast<int64_t>(b) * (E_log + 1) + E_log] = static_cast<int32_t>(s_err);

    if (!layout_grid_barrier(a.ws_barrier, static_cast<uint32_t>(a.G) + a.barrier_extra, a.barrier_limit_ns)) {
        if (tid == 0)
            atomicOr(a.out.status, MOE_DEV_TIMEOUT);
        return;
    }

    // ---- phase 2a: block prefix and totals per logical expert
    for (int e = tid; e < E_log; e += LAYOUT_THREADS) {
        int32_t pre = 0, tot = 0;
        for (int bb = 0; bb < a.G; ++bb) {
            const int32_t c = __ldcg(a.ws_counts + static_cast<int64_t>(bb) * (E_log + 1) + e);
            pre += bb < b ? c : 0;
            tot += c;
        }
        s_pre[e] = pre;
        s_cnt[e] = tot;
        s_repl[e] = -1;
    }
    if (tid == 0) {
        uint32_t all = 0;
        for (int bb = 0; bb < a.G; ++bb)
            all |= static_cast<uint32_t>(__ldcg(a.ws_counts + static_cast<int64_t>(bb) * (E_log + 1) + E_log));
        s_err = all;
    }
    __syncthreads();

    // ---- phase 2b: hot experts and placement
    if (a.num_replicas > 0)
        layout_placement(a, s_cnt, s_repl, s_load, s_free, s_hot);
    __syncthreads();

    // ---- phase 2c: physical counts, scan, splits
    for (int q = tid; q < E; q += LAYOUT_THREADS) {
        const int r = q / a.E_loc, i = q - r * a.E_loc;
        int32_t c = 0;
        if (i < a.M) {
            const int e = r * a.M + i;
            c = s_cnt[e];
            if (s_repl[e] >= 0)
                c = (c + 1) / 2;
        }
        s_raw[q] = c;
    }
    __syncthreads();
    if (a.num_replicas > 0) {
        for (int e = tid; e < E_log; e += LAYOUT_THREADS)
            if (s_repl[e] >= 0)
                s_raw[s_repl[e]] = s_cnt[e] / 2;
        __syncthreads();
    }
    // exclusive scan of the rows each expert owns (C rows each when capped)
    {
        constexpr int PER = 8; // E <= 4096 = LAYOUT_THREADS * PER
        const int q0 = tid * PER;
        int32_t v[PER];
        int32_t sum = 0;
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int q = q0 + u;
            v[u] = q < E ? (a.C > 0 ? a.C : s_raw[q]) : 0;
            sum += v[u];
        }
        // warp inclusive scan of the per-thread sums
        int32_t inc = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t n = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o)
                inc += n;
        }
        __shared__ int32_t s_warp_tot[LAYOUT_WARPS];
        if (lane == 31)
            s_warp_tot[warp] = inc;
        __syncthreads();
        int32_t wpre = 0;
        for (int w = 0; w < warp; ++w)
            wpre += s_warp_tot[w];
        int32_t run = wpre + inc - sum;
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int q = q0 + u;
            if (q < E)
                s_off[q] = run;
            run += v[u];
        }
        if (tid == LAYOUT_THREADS - 1)
            s_off[E] = run;
    }
    int32_t my_valid = 0, my_kept = 0;
    for (int e = tid; e < E_log; e += LAYOUT_THREADS)
        my_valid += s_cnt[e];
    for (int q = tid; q < E; q += LAYOUT_THREADS)
        my_kept += a.C > 0 ? min(s_raw[q], a.C) : s_raw[q];
    const int32_t total_valid = layout_block_sum(my_valid, s_scratch);
    const int32_t total_kept = layout_block_sum(my_kept, s_scratch);
    __syncthreads();

    const moe_layout_t &o = a.out;
    if (b == 0) {
        for (int e = tid; e < E_log; e += LAYOUT_THREADS) {
            o.counts_logical[e] = s_cnt[e];
            o.placement[e] = s_repl[e];
        }
        for (int q = tid; q < E; q += LAYOUT_THREADS) {
            o.counts_raw[q] = s_raw[q];
            o.tokens_per_expert[q] = a.C > 0 ? min(s_raw[q], a.C) : s_raw[q];
        }
        for (int q = tid; q <= E; q += LAYOUT_THREADS)
            o.expert_offsets[q] = s_off[q];
        for (int r = tid; r < a.R; r += LAYOUT_THREADS) {
            const int32_t split = s_off[(r + 1) * a.E_loc] - s_off[r * a.E_loc];
            o.input_splits[r] = split;
            o.output_splits[r] = split;
            o.rank_offsets[r] = s_off[r * a.E_loc];
        }
        if (tid == 0) {
            o.rank_offsets[a.R] = s_off[E];
            *o.num_rows = s_off[E];
            o.counters[0] = total_valid;
            o.counters[1] = total_kept;
            o.counters[2] = total_valid - total_kept;
            o.counters[3] = static_cast<int32_t>(a.rows_max - total_kept);
            o.counters[4] = s_off[E];
            o.counters[5] = s_off[E];
            o.counters[6] = s_off[E];
            o.counters[7] = static_cast<int32_t>(s_err);
            if (s_err)
                atomicOr(o.status, s_err);
        }
    }

    // ---- phase 2d: per-assignment pass over this warp's slice
    const uint32_t lt = lanemask_lt();
    for (int it = 0; it < a.sub; it += 32) {
        const int64_t i = base + it + lane;
        int e = -1;
        if (i < a.NK) {
            e = __ldg(a.topk_idx + i);
            if (e < -1 || e >= E_log)
                e = -1;
        }
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        const uint32_t wbase = e >= 0 ? wcnt[warp * E_log + e] : 0u;
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1)
            wcnt[warp * E_log + e] = wbase + __popc(peers);
        __syncwarp();
        if (i >= a.NK)
            continue;
        int32_t q = -1, ord = -1, dest = -1;
        uint8_t drop = 0;
        if (e >= 0) {
            const int32_t lo = s_pre[e] + static_cast<int32_t>(wbase) + __popc(peers & lt);
            const int32_t master = (e / a.M) * a.E_loc + (e % a.M);
            const int32_t repl = s_repl[e];
            if (repl >= 0) {
                q = (lo & 1) ? repl : master;
                ord = lo >> 1;
            } else {
                q = master;
                ord = lo;
            }
            drop = (a.C > 0 && ord >= a.C) ? 1 : 0;
            if (!drop)
                dest = s_off[q] + ord;
            if (dest >= a.rows_max) { // cannot happen for consistent counts; never write out of bounds
                atomicOr(o.status, MOE_DEV_ROW_RANGE);
                dest = -1;
            }
        }
        o.phys_idx[i] = q;
        o.ordinal[i] = ord;
        o.drop_mask[i] = drop;
        o.dest_row[i] = dest;
        if (dest >= 0) {
            const int32_t t = static_cast<int32_t>(i / a.k);
            o.row_token[dest] = t;
            o.row_slot[dest] = static_cast<int32_t>(i - static_cast<int64_t>(t) * a.k);
            o.row_prob[dest] = a.topk_probs != nullptr ? __ldg(a.topk_probs + i) : 0.0f;
            o.row_local_expert[dest] = q % a.E_loc;
            o.pad_mask[dest] = 0;
        }
        if (o.local_topk != nullptr) {
            const int owner = dest >= 0 ? q / a.E_loc : -1;
            for (int r = 0; r < a.R; ++r)
                o.local_topk[static_cast<int64_t>(r) * a.NK + i] = (r == owner) ? q - r * a.E_loc : -1;
        }
    }

    // ---- phase 2e: pad rows (capacity slots left empty) and the tail
    const int64_t stride = static_cast<int64_t>(a.G) * LAYOUT_THREADS;
    const int64_t start = a.C > 0 ? 0 : s_off[E];
    for (int64_t row = start + static_cast<int64_t>(b) * LAYOUT_THREADS + tid; row < a.rows_max; row += stride) {
        bool pad = true;
        if (a.C > 0) {
            const int32_t q = static_cast<int32_t>(row / a.C);
            const int32_t slot = static_cast<int32_t>(row - static_cast<int64_t>(q) * a.C);
            pad = slot >= min(s_raw[q], a.C);
        }
        if (pad) {
            o.row_token[row] = -1;
            o.row_slot[row] = -1;
            o.row_local_expert[row] = -1;
            o.row_prob[row] = 0.0f;
            o.pad_mask[row] = 1;
        }
    }
}

} // namespace moert
