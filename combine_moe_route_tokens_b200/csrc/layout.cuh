// layout.cuh — the dispatch layout in one cooperative launch.
//
// Steps (page citations in moe_rt.h, moe_dispatch_layout):
//   phase 1  each warp loads its contiguous slice of the flattened [N,k]
//            assignments (ids and probs, kept in registers), ranks every
//            assignment among the earlier ones of its warp with the same id
//            (__match_any_sync + popc, one shared-memory counter update per
//            distinct id), then the block turns its per-warp counts into
//            per-warp exclusive prefixes and publishes its per-expert total;
//   barrier  bounded grid barrier (acquire/release atomics; co-residency is
//            guaranteed by the cooperative launch);
//   phase 2  every block reads all block totals (16-byte loads, up to eight in
//            flight per thread), so it knows per logical expert the total count and the count in
//            earlier blocks; it derives the hot-expert placement, physical
//            counts, capacity, the exclusive scan and the rank splits (block 0
//            publishes them); then, with no further global reads, it writes
//            every per-assignment and per-row output: the stable logical
//            ordinal is  earlier blocks + earlier warps + earlier items of the
//            same warp, and the physical ordinal, drop flag and row follow in
//            closed form. Finally the pad / tail rows of the row maps.
//
// Closed forms used by phase 2 (equal to counting physical ordinals
// directly, as the CPU definition does): a hot expert's assignment with
// logical ordinal o goes to the master if o is even, else to the replica, at
// physical ordinal o/2; so the master holds ceil(c/2) and the replica
// floor(c/2) of the expert's c assignments.
#pragma once

#include <cstdint>
#include <type_traits>

#include "moe_rt.h"
#include "grid_barrier.cuh"
#include "ptx.cuh"

namespace moert {

constexpr int LAYOUT_THREADS = 512;
constexpr int LAYOUT_WARPS = LAYOUT_THREADS / 32;
constexpr int LAYOUT_MAX_BLOCKS = 128;
constexpr int LAYOUT_MAX_E_LOG = 2048;
constexpr int LAYOUT_MAX_PLACEMENT_RANKS = 64;
constexpr int LAYOUT_MAX_IPL = 8; // assignments per lane held in registers
constexpr int LAYOUT_ITEMS_PER_BLOCK = 512; // target slice per block before the block cap

struct LayoutArgs {
    const int32_t *topk_idx; // [N, k]
    const float *topk_probs; // [N, k] or null
    int64_t NK;
    int64_t rows_max;
    int32_t k, E_log, E, R, E_loc, M, S, num_replicas, C;
    int32_t A;       // row alignment (1 = none)
    int32_t T;       // TP folding peers (1 = none)
    int32_t tp_rank; // this peer
    int32_t C_local; // capacity slots per expert in this peer's buffer: ceil(C / T)
    int32_t sub; // assignments per warp slice, a multiple of 32
    int32_t G;   // blocks
    int32_t *ws_counts;   // [G][E_log]: per-block logical totals
    uint32_t *ws_barrier; // [3]: arrival ticket word, (unused), error bits of this call
    uint64_t barrier_limit_ns;
    uint32_t barrier_extra; // test hook: extra arrivals the barrier waits for
    moe_layout_t out;
};

// Dynamic shared memory, in 32-bit words.
__host__ __device__ inline size_t layout_smem_words(int E_log, int E)
{
    return static_cast<size_t>(LAYOUT_WARPS) * E_log // per-warp counters, then prefixes
           + 3 * static_cast<size_t>(E_log)          // block prefix, totals, placement
           + 2 * static_cast<size_t>(E) + 1;         // physical counts, offsets
}

// Rows this peer keeps of an expert with `raw` assignments: the capacity-kept
// ones (min(raw, C)) whose ordinal is congruent to tp_rank modulo T.
__device__ __forceinline__ int32_t layout_local_tokens(const LayoutArgs &a, int32_t raw)
{
    const int32_t t = a.C > 0 ? min(raw, a.C) : raw;
    if (a.T == 1) // no folding: skip the division
        return t;
    return t > a.tp_rank ? (t - a.tp_rank + a.T - 1) / a.T : 0;
}

__device__ __forceinline__ uint32_t lanemask_lt()
{
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Hot set with the counts held in registers (E_log <= 32 * CPL): lane l holds
// experts l, l + 32, ...; each round takes the warp's largest count (equal
// counts: the lowest id, from a second reduction) and clears it.
template <int CPL>
__device__ __forceinline__ void layout_hot_set_regs(const LayoutArgs &a, const int32_t *s_cnt, int32_t *s_hot)
{
    const int lane = threadIdx.x & 31;
    uint32_t c[CPL];
#pragma unroll
    for (int u = 0; u < CPL; ++u) {
        const int e = u * 32 + lane;
        c[u] = e < a.E_log ? static_cast<uint32_t>(s_cnt[e]) + 1u : 0u; // +1: 0 marks "none"
    }
    for (int h = 0; h < a.num_replicas; ++h) {
        uint32_t best = 0;
        int bu = 0;
#pragma unroll
        for (int u = 0; u < CPL; ++u) {
            const bool better = c[u] > best;
            best = better ? c[u] : best;
            bu = better ? u : bu;
        }
        const uint32_t wmax = __reduce_max_sync(0xffffffffu, best);
        const uint32_t cand = (best == wmax && best != 0u) ? ~static_cast<uint32_t>(bu * 32 + lane) : 0u;
        const int e = static_cast<int>(~__reduce_max_sync(0xffffffffu, cand));
        const bool mine = (e & 31) == lane;
#pragma unroll
        for (int u = 0; u < CPL; ++u)
            c[u] = (mine && u == (e >> 5)) ? 0u : c[u];
        if (lane == 0)
            s_hot[h] = e;
    }
}

// Hot set for any E_log <= 2048: the counts are read from shared memory each round.
__device__ __forceinline__ void layout_hot_set_smem(const LayoutArgs &a, const int32_t *s_cnt, int32_t *s_hot)
{
    const int lane = threadIdx.x & 31;
    uint64_t taken = 0; // bit u: expert lane + 32u already chosen (E_log <= 2048)
    for (int h = 0; h < a.num_replicas; ++h) {
        uint32_t best = 0;
        int be = -1;
        for (int u = 0, e = lane; e < a.E_log; ++u, e += 32) {
            const uint32_t c = static_cast<uint32_t>(s_cnt[e]) + 1u; // +1: 0 marks "none"
            if (!((taken >> u) & 1ull) && c > best) {
                best = c;
                be = e;
            }
        }
        const uint32_t wmax = __reduce_max_sync(0xffffffffu, best);
        const uint32_t cand = (best == wmax && be >= 0) ? ~static_cast<uint32_t>(be) : 0u;
        const int e = static_cast<int>(~__reduce_max_sync(0xffffffffu, cand));
        if ((e & 31) == lane)
            taken |= 1ull << (e >> 5);
        if (lane == 0)
            s_hot[h] = e;
    }
}

// Hot experts and their replica placement, by warp 0 (readings of the UltraEP
// page): the num_replicas largest logical counts, lowest id on ties; in that
// order: the least-loaded rank (lowest id on ties) among the ranks other than
// the master's that still have a free replica slot, else the master's own
// rank; then floor(c/2) of load moves from the master's rank to it.
__device__ void layout_placement(const LayoutArgs &a, const int32_t *s_cnt, int32_t *s_repl, int32_t *s_hot)
{
    const int lane = threadIdx.x & 31;
    if (threadIdx.x >= 32)
        return;
    if (a.E_log <= 32)
        layout_hot_set_regs<1>(a, s_cnt, s_hot);
    else if (a.E_log <= 64)
        layout_hot_set_regs<2>(a, s_cnt, s_hot);
    else if (a.E_log <= 128)
        layout_hot_set_regs<4>(a, s_cnt, s_hot);
    else if (a.E_log <= 256)
        layout_hot_set_regs<8>(a, s_cnt, s_hot);
    else
        layout_hot_set_smem(a, s_cnt, s_hot);
    __syncwarp();
    // lane owns ranks lane and lane + 32
    uint32_t load0 = 0, load1 = 0;
    int free0 = a.S, free1 = a.S;
    if (lane < a.R)
        for (int i = 0; i < a.M; ++i)
            load0 += static_cast<uint32_t>(s_cnt[lane * a.M + i]);
    if (lane + 32 < a.R)
        for (int i = 0; i < a.M; ++i)
            load1 += static_cast<uint32_t>(s_cnt[(lane + 32) * a.M + i]);
    // lane h < 32 holds hot expert h, its home rank and the load it moves, so each
    // round's dependent chain starts at the reductions
    int hot_e = 0, hot_home = 0;
    uint32_t hot_moved = 0;
    if (lane < a.num_replicas) {
        hot_e = s_hot[lane];
        hot_home = hot_e / a.M;
        hot_moved = static_cast<uint32_t>(s_cnt[hot_e]) / 2u;
    }
    for (int h = 0; h < a.num_replicas; ++h) {
        int e, home;
        uint32_t moved;
        if (h < 32) { // uniform over the warp
            e = __shfl_sync(0xffffffffu, hot_e, h);
            home = __shfl_sync(0xffffffffu, hot_home, h);
            moved = __shfl_sync(0xffffffffu, hot_moved, h);
        } else {
            e = s_hot[h];
            home = e / a.M;
            moved = static_cast<uint32_t>(s_cnt[e]) / 2u;
        }
        const uint32_t c0 = (lane < a.R && free0 > 0 && lane != home) ? load0 : 0xFFFFFFFFu;
        const uint32_t c1 = (lane + 32 < a.R && free1 > 0 && lane + 32 != home) ? load1 : 0xFFFFFFFFu;
        const uint32_t m = __reduce_min_sync(0xffffffffu, min(c0, c1));
        int best;
        if (m == 0xFFFFFFFFu) {
            best = home;
        } else {
            const uint32_t r0 = c0 == m ? static_cast<uint32_t>(lane) : 0xFFFFFFFFu;
            const uint32_t r1 = c1 == m ? static_cast<uint32_t>(lane + 32) : 0xFFFFFFFFu;
            best = static_cast<int>(__reduce_min_sync(0xffffffffu, min(r0, r1)));
        }
        const int owner_free = __shfl_sync(0xffffffffu, best < 32 ? free0 : free1, best & 31);
        const int slot = a.S - owner_free;
        if (lane == (best & 31)) {
            if (best < 32) {
                free0 -= 1;
                load0 += moved;
            } else {
                free1 -= 1;
                load1 += moved;
            }
        }
        if (lane == (home & 31)) {
            if (home < 32)
                load0 -= moved;
            else
                load1 -= moved;
        }
        if (lane == 0)
            s_repl[e] = best * a.E_loc + a.M + slot;
    }
}

template <int IPL> // IPL > 0: each lane keeps IPL assignments in registers (sub = 32 * IPL); 0: any sub
__global__ void __launch_bounds__(LAYOUT_THREADS, 1) layout_kernel(LayoutArgs a)
{
    extern __shared__ __align__(16) uint32_t layout_smem[];
    const int E_log = a.E_log, E = a.E;
    uint32_t *wcnt = layout_smem;                                                // [WARPS][E_log]
    int32_t *s_pre = reinterpret_cast<int32_t *>(wcnt + LAYOUT_WARPS * E_log); // [E_log]
    int32_t *s_cnt = s_pre + E_log;                                            // [E_log]
    int32_t *s_repl = s_cnt + E_log;                                           // [E_log]
    int32_t *s_raw = s_repl + E_log;                                           // [E]
    int32_t *s_off = s_raw + E;                                                // [E+1]
    __shared__ int32_t s_hot[LAYOUT_MAX_E_LOG];
    __shared__ __align__(16) int32_t s_part[2][4 * LAYOUT_THREADS]; // phase 2a partial sums
    __shared__ int32_t s_wsum[4][LAYOUT_WARPS];
    __shared__ uint32_t s_err;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x;
    const uint32_t lt = lanemask_lt();

    for (int i = tid; i < LAYOUT_WARPS * E_log; i += LAYOUT_THREADS)
        wcnt[i] = 0;
    if (tid == 0)
        s_err = 0;
    __syncthreads();

    const int64_t base = (static_cast<int64_t>(b) * LAYOUT_WARPS + warp) * a.sub;
    uint32_t *my_cnt = wcnt + warp * E_log;
    pdl_trigger();
    pdl_wait(); // inputs and the workspace may have been written by the previous kernel

    // ---- phase 1: load the slice, rank within the warp, per-warp counts
    constexpr int NR = IPL > 0 ? IPL : 1;
    int32_t ids[NR];
    float prs[NR];
    int32_t wrank[NR]; // rank among earlier assignments of this warp with the same id
    uint32_t err = 0;
    auto load_item = [&](int64_t i, int32_t &e, float &p) {
        e = -1;
        p = 0.0f;
        if (i < a.NK) {
            e = __ldg(a.topk_idx + i);
            if (a.topk_probs != nullptr)
                p = __ldg(a.topk_probs + i);
            if (e < -1 || e >= E_log) {
                err |= MOE_DEV_EXPERT_RANGE;
                e = -1;
            }
        }
    };
    // Rank of id e among the earlier items of this warp (counter value before
    // this round + earlier lanes with the same id); advances the counter.
    auto rank_item = [&](int32_t e) -> int32_t {
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        const uint32_t before = e >= 0 ? my_cnt[e] : 0u;
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1)
            my_cnt[e] = before + __popc(peers);
        __syncwarp(); // the next update of this counter may come from another lane
        return static_cast<int32_t>(before + __popc(peers & lt));
    };
    if constexpr (IPL > 0) {
#pragma unroll
        for (int u = 0; u < IPL; ++u)
            load_item(base + u * 32 + lane, ids[u], prs[u]);
#pragma unroll
        for (int u = 0; u < IPL; ++u)
            wrank[u] = rank_item(ids[u]);
    } else {
        for (int it = 0; it < a.sub; it += 32) {
            load_item(base + it + lane, ids[0], prs[0]);
            (void)rank_item(ids[0]);
        }
    }
    err = __reduce_or_sync(0xffffffffu, err);
    if (lane == 0 && err)
        atomicOr(&s_err, err);
    __syncthreads();
    // per-warp counts -> exclusive prefix over warps; block total to the workspace
    for (int e = tid; e < E_log; e += LAYOUT_THREADS) {
        uint32_t c[LAYOUT_WARPS];
#pragma unroll
        for (int w = 0; w < LAYOUT_WARPS; ++w)
            c[w] = wcnt[w * E_log + e];
        uint32_t run = 0;
#pragma unroll
        for (int w = 0; w < LAYOUT_WARPS; ++w) {
            wcnt[w * E_log + e] = run;
            run += c[w];
        }
        a.ws_counts[static_cast<int64_t>(b) * E_log + e] = static_cast<int32_t>(run);
    }
    if (tid == 0 && s_err != 0)
        atomicOr(a.ws_barrier + 2, s_err);

    if (!grid_barrier_ticket(a.ws_barrier, static_cast<uint32_t>(a.G), a.barrier_extra, a.barrier_limit_ns)) {
        if (tid == 0)
            atomicOr(a.out.status, MOE_DEV_TIMEOUT);
        return;
    }

    // ---- phase 2a: block prefix and totals per logical expert. With E_log a
    // multiple of 4, thread (group g, column c) sums experts 4c..4c+3 over the
    // blocks g, g+P, ... with 16-byte loads (up to 8 in flight), then the P
    // groups are merged through shared memory. Otherwise P threads share an
    // expert and read it 4 bytes at a time.
    if ((E_log & 3) == 0) {
        const int E4 = E_log >> 2;
        const int P = min(32, LAYOUT_THREADS / E4); // E4 <= 512 = LAYOUT_THREADS
        if (tid < P * E4) {
            const int c = tid % E4, g = tid / E4;
            const int4 *col = reinterpret_cast<const int4 *>(a.ws_counts) + c;
            int4 pre = make_int4(0, 0, 0, 0), tot = make_int4(0, 0, 0, 0);
            for (int bb0 = g; bb0 < a.G; bb0 += 8 * P) {
                int4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int bb = bb0 + u * P;
                    v[u] = bb < a.G ? __ldcg(col + static_cast<int64_t>(bb) * E4) : make_int4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const bool before = bb0 + u * P < b;
                    tot.x += v[u].x;
                    tot.y += v[u].y;
                    tot.z += v[u].z;
                    tot.w += v[u].w;
                    pre.x += before ? v[u].x : 0;
                    pre.y += before ? v[u].y : 0;
                    pre.z += before ? v[u].z : 0;
                    pre.w += before ? v[u].w : 0;
                }
            }
            // g * E_log + 4c + i < P * E_log <= 4 * LAYOUT_THREADS: in bounds
            reinterpret_cast<int4 *>(&s_part[0][0])[tid] = pre;
            reinterpret_cast<int4 *>(&s_part[1][0])[tid] = tot;
        }
        if (b == 0 && tid == LAYOUT_THREADS - 1) {
            // every block OR-ed its error bits in before the barrier; block 0 reports and clears them
            s_err = __ldcg(a.ws_barrier + 2);
            a.ws_barrier[2] = 0;
        }
        __syncthreads();
        for (int e = tid; e < E_log; e += LAYOUT_THREADS) {
            int32_t pre = 0, tot = 0;
            for (int g = 0; g < P; ++g) {
                pre += s_part[0][g * E_log + e];
                tot += s_part[1][g * E_log + e];
            }
            s_pre[e] = pre;
            s_cnt[e] = tot;
            s_repl[e] = -1;
        }
        __syncthreads();
    } else {
        const int P = E_log >= LAYOUT_THREADS ? 1 : min(32, LAYOUT_THREADS / E_log);
        for (int item = tid; item < E_log * P; item += LAYOUT_THREADS) {
            const int e = item % E_log, part = item / E_log;
            int32_t pre = 0, tot = 0;
            for (int bb0 = part; bb0 < a.G; bb0 += 32 * P) {
                int32_t c[32];
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    const int bb = bb0 + u * P;
                    c[u] = bb < a.G ? __ldcg(a.ws_counts + static_cast<int64_t>(bb) * E_log + e) : 0;
                }
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    tot += c[u];
                    pre += (bb0 + u * P < b) ? c[u] : 0;
                }
            }
            if (P == 1) {
                s_pre[e] = pre;
                s_cnt[e] = tot;
                s_repl[e] = -1;
            } else { // E_log * P <= LAYOUT_THREADS: item indexes the scratch in bounds
                s_part[0][item] = pre;
                s_part[1][item] = tot;
            }
        }
        if (b == 0 && tid == LAYOUT_THREADS - 1) {
            s_err = __ldcg(a.ws_barrier + 2);
            a.ws_barrier[2] = 0;
        }
        __syncthreads();
        if (P > 1) {
            for (int e = tid; e < E_log; e += LAYOUT_THREADS) {
                int32_t pre = 0, tot = 0;
                for (int part = 0; part < P; ++part) {
                    pre += s_part[0][part * E_log + e];
                    tot += s_part[1][part * E_log + e];
                }
                s_pre[e] = pre;
                s_cnt[e] = tot;
                s_repl[e] = -1;
            }
            __syncthreads();
        }
    }

    // ---- phase 2b: hot experts and placement
    if (a.num_replicas > 0) {
        layout_placement(a, s_cnt, s_repl, s_hot);
        __syncthreads();
    }

    // ---- phase 2c: physical counts, scan of the rows each expert owns (C, or its
    // count rounded up to the row alignment), totals
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
    // exclusive scan of the rows each physical expert owns; the valid / kept /
    // dropped totals only in block 0, which publishes them. PER experts per
    // thread: 1 when E <= LAYOUT_THREADS, else 8 (E <= 4096).
    int32_t total_valid = 0, total_kept = 0, total_dropped = 0;
    auto scan_rows = [&](auto per_tag) {
        constexpr int PER = decltype(per_tag)::value;
        const int q0 = tid * PER;
        int32_t rows[PER];
        int32_t sum = 0, valid = 0, kept = 0, dropped = 0;
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int q = q0 + u;
            const int32_t raw = q < E ? s_raw[q] : 0;
            const int32_t local = layout_local_tokens(a, raw);
            rows[u] = q >= E ? 0 : a.C > 0 ? a.C_local : a.A == 1 ? local : ((local + a.A - 1) / a.A) * a.A;
            sum += rows[u];
            valid += raw;
            kept += local;
            dropped += a.C > 0 ? max(raw - a.C, 0) : 0;
        }
        int32_t inc = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t n = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o)
                inc += n;
        }
        if (b == 0) { // block-uniform
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                valid += __shfl_xor_sync(0xffffffffu, valid, o);
                kept += __shfl_xor_sync(0xffffffffu, kept, o);
                dropped += __shfl_xor_sync(0xffffffffu, dropped, o);
            }
            if (lane == 0) {
                s_wsum[1][warp] = valid;
                s_wsum[2][warp] = kept;
                s_wsum[3][warp] = dropped;
            }
        }
        if (lane == 31)
            s_wsum[0][warp] = inc;
        __syncthreads();
        int32_t wpre = 0;
#pragma unroll
        for (int w = 0; w < LAYOUT_WARPS; ++w)
            wpre += w < warp ? s_wsum[0][w] : 0;
        if (b == 0) {
#pragma unroll
            for (int w = 0; w < LAYOUT_WARPS; ++w) {
                total_valid += s_wsum[1][w];
                total_kept += s_wsum[2][w];
                total_dropped += s_wsum[3][w];
            }
        }
        int32_t run = wpre + inc - sum;
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int q = q0 + u;
            if (q < E)
                s_off[q] = run;
            run += rows[u];
        }
        if (tid == LAYOUT_THREADS - 1)
            s_off[E] = run;
    };
    if (E <= LAYOUT_THREADS)
        scan_rows(std::integral_constant<int, 1>{});
    else
        scan_rows(std::integral_constant<int, 8>{});
    __syncthreads();

    const moe_layout_t &o = a.out;
    if (b == 0) {
        for (int e = tid; e < E_log; e += LAYOUT_THREADS) {
            o.counts_logical[e] = s_cnt[e];
            o.placement[e] = s_repl[e];
        }
        for (int q = tid; q < E; q += LAYOUT_THREADS) {
            o.counts_raw[q] = s_raw[q];
            o.tokens_per_expert[q] = layout_local_tokens(a, s_raw[q]);
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
            o.counters[2] = total_dropped;
            o.counters[3] = static_cast<int32_t>(a.rows_max - total_kept);
            o.counters[4] = s_off[E];
            o.counters[5] = s_off[E];
            o.counters[6] = s_off[E];
            o.counters[7] = static_cast<int32_t>(s_err);
            if (s_err)
                atomicOr(o.status, s_err);
        }
    }

    // ---- phase 2d: per-assignment outputs. `in_block` = rank of the assignment
    // among the earlier ones of its block with the same logical id.
    // without capacity or alignment the kept rows are dense ([0, num_rows)): 2d writes
    // their expert, and 2e needs no search
    const bool rows_dense = a.C == 0 && a.A == 1;
    auto emit = [&](int64_t i, int32_t e, float p, int32_t in_block) {
        int32_t q = -1, ord = -1, dest = -1;
        uint8_t drop = 0;
        if (e >= 0) {
            const int32_t lo = s_pre[e] + in_block;
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
            if (!drop && (a.T == 1 || ord % a.T == a.tp_rank)) // this peer's share under TP folding
                dest = s_off[q] + (a.T == 1 ? ord : ord / a.T);
            if (dest >= a.rows_max) { // cannot happen for consistent counts; never write out of bounds
                atomicOr(o.status, MOE_DEV_ROW_RANGE);
                dest = -1;
            }
        }
        o.phys_idx[i] = q;
        o.ordinal[i] = ord;
        o.drop_mask[i] = drop;
        o.dest_row[i] = dest;
        if (dest >= 0) { // scattered: the rest of the row maps is written row by row below
            const int32_t t = static_cast<int32_t>(i) / a.k;
            o.row_token[dest] = t;
            o.row_slot[dest] = static_cast<int32_t>(i) - t * a.k;
            o.row_prob[dest] = p;
            if (rows_dense) // no padding inside the buffer: the row's expert is known here
                o.row_local_expert[dest] = q - (q / a.E_loc) * a.E_loc;
        }
        if (o.local_topk != nullptr) {
            const int owner = dest >= 0 ? q / a.E_loc : -1;
            for (int r = 0; r < a.R; ++r)
                o.local_topk[static_cast<int64_t>(r) * a.NK + i] = (r == owner) ? q - r * a.E_loc : -1;
        }
    };
    if constexpr (IPL > 0) {
        // wcnt now holds the exclusive prefix over earlier warps and is not modified any more
#pragma unroll
        for (int u = 0; u < IPL; ++u) {
            const int64_t i = base + u * 32 + lane;
            if (i < a.NK)
                emit(i, ids[u], prs[u], ids[u] >= 0 ? static_cast<int32_t>(my_cnt[ids[u]]) + wrank[u] : 0);
        }
    } else {
        // slices too long for registers: reload and rank again; the counters now
        // start from the warp's exclusive prefix, so the rank includes it
        for (int it = 0; it < a.sub; it += 32) {
            const int64_t i = base + it + lane;
            int32_t e;
            float p;
            load_item(i, e, p);
            const int32_t in_block = rank_item(e);
            if (i < a.NK)
                emit(i, e, p, in_block);
        }
    }

    // ---- phase 2e: per-row outputs that depend on the row index only, written
    // in row order: pad_mask and 0 / -1 / 0 in pad rows; with padding inside the
    // buffer also the owning expert (capacity slot, or a binary search of the
    // offsets) and the rank-local expert id (dense rows got theirs in 2d).
    const int64_t stride = static_cast<int64_t>(a.G) * LAYOUT_THREADS;
    const int32_t num_rows = s_off[E];
    for (int64_t row = static_cast<int64_t>(b) * LAYOUT_THREADS + tid; row < a.rows_max; row += stride) {
        if (rows_dense) {
            const bool tail = row >= num_rows;
            o.pad_mask[row] = tail ? 1 : 0;
            if (tail) {
                o.row_local_expert[row] = -1;
                o.row_token[row] = -1;
                o.row_slot[row] = -1;
                o.row_prob[row] = 0.0f;
            }
            continue;
        }
        int32_t q;
        bool pad;
        if (a.C > 0) {
            q = static_cast<int32_t>(row / a.C_local);
            const int32_t slot = static_cast<int32_t>(row - static_cast<int64_t>(q) * a.C_local);
            pad = slot >= layout_local_tokens(a, s_raw[q]);
        } else if (row >= num_rows) {
            q = -1;
            pad = true;
        } else {
            int32_t lo = 0, hi = E; // last q with s_off[q] <= row
            while (hi - lo > 1) {
                const int32_t mid = (lo + hi) >> 1;
                if (s_off[mid] <= row)
                    lo = mid;
                else
                    hi = mid;
            }
            q = lo;
            pad = row - s_off[q] >= layout_local_tokens(a, s_raw[q]); // alignment pad after the expert's tokens
        }
        o.pad_mask[row] = pad ? 1 : 0;
        o.row_local_expert[row] = pad ? -1 : q - (q / a.E_loc) * a.E_loc;
        if (pad) {
            o.row_token[row] = -1;
            o.row_slot[row] = -1;
            o.row_prob[row] = 0.0f;
        }
    }
}

} // namespace moert
