// layout.cuh — the dispatch layout: a ticket-ordered count pass with a
// decoupled look-back, then a fill pass (or the fused dispatch of dispatch.cuh).
//
// Steps (page citations in moe_rt.h, moe_dispatch_layout):
//
// layout_count_kernel (blocks ordered by an atomic ticket, any grid size):
//   1. each warp loads its contiguous slice of the flattened [N,k] expert ids
//      and ranks every assignment among the earlier ones of its warp with the
//      same logical id (__match_any_sync + popc, one shared-memory counter
//      update per distinct id);
//   2. per expert, the per-warp counts become per-warp exclusive prefixes and
//      the block total is published as the block's look-back word;
//   3. decoupled look-back (lookback.cuh): the block sums its predecessors'
//      words per expert until it meets an inclusive prefix, then publishes its
//      own; the last block's inclusive words are the logical histogram;
//   4. every assignment's stable logical ordinal (earlier blocks + earlier
//      warps + earlier items of its own warp) is written out.
// Every CTA of the next pass then derives the small tables itself from the
// histogram (layout_tables_cta: hot-expert placement, physical counts,
// capacity, the exclusive scan of the rows), so no single block's serial work
// sits between the two passes; its CTA 0 writes the tables out.
// layout_fill_kernel: per assignment the physical expert and ordinal (closed
// form below), drop flag, destination row (expert offset + ordinal), the local
// view and the inverse row maps scattered by row; per row the pad / tail marks.
//
// Closed forms (equal to counting physical ordinals directly, as the CPU
// definition does): a hot expert's assignment with logical ordinal o goes to
// the master if o is even, else to the replica, at physical ordinal o/2; so the
// master holds ceil(c/2) and the replica floor(c/2) of the expert's c
// assignments.
#pragma once

#include <cstdint>

#include "moe_rt.h"
#include "lookback.cuh"
#include "ptx.cuh"

namespace moert {

constexpr int LAYOUT_THREADS = 512;
constexpr int LAYOUT_WARPS = LAYOUT_THREADS / 32;
constexpr int LAYOUT_MAX_BLOCKS = 128;
constexpr int LAYOUT_TARGET_BLOCKS = 32; // up to this many blocks the look-back ends in one round
constexpr int LAYOUT_MAX_E_LOG = 2048;
constexpr int LAYOUT_MAX_PLACEMENT_RANKS = 64;
constexpr int LAYOUT_MAX_IPL = 8;   // assignments per lane held in registers
constexpr int LAYOUT_LB_CHUNK = 16; // predecessors one thread reads per look-back round
constexpr int FILL_THREADS = 256;

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
    int32_t sub;     // assignments per warp slice, a multiple of 32
    int32_t G;       // count blocks
    unsigned long long *ws_ticket; // ticket word (lookback.cuh)
    unsigned long long *ws_flags;  // [G][E_log] look-back words
    uint64_t wait_limit_ns;
    uint32_t test_stall; // test hook: the block with ticket 0 never publishes
    moe_layout_t out;
};

// Look-back parts per expert: the block's threads split each expert's
// predecessors into this many chunks per round (1 when E_log >= LAYOUT_THREADS).
__host__ __device__ inline int layout_lb_parts(int E_log)
{
    if (E_log >= LAYOUT_THREADS)
        return 1;
    const int p = LAYOUT_THREADS / E_log;
    return p > 32 ? 32 : p;
}

// Dynamic shared memory of the count kernel, in 32-bit words: per-warp
// counters, the exclusive prefix, the block totals, the look-back state and
// the per-part sums and flags.
__host__ __device__ inline size_t layout_count_smem_words(int E_log)
{
    const size_t parts = static_cast<size_t>(layout_lb_parts(E_log)) * static_cast<size_t>(E_log);
    return static_cast<size_t>(LAYOUT_WARPS) * E_log + 3 * static_cast<size_t>(E_log) + 2 * parts;
}

// Shared memory of the tables every CTA of the second pass derives, in 32-bit
// words: logical totals and placement [E_log] each, physical counts [E],
// offsets [E+1], hot experts [E_log].
__host__ __device__ inline size_t layout_tables_smem_words(int E_log, int E)
{
    return 3 * static_cast<size_t>(E_log) + 2 * static_cast<size_t>(E) + 1;
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

// Rows an expert with `raw` assignments owns in this peer's buffer: C slots
// with a capacity, else its kept count rounded up to the row alignment.
__device__ __forceinline__ int32_t layout_expert_rows(const LayoutArgs &a, int32_t raw)
{
    const int32_t local = layout_local_tokens(a, raw);
    return a.C > 0 ? a.C_local : (a.A == 1 ? local : ((local + a.A - 1) / a.A) * a.A);
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

// Shared-memory tables of one CTA of the second pass (layout_tables_smem_words).
struct LayoutTables {
    int32_t *cnt;  // [E_log] logical totals
    int32_t *repl; // [E_log] replica slot of a hot expert, else -1
    int32_t *raw;  // [E] physical counts before capacity
    int32_t *off;  // [E+1] first row of each physical expert
    int32_t *hot;  // [E_log] hot experts in placement order
    int32_t valid, kept, dropped; // totals over the experts (assignments with an id, rows kept, drops)
    bool range_err;               // some count block saw an id outside [-1, E_log)
};

__device__ __forceinline__ LayoutTables layout_tables_carve(const LayoutArgs &a, int32_t *smem)
{
    LayoutTables t;
    t.cnt = smem;
    t.repl = t.cnt + a.E_log;
    t.raw = t.repl + a.E_log;
    t.off = t.raw + a.E;
    t.hot = t.off + a.E + 1;
    t.valid = t.kept = t.dropped = 0;
    t.range_err = false;
    return t;
}

// The tables, derived by every CTA of the second pass from the logical
// histogram in the last count block's inclusive look-back words: hot-expert
// placement, physical counts, the exclusive scan of the rows each physical
// expert owns, and the totals. Must be called by every thread of the CTA (any
// block size that is a multiple of 32, up to 1024); ends with the tables in
// shared memory and the CTA synchronised. A word that was never published
// (a count block that ran out of time) reads as 0 and sets MOE_DEV_TIMEOUT.
__device__ void layout_tables_cta(const LayoutArgs &a, LayoutTables &t)
{
    __shared__ int32_t s_red[4][32];
    __shared__ uint32_t s_flag;
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
    const int E_log = a.E_log, E = a.E;
    // the count pass has completed: its ticket word holds the next launch's epoch
    const uint32_t epoch = static_cast<uint32_t>(__ldcg(a.ws_ticket) >> 32) - 1u;
    const unsigned long long *last = a.ws_flags + static_cast<int64_t>(a.G - 1) * E_log;
    if (tid == 0)
        s_flag = 0;
    __syncthreads();
    uint32_t flag = 0;
    for (int e = tid; e < E_log; e += nt) {
        const uint64_t w = __ldcg(last + e);
        const bool ok = lb_ready(w, epoch) && lb_incl(w);
        t.cnt[e] = ok ? static_cast<int32_t>(lb_value(w)) : 0;
        t.repl[e] = -1;
        if (!ok)
            flag |= 1u;
        else if (e == 0 && lb_err(w))
            flag |= 2u;
    }
    if (flag)
        atomicOr(&s_flag, flag);
    __syncthreads();
    t.range_err = (s_flag & 2u) != 0;
    if ((s_flag & 1u) && tid == 0 && blockIdx.x == 0)
        atomicOr(a.out.status, MOE_DEV_TIMEOUT);
    if (a.num_replicas > 0) {
        layout_placement(a, t.cnt, t.repl, t.hot);
        __syncthreads();
    }
    // physical counts: a master keeps its count, or ceil(c/2) of a hot expert's c;
    // the replica slot of a hot expert gets floor(c/2); empty replica slots 0
    for (int q = tid; q < E; q += nt) {
        const int r = q / a.E_loc, i = q - r * a.E_loc;
        int32_t c = 0;
        if (i < a.M) {
            const int e = r * a.M + i;
            c = t.cnt[e];
            if (t.repl[e] >= 0)
                c = (c + 1) / 2;
        }
        t.raw[q] = c;
    }
    __syncthreads();
    if (a.num_replicas > 0) {
        for (int e = tid; e < E_log; e += nt)
            if (t.repl[e] >= 0)
                t.raw[t.repl[e]] = t.cnt[e] / 2;
        __syncthreads();
    }
    // exclusive scan of the rows each physical expert owns: thread tid takes the
    // contiguous experts [tid c, tid c + c), a warp scan and one pass over the
    // warps' sums give its start
    const int c = (E + nt - 1) / nt;
    const int q0 = tid * c;
    int32_t sum = 0, valid = 0, kept = 0, dropped = 0;
    for (int u = 0; u < c; ++u) {
        const int q = q0 + u;
        if (q < E) {
            const int32_t raw = t.raw[q];
            sum += layout_expert_rows(a, raw);
            valid += raw;
            kept += layout_local_tokens(a, raw);
            dropped += a.C > 0 ? max(raw - a.C, 0) : 0;
        }
    }
    int32_t inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o)
            inc += n;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        valid += __shfl_xor_sync(0xffffffffu, valid, o);
        kept += __shfl_xor_sync(0xffffffffu, kept, o);
        dropped += __shfl_xor_sync(0xffffffffu, dropped, o);
    }
    if (lane == 31)
        s_red[0][warp] = inc;
    if (lane == 0) {
        s_red[1][warp] = valid;
        s_red[2][warp] = kept;
        s_red[3][warp] = dropped;
    }
    __syncthreads();
    int32_t run = inc - sum;
    t.valid = t.kept = t.dropped = 0;
    for (int w = 0; w < nw; ++w) {
        run += w < warp ? s_red[0][w] : 0;
        t.valid += s_red[1][w];
        t.kept += s_red[2][w];
        t.dropped += s_red[3][w];
    }
    for (int u = 0; u < c; ++u) {
        const int q = q0 + u;
        if (q < E) {
            t.off[q] = run;
            run += layout_expert_rows(a, t.raw[q]);
        }
    }
    if (q0 < E && q0 + c >= E) // the thread holding the last expert closes the scan
        t.off[E] = run;
    __syncthreads();
}

// Writes the tables (by one CTA): histograms, placement, offsets, splits, counters.
__device__ void layout_tables_store(const LayoutArgs &a, const LayoutTables &t)
{
    const int tid = threadIdx.x, nt = blockDim.x;
    const moe_layout_t &o = a.out;
    const int E = a.E;
    for (int e = tid; e < a.E_log; e += nt) {
        o.counts_logical[e] = t.cnt[e];
        o.placement[e] = t.repl[e];
    }
    for (int q = tid; q < E; q += nt) {
        o.counts_raw[q] = t.raw[q];
        o.tokens_per_expert[q] = layout_local_tokens(a, t.raw[q]);
    }
    for (int q = tid; q <= E; q += nt)
        o.expert_offsets[q] = t.off[q];
    for (int r = tid; r < a.R; r += nt) {
        const int32_t split = t.off[(r + 1) * a.E_loc] - t.off[r * a.E_loc];
        o.input_splits[r] = split;
        o.output_splits[r] = split;
        o.rank_offsets[r] = t.off[r * a.E_loc];
    }
    if (tid == 0) {
        const int32_t rows = t.off[E];
        o.rank_offsets[a.R] = rows;
        *o.num_rows = rows;
        o.counters[0] = t.valid;
        o.counters[1] = t.kept;
        o.counters[2] = t.dropped;
        o.counters[3] = static_cast<int32_t>(a.rows_max - t.kept);
        o.counters[4] = rows;
        o.counters[5] = rows;
        o.counters[6] = rows;
        o.counters[7] = t.range_err ? static_cast<int32_t>(MOE_DEV_EXPERT_RANGE) : 0;
    }
}

// Per-assignment outputs of assignment i from its logical id (validated) and
// logical ordinal: physical expert and ordinal, drop flag, destination row, the
// local view and the inverse row maps at the destination. Returns the row (-1
// if none); with store = false it only computes the row. `dense_rows`: no
// padding inside the buffer, so the row's local expert is written here
// (otherwise by the row pass).
template <bool REROUTE>
__device__ __forceinline__ int32_t layout_emit_assignment(const LayoutArgs &a, const LayoutTables &t, int64_t i,
                                                          int32_t e, int32_t lo, float p, bool dense_rows,
                                                          bool store = true)
{
    const moe_layout_t &o = a.out;
    int32_t q = -1, ord = -1, dest = -1;
    uint8_t drop = 0;
    bool kept = false;
    if (e >= 0) {
        if (REROUTE) {
            const int32_t master = (e / a.M) * a.E_loc + (e % a.M);
            const int32_t repl = t.repl[e];
            q = (repl >= 0 && (lo & 1)) ? repl : master;
            ord = repl >= 0 ? lo >> 1 : lo;
        } else { // no replicas: the physical expert is the logical one
            q = e;
            ord = lo;
        }
        drop = (a.C > 0 && ord >= a.C) ? 1 : 0;
        kept = !drop && (a.T == 1 || ord % a.T == a.tp_rank); // this peer's share under TP folding
    }
    if (kept) {
        const int64_t d = static_cast<int64_t>(t.off[q]) + (a.T == 1 ? ord : ord / a.T);
        if (d < 0 || d >= a.rows_max) { // cannot happen for consistent counts; never write out of bounds
            if (store)
                atomicOr(o.status, MOE_DEV_ROW_RANGE);
        } else {
            dest = static_cast<int32_t>(d);
        }
    }
    if (!store)
        return dest;
    o.phys_idx[i] = q;
    o.ordinal[i] = ord;
    o.drop_mask[i] = drop;
    o.dest_row[i] = dest;
    if (dest >= 0) { // scattered: the rest of the row maps is written row by row
        const int32_t tok = static_cast<int32_t>(i / a.k);
        o.row_token[dest] = tok;
        o.row_slot[dest] = static_cast<int32_t>(i - static_cast<int64_t>(tok) * a.k);
        o.row_prob[dest] = p;
        if (dense_rows)
            o.row_local_expert[dest] = q - (q / a.E_loc) * a.E_loc;
    }
    if (o.local_topk != nullptr) {
        const int owner = dest >= 0 ? q / a.E_loc : -1;
        for (int r = 0; r < a.R; ++r)
            o.local_topk[static_cast<int64_t>(r) * a.NK + i] = (r == owner) ? q - r * a.E_loc : -1;
    }
    return dest;
}

// The row pass for send-buffer row `row`: pad_mask and 0 / -1 / 0 in pad and
// tail rows; with padding inside the buffer also the owning expert (capacity
// slot, or a binary search of the offsets) and its local id. Returns whether
// the row is a pad (or tail) row.
__device__ __forceinline__ bool layout_emit_row(const LayoutArgs &a, const LayoutTables &t, int64_t row,
                                                bool dense_rows)
{
    const moe_layout_t &o = a.out;
    const int32_t E = a.E, num_rows = t.off[E];
    bool pad;
    if (dense_rows) {
        pad = row >= num_rows;
        o.pad_mask[row] = pad ? 1 : 0;
        if (pad)
            o.row_local_expert[row] = -1;
    } else {
        int32_t q;
        if (a.C > 0) {
            q = static_cast<int32_t>(row / a.C_local);
            const int32_t slot = static_cast<int32_t>(row - static_cast<int64_t>(q) * a.C_local);
            pad = slot >= layout_local_tokens(a, t.raw[q]);
        } else if (row >= num_rows) {
            q = -1;
            pad = true;
        } else {
            int32_t lo = 0, hi = E; // last q with off[q] <= row
            while (hi - lo > 1) {
                const int32_t mid = (lo + hi) >> 1;
                if (t.off[mid] <= row)
                    lo = mid;
                else
                    hi = mid;
            }
            q = lo;
            pad = row - t.off[q] >= layout_local_tokens(a, t.raw[q]); // alignment pad after the expert's tokens
        }
        o.pad_mask[row] = pad ? 1 : 0;
        o.row_local_expert[row] = pad ? -1 : q - (q / a.E_loc) * a.E_loc;
    }
    if (pad) {
        o.row_token[row] = -1;
        o.row_slot[row] = -1;
        o.row_prob[row] = 0.0f;
    }
    return pad;
}

// The count kernel (steps 1-4 at the top of this file). IPL > 0: each lane
// keeps IPL ids in registers (sub = 32 * IPL); 0: any sub, the slice is read
// twice. It lets the next kernel launch only after its own wait has returned,
// so that kernel may read the inputs of this call (written before it) early.
// A ticket beyond the grid (only when two calls share one workspace at once,
// which the contract forbids) makes the block report MOE_DEV_TIMEOUT and stop.
template <int IPL>
__global__ void __launch_bounds__(LAYOUT_THREADS, 1) layout_count_kernel(LayoutArgs a)
{
    extern __shared__ __align__(16) uint32_t layout_smem[];
    const int E_log = a.E_log;
    const int P = layout_lb_parts(E_log);
    uint32_t *wcnt = layout_smem;                                               // [WARPS][E_log]
    int32_t *s_excl = reinterpret_cast<int32_t *>(wcnt + LAYOUT_WARPS * E_log); // [E_log] earlier blocks
    int32_t *s_agg = s_excl + E_log;                                            // [E_log] this block
    uint32_t *s_state = reinterpret_cast<uint32_t *>(s_agg + E_log);            // [E_log] look-back state
    uint32_t *s_psum = s_state + E_log;                                         // [P][E_log]
    uint32_t *s_pflag = s_psum + P * E_log;                                     // [P][E_log]
    __shared__ uint32_t s_vb, s_epoch, s_err, s_timeout;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t lt = lanemask_lt();
    for (int i = tid; i < LAYOUT_WARPS * E_log; i += LAYOUT_THREADS)
        wcnt[i] = 0;
    if (tid == 0) {
        s_err = 0;
        s_timeout = 0;
    }
    // The ticket is drawn before the wait: only count passes touch the ticket word,
    // and the next count pass on this workspace launches after this one lets its
    // dependents launch, which happens below, after every ticket of this launch has
    // been drawn (stream order; a kernel launches only once its predecessor let it).
    if (tid == 0) {
        uint32_t vb, epoch;
        lb_take_ticket(a.ws_ticket, static_cast<uint32_t>(a.G), &vb, &epoch);
        s_vb = vb;
        s_epoch = epoch;
    }
    pdl_wait(); // ids and earlier launches' words are settled
    __syncthreads();
    pdl_trigger();
    const uint32_t vb = s_vb, epoch = s_epoch;
    if (vb >= static_cast<uint32_t>(a.G)) { // two calls shared the workspace at once: stay inside it
        if (tid == 0)
            atomicOr(a.out.status, MOE_DEV_TIMEOUT);
        return;
    }
    const int64_t base = (static_cast<int64_t>(vb) * LAYOUT_WARPS + warp) * a.sub;
    uint32_t *my_cnt = wcnt + warp * E_log;

    // ---- 1. load the slice, rank within the warp, per-warp counts
    constexpr int NR = IPL > 0 ? IPL : 1;
    int32_t ids[NR];
    int32_t wrank[NR]; // rank among earlier assignments of this warp with the same id
    uint32_t err = 0;
    auto load_id = [&](int64_t i) -> int32_t {
        int32_t e = -1;
        if (i < a.NK) {
            e = __ldg(a.topk_idx + i);
            if (e < -1 || e >= E_log) {
                err |= MOE_DEV_EXPERT_RANGE;
                e = -1;
            }
        }
        return e;
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
            ids[u] = load_id(base + u * 32 + lane);
#pragma unroll
        for (int u = 0; u < IPL; ++u)
            wrank[u] = rank_item(ids[u]);
    } else {
        for (int it = 0; it < a.sub; it += 32)
            (void)rank_item(load_id(base + it + lane));
    }
    err = __reduce_or_sync(0xffffffffu, err);
    if (lane == 0 && err)
        atomicOr(&s_err, err);
    __syncthreads();
    const bool blk_err = s_err != 0;
    if (tid == 0 && blk_err)
        atomicOr(a.out.status, s_err);

    // ---- 2. per-warp counts -> exclusive prefixes over warps; publish the block total
    const bool publish = !(a.test_stall != 0 && vb == 0);
    unsigned long long *my_words = a.ws_flags + static_cast<int64_t>(vb) * E_log;
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
        s_agg[e] = static_cast<int32_t>(run);
        s_excl[e] = 0;
        s_state[e] = 0;
        if (publish) // the first block's total is already its inclusive prefix
            st_relaxed_u64(my_words + e, lb_word(epoch, vb == 0 ? LB_INCL : LB_AGG, run, blk_err));
    }
    __syncthreads();

    // ---- 3. decoupled look-back: part p of expert e reads the chunk of
    // predecessors [hi - (p+1) W + 1, hi - p W] each round, nearest first;
    // parts are merged in order up to the first one that closed the prefix
    constexpr uint32_t ST_DONE = 1u, ST_ERR = 2u;
    if (vb > 0) {
        int32_t hi = static_cast<int32_t>(vb) - 1;
        for (;;) {
            for (int item = tid; item < P * E_log; item += LAYOUT_THREADS) {
                const int e = item % E_log, p = item / E_log;
                if (s_state[e] & ST_DONE)
                    continue;
                const LbChunk c = lb_scan_chunk<LAYOUT_LB_CHUNK>(a.ws_flags, E_log, e, hi - p * LAYOUT_LB_CHUNK,
                                                                 epoch, a.wait_limit_ns);
                s_psum[item] = c.sum;
                s_pflag[item] = (c.closed ? 1u : 0u) | (c.err ? 2u : 0u);
                if (c.timeout)
                    s_timeout = 1;
            }
            __syncthreads();
            int more = 0;
            for (int e = tid; e < E_log; e += LAYOUT_THREADS) {
                uint32_t st = s_state[e];
                if (st & ST_DONE)
                    continue;
                uint32_t sum = static_cast<uint32_t>(s_excl[e]);
                for (int p = 0; p < P; ++p) {
                    const uint32_t f = s_pflag[p * E_log + e];
                    sum += s_psum[p * E_log + e];
                    st |= (f & 2u) ? ST_ERR : 0u;
                    if (f & 1u) {
                        st |= ST_DONE;
                        break;
                    }
                }
                s_excl[e] = static_cast<int32_t>(sum);
                s_state[e] = st;
                if (st & ST_DONE) {
                    if (publish)
                        st_relaxed_u64(my_words + e, lb_word(epoch, LB_INCL, sum + static_cast<uint32_t>(s_agg[e]),
                                                             blk_err || (st & ST_ERR)));
                } else {
                    more = 1;
                }
            }
            hi -= P * LAYOUT_LB_CHUNK;
            if (!__syncthreads_or(more))
                break;
        }
        if (tid == 0 && s_timeout)
            atomicOr(a.out.status, MOE_DEV_TIMEOUT);
    }

    // ---- 4. stable logical ordinals (the second pass turns them into physical ones)
    if constexpr (IPL > 0) {
        // wcnt holds the exclusive prefix over earlier warps and is not modified any more
#pragma unroll
        for (int u = 0; u < IPL; ++u) {
            const int64_t i = base + u * 32 + lane;
            const int32_t e = ids[u];
            if (i < a.NK)
                a.out.ordinal[i] = e >= 0 ? s_excl[e] + static_cast<int32_t>(my_cnt[e]) + wrank[u] : -1;
        }
    } else {
        // slices too long for registers: reload and rank again; the counters now
        // start from the warp's exclusive prefix, so the rank includes it
        for (int it = 0; it < a.sub; it += 32) {
            const int64_t i = base + it + lane;
            const int32_t e = load_id(i);
            const int32_t in_block = rank_item(e);
            if (i < a.NK)
                a.out.ordinal[i] = e >= 0 ? s_excl[e] + in_block : -1;
        }
    }
}

// The fill kernel: every CTA derives the tables, then one thread per
// assignment (index i < NK) and per send-buffer row (i < rows_max). REROUTE:
// physical expert and ordinal from the placement; DENSE (no capacity, no
// alignment): the kept rows are [0, num_rows) and an assignment writes its
// row's local expert. CTA 0 writes the tables.
template <bool REROUTE, bool DENSE>
__global__ void __launch_bounds__(FILL_THREADS) layout_fill_kernel(LayoutArgs a)
{
    extern __shared__ __align__(16) int32_t fill_smem[];
    const int64_t i = static_cast<int64_t>(blockIdx.x) * FILL_THREADS + threadIdx.x;
    pdl_trigger();
    pdl_wait(); // the count pass is complete
    int32_t e = -1, lo = -1;
    float p = 0.0f;
    if (i < a.NK) { // issued before the tables so that both round trips overlap
        e = __ldg(a.topk_idx + i);
        lo = __ldcg(a.out.ordinal + i);
        if (a.topk_probs != nullptr)
            p = __ldg(a.topk_probs + i);
    }
    LayoutTables t = layout_tables_carve(a, fill_smem);
    layout_tables_cta(a, t);
    if (blockIdx.x == 0)
        layout_tables_store(a, t);
    if (i < a.NK) {
        if (e < -1 || e >= a.E_log) // reported by the count pass
            e = -1;
        layout_emit_assignment<REROUTE>(a, t, i, e, lo, p, DENSE);
    }
    if (i < a.rows_max)
        layout_emit_row(a, t, i, DENSE);
}

} // namespace moert
