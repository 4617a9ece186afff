// lookback.cuh — ticket-ordered decoupled look-back over per-block count vectors.
//
// The stable per-expert ordinals of the dispatch layout (DeepSpeed EP page,
// assignment_ordinals_by_expert) need, for every block of assignments, the
// number of same-expert assignments in all earlier blocks: an exclusive scan
// over blocks, one column per expert. It is computed in a single pass with the
// decoupled look-back of Merrill & Garland ("Single-pass Parallel Prefix Scan
// with Decoupled Look-back", NVIDIA technical report NVR-2016-002):
//
//  * Each block takes a ticket from an atomic counter; the ticket, not
//    blockIdx, is its position in the scan. A block with ticket v therefore
//    only ever waits for blocks with tickets < v, which have all been
//    scheduled already, so no co-residency is needed and any grid size and
//    any number of concurrent launches make progress.
//  * A block publishes, per expert, its own count (AGG) as soon as it has
//    counted, then looks back over its predecessors, summing their AGG words
//    until it meets an inclusive prefix (INCL), and publishes its own INCL.
//  * Status and value share one 64-bit word, written and read whole, so a
//    reader never sees a flag without its value and no fence is needed.
//  * Every word carries the launch's epoch, so words left by earlier launches
//    (or by a launch that timed out) read as "not yet published": the scratch
//    never has to be cleared between calls.
//  * Waits are bounded by %globaltimer; a block that runs out of time treats
//    the word as an empty inclusive prefix, records MOE_DEV_TIMEOUT and goes on.
//
// Word layout: bits 0-30 the count (< 2^31), bit 31 "an expert id out of
// range was seen" (OR-ed along the scan, so the last block learns whether any
// block saw one), bits 32-33 the status (0 none, 1 AGG, 2 INCL), bits 34-63
// the launch epoch modulo 2^30.
//
// Ticket word: low 32 bits count the tickets taken in this launch, high 32
// bits the epoch. The block that draws ticket G-1 (all others are drawn by
// then) moves it to (epoch + 1, 0) for the next launch, which cannot take a
// ticket before this launch has completed (stream order).
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace moert {

constexpr uint64_t LB_AGG = 1ull << 32;
constexpr uint64_t LB_INCL = 2ull << 32;
constexpr uint64_t LB_STATUS_MASK = 3ull << 32;
constexpr uint32_t LB_ERR_BIT = 0x80000000u;
constexpr uint32_t LB_EPOCH_MASK = (1u << 30) - 1u;

__device__ __forceinline__ uint64_t lb_word(uint32_t epoch, uint64_t status, uint32_t value, bool err)
{
    return (static_cast<uint64_t>(epoch & LB_EPOCH_MASK) << 34) | status | (err ? LB_ERR_BIT : 0u) |
           (value & ~LB_ERR_BIT);
}

__device__ __forceinline__ bool lb_ready(uint64_t w, uint32_t epoch)
{
    return (w & LB_STATUS_MASK) != 0 && static_cast<uint32_t>(w >> 34) == (epoch & LB_EPOCH_MASK);
}

__device__ __forceinline__ uint32_t lb_value(uint64_t w) { return static_cast<uint32_t>(w) & ~LB_ERR_BIT; }
__device__ __forceinline__ bool lb_err(uint64_t w) { return (static_cast<uint32_t>(w) & LB_ERR_BIT) != 0; }
__device__ __forceinline__ bool lb_incl(uint64_t w) { return (w & LB_STATUS_MASK) == LB_INCL; }

__device__ __forceinline__ uint64_t ld_relaxed_u64(const unsigned long long *p)
{
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, uint64_t v)
{
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Ticket of this block (thread 0 only): its position in the scan and the
// launch epoch. The block drawing the last ticket rolls the word over.
__device__ __forceinline__ void lb_take_ticket(unsigned long long *ticket_word, uint32_t G, uint32_t *vb,
                                               uint32_t *epoch)
{
    const unsigned long long old = atomicAdd(ticket_word, 1ull);
    *vb = static_cast<uint32_t>(old);
    *epoch = static_cast<uint32_t>(old >> 32);
    if (*vb == G - 1)
        atomicAdd(ticket_word, (1ull << 32) - static_cast<unsigned long long>(G));
}

// Result of scanning one chunk of predecessors for one column.
struct LbChunk {
    uint32_t sum;  // values summed, nearest predecessor first
    bool err;      // OR of the error bits summed
    bool closed;   // an INCL word was met, or the chunk ran past block 0: the prefix is complete
    bool timeout;  // a wait ran out
};

// Sums the words of blocks top, top-1, ..., top-WL+1 (those >= 0) of column
// `col` (stride `ld` words between blocks), nearest first, stopping after the
// first INCL. All WL loads are issued at once; a word that is not yet ready is
// polled again, bounded by limit_ns from the first poll.
template <int WL>
__device__ __forceinline__ LbChunk lb_scan_chunk(const unsigned long long *flags, int64_t ld, int32_t col,
                                                 int32_t top, uint32_t epoch, uint64_t limit_ns)
{
    uint64_t w[WL];
#pragma unroll
    for (int i = 0; i < WL; ++i)
        w[i] = top - i >= 0 ? ld_relaxed_u64(flags + static_cast<int64_t>(top - i) * ld + col) : 0ull;
    LbChunk c{0u, false, false, false};
    uint64_t t0 = 0;
#pragma unroll
    for (int i = 0; i < WL; ++i) {
        if (top - i < 0) { // ran past block 0: everything before this chunk's top is summed
            c.closed = true;
            break;
        }
        uint64_t v = w[i];
        while (!lb_ready(v, epoch)) {
            const uint64_t now = global_timer_ns();
            if (t0 == 0)
                t0 = now;
            else if (now - t0 > limit_ns) {
                c.timeout = true;
                break;
            }
            v = ld_relaxed_u64(flags + static_cast<int64_t>(top - i) * ld + col);
        }
        if (c.timeout) { // give up on this column: what was summed stands as the prefix
            c.closed = true;
            break;
        }
        c.sum += lb_value(v);
        c.err |= lb_err(v);
        if (lb_incl(v)) {
            c.closed = true;
            break;
        }
    }
    return c;
}

} // namespace moert
