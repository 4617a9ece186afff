// grid_barrier.cuh — the bounded grid barrier of the cooperative launches
// (dispatch layout, dedup layout). Co-residency of all blocks is guaranteed by
// the cooperative launch; every wait is bounded by %globaltimer.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace moert {

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t atom_add_acq_rel_u32(uint32_t *p, uint32_t v)
{
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Bounded single-word grid barrier. Each launch adds exactly GRID_BARRIER_SPAN
// to the word when every block has arrived: block 0 adds SPAN - (G - 1) -
// extra, the others 1 each, so every partial sum stays below the launch's
// target and the last arrival completes the barrier by itself (no reset, no
// generation word). `extra` > 0 only for the timeout test: the target is then
// never reached. The word wraps modulo 2^32, which SPAN divides. After a
// timeout the word is inconsistent and the scratch must be zero-filled again.
constexpr uint32_t GRID_BARRIER_SPAN = 1u << 20;

__device__ __forceinline__ bool grid_barrier_ticket(uint32_t *bar, uint32_t G, uint32_t extra, uint64_t limit_ns)
{
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t inc = blockIdx.x == 0 ? GRID_BARRIER_SPAN - (G - 1) - extra : 1u;
        const uint32_t old = atom_add_acq_rel_u32(bar, inc);
        const uint32_t target = (old & ~(GRID_BARRIER_SPAN - 1)) + GRID_BARRIER_SPAN;
        int ok = 1;
        if (old + inc != target) {
            const uint64_t t0 = global_timer_ns();
            while (static_cast<int32_t>(ld_acquire_u32(bar) - target) < 0) {
                if (global_timer_ns() - t0 > limit_ns) {
                    ok = 0;
                    break;
                }
            }
        }
        s_ok = ok;
    }
    __syncthreads();
    return s_ok != 0;
}

} // namespace moert
