// permute.cuh — the dispatch row copy: send[dest_row[t,j]] = hidden[t].
//
// Megatron MoE page, dispatch_postprocess (permuted tokens per expert);
// Megatron MORI page, permute fused into the dispatch node, padded tails
// masked with 0.
//
// Read once, write k times. A group of 32, 64 or 128 threads (the smallest
// that covers the row with PERMUTE_CHUNKS 16-byte chunks per thread; longer
// rows are cut into pieces of 128 x PERMUTE_CHUNKS chunks) copies one token:
// it reads the token's destination rows and its chunks with streaming (L1
// no-allocate) loads, all in flight together (with a capacity, where most
// tokens may keep no slot, the chunks only after the destinations show that
// one is kept), then stores them to each kept destination row; a warp writes
// 512 contiguous bytes per store instruction. A CTA holds 128 / group
// tokens. The leading CTAs zero the pad rows (pad_mask = 1) while the copy
// CTAs stream. Every needed byte of hidden is read once and every byte of
// send written once.
//
// Staging each row through shared memory with bulk (TMA) copies is the fused
// dispatch's opt-in path (dispatch_bulk_kernel); in the replayed steps it is
// slower than this vector copy on every workload measured.
#pragma once

#include <cstdint>
#include <type_traits>

#include "moe_rt.h"
#include "ptx.cuh"

namespace moert {

constexpr int PERMUTE_THREADS = 128;
constexpr int PERMUTE_CHUNKS = 8; // 16-byte chunks per thread per piece: a piece is 16 KB

struct PermuteArgs {
    const uint4 *hidden;     // [N, V]
    uint4 *send;             // [rows_max, V]
    const int32_t *dest_row; // [N, k]
    const uint8_t *pad_mask; // [rows_max]
    uint32_t *status;
    int64_t N;
    int64_t rows_max;
    int32_t k;
    int32_t V;           // 16-byte chunks per row
    int32_t group;       // threads per token piece: 32, 64 or 128
    int32_t pieces;      // pieces per token
    int32_t zero_blocks; // leading CTAs that zero pad rows
    int32_t load_first = 0; // 1: every token keeps a slot (no capacity), so its row is loaded
                            // together with its destinations rather than after them
    // expert-parallel exchange: slot j's row d of expert q goes to the receive
    // buffer of q's owner, row ep_base[q] + d - ep_offsets[q]; the leading CTAs
    // zero this source's padding rows there (rows tokens[q] .. of each expert)
    uint4 *const *ep_peers;     // [R] device pointers
    const int32_t *phys_idx;    // [N, k]
    const int32_t *ep_base;     // [E]
    const int32_t *ep_offsets;  // [E + 1]
    const int32_t *ep_tokens;   // [E] tokens_per_expert
    int64_t recv_max;
    int32_t E, E_loc;
};

// Expert-parallel exchange: zero this source's padding rows of every expert in
// the owners' buffers (receive buffers, or gradient buffers in the same order);
// one warp per expert at a time. Row i of expert q (tokens[q] <= i < its rows)
// sits at base[q] + i in the buffer of q's owner.
__device__ __forceinline__ void ep_zero_pads_warp(uint4 *const *peers, const int32_t *base, const int32_t *offsets,
                                                  const int32_t *tokens, int32_t E, int32_t E_loc, int32_t V,
                                                  int64_t recv_max, uint32_t *status, int64_t worker,
                                                  int64_t nworkers)
{
    const int lane = threadIdx.x & 31;
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int64_t q = worker; q < E; q += nworkers) {
        const int32_t rows = __ldg(offsets + q + 1) - __ldg(offsets + q);
        const int32_t first = __ldg(tokens + q);
        const int64_t b = __ldg(base + q);
        if (b < 0 || b + rows > recv_max) {
            if (lane == 0 && rows > first)
                atomicOr(status, MOE_DEV_ROW_RANGE);
            continue;
        }
        uint4 *dst = peers[q / E_loc];
        for (int32_t i = first; i < rows; ++i)
            for (int32_t c = lane; c < V; c += 32)
                st_u4(dst + (b + i) * V + c, z);
    }
}

// Zero-fill every row r of `base` (V 16-byte chunks each) with pad_mask[r] != 0,
// for r = worker, worker + nworkers, ... ; one warp per worker.
__device__ __forceinline__ void zero_pad_rows_warp(uint4 *base, const uint8_t *pad_mask, int64_t rows_max, int32_t V,
                                                   int64_t worker, int64_t nworkers)
{
    const int lane = threadIdx.x & 31;
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int64_t r0 = worker; r0 < rows_max; r0 += 32 * nworkers) {
        const int64_t r = r0 + lane * nworkers;
        const bool pad = r < rows_max && pad_mask[r] != 0;
        uint32_t ballot = __ballot_sync(0xffffffffu, pad);
        while (ballot) {
            const int src = __ffs(ballot) - 1;
            ballot &= ballot - 1;
            uint4 *row = base + (r0 + static_cast<int64_t>(src) * nworkers) * V;
            for (int32_t c = lane; c < V; c += 32)
                st_u4(row + c, z);
        }
    }
}

// EP: the destinations are rows of the experts' owners' receive buffers.
template <bool EP = false>
__global__ void __launch_bounds__(PERMUTE_THREADS) permute_kernel(PermuteArgs a)
{
    using Dst = typename std::conditional<EP, uint4 *, int32_t>::type;
    __shared__ Dst s_dest[PERMUTE_THREADS / 32][32];
    pdl_trigger();
    pdl_wait();
    if (blockIdx.x < static_cast<uint32_t>(a.zero_blocks)) {
        const int64_t per = PERMUTE_THREADS / 32;
        const int64_t worker = static_cast<int64_t>(blockIdx.x) * per + (threadIdx.x >> 5);
        if constexpr (EP)
            ep_zero_pads_warp(a.ep_peers, a.ep_base, a.ep_offsets, a.ep_tokens, a.E, a.E_loc, a.V, a.recv_max,
                              a.status, worker, static_cast<int64_t>(a.zero_blocks) * per);
        else
            zero_pad_rows_warp(a.send, a.pad_mask, a.rows_max, a.V, worker, static_cast<int64_t>(a.zero_blocks) * per);
        return;
    }
    const int groups = PERMUTE_THREADS / a.group;
    const int g = threadIdx.x / a.group, gt = threadIdx.x - g * a.group;
    const int64_t unit = (static_cast<int64_t>(blockIdx.x) - a.zero_blocks) * groups + g;
    const int64_t units = a.N * a.pieces;
    const bool active = unit < units;
    const int64_t t = active ? unit / a.pieces : 0;
    const int piece = static_cast<int>(unit - t * a.pieces);
    const int32_t c0 = piece * (a.group * PERMUTE_CHUNKS) + gt;
    const uint4 *src = a.hidden + t * a.V;
    uint4 v[PERMUTE_CHUNKS];
    if (active && a.load_first) { // both round trips in flight at once
#pragma unroll
        for (int c = 0; c < PERMUTE_CHUNKS; ++c) {
            const int32_t idx = c0 + c * a.group;
            if (idx < a.V)
                v[c] = ld_stream_u4(src + idx);
        }
    }
    if (active && gt < a.k) {
        int32_t d = __ldg(a.dest_row + t * a.k + gt);
        if (d < -1 || d >= a.rows_max) {
            atomicOr(a.status, MOE_DEV_ROW_RANGE);
            d = -1;
        }
        if constexpr (EP) {
            uint4 *dst = nullptr;
            if (d >= 0) {
                const int32_t q = __ldg(a.phys_idx + t * a.k + gt);
                const int64_t r = q >= 0 && q < a.E
                                      ? static_cast<int64_t>(__ldg(a.ep_base + q)) + d - __ldg(a.ep_offsets + q)
                                      : -1;
                if (r < 0 || r >= a.recv_max)
                    atomicOr(a.status, MOE_DEV_ROW_RANGE);
                else
                    dst = a.ep_peers[q / a.E_loc] + r * a.V;
            }
            s_dest[g][gt] = dst;
        } else {
            s_dest[g][gt] = d;
        }
    }
    __syncthreads();
    if (!active)
        return;
    bool any = false; // a token whose every slot was dropped is not read at all
    for (int j = 0; j < a.k; ++j) {
        if constexpr (EP)
            any |= s_dest[g][j] != nullptr;
        else
            any |= s_dest[g][j] >= 0;
    }
    if (!any)
        return;
    if (!a.load_first) {
#pragma unroll
        for (int c = 0; c < PERMUTE_CHUNKS; ++c) {
            const int32_t idx = c0 + c * a.group;
            if (idx < a.V)
                v[c] = ld_stream_u4(src + idx);
        }
    }
    for (int j = 0; j < a.k; ++j) {
        uint4 *dst;
        if constexpr (EP) {
            dst = s_dest[g][j];
            if (dst == nullptr)
                continue;
        } else {
            const int32_t d = s_dest[g][j];
            if (d < 0)
                continue;
            dst = a.send + static_cast<int64_t>(d) * a.V;
        }
#pragma unroll
        for (int c = 0; c < PERMUTE_CHUNKS; ++c) {
            const int32_t idx = c0 + c * a.group;
            if (idx < a.V)
                st_u4(dst + idx, v[c]);
        }
    }
}

} // namespace moert
