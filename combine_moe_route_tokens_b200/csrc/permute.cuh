// permute.cuh — the dispatch row copy: send[dest_row[t,j]] = hidden[t].
//
// Megatron MoE page, dispatch_postprocess (permuted tokens per expert);
// Megatron MORI page, permute fused into the dispatch node, padded tails
// masked with 0.
//
// Read once, write k times, staged through shared memory by the TMA unit:
// one warp per CTA, several CTAs per SM, persistent over tokens. Lane 0
// issues a bulk global->shared load of each token row (mbarrier completion
// with an evict-first L2 hint, the row is read once) into a ring of STAGES
// slots, then one bulk shared->global store per kept destination row. A slot
// is refilled once the stores that read it have drained
// (cp.async.bulk.wait_group.read), which keeps STAGES-1 loads in flight per
// CTA while the stores stream out. Rows longer than PERMUTE_SEG_BYTES are
// moved in segments. Pad rows are zero-filled by the same CTAs afterwards.
#pragma once

#include <cstdint>

#include "moe_rt.h"
#include "ptx.cuh"

namespace moert {

constexpr int PERMUTE_MAX_STAGES = 4;
constexpr uint32_t PERMUTE_SEG_BYTES = 32768;

struct PermuteArgs {
    const uint8_t *hidden;  // [N, row_bytes]
    uint8_t *send;          // [rows_max, row_bytes]
    const int32_t *dest_row; // [N, k]
    const uint8_t *pad_mask; // [rows_max]
    uint32_t *status;
    int64_t N;
    int64_t rows_max;
    int32_t k;
    uint32_t row_bytes;
    uint32_t seg_bytes; // <= PERMUTE_SEG_BYTES, multiple of 16
    int32_t nseg;       // segments per row
    int32_t stages;
    uint64_t wait_limit_ns;
};

// Zero-fill every row r of `base` (row_bytes each, 16-byte multiple) with
// pad_mask[r] != 0, r = worker, worker + nworkers, ... ; one warp per worker.
__device__ __forceinline__ void zero_pad_rows_warp(uint8_t *base, const uint8_t *pad_mask, int64_t rows_max,
                                                   uint32_t row_bytes, int64_t worker, int64_t nworkers)
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
            uint8_t *row = base + (r0 + static_cast<int64_t>(src) * nworkers) * row_bytes;
            for (uint32_t off = lane * 16u; off < row_bytes; off += 32u * 16u)
                st_u4(row + off, z);
        }
    }
}

__global__ void __launch_bounds__(32) permute_kernel(PermuteArgs a)
{
    extern __shared__ __align__(128) uint8_t permute_smem[];
    __shared__ __align__(8) uint64_t bars[PERMUTE_MAX_STAGES];
    const int lane = threadIdx.x;
    const int S = a.stages;
    const int64_t units = a.N * a.nseg;
    const int64_t stride = gridDim.x;
    int64_t u0 = blockIdx.x;
    bool ok = true;

    if (lane == 0) {
        for (int s = 0; s < S; ++s)
            mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();

    const uint64_t policy = policy_evict_first();
    auto seg_len = [&](int seg) -> uint32_t {
        const uint32_t off = static_cast<uint32_t>(seg) * a.seg_bytes;
        return min(a.seg_bytes, a.row_bytes - off);
    };
    auto issue_load = [&](int s, int64_t u) {
        const int64_t t = u / a.nseg;
        const int seg = static_cast<int>(u - t * a.nseg);
        const uint32_t len = seg_len(seg);
        mbar_arrive_expect_tx(&bars[s], len);
        bulk_g2s(permute_smem + static_cast<size_t>(s) * a.seg_bytes,
                 a.hidden + t * a.row_bytes + static_cast<size_t>(seg) * a.seg_bytes, len, &bars[s], policy);
    };

    // prologue: fill the ring
    if (lane == 0)
        for (int s = 0; s < S; ++s) {
            const int64_t u = u0 + s * stride;
            if (u < units)
                issue_load(s, u);
        }

    int64_t i = 0;
    for (int64_t u = u0; u < units; u += stride, ++i) {
        const int s = static_cast<int>(i % S);
        const uint32_t parity = static_cast<uint32_t>((i / S) & 1);
        const int64_t t = u / a.nseg;
        const int seg = static_cast<int>(u - t * a.nseg);
        const uint32_t len = seg_len(seg);
        // destination rows of this token: lane j holds dest_row[t, j]
        int32_t d = lane < a.k ? __ldg(a.dest_row + t * a.k + lane) : -1;
        if (d < -1 || d >= a.rows_max) {
            atomicOr(a.status, MOE_DEV_ROW_RANGE);
            d = -1;
        }
        uint32_t valid = __ballot_sync(0xffffffffu, d >= 0);
        if (lane == 0) {
            if (!mbar_wait_bounded(&bars[s], parity, a.wait_limit_ns)) {
                atomicOr(a.status, MOE_DEV_TIMEOUT);
                ok = false;
            }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok)
            break;
        // lane 0 issues the stores; every lane takes part in the shuffles
        while (valid) {
            const int j = __ffs(valid) - 1;
            valid &= valid - 1;
            const int32_t row = __shfl_sync(0xffffffffu, d, j);
            if (lane == 0)
                bulk_s2g(a.send + static_cast<int64_t>(row) * a.row_bytes + static_cast<size_t>(seg) * a.seg_bytes,
                         permute_smem + static_cast<size_t>(s) * a.seg_bytes, len);
        }
        if (lane == 0) {
            bulk_commit();
            // refill the slot used by the previous unit once its stores have read it
            if (i >= 1) {
                bulk_wait_read<1>();
                const int ps = static_cast<int>((i - 1) % S);
                const int64_t nu = u - stride + static_cast<int64_t>(S) * stride;
                if (nu < units)
                    issue_load(ps, nu);
            }
        }
        __syncwarp();
    }
    if (lane == 0) {
        bulk_wait_all();
        if (!ok) {
            // Units i .. max(S-1, i+S-2) of this CTA were loaded but not
            // consumed: let those loads land before the CTA's shared memory
            // goes away.
            const int64_t last = i + S - 2 > S - 1 ? i + S - 2 : S - 1;
            for (int64_t v = i; v <= last; ++v)
                if (u0 + v * stride < units)
                    (void)mbar_wait_bounded(&bars[v % S], static_cast<uint32_t>((v / S) & 1), a.wait_limit_ns);
        }
    }
    __syncwarp();

    zero_pad_rows_warp(a.send, a.pad_mask, a.rows_max, a.row_bytes, blockIdx.x, gridDim.x);
}

} // namespace moert
