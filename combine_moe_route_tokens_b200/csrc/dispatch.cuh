// dispatch.cuh — the fused dispatch: the layout's fill pass and the permute in
// one kernel (Megatron MORI page: the permute is fused into the dispatch node;
// Megatron MoE page, dispatch_postprocess: permuted tokens per expert).
//
// Runs after layout_count_kernel. Leading "row" CTAs derive the layout tables,
// CTA 0 of them writes the tables out, and each marks its share of the
// send-buffer rows (pad_mask, 0 / -1 / 0 row maps and zero rows for pad and
// tail rows). Every other CTA copies tokens like permute.cuh: a group of 32, 64
// or 128 threads per token (piece), which loads its token's row before waiting
// for the count pass (the count pass lets this kernel launch only after its
// own wait returned, so every input of the call is complete), derives the
// tables, turns its token's logical ordinals into destination rows, writes the
// per-assignment outputs and the inverse row maps, and stores the row k times.
// The results equal moe_dispatch_layout followed by moe_permute bit for bit.
#pragma once

#include <cstdint>

#include "layout.cuh"
#include "permute.cuh"
#include "ptx.cuh"

namespace moert {

struct DispatchArgs {
    LayoutArgs L;
    const uint4 *hidden; // [N, V]
    uint4 *send;         // [rows_max, V]
    int64_t N;
    int32_t V;        // 16-byte chunks per row
    int32_t group;    // threads per token piece: 32, 64 or 128
    int32_t pieces;   // pieces per token
    int32_t row_ctas; // leading CTAs that handle the row pass (at least 1: CTA 0 writes the tables)
};

// 16-byte load cached in L2 only (issued before the grid dependency wait).
__device__ __forceinline__ uint4 ld_cg_u4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

template <bool REROUTE, bool DENSE>
__global__ void __launch_bounds__(PERMUTE_THREADS) dispatch_kernel(DispatchArgs d)
{
    extern __shared__ __align__(16) int32_t dispatch_smem[];
    __shared__ int32_t s_dest[PERMUTE_THREADS / 32][32];
    const LayoutArgs &a = d.L;
    const int tid = threadIdx.x, lane = tid & 31;
    const bool row_cta = blockIdx.x < static_cast<uint32_t>(d.row_ctas);
    const int groups = PERMUTE_THREADS / d.group;
    const int g = tid / d.group, gt = tid - g * d.group;
    const int64_t unit = (static_cast<int64_t>(blockIdx.x) - d.row_ctas) * groups + g;
    const bool active = !row_cta && unit < d.N * d.pieces;
    const int64_t t = active ? unit / d.pieces : 0;
    const int piece = static_cast<int>(unit - t * d.pieces);
    const int32_t c0 = piece * (d.group * PERMUTE_CHUNKS) + gt;
    const uint4 *src = d.hidden + t * d.V;
    uint4 v[PERMUTE_CHUNKS];
    // Without a capacity every token keeps a slot, so its row is read before the
    // wait; with one, a token whose slots were all dropped is not read at all.
    const bool early = a.C == 0;
    if (active && early) {
#pragma unroll
        for (int c = 0; c < PERMUTE_CHUNKS; ++c) {
            const int32_t idx = c0 + c * d.group;
            if (idx < d.V)
                v[c] = ld_cg_u4(src + idx);
        }
    }
    pdl_trigger();
    pdl_wait(); // the count pass is complete
    // this group's slots: logical id and ordinal (the count pass's output) and prob
    int32_t e = -1, lo = -1;
    float p = 0.0f;
    const int64_t i = t * a.k + gt;
    if (active && gt < a.k) {
        e = __ldg(a.topk_idx + i);
        if (e < -1 || e >= a.E_log) // reported by the count pass
            e = -1;
        lo = __ldcg(a.out.ordinal + i);
        if (a.topk_probs != nullptr)
            p = __ldg(a.topk_probs + i);
    }
    LayoutTables tb = layout_tables_carve(a, dispatch_smem);
    layout_tables_cta(a, tb);

    if (row_cta) {
        if (blockIdx.x == 0)
            layout_tables_store(a, tb);
        // the row pass: classify rows, one per thread; each warp zeroes its pad rows together
        const int64_t stride = static_cast<int64_t>(d.row_ctas) * PERMUTE_THREADS;
        const uint4 z = make_uint4(0, 0, 0, 0);
        for (int64_t r0 = static_cast<int64_t>(blockIdx.x) * PERMUTE_THREADS + (tid & ~31); r0 < a.rows_max;
             r0 += stride) {
            const int64_t row = r0 + lane;
            const bool pad = row < a.rows_max && layout_emit_row(a, tb, row, DENSE);
            uint32_t ballot = __ballot_sync(0xffffffffu, pad);
            while (ballot) {
                const int src = __ffs(ballot) - 1;
                ballot &= ballot - 1;
                uint4 *dst = d.send + (r0 + src) * d.V;
                for (int32_t c = lane; c < d.V; c += 32)
                    st_u4(dst + c, z);
            }
        }
        return;
    }
    if (active && gt < a.k) {
        // piece 0 of the token writes the per-assignment outputs; every piece needs the rows
        s_dest[g][gt] = layout_emit_assignment<REROUTE>(a, tb, i, e, lo, p, DENSE, piece == 0);
    }
    __syncthreads();
    if (!active)
        return;
    if (!early) {
        bool any = false;
        for (int j = 0; j < a.k; ++j)
            any |= s_dest[g][j] >= 0;
        if (!any)
            return;
#pragma unroll
        for (int c = 0; c < PERMUTE_CHUNKS; ++c) {
            const int32_t idx = c0 + c * d.group;
            if (idx < d.V)
                v[c] = ld_stream_u4(src + idx);
        }
    }
    for (int j = 0; j < a.k; ++j) {
        const int32_t row = s_dest[g][j];
        if (row < 0)
            continue;
        uint4 *dst = d.send + static_cast<int64_t>(row) * d.V;
#pragma unroll
        for (int c = 0; c < PERMUTE_CHUNKS; ++c) {
            const int32_t idx = c0 + c * d.group;
            if (idx < d.V)
                st_u4(dst + idx, v[c]);
        }
    }
}

} // namespace moert
