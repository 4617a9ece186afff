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
// dispatch_bulk_kernel (below) is the same work with the rows staged through
// shared memory by bulk copies.
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

// ---- bulk-copy (TMA) helpers: CTA-local shared memory, no multicast
__device__ __forceinline__ uint32_t smem_u32(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
                 : "=r"(ok)
                 : "r"(smem_u32(bar)), "r"(parity)
                 : "memory");
    return ok != 0;
}
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gsrc, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(smem_dst)),
                 "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void bulk_store(void *gdst, const void *smem_src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(smem_u32(smem_src)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

constexpr int TMA_THREADS = 128;
constexpr int TMA_MAX_TOKENS = 8;

// The same work staged through shared memory with bulk copies (MOE_FLAG_DISPATCH_BULK_COPY):
// one thread of a CTA loads the CTA's token rows (or one piece of a long row) into
// shared memory with cp.async.bulk (mbarrier completion, before the wait when every
// token keeps a slot) and, once the rows are known, stores each kept row with a bulk
// shared-to-global copy. 48 registers a thread instead of ~80, but on B200 the bulk
// stores of this one-read / k-write scatter are slower than the vector stores
// (measured in-graph: 4096 x 7168 top-8 step 188.9 us against 178.2 us), so it is
// not the default. d.group = tokens per CTA (tpc), d.pieces = pieces per token
// (tpc == 1 when > 1), d.V = 16-byte chunks per row; piece bytes = ceil(V / pieces) * 16.
template <bool REROUTE, bool DENSE>
__global__ void __launch_bounds__(TMA_THREADS) dispatch_bulk_kernel(DispatchArgs d)
{
    extern __shared__ __align__(16) int32_t bulk_smem[]; // bulk copies need 16-byte alignment
    __shared__ int32_t s_dest[TMA_MAX_TOKENS][32];
    __shared__ __align__(8) uint64_t s_bar;
    const LayoutArgs &a = d.L;
    const int tid = threadIdx.x, lane = tid & 31;
    const bool row_cta = blockIdx.x < static_cast<uint32_t>(d.row_ctas);
    const int tpc = d.group;
    const int32_t pchunks = (d.V + d.pieces - 1) / d.pieces;
    const int64_t cta = static_cast<int64_t>(blockIdx.x) - d.row_ctas;
    // this CTA: tokens [t0, t0 + ntok) and piece `piece` of each
    const int64_t t0 = d.pieces > 1 ? cta / d.pieces : cta * tpc;
    const int piece = d.pieces > 1 ? static_cast<int>(cta - t0 * d.pieces) : 0;
    const int64_t left = d.N - t0;
    const int ntok = row_cta ? 0 : static_cast<int>(left < tpc ? left : tpc);
    const int32_t c_first = piece * pchunks;
    const int32_t nchunks = min(pchunks, d.V - c_first);
    const uint32_t pbytes = static_cast<uint32_t>(nchunks) * 16u;
    LayoutTables tb = layout_tables_carve(a, bulk_smem);
    // the row buffer follows the tables, at a 128-byte offset
    const size_t tw = layout_tables_smem_words(a.E_log, a.E);
    uint4 *s_rows = reinterpret_cast<uint4 *>(bulk_smem + ((tw + 31) & ~size_t(31)));
    const bool early = a.C == 0;
    if (!row_cta && tid == 0) {
        mbar_init(&s_bar, 1);
        mbar_fence_init();
        if (early && ntok > 0) { // the tokens' rows, before the wait
            mbar_expect_tx(&s_bar, pbytes * ntok);
            for (int u = 0; u < ntok; ++u)
                bulk_load(s_rows + static_cast<int64_t>(u) * pchunks, d.hidden + (t0 + u) * d.V + c_first, pbytes,
                          &s_bar);
        }
    }
    pdl_trigger();
    pdl_wait(); // the count pass is complete
    // metadata of this CTA's slots, loaded before the tables so the round trips overlap
    int32_t e[2] = {-1, -1}, lo[2] = {-1, -1};
    float p[2] = {0.0f, 0.0f};
    const int nslots = ntok * a.k;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int s = tid + u * TMA_THREADS;
        if (s < nslots) {
            const int64_t i = t0 * a.k + s;
            e[u] = __ldg(a.topk_idx + i);
            if (e[u] < -1 || e[u] >= a.E_log)
                e[u] = -1;
            lo[u] = __ldcg(a.out.ordinal + i);
            if (a.topk_probs != nullptr)
                p[u] = __ldg(a.topk_probs + i);
        }
    }
    layout_tables_cta(a, tb);

    if (row_cta) {
        if (blockIdx.x == 0)
            layout_tables_store(a, tb);
        const int64_t stride = static_cast<int64_t>(d.row_ctas) * TMA_THREADS;
        const uint4 z = make_uint4(0, 0, 0, 0);
        for (int64_t r0 = static_cast<int64_t>(blockIdx.x) * TMA_THREADS + (tid & ~31); r0 < a.rows_max;
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
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int s = tid + u * TMA_THREADS;
        if (s < nslots)
            s_dest[s / a.k][s % a.k] = layout_emit_assignment<REROUTE>(a, tb, t0 * a.k + s, e[u], lo[u], p[u], DENSE,
                                                                      piece == 0);
    }
    __syncthreads();
    if (tid != 0 || ntok == 0)
        return;
    if (!early) { // load only the tokens that keep a slot
        uint32_t want = 0;
        for (int u = 0; u < ntok; ++u) {
            bool any = false;
            for (int j = 0; j < a.k; ++j)
                any |= s_dest[u][j] >= 0;
            if (any)
                want |= 1u << u;
        }
        if (want == 0)
            return;
        mbar_expect_tx(&s_bar, pbytes * __popc(want));
        for (int u = 0; u < ntok; ++u)
            if (want & (1u << u))
                bulk_load(s_rows + static_cast<int64_t>(u) * pchunks, d.hidden + (t0 + u) * d.V + c_first, pbytes,
                          &s_bar);
    }
    const uint64_t start = global_timer_ns();
    while (!mbar_try_wait(&s_bar, 0)) {
        if (global_timer_ns() - start > a.wait_limit_ns) { // cannot happen for a valid load; never store garbage
            atomicOr(a.out.status, MOE_DEV_TIMEOUT);
            const uint64_t again = global_timer_ns();
            while (!mbar_try_wait(&s_bar, 0) && global_timer_ns() - again < a.wait_limit_ns) {
            }
            return;
        }
    }
    for (int u = 0; u < ntok; ++u)
        for (int j = 0; j < a.k; ++j) {
            const int32_t row = s_dest[u][j];
            if (row >= 0)
                bulk_store(d.send + static_cast<int64_t>(row) * d.V + c_first, s_rows + static_cast<int64_t>(u) * pchunks,
                           pbytes);
        }
    bulk_commit();
    bulk_wait_read_all(); // the shared rows stay valid until the stores have read them
}

} // namespace moert
