// combine.cuh — the combine gather-reduce and both backward passes.
//
// DeepSpeed EP page, restore_combined: weighted expert outputs are added back
// per token one top-k slot at a time in ascending slot order, so the
// accumulation order is fixed. Megatron MoE page, combine. Megatron MORI
// page: backward passes use receiver-side indices and probs.
//
// Combine: one thread per 16-byte column chunk (8 bf16) of one token. All k
// source rows of the chunk are loaded up front (k independent 16-byte
// streaming loads in flight per thread), then accumulated in fp32 with one
// fmaf per kept slot in ascending j from +0, and rounded once to bf16
// (cvt.rn.bf16x2). No atomics: every output element has one writer. A warp
// covers 512 contiguous bytes of each source row. Short rows with one or two
// slots take combine_rows_kernel: several tokens per CTA, four chunks per
// thread, the same arithmetic.
//
// Combine backward: one CTA per token walks the row in 16-byte chunks,
// writes grad_y[dest_row[t,j]] = bf16(fp32(p[t,j] * g)) and accumulates the
// per-slot dot products <g, y[dest_row[t,j]]> in fp32, reduced across the CTA
// in a fixed order (deterministic). Extra CTAs zero the pad rows of grad_y.
#pragma once

#include <cstdint>
#include <type_traits>

#include "moe_rt.h"
#include "permute.cuh"
#include "ptx.cuh"

namespace moert {

constexpr int COMBINE_THREADS = 256; // widest CTA; the host picks 32..256 to split the row evenly
constexpr int COMBINE_BWD_THREADS = 128;
constexpr int COMBINE_MAX_K = 32;

struct CombineArgs {
    const uint4 *y;          // [rows_max, V]
    const int32_t *dest_row; // [N, k]
    const float *probs;      // [N, k] or null (unit weights)
    uint4 *out;              // [N, V]
    uint32_t *status;
    int64_t N;
    int64_t rows_max;
    int32_t k;
    int32_t V;       // 16-byte chunks per row (H / 8)
    int32_t nchunks; // CTAs per token
    int32_t last_first; // 1: tokens are taken last first (see combine_kernel)
    // restore after TP folding: T peer buffers and row maps (y / dest_row unused)
    int32_t T;
    const uint4 *ys[MOE_MAX_TP];
    const int32_t *dests[MOE_MAX_TP];
    // expert-parallel exchange: slot j's row d of expert q sits in the receive
    // buffer of q's owner at row ep_base[q] + d - ep_offsets[q]
    const uint4 *const *ep_peers; // [R] device pointers
    const int32_t *phys_idx;      // [N, k]
    const int32_t *ep_base;       // [E]
    const int32_t *ep_offsets;    // [E + 1]
    int64_t recv_max;
    int32_t E, E_loc;
};

// Where the combine reads slot rows from.
enum CombineSrc : int { SRC_LOCAL = 0, SRC_TP_PEERS = 1, SRC_EP = 2 };

__device__ __forceinline__ void fma8(float (&acc)[8], float p, const uint4 &y)
{
    acc[0] = __fmaf_rn(p, bf16_lo(y.x), acc[0]);
    acc[1] = __fmaf_rn(p, bf16_hi(y.x), acc[1]);
    acc[2] = __fmaf_rn(p, bf16_lo(y.y), acc[2]);
    acc[3] = __fmaf_rn(p, bf16_hi(y.y), acc[3]);
    acc[4] = __fmaf_rn(p, bf16_lo(y.z), acc[4]);
    acc[5] = __fmaf_rn(p, bf16_hi(y.z), acc[5]);
    acc[6] = __fmaf_rn(p, bf16_lo(y.w), acc[6]);
    acc[7] = __fmaf_rn(p, bf16_hi(y.w), acc[7]);
}

__device__ __forceinline__ uint4 pack8(const float (&acc)[8])
{
    return make_uint4(pack_bf16x2_rn(acc[0], acc[1]), pack_bf16x2_rn(acc[2], acc[3]),
                      pack_bf16x2_rn(acc[4], acc[5]), pack_bf16x2_rn(acc[6], acc[7]));
}

// Slot metadata of token t: lane j < k holds dest_row[t,j] and its weight.
__device__ __forceinline__ void load_slot_meta(const int32_t *dest_row, const float *probs, int64_t t, int k,
                                               int64_t rows_max, uint32_t *status, int32_t &d, float &p)
{
    const int lane = threadIdx.x & 31;
    d = -1;
    p = 0.0f;
    if (lane < k) {
        d = __ldg(dest_row + t * k + lane);
        p = probs != nullptr ? __ldg(probs + t * k + lane) : 1.0f;
        if (d < -1 || d >= rows_max) {
            atomicOr(status, MOE_DEV_ROW_RANGE);
            d = -1;
        }
    }
}

// Restore after TP folding: slot j of token t lives in the one peer buffer whose
// row map has a row for it. Lane j < k finds that peer and the row and returns
// the row's address (null if no peer holds the slot), so the per-thread gather
// needs no per-slot peer selection.
__device__ __forceinline__ const uint4 *peer_base(const CombineArgs &a, int32_t src)
{
    const uint4 *base = a.ys[0];
#pragma unroll
    for (int i = 1; i < MOE_MAX_TP; ++i)
        base = (src == i) ? a.ys[i] : base;
    return base;
}

__device__ __forceinline__ void load_slot_meta_peers(const CombineArgs &a, int64_t t, int k, const uint4 *&row,
                                                     float &p)
{
    const int lane = threadIdx.x & 31;
    row = nullptr;
    p = 0.0f;
    if (lane < k) {
        p = a.probs != nullptr ? __ldg(a.probs + t * k + lane) : 1.0f;
        int32_t r[MOE_MAX_TP];
#pragma unroll
        for (int q = 0; q < MOE_MAX_TP; ++q)
            r[q] = q < a.T ? __ldg(a.dests[q] + t * k + lane) : -1;
        int32_t d = -1, src = 0;
#pragma unroll
        for (int q = 0; q < MOE_MAX_TP; ++q) {
            if (r[q] < -1 || r[q] >= a.rows_max) {
                atomicOr(a.status, MOE_DEV_ROW_RANGE);
            } else if (r[q] >= 0 && d < 0) {
                d = r[q];
                src = q;
            }
        }
        if (d >= 0)
            row = peer_base(a, src) + static_cast<int64_t>(d) * a.V;
    }
}

// Expert-parallel exchange: lane j < k finds slot j's row in the receive buffer
// of the rank owning its expert and returns its address (null if the slot has no
// row or the row lies outside the receive buffer, the latter flagged).
__device__ __forceinline__ void load_slot_meta_ep(const CombineArgs &a, int64_t t, int k, const uint4 *&row, float &p)
{
    const int lane = threadIdx.x & 31;
    row = nullptr;
    p = 0.0f;
    if (lane < k) {
        p = a.probs != nullptr ? __ldg(a.probs + t * k + lane) : 1.0f;
        const int32_t d = __ldg(a.dest_row + t * k + lane);
        const int32_t q = d >= 0 ? __ldg(a.phys_idx + t * k + lane) : -1;
        if (d >= 0 && (q < 0 || q >= a.E || d >= a.rows_max)) {
            atomicOr(a.status, MOE_DEV_ROW_RANGE);
        } else if (d >= 0) {
            const int64_t r = static_cast<int64_t>(__ldg(a.ep_base + q)) + d - __ldg(a.ep_offsets + q);
            if (r < 0 || r >= a.recv_max)
                atomicOr(a.status, MOE_DEV_ROW_RANGE);
            else
                row = a.ep_peers[q / a.E_loc] + r * a.V;
        } else if (d < -1) {
            atomicOr(a.status, MOE_DEV_ROW_RANGE);
        }
    }
}

// K > 0: top-k fixed at compile time; K == 0: runtime k <= 32.
// SRC: one buffer, the TP peers' buffers (restore), or the EP receive buffers.
template <int K, int SRC = SRC_LOCAL>
__global__ void __launch_bounds__(COMBINE_THREADS, 4) combine_kernel(CombineArgs a)
{
    pdl_trigger();
    pdl_wait();
    // With last_first, tokens are taken last first: the rows a preceding token-ordered
    // pass (the permute) wrote last are the ones still in L2 when this kernel starts.
    // Each output row has one writer, so the order changes no result.
    const int64_t tb = blockIdx.x / a.nchunks;
    const int c = static_cast<int>(blockIdx.x - tb * a.nchunks);
    const int64_t t = a.last_first ? a.N - 1 - tb : tb;
    const int v = c * blockDim.x + threadIdx.x;
    const int k = K > 0 ? K : a.k;

    // lane j < k: slot j's source row and weight. One buffer: the row index;
    // TP peers: the row's address in the peer buffer that holds it.
    constexpr bool PTR = SRC != SRC_LOCAL; // slots resolved to addresses
    using Src = typename std::conditional<PTR, const uint4 *, int32_t>::type;
    Src src;
    float p;
    if constexpr (SRC == SRC_TP_PEERS) {
        load_slot_meta_peers(a, t, k, src, p);
    } else if constexpr (SRC == SRC_EP) {
        load_slot_meta_ep(a, t, k, src, p);
    } else {
        load_slot_meta(a.dest_row, a.probs, t, k, a.rows_max, a.status, src, p);
    }
    auto shfl_src = [&](int j) -> Src {
        if constexpr (PTR)
            return reinterpret_cast<const uint4 *>(
                __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(src), j));
        else
            return __shfl_sync(0xffffffffu, src, j);
    };
    auto valid = [](Src s) -> bool {
        if constexpr (PTR)
            return s != nullptr;
        else
            return s >= 0;
    };
    auto row_ptr = [&](Src s) -> const uint4 * {
        if constexpr (PTR)
            return s;
        else
            return a.y + static_cast<int64_t>(s) * a.V;
    };
    auto none = []() -> Src {
        if constexpr (PTR)
            return nullptr;
        else
            return -1;
    };

    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
        acc[e] = 0.0f;

    if constexpr (K > 0) {
        Src sj[K];
        float pj[K];
        uint4 yj[K];
#pragma unroll
        for (int j = 0; j < K; ++j) {
            sj[j] = shfl_src(j);
            pj[j] = __shfl_sync(0xffffffffu, p, j);
        }
        if (v >= a.V)
            return;
#pragma unroll
        for (int j = 0; j < K; ++j)
            if (valid(sj[j]))
                yj[j] = ld_stream_u4(row_ptr(sj[j]) + v);
#pragma unroll
        for (int j = 0; j < K; ++j)
            if (valid(sj[j]))
                fma8(acc, pj[j], yj[j]);
    } else {
        const bool active = v < a.V;
        for (int j0 = 0; j0 < k; j0 += 4) {
            Src sj[4];
            float pj[4];
            uint4 yj[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                sj[u] = shfl_src((j0 + u) & 31);
                pj[u] = __shfl_sync(0xffffffffu, p, (j0 + u) & 31);
                if (j0 + u >= k || !active)
                    sj[u] = none();
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (valid(sj[u]))
                    yj[u] = ld_stream_u4(row_ptr(sj[u]) + v);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (valid(sj[u]))
                    fma8(acc, pj[u], yj[u]);
        }
        if (!active)
            return;
    }
    st_u4(a.out + t * a.V + v, pack8(acc));
}

// Combine of short rows with one or two slots (one buffer). With one 16-byte
// chunk per thread such a token gives a CTA at most 32 bytes to load per
// thread, too little in flight to cover the memory latency, and tokens whose
// slots were all dropped only load their metadata and store zeros. Here a
// token's row is covered by V / COMBINE_ROW_CPT threads (whole warps), each
// owning COMBINE_ROW_CPT chunks a row-quarter apart, and a CTA holds several
// tokens: every load of every chunk is issued before the first multiply-add.
// The grid holds four CTAs per SM and each token group walks the tokens with a
// stride, loading the next token's slot metadata while it loads and stores the
// current one, so a token whose slots were all dropped costs only its stores
// (capacity workload, in a replayed step: 16.6 -> 15.8 us).
// The arithmetic per element is the one of combine_kernel (fma chain in
// ascending j from +0, one bf16 rounding). The host takes this kernel for k <= 2
// and V in {128, 256, 512, 1024}, so COMBINE_THREADS is a multiple of the
// threads per token.
constexpr int COMBINE_ROW_CPT = 4;

template <int K>
__global__ void __launch_bounds__(COMBINE_THREADS, 4) combine_rows_kernel(CombineArgs a)
{
    pdl_trigger();
    pdl_wait();
    const int tpt = a.V / COMBINE_ROW_CPT; // threads per token: 32, 64, 128 or 256
    const int groups = COMBINE_THREADS / tpt;
    const int u = static_cast<int>(threadIdx.x) / tpt, l = static_cast<int>(threadIdx.x) - u * tpt;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * groups;
    int64_t tb = static_cast<int64_t>(blockIdx.x) * groups + u;
    if (tb >= a.N) // whole warps: tpt is a multiple of 32
        return;
    auto token = [&](int64_t b) { return a.last_first ? a.N - 1 - b : b; };
    int32_t d;
    float p;
    load_slot_meta(a.dest_row, a.probs, token(tb), K, a.rows_max, a.status, d, p);
    for (; tb < a.N; tb += stride) {
        const int64_t t = token(tb);
        int32_t dj[K];
        float pj[K];
#pragma unroll
        for (int j = 0; j < K; ++j) {
            dj[j] = __shfl_sync(0xffffffffu, d, j);
            pj[j] = __shfl_sync(0xffffffffu, p, j);
        }
        if (tb + stride < a.N) // the next token's slots, while this one is loaded and stored
            load_slot_meta(a.dest_row, a.probs, token(tb + stride), K, a.rows_max, a.status, d, p);
        uint4 yj[K][COMBINE_ROW_CPT];
#pragma unroll
        for (int j = 0; j < K; ++j)
            if (dj[j] >= 0) {
                const uint4 *row = a.y + static_cast<int64_t>(dj[j]) * a.V + l;
#pragma unroll
                for (int i = 0; i < COMBINE_ROW_CPT; ++i)
                    yj[j][i] = ld_stream_u4(row + i * tpt);
            }
        uint4 *out = a.out + t * a.V + l;
#pragma unroll
        for (int i = 0; i < COMBINE_ROW_CPT; ++i) {
            float acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                acc[e] = 0.0f;
#pragma unroll
            for (int j = 0; j < K; ++j)
                if (dj[j] >= 0)
                    fma8(acc, pj[j], yj[j][i]);
            st_u4(out + i * tpt, pack8(acc));
        }
    }
}

struct CombineBwdArgs {
    const uint4 *grad_out;   // [N, V]
    const uint4 *y;          // [rows_max, V]
    const int32_t *dest_row; // [N, k]
    const float *probs;      // [N, k]
    const uint8_t *pad_mask; // [rows_max]
    uint4 *grad_y;           // [rows_max, V]
    float *grad_probs;       // [N, k]
    uint32_t *status;
    int64_t N;
    int64_t rows_max;
    int32_t k;
    int32_t V;
    int32_t zero_blocks; // trailing CTAs that zero pad rows of grad_y
    // expert-parallel exchange: y and grad_y rows live in the owners' buffers
    // (receive order), row ep_base[q] + d - ep_offsets[q] of owner q / E_loc
    const uint4 *const *ep_peer_y; // [R] device pointers
    uint4 *const *ep_peer_gy;      // [R] device pointers
    const int32_t *phys_idx;       // [N, k]
    const int32_t *ep_base;        // [E]
    const int32_t *ep_offsets;     // [E + 1]
    const int32_t *ep_tokens;      // [E]
    int64_t recv_max;
    int32_t E, E_loc, R;
};

__device__ __forceinline__ float dot8(float s, const uint4 &g, const uint4 &y)
{
    s = __fmaf_rn(bf16_lo(g.x), bf16_lo(y.x), s);
    s = __fmaf_rn(bf16_hi(g.x), bf16_hi(y.x), s);
    s = __fmaf_rn(bf16_lo(g.y), bf16_lo(y.y), s);
    s = __fmaf_rn(bf16_hi(g.y), bf16_hi(y.y), s);
    s = __fmaf_rn(bf16_lo(g.z), bf16_lo(y.z), s);
    s = __fmaf_rn(bf16_hi(g.z), bf16_hi(y.z), s);
    s = __fmaf_rn(bf16_lo(g.w), bf16_lo(y.w), s);
    s = __fmaf_rn(bf16_hi(g.w), bf16_hi(y.w), s);
    return s;
}

__device__ __forceinline__ uint4 scale8(float p, const uint4 &g)
{
    return make_uint4(pack_bf16x2_rn(__fmul_rn(p, bf16_lo(g.x)), __fmul_rn(p, bf16_hi(g.x))),
                      pack_bf16x2_rn(__fmul_rn(p, bf16_lo(g.y)), __fmul_rn(p, bf16_hi(g.y))),
                      pack_bf16x2_rn(__fmul_rn(p, bf16_lo(g.z)), __fmul_rn(p, bf16_hi(g.z))),
                      pack_bf16x2_rn(__fmul_rn(p, bf16_lo(g.w)), __fmul_rn(p, bf16_hi(g.w))));
}

// Deterministic CTA-wide sum: warp butterfly, then warps in index order.
__device__ __forceinline__ float cta_sum_fixed(float v, float *s_red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0)
        s_red[warp] = v;
    __syncthreads();
    float total = 0.0f;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w)
        total += s_red[w];
    return total;
}

// EP: y and grad_y rows are in the owners' buffers of the exchange.
template <int K, bool EP = false>
__global__ void __launch_bounds__(COMBINE_BWD_THREADS) combine_backward_kernel(CombineBwdArgs a)
{
    __shared__ float s_red[COMBINE_BWD_THREADS / 32];
    __shared__ float s_part[COMBINE_BWD_THREADS / 32][K > 0 ? K : 1];
    __shared__ const uint4 *s_py[EP ? MOE_MAX_EP_RANKS : 1];
    __shared__ uint4 *s_pg[EP ? MOE_MAX_EP_RANKS : 1];
    pdl_trigger();
    pdl_wait();
    if (blockIdx.x >= a.N) {
        const int64_t workers = static_cast<int64_t>(a.zero_blocks) * (COMBINE_BWD_THREADS / 32);
        const int64_t worker = (blockIdx.x - a.N) * (COMBINE_BWD_THREADS / 32) + (threadIdx.x >> 5);
        if constexpr (EP)
            ep_zero_pads_warp(a.ep_peer_gy, a.ep_base, a.ep_offsets, a.ep_tokens, a.E, a.E_loc, a.V, a.recv_max,
                              a.status, worker, workers);
        else
            zero_pad_rows_warp(a.grad_y, a.pad_mask, a.rows_max, a.V, worker, workers);
        return;
    }
    const int64_t t = blockIdx.x;
    const int k = K > 0 ? K : a.k;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int32_t d;
    float p;
    load_slot_meta(a.dest_row, a.probs, t, k, a.rows_max, a.status, d, p);
    // EP: lane j's slot row in its owner's buffers (row in d, owner in own), -1 if none
    int32_t own = 0;
    if constexpr (EP) {
        if (threadIdx.x < a.R) {
            s_py[threadIdx.x] = a.ep_peer_y[threadIdx.x];
            s_pg[threadIdx.x] = a.ep_peer_gy[threadIdx.x];
        }
        if (d >= 0) {
            const int32_t q = __ldg(a.phys_idx + t * k + lane);
            const int64_t r = q >= 0 && q < a.E
                                  ? static_cast<int64_t>(__ldg(a.ep_base + q)) + d - __ldg(a.ep_offsets + q)
                                  : -1;
            if (r < 0 || r >= a.recv_max) {
                atomicOr(a.status, MOE_DEV_ROW_RANGE);
                d = -1;
            } else {
                d = static_cast<int32_t>(r);
                own = q / a.E_loc;
            }
        }
        __syncthreads();
    }
    auto y_row = [&](int32_t row, int32_t owner) -> const uint4 * {
        if constexpr (EP)
            return s_py[owner] + static_cast<int64_t>(row) * a.V;
        else
            return a.y + static_cast<int64_t>(row) * a.V;
    };
    auto gy_row = [&](int32_t row, int32_t owner) -> uint4 * {
        if constexpr (EP)
            return s_pg[owner] + static_cast<int64_t>(row) * a.V;
        else
            return a.grad_y + static_cast<int64_t>(row) * a.V;
    };
    const uint4 *g_row = a.grad_out + t * a.V;

    if constexpr (K > 0) {
        int32_t dj[K], oj[K];
        float pj[K];
        float part[K];
#pragma unroll
        for (int j = 0; j < K; ++j) {
            dj[j] = __shfl_sync(0xffffffffu, d, j);
            oj[j] = EP ? __shfl_sync(0xffffffffu, own, j) : 0;
            pj[j] = __shfl_sync(0xffffffffu, p, j);
            part[j] = 0.0f;
        }
        for (int v = threadIdx.x; v < a.V; v += COMBINE_BWD_THREADS) {
            const uint4 g = ld_stream_u4(g_row + v);
            uint4 yj[K];
#pragma unroll
            for (int j = 0; j < K; ++j)
                if (dj[j] >= 0)
                    yj[j] = ld_stream_u4(y_row(dj[j], oj[j]) + v);
#pragma unroll
            for (int j = 0; j < K; ++j)
                if (dj[j] >= 0) {
                    st_u4(gy_row(dj[j], oj[j]) + v, scale8(pj[j], g));
                    part[j] = dot8(part[j], g, yj[j]);
                }
        }
#pragma unroll
        for (int j = 0; j < K; ++j) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                part[j] += __shfl_xor_sync(0xffffffffu, part[j], o);
        }
        if (lane == 0) {
#pragma unroll
            for (int j = 0; j < K; ++j)
                s_part[warp][j] = part[j];
        }
        __syncthreads();
        if (threadIdx.x < K) { // lane j of warp 0 holds slot j's own row in d
            const int j = threadIdx.x;
            float total = 0.0f;
            for (int w = 0; w < COMBINE_BWD_THREADS / 32; ++w)
                total += s_part[w][j];
            a.grad_probs[t * K + j] = d >= 0 ? total : 0.0f;
        }
    } else {
        for (int j = 0; j < k; ++j) {
            const int32_t dj = __shfl_sync(0xffffffffu, d, j);
            const int32_t oj = EP ? __shfl_sync(0xffffffffu, own, j) : 0;
            const float pj = __shfl_sync(0xffffffffu, p, j);
            float part = 0.0f;
            if (dj >= 0) {
                for (int v = threadIdx.x; v < a.V; v += COMBINE_BWD_THREADS) {
                    const uint4 g = __ldg(g_row + v);
                    const uint4 y = ld_stream_u4(y_row(dj, oj) + v);
                    st_u4(gy_row(dj, oj) + v, scale8(pj, g));
                    part = dot8(part, g, y);
                }
            }
            const float total = cta_sum_fixed(part, s_red);
            if (threadIdx.x == 0)
                a.grad_probs[t * k + j] = dj >= 0 ? total : 0.0f;
        }
    }
}

} // namespace moert
