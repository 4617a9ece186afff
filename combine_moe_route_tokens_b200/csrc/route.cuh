// route.cuh — router softmax + top-k, one warp per token.
//
// Megatron MoE page, MoELayer.router_and_preprocess: the router turns a
// token into routing probs and a top-k routing map; Megatron MORI page,
// router.py: padding tokens are masked out of routing.
//
// p[t,e] = expf(l - m) / sum_e expf(l - m) with m = max_e l, over all E
// (no renormalisation over the k chosen). The k chosen experts are the k
// largest logits in descending order, equal logits to the lower expert id;
// selection compares logits, so the ids never depend on expf rounding.
//
// Lane l holds experts l, l+32, ... as 32-bit order-preserving keys (0 marks
// an empty or already chosen slot). Each of the k rounds scans the lane's keys
// for its best (first occurrence = lowest id), takes the warp maximum with one
// redux.sync and, among the lanes holding it, the lowest expert id with a
// second; the owner clears that key. The key maps back to the logit exactly, so
// no shuffle is needed; lane j turns the j-th winner into its prob at the end.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace moert {

constexpr int ROUTE_WARPS_PER_BLOCK = 8;

// Order-preserving map float -> uint32 (larger float, larger key; never 0 for
// a real value); -0 is folded onto +0, which compare equal in IEEE.
__device__ __forceinline__ uint32_t route_key(float v)
{
    const uint32_t b = __float_as_uint(v + 0.0f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float route_unkey(uint32_t k)
{
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Lane l loads experts l, l+32, ... of one token's logits (-inf past E).
template <int VPL>
__device__ __forceinline__ void route_load(const float *__restrict__ row, int E, int lane, float (&v)[VPL])
{
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int e = i * 32 + lane;
        v[i] = e < E ? __ldg(row + e) : -INFINITY;
    }
}

// Softmax + top-k of one token held by the warp (route_load layout). Lane j < k
// ends with the j-th chosen expert id and its prob; other lanes get -1 / 0.
// Every lane of the warp must call it.
template <int VPL>
__device__ __forceinline__ void route_select(const float (&v)[VPL], int E, int k, int lane, int32_t &id, float &prob)
{
    float m = v[0];
#pragma unroll
    for (int i = 1; i < VPL; ++i)
        m = fmaxf(m, v[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));

    float s = 0.0f;
    uint32_t key[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const bool in = i * 32 + lane < E;
        s += in ? expf(v[i] - m) : 0.0f;
        key[i] = in ? route_key(v[i]) : 0u;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        s += __shfl_xor_sync(0xffffffffu, s, o);

    int my_id = -1;
    uint32_t my_key = 0;
    bool done = false;
    if constexpr (VPL >= 4) {
        // Candidates first. Every lane holds a key (E > 64), so the k-th largest of
        // the 32 lane maxima, t0, is reached by k distinct keys, and the k-th largest
        // key overall is >= t0: every key the k rounds below can pick, ties included,
        // is >= t0, and any key < t0 is below all of them. When no lane holds more
        // than two keys >= t0 (the usual case), the rounds run over those two
        // registers per lane; otherwise over all of them. Same picks either way.
        if (k <= 16) {
            uint32_t lm = key[0];
#pragma unroll
            for (int i = 1; i < VPL; ++i)
                lm = max(lm, key[i]);
            uint32_t t0 = 0;
            for (int j = 0; j < k; ++j) { // remove one lane maximum per round, largest first
                const uint32_t w = __reduce_max_sync(0xffffffffu, lm);
                const uint32_t holders = __ballot_sync(0xffffffffu, lm == w);
                if (lane == __ffs(holders) - 1)
                    lm = 0;
                t0 = w;
            }
            int c = 0;
#pragma unroll
            for (int i = 0; i < VPL; ++i)
                c += key[i] >= t0 ? 1 : 0;
            if (t0 != 0u && __reduce_max_sync(0xffffffffu, static_cast<uint32_t>(c)) <= 2u) {
                uint32_t k0 = 0, k1 = 0; // this lane's candidates in ascending index
                int i0 = 0, i1 = 0;
#pragma unroll
                for (int i = VPL - 1; i >= 0; --i) {
                    const bool in = key[i] >= t0;
                    k1 = in ? k0 : k1;
                    i1 = in ? i0 : i1;
                    k0 = in ? key[i] : k0;
                    i0 = in ? i : i0;
                }
                for (int j = 0; j < k; ++j) {
                    const bool second = k1 > k0; // equal keys: the lower index (slot 0)
                    const uint32_t best = second ? k1 : k0;
                    const int bi = second ? i1 : i0;
                    const uint32_t wmax = __reduce_max_sync(0xffffffffu, best);
                    const uint32_t cand =
                        (best == wmax && best != 0u) ? ~static_cast<uint32_t>(bi * 32 + lane) : 0u;
                    const int e = static_cast<int>(~__reduce_max_sync(0xffffffffu, cand));
                    if ((e & 31) == lane) {
                        if (second)
                            k1 = 0;
                        else
                            k0 = 0;
                    }
                    if (lane == j) {
                        my_id = e;
                        my_key = wmax;
                    }
                }
                done = true;
            }
        }
    }
    if (!done) {
        for (int j = 0; j < k; ++j) {
            uint32_t best = 0;
            int bi = 0;
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const bool better = key[i] > best;
                best = better ? key[i] : best;
                bi = better ? i : bi;
            }
            const uint32_t wmax = __reduce_max_sync(0xffffffffu, best);
            const uint32_t cand = (best == wmax && best != 0u) ? ~static_cast<uint32_t>(bi * 32 + lane) : 0u;
            const int e = static_cast<int>(~__reduce_max_sync(0xffffffffu, cand));
            const bool mine = (e & 31) == lane;
#pragma unroll
            for (int i = 0; i < VPL; ++i)
                key[i] = (mine && i == (e >> 5)) ? 0u : key[i];
            if (lane == j) {
                my_id = e;
                my_key = wmax;
            }
        }
    }
    id = lane < k ? my_id : -1;
    prob = lane < k ? expf(route_unkey(my_key) - m) / s : 0.0f; // lane j turns the j-th winning logit into its prob
}

template <int VPL> // logits held per lane: E <= 32 * VPL
__global__ void __launch_bounds__(ROUTE_WARPS_PER_BLOCK * 32)
    route_topk_kernel(const float *__restrict__ logits, const uint8_t *__restrict__ mask, int64_t N, int E, int k,
                      int32_t *__restrict__ topk_idx, float *__restrict__ topk_probs)
{
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * ROUTE_WARPS_PER_BLOCK + (threadIdx.x >> 5);
    if (t >= N)
        return;
    int32_t *idx_out = topk_idx + t * k;
    float *prob_out = topk_probs + t * k;
    if (mask != nullptr && mask[t] != 0) {
        if (lane < k) {
            idx_out[lane] = -1;
            prob_out[lane] = 0.0f;
        }
        return;
    }
    float v[VPL];
    route_load(logits + t * E, E, lane, v);
    int32_t id;
    float prob;
    route_select(v, E, k, lane, id, prob);
    if (lane < k) {
        idx_out[lane] = id;
        prob_out[lane] = prob;
    }
}

} // namespace moert
