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
// an empty slot) and sorts them once, descending (equal keys: lower id first),
// with a static bitonic network. Each of the k rounds then compares only the
// lanes' heads: the warp maximum with one redux.sync, and among the lanes
// holding it the lowest expert id with a second; the winning lane shifts its
// list. The key maps back to the logit exactly, so no shuffle is needed.
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

    const float *row = logits + t * E;
    float v[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int e = i * 32 + lane;
        v[i] = e < E ? __ldg(row + e) : -INFINITY;
    }

    float m = v[0];
#pragma unroll
    for (int i = 1; i < VPL; ++i)
        m = fmaxf(m, v[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));

    float s = 0.0f;
    uint32_t key[VPL];
    int slot[VPL]; // i of expert i * 32 + lane
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const bool in = i * 32 + lane < E;
        s += in ? expf(v[i] - m) : 0.0f;
        key[i] = in ? route_key(v[i]) : 0u;
        slot[i] = i;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        s += __shfl_xor_sync(0xffffffffu, s, o);

    // bitonic sort of the lane's keys, descending; equal keys keep the lower slot first
#pragma unroll
    for (int size = 2; size <= VPL; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int j = i ^ stride;
                if (j > i) {
                    const bool first_greater = key[i] > key[j] || (key[i] == key[j] && slot[i] < slot[j]);
                    const bool want_greater_first = (i & size) == 0;
                    if (first_greater != want_greater_first) {
                        const uint32_t tk = key[i];
                        key[i] = key[j];
                        key[j] = tk;
                        const int ts = slot[i];
                        slot[i] = slot[j];
                        slot[j] = ts;
                    }
                }
            }
        }
    }

    int my_id = -1;
    uint32_t my_key = 0;
    for (int j = 0; j < k; ++j) {
        const uint32_t head = key[0];
        const uint32_t wmax = __reduce_max_sync(0xffffffffu, head);
        const uint32_t cand = (head == wmax && head != 0u) ? ~static_cast<uint32_t>(slot[0] * 32 + lane) : 0u;
        const int e = static_cast<int>(~__reduce_max_sync(0xffffffffu, cand));
        if ((e & 31) == lane) {
#pragma unroll
            for (int i = 0; i + 1 < VPL; ++i) {
                key[i] = key[i + 1];
                slot[i] = slot[i + 1];
            }
            key[VPL - 1] = 0u;
        }
        if (lane == j) {
            my_id = e;
            my_key = wmax;
        }
    }
    if (lane < k) { // lane j turns the j-th winning logit into its prob
        idx_out[lane] = my_id;
        prob_out[lane] = expf(route_unkey(my_key) - m) / s;
    }
}

} // namespace moert
