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
#pragma once

#include <cstdint>

namespace moert {

constexpr int ROUTE_WARPS_PER_BLOCK = 8;

// 64-bit selection key: larger logit first, then lower id. The float is
// mapped to an order-preserving unsigned integer; -0 is folded onto +0 so that
// the two compare equal, as they do in IEEE comparison.
__device__ __forceinline__ uint64_t route_key(float v, int e)
{
    uint32_t b = __float_as_uint(v + 0.0f);
    b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return (static_cast<uint64_t>(b) << 32) | static_cast<uint32_t>(~e);
}

template <int VPL> // logits held per lane: E <= 32 * VPL
__global__ void __launch_bounds__(ROUTE_WARPS_PER_BLOCK * 32)
    route_topk_kernel(const float *__restrict__ logits, const uint8_t *__restrict__ mask, int64_t N, int E, int k,
                      int32_t *__restrict__ topk_idx, float *__restrict__ topk_probs)
{
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
#pragma unroll
    for (int i = 0; i < VPL; ++i)
        if (i * 32 + lane < E)
            s += expf(v[i] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        s += __shfl_xor_sync(0xffffffffu, s, o);

    uint64_t key[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i)
        key[i] = (i * 32 + lane < E) ? route_key(v[i], i * 32 + lane) : 0ull;

    int my_id = -1;
    float my_prob = 0.0f;
    for (int j = 0; j < k; ++j) {
        uint64_t best = 0;
#pragma unroll
        for (int i = 0; i < VPL; ++i)
            best = key[i] > best ? key[i] : best;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const uint64_t other = __shfl_xor_sync(0xffffffffu, best, o);
            best = other > best ? other : best;
        }
        const int e = static_cast<int>(~static_cast<uint32_t>(best));
        // the owner of the winning key retires it
        if ((e & 31) == lane) {
#pragma unroll
            for (int i = 0; i < VPL; ++i)
                if (i == (e >> 5))
                    key[i] = 0ull;
        }
        if (lane == j)
            my_id = e;
        // broadcast the winning logit from its owner lane
        float vw = 0.0f;
#pragma unroll
        for (int i = 0; i < VPL; ++i)
            if (i == (e >> 5))
                vw = v[i];
        vw = __shfl_sync(0xffffffffu, vw, e & 31);
        if (lane == j)
            my_prob = expf(vw - m) / s;
    }
    if (lane < k) {
        idx_out[lane] = my_id;
        prob_out[lane] = my_prob;
    }
}

} // namespace moert
