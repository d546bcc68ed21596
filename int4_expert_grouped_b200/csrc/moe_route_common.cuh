// Routing building blocks shared by the batched routing kernels and the
// small-batch (decode) path, so both take every integer decision with the
// same code (inblix article "Perplexity's Lily engine beats MLX by 35% on M5
// Max, no PyTorch needed", paragraph 3: expert routing, prefix scan, scatter
// and block map).
#pragma once

#include "moe_internal.h"

namespace moe {

struct Cand {
    float v;
    int id;  // >= kInvalidId means none
};
constexpr int kInvalidId = 1 << 30;

// (logit descending, id ascending); an invalid candidate loses to any other
__device__ __forceinline__ bool better(const Cand& a, const Cand& b) {
    if (a.id >= kInvalidId) return false;
    if (b.id >= kInvalidId) return true;
    return a.v > b.v || (a.v == b.v && a.id < b.id);
}

// Routing weights of one token by one warp: lane j < k holds the logit of
// slot j; softmax over the k slots, w_j = exp(l_j - l_0) / sum_j' exp(l_j' - l_0),
// the sum in a fixed xor butterfly order.  Returns lane j's weight (0 for
// lanes >= k).  Evaluated in double and rounded once to fp32: l_j - l_0 is
// then exact, whereas in fp32 its rounding alone moves exp(l_j - l_0) by up to
// |l_j - l_0| * 2^-24 relative (3e-6 at a spread of 50).  Only k values per
// token, so the cost does not show.
__device__ __forceinline__ float warp_slot_weights(float my_v, int k, int lane) {
    const double l0 = static_cast<double>(__shfl_sync(0xffffffffu, my_v, 0));
    const double ex = lane < k ? exp(static_cast<double>(my_v) - l0) : 0.0;
    double sum = ex;
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) sum = __dadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, m));
    return lane < k ? __double2float_rn(__ddiv_rn(ex, sum)) : 0.0f;
}

// Top-k of one token's E logits by one warp: lane holds experts lane,
// lane+32, ...; k rounds of a warp-wide arg-max over the unselected experts.
// Routing weights: softmax over the k selected logits,
// w_j = exp(l_j - l_0) / sum_j' exp(l_j' - l_0), the sum in a fixed xor
// butterfly order.  On return lane j < k holds slot j: (id, weight).
__device__ __forceinline__ void warp_topk(const float* __restrict__ row, int E, int k, int lane,
                                          int& my_id, float& my_w) {
    constexpr int kMaxPerLane = kMaxExperts / 32;
    float v[kMaxPerLane];
    bool taken[kMaxPerLane];
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? row[e] : 0.0f;
        taken[i] = e >= E;
    }
    my_id = 0;
    float my_v = 0.0f;
    for (int j = 0; j < k; ++j) {
        Cand best{0.0f, kInvalidId};
#pragma unroll
        for (int i = 0; i < kMaxPerLane; ++i) {
            const Cand c{v[i], taken[i] ? kInvalidId : lane + 32 * i};
            if (better(c, best)) best = c;
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) {
            Cand o;
            o.v = __shfl_xor_sync(0xffffffffu, best.v, m);
            o.id = __shfl_xor_sync(0xffffffffu, best.id, m);
            if (better(o, best)) best = o;
        }
        // every lane now holds the same winner
#pragma unroll
        for (int i = 0; i < kMaxPerLane; ++i)
            if (best.id == lane + 32 * i) taken[i] = true;
        if (lane == j) {
            my_id = best.id;
            my_v = best.v;
        }
    }
    my_w = warp_slot_weights(my_v, k, lane);
}

// Exclusive prefix sum of one int per thread over a CTA of kThreads threads
// (a multiple of 32, at most 1024); *total receives the sum.  sh_warp needs
// kThreads / 32 + 1 ints.  Every thread of the CTA must call it.
template <int kThreads>
__device__ __forceinline__ int block_exclusive_scan(int v, int* sh_warp, int* total) {
    static_assert(kThreads % 32 == 0 && kThreads <= 1024, "whole warps, at most 32");
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) sh_warp[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < (kThreads / 32) ? sh_warp[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        if (lane < (kThreads / 32)) sh_warp[lane] = wi - w;  // exclusive warp offsets
        if (lane == (kThreads / 32) - 1) sh_warp[kThreads / 32] = wi;
    }
    __syncthreads();
    const int res = sh_warp[warp] + inc - v;
    *total = sh_warp[kThreads / 32];
    __syncthreads();
    return res;
}

}  // namespace moe
