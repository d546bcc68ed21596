// Routing stages of the MoE layer (inblix article "Perplexity's Lily engine
// beats MLX by 35% on M5 Max, no PyTorch needed", paragraph 3: expert
// routing, prefix scan, scatter and block map, all kept on the GPU with no
// host round trip):
//   router_logits_kernel  fp32 logits in the fixed chain-and-butterfly order
//   router_topk_kernel    top-k (ties to the lower id), softmax weights,
//                         per-group expert histograms, zeroing of y_acc
//   route_scan_kernel     counts, prefix offsets, per-group scatter bases,
//                         block map
//   route_scatter_kernel  stable scatter into expert order (sorted_assign,
//                         pos)
#include "moe_internal.h"

namespace moe {

// ---------------------------------------------------------------------------
// Router logits.
//
// l[t,e] = S[t,e] + b_r[e] where S sums x[t,i] * W_r[i,e] in fp32 as 32 chains
// (chain p takes i = p, p+32, ... in ascending i, fused multiply-add from 0)
// combined by an xor butterfly over m = 16, 8, 4, 2, 1.  Lane p of a warp
// owns chain p, so the butterfly is a sequence of shuffles.  Each warp
// accumulates 4 tokens x ES experts per lane; the butterfly is done as a
// reduce-scatter (each step keeps half of the values and trades the other
// half with the partner lane), which computes exactly the same sums as the
// full butterfly with 1/16 of the shuffles.
// Grid: (E / ES, ceil(T / 32)), 256 threads: warp w takes tokens
// 32*blockIdx.y + 4w .. +3 and experts ES*blockIdx.x .. +ES-1.
// ---------------------------------------------------------------------------
constexpr int kLogitTokPerWarp = 4;
constexpr int kLogitWarps = 8;
constexpr int kLogitTokPerCta = kLogitTokPerWarp * kLogitWarps;

template <int ES>
__global__ void __launch_bounds__(kLogitWarps * 32)
router_logits_kernel(const uint16_t* __restrict__ x, const float* __restrict__ W,
                     const float* __restrict__ b, float* __restrict__ logits, int T, int d,
                     int E, int32_t* __restrict__ hist, int hist_n,
                     int32_t* __restrict__ status) {
    constexpr int V = kLogitTokPerWarp * ES;  // values per lane before the butterfly
    static_assert(V % 32 == 0, "reduce-scatter needs a multiple of 32 values");
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;

    if (blockIdx.x == 0 && blockIdx.y == 0) {
        for (int i = threadIdx.x; i < hist_n; i += blockDim.x) hist[i] = 0;
        // the status word reports the most recent call: clear it here, in the
        // first kernel of every call
        if (threadIdx.x < 2) status[threadIdx.x] = 0;
    }

    const int t0 = blockIdx.y * kLogitTokPerCta + warp * kLogitTokPerWarp;
    const int e0 = blockIdx.x * ES;
    if (t0 >= T) return;

    float acc[V];
#pragma unroll
    for (int j = 0; j < V; ++j) acc[j] = 0.0f;

    const uint16_t* xr[kLogitTokPerWarp];
    bool tv[kLogitTokPerWarp];
#pragma unroll
    for (int tt = 0; tt < kLogitTokPerWarp; ++tt) {
        tv[tt] = (t0 + tt) < T;
        xr[tt] = x + static_cast<size_t>(tv[tt] ? t0 + tt : t0) * d;
    }

    const int steps = d >> 5;
#pragma unroll 2
    for (int s = 0; s < steps; ++s) {
        const int i = (s << 5) + lane;
        float xv[kLogitTokPerWarp];
#pragma unroll
        for (int tt = 0; tt < kLogitTokPerWarp; ++tt)
            xv[tt] = tv[tt] ? bf16_bits_to_float(__ldg(xr[tt] + i)) : 0.0f;
        float wv[ES];
        const float4* wrow = reinterpret_cast<const float4*>(W + static_cast<size_t>(i) * E + e0);
#pragma unroll
        for (int q = 0; q < ES / 4; ++q) {
            const float4 w4 = __ldg(wrow + q);
            wv[4 * q + 0] = w4.x;
            wv[4 * q + 1] = w4.y;
            wv[4 * q + 2] = w4.z;
            wv[4 * q + 3] = w4.w;
        }
#pragma unroll
        for (int tt = 0; tt < kLogitTokPerWarp; ++tt)
#pragma unroll
            for (int ee = 0; ee < ES; ++ee)
                acc[tt * ES + ee] = __fmaf_rn(xv[tt], wv[ee], acc[tt * ES + ee]);
    }

    // reduce-scatter butterfly: after the step with distance m the lane keeps
    // the half of its values selected by bit log2(m) of its lane id.
    int cnt = V;
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
        const bool upper = (lane & m) != 0;
        const int half = cnt >> 1;
#pragma unroll
        for (int j = 0; j < V / 2; ++j) {
            if (j < half) {
                const float lo = acc[j];
                const float hi = acc[j + half];
                const float send = upper ? lo : hi;
                const float keep = upper ? hi : lo;
                const float recv = __shfl_xor_sync(0xffffffffu, send, m);
                acc[j] = __fadd_rn(keep, recv);
            }
        }
        cnt = half;
    }
    // lane now holds elements lane * (V/32) + j, j < V/32; element = tt*ES + ee
#pragma unroll
    for (int j = 0; j < V / 32; ++j) {
        const int el = lane * (V / 32) + j;
        const int tt = el / ES;
        const int ee = el % ES;
        const int t = t0 + tt;
        if (t < T) {
            float l = acc[j];
            if (b != nullptr) l = __fadd_rn(l, __ldg(b + e0 + ee));
            logits[static_cast<size_t>(t) * E + e0 + ee] = l;
        }
    }
}

// ---------------------------------------------------------------------------
// Top-k and routing weights.  One warp per token: lane holds experts
// lane, lane+32, ...; k rounds of a warp-wide arg-max over the unselected
// experts by (logit descending, id ascending).  Weights: softmax over the k
// selected logits, w_j = exp(l_j - l_0) / sum_j' exp(l_j' - l_0), with the sum
// taken in a fixed butterfly order.  Each selected expert adds one to the
// histogram of the token's group of kRouteGroupT tokens (integer atomics, so
// the counts do not depend on their order).  The warp also zeroes row t of
// the fp32 combine accumulator y_acc (when given).
// ---------------------------------------------------------------------------
constexpr int kTopkWarps = 8;

struct Cand {
    float v;
    int id;  // >= kInvalidId means none
};
constexpr int kInvalidId = 1 << 30;

__device__ __forceinline__ bool better(const Cand& a, const Cand& b) {
    if (a.id >= kInvalidId) return false;
    if (b.id >= kInvalidId) return true;
    return a.v > b.v || (a.v == b.v && a.id < b.id);
}

__global__ void __launch_bounds__(kTopkWarps * 32)
router_topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                   int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                   int32_t* __restrict__ hist, float* __restrict__ y_acc, int d) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int t = blockIdx.x * kTopkWarps + warp;
    if (t >= T) return;

    constexpr int kMaxPerLane = kMaxExperts / 32;
    float v[kMaxPerLane];
    bool taken[kMaxPerLane];
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? logits[static_cast<size_t>(t) * E + e] : 0.0f;
        taken[i] = e >= E;
    }

    int my_id = 0;
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

    const float l0 = __shfl_sync(0xffffffffu, my_v, 0);
    float ex = lane < k ? expf(__fsub_rn(my_v, l0)) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) sum = __fadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, m));
    if (lane < k) {
        topk_idx[static_cast<size_t>(t) * k + lane] = my_id;
        topk_w[static_cast<size_t>(t) * k + lane] = __fdiv_rn(ex, sum);
        atomicAdd(hist + static_cast<size_t>(t / kRouteGroupT) * E + my_id, 1);
    }
    if (y_acc != nullptr) {
        float4* row = reinterpret_cast<float4*>(y_acc + static_cast<size_t>(t) * d);
        for (int i = lane; i < (d >> 2); i += 32) row[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// ---------------------------------------------------------------------------
// Counts, prefix scan and block map.  One CTA of kScanThreads threads;
// thread e owns expert e.
//   counts[e]  = sum over groups of hist[g][e]
//   offsets    = exclusive scan of counts (offsets[E] = T*k)
//   gbase[g][e]= offsets[e] + sum_{g' < g} hist[g'][e]   (scatter bases)
//   block map  = ceil(counts[e] / BT) tiles per expert, ascending expert
// ---------------------------------------------------------------------------
constexpr int kScanThreads = 256;

__device__ __forceinline__ int block_exclusive_scan(int v, int* sh_warp, int* total) {
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
        int w = lane < (kScanThreads / 32) ? sh_warp[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        if (lane < (kScanThreads / 32)) sh_warp[lane] = wi - w;  // exclusive warp offsets
        if (lane == (kScanThreads / 32) - 1) sh_warp[kScanThreads / 32] = wi;
    }
    __syncthreads();
    const int res = sh_warp[warp] + inc - v;
    *total = sh_warp[kScanThreads / 32];
    __syncthreads();
    return res;
}

__global__ void __launch_bounds__(kScanThreads)
route_scan_kernel(const int32_t* __restrict__ hist, int ng, int E, int BT,
                  int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                  int32_t* __restrict__ gbase, int32_t* __restrict__ block_offsets,
                  int32_t* __restrict__ block_map, int32_t* __restrict__ num_blocks,
                  int max_blocks, int32_t* status) {
    __shared__ int sh_warp[kScanThreads / 32 + 1];
    const int e = threadIdx.x;
    int c = 0;
    if (e < E)
        for (int g = 0; g < ng; ++g) c += hist[static_cast<size_t>(g) * E + e];
    int total = 0;
    const int off = block_exclusive_scan(e < E ? c : 0, sh_warp, &total);
    if (e < E) {
        counts[e] = c;
        offsets[e] = off;
        int run = off;
        for (int g = 0; g < ng; ++g) {
            gbase[static_cast<size_t>(g) * E + e] = run;
            run += hist[static_cast<size_t>(g) * E + e];
        }
    }
    if (e == 0) offsets[E] = total;

    const int nt = e < E ? (c + BT - 1) / BT : 0;
    int nb_total = 0;
    const int bo = block_exclusive_scan(nt, sh_warp, &nb_total);
    if (e < E) {
        block_offsets[e] = bo;
        for (int i = 0; i < nt; ++i) {
            const int idx = bo + i;
            if (idx >= max_blocks) {
                report_error(status, MOE_ERR_DEVICE_BOUNDS, 1);
                break;
            }
            block_map[3 * idx + 0] = e;
            block_map[3 * idx + 1] = off + i * BT;
            block_map[3 * idx + 2] = min(BT, c - i * BT);
        }
    }
    if (e == 0) {
        block_offsets[E] = nb_total;
        num_blocks[0] = min(nb_total, max_blocks);
    }
}

// ---------------------------------------------------------------------------
// Scatter: visit assignments a = t*k + j in ascending order and place each at
// the next free row of its expert, so rows of one expert are in ascending a.
// One warp per group of kRouteGroupT tokens, starting from the group's bases;
// inside a 32-assignment chunk the lanes of one expert are ranked by lane id.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32)
route_scatter_kernel(const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ gbase,
                     int T, int k, int E, int32_t* __restrict__ sorted_assign,
                     int32_t* __restrict__ pos, int32_t* status) {
    __shared__ int running[kMaxExperts];
    const int lane = threadIdx.x;
    const int g = blockIdx.x;
    for (int e = lane; e < E; e += 32) running[e] = gbase[static_cast<size_t>(g) * E + e];
    __syncwarp();
    const long total = static_cast<long>(T) * k;
    const long a_begin = static_cast<long>(g) * kRouteGroupT * k;
    const long a_end = min(total, a_begin + static_cast<long>(kRouteGroupT) * k);
    const unsigned lt_mask = (1u << lane) - 1u;
    for (long a0 = a_begin; a0 < a_end; a0 += 32) {
        const long a = a0 + lane;
        const bool valid = a < a_end;
        int e = valid ? topk_idx[a] : E + lane;  // distinct non-experts for idle lanes
        if (valid && (e < 0 || e >= E)) {
            report_error(status, MOE_ERR_DEVICE_BOUNDS, 2);
            e = E + lane;
        }
        const bool real = e < E;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & lt_mask);
        const int base = real ? running[e] : 0;
        __syncwarp();
        if (real) {
            const int p = base + rank;
            if (p < 0 || p >= total) {
                report_error(status, MOE_ERR_DEVICE_BOUNDS, 3);
            } else {
                sorted_assign[p] = static_cast<int>(a);
                pos[a] = p;
            }
            if (lane == __ffs(peers) - 1) running[e] = base + __popc(peers);
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
cudaError_t launch_router_logits(const uint16_t* x, const float* W, const float* b,
                                 float* logits, int T, int d, int E, int32_t* hist, int hist_n,
                                 int32_t* status, cudaStream_t st) {
    const int ty = T > 0 ? (T + kLogitTokPerCta - 1) / kLogitTokPerCta : 1;
    if (E % 16 == 0) {
        dim3 grid(E / 16, ty);
        router_logits_kernel<16><<<grid, kLogitWarps * 32, 0, st>>>(x, W, b, logits, T, d, E,
                                                                    hist, hist_n, status);
    } else {
        dim3 grid(E / 8, ty);
        router_logits_kernel<8><<<grid, kLogitWarps * 32, 0, st>>>(x, W, b, logits, T, d, E,
                                                                   hist, hist_n, status);
    }
    return cudaGetLastError();
}

cudaError_t launch_router_topk(const float* logits, int T, int E, int k, int32_t* topk_idx,
                               float* topk_w, int32_t* hist, float* y_acc, int d,
                               cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int grid = (T + kTopkWarps - 1) / kTopkWarps;
    router_topk_kernel<<<grid, kTopkWarps * 32, 0, st>>>(logits, T, E, k, topk_idx, topk_w, hist,
                                                         y_acc, d);
    return cudaGetLastError();
}

cudaError_t launch_route_scan(const int32_t* hist, int ng, int E, int BT, int32_t* counts,
                              int32_t* offsets, int32_t* gbase, int32_t* block_offsets,
                              int32_t* block_map, int32_t* num_blocks, int max_blocks,
                              int32_t* status, cudaStream_t st) {
    route_scan_kernel<<<1, kScanThreads, 0, st>>>(hist, ng, E, BT, counts, offsets, gbase,
                                                  block_offsets, block_map, num_blocks,
                                                  max_blocks, status);
    return cudaGetLastError();
}

cudaError_t launch_route_scatter(const int32_t* topk_idx, const int32_t* gbase, int T, int k,
                                 int E, int32_t* sorted_assign, int32_t* pos, int32_t* status,
                                 cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int ng = (T + kRouteGroupT - 1) / kRouteGroupT;
    route_scatter_kernel<<<ng, 32, 0, st>>>(topk_idx, gbase, T, k, E, sorted_assign, pos, status);
    return cudaGetLastError();
}

}  // namespace moe
