// Routing stages of the MoE layer (inblix article "Perplexity's Lily engine
// beats MLX by 35% on M5 Max, no PyTorch needed", paragraph 3: expert
// routing, prefix scan, scatter and block map, all kept on the GPU with no
// host round trip):
//   router_logits_kernel  fp32 logits in the fixed chain-and-butterfly order
//   router_topk_kernel    top-k (ties to the lower id), softmax weights,
//                         per-group expert histograms
//   route_scan_kernel     counts, prefix offsets, per-group scatter bases,
//                         block map
//   route_scatter_kernel  stable scatter into expert order (sorted_assign,
//                         pos)
#include <atomic>

#include "moe_route_common.cuh"

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
    pdl_launch_dependents();
    pdl_wait();

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
// Router logits for larger batches (same summation order as above).
//
// Each CTA owns one slice of ES experts and keeps that slice of W_r in
// shared memory for its whole life (rows padded to ES+4 floats so the 32
// lanes, which read 32 different rows, hit distinct banks).  It sweeps token
// tiles of 64: every warp takes 8 tokens of the tile, lane p accumulates chain
// p of all 8 x ES (token, expert) pairs, and the tile's x rows stream through a
// double-buffered shared-memory ring of 256-wide K chunks (cp.async).
// Grid: (E / ES) * ctas_per_slice; CTA c serves slice c % (E / ES) and tiles
// c / (E / ES), c / (E / ES) + ctas_per_slice, ...
// ---------------------------------------------------------------------------
// Configuration: ES experts per slice, TT tokens per warp, WARPS warps, K
// chunks of KC.  A tile is TT * WARPS tokens.
template <int ES_, int TT_, int WARPS_, int KC_>
struct RouterCfg {
    static constexpr int ES = ES_, TT = TT_, WARPS = WARPS_, KC = KC_;
    static constexpr int kTile = TT * WARPS;
    static constexpr int smem_bytes(int d) { return d * (ES + 4) * 4 + 2 * kTile * KC * 2; }
};
using RouterCfg16 = RouterCfg<16, 8, 8, 256>;
using RouterCfg8 = RouterCfg<8, 8, 16, 128>;
// few tokens: half the experts per slice and 64-token tiles, so twice as many
// CTAs share the work (each loads a W_r slice half as large)
using RouterCfg8s = RouterCfg<8, 8, 8, 256>;
constexpr int kRouterMinTile = 64;  // smallest tile of the configurations above

template <class RC>
__global__ void __launch_bounds__(RC::WARPS * 32, 1)
router_logits_smem_kernel(const uint16_t* __restrict__ x, const float* __restrict__ W,
                          const float* __restrict__ b, float* __restrict__ logits, int T, int d,
                          int E, int32_t* __restrict__ hist, int hist_n,
                          int32_t* __restrict__ status) {
    constexpr int ES = RC::ES;
    constexpr int TT = RC::TT;                      // tokens per warp
    constexpr int kRouterTile = RC::kTile;
    constexpr int kRouterKc = RC::KC;
    constexpr int kRouterWarps = RC::WARPS;
    constexpr int V = TT * ES;                      // values per lane
    static_assert((kRouterTile * kRouterKc * 2 / 16) % (kRouterWarps * 32) == 0,
                  "whole 16-byte pieces per thread and chunk");
    constexpr int WS = ES + 4;                      // padded W row (floats)
    static_assert(V % 32 == 0, "reduce-scatter needs a multiple of 32 values");
    extern __shared__ __align__(16) uint8_t rsm[];
    float* Ws = reinterpret_cast<float*>(rsm);
    uint16_t* xs = reinterpret_cast<uint16_t*>(rsm + static_cast<size_t>(d) * WS * 4);
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nslices = E / ES;
    const int slice = blockIdx.x % nslices;
    const int cta = blockIdx.x / nslices;
    const int ctas = gridDim.x / nslices;
    const int e0 = slice * ES;

    pdl_launch_dependents();
    // the W_r slice, row i -> Ws[i * WS .. + ES) (an input: loaded while the
    // previous kernel in the stream finishes), as asynchronous 16-byte copies
    // that are all in flight at once
    {
        const uint32_t ws_base = smem_u32(Ws);
        for (int idx = threadIdx.x; idx < d * (ES / 4); idx += blockDim.x) {
            const int i = idx / (ES / 4);
            const int q = idx % (ES / 4);
            cp_async_16(ws_base + (i * WS + 4 * q) * 4, W + static_cast<size_t>(i) * E + e0 + 4 * q, 16u);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    pdl_wait();
    if (blockIdx.x == 0) {
        for (int i = threadIdx.x; i < hist_n; i += blockDim.x) hist[i] = 0;
        if (threadIdx.x < 2) status[threadIdx.x] = 0;
    }
    __syncthreads();

    const int ntiles = (T + kRouterTile - 1) / kRouterTile;
    const int nkc = d / kRouterKc;
    const uint32_t xs_base = smem_u32(xs);
    // one K chunk of the tile: 64 rows x 512 bytes = 2048 16-byte pieces, 8 per thread
    auto load_chunk = [&](int t0, int kc, int buf) {
#pragma unroll
        for (int j = 0; j < (kRouterTile * kRouterKc * 2 / 16) / (kRouterWarps * 32); ++j) {
            const int piece = threadIdx.x + j * kRouterWarps * 32;
            const int row = piece / (kRouterKc * 2 / 16);
            const int col = piece % (kRouterKc * 2 / 16);
            const int t = t0 + row;
            const uint16_t* src = x + static_cast<size_t>(t < T ? t : 0) * d + kc * kRouterKc + col * 8;
            cp_async_16(xs_base + ((buf * kRouterTile + row) * kRouterKc + col * 8) * 2, src,
                        t < T ? 16u : 0u);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    for (int tile = cta; tile < ntiles; tile += ctas) {
        const int t0 = tile * kRouterTile;
        // accumulators of experts (2q, 2q+1) of token tt are the pair acc2[tt*ES/2 + q],
        // advanced together by one packed fp32 fused multiply-add (each half
        // rounds exactly like a scalar fmaf)
        float2 acc2[V / 2];
#pragma unroll
        for (int j = 0; j < V / 2; ++j) acc2[j] = make_float2(0.0f, 0.0f);
        load_chunk(t0, 0, 0);
        for (int kc = 0; kc < nkc; ++kc) {
            if (kc + 1 < nkc) {
                load_chunk(t0, kc + 1, (kc + 1) & 1);
                asm volatile("cp.async.wait_group 1;" ::: "memory");
            } else {
                asm volatile("cp.async.wait_group 0;" ::: "memory");
            }
            __syncthreads();
            const uint16_t* xb = xs + ((kc & 1) * kRouterTile + warp * TT) * kRouterKc;
            const float* wb = Ws + static_cast<size_t>(kc * kRouterKc) * WS;
#pragma unroll 2
            for (int s = 0; s < kRouterKc / 32; ++s) {
                const int il = s * 32 + lane;
                float xv[TT];
#pragma unroll
                for (int tt = 0; tt < TT; ++tt) xv[tt] = bf16_bits_to_float(xb[tt * kRouterKc + il]);
                float2 wv[ES / 2];
#pragma unroll
                for (int q = 0; q < ES / 4; ++q) {
                    const float4 w4 = *reinterpret_cast<const float4*>(wb + il * WS + 4 * q);
                    wv[2 * q + 0] = make_float2(w4.x, w4.y);
                    wv[2 * q + 1] = make_float2(w4.z, w4.w);
                }
#pragma unroll
                for (int tt = 0; tt < TT; ++tt) {
                    const float2 xx = make_float2(xv[tt], xv[tt]);
#pragma unroll
                    for (int q = 0; q < ES / 2; ++q)
                        acc2[tt * (ES / 2) + q] = __ffma2_rn(xx, wv[q], acc2[tt * (ES / 2) + q]);
                }
            }
            __syncthreads();  // the buffer is refilled by the next chunk's copies
        }
        float acc[V];
#pragma unroll
        for (int j = 0; j < V / 2; ++j) {
            acc[2 * j] = acc2[j].x;
            acc[2 * j + 1] = acc2[j].y;
        }
        // reduce-scatter butterfly (see router_logits_kernel)
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
#pragma unroll
        for (int j = 0; j < V / 32; ++j) {
            const int el = lane * (V / 32) + j;
            const int tt = el / ES;
            const int ee = el % ES;
            const int t = t0 + warp * TT + tt;
            if (t < T) {
                float l = acc[j];
                if (b != nullptr) l = __fadd_rn(l, __ldg(b + e0 + ee));
                logits[static_cast<size_t>(t) * E + e0 + ee] = l;
            }
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
// the counts do not depend on their order).
// ---------------------------------------------------------------------------
constexpr int kTopkWarps = 8;

__global__ void __launch_bounds__(kTopkWarps * 32)
router_topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                   int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                   int32_t* __restrict__ hist) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    pdl_launch_dependents();
    pdl_wait();
    const int t = blockIdx.x * kTopkWarps + warp;
    if (t >= T) return;
    int my_id;
    float my_w;
    warp_topk(logits + static_cast<size_t>(t) * E, E, k, lane, my_id, my_w);
    if (lane < k) {
        topk_idx[static_cast<size_t>(t) * k + lane] = my_id;
        topk_w[static_cast<size_t>(t) * k + lane] = my_w;
        atomicAdd(hist + static_cast<size_t>(t / kRouteGroupT) * E + my_id, 1);
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


__global__ void __launch_bounds__(kScanThreads)
route_scan_kernel(const int32_t* __restrict__ hist, int ng, int E, int BT,
                  int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                  int32_t* __restrict__ gbase, int32_t* __restrict__ block_offsets,
                  int32_t* __restrict__ block_map, int32_t* __restrict__ num_blocks,
                  int max_blocks, int32_t* status) {
    __shared__ int sh_warp[kScanThreads / 32 + 1];
    pdl_launch_dependents();
    pdl_wait();
    const int e = threadIdx.x;
    int c = 0;
    if (e < E)
        for (int g = 0; g < ng; ++g) c += hist[static_cast<size_t>(g) * E + e];
    int total = 0;
    const int off = block_exclusive_scan<kScanThreads>(e < E ? c : 0, sh_warp, &total);
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
    const int bo = block_exclusive_scan<kScanThreads>(nt, sh_warp, &nb_total);
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
// One CTA of kScatterWarps warps per group of kRouteGroupT tokens; warp w
// owns a contiguous slice of the group's assignments.  Pass 1 counts each
// warp's assignments per expert, the warps' bases follow from the group's base
// (gbase) by a scan over warps, and pass 2 places every assignment: inside a
// 32-assignment chunk the lanes of one expert are ranked by lane id.
// ---------------------------------------------------------------------------
constexpr int kScatterWarps = 32;

__global__ void __launch_bounds__(kScatterWarps * 32)
route_scatter_kernel(const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ gbase,
                     int T, int k, int E, int32_t* __restrict__ sorted_assign,
                     int32_t* __restrict__ pos, int32_t* status) {
    __shared__ int cnt[kScatterWarps][kMaxExperts];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    pdl_launch_dependents();
    pdl_wait();
    const int g = blockIdx.x;
    const long total = static_cast<long>(T) * k;
    const long a_begin = static_cast<long>(g) * kRouteGroupT * k;
    const long a_end = min(total, a_begin + static_cast<long>(kRouteGroupT) * k);
    const long per_warp = (static_cast<long>(kRouteGroupT) * k + kScatterWarps - 1) / kScatterWarps;
    const long w_begin = a_begin + warp * per_warp;
    const long w_end = min(a_end, w_begin + per_warp);
    const unsigned lt_mask = (1u << lane) - 1u;

    for (int e = lane; e < E; e += 32) cnt[warp][e] = 0;
    __syncwarp();
    for (long a0 = w_begin; a0 < w_end; a0 += 32) {
        const long a = a0 + lane;
        int e = a < w_end ? topk_idx[a] : E + lane;
        if (e < 0 || (e >= E && a < w_end)) {
            report_error(status, MOE_ERR_DEVICE_BOUNDS, 2);
            e = E + lane;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e < E && lane == __ffs(peers) - 1) cnt[warp][e] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    // per-warp bases: exclusive scan over warps, starting at the group's base
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = gbase[static_cast<size_t>(g) * E + e];
        for (int w = 0; w < kScatterWarps; ++w) {
            const int c = cnt[w][e];
            cnt[w][e] = run;
            run += c;
        }
    }
    __syncthreads();
    for (long a0 = w_begin; a0 < w_end; a0 += 32) {
        const long a = a0 + lane;
        int e = a < w_end ? topk_idx[a] : E + lane;
        if (e < 0 || e > E + 31) e = E + lane;
        const bool real = e < E;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & lt_mask);
        const int base = real ? cnt[warp][e] : 0;
        __syncwarp();
        if (real) {
            const int p = base + rank;
            if (p < 0 || p >= total) {
                report_error(status, MOE_ERR_DEVICE_BOUNDS, 3);
            } else {
                sorted_assign[p] = static_cast<int>(a);
                pos[a] = p;
            }
            if (lane == __ffs(peers) - 1) cnt[warp][e] = base + __popc(peers);
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
// per-device set-up of the shared-memory router: opt in to large dynamic
// shared memory once per device and remember the SM count
template <class RC>
static cudaError_t router_smem_setup(int* num_sms) {
    static std::atomic<int> ready[64];
    static std::atomic<int> sms[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (ready[dev].load(std::memory_order_acquire) == 0) {
        e = cudaFuncSetAttribute(router_logits_smem_kernel<RC>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        int n = 0;
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        sms[dev].store(n);
        ready[dev].store(1, std::memory_order_release);
    }
    *num_sms = sms[dev].load();
    return cudaSuccess;
}

template <class RC>
static cudaError_t launch_router_smem(const uint16_t* x, const float* W, const float* b,
                                      float* logits, int T, int d, int E, int32_t* hist,
                                      int hist_n, int32_t* status, cudaStream_t st) {
    const int smem = RC::smem_bytes(d);
    int num_sms = 0;
    const cudaError_t e = router_smem_setup<RC>(&num_sms);
    if (e != cudaSuccess) return e;
    const int nslices = E / RC::ES;
    const int ntiles = (T + RC::kTile - 1) / RC::kTile;
    int per_slice = num_sms / nslices;
    if (per_slice < 1) per_slice = 1;
    if (per_slice > ntiles) per_slice = ntiles;
    return launch_pdl(router_logits_smem_kernel<RC>, dim3(nslices * per_slice), dim3(RC::WARPS * 32),
                      smem, st, x, W, b, logits, T, d, E, hist, hist_n, status);
}

cudaError_t prepare_router() {
    int n = 0;
    cudaError_t e = router_smem_setup<RouterCfg16>(&n);
    if (e == cudaSuccess) e = router_smem_setup<RouterCfg8>(&n);
    if (e == cudaSuccess) e = router_smem_setup<RouterCfg8s>(&n);
    return e;
}

cudaError_t launch_router_logits(const uint16_t* x, const float* W, const float* b,
                                 float* logits, int T, int d, int E, int32_t* hist, int hist_n,
                                 int32_t* status, cudaStream_t st) {
    // batches of at least one tile per SM use the shared-memory kernel
    if (T >= kRouterMinTile * 2) {
        if (T <= 1024 && E % 8 == 0 && RouterCfg8s::smem_bytes(d) <= 227 * 1024)
            return launch_router_smem<RouterCfg8s>(x, W, b, logits, T, d, E, hist, hist_n, status,
                                                   st);
        if (E % 16 == 0 && RouterCfg16::smem_bytes(d) <= 227 * 1024)
            return launch_router_smem<RouterCfg16>(x, W, b, logits, T, d, E, hist, hist_n, status,
                                                   st);
        if (RouterCfg8::smem_bytes(d) <= 227 * 1024)
            return launch_router_smem<RouterCfg8>(x, W, b, logits, T, d, E, hist, hist_n, status, st);
    }
    const int ty = T > 0 ? (T + kLogitTokPerCta - 1) / kLogitTokPerCta : 1;
    if (E % 16 == 0)
        return launch_pdl(router_logits_kernel<16>, dim3(E / 16, ty), dim3(kLogitWarps * 32), 0, st,
                          x, W, b, logits, T, d, E, hist, hist_n, status);
    return launch_pdl(router_logits_kernel<8>, dim3(E / 8, ty), dim3(kLogitWarps * 32), 0, st, x, W,
                      b, logits, T, d, E, hist, hist_n, status);
}

cudaError_t launch_router_topk(const float* logits, int T, int E, int k, int32_t* topk_idx,
                               float* topk_w, int32_t* hist, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int grid = (T + kTopkWarps - 1) / kTopkWarps;
    return launch_pdl(router_topk_kernel, dim3(grid), dim3(kTopkWarps * 32), 0, st, logits, T, E, k,
                      topk_idx, topk_w, hist);
}

cudaError_t launch_route_scan(const int32_t* hist, int ng, int E, int BT, int32_t* counts,
                              int32_t* offsets, int32_t* gbase, int32_t* block_offsets,
                              int32_t* block_map, int32_t* num_blocks, int max_blocks,
                              int32_t* status, cudaStream_t st) {
    return launch_pdl(route_scan_kernel, dim3(1), dim3(kScanThreads), 0, st, hist, ng, E, BT, counts,
                      offsets, gbase, block_offsets, block_map, num_blocks, max_blocks, status);
}

cudaError_t launch_route_scatter(const int32_t* topk_idx, const int32_t* gbase, int T, int k,
                                 int E, int32_t* sorted_assign, int32_t* pos, int32_t* status,
                                 cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int ng = (T + kRouteGroupT - 1) / kRouteGroupT;
    return launch_pdl(route_scatter_kernel, dim3(ng), dim3(kScatterWarps * 32), 0, st, topk_idx,
                      gbase, T, k, E, sorted_assign, pos, status);
}

}  // namespace moe
