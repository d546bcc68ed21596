// Dispatch and combine around the grouped GEMMs (inblix article "Perplexity's
// Lily engine beats MLX by 35% on M5 Max, no PyTorch needed", paragraph 3:
// scatter of the routed tokens into expert-contiguous order, and the
// routing-weighted sum of the expert outputs).
//
//   dispatch_kernel   xs[p] = x[sorted_assign[p] / k]        p < T*k
//   combine_kernel    y[t]  = bf16( sum_{j<k} w[t,j] * o[pos[t,j]] )
//
// Both are bound by HBM bandwidth and move 16-byte vectors, consecutive
// threads on consecutive vectors of a row.  Copying the token rows into
// expert order once lets both grouped GEMMs read their token operand as dense
// 2-D TMA tiles (a gather of single rows runs at a small fraction of that
// rate), and writing the down outputs per assignment lets the sum over a
// token's experts run in a fixed order with no atomics.
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint4 ld_nc_v4(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// One warp per row (grid-stride): lane l moves 16-byte vectors l, l + 32, ...
// of the row, up to kDispatchVecs of them loaded before the first store (all
// of a row for d <= 2048), with the next row's source index read before the
// stores.
constexpr int kDispatchVecs = 8;

__global__ void __launch_bounds__(kThreads)
dispatch_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ sorted_assign, int Tk,
                int k, int d, uint16_t* __restrict__ xs, int32_t* status) {
    const int lane = threadIdx.x & 31;
    const int nv = d >> 3;  // 16-byte vectors per row
    const int warps = gridDim.x * (kThreads / 32);
    pdl_launch_dependents();
    pdl_wait();
    const uint4* x4 = reinterpret_cast<const uint4*>(x);
    uint4* xs4 = reinterpret_cast<uint4*>(xs);
    int p = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    int a = p < Tk ? sorted_assign[p] : 0;
    for (; p < Tk; p += warps) {
        const int a_next = p + warps < Tk ? sorted_assign[p + warps] : 0;
        if (static_cast<unsigned>(a) >= static_cast<unsigned>(Tk)) {
            if (lane == 0) report_error(status, MOE_ERR_DEVICE_BOUNDS, 300);
            a = 0;
        }
        const uint4* src = x4 + static_cast<size_t>(a / k) * nv;
        uint4* dst = xs4 + static_cast<size_t>(p) * nv;
        for (int i0 = 0; i0 < nv; i0 += 32 * kDispatchVecs) {
            uint4 v[kDispatchVecs];
#pragma unroll
            for (int u = 0; u < kDispatchVecs; ++u) {
                const int i = i0 + 32 * u + lane;
                v[u] = i < nv ? ld_nc_v4(src + i) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < kDispatchVecs; ++u) {
                const int i = i0 + 32 * u + lane;
                if (i < nv) dst[i] = v[u];
            }
        }
        a = a_next;
    }
}

union BF8 {
    uint4 u;
    __nv_bfloat162 h[4];
};

// acc[0..7] = fma(w, bf16 vector v, acc)
__device__ __forceinline__ void fma8(float* acc, float w, const uint4& v) {
    BF8 b;
    b.u = v;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(b.h[e]);
        acc[2 * e] = fmaf(w, f.x, acc[2 * e]);
        acc[2 * e + 1] = fmaf(w, f.y, acc[2 * e + 1]);
    }
}

// One CTA per token (grid-stride over tokens): the token's k positions and
// weights go to shared memory, then thread i sums the 8 features of vector i
// over the slots in order j = 0 .. k-1 (fp32 fused multiply-add), with the
// loads of up to 8 slots issued before the first of them is used.
__global__ void __launch_bounds__(kThreads)
combine_kernel(const uint16_t* __restrict__ o, const int32_t* __restrict__ pos,
               const float* __restrict__ topk_w, int T, int k, int d, uint16_t* __restrict__ y,
               int32_t* status) {
    __shared__ int32_t sp[kMaxTopk];
    __shared__ float sw[kMaxTopk];
    const int nv = d >> 3;
    const int Tk = T * k;
    const uint4* o4 = reinterpret_cast<const uint4*>(o);
    pdl_launch_dependents();
    pdl_wait();
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        __syncthreads();  // the previous token's slots are no longer read
        if (threadIdx.x < k) {
            int p = pos[static_cast<size_t>(t) * k + threadIdx.x];
            float w = topk_w[static_cast<size_t>(t) * k + threadIdx.x];
            if (static_cast<unsigned>(p) >= static_cast<unsigned>(Tk)) {
                report_error(status, MOE_ERR_DEVICE_BOUNDS, 301);
                p = 0;
                w = 0.0f;
            }
            sp[threadIdx.x] = p;
            sw[threadIdx.x] = w;
        }
        __syncthreads();
        uint4* dst = reinterpret_cast<uint4*>(y + static_cast<size_t>(t) * d);
        for (int i = threadIdx.x; i < nv; i += kThreads) {
            float acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
            for (int j0 = 0; j0 < k; j0 += 8) {
                uint4 v[8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                    v[jj] = j0 + jj < k ? ld_nc_v4(o4 + static_cast<size_t>(sp[j0 + jj]) * nv + i)
                                        : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                    if (j0 + jj < k) fma8(acc, sw[j0 + jj], v[jj]);
            }
            BF8 r;
#pragma unroll
            for (int e = 0; e < 4; ++e) r.h[e] = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
            dst[i] = r.u;
        }
    }
}

__global__ void __launch_bounds__(kThreads)
block_map_check_kernel(const int32_t* __restrict__ block_map, const int32_t* __restrict__ num_blocks,
                       int max_blocks, int n_rows, int E, int block_t, int32_t* __restrict__ nb_out,
                       int32_t* status) {
    __shared__ int bad;
    if (threadIdx.x == 0) {
        bad = 0;
        status[0] = 0;  // the status word reports the most recent call
        status[1] = 0;
    }
    __syncthreads();
    const int nb = *num_blocks;
    if (nb < 0 || nb > max_blocks) {
        if (threadIdx.x == 0) bad = 1;
    } else {
        for (int i = threadIdx.x; i < nb; i += blockDim.x) {
            const int e = block_map[3 * i];
            const int r0 = block_map[3 * i + 1];
            const int n = block_map[3 * i + 2];
            if (e < 0 || e >= E || r0 < 0 || n < 0 || n > block_t || r0 > n_rows - n) atomicOr(&bad, 1);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        *nb_out = bad ? 0 : nb;
        if (bad) report_error(status, MOE_ERR_DEVICE_BOUNDS, 400);
    }
}

}  // namespace

cudaError_t launch_block_map_check(const int32_t* block_map, const int32_t* num_blocks, int max_blocks,
                                   int n_rows, int E, int block_t, int32_t* nb_out, int32_t* status,
                                   cudaStream_t st) {
    block_map_check_kernel<<<1, kThreads, 0, st>>>(block_map, num_blocks, max_blocks, n_rows, E, block_t,
                                                   nb_out, status);
    return cudaGetLastError();
}

cudaError_t launch_dispatch(const uint16_t* x, const int32_t* sorted_assign, int Tk, int k, int d,
                            uint16_t* xs, int32_t* status, int num_sms, cudaStream_t st) {
    if (Tk <= 0) return cudaSuccess;
    const long need = (static_cast<long>(Tk) + kThreads / 32 - 1) / (kThreads / 32);
    const long cap = static_cast<long>(num_sms) * 8;  // 8 CTAs of 8 warps per SM
    const int grid = static_cast<int>(need < cap ? need : cap);
    return launch_pdl(dispatch_kernel, dim3(grid), dim3(kThreads), 0, st, x, sorted_assign, Tk, k, d, xs,
                      status);
}

cudaError_t launch_combine(const uint16_t* o, const int32_t* pos, const float* topk_w, int T, int k,
                           int d, uint16_t* y, int32_t* status, int num_sms, cudaStream_t st) {
    if (T <= 0) return cudaSuccess;
    const long cap = static_cast<long>(num_sms) * 8;
    const int grid = static_cast<int>(T < cap ? T : cap);
    combine_kernel<<<grid, kThreads, 0, st>>>(o, pos, topk_w, T, k, d, y, status);
    return cudaGetLastError();
}

}  // namespace moe
