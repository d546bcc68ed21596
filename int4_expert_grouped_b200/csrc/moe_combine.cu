// Dispatch and combine around the grouped GEMMs (inblix article "Perplexity's
// Lily engine beats MLX by 35% on M5 Max, no PyTorch needed", paragraph 3:
// scatter of the routed tokens into expert-contiguous order, and the
// routing-weighted sum of the expert outputs).
//
//   dispatch_kernel   xs[p] = x[sorted_assign[p] / k]        p < T*k
//   combine_kernel    y[t]  = bf16( sum_{j<k} w[t,j] * o[pos[t,j]] )
//
// Both are bound by HBM bandwidth: one warp moves one row of d bf16 values
// with 16-byte accesses, so every warp instruction touches 512 contiguous
// bytes.  Copying the token rows into expert order once lets both grouped
// GEMMs read their token operand as dense 2-D TMA tiles (a gather of single
// rows runs at a small fraction of that rate), and writing the down outputs
// per assignment lets the sum over a token's experts run in a fixed order
// with no atomics.
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kRowWarps = 8;  // warps per CTA, one row (token) per warp at a time

__device__ __forceinline__ uint4 ld_nc_v4(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__global__ void __launch_bounds__(kRowWarps * 32)
dispatch_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ sorted_assign, int Tk,
                int k, int d, uint16_t* __restrict__ xs, int32_t* status) {
    const int lane = threadIdx.x & 31;
    const int nv = d >> 3;  // 16-byte vectors per row
    for (int p = blockIdx.x * kRowWarps + (threadIdx.x >> 5); p < Tk; p += gridDim.x * kRowWarps) {
        const int a = sorted_assign[p];
        if (static_cast<unsigned>(a) >= static_cast<unsigned>(Tk)) {
            if (lane == 0) report_error(status, MOE_ERR_DEVICE_BOUNDS, 300);
            continue;
        }
        const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(a / k) * d);
        uint4* dst = reinterpret_cast<uint4*>(xs + static_cast<size_t>(p) * d);
        int i = lane;
        for (; i + 96 < nv; i += 128) {
            const uint4 v0 = ld_nc_v4(src + i);
            const uint4 v1 = ld_nc_v4(src + i + 32);
            const uint4 v2 = ld_nc_v4(src + i + 64);
            const uint4 v3 = ld_nc_v4(src + i + 96);
            dst[i] = v0;
            dst[i + 32] = v1;
            dst[i + 64] = v2;
            dst[i + 96] = v3;
        }
        for (; i < nv; i += 32) dst[i] = ld_nc_v4(src + i);
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

// One warp per token.  Lane j < k holds the position and weight of slot j;
// each lane then sums 8 features at a time over the slots in order
// j = 0 .. k-1 (fp32 fused multiply-add), loading up to 8 slots' vectors
// before using any of them.
__global__ void __launch_bounds__(kRowWarps * 32)
combine_kernel(const uint16_t* __restrict__ o, const int32_t* __restrict__ pos,
               const float* __restrict__ topk_w, int T, int k, int d, uint16_t* __restrict__ y,
               int32_t* status) {
    const int lane = threadIdx.x & 31;
    const int nv = d >> 3;
    const int Tk = T * k;
    for (int t = blockIdx.x * kRowWarps + (threadIdx.x >> 5); t < T; t += gridDim.x * kRowWarps) {
        int my_p = 0;
        float my_w = 0.0f;
        if (lane < k) {
            my_p = pos[static_cast<size_t>(t) * k + lane];
            my_w = topk_w[static_cast<size_t>(t) * k + lane];
            if (static_cast<unsigned>(my_p) >= static_cast<unsigned>(Tk)) {
                report_error(status, MOE_ERR_DEVICE_BOUNDS, 301);
                my_p = 0;
                my_w = 0.0f;
            }
        }
        uint4* dst = reinterpret_cast<uint4*>(y + static_cast<size_t>(t) * d);
        for (int i = lane; i < nv; i += 32) {
            float acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
            for (int j0 = 0; j0 < k; j0 += 8) {
                uint4 v[8];
                float w[8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const int j = j0 + jj;
                    const int p = __shfl_sync(0xffffffffu, my_p, j & 31);
                    w[jj] = __shfl_sync(0xffffffffu, my_w, j & 31);
                    v[jj] = j < k ? ld_nc_v4(reinterpret_cast<const uint4*>(o + static_cast<size_t>(p) * d) + i)
                                  : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                    if (j0 + jj < k) fma8(acc, w[jj], v[jj]);
            }
            BF8 r;
#pragma unroll
            for (int e = 0; e < 4; ++e) r.h[e] = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
            dst[i] = r.u;
        }
    }
}

int row_grid(long rows, int num_sms) {
    const long need = (rows + kRowWarps - 1) / kRowWarps;
    const long cap = static_cast<long>(num_sms) * 8;  // 8 CTAs of 8 warps per SM
    return static_cast<int>(need < cap ? need : cap);
}

}  // namespace

cudaError_t launch_dispatch(const uint16_t* x, const int32_t* sorted_assign, int Tk, int k, int d,
                            uint16_t* xs, int32_t* status, int num_sms, cudaStream_t st) {
    if (Tk <= 0) return cudaSuccess;
    dispatch_kernel<<<row_grid(Tk, num_sms), kRowWarps * 32, 0, st>>>(x, sorted_assign, Tk, k, d, xs,
                                                                      status);
    return cudaGetLastError();
}

cudaError_t launch_combine(const uint16_t* o, const int32_t* pos, const float* topk_w, int T, int k,
                           int d, uint16_t* y, int32_t* status, int num_sms, cudaStream_t st) {
    if (T <= 0) return cudaSuccess;
    combine_kernel<<<row_grid(T, num_sms), kRowWarps * 32, 0, st>>>(o, pos, topk_w, T, k, d, y,
                                                                    status);
    return cudaGetLastError();
}

}  // namespace moe
