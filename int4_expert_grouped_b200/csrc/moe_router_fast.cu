// Router for larger batches with exact results at tensor-core speed (inblix
// article "Perplexity's Lily engine beats MLX by 35% on M5 Max, no PyTorch
// needed", paragraph 3: expert routing kept on the GPU; the ai.jakubjirak.com
// post, section "Why one model on one chip is faster": routing hard-coded for
// the one model).
//
// The routing decision needs the logits in the router's fixed fp32 order
// (32 fused-multiply-add chains, chain p over i = p, p + 32, ..., combined by
// an xor butterfly m = 16..1, plus the bias), because the top-k indices must
// be reproducible bit for bit.  Evaluating that order for every (token,
// expert) pair is 2 T E d fp32 FMAs on the CUDA cores.  Here it is evaluated
// only where the choice could depend on it:
//
//   router_prep_kernel      per token: a power-of-two scale s_t and two int8
//                           digits a, b with x' = s_t (a + b / 128); per
//                           expert likewise u_e, c, d for W_r's column; exact
//                           bounds of what the digits leave out
//   router_approx_kernel    l' = x' . w' + b_r exactly: four int8 tcgen05 MMAs
//                           (a c, a d, b c, b d) accumulate in int32 in TMEM,
//                           so the only error against the exact dot product
//                           is the digits' remainder, which is bounded
//   router_select_kernel    one warp per token: the bounds delta, the k-th
//                           largest lower bound l' - delta (theta), the
//                           candidates (upper bound l' + delta >= theta, a
//                           few per token), their fixed-order fp32 logits
//                           (lane p runs chain p over the transposed W_r
//                           column, then the butterfly and the bias), top-k
//                           among them by (logit desc, id asc), the softmax
//                           weights and the per-group histograms
//
// Why the selection is exact: with delta_te >= |l_te - l'_te| for every pair,
// at least k experts have l >= theta_t (the k-th largest lower bound), so
// every expert of the true top-k has l >= theta_t and hence upper >= theta_t:
// the candidates contain the true top-k, and ranking the candidates by their
// exact logits gives it, ties included.
//
// The bound delta_te is the sum of
//   F_e * A_t    x' times W_r's remainder  (F_e = max |w - w'|, A_t >= sum |x'|)
//   E_t * B_e    x's remainder times W_r    (E_t = max |x - x'|, B_e >= sum |w|)
//   gamma_72 * (N_t * Wn_e + |b_e|)   the fixed order's own rounding against
//                the exact sum (64 fused multiply-adds per chain, 5 butterfly
//                levels and the bias add; |sum x w| <= ||x|| ||w||)
//   2^-23 |l'|   rounding l' to fp32
// all evaluated with upward rounding.
#include <algorithm>
#include <atomic>

#include "moe_route_common.cuh"

namespace moe {
namespace {

struct ApproxArgs {
    CUtensorMap map_wc, map_wd;   // expert digits c, d: int8 [E][d], boxes of 128 K x 128 experts
    CUtensorMap map_xa, map_xb;   // token digits a, b: int8 [T][d], boxes of 128 K x 64 tokens
    const float* s_t;
    const float* u_e;
    const float* b_r;
    float* L;                     // [T][E] approximate logits with the bias
    int T, d, E;
    int32_t* status;
};

// ---------------------------------------------------------------------------
// Prep.  Blocks [0, nxb): eight tokens each (warp per token; the row stays in
// registers, 16-byte vectors v = lane, lane + 32, ...).  Blocks [nxb, nxb + E):
// one expert each (thread t holds rows t, t + 256, ... of the column).
// ---------------------------------------------------------------------------
constexpr int kPrepThreads = 256;
constexpr int kPrepMaxVec = 8;    // 16-byte vectors of a token row per lane: d <= 2048
constexpr int kPrepMaxRows = 8;   // W_r rows per thread of an expert block: d <= 2048

// power of two p with m < 2^span_log2 * p (m > 0); exact
__device__ __forceinline__ float pow2_scale(float m, int span_log2) {
    int ex;
    frexpf(m, &ex);  // m = f 2^ex, f in [0.5, 1): m < 2^ex
    return ldexpf(1.0f, ex - span_log2);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__global__ void __launch_bounds__(kPrepThreads, 2)
router_prep_kernel(const uint16_t* __restrict__ x, const float* __restrict__ W, int T, int d, int E,
                   int nxb, RouterFastWs ws, int32_t* __restrict__ hist, int hist_n,
                   int32_t* __restrict__ status) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    pdl_launch_dependents();
    pdl_wait();
    if (blockIdx.x == 0) {
        for (int i = threadIdx.x; i < hist_n; i += blockDim.x) hist[i] = 0;
        // the status word reports the most recent call: cleared by the first kernel
        if (threadIdx.x < 2) status[threadIdx.x] = 0;
    }
    if (static_cast<int>(blockIdx.x) < nxb) {
        const int t = blockIdx.x * 8 + warp;
        if (t >= T) return;
        const uint4* row = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d);
        const int nv = d >> 3;
        uint4 q[kPrepMaxVec];
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < kPrepMaxVec; ++j) {
            const int v = lane + 32 * j;
            q[j] = v < nv ? __ldg(row + v) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int j = 0; j < kPrepMaxVec; ++j) {
            const uint32_t w[4] = {q[j].x, q[j].y, q[j].z, q[j].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        // |x / s| < 128; a = round(x / s) clamped to +-127 (only +-127.5 is
        // clamped, leaving a remainder of 0.5), b = round(128 (x / s - a))
        const float s = m > 0.0f ? pow2_scale(m, 7) : 1.0f;
        const float inv = 1.0f / s;  // exact: a power of two
        double sabs = 0.0, ssq = 0.0;
        float emax = 0.0f;
        int8_t* pa = ws.xa + static_cast<size_t>(t) * d;
        int8_t* pb = ws.xb + static_cast<size_t>(t) * d;
#pragma unroll
        for (int j = 0; j < kPrepMaxVec; ++j) {
            const int v = lane + 32 * j;
            if (v >= nv) continue;
            const uint32_t w[4] = {q[j].x, q[j].y, q[j].z, q[j].w};
            uint32_t oa[2] = {0u, 0u}, ob[2] = {0u, 0u};
            float fs = 0.0f, fq = 0.0f;  // exact: eight bf16 values
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float xv = i & 1 ? bf16_hi(w[i >> 1]) : bf16_lo(w[i >> 1]);
                const float z = xv * inv;                     // exact
                const float a = fminf(fmaxf(rintf(z), -127.0f), 127.0f);
                const float r = z - a;                        // exact, |r| <= 0.5
                const float b = rintf(r * 128.0f);            // |b| <= 64
                emax = fmaxf(emax, fabsf(s * (r - b * 0.0078125f)));  // exact: the remainder of x
                fs += fabsf(xv);
                fq = fmaf(xv, xv, fq);
                oa[i >> 2] |= (static_cast<uint32_t>(static_cast<int>(a)) & 0xFFu) << (8 * (i & 3));
                ob[i >> 2] |= (static_cast<uint32_t>(static_cast<int>(b)) & 0xFFu) << (8 * (i & 3));
            }
            sabs += static_cast<double>(fs);
            ssq += static_cast<double>(fq);
            *reinterpret_cast<uint2*>(pa + 8 * v) = make_uint2(oa[0], oa[1]);
            *reinterpret_cast<uint2*>(pb + 8 * v) = make_uint2(ob[0], ob[1]);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            sabs += __shfl_xor_sync(0xffffffffu, sabs, o);
            ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
            emax = fmaxf(emax, __shfl_xor_sync(0xffffffffu, emax, o));
        }
        if (lane == 0) {
            ws.s_t[t] = s;
            ws.E_t[t] = emax;
            // sum |x'| <= sum |x| + d max|x - x'|; eight-term fp32 partial sums
            // and the double sums are off by far less than the 1e-6 margin
            ws.A_t[t] = __double2float_ru((sabs + static_cast<double>(d) * emax) * (1.0 + 1e-6));
            ws.N_t[t] = __double2float_ru(sqrt(ssq) * (1.0 + 1e-6));
        }
        return;
    }
    // expert e: thread t holds rows i = t + 256 j (also written out as row e
    // of the transposed W_r, read by the selection kernel's exact logits)
    __shared__ float sm_max[kPrepThreads / 32], sm_f[kPrepThreads / 32];
    __shared__ double sm_abs[kPrepThreads / 32], sm_sq[kPrepThreads / 32];
    __shared__ float sm_u;
    const int e = blockIdx.x - nxb;
    float w[kPrepMaxRows];
    float m = 0.0f;
    double sabs = 0.0, ssq = 0.0;
#pragma unroll
    for (int j = 0; j < kPrepMaxRows; ++j) {
        const int i = threadIdx.x + kPrepThreads * j;
        w[j] = i < d ? __ldg(W + static_cast<size_t>(i) * E + e) : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < kPrepMaxRows; ++j) {
        const int i = threadIdx.x + kPrepThreads * j;
        if (i < d) ws.wt[static_cast<size_t>(e) * d + i] = w[j];
        m = fmaxf(m, fabsf(w[j]));
        sabs += fabs(static_cast<double>(w[j]));
        ssq += static_cast<double>(w[j]) * w[j];
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        sabs += __shfl_xor_sync(0xffffffffu, sabs, o);
        ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
    }
    if (lane == 0) {
        sm_max[warp] = m;
        sm_abs[warp] = sabs;
        sm_sq[warp] = ssq;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float mm = 0.0f;
        double a = 0.0, q = 0.0;
        for (int i = 0; i < kPrepThreads / 32; ++i) {
            mm = fmaxf(mm, sm_max[i]);
            a += sm_abs[i];
            q += sm_sq[i];
        }
        // |w / u| < 64: c = round(w / u), remainder r with |r| <= 0.5,
        // d = round(128 r), |d| <= 64, no clamping
        const float u = mm > 0.0f ? pow2_scale(mm, 6) : 1.0f;
        sm_u = u;
        ws.u_e[e] = u;
        ws.B_e[e] = __double2float_ru(a * (1.0 + 1e-9));
        ws.Wn_e[e] = __double2float_ru(sqrt(q) * (1.0 + 1e-9));
    }
    __syncthreads();
    const float u = sm_u;
    const float inv = 1.0f / u;
    float fmax_ = 0.0f;
#pragma unroll
    for (int j = 0; j < kPrepMaxRows; ++j) {
        const int i = threadIdx.x + kPrepThreads * j;
        if (i >= d) continue;
        const float z = w[j] * inv;            // exact
        const float c = rintf(z);
        const float r = z - c;                 // exact
        const float dd = rintf(r * 128.0f);
        fmax_ = fmaxf(fmax_, fabsf(u * (r - dd * 0.0078125f)));  // exact remainder of w
        ws.wc[static_cast<size_t>(e) * d + i] = static_cast<int8_t>(static_cast<int>(c));
        ws.wd[static_cast<size_t>(e) * d + i] = static_cast<int8_t>(static_cast<int>(dd));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) fmax_ = fmaxf(fmax_, __shfl_xor_sync(0xffffffffu, fmax_, o));
    if (lane == 0) sm_f[warp] = fmax_;
    __syncthreads();
    if (threadIdx.x == 0) {
        float f = 0.0f;
        for (int i = 0; i < kPrepThreads / 32; ++i) f = fmaxf(f, sm_f[i]);
        ws.F_e[e] = f;
    }
}

// ---------------------------------------------------------------------------
// Approximate logits on the tensor cores.  One CTA per 64 tokens x 128
// experts.  Operands (int8, K-major rows of 128 bytes, 128-byte swizzle) are
// brought in by TMA, 128 K per stage: the expert digits c, d (A, M = 128) and
// the token digits a, b (B, N = 64).  Per 32-wide K step four MMAs accumulate
// P += a c, Q += a d + b c, R += b d in int32 (TMEM columns 0, 64, 128), so
//   x' . w' = s_t u_e (P + Q / 128 + R / 16384)
// exactly; the epilogue forms it in double (exact: P, Q, R < 2^31, s_t u_e a
// power of two), adds the bias and rounds once to fp32.
// Warps: 0 TMA producer, 1 TMEM allocation and MMA issue, 2-5 epilogue (TMEM
// lane quadrant = warp % 4).
// ---------------------------------------------------------------------------
constexpr int kApN = 64;
constexpr int kApStages = 3;
constexpr int kApATile = 128 * 128;
constexpr int kApBTile = kApN * 128;
constexpr int kApStageBytes = 2 * kApATile + 2 * kApBTile;
constexpr int kApThreads = 192;
constexpr int kApSmem = kApStages * kApStageBytes + 1024 + 256;

__device__ __forceinline__ uint32_t make_idesc_s8(int M, int N) {
    return (2u << 4)                                   // D format s32
           | (1u << 7)                                 // A signed 8-bit
           | (1u << 10)                                // B signed 8-bit
           | (static_cast<uint32_t>(N >> 3) << 17)
           | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_s8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 TMEM lanes x 16 columns: thread i of the warp holds lane (base + i),
// columns col .. col + 15
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__global__ void __launch_bounds__(kApThreads, 1)
router_approx_kernel(const __grid_constant__ ApproxArgs a) {
    extern __shared__ uint8_t ap_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ap_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    pdl_launch_dependents();
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t bar0 = sbase + kApStages * kApStageBytes;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (kApStages + s); };
    const uint32_t accfull = bar0 + 8u * (2 * kApStages);
    const uint32_t drain = accfull + 8u;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kApStages * kApStageBytes + 8 * (2 * kApStages + 2));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kApStages; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(accfull, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();  // the digits come from the prep kernel
    const int t0 = blockIdx.x * kApN;
    const int e0 = blockIdx.y * 128;
    const int KC = a.d / 128;
    if (warp == 0) {
        int issued = 0;
        bool ok = true;
        for (int c = 0; c < KC; ++c) {
            const int s = c % kApStages;
            if (!__all_sync(0xffffffffu, mbar_wait(empty(s), ((c / kApStages) & 1) ^ 1, abort_flag))) {
                ok = false;
                break;
            }
            if (elect_one()) {
                const uint32_t st = sbase + s * kApStageBytes;
                mbar_arrive_expect_tx(full(s), kApStageBytes);
                tma_load_2d(st, &a.map_wc, c * 128, e0, full(s));
                tma_load_2d(st + kApATile, &a.map_wd, c * 128, e0, full(s));
                tma_load_2d(st + 2 * kApATile, &a.map_xa, c * 128, t0, full(s));
                tma_load_2d(st + 2 * kApATile + kApBTile, &a.map_xb, c * 128, t0, full(s));
            }
            __syncwarp();
            ++issued;
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            report_error(a.status, MOE_ERR_DEVICE_TIMEOUT, 600);
            for (int i = issued > kApStages ? issued - kApStages : 0; i < issued; ++i) {
                const uint64_t tt = globaltimer();
                while (!mbar_try_wait(full(i % kApStages), (i / kApStages) & 1))
                    if (globaltimer() - tt > 200000000ull) break;
            }
        }
    } else if (warp == 1) {
        const uint32_t idesc = make_idesc_s8(128, kApN);
        const uint32_t P = tmem, Q = tmem + kApN, R = tmem + 2 * kApN;
        bool ok = true;
        for (int c = 0; c < KC; ++c) {
            const int s = c % kApStages;
            if (!__all_sync(0xffffffffu, mbar_wait(full(s), (c / kApStages) & 1, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t st = sbase + s * kApStageBytes;
            const uint64_t dc = make_sw128_desc(st), dd = make_sw128_desc(st + kApATile);
            const uint64_t da = make_sw128_desc(st + 2 * kApATile);
            const uint64_t db = make_sw128_desc(st + 2 * kApATile + kApBTile);
            if (elect_one()) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint32_t acc = (c > 0 || ks > 0) ? 1u : 0u;
                    mma_s8(P, dc + 2 * ks, da + 2 * ks, idesc, acc);
                    mma_s8(Q, dd + 2 * ks, da + 2 * ks, idesc, acc);
                    mma_s8(Q, dc + 2 * ks, db + 2 * ks, idesc, 1u);
                    mma_s8(R, dd + 2 * ks, db + 2 * ks, idesc, acc);
                }
                mma_commit(empty(s));
            }
            __syncwarp();
        }
        if (elect_one()) mma_commit(ok ? accfull : drain);
        __syncwarp();
        if (!ok) {
            if (lane == 0) {
                *abort_flag = 1;
                report_error(a.status, MOE_ERR_DEVICE_TIMEOUT, 601);
            }
            const uint64_t tt = globaltimer();
            while (!mbar_try_wait(drain, 0))
                if (globaltimer() - tt > 200000000ull) break;
        }
    } else {
        const int q = warp & 3;
        const int e = e0 + 32 * q + lane;
        if (__all_sync(0xffffffffu, mbar_wait(accfull, 0, abort_flag))) {
            tc_fence_after();
            const double su = e < a.E ? static_cast<double>(__ldg(a.u_e + e)) : 0.0;
            const double be = (e < a.E && a.b_r != nullptr) ? static_cast<double>(__ldg(a.b_r + e)) : 0.0;
            const uint32_t lb = static_cast<uint32_t>(32 * q) << 16;
#pragma unroll 1
            for (int cb = 0; cb < kApN / 16; ++cb) {
                uint32_t p[16], qq[16], r[16];
                tmem_ld_32x32b_x16(tmem + lb + cb * 16, p);
                tmem_ld_32x32b_x16(tmem + lb + kApN + cb * 16, qq);
                tmem_ld_32x32b_x16(tmem + lb + 2 * kApN + cb * 16, r);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int t = t0 + cb * 16 + j;
                    if (t < a.T && e < a.E) {
                        const double v = static_cast<double>(static_cast<int32_t>(p[j])) +
                                         static_cast<double>(static_cast<int32_t>(qq[j])) * 0.0078125 +
                                         static_cast<double>(static_cast<int32_t>(r[j])) * 6.103515625e-05;
                        const double l = v * (static_cast<double>(__ldg(a.s_t + t)) * su) + be;
                        a.L[static_cast<size_t>(t) * a.E + e] = static_cast<float>(l);
                    }
                }
            }
        } else if (lane == 0) {
            report_error(a.status, MOE_ERR_DEVICE_TIMEOUT, 602);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ---------------------------------------------------------------------------
// The bound delta (upward rounding throughout).  gamma_72 = 72 u / (1 - 72 u),
// u = 2^-24, rounded up.
// ---------------------------------------------------------------------------
constexpr float kGamma72 = 4.2916e-6f;

__device__ __forceinline__ float route_delta(float L, float A_t, float E_t, float N_t, float F_e,
                                             float B_e, float Wn_e, float babs) {
    const float d1 = __fmul_ru(F_e, A_t);
    const float d2 = __fmul_ru(E_t, B_e);
    const float d3 = __fmul_ru(kGamma72, __fadd_ru(__fmul_ru(N_t, Wn_e), babs));
    const float d4 = __fmul_ru(1.1920929e-07f, fabsf(L));  // 2^-23 |L|
    return __fadd_ru(__fadd_ru(d1, d2), __fadd_ru(d3, __fadd_ru(d4, 1e-30f)));
}

// ---------------------------------------------------------------------------
// Selection, one warp per token.
// ---------------------------------------------------------------------------
constexpr int kSelWarps = 8;
constexpr int kSelPer = kMaxExperts / 32;   // experts per lane
constexpr int kSelXPer = 64;                // x values per lane: d <= 2048
constexpr int kSelChunk = 16;               // column loads in flight per candidate

__global__ void __launch_bounds__(kSelWarps * 32)
router_select_kernel(const uint16_t* __restrict__ x, RouterFastWs ws, const float* __restrict__ b_r, int T,
                     int d, int E, int k, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                     int32_t* __restrict__ hist) {
    __shared__ float rows[kSelWarps][kMaxExperts];
    __shared__ __align__(16) uint16_t xsm[kSelWarps][32 * kSelXPer];
    __shared__ int clist[kSelWarps][kMaxExperts];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    pdl_launch_dependents();
    pdl_wait();
    const int t = blockIdx.x * kSelWarps + warp;
    if (t >= T) return;
    // the token's x row into shared memory (16-byte pieces)
    const int steps = d >> 5;
    {
        const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d);
        uint4* dst = reinterpret_cast<uint4*>(xsm[warp]);
        for (int v = lane; v < d / 8; v += 32) dst[v] = __ldg(src + v);
    }
    // bounds: lower / upper of every expert
    const float A = ws.A_t[t], Et = ws.E_t[t], N = ws.N_t[t];
    float lo[kSelPer], up[kSelPer], lw[kSelPer];
#pragma unroll
    for (int i = 0; i < kSelPer; ++i) {
        const int e = lane + 32 * i;
        lo[i] = up[i] = -INFINITY;
        if (e < E) {
            const float L = ws.L[static_cast<size_t>(t) * E + e];
            const float babs = b_r != nullptr ? fabsf(__ldg(b_r + e)) : 0.0f;
            const float dl = route_delta(L, A, Et, N, ws.F_e[e], ws.B_e[e], ws.Wn_e[e], babs);
            lo[i] = __fsub_rd(L, dl);
            up[i] = __fadd_ru(L, dl);
        }
        lw[i] = lo[i];
    }
    // theta: the k-th largest lower bound (k rounds of a warp arg-max)
    float theta = -INFINITY;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = 1 << 30;
#pragma unroll
        for (int i = 0; i < kSelPer; ++i) {
            const int id = lane + 32 * i;
            if (id < E && (lw[i] > bv || (lw[i] == bv && id < bi))) {
                bv = lw[i];
                bi = id;
            }
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, m);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, m);
            if (ov > bv || (ov == bv && oi < bi)) {
                bv = ov;
                bi = oi;
            }
        }
#pragma unroll
        for (int i = 0; i < kSelPer; ++i)
            if (lane + 32 * i == bi) lw[i] = -INFINITY;
        theta = bv;
    }
    // the candidates' fixed-order logits; the other experts read as -inf
    for (int e = lane; e < E; e += 32) rows[warp][e] = -INFINITY;
    // candidate list (ascending id) in this warp's shared list
    int nc = 0;
#pragma unroll
    for (int i = 0; i < kSelPer; ++i) {
        const unsigned cand = __ballot_sync(0xffffffffu, lane + 32 * i < E && up[i] >= theta);
        if ((cand >> lane) & 1u) clist[warp][nc + __popc(cand & ((1u << lane) - 1u))] = 32 * i + lane;
        nc += __popc(cand);
    }
    __syncwarp();  // the x row and the list are in shared memory
    // two candidates at a time; lane p runs chain p = fma(x[p + 32 m],
    // W_r[p + 32 m][e], chain p) in ascending m for each, with the column's
    // loads issued sixteen at a time ahead of their multiply-adds
    const uint16_t* xw = xsm[warp] + lane;
    for (int c0 = 0; c0 < nc; c0 += 2) {
        const int e0 = clist[warp][c0];
        const int e1 = c0 + 1 < nc ? clist[warp][c0 + 1] : e0;
        const float* w0 = ws.wt + static_cast<size_t>(e0) * d + lane;
        const float* w1 = ws.wt + static_cast<size_t>(e1) * d + lane;
        float a0 = 0.0f, a1 = 0.0f;
        for (int m0 = 0; m0 < steps; m0 += kSelChunk) {
            float v0[kSelChunk], v1[kSelChunk];
            if (m0 + kSelChunk <= steps) {
#pragma unroll
                for (int j = 0; j < kSelChunk; ++j) {
                    v0[j] = __ldg(w0 + 32 * (m0 + j));
                    v1[j] = __ldg(w1 + 32 * (m0 + j));
                }
#pragma unroll
                for (int j = 0; j < kSelChunk; ++j) {
                    const float xv = bf16_bits_to_float(xw[32 * (m0 + j)]);
                    a0 = __fmaf_rn(xv, v0[j], a0);
                    a1 = __fmaf_rn(xv, v1[j], a1);
                }
            } else {
                for (int m = m0; m < steps; ++m) {
                    const float xv = bf16_bits_to_float(xw[32 * m]);
                    a0 = __fmaf_rn(xv, __ldg(w0 + 32 * m), a0);
                    a1 = __fmaf_rn(xv, __ldg(w1 + 32 * m), a1);
                }
            }
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) {
            a0 = __fadd_rn(a0, __shfl_xor_sync(0xffffffffu, a0, m));
            a1 = __fadd_rn(a1, __shfl_xor_sync(0xffffffffu, a1, m));
        }
        if (lane == 0) {
            rows[warp][e0] = b_r != nullptr ? __fadd_rn(a0, __ldg(b_r + e0)) : a0;
            rows[warp][e1] = b_r != nullptr ? __fadd_rn(a1, __ldg(b_r + e1)) : a1;
        }
    }
    __syncwarp();
    int my_id;
    float my_w;
    warp_topk(rows[warp], E, k, lane, my_id, my_w);
    if (lane < k) {
        topk_idx[static_cast<size_t>(t) * k + lane] = my_id;
        topk_w[static_cast<size_t>(t) * k + lane] = my_w;
        atomicAdd(hist + static_cast<size_t>(t / kRouteGroupT) * E + my_id, 1);
    }
}

}  // namespace

bool router_fast_supported(int T, int d, int E) {
    return T >= kFastRouterMinT && E % 8 == 0 && E <= kMaxExperts && d % 128 == 0 &&
           d <= kPrepThreads * kPrepMaxRows && d <= 8 * 32 * kPrepMaxVec && d <= 32 * kSelXPer;
}

size_t router_fast_ws_bytes(int T, int d, int E) {
    auto r = [](size_t v) { return (v + 255) / 256 * 256; };
    const size_t t = static_cast<size_t>(T), dd = static_cast<size_t>(d), e = static_cast<size_t>(E);
    return 2 * r(t * dd) + 2 * r(e * dd) + 4 * r(t * 4) + 4 * r(e * 4) + r(e * dd * 4);
}

RouterFastWs router_fast_ws(uint8_t* base, float* L, int T, int d, int E) {
    auto r = [](size_t v) { return (v + 255) / 256 * 256; };
    const size_t t = static_cast<size_t>(T), dd = static_cast<size_t>(d), e = static_cast<size_t>(E);
    RouterFastWs w;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        uint8_t* p = base + o;
        o += r(bytes);
        return p;
    };
    w.xa = reinterpret_cast<int8_t*>(take(t * dd));
    w.xb = reinterpret_cast<int8_t*>(take(t * dd));
    w.wc = reinterpret_cast<int8_t*>(take(e * dd));
    w.wd = reinterpret_cast<int8_t*>(take(e * dd));
    w.s_t = reinterpret_cast<float*>(take(t * 4));
    w.E_t = reinterpret_cast<float*>(take(t * 4));
    w.A_t = reinterpret_cast<float*>(take(t * 4));
    w.N_t = reinterpret_cast<float*>(take(t * 4));
    w.u_e = reinterpret_cast<float*>(take(e * 4));
    w.F_e = reinterpret_cast<float*>(take(e * 4));
    w.B_e = reinterpret_cast<float*>(take(e * 4));
    w.Wn_e = reinterpret_cast<float*>(take(e * 4));
    w.wt = reinterpret_cast<float*>(take(e * dd * 4));
    w.L = L;
    return w;
}

static cudaError_t router_fast_setup(int* num_sms) {
    static std::atomic<int> ready[64];
    static std::atomic<int> sms[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (ready[dev].load(std::memory_order_acquire) == 0) {
        e = cudaFuncSetAttribute(router_approx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kApSmem);
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

cudaError_t prepare_router_fast() {
    int n = 0;
    return router_fast_setup(&n);
}

cudaError_t launch_router_fast(const uint16_t* x, const float* W, const float* b, int T, int d, int E,
                               int k, const RouterFastWs& ws, int32_t* topk_idx, float* topk_w,
                               int32_t* hist, int hist_n, int32_t* status, cudaStream_t st) {
    int num_sms = 0;
    cudaError_t e = router_fast_setup(&num_sms);
    if (e != cudaSuccess) return e;
    const int nxb = (T + 7) / 8;
    e = launch_pdl(router_prep_kernel, dim3(nxb + E), dim3(kPrepThreads), 0, st, x, W, T, d, E, nxb, ws,
                   hist, hist_n, status);
    if (e != cudaSuccess) return e;
    ApproxArgs a{};
    if ((e = encode_u8_rows_map(&a.map_wc, ws.wc, E, d, 128)) != cudaSuccess) return e;
    if ((e = encode_u8_rows_map(&a.map_wd, ws.wd, E, d, 128)) != cudaSuccess) return e;
    if ((e = encode_u8_rows_map(&a.map_xa, ws.xa, T, d, kApN)) != cudaSuccess) return e;
    if ((e = encode_u8_rows_map(&a.map_xb, ws.xb, T, d, kApN)) != cudaSuccess) return e;
    a.s_t = ws.s_t;
    a.u_e = ws.u_e;
    a.b_r = b;
    a.L = ws.L;
    a.T = T;
    a.d = d;
    a.E = E;
    a.status = status;
    e = launch_pdl(router_approx_kernel, dim3((T + kApN - 1) / kApN, (E + 127) / 128), dim3(kApThreads),
                   kApSmem, st, a);
    if (e != cudaSuccess) return e;
    const int sel_grid = (T + kSelWarps - 1) / kSelWarps;
    return launch_pdl(router_select_kernel, dim3(sel_grid), dim3(kSelWarps * 32), 0, st, x, ws, b, T, d, E, k,
                      topk_idx, topk_w, hist);
}

}  // namespace moe
