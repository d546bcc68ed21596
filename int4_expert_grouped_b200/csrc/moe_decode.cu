// Small-batch (decode) path of the MoE layer: the same operation as the
// batched path (inblix article "Perplexity's Lily engine beats MLX by 35% on
// M5 Max, no PyTorch needed", paragraph 3: routing, prefix scan, scatter,
// block map, dequantisation-fused expert GEMMs, weighted combine) for a few
// tokens, where the layer is bound by reading the selected experts' int4
// weights from HBM.  Three launches chained with programmatic dependent
// launch, so each one's start-up overlaps the previous one's tail:
//
//   decode_route_kernel    one cluster of 8 CTAs: each CTA runs the 32 fp32
//                          fused-multiply-add chains of its E/8 experts
//                          (lanes over experts, so W_r is read in row
//                          segments), combines them with the router's fixed
//                          butterfly tree and writes the logits into CTA 0's
//                          shared memory; CTA 0 then does top-k, counts,
//                          scan, block map and scatter and writes them out
//   decode_gateup_kernel   one warp per weight row (8 gate and 8 up rows per
//                          CTA) streams its int4 row and dots it with the
//                          block's x rows, group by group (scale and bias
//                          applied to each group's sum); SwiGLU gives bf16
//                          rows of h
//   decode_down_kernel     one warp per output feature (16 per CTA): the down
//                          row of every selected expert against that expert's
//                          h rows, each output rounded to bf16, then the
//                          routing-weighted sum over a token's slots in order
//
// The expert kernels are instantiated per batch size, so their loops over the
// batch's rows are fully unrolled without dead code.  The weights are read in
// the prepacked block layout of the batched path, so one packed copy serves
// both.  Rounding differs from the batched path only in the weights: there
// each dequantised weight is rounded to bf16 before the MMA, here the exact
// codes meet the operands and each group's scale and bias apply to its fp32
// sum (closer to the unrounded q*s + b).  Both keep fp32 sums, bf16 h, bf16
// expert outputs and the fp32 slot-order combine.
#include <cooperative_groups.h>

#include <algorithm>

#include "moe_route_common.cuh"

namespace moe {
namespace {

constexpr int kDecodeMaxAssign = kDecodeMaxT * kMaxTopk;
constexpr int kRouteCtas = 8;       // cluster size of the routing kernel: E/8 experts each
constexpr int kRowThreads = 512;    // 16 warps, one weight row each
constexpr int kGuVecs = 2;          // 16-byte nibble vectors per lane and gate/up row: d <= 2048
constexpr int kDnVecs = 1;          // 16-byte nibble vectors per lane and down row: f <= 1024
// experts whose down loads a lane issues together (fewer for larger batches,
// whose operand loops need the registers)
template <int kT>
constexpr int dn_block_batch() { return kT <= 4 ? 8 : 4; }


__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ld_nc_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// sum of the 8 products of bf16 vectors w and x, added to acc
__device__ __forceinline__ float dot8(const uint4& w, const uint4& x, float acc) {
    const uint32_t wa[4] = {w.x, w.y, w.z, w.w};
    const uint32_t xa[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        BF2 a, b;
        a.u = wa[i];
        b.u = xa[i];
        const float2 af = __bfloat1622float2(a.h);
        const float2 bf = __bfloat1622float2(b.h);
        acc = fmaf(af.x, bf.x, acc);
        acc = fmaf(af.y, bf.y, acc);
    }
    return acc;
}

// copy n 16-byte vectors global -> shared by the whole CTA, four loads in
// flight per thread before their stores
__device__ __forceinline__ void cta_copy16(void* dst, const void* src, int n) {
    const uint4* s = reinterpret_cast<const uint4*>(src);
    uint4* d = reinterpret_cast<uint4*>(dst);
    const int stride = blockDim.x;
    for (int i0 = threadIdx.x; i0 < n; i0 += 4 * stride) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (i0 + u * stride < n) v[u] = ld_nc_v4(s + i0 + u * stride);
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (i0 + u * stride < n) d[i0 + u * stride] = v[u];
    }
}

// Copy rows of bf16 operands into shared memory with each row's 16-byte
// pieces reordered: piece v = 4q + w (K 32q + 8w .. + 7) goes to slot
// w * nvec + q, so the lanes of a warp, which own consecutive vectors q and
// read piece w of each at the same time, touch consecutive 16-byte slots.
// nvec = row length / 32; n_rows rows of 4 * nvec pieces.
__device__ __forceinline__ void cta_copy_rows_by_vector(void* dst, const void* src, int n_rows,
                                                        int nvec) {
    const uint4* s = reinterpret_cast<const uint4*>(src);
    uint4* d = reinterpret_cast<uint4*>(dst);
    const int per_row = 4 * nvec;
    const int n = n_rows * per_row;
    const int stride = blockDim.x;
    for (int i0 = threadIdx.x; i0 < n; i0 += 4 * stride) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (i0 + u * stride < n) v[u] = ld_nc_v4(s + i0 + u * stride);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * stride;
            if (i < n) {
                const int r = i / per_row;
                const int pv = i - r * per_row;
                d[r * per_row + (pv & 3) * nvec + (pv >> 2)] = v[u];
            }
        }
    }
}

__device__ __forceinline__ uint16_t bf16_round_bits(float v) {
    const __nv_bfloat16 b = __float2bfloat16_rn(v);
    return *reinterpret_cast<const uint16_t*>(&b);
}

// ---------------------------------------------------------------------------
// Routing of the few tokens in shared memory (CTA 0 of the routing cluster,
// kRowThreads threads) from the logits lg [T][E]: top-k (each (token, expert)
// pair finds its slot in parallel; the warp of a token then forms the
// weights), counts (integer atomics), offsets (exclusive scan), block map
// (ceil(count / kBlockT) tiles per expert in ascending expert order), and the
// stable scatter (the rank of assignment a within its expert is the number of
// earlier assignments to that expert).
// ---------------------------------------------------------------------------
struct DecodeRoute {
    float lg[kDecodeMaxT * kMaxExperts];
    float sel[kDecodeMaxAssign];  // logit of each selected slot
    int idx[kDecodeMaxAssign];
    float w[kDecodeMaxAssign];
    int sa[kDecodeMaxAssign];
    int pos[kDecodeMaxAssign];
    int cnt[kMaxExperts];
    int off[kMaxExperts + 1];
    int bo[kMaxExperts + 1];
    int bm[3 * kDecodeMaxAssign];
    int nb;
    int sh_warp[kRowThreads / 32 + 1];
};

__device__ void route_from_logits(int T, int E, int k, int max_blocks, DecodeRoute& R) {
    static_assert(kRowThreads >= kMaxExperts, "one thread per expert");
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int tid = threadIdx.x;
    const int Tk = T * k;
    if (tid < E) R.cnt[tid] = 0;
    for (int it = tid; it < T * E; it += kRowThreads) {
        const int t = it / E;
        const int e = it - t * E;
        const int slot = expert_slot(R.lg + t * E, E, e);
        if (slot < k) {
            R.idx[t * k + slot] = e;
            R.sel[t * k + slot] = R.lg[it];
        }
    }
    __syncthreads();
    for (int t = warp; t < T; t += kRowThreads / 32) {
        const float wt = warp_slot_weights(lane < k ? R.sel[t * k + lane] : 0.0f, k, lane);
        if (lane < k) R.w[t * k + lane] = wt;
    }
    __syncthreads();
    for (int a = tid; a < Tk; a += kRowThreads) atomicAdd(&R.cnt[R.idx[a]], 1);
    __syncthreads();
    const int c = tid < E ? R.cnt[tid] : 0;
    int total = 0;
    const int off = block_exclusive_scan<kRowThreads>(c, R.sh_warp, &total);
    if (tid < E) R.off[tid] = off;
    if (tid == 0) R.off[E] = total;
    const int nt = (c + kBlockT - 1) / kBlockT;
    int nb_total = 0;
    const int bo = block_exclusive_scan<kRowThreads>(tid < E ? nt : 0, R.sh_warp, &nb_total);
    if (tid < E) {
        R.bo[tid] = bo;
        for (int i = 0; i < nt && bo + i < max_blocks && bo + i < kDecodeMaxAssign; ++i) {
            R.bm[3 * (bo + i) + 0] = tid;
            R.bm[3 * (bo + i) + 1] = off + i * kBlockT;
            R.bm[3 * (bo + i) + 2] = min(kBlockT, c - i * kBlockT);
        }
    }
    if (tid == 0) {
        R.bo[E] = nb_total;
        R.nb = min(min(nb_total, max_blocks), kDecodeMaxAssign);
    }
    for (int a = tid; a < Tk; a += kRowThreads) {
        const int e = R.idx[a];
        int rank = 0;
        for (int a2 = 0; a2 < a; ++a2) rank += R.idx[a2] == e;
        const int p = R.off[e] + rank;
        R.sa[p] = a;
        R.pos[a] = p;
    }
    __syncthreads();
}

struct DecodeRouteOut {
    int32_t* topk_idx;
    float* topk_w;
    int32_t* counts;
    int32_t* offsets;
    int32_t* sorted_assign;
    int32_t* pos;
    int32_t* block_offsets;
    int32_t* block_map;
    int32_t* num_blocks;
};

__device__ void write_route(const DecodeRoute& R, const DecodeRouteOut& o, int Tk, int E) {
    for (int a = threadIdx.x; a < Tk; a += blockDim.x) {
        o.topk_idx[a] = R.idx[a];
        o.topk_w[a] = R.w[a];
        o.sorted_assign[a] = R.sa[a];
        o.pos[a] = R.pos[a];
    }
    for (int e = threadIdx.x; e <= E; e += blockDim.x) {
        if (e < E) o.counts[e] = R.cnt[e];
        o.offsets[e] = R.off[e];
        o.block_offsets[e] = R.bo[e];
    }
    for (int i = threadIdx.x; i < 3 * R.nb; i += blockDim.x) o.block_map[i] = R.bm[i];
    if (threadIdx.x == 0) o.num_blocks[0] = R.nb;
}

// ---------------------------------------------------------------------------
// Routing.  One cluster of kRouteCtas CTAs; CTA c owns experts
// [c*EC, (c+1)*EC), EC = E / kRouteCtas <= 32.  The logit of (t, e) is 32
// chains, chain p taking i = p, p+32, ... in ascending i with fused
// multiply-add from 0, combined by the xor butterfly m = 16..1 (the value
// lane p holds after step m is v_p + v_{p^m}, so the result is the tree that
// adds chains q and q + m for q < m, m = 16..1), plus the bias.  Item
// (p, el) of a CTA runs chain p of expert e0 + el for all T tokens: a group
// of EC lanes reads EC consecutive floats of a W_r row per step, from a copy
// of the CTA's W_r columns that all threads load with 16-byte vectors first.
// The logits go to CTA 0's shared memory (distributed shared memory), which
// then routes.  Dynamic shared memory: x [T][d] bf16, the W_r columns [d][EC]
// fp32, the chains [T][32][33] fp32.
// ---------------------------------------------------------------------------
__global__ void __cluster_dims__(kRouteCtas, 1, 1) __launch_bounds__(kRowThreads)
decode_route_kernel(const uint16_t* __restrict__ x, const float* __restrict__ W,
                    const float* __restrict__ bias, int T, int d, int E, int k, int max_blocks,
                    DecodeRouteOut ro, int32_t* __restrict__ status) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    __shared__ DecodeRoute R;
    extern __shared__ __align__(16) uint8_t dsm[];
    const uint16_t* xs = reinterpret_cast<const uint16_t*>(dsm);
    float* ws = reinterpret_cast<float*>(dsm + static_cast<size_t>(T) * d * 2);  // [i][EC]
    float* cs = ws + static_cast<size_t>(d) * (E / kRouteCtas);                  // [t][p][33]
    pdl_launch_dependents();
    const int rank = static_cast<int>(cluster.block_rank());
    const int EC = E / kRouteCtas;
    const int e0 = rank * EC;
    const int nsteps = d >> 5;
    const int items = 32 * EC;
    cta_copy16(dsm, x, T * d / 8);
    {
        // W_r[:, e0 .. e0+EC) -> ws: 16-byte vectors (EC % 4 == 0), 16 in
        // flight per thread before their stores
        const int nv = d * (EC / 4);
        const int vrow = EC / 4;
        for (int v0 = threadIdx.x; v0 < nv; v0 += 16 * kRowThreads) {
            float4 v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int vi = v0 + u * kRowThreads;
                if (vi < nv) {
                    const int i = vi / vrow;
                    v[u] = __ldg(reinterpret_cast<const float4*>(W + static_cast<size_t>(i) * E + e0) +
                                 (vi - i * vrow));
                }
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int vi = v0 + u * kRowThreads;
                if (vi < nv) reinterpret_cast<float4*>(ws)[vi] = v[u];
            }
        }
    }
    __syncthreads();
    for (int it = threadIdx.x; it < items; it += kRowThreads) {
        const int p = it / EC;
        const int el = it - p * EC;
#pragma unroll 1
        for (int t = 0; t < T; ++t) {
            float a = 0.0f;
#pragma unroll 16
            for (int s = 0; s < nsteps; ++s)
                a = __fmaf_rn(bf16_bits_to_float(xs[t * d + 32 * s + p]), ws[(32 * s + p) * EC + el], a);
            cs[(t * 32 + p) * 33 + el] = a;
        }
    }
    __syncthreads();
    float* lg0 = cluster.map_shared_rank(R.lg, 0);
    for (int it = threadIdx.x; it < T * EC; it += kRowThreads) {
        const int t = it / EC;
        const int el = it - t * EC;
        float v[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) v[q] = cs[(t * 32 + q) * 33 + el];
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1)
#pragma unroll
            for (int q = 0; q < m; ++q) v[q] = __fadd_rn(v[q], v[q + m]);
        lg0[t * E + e0 + el] = bias ? __fadd_rn(v[0], bias[e0 + el]) : v[0];
    }
    cluster.sync();  // all logits are in CTA 0; no CTA touches another's memory after this
    if (rank != 0) return;
    // everything above reads only the layer's inputs; the outputs below are
    // read by the previous call's kernels, which must have finished
    pdl_wait();
    // the status word reports the most recent call: the first kernel clears it
    if (threadIdx.x < 2) status[threadIdx.x] = 0;
    route_from_logits(T, E, k, max_blocks, R);
    write_route(R, ro, T * k, E);
}

// ---------------------------------------------------------------------------
// One packed weight row against kT bf16 operand rows, by one warp.  The row
// lives in blocks base + c * chunk_stride (one per 64-wide K chunk c) at
// packed row prow: 32 bytes of nibbles per chunk, then the (scale, bias)
// entries.  Vector q (16 bytes, K 32q .. 32q+31) is half q % 2 of chunk q / 2;
// its (scale, bias) pair is the row's entry for the group holding that half.
// Lane l owns vectors l, l + 32, ... (< nv): row_load issues all their loads
// at once; row_dots expands each vector once and dots it with every operand
// row (stored by cta_copy_rows_by_vector) into the lane's acc[i].
// ---------------------------------------------------------------------------
template <int kV>
struct RowLoads {
    uint4 nib[kV];
    uint32_t sb[kV];
};

template <int kV>
__device__ __forceinline__ void row_load(RowLoads<kV>& L, const uint8_t* __restrict__ base,
                                         size_t chunk_stride, int prow, int nib_bytes, int gpc,
                                         int nv, int lane) {
#pragma unroll
    for (int u = 0; u < kV; ++u) {
        const int q = lane + 32 * u;
        if (q < nv) {
            const uint8_t* blk = base + static_cast<size_t>(q >> 1) * chunk_stride;
            const int half = q & 1;
            L.nib[u] = ld_nc_v4(blk + prow * 32 + half * 16);
            L.sb[u] = ld_nc_u32(blk + nib_bytes + (prow * gpc + half * (gpc - 1)) * 4);
        }
    }
}

// Dot products of one packed row with every operand row, factored by group:
// with w = q*s + b, sum_k w_k x_k over the vector's 32 K values (one group, or
// half of a 64-wide group with the same s and b) is s * sum_k q_k x_k +
// b * sum_k x_k.  The nibbles become fp32 128 + q exactly (q in mantissa
// bits 16-19 of 128.0), pairs of them meet pairs of operands in packed fp32
// FMAs, and 128 * sum_k x_k (sums: per row and vector) is taken off at the
// end.  The weights are not rounded to bf16 on this path.
template <int kT, int kV>
__device__ __forceinline__ void row_dots(const RowLoads<kV>& L, const uint16_t* const* rows,
                                         const float* const* sums, int nv, int lane, float* acc) {
#pragma unroll
    for (int u = 0; u < kV; ++u) {
        const int q = lane + 32 * u;
        if (q < nv) {
            const float s = __uint_as_float(L.sb[u] << 16);
            const float b = __uint_as_float(L.sb[u] & 0xFFFF0000u);
            float2 a2[kT];
#pragma unroll
            for (int t = 0; t < kT; ++t) a2[t] = make_float2(0.0f, 0.0f);
            const uint32_t words[4] = {L.nib[u].x, L.nib[u].y, L.nib[u].z, L.nib[u].w};
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
                const uint32_t w = words[wi];  // K 32q + 8wi + 2i (bits 4i), + 2i + 1 (bits 16+4i)
                float2 wp[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    wp[i].x = __uint_as_float(((w << (16 - 4 * i)) & 0x000F0000u) | 0x43000000u);
                    wp[i].y = __uint_as_float(((w >> (4 * i)) & 0x000F0000u) | 0x43000000u);
                }
#pragma unroll
                for (int t = 0; t < kT; ++t) {
                    const uint4 xv = *reinterpret_cast<const uint4*>(rows[t] + 8 * (wi * nv + q));
                    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float2 xf = make_float2(__uint_as_float(xw[i] << 16),
                                                      __uint_as_float(xw[i] & 0xFFFF0000u));
                        a2[t] = __ffma2_rn(wp[i], xf, a2[t]);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < kT; ++t) {
                const float xs = sums[t][q];
                acc[t] = fmaf(s, a2[t].x + a2[t].y - 128.0f * xs, fmaf(b, xs, acc[t]));
            }
        }
    }
}

// sums[r * nvec + q] = sum of the 32 operand values of vector q of row r
// (operand rows stored by cta_copy_rows_by_vector)
__device__ __forceinline__ void cta_vector_sums(const uint16_t* rows, int n_rows, int nvec,
                                                float* sums) {
    for (int it = threadIdx.x; it < n_rows * nvec; it += blockDim.x) {
        const int r = it / nvec;
        const int q = it - r * nvec;
        const uint16_t* row = rows + static_cast<size_t>(r) * nvec * 32;
        float acc = 0.0f;
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            const uint4 v = *reinterpret_cast<const uint4*>(row + 8 * (wi * nvec + q));
            const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc += __uint_as_float(vw[i] << 16) + __uint_as_float(vw[i] & 0xFFFF0000u);
        }
        sums[it] = acc;
    }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
    return v;
}

// ---------------------------------------------------------------------------
// Gate/up and SwiGLU for a batch of kT tokens.  Grid: min(E, kT*k) blocks x
// f/16 feature slices (CTAs past the number of blocks return).  Warp r takes
// feature 16q' + r of tile j: its gate row and its up row, so SwiGLU needs
// no exchange between warps.  Rows of the block beyond its count repeat its
// first row and are not stored.  Dynamic shared memory: x [kT][d].
// ---------------------------------------------------------------------------
template <int kT>
__global__ void __launch_bounds__(kRowThreads)
decode_gateup_kernel(const uint16_t* __restrict__ x, const uint8_t* __restrict__ wpack, int d,
                     int k, int f, int group, int bb, DecodeRouteOut ro, uint16_t* __restrict__ h) {
    __shared__ int sblk[3 + kT];  // expert, first row, rows, token of each row
    __shared__ float xsum[kT * 64];  // per token and 32-wide vector (d <= 2048)
    extern __shared__ __align__(16) uint8_t dsm[];
    const uint16_t* xs = reinterpret_cast<const uint16_t*>(dsm);
    pdl_launch_dependents();
    // x does not depend on the routing kernel
    cta_copy_rows_by_vector(dsm, x, kT, d / 32);
    __syncthreads();
    cta_vector_sums(xs, kT, d / 32, xsum);
    pdl_wait();
    const int nq = f / 16;
    const int b = blockIdx.x / nq;
    const int q = blockIdx.x - b * nq;
    if (b >= min(ro.num_blocks[0], kDecodeMaxAssign)) return;
    if (threadIdx.x < 3) sblk[threadIdx.x] = ro.block_map[3 * b + threadIdx.x];
    __syncthreads();
    const int row0 = sblk[1];
    const int nrows = min(sblk[2], kT);
    if (threadIdx.x < kT)
        sblk[3 + threadIdx.x] =
            ro.sorted_assign[row0 + min(static_cast<int>(threadIdx.x), nrows - 1)] / k;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int j = q >> 3;
    const int feat = (q & 7) * 16 + warp;  // feature within tile j
    const int NT = f / 128;
    const int KC = d / kKChunk;
    const int gpc = kKChunk / group;
    const uint8_t* base = wpack + (static_cast<size_t>(sblk[0]) * NT + j) * KC * bb;
    RowLoads<kGuVecs> Lg, Lu;
    row_load(Lg, base, bb, feat, 2 * 128 * 32, gpc, d / 32, lane);
    row_load(Lu, base, bb, 128 + feat, 2 * 128 * 32, gpc, d / 32, lane);
    const uint16_t* rows[kT];
    const float* sums[kT];
    float ag[kT], au[kT];
#pragma unroll
    for (int i = 0; i < kT; ++i) {
        rows[i] = xs + static_cast<size_t>(sblk[3 + i]) * d;
        sums[i] = xsum + sblk[3 + i] * (d / 32);
        ag[i] = 0.0f;
        au[i] = 0.0f;
    }
    row_dots<kT>(Lg, rows, sums, d / 32, lane, ag);
    row_dots<kT>(Lu, rows, sums, d / 32, lane, au);
#pragma unroll
    for (int i = 0; i < kT; ++i) {
        const float gv = warp_sum(ag[i]);
        const float uv = warp_sum(au[i]);
        if (lane == 0 && i < nrows)
            h[static_cast<size_t>(row0 + i) * f + j * 128 + feat] =
                bf16_round_bits(__fdividef(gv * uv, 1.0f + __expf(-gv)));
    }
}

// ---------------------------------------------------------------------------
// Down projection and combine for a batch of kT tokens.  Grid: d/16 CTAs;
// warp r of CTA m owns output feature 16m + r (row (16m + r) % (128 *
// kDownTiles) of down block (16m + r) / (128 * kDownTiles)).  For every block (expert) the warp dots that
// expert's row with the block's h rows, rounds each sum to bf16 (the expert
// output o), and after all blocks thread (t, r) sums o over token t's slots
// in slot order.  Dynamic shared memory: h [kT*k][f] bf16, then the fp32 sums
// of each h row's 32-wide vectors [kT*k][f/32].
// ---------------------------------------------------------------------------
template <int kT>
__global__ void __launch_bounds__(kRowThreads)
decode_down_kernel(const uint8_t* __restrict__ wpack, const uint16_t* __restrict__ h, int d, int k,
                   int f, int group, int bb, int nb_max, DecodeRouteOut ro,
                   uint16_t* __restrict__ y) {
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ int spos[kT * kMaxTopk];
    __shared__ float sw[kT * kMaxTopk];
    __shared__ int sbm[3 * kT * kMaxTopk];
    __shared__ float os[kT * kMaxTopk][16];
    __shared__ int snb;
    const int Tk = kT * k;
    const uint16_t* hs = reinterpret_cast<const uint16_t*>(dsm);
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    pdl_wait();  // h and the routing
    if (threadIdx.x == 0) snb = min(ro.num_blocks[0], nb_max);
    for (int i = threadIdx.x; i < Tk; i += blockDim.x) {
        spos[i] = ro.pos[i];
        sw[i] = ro.topk_w[i];
    }
    for (int i = threadIdx.x; i < 3 * nb_max; i += blockDim.x) sbm[i] = ro.block_map[i];
    cta_copy_rows_by_vector(dsm, h, Tk, f / 32);
    __syncthreads();
    float* hsum = reinterpret_cast<float*>(dsm + static_cast<size_t>(Tk) * f * 2);
    cta_vector_sums(hs, Tk, f / 32, hsum);
    __syncthreads();
    const int nb = snb;
    const int m = blockIdx.x * 16 + warp;
    const int jd = m / (128 * kDownTiles);
    const int prow = m % (128 * kDownTiles);
    const int NTd = d / (128 * kDownTiles);
    const int KCd = f / kKChunk;
    const int nv = f / 32;  // 16-byte nibble vectors per down row
    constexpr int kDnBlockBatch = dn_block_batch<kT>();
    for (int b0 = 0; b0 < nb; b0 += kDnBlockBatch) {
        RowLoads<kDnVecs> L[kDnBlockBatch];
#pragma unroll
        for (int u = 0; u < kDnBlockBatch; ++u)
            if (b0 + u < nb)
                row_load(L[u], wpack + (static_cast<size_t>(sbm[3 * (b0 + u)]) * NTd + jd) * KCd * bb,
                         bb, prow, 128 * kDownTiles * 32, kKChunk / group, nv, lane);
#pragma unroll
        for (int u = 0; u < kDnBlockBatch; ++u) {
            if (b0 + u < nb) {
                const int brow0 = sbm[3 * (b0 + u) + 1];
                const int brows = min(sbm[3 * (b0 + u) + 2], kT);
                const uint16_t* rows[kT];
                const float* sums[kT];
                float acc[kT];
#pragma unroll
                for (int i = 0; i < kT; ++i) {
                    const int p = brow0 + min(i, brows - 1);
                    rows[i] = hs + static_cast<size_t>(p) * f;
                    sums[i] = hsum + p * nv;
                    acc[i] = 0.0f;
                }
                row_dots<kT>(L[u], rows, sums, nv, lane, acc);
#pragma unroll
                for (int i = 0; i < kT; ++i) {
                    const float v = warp_sum(acc[i]);
                    if (lane == 0 && i < brows) os[brow0 + i][warp] = __bfloat162float(__float2bfloat16_rn(v));
                }
            }
        }
    }
    __syncthreads();
    if (threadIdx.x < 16 * kT) {
        const int t = threadIdx.x >> 4;
        const int r = threadIdx.x & 15;
        float acc = 0.0f;
        for (int jj = 0; jj < k; ++jj) acc = fmaf(sw[t * k + jj], os[spos[t * k + jj]][r], acc);
        y[static_cast<size_t>(t) * d + blockIdx.x * 16 + r] = bf16_round_bits(acc);
    }
}


constexpr size_t kDecodeSmemLimit = 112 * 1024;
constexpr size_t kRouteSmemLimit = 200 * 1024;

// gate/up: the batch's x rows; down: every assignment's h row and its vector sums
size_t gateup_smem_bytes(const moe_shape_t& s, int T) { return static_cast<size_t>(T) * s.d * 2; }
size_t down_smem_bytes(const moe_shape_t& s, int T) {
    return static_cast<size_t>(T) * s.k * (static_cast<size_t>(s.f) * 2 + (s.f / 32) * 4);
}

size_t route_smem_bytes(const moe_shape_t& s, int T) {
    return static_cast<size_t>(T) * s.d * 2 + static_cast<size_t>(s.d) * (s.E / kRouteCtas) * 4 +
           static_cast<size_t>(T) * 32 * 33 * 4;
}

template <int kT>
cudaError_t set_expert_kernel_smem() {
    cudaError_t e = cudaFuncSetAttribute(decode_gateup_kernel<kT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kDecodeSmemLimit));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(decode_down_kernel<kT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kDecodeSmemLimit));
}

template <int kT>
cudaError_t launch_experts(const DecodeArgs& a, const DecodeRouteOut& ro, cudaStream_t st,
                           void* ev_gate_up) {
    const moe_shape_t& s = a.s;
    const int nb_max = std::min(s.E, kT * s.k);
    cudaError_t e = launch_pdl(decode_gateup_kernel<kT>, dim3(nb_max * (s.f / 16)), kRowThreads,
                               gateup_smem_bytes(s, kT), st, a.x, a.wpack_gu, s.d, s.k,
                               s.f, s.group, a.gu_block_bytes, ro, a.h);
    if (e != cudaSuccess) return e;
    if (ev_gate_up && (e = cudaEventRecord(static_cast<cudaEvent_t>(ev_gate_up), st)) != cudaSuccess)
        return e;
    return launch_pdl(decode_down_kernel<kT>, dim3(s.d / 16), kRowThreads,
                      down_smem_bytes(s, kT), st, a.wpack_dn,
                      static_cast<const uint16_t*>(a.h), s.d, s.k, s.f, s.group, a.dn_block_bytes,
                      nb_max, ro, a.y);
}

}  // namespace

bool decode_supported(const moe_shape_t& s, int T) {
    if (T < 1 || T > kDecodeMaxT) return false;
    if (T * s.k > kDecodeMaxAssign || s.E > kMaxExperts) return false;
    // whole 16-byte vectors of W_r columns per routing CTA
    if (s.E % (4 * kRouteCtas) != 0 || route_smem_bytes(s, T) > kRouteSmemLimit) return false;
    // 16-byte nibble vectors (32 K values each) per lane and row
    if (s.d > 32 * 32 * kGuVecs || s.f > 32 * 32 * kDnVecs) return false;
    return gateup_smem_bytes(s, T) <= kDecodeSmemLimit && down_smem_bytes(s, T) <= kDecodeSmemLimit;
}

cudaError_t prepare_decode_kernels() {
    cudaError_t e = cudaFuncSetAttribute(decode_route_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kRouteSmemLimit));
    if (e != cudaSuccess) return e;
    static_assert(kDecodeMaxT == 8, "one instantiation per batch size");
    if ((e = set_expert_kernel_smem<1>()) != cudaSuccess) return e;
    if ((e = set_expert_kernel_smem<2>()) != cudaSuccess) return e;
    if ((e = set_expert_kernel_smem<3>()) != cudaSuccess) return e;
    if ((e = set_expert_kernel_smem<4>()) != cudaSuccess) return e;
    if ((e = set_expert_kernel_smem<5>()) != cudaSuccess) return e;
    if ((e = set_expert_kernel_smem<6>()) != cudaSuccess) return e;
    if ((e = set_expert_kernel_smem<7>()) != cudaSuccess) return e;
    return set_expert_kernel_smem<8>();
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st, void* ev_routed, void* ev_gate_up) {
    const moe_shape_t& s = a.s;
    const int T = a.T;
    const DecodeRouteOut ro{a.topk_idx, a.topk_w,        a.counts,    a.offsets,   a.sorted_assign,
                            a.pos,      a.block_offsets, a.block_map, a.num_blocks};
    const size_t route_smem = route_smem_bytes(s, T);
    cudaError_t e = launch_pdl(decode_route_kernel, dim3(kRouteCtas), dim3(kRowThreads), route_smem, st,
                               a.x, a.W_r, a.b_r, T, s.d, s.E, s.k, a.max_blocks, ro, a.status);
    if (e != cudaSuccess) return e;
    if (ev_routed && (e = cudaEventRecord(static_cast<cudaEvent_t>(ev_routed), st)) != cudaSuccess)
        return e;
    switch (T) {
        case 1: return launch_experts<1>(a, ro, st, ev_gate_up);
        case 2: return launch_experts<2>(a, ro, st, ev_gate_up);
        case 3: return launch_experts<3>(a, ro, st, ev_gate_up);
        case 4: return launch_experts<4>(a, ro, st, ev_gate_up);
        case 5: return launch_experts<5>(a, ro, st, ev_gate_up);
        case 6: return launch_experts<6>(a, ro, st, ev_gate_up);
        case 7: return launch_experts<7>(a, ro, st, ev_gate_up);
        case 8: return launch_experts<8>(a, ro, st, ev_gate_up);
    }
    return cudaErrorInvalidValue;
}

}  // namespace moe
