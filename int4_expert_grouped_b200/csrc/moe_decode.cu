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
//   decode_gateup_kernel   per (block, 8 features): the gate and up rows as
//                          one 16-row tile of the warp-level tensor-core MMA
//                          against the block's x rows (the MMA's 8 columns),
//                          int4 codes unpacked straight into its registers;
//                          each 32-wide vector's sum takes its group's scale
//                          and bias; SwiGLU gives bf16 rows of h
//   decode_down_kernel     per 16 output features: the same tile MMA for
//                          every selected expert against that expert's h
//                          rows, each output rounded to bf16, then the
//                          routing-weighted sum over a token's slots in order
//
// The MMA's 8 columns hold a block's rows (one per token), so the instruction
// count does not grow with the batch up to 8 tokens.  The weights are read in
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
constexpr int kRouteRowsPerLoad = 256;  // W_r rows per tensor load (the box height limit)
constexpr int kRowThreads = 512;    // threads of a routing CTA


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
    int cta_err[kRouteCtas];  // CTA r's copy of its W_r columns timed out (written every call)
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
// of the CTA's W_r columns that the tensor-memory-access unit brings in, 256
// rows per load (the load/store units reach a fraction of its rate for this
// strided copy).  The logits go to CTA 0's shared memory (distributed shared
// memory), which then routes.  Dynamic shared memory (128-byte aligned): the
// W_r columns [d][EC] fp32, x [T][d] bf16, the chains [T][32][33] fp32.
// ---------------------------------------------------------------------------
__global__ void __cluster_dims__(kRouteCtas, 1, 1) __launch_bounds__(kRowThreads)
decode_route_kernel(const __grid_constant__ CUtensorMap wmap, const uint16_t* __restrict__ x,
                    const float* __restrict__ bias, int T, int d, int E, int k, int max_blocks,
                    DecodeRouteOut ro, int32_t* __restrict__ status) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    __shared__ DecodeRoute R;
    __shared__ __align__(8) uint64_t wbar;
    __shared__ int no_abort;
    extern __shared__ __align__(16) uint8_t dsm_raw[];
    uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 127) &
                                              ~static_cast<uintptr_t>(127));
    const int EC = E / kRouteCtas;
    float* ws = reinterpret_cast<float*>(dsm);  // [i][EC]
    uint16_t* xs = reinterpret_cast<uint16_t*>(dsm + static_cast<size_t>(d) * EC * 4);
    float* cs = reinterpret_cast<float*>(dsm + static_cast<size_t>(d) * EC * 4 +
                                         static_cast<size_t>(T) * d * 2);  // [t][p][33]
    pdl_launch_dependents();
    const int rank = static_cast<int>(cluster.block_rank());
    const int e0 = rank * EC;
    const int nsteps = d >> 5;
    const int items = 32 * EC;
    const uint32_t bar = smem_u32(&wbar);
    if (threadIdx.x == 0) {
        // W_r[:, e0 .. e0+EC) -> ws in loads of 256 rows (e0 * 4 bytes is a
        // multiple of 16: EC % 4 == 0)
        no_abort = 0;
        mbar_init(bar, 1);
        fence_mbarrier_init();
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(d) * EC * 4);
        for (int r0 = 0; r0 < d; r0 += kRouteRowsPerLoad)
            tma_load_2d(smem_u32(ws + static_cast<size_t>(r0) * EC), &wmap, e0, r0, bar);
    }
    // x may be the output of the previous kernel in the stream (for example
    // y of the previous call), so it is read only after that kernel has
    // completed; W_r and the bias are never written by this library
    pdl_wait();
    cta_copy16(xs, x, T * d / 8);
    __syncthreads();  // x in place; the barrier initialised
    const bool w_ok = mbar_wait(bar, 0, &no_abort);
    if (threadIdx.x == 0) cluster.map_shared_rank(R.cta_err, 0)[rank] = w_ok ? 0 : 1;
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
    // the status word reports the most recent call: the first kernel clears it
    if (threadIdx.x < 2) status[threadIdx.x] = 0;
    __syncthreads();
    if (threadIdx.x < kRouteCtas && R.cta_err[threadIdx.x])
        report_error(status, MOE_ERR_DEVICE_TIMEOUT, 400 + threadIdx.x);
    route_from_logits(T, E, k, max_blocks, R);
    write_route(R, ro, T * k, E);
}

// ---------------------------------------------------------------------------
// Expert GEMVs on the warp-level tensor-core MMA (m16n8k16, bf16 operands from
// registers, fp32 accumulators).  A 16-row tile of packed weights is the A
// operand and up to 8 operand rows (a block's tokens) are the 8 columns of B,
// so the instruction count does not grow with the batch.
//
// Fragments (thread t of the warp: g = t / 4, c = t % 4): A holds rows g and
// g + 8, logical K pairs c and c + 4; B holds column g, the same K pairs; the
// accumulator holds rows g, g + 8 x columns 2c, 2c + 1.  Any one-to-one map of
// the 16 logical K onto the data's K gives the same sum, so thread c takes word
// c of a 32-wide nibble vector (K 8c .. 8c+7: nibble pair i is K 8c+2i at bits
// 4i and 8c+2i+1 at bits 16+4i) for both of its rows: pairs 0 and 1 feed the
// first MMA, pairs 2 and 3 the second, and its operand piece is the 16 bytes of
// K 8c .. 8c+7 of its column.  A nibble pair becomes two bf16 values 128 + q
// exactly (q in the mantissa of 128.0), so the MMA gives sum (128 + q) x; with
// w = q s + b a group's dot product is s * D + (b - 128 s) * sum x, formed in
// fp32 once per group (the MMAs of a 64-wide group accumulate together).  The
// weights are not rounded to bf16 on this path.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// nibble pair i of a packed word as bf16 (128 + q_lo, 128 + q_hi)
__device__ __forceinline__ uint32_t nib_pair(uint32_t w, int i) {
    return ((w >> (4 * i)) & 0x000F000Fu) | 0x43004300u;
}

// D += sum (128 + q) x over one 32-wide vector: wa, wb = word c of the vector
// in rows g and g + 8; xb = the column's operands K 8c .. 8c+7
__device__ __forceinline__ void vector_mma(float (&D)[4], uint32_t wa, uint32_t wb, const uint4& xb) {
    mma_16816(D, nib_pair(wa, 0), nib_pair(wb, 0), nib_pair(wa, 1), nib_pair(wb, 1), xb.x, xb.y);
    mma_16816(D, nib_pair(wa, 2), nib_pair(wb, 2), nib_pair(wa, 3), nib_pair(wb, 3), xb.z, xb.w);
}

// acc += s * D + (b - 128 s) * sum x for one group: sa, sb = the (scale,
// bias) words of rows g and g + 8; xs0, xs1 = the group's operand sums of
// columns 2c, 2c + 1
__device__ __forceinline__ void group_fold(float (&acc)[4], const float (&D)[4], uint32_t sa,
                                           uint32_t sb, float xs0, float xs1) {
    const float s0 = __uint_as_float(sa << 16);
    const float s1 = __uint_as_float(sb << 16);
    const float c0 = fmaf(-128.0f, s0, __uint_as_float(sa & 0xFFFF0000u));
    const float c1 = fmaf(-128.0f, s1, __uint_as_float(sb & 0xFFFF0000u));
    acc[0] = fmaf(s0, D[0], fmaf(c0, xs0, acc[0]));
    acc[1] = fmaf(s0, D[1], fmaf(c0, xs1, acc[1]));
    acc[2] = fmaf(s1, D[2], fmaf(c1, xs0, acc[2]));
    acc[3] = fmaf(s1, D[3], fmaf(c1, xs1, acc[3]));
}

// Loads of one 16-row tile over a range of 64-wide K chunks: the tile's rows
// g and g + 8 are packed rows pa and pb of blocks base + ch * bb; per chunk
// word c of both halves of both rows, and the rows' (scale, bias) words.
template <int kChunks, int kGpc>
struct TileLoads {
    uint32_t w[kChunks][4];         // row a half 0, row a half 1, row b half 0, row b half 1
    uint32_t sc[kChunks][2 * kGpc];  // row a groups, row b groups
};

template <int kChunks, int kGpc>
__device__ __forceinline__ void tile_load(TileLoads<kChunks, kGpc>& L, const uint8_t* base, int bb,
                                          int nib_bytes, int pa, int pb, int ch0, int ch_step,
                                          int KC, int c) {
#pragma unroll
    for (int u = 0; u < kChunks; ++u) {
        const int ch = ch0 + u * ch_step;
        if (ch < KC) {
            const uint8_t* blk = base + static_cast<size_t>(ch) * bb;
            L.w[u][0] = ld_nc_u32(blk + pa * 32 + 4 * c);
            L.w[u][1] = ld_nc_u32(blk + pa * 32 + 16 + 4 * c);
            L.w[u][2] = ld_nc_u32(blk + pb * 32 + 4 * c);
            L.w[u][3] = ld_nc_u32(blk + pb * 32 + 16 + 4 * c);
#pragma unroll
            for (int q = 0; q < kGpc; ++q) {
                L.sc[u][q] = ld_nc_u32(blk + nib_bytes + (pa * kGpc + q) * 4);
                L.sc[u][kGpc + q] = ld_nc_u32(blk + nib_bytes + (pb * kGpc + q) * 4);
            }
        }
    }
}

// acc += the tile's dot products over the loaded chunks.  xrow: the thread's
// column in shared memory, advanced to K 8c; xs0, xs1: vector sums of columns
// 2c and 2c + 1.
template <int kChunks, int kGpc>
__device__ __forceinline__ void tile_dots(float (&acc)[4], const TileLoads<kChunks, kGpc>& L,
                                          const uint16_t* xrow, const float* xs0, const float* xs1,
                                          int ch0, int ch_step, int KC) {
#pragma unroll
    for (int u = 0; u < kChunks; ++u) {
        const int ch = ch0 + u * ch_step;
        if (ch < KC) {
            const int v = 2 * ch;
            const uint4 xb0 = *reinterpret_cast<const uint4*>(xrow + 32 * v);
            const uint4 xb1 = *reinterpret_cast<const uint4*>(xrow + 32 * v + 32);
            float D[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            vector_mma(D, L.w[u][0], L.w[u][2], xb0);
            if (kGpc == 2) {  // a group per vector
                group_fold(acc, D, L.sc[u][0], L.sc[u][2], xs0[v], xs1[v]);
                D[0] = D[1] = D[2] = D[3] = 0.0f;
                vector_mma(D, L.w[u][1], L.w[u][3], xb1);
                group_fold(acc, D, L.sc[u][1], L.sc[u][3], xs0[v + 1], xs1[v + 1]);
            } else {  // one group for the chunk: its four MMAs share the fold
                vector_mma(D, L.w[u][1], L.w[u][3], xb1);
                group_fold(acc, D, L.sc[u][0], L.sc[u][1], xs0[v] + xs0[v + 1], xs1[v] + xs1[v + 1]);
            }
        }
    }
}

// Rows of bf16 operands (n_rows of w elements, row r at src row row_of(r))
// into shared memory with a row stride of w + 32 elements (64 bytes of pad,
// so the 8 columns' 16-byte reads fall in distinct banks), and each 32-wide
// vector's sum (fp32, in K order) into sums [r][w/32].
template <class RowOf>
__device__ __forceinline__ void cta_stage_rows(uint16_t* dst, float* sums, const uint16_t* src,
                                               int n_rows, int w, RowOf row_of) {
    const int nv = w / 32;
    for (int it = threadIdx.x; it < n_rows * nv; it += blockDim.x) {
        const int r = it / nv;
        const int v = it - r * nv;
        const uint8_t* s = reinterpret_cast<const uint8_t*>(src + static_cast<size_t>(row_of(r)) * w + 32 * v);
        uint4 p[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) p[q] = ld_nc_v4(s + 16 * q);
        uint4* d4 = reinterpret_cast<uint4*>(dst + static_cast<size_t>(r) * (w + 32) + 32 * v);
        float acc = 0.0f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            d4[q] = p[q];
            const uint32_t pw[4] = {p[q].x, p[q].y, p[q].z, p[q].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc += __uint_as_float(pw[i] << 16);
                acc += __uint_as_float(pw[i] & 0xFFFF0000u);
            }
        }
        sums[it] = acc;
    }
}

constexpr int kGuWarps = 4;   // K split of a gate/up CTA
constexpr int kGuChunks = 8;  // 64-wide K chunks per warp: d <= 4 * 8 * 64
constexpr int kGuFeat = 8;    // features per gate/up CTA: 8 gate + 8 up rows, one MMA tile
constexpr int kDnWarps = 16;  // blocks in flight per down CTA
template <int kGpc>
constexpr int dn_chunks() { return kGpc == 1 ? 8 : 6; }  // down K chunks loaded together

// ---------------------------------------------------------------------------
// Gate/up and SwiGLU.  Grid: min(E, T*k) blocks x f/8 feature groups (CTAs
// past the number of blocks return).  The MMA tile's rows g and g + 8 are the
// gate and up rows of feature 8q + g, so SwiGLU happens in the thread that
// holds both sums.  The four warps split K; their sums are added in warp
// order.  Columns beyond the block's rows repeat its last row and are not
// stored.  Dynamic shared memory: the block's x rows [T][d + 32] bf16, then
// their vector sums [T][d/32] fp32.
// ---------------------------------------------------------------------------
template <int kGpc>
__global__ void __launch_bounds__(kGuWarps * 32, kGpc == 1 ? 6 : 4)
decode_gateup_kernel(const uint16_t* __restrict__ x, const uint8_t* __restrict__ wpack, int T,
                     int d, int k, int f, int bb, DecodeRouteOut ro, uint16_t* __restrict__ h) {
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ float red[kGuWarps - 1][4][32];
    pdl_launch_dependents();
    pdl_wait();
    const int nfq = f / kGuFeat;
    const int b = blockIdx.x / nfq;
    const int fq = blockIdx.x - b * nfq;
    const int nb = ro.num_blocks[0];
    const int e = ro.block_map[3 * b];
    const int row0 = ro.block_map[3 * b + 1];
    const int cnt = ro.block_map[3 * b + 2];
    if (b >= min(nb, kDecodeMaxAssign)) return;
    const int nrows = min(cnt, T);  // a block holds at most one row per token
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int g = lane >> 2;
    const int c = lane & 3;
    const int KC = d / kKChunk;
    const int j = fq * kGuFeat / 128;
    const int pa = fq * kGuFeat % 128 + g;  // gate row; the up row is 128 further
    const uint8_t* base = wpack + (static_cast<size_t>(e) * (f / 128) + j) * KC * bb;
    TileLoads<kGuChunks, kGpc> L;
    tile_load(L, base, bb, 2 * 128 * 32, pa, 128 + pa, warp, kGuWarps, KC, c);
    uint16_t* xsh = reinterpret_cast<uint16_t*>(dsm);
    float* xss = reinterpret_cast<float*>(dsm + static_cast<size_t>(T) * (d + 32) * 2);
    const int32_t* sa = ro.sorted_assign + row0;
    cta_stage_rows(xsh, xss, x, nrows, d, [&](int r) { return sa[r] / k; });
    __syncthreads();
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const int nv = d / 32;
    tile_dots(acc, L, xsh + min(g, nrows - 1) * (d + 32) + 8 * c, xss + min(2 * c, nrows - 1) * nv,
              xss + min(2 * c + 1, nrows - 1) * nv, warp, kGuWarps, KC);
    if (warp > 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) red[warp - 1][i][lane] = acc[i];
    }
    __syncthreads();
    if (warp != 0) return;
#pragma unroll
    for (int w = 0; w < kGuWarps - 1; ++w)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] += red[w][i][lane];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int r = 2 * c + i;
        if (r < nrows) {
            const float gv = acc[i];
            const float uv = acc[2 + i];
            h[static_cast<size_t>(row0 + r) * f + fq * kGuFeat + g] =
                bf16_round_bits(__fdividef(gv * uv, 1.0f + __expf(-gv)));
        }
    }
}

// ---------------------------------------------------------------------------
// Down projection and combine.  Grid: d/16 CTAs; CTA m owns output features
// 16m .. 16m+15 (one MMA tile: rows 16m % 128 + g and + 8 of down tile
// 16m / 128).  The tile against a block's h rows gives each of the block's
// assignments its 16 outputs.  With at most 8 blocks a pair of warps takes a
// block, one K half each; otherwise warp w takes blocks w, w + 16, ... over
// all of K.  The two halves' sums (the second is zero for a whole-K warp) are
// added and rounded to bf16 (the expert output o), then thread (t, r) sums o
// over token t's slots in slot order.  Dynamic shared memory: h [T*k][f + 32]
// bf16, then its vector sums [T*k][f/32] fp32.
// ---------------------------------------------------------------------------
template <int kGpc>
__global__ void __launch_bounds__(kDnWarps * 32, 1)
decode_down_kernel(const uint8_t* __restrict__ wpack, const uint16_t* __restrict__ h, int T,
                   int d, int k, int f, int bb, int nb_max, DecodeRouteOut ro,
                   uint16_t* __restrict__ y) {
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ int spos[kDecodeMaxAssign];
    __shared__ float sw[kDecodeMaxAssign];
    __shared__ int sbm[3 * kDecodeMaxAssign];
    __shared__ float op[2][kDecodeMaxAssign][16];  // K-half sums of each assignment's outputs
    __shared__ int snb;
    const int Tk = T * k;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int g = lane >> 2;
    const int c = lane & 3;
    pdl_wait();  // h and the routing
    if (threadIdx.x == 0) snb = min(ro.num_blocks[0], nb_max);
    for (int i = threadIdx.x; i < Tk; i += blockDim.x) {
        spos[i] = ro.pos[i];
        sw[i] = ro.topk_w[i];
    }
    for (int i = threadIdx.x; i < 3 * nb_max; i += blockDim.x) sbm[i] = ro.block_map[i];
    uint16_t* hsh = reinterpret_cast<uint16_t*>(dsm);
    float* hss = reinterpret_cast<float*>(dsm + static_cast<size_t>(Tk) * (f + 32) * 2);
    cta_stage_rows(hsh, hss, h, Tk, f, [](int r) { return r; });
    __syncthreads();
    const int nb = snb;
    const int m0 = blockIdx.x * 16;
    const int jd = m0 / 128;
    const int pa = m0 % 128 + g;
    const int KC = f / kKChunk;
    const int nv = f / 32;
    constexpr int kCh = dn_chunks<kGpc>();
    const int split = nb <= kDnWarps / 2 ? 2 : 1;
    const int part = warp % split;
    const int kc_part = (KC + split - 1) / split;
    const int ch_begin = part * kc_part;
    const int ch_end = min(KC, ch_begin + kc_part);
    for (int b = warp / split; b < nb; b += kDnWarps / split) {
        const int brow0 = sbm[3 * b + 1];
        const int brows = min(sbm[3 * b + 2], T);
        const uint8_t* base = wpack + (static_cast<size_t>(sbm[3 * b]) * (d / 128) + jd) * KC * bb;
        const uint16_t* xrow = hsh + (brow0 + min(g, brows - 1)) * (f + 32) + 8 * c;
        const float* xs0 = hss + (brow0 + min(2 * c, brows - 1)) * nv;
        const float* xs1 = hss + (brow0 + min(2 * c + 1, brows - 1)) * nv;
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int ch0 = ch_begin; ch0 < ch_end; ch0 += kCh) {
            TileLoads<kCh, kGpc> L;
            tile_load(L, base, bb, 128 * 32, pa, pa + 8, ch0, 1, ch_end, c);
            tile_dots(acc, L, xrow, xs0, xs1, ch0, 1, ch_end);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int r = 2 * c + i;
            if (r < brows) {
                op[part][brow0 + r][g] = acc[i];
                op[part][brow0 + r][g + 8] = acc[2 + i];
            }
        }
    }
    if (split == 1) {  // whole-K sums: the second half is zero (no warp writes op[1])
        for (int i = threadIdx.x; i < Tk * 16; i += blockDim.x) op[1][i >> 4][i & 15] = 0.0f;
    }
    __syncthreads();
    if (threadIdx.x < 16 * T) {
        const int t = threadIdx.x >> 4;
        const int r = threadIdx.x & 15;
        float acc = 0.0f;
        for (int jj = 0; jj < k; ++jj) {
            const int pj = spos[t * k + jj];
            const float o = __bfloat162float(__float2bfloat16_rn(op[0][pj][r] + op[1][pj][r]));
            acc = fmaf(sw[t * k + jj], o, acc);
        }
        y[static_cast<size_t>(t) * d + m0 + r] = bf16_round_bits(acc);
    }
}

constexpr size_t kGuSmemLimit = 64 * 1024;
constexpr size_t kDnSmemLimit = 180 * 1024;
constexpr size_t kRouteSmemLimit = 200 * 1024;

size_t route_smem_bytes(const moe_shape_t& s, int T) {
    return 128 + static_cast<size_t>(T) * s.d * 2 + static_cast<size_t>(s.d) * (s.E / kRouteCtas) * 4 +
           static_cast<size_t>(T) * 32 * 33 * 4;  // + slack to align the base
}

// gate/up: the block's x rows (at most T) and their vector sums; down: every
// assignment's h row and its vector sums
size_t gateup_smem_bytes(const moe_shape_t& s, int T) {
    return static_cast<size_t>(T) * ((s.d + 32) * 2 + (s.d / 32) * 4);
}
size_t down_smem_bytes(const moe_shape_t& s, int T) {
    return static_cast<size_t>(T) * s.k * ((s.f + 32) * 2 + (s.f / 32) * 4);
}

template <int kGpc>
cudaError_t set_expert_kernel_smem() {
    cudaError_t e = cudaFuncSetAttribute(decode_gateup_kernel<kGpc>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kGuSmemLimit));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(decode_down_kernel<kGpc>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kDnSmemLimit));
}

template <int kGpc>
cudaError_t launch_experts(const DecodeArgs& a, const DecodeRouteOut& ro, cudaStream_t st,
                           void* ev_gate_up) {
    const moe_shape_t& s = a.s;
    const int nb_max = std::min(s.E, a.T * s.k);
    cudaError_t e = launch_pdl(decode_gateup_kernel<kGpc>, dim3(nb_max * (s.f / kGuFeat)),
                               dim3(kGuWarps * 32), gateup_smem_bytes(s, a.T), st, a.x, a.wpack_gu,
                               a.T, s.d, s.k, s.f, a.gu_block_bytes, ro, a.h);
    if (e != cudaSuccess) return e;
    if (ev_gate_up && (e = cudaEventRecord(static_cast<cudaEvent_t>(ev_gate_up), st)) != cudaSuccess)
        return e;
    return launch_pdl(decode_down_kernel<kGpc>, dim3(s.d / 16), dim3(kDnWarps * 32),
                      down_smem_bytes(s, a.T), st, a.wpack_dn, static_cast<const uint16_t*>(a.h),
                      a.T, s.d, s.k, s.f, a.dn_block_bytes, nb_max, ro, a.y);
}

}  // namespace

bool decode_supported(const moe_shape_t& s, int T) {
    if (T < 1 || T > kDecodeMaxT) return false;
    if (T * s.k > kDecodeMaxAssign || s.E > kMaxExperts) return false;
    // whole 16-byte vectors of W_r columns per routing CTA
    if (s.E % (4 * kRouteCtas) != 0 || route_smem_bytes(s, T) > kRouteSmemLimit) return false;
    // (groups of 32 or 64 and d, f in whole tiles hold for every plan) a
    // gate/up warp's K chunks fit in its registers
    if (s.d > kGuWarps * kGuChunks * kKChunk) return false;
    return gateup_smem_bytes(s, T) <= kGuSmemLimit && down_smem_bytes(s, T) <= kDnSmemLimit;
}

cudaError_t prepare_decode_kernels() {
    cudaError_t e = cudaFuncSetAttribute(decode_route_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kRouteSmemLimit));
    if (e != cudaSuccess) return e;
    if ((e = set_expert_kernel_smem<1>()) != cudaSuccess) return e;
    return set_expert_kernel_smem<2>();
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st, void* ev_routed, void* ev_gate_up) {
    const moe_shape_t& s = a.s;
    const int T = a.T;
    const DecodeRouteOut ro{a.topk_idx, a.topk_w,        a.counts,    a.offsets,   a.sorted_assign,
                            a.pos,      a.block_offsets, a.block_map, a.num_blocks};
    const size_t route_smem = route_smem_bytes(s, T);
    CUtensorMap wmap;
    cudaError_t e = encode_f32_cols_map(&wmap, a.W_r, s.d, s.E, s.E / kRouteCtas, kRouteRowsPerLoad);
    if (e != cudaSuccess) return e;
    e = launch_pdl(decode_route_kernel, dim3(kRouteCtas), dim3(kRowThreads), route_smem, st, wmap, a.x,
                   a.b_r, T, s.d, s.E, s.k, a.max_blocks, ro, a.status);
    if (e != cudaSuccess) return e;
    if (ev_routed && (e = cudaEventRecord(static_cast<cudaEvent_t>(ev_routed), st)) != cudaSuccess)
        return e;
    return s.group == 64 ? launch_experts<1>(a, ro, st, ev_gate_up)
                         : launch_experts<2>(a, ro, st, ev_gate_up);
}

}  // namespace moe
