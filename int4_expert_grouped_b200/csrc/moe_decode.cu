// Small-batch (decode) path of the MoE layer: the same operation as the
// batched path (inblix article "Perplexity's Lily engine beats MLX by 35% on
// M5 Max, no PyTorch needed", paragraph 3: routing, prefix scan, scatter,
// block map, dequantisation-fused expert GEMMs, weighted combine) for at most
// eight tokens, where the layer is bound by reading the selected experts'
// int4 weights from HBM (wpnews page "Perplexity Lily: 1.35x Faster Local AI
// Than MLX on Mac", section "Why MLX Falls Behind": prefill and decode are
// separate workloads).
//
// One persistent kernel, one CTA per SM, in four phases separated by flags in
// the workspace (no host round trip, no second launch):
//
//   1. router partials  CTA c owns routing item c (8 experts x one residue
//                       class r of the 32 fp32 chains): it brings its W_r
//                       piece in by one tensor load, runs the chains
//                       p = r, r+8, r+16, r+24 over all tokens and combines
//                       them by the first two levels of the router's
//                       butterfly; the partial u_r goes to the workspace
//   2. routing          every CTA, once all items are in: the last three
//                       butterfly levels and the bias give the logits; top-k,
//                       weights, counts, offsets, block map and scatter are
//                       computed in every CTA identically (CTA 0 writes them)
//   3. experts          the units (one expert's 64-feature slice: its 64 gate
//                       and 64 up rows over all of K, then the 64 matching
//                       columns of W_down for every output tile) are dealt
//                       round robin to the CTAs.  A producer warp streams
//                       each unit's weights into a shared-memory ring with
//                       bulk copies, as far ahead as the ring allows, so every
//                       SM keeps its share of the weights in flight; eight
//                       warps multiply them on the warp-level tensor-core MMA,
//                       each warp a share of the K chunks (gate/up) or of the
//                       output tiles (down) with all of the slice's rows, so
//                       its eight row tiles are independent chains.
//                       SwiGLU of the slice stays in shared memory (no h round
//                       trip); the slice's down partial sums go to the
//                       workspace
//   4. combine          after a grid-wide count of finished CTAs, every CTA
//                       adds, for its share of the outputs, each expert's
//                       slice partials in slice order, rounds the expert output
//                       to bf16 and sums a token's slots in slot order into y;
//                       the last CTA to leave resets the flags for the next
//                       call
//
// MMA form (m16n8k16, bf16 operands from registers, fp32 accumulators): a
// 16-row tile of packed weights is A, the rows of one expert's block (at most
// eight tokens) are the eight columns of B.  A nibble pair becomes two bf16
// values 128 + q exactly, so the MMA gives sum (128 + q) x; with
// w = q s + b a group's dot product is s * D + (b - 128 s) * sum x, formed in
// fp32 once per group.  The weights are not rounded to bf16 on this path
// (closer to the unrounded q s + b than the batched path's rounding); h and
// each expert output are rounded to bf16 and a token's slots are summed in
// slot order, as in the batched path.
//
// Every wait is bounded (%globaltimer): a CTA that gives up records
// MOE_ERR_DEVICE_TIMEOUT, raises an abort flag the others poll, and still
// takes part in the exit count.
#include <algorithm>

#include "moe_route_common.cuh"

namespace moe {
namespace {

constexpr int kDecComputeWarps = 16;
constexpr int kDecThreads = (kDecComputeWarps + 1) * 32;  // + one producer warp
constexpr int kDecProducerWarp = kDecComputeWarps;
constexpr int kDecComputeThreads = kDecComputeWarps * 32;
constexpr int kDecStages = 8;
// One stage = four 64-wide K chunks of a slice's 64 gate and 64 up rows (four
// consecutive half-blocks), or up to four down blocks (128 rows x 64 K each;
// a slice's blocks are consecutive over the output tiles): one bulk copy of
// at most 4 * half_block_bytes(group) bytes.  Copies of 16 KB and more keep
// the per-SM copy rate near its maximum; 4.6 KB copies ran at half of it.
constexpr int kDecChunks = 4;
constexpr int kDecStageBytes = kDecChunks * half_block_bytes(32);
constexpr int kDecMaxAssign = 64;                          // T * k the path takes
constexpr int kDecSlice = 64;                              // features per unit
constexpr int kDecMaxSlices = 32;                          // f / 64
constexpr int kDecMaxNTd = 64;                             // d / 128
constexpr int kDecHStride = kDecSlice + 32;                // h row stride (elements) in shared memory
constexpr int kDecRowTiles = kDecSlice / 8;                // 16-row MMA tiles of a slice: 8 gate + 8 up rows each
constexpr int kDecKHalves = kDecComputeWarps / kDecRowTiles;  // compute warps per MMA row tile
static_assert(kDecKHalves == 2 && kDecChunks % kDecKHalves == 0,
              "compute warps w and w + 8 own MMA row tile w % 8, each half of every stage");
constexpr int kDecWRows = 256;                             // W_r rows per tensor load (box limit)
constexpr uint32_t kDecMagic0 = 0x4D6F4544u, kDecMagic1 = 0x53796E63u;

// Flags in the workspace's decode region (int32 offsets).
constexpr int kSyncMagic = 0;     // two words: the region has been initialised
constexpr int kSyncRoute = 2;     // routing items published
constexpr int kSyncExit = 3;      // CTAs that have finished
constexpr int kSyncAbort = 4;     // a CTA gave up waiting
constexpr int kSyncUnits = 5;     // CTAs done with their units
constexpr int kSyncInts = 8;
static_assert(kSyncInts * 4 <= kDecodeSyncBytes, "decode flags fit their workspace region");

__device__ __forceinline__ uint4 ld_cg_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ float ld_cg_f32(const float* p) {
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_release_add(int* p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int atom_acq_rel_add(int* p, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ void st_release(int* p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// barrier of the eight compute warps (the producer warp does not take part)
__device__ __forceinline__ void compute_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kDecComputeThreads) : "memory");
}

// 3-D tensor load (TMA): coordinates c0 (innermost), c1, c2.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, int c0, int c1, int c2,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ uint16_t bf16_round_bits(float v) {
    const __nv_bfloat16 b = __float2bfloat16_rn(v);
    return *reinterpret_cast<const uint16_t*>(&b);
}
__device__ __forceinline__ float bf16_round(float v) {
    return __bfloat162float(__float2bfloat16_rn(v));
}

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// nibble pair i of a packed word as bf16 (128 + q_lo, 128 + q_hi)
__device__ __forceinline__ uint32_t nib_pair(uint32_t w, int i) { return nibble_pair_bf16(w, i); }

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
    // the scales (low halves) by an integer multiply, which may issue on the
    // FMA pipe; the logic pipe is the busier one in these calls
    const float s0 = __uint_as_float(sa * 65536u);
    const float s1 = __uint_as_float(sb * 65536u);
    const float c0 = fmaf(-128.0f, s0, __uint_as_float(sa & 0xFFFF0000u));
    const float c1 = fmaf(-128.0f, s1, __uint_as_float(sb & 0xFFFF0000u));
    acc[0] = fmaf(s0, D[0], fmaf(c0, xs0, acc[0]));
    acc[1] = fmaf(s0, D[1], fmaf(c0, xs1, acc[1]));
    acc[2] = fmaf(s1, D[2], fmaf(c1, xs0, acc[2]));
    acc[3] = fmaf(s1, D[3], fmaf(c1, xs1, acc[3]));
}

__device__ __forceinline__ uint32_t lds_u32(const uint8_t* p) {
    return *reinterpret_cast<const uint32_t*>(p);
}

// One 64-wide K chunk of a 16-row tile held in shared memory: blk = the
// packed block (rows x 32 bytes of nibbles, then per row and group a (scale,
// bias) word), rows ra and ra + 8; xrow = the thread's B column at K 8c of
// this chunk; xs0, xs1 = the 32-wide vector sums of columns 2c, 2c + 1 at
// this chunk's first vector.
template <int kGpc>
__device__ __forceinline__ void chunk_mma(float (&acc)[4], const uint8_t* blk, int nib_bytes, int ra,
                                          int c, const uint16_t* xrow, const float* xs0,
                                          const float* xs1) {
    const int rb = ra + 8;
    const uint32_t wa0 = lds_u32(blk + ra * 32 + 4 * c);
    const uint32_t wa1 = lds_u32(blk + ra * 32 + 16 + 4 * c);
    const uint32_t wb0 = lds_u32(blk + rb * 32 + 4 * c);
    const uint32_t wb1 = lds_u32(blk + rb * 32 + 16 + 4 * c);
    const uint4 xb0 = *reinterpret_cast<const uint4*>(xrow);
    const uint4 xb1 = *reinterpret_cast<const uint4*>(xrow + 32);
    float D[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    vector_mma(D, wa0, wb0, xb0);
    if constexpr (kGpc == 2) {  // a group per 32-wide vector
        group_fold(acc, D, lds_u32(blk + nib_bytes + (ra * 2) * 4), lds_u32(blk + nib_bytes + (rb * 2) * 4),
                   xs0[0], xs1[0]);
        D[0] = D[1] = D[2] = D[3] = 0.0f;
        vector_mma(D, wa1, wb1, xb1);
        group_fold(acc, D, lds_u32(blk + nib_bytes + (ra * 2 + 1) * 4),
                   lds_u32(blk + nib_bytes + (rb * 2 + 1) * 4), xs0[1], xs1[1]);
    } else {  // one group for the chunk: its four MMAs share the fold
        vector_mma(D, wa1, wb1, xb1);
        group_fold(acc, D, lds_u32(blk + nib_bytes + ra * 4), lds_u32(blk + nib_bytes + rb * 4),
                   xs0[0] + xs0[1], xs1[0] + xs1[1]);
    }
}

// The same for rows held apart (the gate and the up rows of a slice): na, nb
// = the two rows' 32 bytes of nibbles, sa, sb = their (scale, bias) words.
template <int kGpc>
__device__ __forceinline__ void chunk_mma_rows(float (&acc)[4], const uint8_t* na, const uint8_t* nb,
                                               const uint8_t* sa, const uint8_t* sb, int c,
                                               const uint16_t* xrow, const float* xs0, const float* xs1) {
    const uint32_t wa0 = lds_u32(na + 4 * c);
    const uint32_t wa1 = lds_u32(na + 16 + 4 * c);
    const uint32_t wb0 = lds_u32(nb + 4 * c);
    const uint32_t wb1 = lds_u32(nb + 16 + 4 * c);
    const uint4 xb0 = *reinterpret_cast<const uint4*>(xrow);
    const uint4 xb1 = *reinterpret_cast<const uint4*>(xrow + 32);
    float D[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    vector_mma(D, wa0, wb0, xb0);
    if constexpr (kGpc == 2) {
        group_fold(acc, D, lds_u32(sa), lds_u32(sb), xs0[0], xs1[0]);
        D[0] = D[1] = D[2] = D[3] = 0.0f;
        vector_mma(D, wa1, wb1, xb1);
        group_fold(acc, D, lds_u32(sa + 4), lds_u32(sb + 4), xs0[1], xs1[1]);
    } else {
        vector_mma(D, wa1, wb1, xb1);
        group_fold(acc, D, lds_u32(sa), lds_u32(sb), xs0[0] + xs0[1], xs1[0] + xs1[1]);
    }
}

// Rows of bf16 operands into shared memory with a row stride of w + 32
// elements (the eight columns' 16-byte reads then fall in distinct banks),
// and each 32-wide vector's fp32 sum in K order into sums[r][w / 32].
// Reads through L2 (the rows may have been written by other CTAs).
template <class RowOf>
__device__ __forceinline__ void stage_rows(uint16_t* dst, float* sums, const uint16_t* src, int n_rows,
                                           int w, RowOf row_of, int tid, int nthreads) {
    const int nv = w / 32;
    for (int it = tid; it < n_rows * nv; it += nthreads) {
        const int r = it / nv;
        const int v = it - r * nv;
        const uint8_t* s = reinterpret_cast<const uint8_t*>(src + static_cast<size_t>(row_of(r)) * w + 32 * v);
        uint4 p[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) p[q] = ld_cg_v4(s + 16 * q);
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

// Routing of the few tokens, in shared memory (identical in every CTA).
struct DecRoute {
    float sel[kDecMaxAssign];  // logit of each selected slot
    int idx[kDecMaxAssign];
    float w[kDecMaxAssign];
    int sa[kDecMaxAssign];
    int pos[kDecMaxAssign];
    int cnt[kMaxExperts];
    int off[kMaxExperts + 1];
    int bo[kMaxExperts + 1];
    int blk_e[kDecMaxAssign];  // block b: expert, first row, rows (one block per selected expert)
    int blk_row0[kDecMaxAssign];
    int blk_n[kDecMaxAssign];
    int nb;
    int sh_warp[kDecThreads / 32 + 1];
    int flag;                  // broadcast of a thread-0 decision to the compute warps
    int hok;                   // the h rows of a block became ready
    int fail;                  // a compute warp gave up on the current unit
    int abort_local;           // this CTA gave up
};

// top-k (each (token, expert) pair finds its slot by counting the experts
// ahead of it, P threads per pair over E / P experts each; ties go to the
// lower id; measured faster here than a warp top-k per token), counts
// (integer atomics, taken with the slots), the softmax weights over the k
// slots, offsets and the block map (one exclusive scan of counts | blocks
// << 16: counts sum to at most 64, blocks to at most E), one block per expert
// with rows (ascending expert), and the stable scatter (rank of assignment a
// = number of earlier assignments to its expert).  All kDecThreads threads;
// R.cnt is zero on entry.
__device__ void route_small(const float* lg, int T, int E, int k, DecRoute& R) {
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int Tk = T * k;
    int P = 1;
    while (P < 8 && 2 * P * T * E <= kDecThreads && (E / (2 * P)) % 4 == 0) P *= 2;
    const int per = E / P;
    const int n_it = T * E * P;
    for (int base = warp * 32; base < n_it; base += kDecThreads) {  // warp-uniform: the shuffles below
        const int it = base + lane;
        const bool valid = it < n_it;  // whole groups of P lanes: n_it is a multiple of P
        const int pair = it / P;
        const int part = it - pair * P;
        const int t = valid ? pair / E : 0;
        const int e = valid ? pair - t * E : 0;
        const float* row = lg + t * E;
        const float v = row[e];
        int r = 0;
        if (valid) {
            const float4* r4 = reinterpret_cast<const float4*>(row + part * per);
            for (int j = 0; j < per / 4; ++j) {
                const float4 u = r4[j];
                const int e2 = part * per + 4 * j;
                r += (u.x > v) | ((u.x == v) & (e2 < e));
                r += (u.y > v) | ((u.y == v) & (e2 + 1 < e));
                r += (u.z > v) | ((u.z == v) & (e2 + 2 < e));
                r += (u.w > v) | ((u.w == v) & (e2 + 3 < e));
            }
        }
        for (int m = 1; m < P; m <<= 1) r += __shfl_xor_sync(0xffffffffu, r, m);
        if (valid && part == 0 && r < k) {
            R.idx[t * k + r] = e;
            R.sel[t * k + r] = v;
            atomicAdd(&R.cnt[e], 1);
        }
    }
    __syncthreads();
    for (int t = warp; t < T; t += kDecThreads / 32) {
        const float wt = warp_slot_weights(lane < k ? R.sel[t * k + lane] : 0.0f, k, lane);
        if (lane < k) R.w[t * k + lane] = wt;
    }
    const int c = tid < E ? R.cnt[tid] : 0;
    const int nt = c > 0 ? 1 : 0;  // at most T <= 8 rows per expert: one block each
    int total = 0;
    const int packed = block_exclusive_scan<kDecThreads>(c | (nt << 16), R.sh_warp, &total);
    const int off = packed & 0xFFFF, bo = packed >> 16;
    const int nb = total >> 16;
    if (tid < E) {
        R.off[tid] = off;
        R.bo[tid] = bo;
        if (nt) {
            R.blk_e[bo] = tid;
            R.blk_row0[bo] = off;
            R.blk_n[bo] = c;
        }
    }
    if (tid == 0) {
        R.off[E] = total & 0xFFFF;
        R.bo[E] = nb;
        R.nb = nb;
    }
    __syncthreads();
    for (int a = tid; a < Tk; a += kDecThreads) {
        const int e = R.idx[a];
        int rank = 0;
        for (int a2 = 0; a2 < a; ++a2) rank += R.idx[a2] == e;
        const int p = R.off[e] + rank;
        R.sa[p] = a;
        R.pos[a] = p;
    }
    __syncthreads();
}

// Layout of the dynamic shared memory (byte offsets; the base is 1024-aligned).
struct DecSmem {
    int ring, x, xsum, h, hsum, lg, red, route, bars, total;
};
__host__ __device__ inline DecSmem dec_smem_layout(int T, int d, int E, int f) {
    DecSmem L;
    int o = 0;
    auto take = [&](int bytes) {
        const int r = o;
        o = (o + bytes + 127) / 128 * 128;
        return r;
    };
    L.ring = take(kDecStages * kDecStageBytes);
    L.x = take(T * (d + 32) * 2);
    L.xsum = take(T * (d / 32) * 4);
    L.h = take(kDecodeMaxT * kDecHStride * 2);
    L.hsum = take(kDecodeMaxT * (kDecSlice / 32) * 4);
    L.lg = take(T * E * 4);
    L.red = take(kDecRowTiles * 4 * 32 * 4);  // second-half gate/up sums
    L.route = take(static_cast<int>(sizeof(DecRoute)));
    L.bars = take((2 * kDecStages + 1) * 8);
    L.total = o + 1024;  // + slack to align the base
    return L;
}

struct DecParams {
    int T, d, E, k, f;
    const uint16_t* x;
    const float* b_r;
    const uint8_t* wgu;   // packed gate/up blocks [E][f/128][d/64][bb_gu]
    const uint8_t* wdn;   // packed down blocks [E][f/64][d/128][bb_dn]
    int bb_gu, bb_dn;
    int32_t *topk_idx, *counts, *offsets, *sorted_assign, *pos, *block_offsets, *block_map,
        *num_blocks;
    float* topk_w;
    float* U;             // router partials [T][E][8]
    float* pdn;           // down partial sums [T*k][f/64][d]: one per (row, slice)
    uint16_t* y;          // [T][d]
    int32_t* status;
    int32_t* sync;        // the decode flags
};

// Wait until *flag >= target (thread-level, bounded; also gives up when the
// call's abort flag is raised).  Returns false on giving up.
__device__ __forceinline__ bool wait_flag(const int* flag, int target, const int* abort) {
    if (ld_acquire(flag) >= target) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t n = 1;; ++n) {
        if (ld_acquire(flag) >= target) return true;
        if ((n & 15u) == 0) {
            if (ld_acquire(abort) != 0) return false;
            if (globaltimer() - t0 > kWaitTimeoutNs) return false;
        }
        __nanosleep(32);
    }
}

// Wait until the flags region carries both magic words (CTA 0 writes them
// after zeroing the region, the second one last, with release order).
__device__ __forceinline__ bool wait_magic(const int* sync, const int* abort) {
    const uint64_t t0 = globaltimer();
    for (uint32_t n = 0;; ++n) {
        if (static_cast<uint32_t>(ld_acquire(sync + kSyncMagic + 1)) == kDecMagic1 &&
            static_cast<uint32_t>(ld_acquire(sync + kSyncMagic)) == kDecMagic0)
            return true;
        if ((n & 15u) == 15u) {
            if (ld_acquire(abort) != 0) return false;
            if (globaltimer() - t0 > kWaitTimeoutNs) return false;
        }
        __nanosleep(32);
    }
}

__device__ __forceinline__ int vload(const int& v) { return *reinterpret_cast<const volatile int*>(&v); }

// the thread that gives up: record the error and stop every CTA of the call
__device__ __forceinline__ void dec_fail(const DecParams& p, DecRoute& R, int detail) {
    report_error(p.status, MOE_ERR_DEVICE_TIMEOUT, detail);
    st_release(p.sync + kSyncAbort, 1);
    R.abort_local = 1;
}

template <int kGpc>
__global__ void __launch_bounds__(kDecThreads, 1)
decode_layer_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ DecParams p) {
    extern __shared__ uint8_t dsm_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    pdl_launch_dependents();
    const int T = p.T, d = p.d, E = p.E, k = p.k, f = p.f;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int G = gridDim.x;
    const int cta = blockIdx.x;
    const DecSmem L = dec_smem_layout(T, d, E, f);
    uint8_t* ring = smem + L.ring;
    uint16_t* xsh = reinterpret_cast<uint16_t*>(smem + L.x);
    float* xsum = reinterpret_cast<float*>(smem + L.xsum);
    uint16_t* hsh = reinterpret_cast<uint16_t*>(smem + L.h);
    float* hsum = reinterpret_cast<float*>(smem + L.hsum);
    float* lg = reinterpret_cast<float*>(smem + L.lg);
    DecRoute& R = *reinterpret_cast<DecRoute*>(smem + L.route);
    const uint32_t bar0 = smem_u32(smem + L.bars);
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (kDecStages + s); };
    const uint32_t wbar = bar0 + 8u * (2 * kDecStages);
    int32_t* sync = p.sync;
    const int* abort_g = sync + kSyncAbort;

    // routing items of this CTA: item i = (octet i >> 3, residue i & 7)
    const int my_items = cta < E ? (E - 1 - cta) / G + 1 : 0;
    const int item_bytes = (d / 8) * 32;
    if (tid == 0) {
        for (int s = 0; s < kDecStages; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), kDecComputeWarps);  // every compute warp uses every stage
        }
        mbar_init(wbar, 1);
        R.abort_local = 0;
        fence_mbarrier_init();
        // W_r pieces (model weights, never written by this library: loaded
        // before waiting for the previous kernel): rows i = 8j + r, j < d/8,
        // of the item's 8 experts, [j][8] fp32
        if (my_items > 0) {
            mbar_arrive_expect_tx(wbar, static_cast<uint32_t>(my_items * item_bytes));
            for (int ii = 0; ii < my_items; ++ii) {
                const int item = cta + ii * G;
                for (int j0 = 0; j0 < d / 8; j0 += kDecWRows)
                    tma_load_3d(smem_u32(ring + ii * item_bytes + j0 * 32), &wmap, 8 * (item >> 3), item & 7,
                                j0, wbar);
            }
        }
    }
    // x may be the output of the previous kernel in the stream (for example
    // y of the previous call): read it, and the workspace, only after that
    // kernel has completed
    pdl_wait();
    stage_rows(xsh, xsum, p.x, T, d, [](int r) { return r; }, tid, kDecThreads);
    if (cta == 0 && tid == 0) {
        // the status word reports the most recent call; the flags region is
        // zeroed on first use (and reset by the last CTA of every call)
        p.status[0] = 0;
        p.status[1] = 0;
        R.flag = !(static_cast<uint32_t>(sync[kSyncMagic]) == kDecMagic0 &&
                   static_cast<uint32_t>(sync[kSyncMagic + 1]) == kDecMagic1);
    }
    __syncthreads();
    if (cta == 0 && vload(R.flag)) {
        for (int i = tid + 2; i < kSyncInts; i += kDecThreads) sync[i] = 0;
        __threadfence();
        __syncthreads();
        if (tid == 0) {
            sync[kSyncMagic] = static_cast<int>(kDecMagic0);
            __threadfence();
            st_release(sync + kSyncMagic + 1, static_cast<int>(kDecMagic1));
        }
    }

    // ---- phase 1: router partials ----------------------------------------
    // chain p = r + 8q (q < 4) of expert 8o + el and token t runs
    // i = p, p + 32, ... with fused multiply-add from 0; lanes 4m .. 4m + 3
    // hold q = 0..3 of one (t, el), and u_r = (c_r + c_{r+16}) + (c_{r+8} + c_{r+24})
    // is the value the router's butterfly holds at chain r after its levels
    // 16 and 8
    if (my_items > 0) {
        // every thread waits; the outcome is made uniform before any shuffle
        const bool w_ok = __syncthreads_and(mbar_wait(wbar, 0, &R.abort_local)) != 0;
        if (!w_ok && tid == 0) dec_fail(p, R, 500);
        if (w_ok) {
            for (int ii = 0; ii < my_items; ++ii) {
                const int item = cta + ii * G;
                const int o = item >> 3;
                const int r = item & 7;
                const float* wsl = reinterpret_cast<const float*>(ring + ii * item_bytes);
                for (int ch = tid; ch < T * 32; ch += kDecThreads) {  // T * 32 <= 256: one pass
                    const int q = ch & 3;
                    const int el = (ch >> 2) & 7;
                    const int t = ch >> 5;
                    const uint16_t* xr = xsh + t * (d + 32) + r + 8 * q;
                    const float* wr = wsl + q * 8 + el;
                    float acc = 0.0f;
#pragma unroll 8
                    for (int m = 0; m < d / 32; ++m)
                        acc = __fmaf_rn(bf16_bits_to_float(xr[32 * m]), wr[32 * m], acc);
                    const float s02 = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, 2));
                    const float u = __fadd_rn(s02, __shfl_xor_sync(0xffffffffu, s02, 1));
                    if (q == 0) p.U[(static_cast<size_t>(t) * E + 8 * o + el) * 8 + r] = u;
                }
            }
        }
        __threadfence();
    }
    __syncthreads();
    if (tid == 0) {
        bool ok = !vload(R.abort_local);
        if (ok && !wait_magic(sync, abort_g)) {
            dec_fail(p, R, 501);
            ok = false;
        }
        if (my_items > 0) red_release_add(sync + kSyncRoute, my_items);  // counted even on failure
        if (ok && !wait_flag(sync + kSyncRoute, E, abort_g)) dec_fail(p, R, 502);
    }
    __syncthreads();

    // ---- phase 2: routing (every CTA) ---------------------------------------
    if (!vload(R.abort_local)) {
        for (int it = tid; it < T * E; it += kDecThreads) {
            const uint4 ua = ld_cg_v4(p.U + static_cast<size_t>(it) * 8);
            const uint4 ub = ld_cg_v4(p.U + static_cast<size_t>(it) * 8 + 4);
            const float4 a = make_float4(__uint_as_float(ua.x), __uint_as_float(ua.y),
                                         __uint_as_float(ua.z), __uint_as_float(ua.w));
            const float4 b = make_float4(__uint_as_float(ub.x), __uint_as_float(ub.y),
                                         __uint_as_float(ub.z), __uint_as_float(ub.w));
            // levels 4, 2, 1 of the butterfly: ((u0+u4) + (u2+u6)) + ((u1+u5) + (u3+u7))
            const float S = __fadd_rn(__fadd_rn(__fadd_rn(a.x, b.x), __fadd_rn(a.z, b.z)),
                                      __fadd_rn(__fadd_rn(a.y, b.y), __fadd_rn(a.w, b.w)));
            lg[it] = p.b_r != nullptr ? __fadd_rn(S, __ldg(p.b_r + (it % E))) : S;
        }
    }
    if (tid < E) R.cnt[tid] = 0;
    __syncthreads();
    const bool routed = !vload(R.abort_local);
    if (routed) route_small(lg, T, E, k, R);
    const int nb = routed ? R.nb : 0;
    const int Tk = T * k;
    if (cta == 0 && routed) {
        for (int a = tid; a < Tk; a += kDecThreads) {
            p.topk_idx[a] = R.idx[a];
            p.topk_w[a] = R.w[a];
            p.sorted_assign[a] = R.sa[a];
            p.pos[a] = R.pos[a];
        }
        for (int e = tid; e <= E; e += kDecThreads) {
            if (e < E) p.counts[e] = R.cnt[e];
            p.offsets[e] = R.off[e];
            p.block_offsets[e] = R.bo[e];
        }
        for (int b = tid; b < nb; b += kDecThreads) {
            p.block_map[3 * b + 0] = R.blk_e[b];
            p.block_map[3 * b + 1] = R.blk_row0[b];
            p.block_map[3 * b + 2] = R.blk_n[b];
        }
        if (tid == 0) p.num_blocks[0] = nb;
    }

    // ---- phase 3: expert units ------------------------------------------------
    // unit u = (block u / S, slice u % S); S = f / 64 slices per expert
    const int NT = f / 128, KC = d / kKChunk, NTd = d / 128, KCd = f / kKChunk;
    const int S = f / kDecSlice;
    const int u_total = nb * S;
    const int NSd = (NTd + kDecChunks - 1) / kDecChunks;  // down stages per unit

    if (warp == kDecProducerWarp) {
        // the whole warp runs the loop; one elected lane issues the copies
        uint32_t q = 0;
        bool ok = true;
        for (int u = cta; ok && u < u_total; u += G) {
            const int b = u / S;
            const int fs = u - b * S;
            const int e = R.blk_e[b];
            const int j = fs >> 1, hh = fs & 1;  // 128-feature tile, half of it
            const uint8_t* gsrc = p.wgu + ((static_cast<size_t>(e) * NT + j) * 2 + hh) * KC * p.bb_dn;
            const uint8_t* dsrc = p.wdn + (static_cast<size_t>(e) * KCd + fs) * NTd * p.bb_dn;
            for (int st = 0; st < KC / kDecChunks + NSd; ++st, ++q) {
                const int slot = q % kDecStages;
                if (!__all_sync(0xffffffffu, mbar_wait(empty(slot), ((q / kDecStages) & 1) ^ 1, &R.abort_local))) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    const uint32_t dst = smem_u32(ring + slot * kDecStageBytes);
                    // gate/up: K chunks 4 st .. 4 st + 3 of the slice; down:
                    // output tiles 4 sd .. of K chunk fs; consecutive blocks
                    const bool gu = st < KC / kDecChunks;
                    const int first = gu ? kDecChunks * st : kDecChunks * (st - KC / kDecChunks);
                    const int nblk = gu ? kDecChunks : min(kDecChunks, NTd - first);
                    const uint32_t bytes = static_cast<uint32_t>(nblk * p.bb_dn);
                    mbar_arrive_expect_tx(full(slot), bytes);
                    bulk_copy_g2s(dst, (gu ? gsrc : dsrc) + static_cast<size_t>(first) * p.bb_dn, bytes,
                                  full(slot));
                }
                __syncwarp();
            }
        }
        if (!ok && lane == 0) {
            if (!vload(R.abort_local)) dec_fail(p, R, 503);
            // let the copies already issued land before the CTA exits
            const uint32_t first = q > kDecStages ? q - kDecStages : 0;
            for (uint32_t i = first; i < q; ++i) {
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(full(i % kDecStages), (i / kDecStages) & 1))
                    if (globaltimer() - t0 > 200000000ull) break;
            }
        }
    } else {
        // compute warps: MMA fragment coordinates.  Every compute warp takes
        // every stage of the ring; warps w and w + 8 own MMA row tile r = w % 8:
        // gate rows of features 8r .. 8r + 7 as rows g and their up rows as
        // g + 8 (gate/up stages), rows 16r .. 16r + 15 of each 128-row output
        // tile (down stages); warp w < 8 takes the first half of each stage's
        // K chunks or output tiles, warp w + 8 the second.  A warp waits on a
        // stage's phase only after it has used the slot's previous phase, so
        // no wait runs two phases ahead.
        const int g = lane >> 2;
        const int c = lane & 3;
        const int rt = warp % kDecRowTiles;   // MMA row tile
        const int kh = warp / kDecRowTiles;   // which half of each stage's chunks / tiles
        const int fr = 8 * rt + g;
        float* red = reinterpret_cast<float*>(smem + L.red);
        constexpr int kHalf = kDecChunks / kDecKHalves;  // chunks or tiles per warp and stage
        uint32_t q = 0;
        const int nvd = d / 32;
        for (int u = cta; u < u_total; u += G) {
            const int b = u / S;
            const int fs = u - b * S;
            const int row0 = R.blk_row0[b];
            const int n = R.blk_n[b];
            if (tid == 0) R.fail = 0;
            compute_sync();  // also: every warp is done with the previous unit's h rows
            const int cg = min(g, n - 1), c0 = min(2 * c, n - 1), c1 = min(2 * c + 1, n - 1);
            const uint16_t* brow = xsh + (R.sa[row0 + cg] / k) * (d + 32) + 8 * c;
            const float* bs0 = xsum + (R.sa[row0 + c0] / k) * nvd;
            const float* bs1 = xsum + (R.sa[row0 + c1] / k) * nvd;
            // gate/up: this warp's half of each stage's K chunks, in order,
            // into one accumulator
            float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            bool ok = true;
            for (int st = 0; st < KC / kDecChunks; ++st, ++q) {
                const int slot = q % kDecStages;
                if (!__all_sync(0xffffffffu, mbar_wait(full(slot), (q / kDecStages) & 1, &R.abort_local))) {
                    ok = false;
                    break;
                }
#pragma unroll
                for (int ci = 0; ci < kHalf; ++ci) {
                    const int cc = kh * kHalf + ci;
                    const uint8_t* hb = ring + slot * kDecStageBytes + cc * p.bb_dn;  // half-block of chunk kc
                    const int kc = kDecChunks * st + cc;
                    chunk_mma_rows<kGpc>(acc, hb + gu_nib_offset(0, fr), hb + gu_nib_offset(1, fr),
                                         hb + gu_word_offset(0, fr, 0, kGpc), hb + gu_word_offset(1, fr, 0, kGpc),
                                         c, brow + kKChunk * kc, bs0 + 2 * kc, bs1 + 2 * kc);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty(slot));
            }
            if (!ok) {
                if (lane == 0) {
                    R.fail = 1;
                    if (!vload(R.abort_local)) dec_fail(p, R, 505);
                }
            }
            // the two halves' sums, first half + second half
            if (kh == 1)
#pragma unroll
                for (int i = 0; i < 4; ++i) red[(rt * 4 + i) * 32 + lane] = acc[i];
            compute_sync();
            if (vload(R.fail)) break;
            // SwiGLU of the row tile's eight features, rounded to bf16, into
            // shared memory [token][64]
            if (kh == 0) {
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i] += red[(rt * 4 + i) * 32 + lane];
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    const int col = 2 * c + e2;
                    if (col < n)
                        hsh[col * kDecHStride + fr] =
                            bf16_round_bits(__fdividef(acc[e2] * acc[2 + e2], 1.0f + __expf(-acc[e2])));
                }
            }
            compute_sync();
            // the 32-wide vector sums of the h rows, for the group folds: warp
            // 2 col + v sums vector v of row col with an xor butterfly (a fixed
            // order)
            if (warp < 2 * n) {
                const int col = warp >> 1, v = warp & 1;
                float sacc = bf16_bits_to_float(hsh[col * kDecHStride + 32 * v + lane]);
#pragma unroll
                for (int m = 16; m >= 1; m >>= 1) sacc = __fadd_rn(sacc, __shfl_xor_sync(0xffffffffu, sacc, m));
                if (lane == 0) hsum[col * 2 + v] = sacc;
            }
            compute_sync();
            // down: up to four 128-row output tiles per stage, K = the slice
            const uint16_t* hrow = hsh + cg * kDecHStride + 8 * c;
            const float* hs0 = hsum + c0 * 2;
            const float* hs1 = hsum + c1 * 2;
            for (int sd = 0; sd < NSd; ++sd, ++q) {
                const int slot = q % kDecStages;
                if (!__all_sync(0xffffffffu, mbar_wait(full(slot), (q / kDecStages) & 1, &R.abort_local))) {
                    if (lane == 0) {
                        R.fail = 1;
                        if (!vload(R.abort_local)) dec_fail(p, R, 506);
                    }
                    break;
                }
                const int nblk = min(kDecChunks, NTd - kDecChunks * sd);
                for (int h = kh * kHalf; h < min(nblk, (kh + 1) * kHalf); ++h) {
                    const int jd = kDecChunks * sd + h;
                    const uint8_t* stage = ring + slot * kDecStageBytes + h * p.bb_dn;
                    float o[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                    chunk_mma<kGpc>(o, stage, 128 * 32, 16 * rt + g, c, hrow, hs0, hs1);
#pragma unroll
                    for (int e2 = 0; e2 < 2; ++e2) {
                        const int col = 2 * c + e2;
                        if (col < n) {
                            float* dst = p.pdn + (static_cast<size_t>(row0 + col) * S + fs) * d + jd * 128 + 16 * rt;
                            dst[g] = o[e2];
                            dst[g + 8] = o[2 + e2];
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty(slot));
            }
            compute_sync();
            if (vload(R.fail)) break;
        }
    }

    // ---- phase 4: combine, after every CTA is done with its units ----------
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        red_release_add(sync + kSyncUnits, 1);
        R.hok = routed && !vload(R.abort_local);
        if (R.hok && !wait_flag(sync + kSyncUnits, G, abort_g)) {
            dec_fail(p, R, 507);
            R.hok = 0;
        }
    }
    __syncthreads();
    if (vload(R.hok)) {
        // this CTA's outputs: flattened (t, m) in [o0, o1); first each
        // (output, slot) pair's expert output (the slice partials summed in
        // slice order, rounded to bf16), then each output's slots in order
        float* ob = reinterpret_cast<float*>(ring);  // the ring is idle now
        const int per = (T * d + G - 1) / G;
        const int o0 = cta * per;
        const int o1 = min(T * d, o0 + per);
        const int cnt = max(o1 - o0, 0);
        for (int it = tid; it < cnt * k; it += kDecThreads) {
            const int jj = it / cnt;
            const int li = it - jj * cnt;
            const int oi = o0 + li;
            const int t = oi / d;
            const int m = oi - t * d;
            const float* src = p.pdn + static_cast<size_t>(R.pos[t * k + jj]) * S * d + m;
            float v[kDecMaxSlices];
#pragma unroll
            for (int sl = 0; sl < kDecMaxSlices; ++sl)
                if (sl < S) v[sl] = ld_cg_f32(src + static_cast<size_t>(sl) * d);
            float sum = v[0];
#pragma unroll
            for (int sl = 1; sl < kDecMaxSlices; ++sl)
                if (sl < S) sum += v[sl];
            ob[jj * cnt + li] = bf16_round(sum);
        }
        __syncthreads();
        for (int li = tid; li < cnt; li += kDecThreads) {
            const int oi = o0 + li;
            const int t = oi / d;
            const int m = oi - t * d;
            float yv = 0.0f;
            for (int jj = 0; jj < k; ++jj) yv = fmaf(R.w[t * k + jj], ob[jj * cnt + li], yv);
            p.y[static_cast<size_t>(t) * d + m] = bf16_round_bits(yv);
        }
    }

    // ---- exit: the last CTA resets the flags --------------------------------
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        R.flag = atom_acq_rel_add(sync + kSyncExit, 1) == G - 1;
    }
    __syncthreads();
    if (vload(R.flag)) {
        for (int i = tid + 2; i < kSyncInts; i += kDecThreads) sync[i] = 0;
        __threadfence();
    }
}

constexpr int kDecSmemLimit = 227 * 1024;

}  // namespace

bool decode_supported(const moe_shape_t& s, int T) {
    if (T < 1 || T > kDecodeMaxT) return false;
    if (T * s.k > kDecMaxAssign || s.E > kMaxExperts || s.E % 8 != 0) return false;
    if (s.f / kDecSlice > kDecMaxSlices || s.d / 128 > kDecMaxNTd) return false;
    return dec_smem_layout(T, s.d, s.E, s.f).total <= kDecSmemLimit;
}

size_t decode_workspace_bytes(const moe_shape_t& s, int T_max) {
    const size_t T = static_cast<size_t>(std::min(T_max, kDecodeMaxT));
    const size_t Tk = T * s.k;
    auto r256 = [](size_t v) { return (v + 255) / 256 * 256; };
    return r256(T * s.E * 8 * 4) + r256(Tk * (s.f / kDecSlice) * s.d * 4);
}

cudaError_t prepare_decode_kernels() {
    cudaError_t e = cudaFuncSetAttribute(decode_layer_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kDecSmemLimit);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(decode_layer_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kDecSmemLimit);
}

cudaError_t launch_decode(const DecodeArgs& a, int num_sms, cudaStream_t st) {
    const moe_shape_t& s = a.s;
    CUtensorMap wmap;
    cudaError_t e = encode_f32_3d_map(&wmap, a.W_r, static_cast<uint64_t>(s.E), 8, static_cast<uint64_t>(s.d / 8),
                                      8, 1, static_cast<uint32_t>(std::min(s.d / 8, kDecWRows)));
    if (e != cudaSuccess) return e;
    DecParams p{};
    p.T = a.T;
    p.d = s.d;
    p.E = s.E;
    p.k = s.k;
    p.f = s.f;
    p.x = a.x;
    p.b_r = a.b_r;
    p.wgu = a.wpack_gu;
    p.wdn = a.wpack_dn;
    p.bb_gu = a.gu_block_bytes;
    p.bb_dn = a.dn_block_bytes;
    p.topk_idx = a.topk_idx;
    p.counts = a.counts;
    p.offsets = a.offsets;
    p.sorted_assign = a.sorted_assign;
    p.pos = a.pos;
    p.block_offsets = a.block_offsets;
    p.block_map = a.block_map;
    p.num_blocks = a.num_blocks;
    p.topk_w = a.topk_w;
    const size_t T = static_cast<size_t>(a.T);
    auto r256 = [](size_t v) { return (v + 255) / 256 * 256; };
    uint8_t* scratch = a.scratch;
    p.U = reinterpret_cast<float*>(scratch);
    p.pdn = reinterpret_cast<float*>(scratch + r256(T * s.E * 8 * 4));
    p.y = a.y;
    p.status = a.status;
    p.sync = a.sync;
    const int smem = dec_smem_layout(a.T, s.d, s.E, s.f).total;
    if (s.group == 64)
        return launch_pdl(decode_layer_kernel<1>, dim3(num_sms), dim3(kDecThreads), smem, st, wmap, p);
    return launch_pdl(decode_layer_kernel<2>, dim3(num_sms), dim3(kDecThreads), smem, st, wmap, p);
}

}  // namespace moe
