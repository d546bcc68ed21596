// Grouped GEMM over int4 expert weights, dequantised on chip (inblix article
// "Perplexity's Lily engine beats MLX by 35% on M5 Max, no PyTorch needed",
// paragraph 3: 4-bit dequantisation fused into the grouped GEMM so expanded
// bf16 weights never reach memory).
//
//   prepack_kernel        logical nibbles/scales -> per (expert, tile, K chunk)
//                         contiguous blocks in the order the GEMM reads them
//   grouped_gemm_kernel   persistent, warp-specialised tcgen05 GEMM:
//       gate/up: D0 = Wg xs^T, D1 = Wu xs^T over token rows in expert order,
//                epilogue h = silu(D0) * D1 -> bf16 h rows
//       down:    D = 128-row tiles of Wd (one, or two in the streaming
//                variant) times h^T, epilogue o = bf16(D) rows
//                (the routing-weighted sum over a token's experts is a
//                separate pass, so no output element is ever accumulated by
//                two CTAs)
//
// One gate/up work unit = one block-map tile (<= 256 expert-ordered rows of
// one expert) x one output tile of 128 features (the gate and the up rows of
// those features).  One down unit = one half of a block-map tile (<= 128
// rows) x two adjacent output tiles of 128 features: each token tile then
// serves two output tiles (the down GEMM waited on its token tiles about a
// quarter of the time with one), and the 256-column accumulator leaves room
// for a second, so the epilogue overlaps the next unit.  The weights are the
// MMA A operand (M = 128 per tile), the tokens the B operand (N = rows
// rounded up to 16), so a partly filled tile wastes at most 15 columns.
//
// Shapes are set by two limits measured on B200: expanding int4 costs about
// two instructions per weight, so every expanded weight must serve up to 256
// tokens; and the MMA's shared-memory operand reads share the read port with
// ordinary loads, so each MMA should read as little shared memory per flop as
// possible (M = 128 x N = 256 reads 96 bytes per clock at full rate).
//
// Warp roles (512 threads, one CTA per SM):
//   warp 0       bulk-copies packed weight blocks into the W ring (TMA engine)
//   warp 1       allocates TMEM; runs the MMA loop, one elected lane issues
//                tcgen05.mma and tcgen05.commit
//   warp 2       loads 2-D TMA tiles of the token rows (xs or h) into the
//                B ring (128-byte swizzle); warp 3 has no role
//   warps 4-11   expand int4 -> bf16 from the W ring into the A ring, in two
//                groups that take alternate K chunks
//   warps 12-15  epilogue: TMEM -> registers -> bf16 rows of h or o
// TMEM: gate/up holds one buffer of 2 x 256 columns (gate, up), so its
// epilogue runs between units.  Down with one tile per unit holds two buffers
// of 256 columns, so its epilogue overlaps the next unit's main loop (measured
// faster than two tiles per unit, which halves the token-operand traffic per
// MMA but exposes the epilogue).
#include <cudaTypedefs.h>

#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kWarpWProducer = 0;
constexpr int kWarpMma = 1;
constexpr int kWarpLoader = 2;
constexpr int kWarpIdle = 3;     // no role
constexpr int kWarpTransform0 = 4;
constexpr int kNumTransformWarps = 8;
constexpr int kWarpEpi0 = 12;
constexpr int kNumEpiWarps = 4;
constexpr int kGemmThreads = 16 * 32;
constexpr int kTransformThreads = kNumTransformWarps * 32;
constexpr int kATileBytes = 128 * 128;     // 128 rows x 64 bf16 (128B swizzle)
constexpr int kEpiRowBytes = 80;    // staging row: 32 bf16 + 16 bytes of padding
constexpr uint32_t kTmemCols = 512;

// Per-projection configuration.  kStream: the ring sizes for blocks of few
// rows (a batch of at most 64 rows per expert on average), where the kernel
// is bound by reading the packed weights from HBM: a deep packed-weight ring
// keeps more of them in flight per SM, at the cost of expanded-A and token
// stages that such blocks do not need.
//
// Units.  Gate/up: (block, 128-feature tile): two A tiles (the tile's gate and
// up rows) x the block's rows (N <= 256), one 512-column accumulator.  Down:
// (block, 128-row output tile): one A tile x the block's rows, two 256-column
// accumulators, so the epilogue of one unit overlaps the next unit's MMAs.
// Streaming variant (few rows per expert): units take one half of a block's
// rows (at most 128), so the token stages are half as large and twice as
// many, and two accumulators fit.  Gate/up: (block, half, 128-feature tile).
// Down ("pair" units): (block, half, pair of output tiles): two A tiles (the
// pair's packed blocks, adjacent in memory for one K chunk), so each token
// tile serves two output tiles.  At 512 tokens the down pairs measured 72
// against 89 us; with large blocks N = 128 doubles the A operand's
// shared-memory reads per flop and the expansion per token (319 against
// 250 us at 8192 tokens).
template <bool kDown, bool kStream>
struct Cfg {
    static constexpr bool kPair = kDown && kStream;
    static constexpr int kTiles = (kDown && !kPair) ? kDownTiles : 2;  // A tiles (of 128 rows) per unit
    static constexpr bool kOneTile = kTiles == 1;
    static constexpr int kBlockN = kStream ? kBlockT / 2 : kBlockT;  // token rows per unit (MMA N at most)
    static constexpr int kNW = kStream ? (kOneTile ? 20 : 8) : (kOneTile ? 4 : 2);  // packed weight ring
    static constexpr int kNA = kStream ? 2 : (kOneTile ? 4 : 3);  // expanded bf16 A ring
    static constexpr int kNB = kStream ? 4 : 3;                   // token B ring
    static constexpr int kAccBufs = (kDown || kStream) ? 2 : 1;   // TMEM accumulator buffers
    static constexpr int kAccCols = kTiles * kBlockN;         // columns per buffer
    static constexpr int kBStageBytes = kBlockN * 128;        // token rows x 64 bf16
    static constexpr int kAStageBytes = kTiles * kATileBytes;
    static constexpr int kWStageBytes = packed_block_bytes(kTiles, 32);  // largest (group 32)
    static constexpr int kEpiWarpBytes = 32 * kEpiRowBytes;
    // transform warp groups; group g expands the chunks it with it % kGroups == g
    static constexpr int kGroups = kOneTile ? 2 : 1;
    static constexpr int kGroupThreads = kTransformThreads / kGroups;
    static constexpr int kTasks = kTiles * 256 / kGroupThreads;  // (row, half) tasks per thread

    static constexpr int kOffA = 0;
    static constexpr int kOffB = kOffA + kNA * kAStageBytes;
    static constexpr int kOffW = kOffB + kNB * kBStageBytes;
    static constexpr int kOffEpi = kOffW + kNW * kWStageBytes;
    static constexpr int kOffBar = kOffEpi + kNumEpiWarps * kEpiWarpBytes;
    static constexpr int kNumBars = 2 * kNW + 2 * kNA + 2 * kNB + 2 * kAccBufs + 1;
    static constexpr int kOffMisc = kOffBar + 8 * kNumBars;
    static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + slack to align the base

    static_assert(kOffA % 1024 == 0 && kOffB % 1024 == 0 && kAStageBytes % 1024 == 0,
                  "UMMA tiles need 1024-byte alignment");
    static_assert(kOffW % 16 == 0 && kWStageBytes % 16 == 0, "bulk copies need 16-byte alignment");
    static_assert(kOffBar % 8 == 0, "mbarriers are 8-byte aligned");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
    static_assert(kAccBufs * kAccCols <= static_cast<int>(kTmemCols), "TMEM budget");
    // mbarrier parity waits only tell a phase from the one before it, so no
    // waiter may ever be two phases ahead of a barrier.  Transform groups take
    // alternate chunks; with ring sizes that are multiples of the group count
    // every W and A stage is filled and released by one group only, which
    // keeps each group at most one phase ahead.  (A shared A ring with three
    // or four groups deadlocks in a discrete-event model of this protocol.)
    static_assert(kNW % kGroups == 0 && kNA % kGroups == 0,
                  "transform groups must not alias mbarrier phases");
    static_assert(kTasks * kGroupThreads == kTiles * 256, "transform task split");
};

static_assert(kWarpIdle + 1 == kWarpTransform0 && kWarpEpi0 % 4 == 0 &&
                  kWarpEpi0 + kNumEpiWarps == kGemmThreads / 32,
              "every warp has exactly one role; epilogue warps cover TMEM quadrants 0..3");

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// mbar_wait for a whole converged warp: every lane waits and the outcome is
// voted, so the warp takes the same branch whatever happens at a timeout.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, limit_ns));
}

// Wait used only while shutting down after an abort: ignores the abort flag.
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > 200000000ull) return false;
    }
    return true;
}

template <bool kDown, bool kStream>
__global__ void __launch_bounds__(kGemmThreads, 1) grouped_gemm_kernel(const __grid_constant__ GemmArgs a) {
    using C = Cfg<kDown, kStream>;
    extern __shared__ uint8_t smem_raw[];
    pdl_launch_dependents();
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // barrier addresses
    const uint32_t bar0 = sbase + C::kOffBar;
    auto wfull = [&](int s) { return bar0 + 8u * s; };
    auto wempty = [&](int s) { return bar0 + 8u * (C::kNW + s); };
    auto afull = [&](int s) { return bar0 + 8u * (2 * C::kNW + s); };
    auto aempty = [&](int s) { return bar0 + 8u * (2 * C::kNW + C::kNA + s); };
    auto bfull = [&](int s) { return bar0 + 8u * (2 * C::kNW + 2 * C::kNA + s); };
    auto bempty = [&](int s) { return bar0 + 8u * (2 * C::kNW + 2 * C::kNA + C::kNB + s); };
    auto accfull = [&](int s) { return bar0 + 8u * (2 * C::kNW + 2 * C::kNA + 2 * C::kNB + s); };
    auto accempty = [&](int s) {
        return bar0 + 8u * (2 * C::kNW + 2 * C::kNA + 2 * C::kNB + C::kAccBufs + s);
    };
    const uint32_t drain_bar = bar0 + 8u * (C::kNumBars - 1);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kNW; ++s) {
            mbar_init(wfull(s), 1);
            mbar_init(wempty(s), kNumTransformWarps / C::kGroups);
        }
        for (int s = 0; s < C::kNA; ++s) {
            mbar_init(afull(s), kNumTransformWarps / C::kGroups);
            mbar_init(aempty(s), 1);
        }
        for (int s = 0; s < C::kNB; ++s) {
            mbar_init(bfull(s), 1);
            mbar_init(bempty(s), 1);
        }
        for (int s = 0; s < C::kAccBufs; ++s) {
            mbar_init(accfull(s), 1);
            mbar_init(accempty(s), kNumEpiWarps);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();  // the block map, the token rows and (down) h come from earlier kernels

    const int NT = a.NT;
    const int KC = a.K / kKChunk;
    const int num_units = min(*a.num_blocks * NT, a.max_units);

    auto fail = [&](int where) {
        *abort_flag = 1;
        report_error(a.status, MOE_ERR_DEVICE_TIMEOUT, (kDown ? 200 : 100) + where);
    };
    // unit u: block b = u / NT, output tile j = u % NT.  Streaming variant:
    // first every block's first half of rows, then every block's second half
    // (units u and u + nblk * NT / 2 are the two halves of one (block, tile)),
    // with output tile (gate/up) or tile pair (down) j; so the units that are
    // empty (a second half of a block of <= 128 rows) come last and the
    // persistent grid deals the others out evenly.  Every role skips the same
    // empty units.
    const int nhu = *a.num_blocks * (NT / 2);  // units per half (streaming variant)
    struct Unit {
        int b, j, row0, rows;
    };
    auto unit_of = [&](int u) {
        Unit x;
        int r;
        int half = 0;
        if constexpr (kStream) {
            half = u >= nhu ? 1 : 0;
            const int v = u - half * nhu;
            x.b = v / (NT / 2);
            r = v - x.b * (NT / 2);
        } else {
            x.b = u / NT;
            r = u - x.b * NT;
        }
        const int row0 = a.block_map[3 * x.b + 1];
        const int rows = a.block_map[3 * x.b + 2];
        if constexpr (kStream) {
            x.j = r;
            x.row0 = row0 + half * C::kBlockN;
            x.rows = min(C::kBlockN, rows - half * C::kBlockN);
        } else {
            x.j = r;
            x.row0 = row0;
            x.rows = rows;
        }
        return x;
    };

    if (warp == kWarpWProducer) {
        // the whole warp runs the loop; one elected lane issues the copies
        uint32_t it = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
            const Unit un = unit_of(u);
            if (un.rows <= 0) continue;
            const int j = un.j;
            const int e = a.block_map[3 * un.b];
            // down: blocks (e, c, kTiles j ..) for chunk c, adjacent (a chunk's
            // output tiles are contiguous); gate/up: half-blocks (e, j, 0, c)
            // and (e, j, 1, c)
            const int NTg = kStream ? NT / 2 : NT;  // gate/up feature tiles of an expert
            const uint8_t* src = a.wpack + (static_cast<size_t>(e) * NTg + j) * KC * a.block_bytes;
            const size_t half_stride = static_cast<size_t>(KC) * (a.block_bytes / 2);
            for (int c = 0; c < KC; ++c, ++it) {
                const int s = it % C::kNW;
                if (!warp_wait(wempty(s), ((it / C::kNW) & 1) ^ 1, abort_flag, a.wait_ns)) {
                    fail(1);
                    ok = false;
                    break;
                }
                // test hook: withhold the first stage, so its consumers' waits run out
                if (a.withhold_first && it == 0) continue;
                if (elect_one()) {
                    const uint32_t dst = sbase + C::kOffW + s * C::kWStageBytes;
                    if constexpr (kDown) {
                        // the unit's kTiles output tiles of chunk c, adjacent blocks
                        const uint32_t bytes = C::kTiles * a.block_bytes;
                        mbar_arrive_expect_tx(wfull(s), bytes);
                        bulk_copy_g2s(dst,
                                      a.wpack + ((static_cast<size_t>(e) * KC + c) * NT + C::kTiles * j) * a.block_bytes,
                                      bytes, wfull(s));
                    } else {
                        mbar_arrive_expect_tx(wfull(s), a.block_bytes);
                        const uint32_t hb = a.block_bytes / 2;
                        bulk_copy_g2s(dst, src + c * hb, hb, wfull(s));
                        bulk_copy_g2s(dst + hb, src + half_stride + c * hb, hb, wfull(s));
                    }
                }
                __syncwarp();
            }
        }
        if (!ok && lane == 0) {
            // let the copies already issued land before the CTA exits
            const uint32_t first = it > C::kNW ? it - C::kNW : 0;
            for (uint32_t i = first; i < it; ++i)
                if (!(a.withhold_first && i == 0)) mbar_wait_drain(wfull(i % C::kNW), (i / C::kNW) & 1);
        }
    } else if (warp == kWarpMma) {
        // The whole warp runs the issue loop so descriptors and ring indices
        // stay warp-uniform; one elected lane issues each MMA and commit.
        uint32_t it = 0, ucount = 0;
        bool ok = true;
        bool ready = false;  // the current stage was already seen full
        for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
            const Unit un = unit_of(u);
            if (un.rows <= 0) continue;
            const int N = (un.rows + 15) & ~15;
            const uint32_t idesc = make_idesc_bf16(128, N);
            const int buf = ucount % C::kAccBufs;
            const uint32_t use = ucount / C::kAccBufs;
            if (!warp_wait(accempty(buf), (use & 1) ^ 1, abort_flag, a.wait_ns)) {
                fail(2);
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t dacc = tmem + buf * C::kAccCols;
            for (int c = 0; c < KC; ++c, ++it) {
                const int sa = it % C::kNA;
                const int sb = it % C::kNB;
                if (!ready && (!warp_wait(afull(sa), (it / C::kNA) & 1, abort_flag, a.wait_ns) ||
                               !warp_wait(bfull(sb), (it / C::kNB) & 1, abort_flag, a.wait_ns))) {
                    fail(3);
                    ok = false;
                    break;
                }
                // order the asynchronous MMAs after the waits (the transform
                // warps fence their generic-proxy stores to A before arriving;
                // B arrives through the TMA, already in the async proxy)
                tc_fence_after();
                // Test the next stage now and look at the answer only after this
                // stage's MMAs are issued: a barrier read stalls the issuing
                // thread for about as long as one MMA runs, and the tensor core's
                // queue is too short to hide it.
                const uint32_t nx = it + 1;
                const uint32_t ra = mbar_test(afull(nx % C::kNA), (nx / C::kNA) & 1);
                const uint32_t rb = mbar_test(bfull(nx % C::kNB), (nx / C::kNB) & 1);
                const uint32_t abase = sbase + C::kOffA + sa * C::kAStageBytes;
                const uint64_t db = make_sw128_desc(sbase + C::kOffB + sb * C::kBStageBytes);
                uint64_t da[C::kTiles];
#pragma unroll
                for (int t = 0; t < C::kTiles; ++t) da[t] = make_sw128_desc(abase + t * kATileBytes);
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < kKChunk / 16; ++kk) {
                        const uint32_t acc = (c > 0 || kk > 0) ? 1u : 0u;
#pragma unroll
                        for (int t = 0; t < C::kTiles; ++t)
                            mma_bf16(dacc + t * C::kBlockN, da[t] + 2 * kk, db + 2 * kk, idesc, acc);
                    }
                    mma_commit(aempty(sa));
                    mma_commit(bempty(sb));
                }
                ready = __all_sync(0xffffffffu, (ra & rb) != 0);
            }
            if (ok && elect_one()) mma_commit(accfull(buf));
            __syncwarp();
            ++ucount;
        }
        if (!ok) {
            if (elect_one()) mma_commit(drain_bar);
            __syncwarp();
            mbar_wait_drain(drain_bar, 0);
        }
    } else if (warp == kWarpLoader) {
        // one 2-D TMA tile of token rows per stage, 256, 128, 64 or 32 rows: the
        // smallest that covers the N rows the MMA reads (rows past the block
        // belong to the next expert or lie past the end and are zero-filled;
        // the MMA ignores columns >= N and the epilogue columns >= rows)
        uint32_t it = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
            const Unit un = unit_of(u);
            if (un.rows <= 0) continue;
            const int row0 = un.row0;
            // the smallest box (256 >> bi rows) that covers the N rows the MMA
            // reads (N <= kBlockN, so the box fits the stage)
            const int N = (un.rows + 15) & ~15;
            int bi = 0;
            while (bi + 1 < kBoxSizes && (kBlockT >> (bi + 1)) >= N) ++bi;
            const uint32_t box_bytes = static_cast<uint32_t>(kBlockT >> bi) * (kKChunk * 2);
            for (int c = 0; c < KC; ++c, ++it) {
                const int s = it % C::kNB;
                if (!warp_wait(bempty(s), ((it / C::kNB) & 1) ^ 1, abort_flag, a.wait_ns)) {
                    fail(4);
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    mbar_arrive_expect_tx(bfull(s), box_bytes);
                    tma_load_2d(sbase + C::kOffB + s * C::kBStageBytes, &a.bmap[bi], c * kKChunk, row0, bfull(s));
                }
                __syncwarp();
            }
        }
        if (!ok && lane == 0) {
            const uint32_t first = it > C::kNB ? it - C::kNB : 0;
            for (uint32_t i = first; i < it; ++i)
                mbar_wait_drain(bfull(i % C::kNB), (i / C::kNB) & 1);
        }
    } else if (warp >= kWarpTransform0 && warp < kWarpTransform0 + kNumTransformWarps) {
        // One-tile units: two groups of transform warps take alternate chunks,
        // so each warp pays one round of barrier waits per two chunks; two-tile
        // units: all eight warps expand each chunk.
        const int ttid = threadIdx.x - kWarpTransform0 * 32;
        const int grp = ttid / C::kGroupThreads;
        const int gtid = ttid % C::kGroupThreads;
        const int gpc = kKChunk / a.group;
        uint32_t it = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
            if (unit_of(u).rows <= 0) continue;
            for (int c = 0; c < KC; ++c, ++it) {
                if (static_cast<int>(it % C::kGroups) != grp) continue;
                const int sw = it % C::kNW;
                const int sa = it % C::kNA;
                if (!warp_wait(wfull(sw), (it / C::kNW) & 1, abort_flag, a.wait_ns) ||
                    !warp_wait(aempty(sa), ((it / C::kNA) & 1) ^ 1, abort_flag, a.wait_ns)) {
                    fail(5);
                    ok = false;
                    break;
                }
                const uint8_t* wst = smem + C::kOffW + sw * C::kWStageBytes;
                const uint32_t ast = sbase + C::kOffA + sa * C::kAStageBytes;
                // Task rep of this thread: packed row (gtid + kGroupThreads*rep) / 2
                // (tile row >> 7, row & 127 within it), K half gtid & 1.  All
                // loads of the chunk are issued before the first store so their
                // latencies overlap.
                const int half = gtid & 1;       // K 0..31 or 32..63 of the chunk
                const int g = half * (gpc - 1);  // group 64: 0; group 32: half
                const int hbytes = a.block_bytes / 2;  // gate/up half-block
                uint4 pk[C::kTasks];
                uint32_t sb[C::kTasks];
#pragma unroll
                for (int rep = 0; rep < C::kTasks; ++rep) {
                    const int row = (gtid + C::kGroupThreads * rep) >> 1;
                    int nib_off, w_off;
                    if constexpr (kDown) {  // row: block (output tile) row >> 7 of the stage, row & 127 in it
                        const int boff = (row >> 7) * a.block_bytes;
                        nib_off = boff + (row & 127) * 32;
                        w_off = boff + 128 * 32 + ((row & 127) * gpc + g) * 4;
                    } else {  // row: tile row >> 7, feature row & 127 in half-block (row & 127) >> 6
                        const int hoff = ((row & 127) >> 6) * hbytes;
                        nib_off = hoff + gu_nib_offset(row >> 7, row & 63);
                        w_off = hoff + gu_word_offset(row >> 7, row & 63, g, gpc);
                    }
                    pk[rep] = *reinterpret_cast<const uint4*>(wst + nib_off + half * 16);
                    sb[rep] = *reinterpret_cast<const uint32_t*>(wst + w_off);
                }
#pragma unroll
                for (int rep = 0; rep < C::kTasks; ++rep) {
                    const int row = (gtid + C::kGroupThreads * rep) >> 1;
                    BF2 s2, b2;
                    s2.u = __byte_perm(sb[rep], 0, 0x1010);
                    b2.u = __byte_perm(sb[rep], 0, 0x3232);
                    const uint32_t arow = ast + (row >> 7) * kATileBytes + (row & 127) * 128;
                    const int rsw = row & 7;
                    st_shared_v4(arow + (((half * 4 + 0) ^ rsw) << 4), expand8(pk[rep].x, s2.h, b2.h));
                    st_shared_v4(arow + (((half * 4 + 1) ^ rsw) << 4), expand8(pk[rep].y, s2.h, b2.h));
                    st_shared_v4(arow + (((half * 4 + 2) ^ rsw) << 4), expand8(pk[rep].z, s2.h, b2.h));
                    st_shared_v4(arow + (((half * 4 + 3) ^ rsw) << 4), expand8(pk[rep].w, s2.h, b2.h));
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(afull(sa));
                    mbar_arrive(wempty(sw));
                }
            }
        }
    } else if (warp >= kWarpEpi0) {
        // Epilogue warps: warp % 4 selects the TMEM lane quadrant, i.e. output
        // features q*32 .. q*32+31 of the tile; the accumulator is
        // D[feature][token].  Per block of 32 tokens the warp reads two 16-lane
        // halves in the m16n8 fragment layout, rounds pairs of neighbouring
        // tokens to bf16x2, and writes them transposed with stmatrix into a
        // staging tile [token][32 features]; each lane then copies one
        // token's 64 bytes to global memory.
        const int q = warp & 3;
        const uint32_t stg = sbase + C::kOffEpi + (warp - kWarpEpi0) * C::kEpiWarpBytes;
        // stmatrix row address of this thread: matrix m = lane / 8 is the
        // feature octet (16 bytes), row c = lane % 8 the token within a group of 8
        const uint32_t st_addr = stg + (lane & 7) * kEpiRowBytes + (lane >> 3) * 16;
        uint32_t ucount = 0;
        for (int u = blockIdx.x; u < num_units; u += gridDim.x) {
            const Unit un = unit_of(u);
            if (un.rows <= 0) continue;
            const int j = un.j;
            const int row0 = un.row0;
            const int rows = un.rows;
            const int ncb = (rows + 31) >> 5;
            const int buf = ucount % C::kAccBufs;
            const uint32_t use = ucount / C::kAccBufs;
            if (!warp_wait(accfull(buf), use & 1, abort_flag, a.wait_ns)) {
                fail(6);
                break;
            }
            tc_fence_after();
            // gate/up: one output tile (gate at column 0, up at kBlockN); down:
            // kTiles output tiles of 128 features at columns t * kBlockN
            constexpr int kOutTiles = kDown ? C::kTiles : 1;
#pragma unroll 1
            for (int it = 0; it < kOutTiles * ncb; ++it) {
                const int t = it / ncb;
                const int cb = it - t * ncb;
                const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * C::kAccCols +
                                    t * C::kBlockN;
                // p[h][i]: lane half h (features 16h + t/4 (+8)), register i
                uint32_t p[2][8];
                if constexpr (kDown) {
                    // both lane halves in flight before the one wait
                    uint32_t v[2][16];
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        tmem_ld_16x256b_x4(tb + (static_cast<uint32_t>(16 * h) << 16) + cb * 32, v[h]);
                    tmem_ld_wait();
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            BF2 o;
                            o.h = __floats2bfloat162_rn(__uint_as_float(v[h][2 * i]),
                                                        __uint_as_float(v[h][2 * i + 1]));
                            p[h][i] = o.u;
                        }
                } else {
                    // gate and up of both lane halves in flight before one wait
                    uint32_t v[2][16], uu[2][16];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t ta = tb + (static_cast<uint32_t>(16 * h) << 16) + cb * 32;
                        tmem_ld_16x256b_x4(ta, v[h]);
                        tmem_ld_16x256b_x4(ta + C::kBlockN, uu[h]);
                    }
                    tmem_ld_wait();
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            float hv[2];
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const float gv = __uint_as_float(v[h][2 * i + e]);
                                const float uv = __uint_as_float(uu[h][2 * i + e]);
                                hv[e] = __fdividef(gv * uv, 1.0f + __expf(-gv));
                            }
                            BF2 o;
                            o.h = __floats2bfloat162_rn(hv[0], hv[1]);
                            p[h][i] = o.u;
                        }
                }
                if (it == kOutTiles * ncb - 1) {
                    // every TMEM read of this unit has completed: hand the
                    // accumulator back to the MMA warp before the last stores
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(accempty(buf));
                }
                // token group g (8 tokens): matrices (h, octet) = registers
                // p[h][2g] (features 16h + 0..7) and p[h][2g+1] (16h + 8..15)
#pragma unroll
                for (int g = 0; g < 4; ++g)
                    stmatrix_x4_trans(st_addr + g * 8 * kEpiRowBytes, p[0][2 * g], p[0][2 * g + 1],
                                      p[1][2 * g], p[1][2 * g + 1]);
                __syncwarp();
                const int c = cb * 32 + lane;
                if (c < rows) {
                    const uint4* s4 = reinterpret_cast<const uint4*>(
                        smem + C::kOffEpi + (warp - kWarpEpi0) * C::kEpiWarpBytes + lane * kEpiRowBytes);
                    uint4* d4 = reinterpret_cast<uint4*>(a.out + static_cast<size_t>(row0 + c) * a.out_ld +
                                                         (j * kOutTiles + t) * 128 + q * 32);
                    d4[0] = s4[0];
                    d4[1] = s4[1];
                    d4[2] = s4[2];
                    d4[3] = s4[3];
                }
                __syncwarp();
            }
            if (ncb == 0) {  // a unit always has rows; keep the hand-back unconditional
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(accempty(buf));
            }
            ++ucount;
        }
    }

    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// One thread per (expert, tile, K chunk, packed row): writes 8 words of
// nibbles and the row's (scale, bias) pairs of that chunk.  A block holds
// s.tiles tiles of 128 rows; packed row rr comes from tile rr / 128.
__global__ void prepack_kernel(const PrepackSource s, int E, int group, uint8_t* __restrict__ out) {
    const int KC = s.K / kKChunk;
    const int gpc = kKChunk / group;
    const int bb = packed_block_bytes(s.tiles, group);
    const int rows = 128 * s.tiles;
    const int nibble_bytes = rows * 32;
    const long total = static_cast<long>(E) * s.NT * KC * rows;
    for (long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += static_cast<long>(gridDim.x) * blockDim.x) {
        const int rr = static_cast<int>(idx % rows);
        long blk = idx / rows;
        const int c = static_cast<int>(blk % KC);
        blk /= KC;
        const int j = static_cast<int>(blk % s.NT);
        const int e = static_cast<int>(blk / s.NT);
        const bool second = rr >= 128;
        const int n = j * s.row_step + (second ? s.a1_off : 0) + (rr & 127);
        const uint8_t* qsrc = second ? s.q1 : s.q0;
        const uint16_t* ssrc = second ? s.s1 : s.s0;
        const uint16_t* bsrc = second ? s.b1 : s.b0;
        const size_t row = static_cast<size_t>(e) * s.N + n;
        const uint8_t* qrow = qsrc + row * (s.K / 2) + c * 32;
        // down: block (e, c, j); gate/up: half-block (e, j, half, c) (see packed_block_bytes)
        const int f = rr & 127;
        const int hb = half_block_bytes(group);
        uint8_t* dst = s.tiles == 1
                           ? out + ((static_cast<size_t>(e) * KC + c) * s.NT + j) * bb
                           : out + (((static_cast<size_t>(e) * s.NT + j) * 2 + (f >> 6)) * KC + c) * hb;
        const int nib_off = s.tiles == 1 ? rr * 32 : gu_nib_offset(second ? 1 : 0, f & 63);
        uint32_t words[8];
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            uint32_t word = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t byte = qrow[4 * w + i];  // K = 8w+2i (low), 8w+2i+1 (high)
                word |= (byte & 0xFu) << (4 * i);
                word |= (byte >> 4) << (16 + 4 * i);
            }
            words[w] = word;
        }
        uint4* d4 = reinterpret_cast<uint4*>(dst + nib_off);
        d4[0] = make_uint4(words[0], words[1], words[2], words[3]);
        d4[1] = make_uint4(words[4], words[5], words[6], words[7]);
        const size_t grow = row * (s.K / group) + static_cast<size_t>(c) * gpc;
        for (int g = 0; g < gpc; ++g) {
            const uint32_t sv = ssrc[grow + g];
            const uint32_t bv = bsrc[grow + g];
            const int w_off = s.tiles == 1 ? nibble_bytes + (rr * gpc + g) * 4
                                           : gu_word_offset(second ? 1 : 0, f & 63, g, gpc);
            *reinterpret_cast<uint32_t*>(dst + w_off) = sv | (bv << 16);
        }
    }
}

}  // namespace

cudaError_t prepare_gemm_kernels() {
    cudaError_t e;
#define MOE_SET_SMEM(D, S)                                                                     \
    e = cudaFuncSetAttribute(grouped_gemm_kernel<D, S>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             Cfg<D, S>::kSmemBytes);                                           \
    if (e != cudaSuccess) return e;
    MOE_SET_SMEM(false, false)
    MOE_SET_SMEM(true, false)
    MOE_SET_SMEM(false, true)
    MOE_SET_SMEM(true, true)
#undef MOE_SET_SMEM
    return cudaSuccess;
}

static cudaError_t tensor_map_encoder(PFN_cuTensorMapEncodeTiled_v12000* out) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (encode == nullptr) {
        cudaDriverEntryPointQueryResult q;
        void* fn = nullptr;
        const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr)
            return e != cudaSuccess ? e : cudaErrorInvalidValue;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    *out = encode;
    return cudaSuccess;
}

cudaError_t encode_f32_cols_map(CUtensorMap* map, const float* base, uint64_t rows, uint64_t cols,
                                uint32_t box_cols, uint32_t box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    const cudaError_t e = tensor_map_encoder(&encode);
    if (e != cudaSuccess) return e;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 4};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_u8_rows_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                               uint32_t box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    const cudaError_t e = tensor_map_encoder(&encode);
    if (e != cudaSuccess) return e;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {128, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_f32_3d_map(CUtensorMap* map, const float* base, uint64_t d0, uint64_t d1, uint64_t d2,
                              uint32_t b0, uint32_t b1, uint32_t b2) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    const cudaError_t e = tensor_map_encoder(&encode);
    if (e != cudaSuccess) return e;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {d0 * 4, d0 * d1 * 4};
    const cuuint32_t box[3] = {b0, b1, b2};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_bf16_rows_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                                 uint32_t box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    const cudaError_t e = tensor_map_encoder(&encode);
    if (e != cudaSuccess) return e;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kKChunk), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_prepack(const PrepackSource& src, int E, int group, uint8_t* out,
                           cudaStream_t st) {
    const long total = static_cast<long>(E) * src.NT * (src.K / kKChunk) * 128 * src.tiles;
    const int threads = 256;
    const long blocks = (total + threads - 1) / threads;
    prepack_kernel<<<static_cast<int>(blocks < 65535 * 16 ? blocks : 65535 * 16), threads, 0, st>>>(
        src, E, group, out);
    return cudaGetLastError();
}

template <bool kDown, bool kStream>
static cudaError_t launch_gemm_t(const GemmArgs& a, int num_sms, cudaStream_t st) {
    const int grid = a.max_units < num_sms ? a.max_units : num_sms;
    // Plain launches: letting the next kernel's CTAs be scheduled early measured
    // slower around the GEMMs (their pdl_wait then returns at once).
    grouped_gemm_kernel<kDown, kStream><<<grid, kGemmThreads, Cfg<kDown, kStream>::kSmemBytes, st>>>(a);
    return cudaGetLastError();
}

static cudaError_t launch_gemm(const GemmArgs& a, int num_sms, bool down, cudaStream_t st) {
    if (a.max_units <= 0) return cudaSuccess;
    if (down)
        return a.stream ? launch_gemm_t<true, true>(a, num_sms, st) : launch_gemm_t<true, false>(a, num_sms, st);
    return a.stream ? launch_gemm_t<false, true>(a, num_sms, st) : launch_gemm_t<false, false>(a, num_sms, st);
}

cudaError_t launch_gemm_gateup(const GemmArgs& a, int num_sms, cudaStream_t st) {
    return launch_gemm(a, num_sms, false, st);
}

cudaError_t launch_gemm_down(const GemmArgs& a, int num_sms, cudaStream_t st) {
    return launch_gemm(a, num_sms, true, st);
}

}  // namespace moe
