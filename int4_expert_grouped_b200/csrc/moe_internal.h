// Internal constants and kernel launchers shared by the host API and the
// kernel files.  Not part of the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "moe_common.cuh"

// Plan of one layer shape (opaque to callers of the C ABI).
struct moe_plan {
    moe_shape_t s;
    int block_t;
    int max_blocks;
    int ng_max;
    int group_bytes;  // packed block bytes, gate/up (two tiles)
    int down_block_bytes;  // packed block bytes, down (one tile)
    size_t gu_packed;  // bytes of the gate/up packed blocks
    size_t dn_packed;
    size_t packed_bytes;
    // workspace offsets
    size_t o_status, o_dsync, o_dscr, o_logits, o_hist, o_gbase, o_idx, o_w, o_counts, o_offsets, o_bo, o_nb,
        o_sa, o_pos, o_bm, o_xs, o_h, o_rfast, ws_bytes;
    size_t o_xstage, o_ystage, host_ws_bytes;
};

namespace moe {

// Launch with programmatic stream serialization: the kernel may be scheduled
// while its predecessor in the stream finishes, and waits for it in pdl_wait.
template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

constexpr int kMaxExperts = 256;  // experts per layer the routing kernels hold
constexpr int kMaxTopk = 32;      // one warp lane per selected expert
constexpr int kRouteGroupT = 256; // tokens per scatter group (one histogram row)
constexpr int kBlockT = 256;      // block map tile height = largest MMA N
constexpr int kKChunk = 64;       // K elements per pipeline stage (128 bytes bf16)
constexpr int kDecodeMaxT = 8;    // largest batch the small-batch (decode) path takes
constexpr int kDownTiles = 1;     // 128-row down-projection tiles per packed block
constexpr int kBoxSizes = 4;      // token-tile boxes of 256, 128, 64 and 32 rows
constexpr int kDecodeSyncBytes = 8192;  // flags of the small-batch kernel (workspace bytes 256 ..)

// Packed weight block: `tiles` 128-row A tiles of one 64-wide K chunk
// (gate/up: the gate and the up rows of 128 features; down: 128 rows).
// A down block is 128 rows x 32 bytes of nibbles, then per row and group one
// (scale, bias) bf16 pair; the blocks of one K chunk (a 64-feature slice of
// h) are stored over all output tiles in a row (layout [E][f/64][d/128][block]).
// A gate/up block is two half-blocks of the same
// form, one per 64 features: [64 gate rows][64 up rows] of nibbles, then the
// gate rows' and the up rows' words; each half-block is stored with the same
// half of the expert's other K chunks (layout [E][f/128][2][d/64][half-block]),
// so the 64-feature slice of an expert is contiguous over K.
__host__ __device__ constexpr int packed_block_bytes(int tiles, int group) {
    return 128 * tiles * 32 + 128 * tiles * (kKChunk / group) * 4;
}
__host__ __device__ constexpr int half_block_bytes(int group) { return packed_block_bytes(1, group); }
// Byte offsets, inside a gate/up half-block, of the nibbles of row fl (< 64)
// of tile t (0 gate, 1 up) and of its word for group g of the chunk.
__host__ __device__ inline int gu_nib_offset(int t, int fl) { return t * 64 * 32 + fl * 32; }
__host__ __device__ inline int gu_word_offset(int t, int fl, int g, int gpc) {
    return 128 * 32 + (t * 64 + fl) * gpc * 4 + g * 4;
}

// ---- routing (moe_route.cu) ----
cudaError_t launch_router_logits(const uint16_t* x, const float* W, const float* b, float* logits,
                                 int T, int d, int E, int32_t* hist, int hist_n, int32_t* status,
                                 cudaStream_t st);
cudaError_t launch_router_topk(const float* logits, int T, int E, int k, int32_t* topk_idx,
                               float* topk_w, int32_t* hist, cudaStream_t st);
cudaError_t launch_route_scan(const int32_t* hist, int ng, int E, int BT, int32_t* counts,
                              int32_t* offsets, int32_t* gbase, int32_t* block_offsets,
                              int32_t* block_map, int32_t* num_blocks, int max_blocks,
                              int32_t* status, cudaStream_t st);
cudaError_t launch_route_scatter(const int32_t* topk_idx, const int32_t* gbase, int T, int k,
                                 int E, int32_t* sorted_assign, int32_t* pos, int32_t* status,
                                 cudaStream_t st);

// ---- router with exact near-tie recheck (moe_router_fast.cu) ----
constexpr int kFastRouterMinT = 1024;  // smallest batch the int8 tensor-core router takes
struct RouterFastWs {
    int8_t *xa, *xb;            // token digits [T][d]
    int8_t *wc, *wd;            // expert digits [E][d]
    float *s_t, *E_t, *A_t, *N_t;  // per token: scale, remainder max, sum |x'|, ||x||
    float *u_e, *F_e, *B_e, *Wn_e;         // per expert: scale, remainder max, sum |w|, ||w||
    float* L;                   // [T][E] approximate logits with the bias
    float* wt;                  // [E][d] W_r transposed (fp32, exact copy)
};
bool router_fast_supported(int T, int d, int E);
size_t router_fast_ws_bytes(int T, int d, int E);
// Carve the router's scratch out of `base` (router_fast_ws_bytes); L is the
// [T][E] logits buffer.
RouterFastWs router_fast_ws(uint8_t* base, float* L, int T, int d, int E);
cudaError_t prepare_router_fast();
// Shared-memory attributes of every fp32 router tiling (also run on a call's
// first use of a tiling; done up front so that no later call makes it inside
// a stream capture).
cudaError_t prepare_router();
// Top-k indices and weights and the per-group histograms (cleared here, as is
// the status word) for T >= kFastRouterMinT tokens.
cudaError_t launch_router_fast(const uint16_t* x, const float* W, const float* b, int T, int d, int E,
                               int k, const RouterFastWs& ws, int32_t* topk_idx, float* topk_w,
                               int32_t* hist, int hist_n, int32_t* status, cudaStream_t st);

// ---- weights and GEMM (moe_gemm.cu) ----
struct PrepackSource {
    const uint8_t* q0;   // A0 rows come from this projection
    const uint16_t* s0;
    const uint16_t* b0;
    const uint8_t* q1;   // A1 rows come from this projection
    const uint16_t* s1;
    const uint16_t* b1;
    int N;               // rows per expert of the source projections
    int K;               // reduction length
    int row_step;        // source row of tile j, row r: j*row_step + r (A0), + a1_off (A1)
    int a1_off;
    int NT;              // output tiles per expert
    int tiles;           // 128-row A tiles per packed block (1 or 2)
};
cudaError_t launch_prepack(const PrepackSource& src, int E, int group, uint8_t* out,
                           cudaStream_t st);

struct GemmArgs {
    // B operand (token rows in expert order) for 2-D TMA tiles of 64 columns
    // with the 128-byte swizzle, the K-major layout the MMA reads: gate/up
    // reads xs [T*k, d], down reads h [T*k, f].  bmap[i] has boxes of
    // kBlockT >> i rows; a unit loads the smallest box that covers its rows.
    CUtensorMap bmap[kBoxSizes];
    const uint8_t* wpack;          // packed blocks [E][NT][K/64][block_bytes]
    const int32_t* block_map;      // [num_blocks, 3]
    const int32_t* num_blocks;     // [1], device
    uint16_t* out;                 // h [T*k, f] (gate/up) or o [T*k, d] (down), bf16
    int32_t* status;
    int K;                         // reduction length
    int NT;                        // output tiles of 128 features per expert
    int out_ld;                    // f (gate/up) or d (down)
    int group;
    int block_bytes;
    int max_units;                 // upper bound of num_blocks * NT
    int stream;                    // ring sizes for blocks of few rows (weight streaming)
    int withhold_first;            // test hook: the weight producer skips its first copy
    uint64_t wait_ns;              // limit of every device-side wait
};
// Encode the tensor map of a row-major fp32 matrix [rows, cols] read in boxes
// of box_cols columns x box_rows rows, unswizzled.
cudaError_t encode_f32_cols_map(CUtensorMap* map, const float* base, uint64_t rows, uint64_t cols,
                                uint32_t box_cols, uint32_t box_rows);
// Encode the tensor map of a row-major int8 matrix [rows, cols] read in boxes
// of 128 columns (bytes) x box_rows rows with the 128-byte swizzle.
cudaError_t encode_u8_rows_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                               uint32_t box_rows);
// Encode the tensor map of a 3-D fp32 tensor with dims d0 (innermost,
// contiguous) x d1 x d2, read in unswizzled boxes b0 x b1 x b2.
cudaError_t encode_f32_3d_map(CUtensorMap* map, const float* base, uint64_t d0, uint64_t d1, uint64_t d2,
                              uint32_t b0, uint32_t b1, uint32_t b2);
// Encode the tensor map of a row-major bf16 matrix [rows, cols] read in boxes
// of 64 columns x box_rows rows with the 128-byte swizzle.
cudaError_t encode_bf16_rows_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                                 uint32_t box_rows);

cudaError_t launch_gemm_gateup(const GemmArgs& a, int num_sms, cudaStream_t st);
cudaError_t launch_gemm_down(const GemmArgs& a, int num_sms, cudaStream_t st);
cudaError_t prepare_gemm_kernels();

// ---- dispatch and combine (moe_combine.cu) ----
// xs[p] = x[sorted_assign[p] / k] for p < T*k
cudaError_t launch_dispatch(const uint16_t* x, const int32_t* sorted_assign, int Tk, int k, int d,
                            uint16_t* xs, int32_t* status, int num_sms, cudaStream_t st);
// Check a caller-built block map before the GEMMs read it (moe_experts_forward):
// at most max_blocks entries, each with expert < E, first row >= 0,
// 0 <= rows <= block_t and first row + rows <= n_rows.  Clears the status
// word (the call's first kernel), then writes the entry count to *nb_out, or
// 0 with MOE_ERR_DEVICE_BOUNDS (detail 400) if any entry is out of range.
cudaError_t launch_block_map_check(const int32_t* block_map, const int32_t* num_blocks, int max_blocks,
                                   int n_rows, int E, int block_t, int32_t* nb_out, int32_t* status,
                                   cudaStream_t st);
// y[t] = bf16(sum_i topk_w[t*k+i] * o[pos[t*k+i]])
cudaError_t launch_combine(const uint16_t* o, const int32_t* pos, const float* topk_w, int T,
                           int k, int d, uint16_t* y, int32_t* status, int num_sms,
                           cudaStream_t st);

// ---- small-batch path (moe_decode.cu) ----
struct DecodeArgs {
    moe_shape_t s;
    int T;
    const uint16_t* x;
    const float* W_r;
    const float* b_r;
    const uint8_t* wpack_gu;     // packed gate/up blocks
    const uint8_t* wpack_dn;     // packed down blocks
    int gu_block_bytes;
    int dn_block_bytes;
    int32_t *topk_idx, *counts, *offsets, *sorted_assign, *pos, *block_offsets, *block_map,
        *num_blocks;
    float* topk_w;
    uint16_t* h;                 // workspace [T*k, f]
    uint16_t* y;                 // [T, d]
    int32_t* status;
    int32_t* sync;               // workspace flags (kDecodeSyncBytes, zero or left by this kernel)
    uint8_t* scratch;            // workspace, decode_workspace_bytes
};
// Whether the small-batch kernel takes this shape at batch T (otherwise the
// batched path runs).
bool decode_supported(const moe_shape_t& s, int T);
// Workspace bytes of the small-batch kernel's partial sums for batches up to T_max.
size_t decode_workspace_bytes(const moe_shape_t& s, int T_max);
cudaError_t prepare_decode_kernels();
cudaError_t launch_decode(const DecodeArgs& a, int num_sms, cudaStream_t st);

}  // namespace moe
