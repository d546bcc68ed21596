/*
 * int4 expert-grouped mixture-of-experts layer for NVIDIA B200 (sm_100a).
 *
 * C ABI of libmoe_b200.so.  One call runs one MoE layer:
 *   routing (softmax top-k) -> per-expert counts and prefix scan ->
 *   scatter into expert-contiguous order with a tile block map ->
 *   grouped GEMM over 4-bit group-quantised expert weights (gate/up with
 *   SwiGLU, then down) whose weights are expanded to bf16 on chip only ->
 *   routing-weighted combine.
 * The step list is the one the inblix article "Perplexity's Lily engine
 * beats MLX by 35% on M5 Max, no PyTorch needed" credits for prefill speed
 * (paragraph 3: dequantisation fused into the grouped GEMM so expanded
 * bf16 weights never reach memory; expert routing, prefix scan, scatter and
 * block map kept on the GPU in one submission).
 *
 * Conventions for every entry point:
 *   - Device pointers, host pointers and streams are owned by the caller.
 *     The library never allocates device memory.  moe_route and
 *     moe_forward never synchronise and never read device data on the host;
 *     everything runs on the caller's stream in order.
 *   - Every call returns a moe_status_t.  Argument errors are reported
 *     before anything is launched.  Errors found on the device (a wait that
 *     timed out, an index out of range) are written to a status word in
 *     the workspace; read it with moe_read_status after synchronising.
 *   - Streams are passed as void* (a cudaStream_t; NULL = legacy default).
 *   - bf16 values are passed as uint16_t bit patterns.
 *   - Device pointers must be 16-byte aligned (MOE_ERR_ALIGNMENT).
 *   - A plan is immutable once built and may be used from several host
 *     threads; calls that share a workspace must not overlap on the GPU.
 */
#ifndef INT4_EXPERT_GROUPED_MOE_H
#define INT4_EXPERT_GROUPED_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 1

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,       /* null pointer, T < 0 or T > T_max, ... */
    MOE_ERR_UNSUPPORTED_SHAPE = 2, /* shape outside what the kernels tile  */
    MOE_ERR_ALIGNMENT = 3,         /* a device pointer not 16-byte aligned */
    MOE_ERR_WORKSPACE_TOO_SMALL = 4,
    MOE_ERR_CUDA = 5,              /* a CUDA runtime call or launch failed */
    MOE_ERR_DEVICE_TIMEOUT = 6,    /* a device-side wait gave up (status word) */
    MOE_ERR_DEVICE_BOUNDS = 7      /* a device-side index check failed (status word) */
} moe_status_t;

/*
 * Layer shape.  Supported (the tile sizes are fixed for these shapes, as a
 * single-model engine fixes them; the ai.jakubjirak.com post "Perplexity's
 * Lily beats MLX by 1.35x ...", section "Why one model on one chip is
 * faster"):
 *   d % 256 == 0, f % 128 == 0, group in {32, 64},
 *   1 <= k <= E, E % 8 == 0, E <= 256, k <= 32, 0 < T_max <= 2^24 / k.
 */
typedef struct moe_shape {
    int32_t T_max; /* largest token count any call will pass              */
    int32_t d;     /* hidden size                                          */
    int32_t E;     /* number of experts                                    */
    int32_t k;     /* experts per token                                    */
    int32_t f;     /* expert intermediate size                             */
    int32_t group; /* int4 group size along the reduction dimension        */
    uint32_t flags;/* 0, or MOE_SHAPE_TEST_TIMEOUT                         */
} moe_shape_t;

/*
 * Test hook, not for production plans: in moe_forward's batched path the
 * gate/up grouped GEMM's weight producer withholds its first copy and every
 * wait of that kernel gives up after 5 ms, so the call records
 * MOE_ERR_DEVICE_TIMEOUT (detail 101..106: the role that gave up) in the
 * workspace status word instead of a result.  It exercises the bounded-wait
 * and abort path without faulting or hanging the GPU; the workspace stays
 * usable for the next call.
 */
#define MOE_SHAPE_TEST_TIMEOUT 1u

typedef struct moe_plan moe_plan_t;

/* What a plan needs from the caller (all sizes in bytes). */
typedef struct moe_plan_info {
    size_t workspace_bytes;      /* device scratch for moe_route / moe_forward */
    size_t host_workspace_bytes; /* device scratch for moe_forward_host        */
    size_t packed_weight_bytes;  /* output of moe_prepack_weights              */
    int32_t block_t;             /* tile height of the block map (rows)        */
    int32_t max_blocks;          /* capacity the block map needs for T_max     */
} moe_plan_info_t;

/*
 * One int4 projection of all experts in logical layout (device pointers):
 *   q     [E, N, K/2] bytes: weight (n, kk) is the low nibble of byte
 *         q[e, n, kk/2] when kk is even, the high nibble when kk is odd;
 *   scale [E, N, K/group] bf16;  bias [E, N, K/group] bf16;
 *   weight value = nibble * scale + bias of its group along K.
 * Gate and up have N = f, K = d; down has N = d, K = f.
 */
typedef struct moe_projection {
    const uint8_t *q;
    const uint16_t *scale;
    const uint16_t *bias;
} moe_projection_t;

typedef struct moe_expert_weights {
    moe_projection_t gate, up, down;
} moe_expert_weights_t;

/*
 * Routing results (device pointers, caller-owned).  With T tokens:
 *   topk_idx      int32 [T, k]   experts per token, best first; ties go to
 *                                the lower expert id
 *   topk_w        fp32  [T, k]   softmax over the k selected logits (evaluated
 *                                in double, rounded once to fp32)
 *   counts        int32 [E]      assignments per expert
 *   offsets       int32 [E+1]    exclusive prefix sum of counts
 *   sorted_assign int32 [T*k]    assignment a = t*k + j at expert-ordered row
 *                                p; ascending a within an expert
 *   pos           int32 [T*k]    inverse of sorted_assign
 *   block_offsets int32 [E+1]    first block map entry of each expert
 *   block_map     int32 [max_blocks, 3]  (expert, first row, rows) per tile
 *                                of at most block_t rows, ascending expert
 *   num_blocks    int32 [1]      number of block map entries
 */
typedef struct moe_route_out {
    int32_t *topk_idx;
    float *topk_w;
    int32_t *counts;
    int32_t *offsets;
    int32_t *sorted_assign;
    int32_t *pos;
    int32_t *block_offsets;
    int32_t *block_map;
    int32_t *num_blocks;
} moe_route_out_t;

MOE_API int moe_abi_version(void);
MOE_API const char *moe_status_str(moe_status_t s);

/*
 * Build a plan for a shape.  Host only: launches nothing, touches no GPU
 * state.  Fills *info (may be NULL).  MOE_ERR_UNSUPPORTED_SHAPE if the
 * shape is outside the list above.
 */
MOE_API moe_status_t moe_plan_create(const moe_shape_t *shape, moe_plan_t **plan,
                             moe_plan_info_t *info);
MOE_API moe_status_t moe_plan_info(const moe_plan_t *plan, moe_plan_info_t *info);
MOE_API void moe_plan_destroy(moe_plan_t *plan);

/*
 * Repack the logical int4 weights into the order the grouped GEMM reads
 * (one contiguous block per expert, output tile and 64-wide K chunk, with
 * the nibbles of each 32-bit word arranged for the on-chip expansion), as a
 * single-model engine lays weights out in the order its kernels read them
 * fastest (ai.jakubjirak.com post, section "Why one model on one chip is
 * faster").  One-time, on `stream`; packed_out needs packed_weight_bytes.
 */
MOE_API moe_status_t moe_prepack_weights(const moe_plan_t *plan,
                                 const moe_expert_weights_t *logical,
                                 void *packed_out, void *stream);

/*
 * Routing steps only (inblix, paragraph 3: expert routing, prefix scan,
 * scatter, block map), for T tokens (0 <= T <= T_max):
 *   x    bf16 [T, d] device;  W_r fp32 [d, E] device (row-major);
 *   b_r  fp32 [E] device router bias, or NULL for none.
 * The router logit of (t, e) is x[t,:] . W_r[:,e] summed in fp32 as 32
 * fused-multiply-add chains (chain p takes i = p, p+32, ... in ascending i)
 * combined by an xor butterfly (m = 16, 8, 4, 2, 1), plus b_r[e]; every
 * integer output is therefore reproducible bit for bit.
 * All fields of *out are required.  ws: workspace_bytes of device memory.
 */
MOE_API moe_status_t moe_route(const moe_plan_t *plan, int32_t T, const uint16_t *x,
                       const float *W_r, const float *b_r,
                       const moe_route_out_t *out, void *ws, size_t ws_bytes,
                       void *stream);

/*
 * The whole layer: y = sum_j topk_w[t,j] * expert_{topk_idx[t,j]}(x[t]),
 * expert(x) = W_down (silu(W_gate x) * (W_up x)), for T tokens
 * (0 <= T <= T_max).
 *   packed_w: moe_prepack_weights output; y: bf16 [T, d] device (written).
 *   route_out: NULL, or buffers that receive the routing results.
 * Rounding: x is bf16, weights are expanded to bf16 (one rounding of
 * nibble*scale+bias), products accumulate in fp32, the SwiGLU output is
 * rounded to bf16 before the down projection, each expert's down output is
 * rounded to bf16, the k weighted outputs of a token are summed in fp32 in
 * slot order j = 0..k-1 and y is rounded to bf16.  The small-batch kernels
 * (moe_forward_path == 1) do not round the weights: each group's fp32 sum of
 * nibble * x takes the group's scale and bias (scale * sum + bias * sum x);
 * the later roundings are the same.
 */
MOE_API moe_status_t moe_forward(const moe_plan_t *plan, int32_t T, const uint16_t *x,
                         const float *W_r, const float *b_r,
                         const void *packed_w, uint16_t *y,
                         const moe_route_out_t *route_out, void *ws,
                         size_t ws_bytes, void *stream);

/*
 * Optional stage timing for moe_forward_timed: CUDA events (cudaEvent_t as
 * void*, created by the caller) recorded on the stream at stage boundaries.
 * Any field may be NULL.
 */
typedef struct moe_stage_events {
    void *start;   /* before the routing kernels                         */
    void *routed;  /* after top-k, prefix scan, scatter, block map and
                      the copy of the token rows into expert order       */
    void *gate_up; /* after the gate/up grouped GEMM (SwiGLU fused)      */
    void *down;    /* after the down grouped GEMM                        */
    void *end;     /* after the routing-weighted combine into y          */
} moe_stage_events_t;

/* moe_forward, also recording *events (may be NULL) between the stages. */
MOE_API moe_status_t moe_forward_timed(const moe_plan_t *plan, int32_t T,
                                       const uint16_t *x, const float *W_r,
                                       const float *b_r, const void *packed_w,
                                       uint16_t *y,
                                       const moe_route_out_t *route_out,
                                       void *ws, size_t ws_bytes, void *stream,
                                       const moe_stage_events_t *events);

/*
 * moe_forward from HOST buffers: copies x_host (bf16 [T, d], ideally
 * pinned) to the device, runs the layer, copies y back into y_host and
 * synchronises the stream before returning.  W_r, b_r and packed_w stay
 * device pointers (model state).  ws: host_workspace_bytes of device memory.
 */
MOE_API moe_status_t moe_forward_host(const moe_plan_t *plan, int32_t T,
                              const uint16_t *x_host, const float *W_r,
                              const float *b_r, const void *packed_w,
                              uint16_t *y_host, void *ws, size_t ws_bytes,
                              void *stream);

/*
 * Expert parallelism: the layer's experts split over ranks (one process per
 * GPU), rank r holding a contiguous range of them.  The scatter already puts
 * the rows for one rank's experts next to each other, so each rank runs
 *   moe_route            routing of its own tokens over all E experts
 *   moe_dispatch         its token rows in expert order (one segment per rank)
 *   (the caller sends segment r to rank r, e.g. an NCCL all-to-all)
 *   moe_experts_forward  the grouped GEMMs over the rows it received, for its
 *                        own experts (a plan and packed weights of just those)
 *   (the caller sends the outputs back the same way)
 *   moe_combine          the routing-weighted sum of its tokens' outputs
 * The scatter with its block map (inblix, paragraph 3) is the step the
 * exchange hangs on; the exchange itself is the caller's (NCCL over NVLink
 * in int4_expert_grouped_b200/ep.py).  The three entries below run one part
 * of moe_forward each, with the same arithmetic.
 *
 * moe_dispatch: xs[p] = x[sorted_assign[p] / k] for p < T*k.
 *   x bf16 [T, d]; sorted_assign int32 [T*k] (from moe_route, values < T*k,
 *   else MOE_ERR_DEVICE_BOUNDS detail 300 and row 0 is copied);
 *   xs bf16 [T*k, d] (written).  ws: workspace_bytes (status word only).
 */
MOE_API moe_status_t moe_dispatch(const moe_plan_t *plan, int32_t T, const uint16_t *x,
                                  const int32_t *sorted_assign, uint16_t *xs, void *ws,
                                  size_t ws_bytes, void *stream);

/*
 * moe_experts_forward: o[p] = bf16(W_down^e (bf16(silu(W_gate^e xs[p]) *
 * (W_up^e xs[p])))) for every row p of every block map entry (e, first row,
 * rows); the expert ids index this plan's experts (its E, its packed
 * weights).  Rounding as moe_forward's batched path.
 *   rows      rows of xs and o, 0 <= rows <= T_max * k;
 *   xs        bf16 [rows, d] device, the rows in any order;
 *   block_map int32 [max_blocks, 3] device: entries of at most block_t rows
 *             (moe_plan_info), each with expert < E, first row >= 0 and first
 *             row + rows <= rows of xs; num_blocks int32 [1] device, at most
 *             max_blocks.  A map out of range is not used: the call records
 *             MOE_ERR_DEVICE_BOUNDS (detail 400) and writes nothing to o.
 *             Rows outside every entry are left as they were in o.
 *   o         bf16 [rows, d] device (written).
 *   ws        workspace_bytes of device memory for this plan.
 */
MOE_API moe_status_t moe_experts_forward(const moe_plan_t *plan, int32_t rows,
                                         const uint16_t *xs, const int32_t *block_map,
                                         const int32_t *num_blocks, int32_t max_blocks,
                                         const void *packed_w, uint16_t *o, void *ws,
                                         size_t ws_bytes, void *stream);

/*
 * moe_combine: y[t] = bf16(sum_{j<k} topk_w[t,j] * o[pos[t*k+j]]), the sum in
 * fp32 in slot order.  o bf16 [T*k, d] (row p = the expert output of
 * expert-ordered row p); pos and topk_w from moe_route (pos values < T*k,
 * else MOE_ERR_DEVICE_BOUNDS detail 301 and that slot counts as 0);
 * y bf16 [T, d] (written).  ws: workspace_bytes (status word only).
 */
MOE_API moe_status_t moe_combine(const moe_plan_t *plan, int32_t T, const uint16_t *o,
                                 const int32_t *pos, const float *topk_w, uint16_t *y, void *ws,
                                 size_t ws_bytes, void *stream);

/*
 * moe_route without a workspace, for callers that cannot allocate device
 * memory (code running under a stream capture that forbids allocation, a
 * runtime that owns every byte of device memory, a plugin host that hands a
 * kernel only its inputs and outputs).  The pages describe no such entry
 * point; it has no counterpart there.
 *   Arguments and outputs: as moe_route, without ws / ws_bytes.
 *   Scratch: a fixed 4 MiB array inside the library, per GPU, held until the
 *     process exits.  A call needs 256 + 4*T*E + 8*ceil(T/256)*E bytes of it
 *     (each part rounded up to 256); larger calls return
 *     MOE_ERR_WORKSPACE_TOO_SMALL before launching anything.
 *   The first call on a device looks up the array's device address (with
 *     that device current) and sets the router kernels' attributes for every
 *     batch size; make it before any stream capture begins.
 *   Every call shares the one array: calls that overlap on the GPU (other
 *     streams, other host threads) race and must be serialised by the caller.
 *   Device-side errors are recorded in the array and cannot be read back.
 *   It allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 *     call.
 */
MOE_API moe_status_t moe_route_noalloc(const moe_plan_t *plan, int32_t T,
                                       const uint16_t *x, const float *W_r,
                                       const float *b_r,
                                       const moe_route_out_t *out, void *stream);

/*
 * Read the device status word of a workspace (synchronises `stream`
 * first).  *code is a moe_status_t (MOE_OK if no device error was
 * recorded); *detail says where.  clear != 0 resets the word afterwards.
 */
MOE_API moe_status_t moe_read_status(const void *ws, int32_t *code, int32_t *detail,
                             int32_t clear, void *stream);

/*
 * Which kernels moe_forward runs at batch T for this plan:
 *   1  the small-batch (decode) kernel, one launch, which streams the
 *      selected experts' weights (wpnews page "Perplexity Lily: 1.35x Faster
 *      Local AI Than MLX on Mac", section "Why MLX Falls Behind": prefill and
 *      decode are separate workloads);
 *   0  the batched grouped-GEMM kernels with the fp32 router: eight launches
 *      (router logits, top-k, scan, scatter, dispatch, gate/up GEMM, down
 *      GEMM, combine);
 *   2  the batched kernels with the int8 tensor-core router and its exact
 *      recheck (T >= 1024): nine launches (router prep, approximate logits,
 *      selection, then as for 0 from the scan on);
 *  -1  plan is NULL or T is outside 0..T_max.
 * All three give the same routing results.  Host only; launches nothing.
 */
MOE_API int moe_forward_path(const moe_plan_t *plan, int32_t T);

#ifdef __cplusplus
}
#endif

#endif /* INT4_EXPERT_GROUPED_MOE_H */
