// Host side of the C ABI declared in include/moe.h: shape checks, plan and
// workspace layout, argument validation before any launch, and the launch
// sequence of one layer on the caller's stream (no host synchronisation and
// no host read of device data between the routing stages and the GEMMs, as
// the inblix article "Perplexity's Lily engine beats MLX by 35% on M5 Max, no
// PyTorch needed" describes for expert routing, prefix scan, scatter and
// block map in paragraph 3).
#include <algorithm>
#include <atomic>
#include <cstring>
#include <new>

#include "moe_internal.h"

namespace {

using moe::kBlockT;
using moe::kRouteGroupT;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status_t check_shape(const moe_shape_t& s) {
    if ((s.flags & ~static_cast<uint32_t>(MOE_SHAPE_TEST_TIMEOUT)) != 0) return MOE_ERR_INVALID_ARG;
    if (s.T_max <= 0 || s.d <= 0 || s.E <= 0 || s.k <= 0 || s.f <= 0) return MOE_ERR_INVALID_ARG;
    if (s.k > s.E) return MOE_ERR_INVALID_ARG;
    if (s.group != 32 && s.group != 64) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (s.d % 256 != 0 || s.f % 128 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (s.E % 8 != 0 || s.E > moe::kMaxExperts || s.k > moe::kMaxTopk)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (static_cast<long long>(s.T_max) * s.k > (1ll << 24)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (static_cast<long long>(s.d) * s.f > (1ll << 26)) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

struct DeviceCache {
    std::atomic<int> sms{0};
    std::atomic<int> prepared{0};
};
DeviceCache g_dev[64];

moe_status_t device_setup(int* num_sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    DeviceCache& c = g_dev[dev];
    if (c.prepared.load() == 0) {
        if (moe::prepare_gemm_kernels() != cudaSuccess) return MOE_ERR_CUDA;
        if (moe::prepare_decode_kernels() != cudaSuccess) return MOE_ERR_CUDA;
        if (moe::prepare_router_fast() != cudaSuccess) return MOE_ERR_CUDA;
        if (moe::prepare_router() != cudaSuccess) return MOE_ERR_CUDA;
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        c.sms.store(sms);
        c.prepared.store(1);
    }
    *num_sms = c.sms.load();
    return MOE_OK;
}

template <class T>
T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

struct RoutePtrs {
    int32_t* idx;
    float* w;
    int32_t* counts;
    int32_t* offsets;
    int32_t* sa;
    int32_t* pos;
    int32_t* bo;
    int32_t* bm;
    int32_t* nb;
};

RoutePtrs route_ptrs(const moe_plan* p, void* ws, const moe_route_out_t* out) {
    if (out != nullptr)
        return {out->topk_idx, out->topk_w,        out->counts,    out->offsets, out->sorted_assign,
                out->pos,      out->block_offsets, out->block_map, out->num_blocks};
    return {at<int32_t>(ws, p->o_idx),    at<float>(ws, p->o_w),       at<int32_t>(ws, p->o_counts),
            at<int32_t>(ws, p->o_offsets), at<int32_t>(ws, p->o_sa),    at<int32_t>(ws, p->o_pos),
            at<int32_t>(ws, p->o_bo),      at<int32_t>(ws, p->o_bm),    at<int32_t>(ws, p->o_nb)};
}

moe_status_t check_route_out(const moe_route_out_t* o) {
    const void* ps[] = {o->topk_idx, o->topk_w,        o->counts,    o->offsets,   o->sorted_assign,
                        o->pos,      o->block_offsets, o->block_map, o->num_blocks};
    for (const void* q : ps) {
        if (q == nullptr) return MOE_ERR_INVALID_ARG;
        if (!aligned16(q)) return MOE_ERR_ALIGNMENT;
    }
    return MOE_OK;
}

#define MOE_CUDA(call)                          \
    do {                                        \
        if ((call) != cudaSuccess) return MOE_ERR_CUDA; \
    } while (0)

// Steps 1-4 (routing).
moe_status_t run_route(const moe_plan* p, int T, const uint16_t* x, const float* W_r,
                       const float* b_r, const RoutePtrs& r, void* ws, cudaStream_t st) {
    const moe_shape_t& s = p->s;
    int32_t* status = at<int32_t>(ws, p->o_status);
    int32_t* hist = at<int32_t>(ws, p->o_hist);
    const int ng = (T + kRouteGroupT - 1) / kRouteGroupT;
    if (moe::router_fast_supported(T, s.d, s.E)) {
        // int8 tensor-core logits with a proven error bound; the fixed-order
        // fp32 logits only for the pairs the bound cannot settle
        const moe::RouterFastWs fw = moe::router_fast_ws(at<uint8_t>(ws, p->o_rfast),
                                                         at<float>(ws, p->o_logits), T, s.d, s.E);
        MOE_CUDA(moe::launch_router_fast(x, W_r, b_r, T, s.d, s.E, s.k, fw, r.idx, r.w, hist,
                                         std::max(ng, 1) * s.E, status, st));
    } else {
        MOE_CUDA(moe::launch_router_logits(x, W_r, b_r, at<float>(ws, p->o_logits), T, s.d, s.E, hist,
                                           std::max(ng, 1) * s.E, status, st));
        MOE_CUDA(moe::launch_router_topk(at<float>(ws, p->o_logits), T, s.E, s.k, r.idx, r.w, hist,
                                         st));
    }
    MOE_CUDA(moe::launch_route_scan(hist, ng, s.E, p->block_t, r.counts, r.offsets,
                                    at<int32_t>(ws, p->o_gbase), r.bo, r.bm, r.nb, p->max_blocks,
                                    status, st));
    MOE_CUDA(moe::launch_route_scatter(r.idx, at<int32_t>(ws, p->o_gbase), T, s.k, s.E, r.sa,
                                       r.pos, status, st));
    return MOE_OK;
}

int max_blocks_for(const moe_shape_t& s, int T) {
    const long long tk = static_cast<long long>(T) * s.k;
    return static_cast<int>((tk + kBlockT - 1) / kBlockT + std::min<long long>(s.E, tk));
}

}  // namespace

extern "C" {

int moe_abi_version(void) { return MOE_ABI_VERSION; }

const char* moe_status_str(moe_status_t s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case MOE_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case MOE_ERR_CUDA: return "CUDA runtime error";
        case MOE_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        case MOE_ERR_DEVICE_BOUNDS: return "device-side index out of range";
    }
    return "unknown status";
}

moe_status_t moe_plan_create(const moe_shape_t* shape, moe_plan_t** plan, moe_plan_info_t* info) {
    if (shape == nullptr || plan == nullptr) return MOE_ERR_INVALID_ARG;
    *plan = nullptr;
    const moe_status_t st = check_shape(*shape);
    if (st != MOE_OK) return st;
    moe_plan* p = new (std::nothrow) moe_plan();
    if (p == nullptr) return MOE_ERR_INVALID_ARG;
    const moe_shape_t& s = *shape;
    p->s = s;
    p->block_t = kBlockT;
    p->max_blocks = max_blocks_for(s, s.T_max);
    p->ng_max = (s.T_max + kRouteGroupT - 1) / kRouteGroupT;
    p->group_bytes = moe::packed_block_bytes(2, s.group);
    p->down_block_bytes = moe::packed_block_bytes(moe::kDownTiles, s.group);
    const size_t E = s.E;
    p->gu_packed = E * (s.f / 128) * (s.d / moe::kKChunk) * p->group_bytes;
    p->dn_packed = E * (s.d / (128 * moe::kDownTiles)) * (s.f / moe::kKChunk) * p->down_block_bytes;
    p->packed_bytes = align_up(p->gu_packed, 256) + p->dn_packed;

    const size_t T = s.T_max, k = s.k;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t r = o;
        o = align_up(o + bytes, 256);
        return r;
    };
    p->o_status = take(256);
    p->o_dsync = take(moe::kDecodeSyncBytes);  // offset 256: flags of the small-batch kernel
    p->o_dscr = take(moe::decode_workspace_bytes(s, s.T_max));
    p->o_logits = take(T * E * 4);
    p->o_hist = take(static_cast<size_t>(p->ng_max) * E * 4);
    p->o_gbase = take(static_cast<size_t>(p->ng_max) * E * 4);
    p->o_idx = take(T * k * 4);
    p->o_w = take(T * k * 4);
    p->o_counts = take(E * 4);
    p->o_offsets = take((E + 1) * 4);
    p->o_bo = take((E + 1) * 4);
    p->o_nb = take(16);
    p->o_sa = take(T * k * 4);
    p->o_pos = take(T * k * 4);
    p->o_bm = take(static_cast<size_t>(p->max_blocks) * 12);
    p->o_xs = take(T * k * s.d * 2);  // x rows in expert order, later the down outputs o
    p->o_h = take(T * k * s.f * 2);
    p->o_rfast = take(moe::router_fast_supported(s.T_max, s.d, s.E)
                          ? moe::router_fast_ws_bytes(s.T_max, s.d, s.E)
                          : 0);
    p->ws_bytes = o;
    p->o_xstage = take(T * s.d * 2);
    p->o_ystage = take(T * s.d * 2);
    p->host_ws_bytes = o;
    *plan = p;
    return moe_plan_info(p, info);
}

moe_status_t moe_plan_info(const moe_plan_t* plan, moe_plan_info_t* info) {
    if (plan == nullptr) return MOE_ERR_INVALID_ARG;
    if (info != nullptr) {
        info->workspace_bytes = plan->ws_bytes;
        info->host_workspace_bytes = plan->host_ws_bytes;
        info->packed_weight_bytes = plan->packed_bytes;
        info->block_t = plan->block_t;
        info->max_blocks = plan->max_blocks;
    }
    return MOE_OK;
}

void moe_plan_destroy(moe_plan_t* plan) { delete plan; }

moe_status_t moe_prepack_weights(const moe_plan_t* plan, const moe_expert_weights_t* lw,
                                 void* packed_out, void* stream) {
    if (plan == nullptr || lw == nullptr || packed_out == nullptr) return MOE_ERR_INVALID_ARG;
    const moe_projection_t* ps[] = {&lw->gate, &lw->up, &lw->down};
    for (const moe_projection_t* pr : ps) {
        if (pr->q == nullptr || pr->scale == nullptr || pr->bias == nullptr)
            return MOE_ERR_INVALID_ARG;
        if (!aligned16(pr->q) || !aligned16(pr->scale) || !aligned16(pr->bias))
            return MOE_ERR_ALIGNMENT;
    }
    if (!aligned16(packed_out)) return MOE_ERR_ALIGNMENT;
    const moe_shape_t& s = plan->s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* out = static_cast<uint8_t*>(packed_out);
    moe::PrepackSource gu{lw->gate.q, lw->gate.scale, lw->gate.bias, lw->up.q, lw->up.scale,
                          lw->up.bias, s.f, s.d, 128, 0, s.f / 128, 2};
    MOE_CUDA(moe::launch_prepack(gu, s.E, s.group, out, st));
    moe::PrepackSource dn{lw->down.q, lw->down.scale, lw->down.bias, lw->down.q, lw->down.scale,
                          lw->down.bias, s.d, s.f, 128 * moe::kDownTiles, 128,
                          s.d / (128 * moe::kDownTiles), moe::kDownTiles};
    MOE_CUDA(moe::launch_prepack(dn, s.E, s.group, out + align_up(plan->gu_packed, 256), st));
    return MOE_OK;
}

moe_status_t moe_route(const moe_plan_t* plan, int32_t T, const uint16_t* x, const float* W_r,
                       const float* b_r, const moe_route_out_t* out, void* ws, size_t ws_bytes,
                       void* stream) {
    if (plan == nullptr || out == nullptr || ws == nullptr || W_r == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (T < 0 || T > plan->s.T_max) return MOE_ERR_INVALID_ARG;
    if (T > 0 && x == nullptr) return MOE_ERR_INVALID_ARG;
    const moe_status_t c = check_route_out(out);
    if (c != MOE_OK) return c;
    if (!aligned16(ws) || !aligned16(W_r) || (x && !aligned16(x)) || (b_r && !aligned16(b_r)))
        return MOE_ERR_ALIGNMENT;
    if (ws_bytes < plan->ws_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
    return run_route(plan, T, x, W_r, b_r, route_ptrs(plan, ws, out), ws,
                     static_cast<cudaStream_t>(stream));
}

// Steps 6-7: the gate/up GEMM (SwiGLU fused) and the down GEMM over
// expert-ordered rows xs [rows, d] tiled by block_map (num_blocks entries on
// the device, at most mb); h [rows, f] is scratch and o [rows, d] receives the
// expert outputs (o may be xs: gate/up has finished reading xs when the down
// GEMM starts).  after_gate_up: an event recorded between the two, or NULL.
static moe_status_t run_experts(const moe_plan* plan, int rows, const uint16_t* xs, const int32_t* block_map,
                         const int32_t* num_blocks, int mb, const void* packed_w, uint16_t* h, uint16_t* o,
                         int32_t* status, bool test_timeout, int num_sms, cudaStream_t st,
                         cudaEvent_t after_gate_up) {
    const moe_shape_t& s = plan->s;
    const uint8_t* wp = static_cast<const uint8_t*>(packed_w);
    moe::GemmArgs g{};
    g.wpack = wp;
    g.block_map = block_map;
    g.num_blocks = num_blocks;
    g.out = h;
    g.status = status;
    // at most 64 rows per expert on average: the GEMMs are bound by reading the
    // weights, so they keep more packed-weight stages in flight, and each unit
    // takes one half (<= 128 rows) of a block
    g.stream = static_cast<long long>(rows) < 64ll * s.E ? 1 : 0;
    g.K = s.d;
    g.NT = (s.f / 128) * (g.stream ? 2 : 1);  // units per block: feature tiles (x halves)
    g.out_ld = s.f;
    g.group = s.group;
    g.block_bytes = plan->group_bytes;
    g.max_units = mb * g.NT;
    // test hook (MOE_SHAPE_TEST_TIMEOUT): the gate/up GEMM withholds a stage and
    // its waits give up after 5 ms
    g.withhold_first = test_timeout ? 1 : 0;
    g.wait_ns = test_timeout ? 5000000ull : moe::kWaitTimeoutNs;
    for (int i = 0; i < moe::kBoxSizes; ++i)
        MOE_CUDA(moe::encode_bf16_rows_map(&g.bmap[i], xs, static_cast<uint64_t>(rows), s.d, moe::kBlockT >> i));
    MOE_CUDA(moe::launch_gemm_gateup(g, num_sms, st));
    if (after_gate_up != nullptr) MOE_CUDA(cudaEventRecord(after_gate_up, st));

    g.wpack = wp + align_up(plan->gu_packed, 256);
    g.out = o;
    g.K = s.f;
    g.NT = s.d / (128 * moe::kDownTiles);
    g.out_ld = s.d;
    g.block_bytes = plan->down_block_bytes;
    g.max_units = mb * g.NT;
    g.withhold_first = 0;
    g.wait_ns = moe::kWaitTimeoutNs;
    for (int i = 0; i < moe::kBoxSizes; ++i)
        MOE_CUDA(moe::encode_bf16_rows_map(&g.bmap[i], h, static_cast<uint64_t>(rows), s.f, moe::kBlockT >> i));
    MOE_CUDA(moe::launch_gemm_down(g, num_sms, st));
    return MOE_OK;
}

moe_status_t moe_forward(const moe_plan_t* plan, int32_t T, const uint16_t* x, const float* W_r,
                         const float* b_r, const void* packed_w, uint16_t* y,
                         const moe_route_out_t* route_out, void* ws, size_t ws_bytes,
                         void* stream) {
    return moe_forward_timed(plan, T, x, W_r, b_r, packed_w, y, route_out, ws, ws_bytes, stream,
                             nullptr);
}

moe_status_t moe_forward_timed(const moe_plan_t* plan, int32_t T, const uint16_t* x,
                               const float* W_r, const float* b_r, const void* packed_w,
                               uint16_t* y, const moe_route_out_t* route_out, void* ws,
                               size_t ws_bytes, void* stream, const moe_stage_events_t* ev) {
    if (plan == nullptr || ws == nullptr || W_r == nullptr || packed_w == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (T < 0 || T > plan->s.T_max) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (x == nullptr || y == nullptr)) return MOE_ERR_INVALID_ARG;
    if (route_out != nullptr) {
        const moe_status_t c = check_route_out(route_out);
        if (c != MOE_OK) return c;
    }
    if (!aligned16(ws) || !aligned16(W_r) || !aligned16(packed_w) || (x && !aligned16(x)) ||
        (y && !aligned16(y)) || (b_r && !aligned16(b_r)))
        return MOE_ERR_ALIGNMENT;
    if (ws_bytes < plan->ws_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
    int num_sms = 0;
    const moe_status_t ds = device_setup(&num_sms);
    if (ds != MOE_OK) return ds;

    const moe_shape_t& s = plan->s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const RoutePtrs r = route_ptrs(plan, ws, route_out);
    uint16_t* xs = at<uint16_t>(ws, plan->o_xs);
    uint16_t* h = at<uint16_t>(ws, plan->o_h);
    int32_t* status = at<int32_t>(ws, plan->o_status);
    auto mark = [&](void* e) -> bool {
        return e == nullptr || cudaEventRecord(static_cast<cudaEvent_t>(e), st) == cudaSuccess;
    };
    if (ev && !mark(ev->start)) return MOE_ERR_CUDA;
    if (moe::decode_supported(s, T)) {
        // a few tokens: one persistent kernel bound by reading the selected
        // experts' weights
        const uint8_t* wp = static_cast<const uint8_t*>(packed_w);
        moe::DecodeArgs da{};
        da.s = s;
        da.T = T;
        da.x = x;
        da.W_r = W_r;
        da.b_r = b_r;
        da.wpack_gu = wp;
        da.wpack_dn = wp + align_up(plan->gu_packed, 256);
        da.gu_block_bytes = plan->group_bytes;
        da.dn_block_bytes = plan->down_block_bytes;
        da.topk_idx = r.idx;
        da.topk_w = r.w;
        da.counts = r.counts;
        da.offsets = r.offsets;
        da.sorted_assign = r.sa;
        da.pos = r.pos;
        da.block_offsets = r.bo;
        da.block_map = r.bm;
        da.num_blocks = r.nb;
        da.h = h;
        da.y = y;
        da.status = status;
        da.sync = at<int32_t>(ws, plan->o_dsync);
        da.scratch = at<uint8_t>(ws, plan->o_dscr);
        MOE_CUDA(moe::launch_decode(da, num_sms, st));
        // one kernel: the stage events all mark its end
        if (ev && !(mark(ev->routed) && mark(ev->gate_up) && mark(ev->down) && mark(ev->end)))
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    moe_status_t rs = run_route(plan, T, x, W_r, b_r, r, ws, st);
    if (rs != MOE_OK) return rs;
    if (T == 0) {
        if (ev && !(mark(ev->routed) && mark(ev->gate_up) && mark(ev->down) && mark(ev->end)))
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    const int Tk = T * s.k;
    // step 5 (dispatch): token rows into expert order, so both GEMMs read
    // their token operand as dense 2-D TMA tiles (a TMA row gather of x
    // measured 2.6x slower in the gate/up GEMM)
    MOE_CUDA(moe::launch_dispatch(x, r.sa, Tk, s.k, s.d, xs, status, num_sms, st));
    if (ev && !mark(ev->routed)) return MOE_ERR_CUDA;

    const bool test_timeout = (s.flags & MOE_SHAPE_TEST_TIMEOUT) != 0;
    // the down outputs o reuse the storage of xs, which gate/up has finished reading
    const moe_status_t es = run_experts(plan, Tk, xs, r.bm, r.nb, max_blocks_for(s, T), packed_w, h, xs,
                                        status, test_timeout, num_sms, st,
                                        ev ? static_cast<cudaEvent_t>(ev->gate_up) : nullptr);
    if (es != MOE_OK) return es;
    if (ev && !mark(ev->down)) return MOE_ERR_CUDA;
    MOE_CUDA(moe::launch_combine(xs, r.pos, r.w, T, s.k, s.d, y, status, num_sms, st));
    if (ev && !mark(ev->end)) return MOE_ERR_CUDA;
    return MOE_OK;
}

moe_status_t moe_dispatch(const moe_plan_t* plan, int32_t T, const uint16_t* x,
                          const int32_t* sorted_assign, uint16_t* xs, void* ws, size_t ws_bytes,
                          void* stream) {
    if (plan == nullptr || ws == nullptr) return MOE_ERR_INVALID_ARG;
    if (T < 0 || T > plan->s.T_max) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (x == nullptr || sorted_assign == nullptr || xs == nullptr)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(ws) || (x && !aligned16(x)) || (sorted_assign && !aligned16(sorted_assign)) ||
        (xs && !aligned16(xs)))
        return MOE_ERR_ALIGNMENT;
    if (ws_bytes < plan->ws_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
    int num_sms = 0;
    const moe_status_t ds = device_setup(&num_sms);
    if (ds != MOE_OK) return ds;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* status = at<int32_t>(ws, plan->o_status);
    MOE_CUDA(cudaMemsetAsync(status, 0, 2 * sizeof(int32_t), st));
    if (T == 0) return MOE_OK;
    MOE_CUDA(moe::launch_dispatch(x, sorted_assign, T * plan->s.k, plan->s.k, plan->s.d, xs, status, num_sms, st));
    return MOE_OK;
}

moe_status_t moe_experts_forward(const moe_plan_t* plan, int32_t rows, const uint16_t* xs,
                                 const int32_t* block_map, const int32_t* num_blocks, int32_t max_blocks,
                                 const void* packed_w, uint16_t* o, void* ws, size_t ws_bytes,
                                 void* stream) {
    if (plan == nullptr || ws == nullptr || packed_w == nullptr) return MOE_ERR_INVALID_ARG;
    const moe_shape_t& s = plan->s;
    if (rows < 0 || static_cast<long long>(rows) > static_cast<long long>(s.T_max) * s.k)
        return MOE_ERR_INVALID_ARG;
    if (max_blocks < 0 || max_blocks > (1 << 24)) return MOE_ERR_INVALID_ARG;
    if (rows > 0 && (xs == nullptr || o == nullptr || block_map == nullptr || num_blocks == nullptr))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(ws) || !aligned16(packed_w) || (xs && !aligned16(xs)) || (o && !aligned16(o)) ||
        (block_map && !aligned16(block_map)) || (num_blocks && !aligned16(num_blocks)))
        return MOE_ERR_ALIGNMENT;
    if (ws_bytes < plan->ws_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
    int num_sms = 0;
    const moe_status_t ds = device_setup(&num_sms);
    if (ds != MOE_OK) return ds;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* status = at<int32_t>(ws, plan->o_status);
    if (rows == 0) {
        MOE_CUDA(cudaMemsetAsync(status, 0, 2 * sizeof(int32_t), st));
        return MOE_OK;
    }
    // the GEMMs read the checked entry count (0 if the map is out of range)
    int32_t* nb_checked = at<int32_t>(ws, plan->o_nb);
    MOE_CUDA(moe::launch_block_map_check(block_map, num_blocks, max_blocks, rows, s.E, kBlockT, nb_checked,
                                         status, st));
    return run_experts(plan, rows, xs, block_map, nb_checked, max_blocks, packed_w,
                       at<uint16_t>(ws, plan->o_h), o, status, false, num_sms, st, nullptr);
}

moe_status_t moe_combine(const moe_plan_t* plan, int32_t T, const uint16_t* o, const int32_t* pos,
                         const float* topk_w, uint16_t* y, void* ws, size_t ws_bytes, void* stream) {
    if (plan == nullptr || ws == nullptr) return MOE_ERR_INVALID_ARG;
    if (T < 0 || T > plan->s.T_max) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (o == nullptr || pos == nullptr || topk_w == nullptr || y == nullptr))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(ws) || (o && !aligned16(o)) || (pos && !aligned16(pos)) || (topk_w && !aligned16(topk_w)) ||
        (y && !aligned16(y)))
        return MOE_ERR_ALIGNMENT;
    if (ws_bytes < plan->ws_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
    int num_sms = 0;
    const moe_status_t ds = device_setup(&num_sms);
    if (ds != MOE_OK) return ds;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* status = at<int32_t>(ws, plan->o_status);
    MOE_CUDA(cudaMemsetAsync(status, 0, 2 * sizeof(int32_t), st));
    if (T == 0) return MOE_OK;
    MOE_CUDA(moe::launch_combine(o, pos, topk_w, T, plan->s.k, plan->s.d, y, status, num_sms, st));
    return MOE_OK;
}

moe_status_t moe_forward_host(const moe_plan_t* plan, int32_t T, const uint16_t* x_host,
                              const float* W_r, const float* b_r, const void* packed_w,
                              uint16_t* y_host, void* ws, size_t ws_bytes, void* stream) {
    if (plan == nullptr || ws == nullptr) return MOE_ERR_INVALID_ARG;
    if (T < 0 || T > plan->s.T_max) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (x_host == nullptr || y_host == nullptr)) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < plan->host_ws_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(ws)) return MOE_ERR_ALIGNMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint16_t* xd = at<uint16_t>(ws, plan->o_xstage);
    uint16_t* yd = at<uint16_t>(ws, plan->o_ystage);
    const size_t bytes = static_cast<size_t>(T) * plan->s.d * 2;
    if (bytes) MOE_CUDA(cudaMemcpyAsync(xd, x_host, bytes, cudaMemcpyHostToDevice, st));
    const moe_status_t r =
        moe_forward(plan, T, xd, W_r, b_r, packed_w, yd, nullptr, ws, plan->ws_bytes, stream);
    if (r != MOE_OK) return r;
    if (bytes) MOE_CUDA(cudaMemcpyAsync(y_host, yd, bytes, cudaMemcpyDeviceToHost, st));
    MOE_CUDA(cudaStreamSynchronize(st));
    return MOE_OK;
}

int moe_forward_path(const moe_plan_t* plan, int32_t T) {
    if (plan == nullptr || T < 0 || T > plan->s.T_max) return -1;
    if (moe::decode_supported(plan->s, T)) return 1;
    return moe::router_fast_supported(T, plan->s.d, plan->s.E) ? 2 : 0;
}

moe_status_t moe_read_status(const void* ws, int32_t* code, int32_t* detail, int32_t clear,
                             void* stream) {
    if (ws == nullptr || code == nullptr) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t h[2] = {0, 0};
    MOE_CUDA(cudaStreamSynchronize(st));
    MOE_CUDA(cudaMemcpy(h, ws, sizeof h, cudaMemcpyDeviceToHost));
    *code = h[0];
    if (detail) *detail = h[1];
    if (clear) MOE_CUDA(cudaMemset(const_cast<void*>(ws), 0, sizeof h));
    return MOE_OK;
}

}  // extern "C"
