// moe_route_noalloc: the routing steps for callers that cannot allocate
// device memory.
//
// Some callers of this library cannot call cudaMalloc: code that runs while
// a stream is being captured into a CUDA graph in a mode that forbids
// allocation, runtimes that hand out all device memory from their own pool
// and forbid side allocations, or plugin hosts that give a kernel only its
// input and output buffers.  moe_route needs a caller-provided workspace for
// its scratch (router logits, per-group expert histograms and scatter bases);
// this variant keeps that scratch in a fixed array inside the library
// instead, so the caller passes only inputs and outputs.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds kNoAllocScratchBytes of it until the process exits, and
// every call shares it.  Host code cannot use the array's name as a device
// address, so the first call on each device (with that device current) looks
// the address up once with cudaGetSymbolAddress and keeps it, and sets the
// routers' kernel attributes for every tiling; make that first call before
// any stream capture begins.
#include <atomic>
#include <mutex>

#include "moe_internal.h"

namespace {

// 4 MiB: enough for T * E * 4 bytes of logits plus two histograms of
// ceil(T / 256) * E counts, e.g. 8,000 tokens with 128 experts.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;

static __device__ __align__(256) unsigned char g_route_scratch[kNoAllocScratchBytes];

struct ScratchAddress {
    std::atomic<int> ready{0};
    void* ptr = nullptr;
    std::mutex lock;
};
ScratchAddress g_scratch_addr[64];

// Device address of g_route_scratch on the current device (looked up once).
moe_status_t scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    ScratchAddress& c = g_scratch_addr[dev];
    if (c.ready.load(std::memory_order_acquire) == 0) {
        std::lock_guard<std::mutex> guard(c.lock);
        if (c.ready.load(std::memory_order_relaxed) == 0) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr)
                return MOE_ERR_CUDA;
            // the routers' one-time kernel attributes, so that no later call
            // sets them inside a stream capture
            if (moe::prepare_router() != cudaSuccess || moe::prepare_router_fast() != cudaSuccess)
                return MOE_ERR_CUDA;
            c.ptr = p;
            c.ready.store(1, std::memory_order_release);
        }
    }
    *out = c.ptr;
    return MOE_OK;
}

size_t round256(size_t v) { return (v + 255) / 256 * 256; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" MOE_API moe_status_t moe_route_noalloc(const moe_plan_t* plan, int32_t T,
                                                  const uint16_t* x, const float* W_r,
                                                  const float* b_r, const moe_route_out_t* out,
                                                  void* stream) {
    if (plan == nullptr || out == nullptr || W_r == nullptr) return MOE_ERR_INVALID_ARG;
    if (T < 0 || T > plan->s.T_max) return MOE_ERR_INVALID_ARG;
    if (T > 0 && x == nullptr) return MOE_ERR_INVALID_ARG;
    const void* outs[] = {out->topk_idx, out->topk_w,        out->counts,    out->offsets,
                          out->sorted_assign, out->pos,      out->block_offsets, out->block_map,
                          out->num_blocks};
    for (const void* p : outs) {
        if (p == nullptr) return MOE_ERR_INVALID_ARG;
        if (!aligned16(p)) return MOE_ERR_ALIGNMENT;
    }
    if (!aligned16(W_r) || (x && !aligned16(x)) || (b_r && !aligned16(b_r)))
        return MOE_ERR_ALIGNMENT;

    // scratch layout: status word | logits [T, E] | histograms | scatter bases
    const moe_shape_t& s = plan->s;
    const int ng = (T + moe::kRouteGroupT - 1) / moe::kRouteGroupT;
    const size_t hist_n = static_cast<size_t>(ng > 0 ? ng : 1) * s.E;
    const size_t o_logits = 256;
    const size_t o_hist = o_logits + round256(static_cast<size_t>(T) * s.E * 4);
    const size_t o_gbase = o_hist + round256(hist_n * 4);
    const size_t need = o_gbase + round256(hist_n * 4);
    if (need > kNoAllocScratchBytes) return MOE_ERR_WORKSPACE_TOO_SMALL;

    void* base = nullptr;
    const moe_status_t st = scratch_address(&base);
    if (st != MOE_OK) return st;
    uint8_t* b = static_cast<uint8_t*>(base);
    int32_t* status = reinterpret_cast<int32_t*>(b);
    float* logits = reinterpret_cast<float*>(b + o_logits);
    int32_t* hist = reinterpret_cast<int32_t*>(b + o_hist);
    int32_t* gbase = reinterpret_cast<int32_t*>(b + o_gbase);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);

    // the logits kernel clears the histograms and the status word before
    // anything reads them, so stale contents of an earlier call do not leak
    if (moe::launch_router_logits(x, W_r, b_r, logits, T, s.d, s.E, hist,
                                  static_cast<int>(hist_n), status, cs) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (moe::launch_router_topk(logits, T, s.E, s.k, out->topk_idx, out->topk_w, hist, cs) !=
        cudaSuccess)
        return MOE_ERR_CUDA;
    if (moe::launch_route_scan(hist, ng, s.E, plan->block_t, out->counts, out->offsets, gbase,
                               out->block_offsets, out->block_map, out->num_blocks,
                               plan->max_blocks, status, cs) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (moe::launch_route_scatter(out->topk_idx, gbase, T, s.k, s.E, out->sorted_assign, out->pos,
                                  status, cs) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}
