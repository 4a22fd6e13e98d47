// route_static.cu -- moe_route_static: routing and permutation for callers that cannot allocate
// device memory.
//
// Some callers can't call cudaMalloc: code that runs inside a memory allocator or pool callback
// (it would re-enter the allocator), serving loops that forbid allocation after start-up
// (cudaMalloc may synchronise the device and stall every stream), and embedders whose device
// memory is reserved up front by another framework's caching allocator.  moe_plan allocates a
// small status word and moe_route needs a caller-sized workspace; this entry point needs
// neither.  Its scratch (the per-token row positions, per-chunk histograms and
// token-tile prefixes that moe_route keeps in the workspace) lives in one file-scope
// __device__ array of fixed size, which every GPU that loads this library holds until the
// process exits.
//
// Properties a caller must know:
//  * Capacity: T*k + ceil(T/256)*E + 2*(E+1) <= kStaticScratchInts (2^19 int32 = 2 MiB);
//    larger problems are rejected with MOE_ERR_UNSUPPORTED before any device work.
//  * The first call in a CUDA context (normally: on a device) looks up the array's device
//    address with cudaGetSymbolAddress (under a lock, with that device current) and keeps it
//    for the context; a call in a new context of the device (after cudaDeviceReset, say) looks
//    it up again.  Make the first call on each device before any stream capture.
//  * `stream` must belong to the current device (its context); a stream of another device is
//    rejected with MOE_ERR_INVALID_ARG, and the buffers must live on the current device too.
//  * Every call on a device shares the one array, and it keeps the previous call's contents.
//    Nothing in it needs to start at zero: each launch writes every entry it later reads.  Two
//    calls whose kernels overlap on the GPU (different streams, no ordering between them)
//    race on the array and give undefined results; serialise them.
//  * No cudaMalloc, cudaFree or allocating library routine is called.
#include "moe_internal.h"

#include <mutex>

namespace moe {

namespace {

constexpr size_t kStaticScratchInts = size_t(1) << 19;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) int32_t g_route_scratch[kStaticScratchInts];

struct ScratchSlot {
    unsigned long long ctx_id;  // context the address was looked up in (0: none yet)
    int32_t *ptr;
};
std::mutex g_scratch_mu;
ScratchSlot g_scratch[kMaxDevices] = {};

// Device address of g_route_scratch in the current context, after checking that `stream`
// belongs to that context.  Looked up once per context.
int scratch_for_current_context(cudaStream_t stream, int32_t **out)
{
    int dev = -1;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    int rc = current_context(&dev, &ctx, &id);
    if (rc != MOE_OK) return rc;
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    rc = stream_in_context(stream, ctx);  // a stream of another device or context is rejected
    if (rc != MOE_OK) return rc;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchSlot &slot = g_scratch[dev];
    if (slot.ctx_id != id || !slot.ptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess) return MOE_ERR_CUDA;
        slot.ptr = static_cast<int32_t *>(p);
        slot.ctx_id = id;
    }
    *out = slot.ptr;
    return MOE_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" int moe_route_static(int32_t T, int32_t E, int32_t k, const float *logits, int32_t *topk_idx,
                                float *topk_w, int32_t *counts, int32_t *offsets, int32_t *perm_tok,
                                moe_stream_t stream)
{
    if (T < 0 || E < 1 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
    if (E > kMaxE || k > kMaxK) return MOE_ERR_UNSUPPORTED;
    const size_t A = (size_t)T * (size_t)k;
    const size_t nch = ((size_t)T + kChunk - 1) / kChunk;
    const size_t need = A + nch * (size_t)E + 2 * ((size_t)E + 1);
    if (need > kStaticScratchInts) return MOE_ERR_UNSUPPORTED;  // beyond the fixed scratch
    if (!counts || !offsets || (T > 0 && (!logits || !topk_idx || !topk_w || !perm_tok))) return MOE_ERR_INVALID_ARG;
    if (!aligned16(logits) || !aligned16(topk_idx) || !aligned16(topk_w) || !aligned16(counts) ||
        !aligned16(offsets) || !aligned16(perm_tok))
        return MOE_ERR_INVALID_ARG;

    cudaStream_t s = (cudaStream_t)stream;
    int32_t *scratch = nullptr;
    const int rc = scratch_for_current_context(s, &scratch);
    if (rc != MOE_OK) return rc;

    RouteBufs b;
    b.topk_idx = topk_idx;
    b.topk_w = topk_w;
    b.counts = counts;
    b.offsets = offsets;
    b.perm_tok = perm_tok;
    b.pos = scratch;
    b.chunk_hist = scratch + A;
    b.ttile_a = b.chunk_hist + nch * (size_t)E;
    b.ttile_b = b.ttile_a + (E + 1);
    const long avg = ((long)T * k + E - 1) / E;
    const int bn = avg > 48 ? 64 : 32;
    cudaError_t e = launch_route(logits, T, E, k, topk_idx, topk_w, s);
    if (e == cudaSuccess) e = launch_permute(b, T, E, k, bn, bn, s);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
