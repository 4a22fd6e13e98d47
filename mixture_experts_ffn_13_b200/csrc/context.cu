// context.cu -- which CUDA context a call runs in, and kernel attributes set once per context.
//
// The driver entry points are taken through the runtime (cudaGetDriverEntryPointByVersion), so
// the library links only libcudart.  A context's id (cuCtxGetId) is unique for the life of the
// process: a context created after cudaDeviceReset gets a new id, so anything cached under the
// old id is looked up or set again.
#include "moe_internal.h"

#include <cudaTypedefs.h>

#include <mutex>

namespace moe {

namespace {

PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;
PFN_cuStreamGetCtx_v9020 g_stream_ctx = nullptr;
std::once_flag g_driver_once;

void load_driver()
{
    auto get = [](const char *name, unsigned ver) -> void * {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion(name, &fn, ver, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return fn;
    };
    g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(get("cuCtxGetCurrent", 4000));
    g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(get("cuCtxGetId", 12000));
    g_stream_ctx = reinterpret_cast<PFN_cuStreamGetCtx_v9020>(get("cuStreamGetCtx", 9020));
}

struct AttrEntry {
    unsigned long long ctx_id;
    const void *func;
    int smem;
};
constexpr int kMaxAttrEntries = 512;
std::mutex g_attr_mu;
AttrEntry g_attr[kMaxAttrEntries];
int g_attr_n = 0;

}  // namespace

int current_context(int *dev, CUcontext *ctx, unsigned long long *id)
{
    std::call_once(g_driver_once, load_driver);
    if (!g_ctx_current || !g_ctx_id || !g_stream_ctx) return MOE_ERR_CUDA;
    if (cudaGetDevice(dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (g_ctx_current(ctx) != CUDA_SUCCESS) return MOE_ERR_CUDA;
    if (!*ctx) {  // no context yet on this thread: cudaSetDevice makes the primary context current
        if (cudaSetDevice(*dev) != cudaSuccess || g_ctx_current(ctx) != CUDA_SUCCESS || !*ctx) return MOE_ERR_CUDA;
    }
    if (g_ctx_id(*ctx, id) != CUDA_SUCCESS) return MOE_ERR_CUDA;
    return MOE_OK;
}

int stream_in_context(cudaStream_t s, CUcontext ctx)
{
    std::call_once(g_driver_once, load_driver);
    if (!g_stream_ctx) return MOE_ERR_CUDA;
    CUcontext sctx = nullptr;
    if (g_stream_ctx(reinterpret_cast<CUstream>(s), &sctx) != CUDA_SUCCESS) return MOE_ERR_INVALID_ARG;
    return sctx == ctx ? MOE_OK : MOE_ERR_INVALID_ARG;
}

cudaError_t set_smem_limit(const void *func, int smem)
{
    int dev = -1;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (current_context(&dev, &ctx, &id) != MOE_OK)  // no context id: set it every time
        return cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    std::lock_guard<std::mutex> lock(g_attr_mu);
    for (int i = 0; i < g_attr_n; ++i)
        if (g_attr[i].ctx_id == id && g_attr[i].func == func && g_attr[i].smem >= smem) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    for (int i = 0; i < g_attr_n; ++i)
        if (g_attr[i].ctx_id == id && g_attr[i].func == func) {
            g_attr[i].smem = smem;
            return e;
        }
    if (g_attr_n < kMaxAttrEntries) g_attr[g_attr_n++] = AttrEntry{id, func, smem};
    return e;
}

}  // namespace moe
