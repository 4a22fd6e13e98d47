// moe_abi.cu -- the C ABI (include/moe_b200.h): plan validation, workspace carving, tensor-map
// encoding and the launch sequence of one layer call.  Host code only.
#include "moe_internal.h"

#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <new>

struct moe_plan_s {
    moe_dims d;
    int device;
    int num_sms;
    int *d_status;  // device status word (4 ints), allocated by moe_plan
    int last_cuda_error;
    size_t ws_bytes;
    int launches;             // kernels launched by the last route/forward call
    bool checked = false;     // checked mode (moe_set_checked): device-side argument checks
    bool prof;                // stage events enabled
    bool prof_recorded;       // the last forward recorded them
    cudaEvent_t ev[8];        // stage boundaries 0..7
};

namespace moe {

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

int nb512(int K) { return (K + kBlockK - 1) / kBlockK; }

// Byte offsets of every workspace buffer for a token count of Tm (the plan's T_max).
struct Layout {
    size_t topk_idx, topk_w, counts, offsets, perm, pos, chunk_hist, ttile_a, ttile_b;
    size_t act, act_scale;       // permuted activations (+ scales for FP8)
    size_t h, h_sh;              // gate|up output, routed / shared
    size_t hq, hq_sh, sh, sh_sh; // quantised h (FP8)
    size_t y;                    // down output rows (routed then shared), fp32
    size_t lg;                   // router logits [T, E] fp32 (moe_forward_x): inside y when they fit
    size_t small;                // the small-batch kernel's partial sums, y rows and barrier
    size_t total;
};

Layout make_layout(const moe_dims &d)
{
    const size_t Tm = (size_t)d.T_max, k = (size_t)d.k, E = (size_t)d.E;
    const size_t H = (size_t)d.H, I = (size_t)d.I, Is = (size_t)d.I_shared;
    const size_t A = Tm * k;
    const size_t R = A + (Is > 0 ? Tm : 0);
    const size_t nch = (Tm + kChunk - 1) / kChunk;
    const bool fp8 = d.wfmt == MOE_W_FP8_SC512;
    Layout L{};
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align_up(o + std::max<size_t>(bytes, 1));
        return at;
    };
    L.topk_idx = take(A * 4);
    L.topk_w = take(A * 4);
    L.counts = take(E * 4);
    L.offsets = take((E + 1) * 4);
    L.perm = take(A * 4);
    L.pos = take(A * 4);
    L.chunk_hist = take(nch * E * 4);
    L.ttile_a = take((E + 1) * 4);
    L.ttile_b = take((E + 1) * 4);
    if (fp8) {
        L.act = take(R * H);
        L.act_scale = take(R * nb512(d.H) * 4);
        L.h = take(A * I * 4);
        L.h_sh = take(Tm * Is * 4);
        L.hq = take(A * I);
        L.hq_sh = take(Tm * Is);
        L.sh = take(A * nb512(d.I) * 4);
        L.sh_sh = take(Tm * nb512(d.I_shared) * 4);
    } else {
        L.act = take(R * H * 2);
        L.act_scale = 0;
        L.h = take(A * I * 2);
        L.h_sh = take(Tm * Is * 2);
        L.hq = L.hq_sh = L.sh = L.sh_sh = 0;
    }
    L.y = take(R * H * 4);
    // moe_forward_x's logits are read only by the route kernel, the first kernel of the
    // forward, and y is written by the down GEMM later on the same stream, so they share y's
    // bytes unless they do not fit there
    L.lg = Tm * E <= R * H ? L.y : take(Tm * E * 4);
    L.small = fp8 ? take(small_batch_workspace(d)) : 0;
    L.total = o;
    return L;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

void load_encode()
{
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int fail_cuda(moe_plan_t *p, cudaError_t e)
{
    p->last_cuda_error = (int)e;
    return MOE_ERR_CUDA;
}

// Tile size along the token dimension from the mean rows per expert group: decode-sized
// groups take 32-row tiles; larger groups take wider tiles so each weight tile staged in
// shared memory feeds more MMA work (the 4-bit kernel stops at 64).
int pick_bn(int T, int k, int E, bool fp8)
{
    const long avg = ((long)T * k + E - 1) / E;
    if (avg <= 48) return fp8 || avg <= 24 ? 32 : 64;
    if (!fp8) return 96;  // 4-bit: one tile per group up to ~1.5x the mean (dequant is per tile)
    return avg <= 96 ? 64 : 192;  // 192: one pass over each weight tile for groups up to 192 rows
    // (the FP8 GEMM also builds 128- and 160-row tiles; both measured slower at prefill, 3.88 and
    // 3.69 against 3.37 ms, and are not picked)
}

}  // namespace

int encode_map_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes, uint64_t inner,
                  uint64_t outer, uint32_t box_inner, uint32_t box_outer, bool swizzle128)
{
    std::call_once(g_encode_once, load_encode);
    if (!g_encode) return MOE_ERR_CUDA;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner * (uint64_t)elem_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE,
                                swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

int encode_map_gateup_ilv(CUtensorMap *map, const void *gate, const void *up, uint64_t K, uint64_t rows, int *up_lo)
{
    std::call_once(g_encode_once, load_encode);
    if (!g_encode) return MOE_ERR_CUDA;
    const uintptr_t g = reinterpret_cast<uintptr_t>(gate), u = reinterpret_cast<uintptr_t>(up);
    const bool lo_up = u < g;
    const uintptr_t base = lo_up ? u : g, dist = lo_up ? g - u : u - g;
    if (dist == 0 || dist % 16 || dist >= (uint64_t(1) << 40) || rows % 64 || K % 16) return MOE_ERR_UNSUPPORTED;
    const cuuint64_t dims[4] = {K, 16, 2, rows / 16};
    const cuuint64_t strides[3] = {K, dist, 16 * K};
    const cuuint32_t box[4] = {128, 16, 2, 4};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, reinterpret_cast<void *>(base), dims, strides,
                                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return MOE_ERR_UNSUPPORTED;
    *up_lo = lo_up ? 1 : 0;
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

const char *moe_strerror(int code)
{
    switch (code) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
        case MOE_ERR_BOUNDS: return "MOE_ERR_BOUNDS";
        default: return "MOE_ERR_UNKNOWN";
    }
}

int moe_plan(const moe_dims *dims, moe_plan_t **out_plan, size_t *workspace_bytes)
{
    if (!dims || !out_plan || !workspace_bytes) return MOE_ERR_INVALID_ARG;
    *out_plan = nullptr;
    const moe_dims d = *dims;
    if (d.T_max < 1 || d.H < 1 || d.E < 1 || d.I < 1 || d.k < 1 || d.I_shared < 0) return MOE_ERR_INVALID_ARG;
    if (d.wfmt < MOE_W_FP8_SC512 || d.wfmt > MOE_W_NVFP4_G16) return MOE_ERR_INVALID_ARG;
    if (d.k > d.E) return MOE_ERR_INVALID_ARG;
    if (d.E > kMaxE || d.k > kMaxK || d.T_max > (1 << 20)) return MOE_ERR_UNSUPPORTED;
    if (d.H % 128 || d.I % 128 || d.I_shared % 128) return MOE_ERR_UNSUPPORTED;
    if (d.H > 8192 || d.I > 8192 || d.I_shared > 8192) return MOE_ERR_UNSUPPORTED;
    // 32-bit row arithmetic inside the kernels
    if ((long long)d.E * std::max(d.I, d.H) >= (1ll << 31) ||
        (long long)d.T_max * (d.k + 1) * std::max(d.I, d.H) >= (1ll << 40))
        return MOE_ERR_UNSUPPORTED;
    moe_plan_t *p = new (std::nothrow) moe_plan_s();
    if (!p) return MOE_ERR_INVALID_ARG;
    p->d = d;
    cudaError_t e = cudaGetDevice(&p->device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&p->num_sms, cudaDevAttrMultiProcessorCount, p->device);
    if (e == cudaSuccess) e = cudaMalloc(&p->d_status, 4 * sizeof(int));
    if (e == cudaSuccess) e = cudaMemset(p->d_status, 0, 4 * sizeof(int));
    if (e != cudaSuccess) {
        if (p->d_status) cudaFree(p->d_status);
        delete p;
        return MOE_ERR_CUDA;
    }
    p->ws_bytes = make_layout(d).total;
    *workspace_bytes = p->ws_bytes;
    *out_plan = p;
    return MOE_OK;
}

void moe_destroy(moe_plan_t *p)
{
    if (!p) return;
    if (p->prof)
        for (cudaEvent_t &e : p->ev) cudaEventDestroy(e);
    if (p->d_status) cudaFree(p->d_status);
    delete p;
}

static const char *kStageNames[7] = {"route", "permute", "quant_x", "gemm_gateup", "quant_h", "gemm_down", "combine"};

const char *moe_profile_stage_name(int i) { return (i >= 0 && i < 7) ? kStageNames[i] : nullptr; }

int moe_launch_count(const moe_plan_t *p) { return p ? p->launches : 0; }

int moe_set_checked(moe_plan_t *p, int enable)
{
    if (!p) return MOE_ERR_INVALID_ARG;
    p->checked = enable != 0;
    return MOE_OK;
}

int moe_profile_enable(moe_plan_t *p, int enable)
{
    if (!p) return MOE_ERR_INVALID_ARG;
    if (enable && !p->prof) {
        for (int i = 0; i < 8; ++i) {
            const cudaError_t e = cudaEventCreate(&p->ev[i]);
            if (e != cudaSuccess) {
                for (int j = 0; j < i; ++j) cudaEventDestroy(p->ev[j]);
                return fail_cuda(p, e);
            }
        }
        p->prof = true;
    } else if (!enable && p->prof) {
        for (cudaEvent_t &e : p->ev) cudaEventDestroy(e);
        p->prof = false;
    }
    p->prof_recorded = false;
    return MOE_OK;
}

int moe_profile_read(moe_plan_t *p, float *ms, int max_stages)
{
    if (!p || !ms || max_stages < 0 || !p->prof || !p->prof_recorded) return MOE_ERR_INVALID_ARG;
    const int n = std::min(max_stages, 7);
    cudaError_t e = cudaEventSynchronize(p->ev[7]);
    for (int i = 0; i < n && e == cudaSuccess; ++i) e = cudaEventElapsedTime(&ms[i], p->ev[i], p->ev[i + 1]);
    if (e != cudaSuccess) return fail_cuda(p, e);
    return n;
}

int moe_last_cuda_error(const moe_plan_t *p) { return p ? p->last_cuda_error : 0; }

int moe_get_status(moe_plan_t *p, moe_stream_t stream)
{
    if (!p) return MOE_ERR_INVALID_ARG;
    int h[4] = {0, 0, 0, 0};
    cudaError_t e = cudaMemcpyAsync(h, p->d_status, sizeof(h), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e == cudaSuccess && h[0] != 0) e = cudaMemsetAsync(p->d_status, 0, sizeof(h), (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return fail_cuda(p, e);
    return h[0];
}

static int check_ws(const moe_plan_t *p, void *ws, size_t ws_bytes)
{
    if (!ws || ws_bytes < p->ws_bytes) return MOE_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) % kAlign) return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

static RouteBufs route_bufs(const Layout &L, uint8_t *ws)
{
    RouteBufs b;
    b.topk_idx = reinterpret_cast<int32_t *>(ws + L.topk_idx);
    b.topk_w = reinterpret_cast<float *>(ws + L.topk_w);
    b.counts = reinterpret_cast<int32_t *>(ws + L.counts);
    b.offsets = reinterpret_cast<int32_t *>(ws + L.offsets);
    b.perm_tok = reinterpret_cast<int32_t *>(ws + L.perm);
    b.pos = reinterpret_cast<int32_t *>(ws + L.pos);
    b.chunk_hist = reinterpret_cast<int32_t *>(ws + L.chunk_hist);
    b.ttile_a = reinterpret_cast<int32_t *>(ws + L.ttile_a);
    b.ttile_b = reinterpret_cast<int32_t *>(ws + L.ttile_b);
    return b;
}

int moe_router_logits(moe_plan_t *p, int32_t T, const uint16_t *x, const uint16_t *w_router, float *logits,
                      moe_stream_t stream)
{
    if (!p) return MOE_ERR_INVALID_ARG;
    if (T < 0 || T > p->d.T_max) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !w_router || !logits)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_router) || !aligned16(logits)) return MOE_ERR_INVALID_ARG;
    p->launches = 0;
    if (T == 0) return MOE_OK;
    const cudaError_t e =
        launch_router_gemm(x, w_router, logits, T, p->d.H, p->d.E, p->d_status, p->num_sms, (cudaStream_t)stream);
    if (e != cudaSuccess) return fail_cuda(p, e);
    p->launches = 1;
    return MOE_OK;
}

int moe_router_topk(moe_plan_t *p, int32_t T, const uint16_t *x, const uint16_t *w_router, float *logits,
                    int32_t *topk_idx, float *topk_w, moe_stream_t stream)
{
    if (!p) return MOE_ERR_INVALID_ARG;
    if (T < 0 || T > p->d.T_max) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !w_router || !logits || !topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_router) || !aligned16(logits) || !aligned16(topk_idx) || !aligned16(topk_w))
        return MOE_ERR_INVALID_ARG;
    p->launches = 0;
    if (T == 0) return MOE_OK;
    const cudaError_t e = launch_router_topk(x, w_router, logits, topk_idx, topk_w, T, p->d.H, p->d.E, p->d.k,
                                             p->d_status, p->num_sms, (cudaStream_t)stream);
    if (e != cudaSuccess) return fail_cuda(p, e);
    p->launches = 2;
    return MOE_OK;
}

int moe_route(moe_plan_t *p, int32_t T, const float *logits, int32_t *topk_idx, float *topk_w, int32_t *counts,
              int32_t *offsets, int32_t *perm_tok, void *workspace, size_t ws_bytes, moe_stream_t stream)
{
    if (!p) return MOE_ERR_INVALID_ARG;
    if (T < 0 || T > p->d.T_max) return MOE_ERR_INVALID_ARG;
    if (!counts || !offsets || (T > 0 && (!logits || !topk_idx || !topk_w || !perm_tok))) return MOE_ERR_INVALID_ARG;
    if (!aligned16(logits) || !aligned16(topk_idx) || !aligned16(topk_w) || !aligned16(counts) ||
        !aligned16(offsets) || !aligned16(perm_tok))
        return MOE_ERR_INVALID_ARG;
    int rc = check_ws(p, workspace, ws_bytes);
    if (rc) return rc;
    const moe_dims &d = p->d;
    const Layout L = make_layout(d);
    RouteBufs b = route_bufs(L, static_cast<uint8_t *>(workspace));
    b.topk_idx = topk_idx;
    b.topk_w = topk_w;
    b.counts = counts;
    b.offsets = offsets;
    b.perm_tok = perm_tok;
    cudaStream_t s = (cudaStream_t)stream;
    const int bn = pick_bn(T, d.k, d.E, d.wfmt == MOE_W_FP8_SC512);
    p->launches = 0;
    cudaError_t e = launch_route_permute(logits, b, T, d.E, d.k, bn, bn, s, p->checked ? p->d_status : nullptr);
    p->launches = route_permute_launches(T, d.E, d.k);
    return e == cudaSuccess ? MOE_OK : fail_cuda(p, e);
}

// The 4-bit layer (int4, MXFP4 or NVFP4): route, permute, gather bf16 rows, 4-bit gate|up
// (h in bf16), 4-bit down, combine.  Stage events: 0 route | 1 permute | 2 gather | 3 gate|up |
// 4 (no h quantiser) | 5 down | 6 combine | 7.
static int forward_w4(moe_plan_t *p, int T, const uint16_t *x, const float *logits, const moe_weights *w,
                        uint16_t *out, uint8_t *ws, cudaStream_t s)
{
    const moe_dims &d = p->d;
    auto mark = [&](int i) {
        if (p->prof) cudaEventRecord(p->ev[i], s);
    };
    const Layout L = make_layout(d);
    const RouteBufs b = route_bufs(L, ws);
    const int H = d.H, I = d.I, Is = d.I_shared, k = d.k, E = d.E;
    const bool shared = Is > 0;
    const int A = T * k;
    const int bn = pick_bn(T, k, E, false);
    mark(0);
    int *chk = p->checked ? p->d_status : nullptr;
    cudaError_t e = launch_route(logits, T, E, k, b.topk_idx, b.topk_w, s, chk);
    mark(1);
    if (e == cudaSuccess) e = launch_permute_any(b, T, E, k, bn, bn, s);
    mark(2);
    if (e != cudaSuccess) return fail_cuda(p, e);
    uint16_t *xp = reinterpret_cast<uint16_t *>(ws + L.act);
    uint16_t *xp_sh = shared ? xp + (size_t)A * H : nullptr;
    e = launch_gather_x_bf16(x, T, H, k, b.pos, xp, xp_sh, d.wfmt == MOE_W_INT4_G128, s);
    mark(3);
    if (e != cudaSuccess) return fail_cuda(p, e);

    uint16_t *h = reinterpret_cast<uint16_t *>(ws + L.h);
    uint16_t *h_sh = reinterpret_cast<uint16_t *>(ws + L.h_sh);
    float *y = reinterpret_cast<float *>(ws + L.y);
    float *y_sh = shared ? y + (size_t)A * H : nullptr;
    const CUtensorMapDataType U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8, BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;

    GemmMaps mg{};
    GemmArgs ag{};
    ag.nseg = shared ? 2 : 1;
    ag.E = E;
    ag.T = T;
    ag.offsets = b.offsets;
    ag.ttile = b.ttile_a;
    ag.status = p->d_status;
    ag.timeout_ns = kDefaultTimeoutNs;
    ag.seg[0] = GemmSeg{I, H, A, w->s_gate, w->s_up, nullptr, h};
    ag.seg[0].ts0 = w->t_gate;
    ag.seg[0].ts1 = w->t_up;
    int rc = encode_map_2d(&mg.a0[0], w->w_gate, U8, 1, H / 2, (uint64_t)E * I, 128, 128, true);
    rc |= encode_map_2d(&mg.a1[0], w->w_up, U8, 1, H / 2, (uint64_t)E * I, 128, 128, true);
    rc |= encode_map_2d(&mg.b[0], xp, BF, 2, H, A, 64, bn, true);
    if (shared) {
        ag.seg[1] = GemmSeg{Is, H, T, w->ss_gate, w->ss_up, nullptr, h_sh};
        ag.seg[1].ts0 = w->ts_gate;
        ag.seg[1].ts1 = w->ts_up;
        rc |= encode_map_2d(&mg.a0[1], w->ws_gate, U8, 1, H / 2, Is, 128, 128, true);
        rc |= encode_map_2d(&mg.a1[1], w->ws_up, U8, 1, H / 2, Is, 128, 128, true);
        rc |= encode_map_2d(&mg.b[1], xp_sh, BF, 2, H, T, 64, bn, true);
    }
    if (rc) return MOE_ERR_CUDA;
    e = launch_gemm_w4(true, d.wfmt, bn, mg, ag, p->num_sms, s);
    mark(4);
    mark(5);
    if (e != cudaSuccess) return fail_cuda(p, e);

    GemmMaps md{};
    GemmArgs ad = ag;
    ad.ttile = b.ttile_b;
    ad.seg[0] = GemmSeg{H, I, A, w->s_down, nullptr, nullptr, y};
    ad.seg[0].ts0 = w->t_down;
    rc = encode_map_2d(&md.a0[0], w->w_down, U8, 1, I / 2, (uint64_t)E * H, 128, 128, true);
    rc |= encode_map_2d(&md.b[0], h, BF, 2, I, A, 64, bn, true);
    if (shared) {
        ad.seg[1] = GemmSeg{H, Is, T, w->ss_down, nullptr, nullptr, y_sh};
        ad.seg[1].ts0 = w->ts_down;
        rc |= encode_map_2d(&md.a0[1], w->ws_down, U8, 1, Is / 2, H, 128, 128, true);
        rc |= encode_map_2d(&md.b[1], h_sh, BF, 2, Is, T, 64, bn, true);
    }
    if (rc) return MOE_ERR_CUDA;
    e = launch_gemm_w4(false, d.wfmt, bn, md, ad, p->num_sms, s);
    mark(6);
    if (e != cudaSuccess) return fail_cuda(p, e);
    e = launch_combine(y, y_sh, b.pos, b.topk_w, T, H, k, out, s, chk);
    mark(7);
    if (e != cudaSuccess) return fail_cuda(p, e);
    p->launches = route_permute_launches(T, E, k) + 1 + 1 + 1 + 1;
    p->prof_recorded = p->prof;
    return MOE_OK;
}

// Weight pointers present (the shared expert's when I_shared > 0, the tensor scales for NVFP4)
// and 16-byte aligned.
static int check_weights(const moe_plan_t *p, const moe_weights *w)
{
    if (!w->w_gate || !w->w_up || !w->w_down || !w->s_gate || !w->s_up || !w->s_down) return MOE_ERR_INVALID_ARG;
    if (p->d.I_shared > 0 &&
        (!w->ws_gate || !w->ws_up || !w->ws_down || !w->ss_gate || !w->ss_up || !w->ss_down))
        return MOE_ERR_INVALID_ARG;
    const void *ptrs[] = {w->w_gate, w->w_up, w->w_down, w->s_gate, w->s_up, w->s_down,
                          w->ws_gate, w->ws_up, w->ws_down, w->ss_gate, w->ss_up, w->ss_down};
    for (const void *q : ptrs)
        if (!aligned16(q)) return MOE_ERR_INVALID_ARG;
    if (p->d.wfmt == MOE_W_NVFP4_G16) {  // the tensor scales are read for NVFP4 only
        if (!w->t_gate || !w->t_up || !w->t_down) return MOE_ERR_INVALID_ARG;
        if (p->d.I_shared > 0 && (!w->ts_gate || !w->ts_up || !w->ts_down)) return MOE_ERR_INVALID_ARG;
        const void *ts[] = {w->t_gate, w->t_up, w->t_down, w->ts_gate, w->ts_up, w->ts_down};
        for (const void *q : ts)
            if (!aligned16(q)) return MOE_ERR_INVALID_ARG;
    }
    return MOE_OK;
}

int moe_forward(moe_plan_t *p, int32_t T, const uint16_t *x, const float *logits, const moe_weights *w,
                uint16_t *out, void *workspace, size_t ws_bytes, moe_stream_t stream)
{
    if (!p || !w) return MOE_ERR_INVALID_ARG;
    const moe_dims &d = p->d;
    if (T < 0 || T > d.T_max) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !logits || !out)) return MOE_ERR_INVALID_ARG;
    const bool shared = d.I_shared > 0;
    if (check_weights(p, w) != MOE_OK) return MOE_ERR_INVALID_ARG;
    const void *ptrs[] = {x, logits, out};
    for (const void *q : ptrs)
        if (!aligned16(q)) return MOE_ERR_INVALID_ARG;
    int rc = check_ws(p, workspace, ws_bytes);
    if (rc) return rc;
    p->launches = 0;
    p->prof_recorded = false;
    if (T == 0) return MOE_OK;

    cudaStream_t s = (cudaStream_t)stream;
    auto mark = [&](int i) {
        if (p->prof) cudaEventRecord(p->ev[i], s);
    };
    if (d.wfmt != MOE_W_FP8_SC512) return forward_w4(p, T, x, logits, w, out, static_cast<uint8_t *>(workspace), s);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const Layout L = make_layout(d);
    // small batches: the whole layer in one kernel (checked mode keeps the regular path, whose
    // kernels carry the device-side checks); the whole call is reported as stage 3
    if (!p->checked && small_batch_fits(T, d)) {
        int launched = 0;
        for (int i = 0; i <= 3; ++i) mark(i);
        const cudaError_t es =
            launch_small_batch(d, T, x, logits, w, out, ws + L.small, p->d_status, p->num_sms, s, &launched);
        if (es == cudaSuccess) {
            for (int i = 4; i <= 7; ++i) mark(i);
            p->launches = 1;
            p->prof_recorded = p->prof;
            return MOE_OK;
        }
        if (launched || es != cudaErrorNotSupported) return fail_cuda(p, es);
        // gate and up weights too far apart for the small kernel's tensor map: regular path
    }
    const RouteBufs b = route_bufs(L, ws);
    const int H = d.H, I = d.I, Is = d.I_shared, k = d.k, E = d.E;
    const int A = T * k;
    const int bn_b = pick_bn(T, k, E, true);
    // gate|up: narrow tiles pair the gate and up tiles (two accumulators per column); 192-row
    // tiles interleave 64 gate and 64 up rows in one 128-row MMA tile
    const int bn_a = bn_b;
    const bool ilv = bn_a > 64;
    const uint32_t wbox = ilv ? 16 : 128;  // weight rows per TMA box (2-D maps)
    const uint32_t kXBox = bn_a;  // activation rows per TMA box: the whole token tile

    // When nearly every expert is picked (T*k >= 2E: each misses with probability < e^-2), the
    // gate|up GEMM's first wave of work items is the leading experts' weight tiles (items run
    // expert by expert).  The route kernel asks L2 for the first ~96 MB of them, so that part of
    // the weight stream overlaps routing, permutation and quantisation instead of following them.
    WeightPrefetch pf;
    if ((int64_t)T * k >= 2 * (int64_t)E && aligned16(w->w_gate) && aligned16(w->w_up)) {
        const size_t per_expert = (size_t)I * H;
        const size_t budget = 48u << 20;  // per matrix
        const size_t n_exp = std::min<size_t>((size_t)E, budget / per_expert);
        pf.a = static_cast<const uint8_t *>(w->w_gate);
        pf.b = static_cast<const uint8_t *>(w->w_up);
        pf.chunks = (uint32_t)(n_exp * per_expert / WeightPrefetch::kChunk);
    }
    mark(0);
    int *chk = p->checked ? p->d_status : nullptr;
    cudaError_t e = launch_route(logits, T, E, k, b.topk_idx, b.topk_w, s, chk, pf);
    mark(1);
    if (e == cudaSuccess) e = launch_permute_any(b, T, E, k, bn_a, bn_b, s);
    mark(2);
    if (e != cudaSuccess) return fail_cuda(p, e);

    // A2: quantise x into permuted rows [0, A) and shared rows [A, A + T)
    uint8_t *xq = ws + L.act;
    float *sx = reinterpret_cast<float *>(ws + L.act_scale);
    const int nbH = nb512(H);
    uint8_t *xq_sh = shared ? xq + (size_t)A * H : nullptr;
    float *sx_sh = shared ? sx + (size_t)A * nbH : nullptr;
    e = launch_quant_x_fp8(x, T, H, k, b.pos, xq, sx, xq_sh, sx_sh, s);
    mark(3);
    if (e != cudaSuccess) return fail_cuda(p, e);

    float *h = reinterpret_cast<float *>(ws + L.h);
    float *h_sh = reinterpret_cast<float *>(ws + L.h_sh);
    uint8_t *hq = ws + L.hq, *hq_sh = ws + L.hq_sh;
    float *sh = reinterpret_cast<float *>(ws + L.sh), *sh_sh = reinterpret_cast<float *>(ws + L.sh_sh);
    float *y = reinterpret_cast<float *>(ws + L.y);
    float *y_sh = shared ? y + (size_t)A * H : nullptr;
    const CUtensorMapDataType U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;

    // A4: gate|up
    GemmMaps mg{};
    GemmArgs ag{};
    ag.nseg = shared ? 2 : 1;
    ag.E = E;
    ag.T = T;
    ag.offsets = b.offsets;
    ag.ttile = b.ttile_a;
    ag.status = p->d_status;
    ag.timeout_ns = kDefaultTimeoutNs;
    ag.seg[0] = GemmSeg{I, H, A, w->s_gate, w->s_up, sx, h};
    // interleaved tiles load gate and up rows with one 4-D map where the two weight arrays'
    // distance allows it, else with 16-row boxes of two 2-D maps
    auto gateup_maps = [&](GemmSeg &sg, CUtensorMap &m0, CUtensorMap &m1, const void *wg, const void *wu,
                           uint64_t rows) {
        if (ilv && encode_map_gateup_ilv(&m0, wg, wu, H, rows, &sg.up_lo) == MOE_OK) {
            sg.ilv4d = 1;
            return 0;
        }
        return encode_map_2d(&m0, wg, U8, 1, H, rows, 128, wbox, true) |
               encode_map_2d(&m1, wu, U8, 1, H, rows, 128, wbox, true);
    };
    rc = gateup_maps(ag.seg[0], mg.a0[0], mg.a1[0], w->w_gate, w->w_up, (uint64_t)E * I);
    rc |= encode_map_2d(&mg.b[0], xq, U8, 1, H, A, 128, kXBox, true);
    if (shared) {
        ag.seg[1] = GemmSeg{Is, H, T, w->ss_gate, w->ss_up, sx_sh, h_sh};
        rc |= gateup_maps(ag.seg[1], mg.a0[1], mg.a1[1], w->ws_gate, w->ws_up, (uint64_t)Is);
        rc |= encode_map_2d(&mg.b[1], xq_sh, U8, 1, H, T, 128, kXBox, true);
    }
    if (rc) return MOE_ERR_CUDA;
    e = launch_gemm_fp8(true, bn_a, mg, ag, p->num_sms, s);
    mark(4);
    if (e != cudaSuccess) return fail_cuda(p, e);

    // quantise h per (row, 512-block)
    e = launch_quant_rows_fp8(h, A, I, hq, sh, shared ? h_sh : nullptr, T, Is, hq_sh, sh_sh, s);
    mark(5);
    if (e != cudaSuccess) return fail_cuda(p, e);

    // A5: down
    GemmMaps md{};
    GemmArgs ad = ag;
    ad.ttile = b.ttile_b;
    ad.seg[0] = GemmSeg{H, I, A, w->s_down, nullptr, sh, y};
    const uint32_t kHBox = bn_b;  // the whole token tile per TMA box
    rc = encode_map_2d(&md.a0[0], w->w_down, U8, 1, I, (uint64_t)E * H, 128, 128, true);
    rc |= encode_map_2d(&md.b[0], hq, U8, 1, I, A, 128, kHBox, true);
    if (shared) {
        ad.seg[1] = GemmSeg{H, Is, T, w->ss_down, nullptr, sh_sh, y_sh};
        rc |= encode_map_2d(&md.a0[1], w->ws_down, U8, 1, Is, H, 128, 128, true);
        rc |= encode_map_2d(&md.b[1], hq_sh, U8, 1, Is, T, 128, kHBox, true);
    }
    if (rc) return MOE_ERR_CUDA;
    e = launch_gemm_fp8(false, bn_b, md, ad, p->num_sms, s);
    mark(6);
    if (e != cudaSuccess) return fail_cuda(p, e);

    // A6: combine
    e = launch_combine(y, y_sh, b.pos, b.topk_w, T, H, k, out, s, chk);
    mark(7);
    if (e != cudaSuccess) return fail_cuda(p, e);
    p->launches = route_permute_launches(T, E, k) + 1 + 1 + 1 + 1 + 1;
    p->prof_recorded = p->prof;
    return MOE_OK;
}

int moe_forward_x(moe_plan_t *p, int32_t T, const uint16_t *x, const uint16_t *w_router, const moe_weights *w,
                  uint16_t *out, void *workspace, size_t ws_bytes, moe_stream_t stream)
{
    if (!p || !w) return MOE_ERR_INVALID_ARG;
    const moe_dims &d = p->d;
    if (T < 0 || T > d.T_max) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !w_router || !out)) return MOE_ERR_INVALID_ARG;
    if (check_weights(p, w) != MOE_OK) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_router) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    int rc = check_ws(p, workspace, ws_bytes);
    if (rc) return rc;
    p->launches = 0;
    if (T == 0) return MOE_OK;
    const Layout L = make_layout(d);
    float *lg = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + L.lg);
    const cudaError_t e =
        launch_router_gemm(x, w_router, lg, T, d.H, d.E, p->d_status, p->num_sms, (cudaStream_t)stream);
    if (e != cudaSuccess) return fail_cuda(p, e);
    rc = moe_forward(p, T, x, lg, w, out, workspace, ws_bytes, stream);
    if (rc == MOE_OK) p->launches += 1;
    return rc;
}


}  // extern "C"
