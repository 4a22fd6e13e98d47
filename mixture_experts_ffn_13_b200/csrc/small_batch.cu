// small_batch.cu -- the whole FP8 layer for small batches (T <= 16 tokens) in one persistent kernel.
//
// Page "TPU推理外部化全面加速：InferenceX首份第三方性能數據發布", sections "优化 MoE 路由与专家内核" and
// "减少填充和低并发开销": at low concurrency the per-step overheads of routing, permutation and
// padding dominate, and for small batches the permutation is done as a one-hot selection
// instead of a sort.  Here, for 2 <= T <= 16, one cooperative launch (one CTA per SM) does the layer:
//  * phase 0a, spread over the grid, one warp per unit: the softmax top-k of one token, or the
//    e4m3 quantisation of one (token, 512-block) of x; results go to the workspace.  Meanwhile
//    every CTA asks L2 to prefetch its slice of the shared expert's weights, which no routing
//    decision can change;
//  * grid barrier (bounded spin on a counter in the workspace; all CTAs are co-resident);
//  * phase 0b, in every CTA: the (expert, token) row order of the regular path from the top-k,
//    and the x codes copied into shared memory as the MMA's B operand (all T tokens, padded to
//    16 columns);
//  * phase 1: gate|up.  Work items are (expert, 64 features of gate and of up, a quarter of K),
//    the shared expert's first; each streams its 128 interleaved weight rows by TMA and
//    multiplies them with all 16 token columns on the tensor cores (the one-hot selection:
//    columns of tokens that did not pick the expert are computed and dropped, which costs
//    nothing here since the weights stream anyway); the epilogue promotes each 512-block and
//    stores the partial G and U of the selected tokens' rows.  Splitting K four ways gives ~4x
//    more items than SMs at T = 1;
//  * grid barrier;
//  * phase 1.5, spread over the epilogue warps of the grid, one warp per (row, 512-block):
//    h = silu(G)*U from the four partials, quantised to e4m3 exactly as the regular path does,
//    into the workspace (each row once, whichever CTAs later stream its expert);
//  * grid barrier;
//  * phase 2: down.  Work items are (expert, 128 rows of H), the shared expert's first, and each
//    CTA takes a contiguous run of them, so consecutive items mostly share an expert.  For each
//    expert of its run a CTA copies the selected rows' h codes into shared memory as the B
//    operand (double-buffered: the next expert's operand is copied while the current one's
//    weights stream); the epilogue promotes and stores y for the selected rows;
//  * grid barrier, then phase 3: out[t] = sum_j p_hat[t,j] * y(t, e_j) + y_shared(t) in fp32,
//    rounded to bf16.
// The producer warp streams phase 2's weights while the barriers before it are pending.  Every wait
// is bounded and reports MOE_ERR_DEVICE_TIMEOUT through the status word; the epilogue warps
// take every wait's outcome together (bar.red), so none is left behind at a named barrier.
#include "moe_internal.h"
#include "gemm_common.cuh"
#include "launch.cuh"
#include "sm100.cuh"

#include <cuda_bf16.h>
#include <math.h>
#include <stdlib.h>

namespace moe {

namespace {

constexpr int kSbT = 16;                        // token columns of every MMA (the batch, padded)
constexpr int kSbKC = 128;                      // K bytes per weight stage
constexpr int kSbSplit = 4;                     // gate|up: K split into quarters
constexpr int kSbStage = 128 * kSbKC;           // 16 KB weight tile per stage
constexpr int kSbNS = 5;                        // weight stages: a smaller shared-memory carve-out leaves more L1 (measured: 5 beats 4, 6, 8 and 9)
constexpr int kSbEW = 4;                        // epilogue warps (one per TMEM lane quarter)
constexpr int kSbWarps = 2 + kSbEW;
constexpr int kSbThreads = 32 * kSbWarps;       // producer, MMA issuer, epilogue
constexpr int kSbMaxH = 4096, kSbMaxI = 2048;   // B operand: 16 x 4096 bytes of x, 2 x 16 x 2048 of h
constexpr int kSbBT = 64 * 1024;                // B operand region
constexpr int kSbMaxKb = 8;                     // 512-blocks of K (<= 4096)
constexpr int kSbMaxG = kSbT * kMaxK + 1;       // groups: selected experts + the shared expert
constexpr int kSbNSLOT = 8;                     // TMEM accumulator slots of 16 columns
constexpr int kBarEpi = 1, kBarEpiVote = 2;     // named barriers among the epilogue warps

struct SmallArgs {
    const uint16_t *x;      // [T, H] bf16
    const float *logits;    // [T, E]
    uint16_t *out;          // [T, H] bf16
    int T, H, E, I, Is, k;
    const float *sg, *su, *sd;     // routed scales: [E, I, H/512] x 2, [E, H, I/512]
    const float *ssg, *ssu, *ssd;  // shared expert's scales
    const uint8_t *wsh[3];         // shared expert's gate, up, down weights (L2 prefetch)
    size_t wsh_bytes[3];
    int up_lo[2];                  // per gate|up map (routed, shared): up rows below gate rows
    int32_t *tk_idx;               // [T, k] selected experts (phase 0a -> 0b)
    float *tk_w;                   // [T, k] p_hat
    uint8_t *xq;                   // [T, H] e4m3 codes of x
    float *xs;                     // [T, H/512] their scales
    float *partG, *partU;          // [kSbSplit][R][Imax] partial gate / up sums
    float *ybuf;                   // [R][H] down outputs of the selected rows
    uint8_t *hq;                   // [R][Imax] e4m3 codes of h (phase 1.5 -> 2)
    float *hs;                     // [R][Imax/512] their scales
    int R, Imax;                   // rows (T*k + T) and features per row of the partial sums
    const uint8_t *ws_warm;        // partials and y rows: pages touched early (address translation)
    size_t ws_warm_bytes;
    unsigned *bar;                 // grid barrier counter (zero before the launch)
    int *status;
    uint64_t timeout_ns;
};

struct SmallMaps {
    CUtensorMap gu[2];  // 4-D interleaved gate|up boxes (routed [E*I rows], shared [Is rows])
    CUtensorMap dn[2];  // down, 128 rows x 128 K bytes (routed [E*H rows], shared [H rows])
};

__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// e4m3 codes of 16 values scaled by 1/sc (sc = amax/448, correctly rounded divisions), packed
// in element order; the regular path's quantisers compute the same codes.
__device__ __forceinline__ uint4 e4m3_codes16(const float *f, float amax, float *sc_out)
{
    uint32_t cw[4] = {0u, 0u, 0u, 0u};
    float sc = 1.0f;
    if (amax > 0.0f) {
        sc = __fdiv_rn(amax, 448.0f);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t lo = cvt_e4m3x2(__fdiv_rn(f[4 * i], sc), __fdiv_rn(f[4 * i + 1], sc));
            const uint32_t hi = cvt_e4m3x2(__fdiv_rn(f[4 * i + 2], sc), __fdiv_rn(f[4 * i + 3], sc));
            cw[i] = lo | (hi << 16);
        }
    }
    *sc_out = sc;
    return make_uint4(cw[0], cw[1], cw[2], cw[3]);
}

// Order-preserving 32-bit key of a logit: a larger float gives a larger key, NaN counts as -inf
// and -0 as +0 (they compare equal as floats, so their tie is broken by index like any other).
__device__ __forceinline__ uint32_t logit_key(float v)
{
    if (v != v) v = -INFINITY;
    if (v == 0.0f) v = 0.0f;
    const uint32_t b = __float_as_uint(v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float logit_of_key(uint32_t key)
{
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Top-k of one token's E logits by one warp: (logit desc, index asc), then p_hat = softmax over
// the k.  Each candidate is the 64-bit key (logit key, ~index), so the largest key is the
// largest logit with ties to the lower index, and a pass is a register max-tree plus a warp
// max; the winner's key is then zeroed (a key of a real logit is never zero).  NPL: logits per
// lane (E <= 32 NPL).
template <int NPL>
__device__ __forceinline__ void topk_token(const float *L, int E, int k, int lane, int32_t *idx_out, float *w_out)
{
    uint64_t key[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        key[i] = e < E ? ((uint64_t)logit_key(__ldg(L + e)) << 32) | (uint32_t)~e : 0ull;
    }
    uint64_t sel = 0;
    for (int j = 0; j < k; ++j) {
        uint64_t t[NPL];
#pragma unroll
        for (int i = 0; i < NPL; ++i) t[i] = key[i];
#pragma unroll
        for (int h = NPL / 2; h >= 1; h >>= 1)
#pragma unroll
            for (int i = 0; i < h; ++i) t[i] = t[i] > t[i + h] ? t[i] : t[i + h];
        uint64_t best = t[0];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const uint64_t o = __shfl_xor_sync(0xffffffffu, best, off);
            best = o > best ? o : best;
        }
#pragma unroll
        for (int i = 0; i < NPL; ++i) key[i] = key[i] == best ? 0ull : key[i];
        if (lane == j) sel = best;
    }
    const float v = logit_of_key((uint32_t)(sel >> 32));
    const float lmax = __shfl_sync(0xffffffffu, v, 0);
    const float ex = lane < k ? expf(v - lmax) : 0.0f;
    float denom = 0.0f;
    for (int j = 0; j < k; ++j) denom += __shfl_sync(0xffffffffu, ex, j);
    if (lane < k) {
        idx_out[lane] = (int32_t)~(uint32_t)sel;
        w_out[lane] = ex / denom;
    }
}

// Byte offset of (row r, K byte b) in a K-major operand laid out as 128-byte-wide chunks of
// 16 rows with the 128-byte swizzle (16-byte piece j of row r stored at piece j ^ (r & 7)).
__device__ __forceinline__ int bt_off(int r, int b)
{
    return (b >> 7) * (kSbT * 128) + r * 128 + ((((b >> 4) & 7) ^ (r & 7)) << 4) + (b & 15);
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync %0, %1;" ::"r"(kBarEpi), "r"(32 * kSbEW) : "memory"); }
__device__ __forceinline__ bool epi_all(bool p) { return bar_all(kBarEpiVote, 32 * kSbEW, p); }

// One CTA's arrival at a grid barrier and its bounded wait for `target` arrivals, by the calling
// thread.  False on a timeout or when the CTA has aborted.
__device__ bool grid_arrive_wait(unsigned *bar, unsigned target, int *status, volatile int *abort, uint64_t tmo)
{
    __threadfence();
    atomicAdd(bar, 1u);
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        unsigned v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
        if (v >= target) return true;
        if (*abort || globaltimer_ns() - t0 > tmo) {
            atomicCAS(status, 0, MOE_ERR_DEVICE_TIMEOUT);
            *abort = 1;
            return false;
        }
        __nanosleep(64);
    }
}

// Grid barrier for every thread of every CTA; the outcome is the same in all threads of a CTA.
__device__ bool grid_sync_all(unsigned *bar, unsigned target, int *status, volatile int *abort, uint64_t tmo)
{
    __syncthreads();
    int ok = 1;
    if (threadIdx.x == 0) ok = grid_arrive_wait(bar, target, status, abort, tmo);
    return __syncthreads_and(ok) != 0;
}

// Grid barrier among the epilogue warps of every CTA; the outcome is the same in all of them.
__device__ bool grid_sync_epi(unsigned *bar, unsigned target, int *status, volatile int *abort, uint64_t tmo)
{
    epi_sync();
    bool ok = true;
    if (threadIdx.x == 64) ok = grid_arrive_wait(bar, target, status, abort, tmo);
    return epi_all(ok && !*abort);
}

__global__ void __launch_bounds__(kSbThreads, 1)
    small_batch_kernel(const __grid_constant__ SmallMaps maps, const __grid_constant__ SmallArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;                                  // kSbNS weight stages
    uint8_t *bt = ring + kSbNS * kSbStage;                 // B operand (x codes, then two h buffers)
    float *bscale = reinterpret_cast<float *>(bt + kSbBT);  // [2][16][kSbMaxKb] scales of the B operand
    int *s_idx = reinterpret_cast<int *>(bscale + 2 * kSbT * kSbMaxKb);  // [16][k] experts
    float *s_w = reinterpret_cast<float *>(s_idx + kSbT * kMaxK);         // [16][k] p_hat
    int *s_pos = reinterpret_cast<int *>(s_w + kSbT * kMaxK);             // [16][k] permuted row
    int *s_cnt = s_pos + kSbT * kMaxK;                                    // [E + 1] counts, then offsets
    int *s_gexp = s_cnt + (kMaxE + 1);                                    // [G] expert of each group
    int *s_gmask = s_gexp + kSbMaxG;                                      // [G] token mask
    int *s_misc = s_gmask + kSbMaxG;                                      // [0] routed groups
    uint64_t *full = reinterpret_cast<uint64_t *>((reinterpret_cast<uintptr_t>(s_misc + 4) + 7) & ~uintptr_t(7));
    uint64_t *empty = full + kSbNS;
    uint64_t *accf = empty + kSbNS;
    uint64_t *acce = accf + kSbNSLOT;
    uint64_t *bready = acce + kSbNSLOT;  // [2]
    uint64_t *bfree = bready + 2;        // [2]
    uint64_t *drain_bar = bfree + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T, H = a.H, E = a.E, I = a.I, Is = a.Is, k = a.k;
    const int nbH = H / kBlockK;
    const unsigned nblk = gridDim.x;
    int *status = a.status;
    const uint64_t tmo = a.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSbNS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < kSbNSLOT; ++s) {
            mbar_init(&accf[s], 1);
            mbar_init(&acce[s], kSbEW);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bready[b], kSbEW);
            mbar_init(&bfree[b], 1);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0)
        for (int i = 0; i < 2; ++i) {
            tma_prefetch_desc(&maps.gu[i]);
            tma_prefetch_desc(&maps.dn[i]);
        }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kSbNSLOT * kSbT);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    griddep_wait();
    griddep_launch_dependents();
    uint32_t issued = 0;

    // ---------------- phase 0a (spread over the grid): top-k, x codes ----------------
    if (threadIdx.x == 32) {
        // The first store into a page whose translation is not cached stalls the storing warp
        // for microseconds (measured ~12 us after a 256 MB sweep of L2): touch every 64 KB of
        // the partial-sum and y regions now, spread over the CTAs, while phase 0 runs.
        for (size_t o = (size_t)blockIdx.x << 16; o < a.ws_warm_bytes; o += (size_t)nblk << 16)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(a.ws_warm + o) : "memory");
        // this CTA's slice of the shared expert's weights into L2
        for (int m = 0; m < 3; ++m) {
            const size_t n = a.wsh_bytes[m];
            const size_t per = ((n + nblk - 1) / nblk + 255) & ~size_t(255);
            const size_t lo = per * blockIdx.x, hi = lo + per < n ? lo + per : n;
            for (size_t o = lo; o < hi; o += 32768) {
                const uint32_t len = (uint32_t)(hi - o < 32768 ? hi - o : 32768);
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.wsh[m] + o), "r"(len) : "memory");
            }
        }
    }
    for (int u = blockIdx.x * kSbWarps + warp; u < T + T * nbH; u += nblk * kSbWarps) {
        if (u < T) {
            const float *L = a.logits + (size_t)u * E;
            if (E <= 256)
                topk_token<8>(L, E, k, lane, a.tk_idx + u * k, a.tk_w + u * k);
            else if (E <= 512)
                topk_token<16>(L, E, k, lane, a.tk_idx + u * k, a.tk_w + u * k);
            else
                topk_token<32>(L, E, k, lane, a.tk_idx + u * k, a.tk_w + u * k);
        } else {
            // x codes of (token t, block kb): lane = 16 consecutive elements
            const int t = (u - T) / nbH, kb = (u - T) - t * nbH;
            const int i0 = kb * kBlockK + lane * 16;
            const uint4 *p = reinterpret_cast<const uint4 *>(a.x + (size_t)t * H + i0);
            const uint4 q0 = __ldg(p), q1 = __ldg(p + 1);
            const uint32_t wv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
            float f[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                f[2 * i] = __uint_as_float(wv[i] << 16);
                f[2 * i + 1] = __uint_as_float(wv[i] & 0xffff0000u);
            }
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            float sc;
            const uint4 cw = e4m3_codes16(f, amax, &sc);
            *reinterpret_cast<uint4 *>(a.xq + (size_t)t * H + i0) = cw;
            if (lane == 0) a.xs[t * nbH + kb] = sc;
        }
    }
    if (!grid_sync_all(a.bar, nblk, status, abort_flag, tmo)) goto done;

    // ---------------- phase 0b (every CTA): permutation, B operand ----------------
    {
        // x codes into the swizzled B layout; rows >= T are never stored, so they stay as they are
        const uint32_t bts = smem_u32(bt);
        const int per_row = H / 16;
        for (int c = threadIdx.x; c < T * per_row; c += kSbThreads) {
            const int t = c / per_row, b = (c - t * per_row) * 16;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(bts + bt_off(t, b)),
                         "l"(a.xq + (size_t)t * H + b)
                         : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    for (int i = threadIdx.x; i < 2 * kSbT * kSbMaxKb; i += kSbThreads) {
        const int t = i / kSbMaxKb, kb = i - t * kSbMaxKb;
        bscale[i] = (i < kSbT * kSbMaxKb && t < T && kb < nbH) ? __ldcg(a.xs + t * nbH + kb) : 1.0f;
    }
    for (int i = threadIdx.x; i < T * k; i += kSbThreads) {
        s_idx[i] = __ldcg(a.tk_idx + i);
        s_w[i] = __ldcg(a.tk_w + i);
    }
    for (int e = threadIdx.x; e <= E; e += kSbThreads) s_cnt[e] = 0;
    __syncthreads();
    // permutation: counts, offsets, rows in (expert, token) order (as the regular path)
    for (int i = threadIdx.x; i < T * k; i += kSbThreads) atomicAdd(&s_cnt[s_idx[i]], 1);
    __syncthreads();
    if (warp == 0) {  // exclusive scan of the counts and the list of touched experts, lane = E/32 experts
        const int per = (E + 31) / 32;
        const int e0 = lane * per, e1 = min(E, e0 + per);
        int sum = 0, ng = 0;
        for (int e = e0; e < e1; ++e) {
            const int c = s_cnt[e];
            sum += c;
            ng += c != 0;
        }
        int isum = sum, ing = ng;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int vs = __shfl_up_sync(0xffffffffu, isum, off), vg = __shfl_up_sync(0xffffffffu, ing, off);
            if (lane >= off) {
                isum += vs;
                ing += vg;
            }
        }
        int run = isum - sum, g = ing - ng;
        for (int e = e0; e < e1; ++e) {
            const int c = s_cnt[e];
            s_cnt[e] = run;
            if (c) {
                s_gexp[g] = e;
                s_gmask[g] = 0;
                ++g;
            }
            run += c;
        }
        if (lane == 31) {
            s_cnt[E] = isum;
            s_misc[0] = ing;
        }
    }
    __syncthreads();
    {
        const int Gr0 = s_misc[0];
        for (int i = threadIdx.x; i < T * k; i += kSbThreads) {
            const int t = i / k, e = s_idx[i];
            int rank = 0;  // tokens below t that chose e
            for (int u = 0; u < t; ++u)
                for (int j = 0; j < k; ++j) rank += s_idx[u * k + j] == e;
            s_pos[i] = s_cnt[e] + rank;
            // group of e: binary search in the sorted expert list
            int lo = 0, hi = Gr0 - 1;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (s_gexp[mid] < e) lo = mid + 1; else hi = mid;
            }
            atomicOr(&s_gmask[lo], 1 << t);
        }
        if (threadIdx.x == 0) {
            s_gexp[Gr0] = -1;  // the shared expert: every token
            s_gmask[Gr0] = (1 << T) - 1;
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // x codes, for the tensor cores
    __syncthreads();
    {
    const int Gr = s_misc[0];
    const int G = Gr + (Is > 0 ? 1 : 0);
    // row of (group g, token t): routed rows from the permutation, shared rows after them
    auto row_of = [&](int g, int t) {
        if (g == Gr) return T * k + t;
        const int e = s_gexp[g];
        int r = s_cnt[e];
        for (int u = 0; u < t; ++u) r += (s_gmask[g] >> u) & 1;
        return r;
    };
    const int nf_r = I / 64, nf_s = Is > 0 ? Is / 64 : 0;  // 64-feature gate|up tiles per group
    const int items1 = (nf_s + Gr * nf_r) * kSbSplit;
    const int kq = H / kSbSplit;  // K bytes of a gate|up item
    // phase-1 item w -> (group, feature tile, K quarter); the shared expert's tiles first
    auto item1 = [&](int w, int &g, int &f, int &sp) {
        sp = w % kSbSplit;
        const int u = w / kSbSplit;
        if (u < nf_s) {
            g = Gr;
            f = u;
        } else {
            g = (u - nf_s) / nf_r;
            f = (u - nf_s) - g * nf_r;
        }
    };
    // phase 2: items (group, 128-row tile of H), the shared expert's first; CTA b takes the
    // contiguous run [w2lo, w2hi), and a run of one group's tiles is one "segment" sharing a B operand
    const int ntile = H / 128;
    const int items2 = G * ntile;
    const int w2lo = (int)(((long long)items2 * blockIdx.x) / nblk);
    const int w2hi = (int)(((long long)items2 * (blockIdx.x + 1)) / nblk);
    auto grp2 = [&](int w) {
        const int gi = w / ntile;
        return Is > 0 ? (gi == 0 ? Gr : gi - 1) : gi;
    };

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            const uint64_t pol_w = l2_policy_evict_first();
            uint32_t it = 0;
            auto stage = [&](const CUtensorMap *map, bool four_d, int x, int y) -> bool {
                const int s = it % kSbNS;
                if (!mbar_wait(&empty[s], ((it / kSbNS) & 1) ^ 1, abort_flag, status, tmo)) return false;
                issued = it + 1;
                mbar_arrive_expect_tx(&full[s], kSbStage);
                if (four_d)
                    tma_load_4d_hint(ring + s * kSbStage, map, &full[s], x, 0, 0, y >> 4, pol_w);
                else
                    tma_load_2d_hint(ring + s * kSbStage, map, &full[s], x, y, pol_w);
                ++it;
                return true;
            };
            for (int w = blockIdx.x; w < items1; w += nblk) {
                int g, f, sp;
                item1(w, g, f, sp);
                const bool sh = g == Gr;
                const int wrow = (sh ? 0 : s_gexp[g] * I) + f * 64;
                for (int x = sp * kq; x < (sp + 1) * kq; x += kSbKC)
                    if (!stage(&maps.gu[sh ? 1 : 0], true, x, wrow)) goto done;
            }
            for (int w = w2lo; w < w2hi; ++w) {
                const int g = grp2(w), nt = w % ntile;
                const bool sh = g == Gr;
                const int K = sh ? Is : I;
                const int wrow = (sh ? 0 : s_gexp[g] * H) + nt * 128;
                for (int x = 0; x < K; x += kSbKC)
                    if (!stage(&maps.dn[sh ? 1 : 0], false, x, wrow)) goto done;
            }
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0) {
            const uint32_t idesc = instr_desc(kTileM, kSbT, 0, 0);
            uint32_t it = 0, ai = 0;
            auto block = [&](const uint8_t *bops, int nstages) -> bool {
                const int slot = ai % kSbNSLOT;
                if (!mbar_wait(&acce[slot], ((ai / kSbNSLOT) & 1) ^ 1, abort_flag, status, tmo)) return false;
                tc_fence_after();
                const uint32_t d = tmem_base + slot * kSbT;
                for (int j = 0; j < nstages; ++j, ++it) {
                    const int s = it % kSbNS;
                    if (!mbar_wait(&full[s], (it / kSbNS) & 1, abort_flag, status, tmo)) return false;
                    tc_fence_after();
                    const uint64_t da = smem_desc_sw128(ring + s * kSbStage);
                    const uint64_t db = smem_desc_sw128(bops + j * (kSbT * 128));
#pragma unroll
                    for (int kk = 0; kk < kSbKC / 32; ++kk)
                        mma_f8(d, da + 2 * kk, db + 2 * kk, idesc, (j > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&empty[s]);
                }
                mma_commit(&accf[slot]);
                ++ai;
                return true;
            };
            for (int w = blockIdx.x; w < items1; w += nblk) {
                int g, f, sp;
                item1(w, g, f, sp);
                for (int x = sp * kq; x < (sp + 1) * kq; x += kBlockK)
                    if (!block(bt + (x >> 7) * (kSbT * 128), kBlockK / kSbKC)) goto done;
            }
            int si = -1, gcur = -2;
            for (int w = w2lo; w < w2hi; ++w) {
                const int g = grp2(w);
                if (g != gcur) {  // a new segment: its operand must be built
                    if (si >= 0) mma_commit(&bfree[si & 1]);
                    ++si;
                    gcur = g;
                    if (!mbar_wait(&bready[si & 1], (si >> 1) & 1, abort_flag, status, tmo)) goto done;
                    tc_fence_after();
                }
                const int K = g == Gr ? Is : I;
                const uint8_t *bops = bt + (si & 1) * (kSbT * kSbMaxI);
                for (int x = 0; x < K; x += kBlockK)
                    if (!block(bops + (x >> 7) * (kSbT * 128), kBlockK / kSbKC)) goto done;
            }
            if (si >= 0) mma_commit(&bfree[si & 1]);
        }
    } else {
        // ------------------------------ epilogue ----------------------------------
        const int q = warp & 3;
        const int r = q * 16 + (lane & 15);  // feature of a gate|up tile; lanes >= 16: the other matrix
        const int et = threadIdx.x - 64;     // 0..127
        const int ew = warp - 2;             // epilogue warp 0..3
        uint32_t ai = 0;
        // phase 1: partial G and U of the selected rows.  This thread's weight scales for an
        // item's blocks are loaded one item ahead (each would otherwise cost the epilogue a DRAM
        // round trip per block, and the stalled epilogue would hold up the TMEM slots).
        constexpr int kB1 = kSbMaxKb / kSbSplit;  // 512-blocks per gate|up item (H / 2048)
        const int nb1 = kq / kBlockK;
        auto scales1 = [&](int w, float(&sc)[kB1]) {
            int g, f, sp;
            item1(w, g, f, sp);
            const bool sh = g == Gr;
            const bool up = (lane >= 16) != (a.up_lo[sh ? 1 : 0] != 0);
            const float *sw = up ? (sh ? a.ssu : a.su) : (sh ? a.ssg : a.sg);
            sw += ((size_t)(sh ? 0 : s_gexp[g]) * (sh ? Is : I) + f * 64 + r) * nbH + sp * nb1;
#pragma unroll
            for (int i = 0; i < kB1; ++i) sc[i] = i < nb1 ? __ldg(sw + i) : 0.0f;
        };
        float scn1[kB1];
        if ((int)blockIdx.x < items1) scales1(blockIdx.x, scn1);
        for (int w = blockIdx.x; w < items1; w += nblk) {
            int g, f, sp;
            item1(w, g, f, sp);
            float sc[kB1];
#pragma unroll
            for (int i = 0; i < kB1; ++i) sc[i] = scn1[i];
            if (w + (int)nblk < items1) scales1(w + nblk, scn1);
            const bool is_up = (lane >= 16) != (a.up_lo[g == Gr ? 1 : 0] != 0);
            const int feat = f * 64 + r;
            float acc[kSbT];
#pragma unroll
            for (int c = 0; c < kSbT; ++c) acc[c] = 0.0f;
#pragma unroll
            for (int i = 0; i < kB1; ++i) {
                if (i >= nb1) break;
                const int kb = sp * nb1 + i;
                const int slot = ai % kSbNSLOT;
                const bool ok = mbar_wait(&accf[slot], (ai / kSbNSLOT) & 1, abort_flag, status, tmo);
                if (!epi_all(ok)) goto done;
                tc_fence_after();
                float v[16];
                tmem_ld16(tmem_base + ((uint32_t)(q * 32) << 16) + slot * kSbT, v);
                tmem_wait_ld(v);
#pragma unroll
                for (int c = 0; c < kSbT; ++c) acc[c] = fmaf(v[c], sc[i] * bscale[c * kSbMaxKb + kb], acc[c]);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acce[slot]);
                ++ai;
            }
            float *part = (is_up ? a.partU : a.partG) + (size_t)sp * a.R * a.Imax;
            const int mask = s_gmask[g];
#pragma unroll
            for (int c = 0; c < kSbT; ++c)
                if (c < T && ((mask >> c) & 1)) part[(size_t)row_of(g, c) * a.Imax + feat] = acc[c];
        }
        if (!grid_sync_epi(a.bar, 2 * nblk, status, abort_flag, tmo)) goto done;
        // phase 1.5, spread over the epilogue warps of the grid: h = silu(G)*U of every row from
        // the four partial sums, e4m3 per 512-block (the regular path's quantiser), into hq/hs;
        // one warp per (row, 512-block), lane = 16 consecutive features
        {
            const int nbI = I / kBlockK, nbS = Is / kBlockK;
            const int units = T * k * nbI + T * nbS;
            for (int u = blockIdx.x * kSbEW + ew; u < units; u += nblk * kSbEW) {
                int row, kb;
                if (u < T * k * nbI) {
                    row = u / nbI;
                    kb = u - row * nbI;
                } else {
                    row = T * k + (u - T * k * nbI) / nbS;
                    kb = (u - T * k * nbI) % nbS;
                }
                const int f0 = kb * kBlockK + lane * 16;
                float4 vg[kSbSplit][4], vu[kSbSplit][4];
#pragma unroll
                for (int sp = 0; sp < kSbSplit; ++sp) {
                    const size_t o = ((size_t)sp * a.R + row) * a.Imax + f0;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        vg[sp][i] = __ldcg(reinterpret_cast<const float4 *>(a.partG + o) + i);
                        vu[sp][i] = __ldcg(reinterpret_cast<const float4 *>(a.partU + o) + i);
                    }
                }
                float h[16], am = 0.0f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float g4[4] = {0.f, 0.f, 0.f, 0.f}, u4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int sp = 0; sp < kSbSplit; ++sp) {
                        g4[0] += vg[sp][i].x;
                        g4[1] += vg[sp][i].y;
                        g4[2] += vg[sp][i].z;
                        g4[3] += vg[sp][i].w;
                        u4[0] += vu[sp][i].x;
                        u4[1] += vu[sp][i].y;
                        u4[2] += vu[sp][i].z;
                        u4[3] += vu[sp][i].w;
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        h[4 * i + j] = silu_mul(g4[j], u4[j]);
                        am = fmaxf(am, fabsf(h[4 * i + j]));
                    }
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
                float sc;
                const uint4 cw = e4m3_codes16(h, am, &sc);
                *reinterpret_cast<uint4 *>(a.hq + (size_t)row * a.Imax + f0) = cw;
                if (lane == 0) a.hs[row * (a.Imax / kBlockK) + kb] = sc;
            }
        }
        if (!grid_sync_epi(a.bar, 3 * nblk, status, abort_flag, tmo)) goto done;
        // phase 2: the B operand of segment si (group g) into buffer si & 1: the codes and scales
        // of the group's selected rows, copied from hq/hs.  Columns of tokens that did not pick
        // the group keep whatever codes the buffer held: an MMA column depends only on its own B
        // row, and those columns are never stored.
        auto load_h = [&](int g, int si) -> bool {
            const int b = si & 1;
            const int nbK = (g == Gr ? Is : I) / kBlockK;
            const uint32_t bops = smem_u32(bt + b * (kSbT * kSbMaxI));
            float *bsc = bscale + b * kSbT * kSbMaxKb;
            if (si >= 2) {
                // the MMAs of segment si - 2 have read the buffer, and (the vote is also a
                // barrier) every epilogue warp has promoted its items with the buffer's scales
                const bool ok = mbar_wait(&bfree[b], ((si >> 1) - 1) & 1, abort_flag, status, tmo);
                if (!epi_all(ok)) return false;
            }
            const int mask = s_gmask[g];
            const int nsel = __popc(mask);
            const int per_row = nbK * (kBlockK / 16);  // 16-byte chunks of a row's codes
            for (int c = et; c < nsel * per_row; c += 32 * kSbEW) {
                const int j = c / per_row, b16 = (c - j * per_row) * 16;
                int m = mask;
                for (int i = 0; i < j; ++i) m &= m - 1;
                const int t = __ffs(m) - 1;
                const int row = row_of(g, t);
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(bops + bt_off(t, b16)),
                             "l"(a.hq + (size_t)row * a.Imax + b16)
                             : "memory");
                if (b16 % kBlockK == 0) bsc[t * kSbMaxKb + b16 / kBlockK] = __ldcg(a.hs + row * (a.Imax / kBlockK) + b16 / kBlockK);
            }
            asm volatile("cp.async.wait_all;" ::: "memory");
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // h codes, for the tensor cores
            __syncwarp();
            if (lane == 0) mbar_arrive(&bready[b]);
            epi_sync();  // the scales are in place for every epilogue warp
            return true;
        };
        // this thread's down-weight scales of item w, loaded one item ahead as in phase 1
        constexpr int kB2 = kSbMaxI / kBlockK;  // 512-blocks per down item (K <= 2048)
        auto scales2 = [&](int w, float(&sc)[kB2]) {
            const int g = grp2(w);
            const bool sh = g == Gr;
            const int nbK = (sh ? Is : I) / kBlockK;
            const int n = (w % ntile) * 128 + q * 32 + lane;
            const float *sw = (sh ? a.ssd : a.sd) + ((size_t)(sh ? 0 : s_gexp[g]) * H + n) * nbK;
#pragma unroll
            for (int i = 0; i < kB2; ++i) sc[i] = i < nbK ? __ldg(sw + i) : 0.0f;
        };
        float scn2[kB2];
        if (w2lo < w2hi) scales2(w2lo, scn2);
        int si = 0;
        if (w2lo < w2hi && !load_h(grp2(w2lo), 0)) goto done;
        for (int w = w2lo; w < w2hi; ++si) {
            const int g = grp2(w);
            const int wend = min(w2hi, (w / ntile + 1) * ntile);  // end of this segment
            if (wend < w2hi && !load_h(grp2(wend), si + 1)) goto done;
            const bool sh = g == Gr;
            const int nbK = (sh ? Is : I) / kBlockK;
            const float *bsc = bscale + (si & 1) * kSbT * kSbMaxKb;
            const int mask = s_gmask[g];
            for (; w < wend; ++w) {
                float sc[kB2];
#pragma unroll
                for (int i = 0; i < kB2; ++i) sc[i] = scn2[i];
                if (w + 1 < w2hi) scales2(w + 1, scn2);
                // promote and store y of the selected rows
                const int n = (w % ntile) * 128 + q * 32 + lane;
                float acc[kSbT];
#pragma unroll
                for (int c = 0; c < kSbT; ++c) acc[c] = 0.0f;
#pragma unroll
                for (int kb = 0; kb < kB2; ++kb) {
                    if (kb >= nbK) break;
                    const int slot = ai % kSbNSLOT;
                    const bool ok = mbar_wait(&accf[slot], (ai / kSbNSLOT) & 1, abort_flag, status, tmo);
                    if (!epi_all(ok)) goto done;
                    tc_fence_after();
                    float v[16];
                    tmem_ld16(tmem_base + ((uint32_t)(q * 32) << 16) + slot * kSbT, v);
                    tmem_wait_ld(v);
#pragma unroll
                    for (int c = 0; c < kSbT; ++c) acc[c] = fmaf(v[c], sc[kb] * bsc[c * kSbMaxKb + kb], acc[c]);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acce[slot]);
                    ++ai;
                }
#pragma unroll
                for (int c = 0; c < kSbT; ++c)
                    if (c < T && ((mask >> c) & 1)) a.ybuf[(size_t)row_of(g, c) * H + n] = acc[c];
            }
        }
        if (!grid_sync_epi(a.bar, 4 * nblk, status, abort_flag, tmo)) goto done;
        // phase 3: combine, 4 hidden features per thread over all CTAs
        for (int i = blockIdx.x * (32 * kSbEW) + et; i < T * H / 4; i += nblk * (32 * kSbEW)) {
            const int t = i / (H / 4), c4 = i - t * (H / 4);
            float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int j = 0; j < k; ++j) {
                const float wj = s_w[t * k + j];
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.ybuf + (size_t)s_pos[t * k + j] * H) + c4);
                s.x = fmaf(wj, v.x, s.x);
                s.y = fmaf(wj, v.y, s.y);
                s.z = fmaf(wj, v.z, s.z);
                s.w = fmaf(wj, v.w, s.w);
            }
            if (Is > 0) {
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.ybuf + (size_t)(T * k + t) * H) + c4);
                s.x += v.x;
                s.y += v.y;
                s.z += v.z;
                s.w += v.w;
            }
            const __nv_bfloat162 lo = __floats2bfloat162_rn(s.x, s.y), hi = __floats2bfloat162_rn(s.z, s.w);
            uint2 o;
            o.x = *reinterpret_cast<const uint32_t *>(&lo);
            o.y = *reinterpret_cast<const uint32_t *>(&hi);
            reinterpret_cast<uint2 *>(a.out + (size_t)t * H)[c4] = o;
        }
    }
    }
done:
    if (warp == 0 && lane == 0)
        for (uint32_t j = issued > (uint32_t)kSbNS ? issued - kSbNS : 0; j < issued; ++j)
            mbar_wait_drain(&full[j % kSbNS], (j / kSbNS) & 1, tmo);
    if (warp == 1 && lane == 0) mma_drain(drain_bar, tmo);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, kSbNSLOT * kSbT);
    }
}

constexpr int kSbSmem = 1024 + kSbNS * kSbStage + kSbBT + 4 * (2 * kSbT * kSbMaxKb) + 4 * 3 * (kSbT * kMaxK) +
                        4 * (kMaxE + 1) + 4 * 2 * kSbMaxG + 16 + 8 +
                        8 * (2 * kSbNS + 2 * kSbNSLOT + 5) + 8;

int env_small_batch()
{
    static const int on = [] {
        const char *v = getenv("MOE_SMALL_BATCH");
        return (v && v[0] == '0') ? 0 : 1;
    }();
    return on;
}

// Workspace carve-up for a batch of T tokens (every region 256-byte aligned; sizes grow with T,
// so the layout for T_max bounds every smaller batch's).
struct SbLayout {
    size_t bar, partG, partU, ybuf, hq, hs, tk_idx, tk_w, xq, xs, total;
};

SbLayout sb_layout(size_t T, const moe_dims &d)
{
    auto al = [](size_t v) { return (v + 255) & ~size_t(255); };
    const size_t R = T * (size_t)(d.k + 1);
    const size_t Imax = (size_t)(d.I > d.I_shared ? d.I : d.I_shared);
    const size_t part = (size_t)kSbSplit * R * Imax * 4;
    SbLayout L;
    L.bar = 0;  // the barrier counter keeps one place whatever the batch
    L.partG = 256;
    L.partU = al(L.partG + part);
    L.ybuf = al(L.partU + part);
    L.hq = al(L.ybuf + R * (size_t)d.H * 4);
    L.hs = al(L.hq + R * Imax);
    L.tk_idx = al(L.hs + R * (Imax / kBlockK) * 4);
    L.tk_w = al(L.tk_idx + T * (size_t)d.k * 4);
    L.xq = al(L.tk_w + T * (size_t)d.k * 4);
    L.xs = al(L.xq + T * (size_t)d.H);
    L.total = al(L.xs + T * (size_t)(d.H / kBlockK) * 4);
    return L;
}

}  // namespace

bool small_batch_fits(int T, const moe_dims &d)
{
    // T = 1 stays on the multi-kernel path, which measured faster there (66.6 against ~70 us on
    // the decode-shaped layer); from 2 to 16 tokens the single kernel is as fast or faster
    return env_small_batch() && d.wfmt == MOE_W_FP8_SC512 && T >= 2 && T <= kSbT && d.H <= kSbMaxH &&
           d.H % (kSbSplit * kBlockK) == 0 && d.I <= kSbMaxI && d.I % kBlockK == 0 &&
           (d.I_shared == 0 || (d.I_shared <= kSbMaxI && d.I_shared % kBlockK == 0)) && d.E <= kMaxE &&
           d.k <= kMaxK;
}

size_t small_batch_workspace(const moe_dims &d)
{
    const size_t T = d.T_max < kSbT ? (size_t)d.T_max : (size_t)kSbT;
    return sb_layout(T, d).total;
}

cudaError_t launch_small_batch(const moe_dims &d, int T, const uint16_t *x, const float *logits,
                               const moe_weights *w, uint16_t *out, void *ws, int *status, int num_sms,
                               cudaStream_t s, int *launched)
{
    *launched = 0;
    SmallMaps maps{};
    SmallArgs a{};
    const int H = d.H, I = d.I, Is = d.I_shared, E = d.E;
    int rc = encode_map_gateup_ilv(&maps.gu[0], w->w_gate, w->w_up, H, (uint64_t)E * I, &a.up_lo[0]);
    if (Is > 0) rc |= encode_map_gateup_ilv(&maps.gu[1], w->ws_gate, w->ws_up, H, Is, &a.up_lo[1]);
    if (rc) return cudaErrorNotSupported;  // the weight arrays are too far apart for one map
    const CUtensorMapDataType U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
    rc = encode_map_2d(&maps.dn[0], w->w_down, U8, 1, I, (uint64_t)E * H, 128, 128, true);
    if (Is > 0) rc |= encode_map_2d(&maps.dn[1], w->ws_down, U8, 1, Is, H, 128, 128, true);
    if (rc) return cudaErrorInvalidValue;
    if (Is == 0) {  // never read: the shared expert's maps mirror the routed ones
        maps.gu[1] = maps.gu[0];
        maps.dn[1] = maps.dn[0];
    }
    a.x = x;
    a.logits = logits;
    a.out = out;
    a.T = T;
    a.H = H;
    a.E = E;
    a.I = I;
    a.Is = Is;
    a.k = d.k;
    a.sg = static_cast<const float *>(w->s_gate);
    a.su = static_cast<const float *>(w->s_up);
    a.sd = static_cast<const float *>(w->s_down);
    a.ssg = static_cast<const float *>(w->ss_gate);
    a.ssu = static_cast<const float *>(w->ss_up);
    a.ssd = static_cast<const float *>(w->ss_down);
    const size_t shared_bytes = Is > 0 ? (size_t)Is * H : 0;  // each of gate, up, down
    a.wsh[0] = static_cast<const uint8_t *>(w->ws_gate);
    a.wsh[1] = static_cast<const uint8_t *>(w->ws_up);
    a.wsh[2] = static_cast<const uint8_t *>(w->ws_down);
    for (int m = 0; m < 3; ++m)  // prefetch needs 16-byte aligned starts (slices are 256-byte multiples)
        a.wsh_bytes[m] = (a.wsh[m] && (reinterpret_cast<uintptr_t>(a.wsh[m]) & 15) == 0) ? shared_bytes : 0;
    a.R = T * (d.k + 1);
    a.Imax = I > Is ? I : Is;
    const SbLayout L = sb_layout((size_t)T, d);
    uint8_t *p = static_cast<uint8_t *>(ws);
    a.partG = reinterpret_cast<float *>(p + L.partG);
    a.partU = reinterpret_cast<float *>(p + L.partU);
    a.ybuf = reinterpret_cast<float *>(p + L.ybuf);
    a.hq = p + L.hq;
    a.hs = reinterpret_cast<float *>(p + L.hs);
    a.bar = reinterpret_cast<unsigned *>(p + L.bar);
    a.tk_idx = reinterpret_cast<int32_t *>(p + L.tk_idx);
    a.tk_w = reinterpret_cast<float *>(p + L.tk_w);
    a.xq = p + L.xq;
    a.xs = reinterpret_cast<float *>(p + L.xs);
    a.ws_warm = p + L.partG;
    a.ws_warm_bytes = L.tk_idx - L.partG;
    a.status = status;
    a.timeout_ns = kDefaultTimeoutNs;
    cudaError_t e = cudaMemsetAsync(a.bar, 0, sizeof(unsigned), s);
    if (e != cudaSuccess) return e;
    e = set_smem_limit(reinterpret_cast<const void *>(small_batch_kernel), kSbSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident at once: the grid barriers
    attr[0].val.cooperative = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms);
    cfg.blockDim = dim3(kSbThreads);
    cfg.dynamicSmemBytes = kSbSmem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, small_batch_kernel, maps, a);
    if (e == cudaSuccess) *launched = 1;
    return e;
}

}  // namespace moe
