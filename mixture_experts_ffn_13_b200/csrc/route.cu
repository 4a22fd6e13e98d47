// route.cu -- step A1 (softmax top-k router) and step A3 (permutation into per-expert groups).
//
// Router: page "把 397B MoE 榨進 TPU7x：Google 拿到 4.7 倍加速", section "稀疏在哪裡": each token
// picks its top experts by softmax probability.  Selection compares the fp32 logits (the
// softmax is monotone in them), ties going to the lower expert index; the k weights are the
// softmax over the selected logits (the full softmax renormalised over the top-k).
//
// Permutation: page "TPU推理外部化全面加速：InferenceX首份第三方性能數據發布", section "优化 MoE
// 路由与专家内核": tokens are collected into contiguous per-expert groups, ordered by a packed
// (expert, token) key.  Here that order is produced without a sort: a per-chunk histogram,
// one prefix sum over (expert, chunk), and an in-order scatter inside each chunk, so the
// result is deterministic and equal to sorting by (expert, token).  Batches of up to 4096
// tokens (token bitmaps within 160 KB of shared memory) permute in one block instead: per-expert
// token bitmaps, one packed scan, and popcount ranks.
#include "launch.cuh"
#include "moe_internal.h"

#include <algorithm>

#include <math.h>

namespace moe {

namespace {

constexpr unsigned kFull = 0xffffffffu;

// Top-k of one token's logits by one warp.  Lane l holds the logits of experts l, l+32, ...;
// k rounds of a warp arg-max (value desc, index asc) pick the experts; lane j < k returns the
// j-th pick in *sel_e and its weight p_hat_j = exp(L_j - L_max) / sum_i exp(L_i - L_max) (the
// sum taken in selection order) in *sel_w.
template <int EPL>
__device__ __forceinline__ void route_one(const float *__restrict__ L, int E, int k, int lane, int *sel_e_out,
                                          float *sel_w_out)
{
    float v[EPL];
    uint32_t taken = 0;  // bit i: element i of this lane is absent or already chosen
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        const float l = (e < E) ? __ldg(L + e) : -INFINITY;
        v[i] = (l != l) ? -INFINITY : l;  // NaN (caller error) ranks lowest: indices stay valid
        if (e >= E) taken |= 1u << i;
    }
    float sel_v = 0.0f;
    int sel_e = 0;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = lane + 32 * i;
            if (!((taken >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < be))) {
                bv = v[i];
                be = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(kFull, bv, off);
            const int oe = __shfl_xor_sync(kFull, be, off);
            if (ov > bv || (ov == bv && oe < be)) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == j) {
            sel_v = bv;
            sel_e = be;
        }
    }
    const float lmax = __shfl_sync(kFull, sel_v, 0);
    const float ex = (lane < k) ? expf(sel_v - lmax) : 0.0f;
    float denom = 0.0f;
    for (int j = 0; j < k; ++j) denom += __shfl_sync(kFull, ex, j);
    *sel_e_out = sel_e;
    *sel_w_out = ex / denom;
}

// One warp per token.
// With `check` set (checked mode), a token whose logits are not all finite records
// MOE_ERR_BOUNDS in *check; selection then proceeds as usual (its result is unspecified).
template <int EPL>
__global__ void __launch_bounds__(256) route_kernel(const float *__restrict__ logits, int T, int E, int k,
                                                    int32_t *__restrict__ topk_idx, float *__restrict__ topk_w,
                                                    int *check, WeightPrefetch pf)
{
    // Blocks past the routing ones only ask L2 for weights that no kernel of this stream writes
    // (before waiting on the previous kernel), so the weight stream overlaps routing, permutation
    // and quantisation without delaying the routing blocks, whose issue is latency-bound.
    const uint32_t nroute = (T + 7) / 8;
    if (blockIdx.x >= nroute) {
        const uint32_t npf = gridDim.x - nroute;
        for (uint32_t c = (blockIdx.x - nroute) + npf * threadIdx.x; c < 2 * pf.chunks; c += npf * blockDim.x) {
            const uint8_t *src = (c & 1 ? pf.b : pf.a) + (size_t)(c >> 1) * WeightPrefetch::kChunk;
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(WeightPrefetch::kChunk)
                         : "memory");
        }
        griddep_launch_dependents();
        return;
    }
    griddep_wait();
    griddep_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= T) return;
    if (check) {
        bool bad = false;
        for (int e = lane; e < E; e += 32) bad |= !isfinite(__ldg(logits + (size_t)t * E + e));
        if (__any_sync(kFull, bad) && lane == 0) atomicCAS(check, 0, MOE_ERR_BOUNDS);
    }
    int e;
    float w;
    route_one<EPL>(logits + (size_t)t * E, E, k, lane, &e, &w);
    if (lane < k) {
        topk_idx[(size_t)t * k + lane] = e;
        topk_w[(size_t)t * k + lane] = w;
    }
}

// Per-chunk expert histogram: chunk_hist[c, e] = assignments to e among tokens of chunk c.
__global__ void __launch_bounds__(kChunk) hist_kernel(const int32_t *__restrict__ topk_idx, int T, int E, int k,
                                                      int32_t *__restrict__ chunk_hist)
{
    __shared__ int h[kMaxE];
    griddep_wait();
    griddep_launch_dependents();
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    const int t = blockIdx.x * kChunk + threadIdx.x;
    if (t < T)
        for (int j = 0; j < k; ++j) atomicAdd(&h[topk_idx[(size_t)t * k + j]], 1);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_hist[(size_t)blockIdx.x * E + e] = h[e];
}

// Exclusive prefix sum over the 1024 threads of a block; returns the thread's exclusive
// prefix and writes the block total to *total.
__device__ int block_exclusive_scan(int v, int *scratch /* 33 ints */, int *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = (lane < (int)(blockDim.x >> 5)) ? scratch[lane] : 0;
        int wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(kFull, wi, off);
            if (lane >= off) wi += o;
        }
        scratch[lane] = wi - w;  // exclusive prefix of warp totals
        if (lane == 31) scratch[32] = wi;
    }
    __syncthreads();
    const int res = scratch[warp] + incl - v;
    *total = scratch[32];
    __syncthreads();
    return res;
}

// The same over 64-bit values: the small-batch permutation scans three packed 21-bit counters
// at once (there T*k <= 4096*32 = 2^17, so each field's block total stays below 2^21 and no
// carry crosses into the next field).
__device__ unsigned long long block_exclusive_scan64(unsigned long long v, unsigned long long *scratch /* 33 */,
                                                     unsigned long long *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned long long incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned long long o = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const unsigned long long w = (lane < (int)(blockDim.x >> 5)) ? scratch[lane] : 0ull;
        unsigned long long wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const unsigned long long o = __shfl_up_sync(kFull, wi, off);
            if (lane >= off) wi += o;
        }
        scratch[lane] = wi - w;
        if (lane == 31) scratch[32] = wi;
    }
    __syncthreads();
    const unsigned long long res = scratch[warp] + incl - v;
    *total = scratch[32];
    __syncthreads();
    return res;
}

// Counts of one expert packed for one scan: rows, token tiles of width bn_a, of width bn_b.
constexpr int kPackBits = 21;
constexpr unsigned long long kPackMask = (1ull << kPackBits) - 1;
__device__ __forceinline__ unsigned long long pack3(int c, int bn_a, int bn_b)
{
    return (unsigned long long)c | ((unsigned long long)((c + bn_a - 1) / bn_a) << kPackBits) |
           ((unsigned long long)((c + bn_b - 1) / bn_b) << (2 * kPackBits));
}
__device__ __forceinline__ int field(unsigned long long v, int i) { return (int)((v >> (i * kPackBits)) & kPackMask); }

// One block of 1024 threads, thread e owns expert e:
//   counts[e] = sum over chunks; offsets = exclusive scan of counts;
//   chunk_hist[c, e] <- offsets[e] + assignments to e in chunks < c  (the chunk's base row);
//   ttile_a / ttile_b = exclusive scans of ceil(counts / bn) (token tiles per group).
__global__ void __launch_bounds__(1024) scan_kernel(int nchunks, int E, int32_t *__restrict__ chunk_hist,
                                                    int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                                                    int bn_a, int32_t *__restrict__ ttile_a, int bn_b,
                                                    int32_t *__restrict__ ttile_b)
{
    __shared__ int scratch[33];
    griddep_wait();
    griddep_launch_dependents();
    // Each thread walks its expert's column of chunk counts.  A store and the next load go
    // through the same pointer, so the compiler keeps them in order; the column is therefore
    // walked kBatch entries at a time, all loads of a batch issued before its stores, so that
    // a long column (4096 chunks at 2^20 tokens) costs nchunks / kBatch memory round trips.
    constexpr int kBatch = 16;
    const int e = threadIdx.x;
    int c = 0;
    if (e < E) {
        int ch = 0;
        for (; ch + kBatch <= nchunks; ch += kBatch) {
            int v[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) v[j] = chunk_hist[(size_t)(ch + j) * E + e];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                chunk_hist[(size_t)(ch + j) * E + e] = c;
                c += v[j];
            }
        }
        for (; ch < nchunks; ++ch) {
            const int v = chunk_hist[(size_t)ch * E + e];
            chunk_hist[(size_t)ch * E + e] = c;
            c += v;
        }
        counts[e] = c;
    }
    int total;
    const int off = block_exclusive_scan(e < E ? c : 0, scratch, &total);
    if (e < E) {
        offsets[e] = off;
        int ch = 0;
        for (; ch + kBatch <= nchunks; ch += kBatch) {
            int v[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) v[j] = chunk_hist[(size_t)(ch + j) * E + e];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) chunk_hist[(size_t)(ch + j) * E + e] = v[j] + off;
        }
        for (; ch < nchunks; ++ch) chunk_hist[(size_t)ch * E + e] += off;
    }
    if (e == 0) offsets[E] = total;
    const int ta = (e < E) ? (c + bn_a - 1) / bn_a : 0;
    const int oa = block_exclusive_scan(ta, scratch, &total);
    if (e < E) ttile_a[e] = oa;
    if (e == 0) ttile_a[E] = total;
    const int tb = (e < E) ? (c + bn_b - 1) / bn_b : 0;
    const int ob = block_exclusive_scan(tb, scratch, &total);
    if (e < E) ttile_b[e] = ob;
    if (e == 0) ttile_b[E] = total;
}

// Scatter of one chunk of 256 tokens (8 warps x 32).  Rows of expert e inside the chunk are
// handed out in token order: warp-level counts, an exclusive scan over the 8 warps (plus the
// chunk's base row), then each warp walks its 32 tokens in order (lane j < k handles slot j;
// the k experts of a token are distinct, so the k lanes never touch the same counter).  Each
// lane loads its 32 expert ids up front so the in-order walks touch shared memory only.
__global__ void __launch_bounds__(kChunk) scatter_kernel(const int32_t *__restrict__ topk_idx, int T, int E, int k,
                                                         const int32_t *__restrict__ chunk_base,
                                                         int32_t *__restrict__ perm_tok, int32_t *__restrict__ pos)
{
    __shared__ int cnt[kChunk / 32][kMaxE];
    griddep_wait();
    griddep_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * kChunk + warp * 32;
    int ids[32];
#pragma unroll
    for (int l = 0; l < 32; ++l) ids[l] = (t0 + l < T && lane < k) ? __ldg(topk_idx + (size_t)(t0 + l) * k + lane) : -1;
    for (int i = threadIdx.x; i < (kChunk / 32) * E; i += blockDim.x) cnt[i / E][i % E] = 0;
    __syncthreads();
#pragma unroll
    for (int l = 0; l < 32; ++l) {
        if (ids[l] >= 0) cnt[warp][ids[l]] += 1;
        __syncwarp();
    }
    __syncthreads();
    const int32_t *base = chunk_base + (size_t)blockIdx.x * E;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = __ldg(base + e);
        for (int w = 0; w < kChunk / 32; ++w) {
            const int c = cnt[w][e];
            cnt[w][e] = run;
            run += c;
        }
    }
    __syncthreads();
#pragma unroll
    for (int l = 0; l < 32; ++l) {
        if (ids[l] >= 0) {
            const int r = cnt[warp][ids[l]]++;
            perm_tok[r] = t0 + l;
            pos[(size_t)(t0 + l) * k + lane] = r;
        }
        __syncwarp();
    }
}

// Small batches: the whole permutation in one block of 1024 threads (after the router).  Each
// assignment sets bit t of its expert's token bitmap (E x ceil(T/32) words in shared memory);
// the row of assignment (t, e) is then offsets[e] + (tokens below t that chose e) = a
// per-(expert, word) prefix of bit counts plus the popcount of the bits below t in t's word --
// the (expert, token) order without a sort or a serial pass.
__global__ void __launch_bounds__(1024) permute_small_kernel(const int32_t *__restrict__ topk_idx, int T, int E,
                                                             int k, int32_t *__restrict__ counts,
                                                             int32_t *__restrict__ offsets,
                                                             int32_t *__restrict__ perm_tok, int32_t *__restrict__ pos,
                                                             int bn_a, int32_t *__restrict__ ttile_a, int bn_b,
                                                             int32_t *__restrict__ ttile_b)
{
    extern __shared__ int sm[];
    const int W = (T + 31) >> 5;
    int *s_scr = sm;                                           // 33 x 64-bit
    int *s_cnt = s_scr + 68;                                   // E
    // word-major [W][E]: in the per-expert prefix pass thread e walks its column, so the 32
    // lanes of a warp touch 32 consecutive words (no bank conflicts)
    uint32_t *mask = reinterpret_cast<uint32_t *>(s_cnt + E);  // W * E
    int *pre = reinterpret_cast<int *>(mask + (size_t)E * W);  // W * E
    int *s_idx = pre + (size_t)E * W;                          // T * k
    const int tid = threadIdx.x;
    griddep_wait();
    griddep_launch_dependents();
    for (int i = tid; i < E; i += 1024) s_cnt[i] = 0;
    for (int i = tid; i < E * W; i += 1024) mask[i] = 0;
    __syncthreads();
    for (int i = tid; i < T * k; i += 1024) {
        const int e = __ldg(topk_idx + i);
        const int t = i / k;
        s_idx[i] = e;
        atomicOr(&mask[(t >> 5) * E + e], 1u << (t & 31));
        atomicAdd(&s_cnt[e], 1);
    }
    __syncthreads();
    const int c = tid < E ? s_cnt[tid] : 0;
    unsigned long long tot;
    const unsigned long long o3 = block_exclusive_scan64(tid < E ? pack3(c, bn_a, bn_b) : 0ull,
                                                         reinterpret_cast<unsigned long long *>(s_scr), &tot);
    if (tid < E) {
        const int off = field(o3, 0);
        counts[tid] = c;
        offsets[tid] = off;
        ttile_a[tid] = field(o3, 1);
        ttile_b[tid] = field(o3, 2);
        int run = off;
        for (int w = 0; w < W; ++w) {
            pre[w * E + tid] = run;
            run += __popc(mask[w * E + tid]);
        }
    }
    if (tid == 0) {
        offsets[E] = field(tot, 0);
        ttile_a[E] = field(tot, 1);
        ttile_b[E] = field(tot, 2);
    }
    __syncthreads();
    for (int i = tid; i < T * k; i += 1024) {
        const int t = i / k;
        const int e = s_idx[i];
        const int w = t >> 5;
        const int r = pre[w * E + e] + __popc(mask[w * E + e] & ((1u << (t & 31)) - 1u));
        perm_tok[r] = t;
        pos[i] = r;
    }
}

size_t small_route_smem(int T, int E, int k)
{
    const size_t W = ((size_t)T + 31) / 32;
    return 4 * (68 + (size_t)E + 2 * (size_t)E * W + (size_t)T * k);
}

}  // namespace

cudaError_t launch_route_permute(const float *logits, const RouteBufs &b, int T, int E, int k, int bn_a, int bn_b,
                                 cudaStream_t s, int *check)
{
    cudaError_t e = launch_route(logits, T, E, k, b.topk_idx, b.topk_w, s, check);
    if (e != cudaSuccess) return e;
    return launch_permute_any(b, T, E, k, bn_a, bn_b, s);
}

cudaError_t launch_permute_any(const RouteBufs &b, int T, int E, int k, int bn_a, int bn_b, cudaStream_t s)
{
    cudaError_t e;
    const size_t smem = small_route_smem(T, E, k);
    if (T < 1 || T > 4096 || smem > 160 * 1024) return launch_permute(b, T, E, k, bn_a, bn_b, s);
    e = set_smem_limit(reinterpret_cast<const void *>(permute_small_kernel), (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(permute_small_kernel, dim3(1), dim3(1024), smem, s, b.topk_idx, T, E, k, b.counts, b.offsets,
                      b.perm_tok, b.pos, bn_a, b.ttile_a, bn_b, b.ttile_b);
}

int route_permute_launches(int T, int E, int k)
{
    if (T < 1) return 1;
    if (T > 4096 || small_route_smem(T, E, k) > 160 * 1024) return 4;
    return 2;
}

cudaError_t launch_route(const float *logits, int T, int E, int k, int32_t *topk_idx, float *topk_w,
                         cudaStream_t s, int *check, WeightPrefetch pf)
{
    if (T <= 0) return cudaSuccess;
    // prefetching blocks: spread over the SMs (a few 64 KB chunks each), since one SM issues
    // bulk prefetches at about its share of the L2 bandwidth
    const int npf = (int)std::min<uint32_t>(128u, 2 * pf.chunks);
    const dim3 grid((T + 7) / 8 + npf), block(256);
    const int epl = (E + 31) / 32;
    auto go = [&](auto kern) {
        return launch_pdl(kern, grid, block, 0, s, logits, T, E, k, topk_idx, topk_w, check, pf);
    };
    if (epl <= 1) return go(route_kernel<1>);
    if (epl <= 2) return go(route_kernel<2>);
    if (epl <= 4) return go(route_kernel<4>);
    if (epl <= 8) return go(route_kernel<8>);
    if (epl <= 16) return go(route_kernel<16>);
    return go(route_kernel<32>);
}

cudaError_t launch_permute(const RouteBufs &b, int T, int E, int k, int bn_a, int bn_b, cudaStream_t s)
{
    const int nchunks = (T + kChunk - 1) / kChunk;
    cudaError_t e = cudaSuccess;
    if (nchunks > 0) e = launch_pdl(hist_kernel, dim3(nchunks), dim3(kChunk), 0, s, b.topk_idx, T, E, k, b.chunk_hist);
    if (e == cudaSuccess)
        e = launch_pdl(scan_kernel, dim3(1), dim3(1024), 0, s, nchunks, E, b.chunk_hist, b.counts, b.offsets, bn_a,
                       b.ttile_a, bn_b, b.ttile_b);
    if (e == cudaSuccess && nchunks > 0)
        e = launch_pdl(scatter_kernel, dim3(nchunks), dim3(kChunk), 0, s, b.topk_idx, T, E, k, b.chunk_hist,
                       b.perm_tok, b.pos);
    return e;
}

}  // namespace moe
