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
// result is deterministic and equal to sorting by (expert, token).
#include "moe_internal.h"

#include <math.h>

namespace moe {

namespace {

constexpr unsigned kFull = 0xffffffffu;

// One warp per token.  Lane l holds the logits of experts l, l+32, ...; k rounds of a warp
// arg-max (value desc, index asc) pick the experts; lane j keeps the j-th pick.
template <int EPL>
__global__ void __launch_bounds__(256) route_kernel(const float *__restrict__ logits, int T, int E, int k,
                                                    int32_t *__restrict__ topk_idx, float *__restrict__ topk_w)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= T) return;
    const float *L = logits + (size_t)t * E;
    float v[EPL];
    uint32_t taken = 0;  // bit i: element i of this lane is absent or already chosen
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        v[i] = (e < E) ? __ldg(L + e) : -INFINITY;
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
    // p_hat_j = exp(L_j - L_max) / sum_i exp(L_i - L_max), the sum taken in selection order.
    const float lmax = __shfl_sync(kFull, sel_v, 0);
    const float ex = (lane < k) ? expf(sel_v - lmax) : 0.0f;
    float denom = 0.0f;
    for (int j = 0; j < k; ++j) denom += __shfl_sync(kFull, ex, j);
    if (lane < k) {
        topk_idx[(size_t)t * k + lane] = sel_e;
        topk_w[(size_t)t * k + lane] = ex / denom;
    }
}

// Per-chunk expert histogram: chunk_hist[c, e] = assignments to e among tokens of chunk c.
__global__ void __launch_bounds__(kChunk) hist_kernel(const int32_t *__restrict__ topk_idx, int T, int E, int k,
                                                      int32_t *__restrict__ chunk_hist)
{
    __shared__ int h[kMaxE];
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
    const int e = threadIdx.x;
    int c = 0;
    if (e < E) {
        for (int ch = 0; ch < nchunks; ++ch) {
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
        for (int ch = 0; ch < nchunks; ++ch) chunk_hist[(size_t)ch * E + e] += off;
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
// handed out in token order: warp-level counts, an exclusive scan over the 8 warps, then each
// warp walks its 32 tokens in order (lane j < k handles slot j; the k experts of a token are
// distinct, so the k lanes never touch the same counter).
__global__ void __launch_bounds__(kChunk) scatter_kernel(const int32_t *__restrict__ topk_idx, int T, int E, int k,
                                                         const int32_t *__restrict__ chunk_base,
                                                         int32_t *__restrict__ perm_tok, int32_t *__restrict__ pos)
{
    __shared__ int cnt[kChunk / 32][kMaxE];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < (kChunk / 32) * E; i += blockDim.x) cnt[i / E][i % E] = 0;
    __syncthreads();
    const int t0 = blockIdx.x * kChunk + warp * 32;
    for (int l = 0; l < 32; ++l) {
        const int t = t0 + l;
        if (t < T && lane < k) cnt[warp][topk_idx[(size_t)t * k + lane]] += 1;
        __syncwarp();
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int w = 0; w < kChunk / 32; ++w) {
            const int c = cnt[w][e];
            cnt[w][e] = run;
            run += c;
        }
    }
    __syncthreads();
    const int32_t *base = chunk_base + (size_t)blockIdx.x * E;
    for (int l = 0; l < 32; ++l) {
        const int t = t0 + l;
        if (t < T && lane < k) {
            const int e = topk_idx[(size_t)t * k + lane];
            const int r = base[e] + cnt[warp][e];
            cnt[warp][e] += 1;
            perm_tok[r] = t;
            pos[(size_t)t * k + lane] = r;
        }
        __syncwarp();
    }
}

}  // namespace

cudaError_t launch_route(const float *logits, int T, int E, int k, int32_t *topk_idx, float *topk_w,
                         cudaStream_t s)
{
    if (T <= 0) return cudaSuccess;
    const dim3 grid((T + 7) / 8), block(256);
    const int epl = (E + 31) / 32;
    if (epl <= 1)
        route_kernel<1><<<grid, block, 0, s>>>(logits, T, E, k, topk_idx, topk_w);
    else if (epl <= 2)
        route_kernel<2><<<grid, block, 0, s>>>(logits, T, E, k, topk_idx, topk_w);
    else if (epl <= 4)
        route_kernel<4><<<grid, block, 0, s>>>(logits, T, E, k, topk_idx, topk_w);
    else if (epl <= 8)
        route_kernel<8><<<grid, block, 0, s>>>(logits, T, E, k, topk_idx, topk_w);
    else if (epl <= 16)
        route_kernel<16><<<grid, block, 0, s>>>(logits, T, E, k, topk_idx, topk_w);
    else
        route_kernel<32><<<grid, block, 0, s>>>(logits, T, E, k, topk_idx, topk_w);
    return cudaGetLastError();
}

cudaError_t launch_permute(const RouteBufs &b, int T, int E, int k, int bn_a, int bn_b, cudaStream_t s)
{
    const int nchunks = (T + kChunk - 1) / kChunk;
    if (nchunks > 0) hist_kernel<<<nchunks, kChunk, 0, s>>>(b.topk_idx, T, E, k, b.chunk_hist);
    scan_kernel<<<1, 1024, 0, s>>>(nchunks, E, b.chunk_hist, b.counts, b.offsets, bn_a, b.ttile_a, bn_b, b.ttile_b);
    if (nchunks > 0) scatter_kernel<<<nchunks, kChunk, 0, s>>>(b.topk_idx, T, E, k, b.chunk_hist, b.perm_tok, b.pos);
    return cudaGetLastError();
}

}  // namespace moe
