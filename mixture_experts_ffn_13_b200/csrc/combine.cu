// combine.cu -- step A6: the probability-weighted un-permute and combine.
//
// Page "TPU推理外部化全面加速：InferenceX首份第三方性能數據發布", section "优化 MoE 路由与专家内核":
// expert outputs are un-permuted back to token order and summed with the top-k weights; the
// shared expert's output is added with weight 1 (page "把 397B MoE 榨進 TPU7x", section
// "稀疏在哪裡": the shared expert runs for every token).  Sums are fp32, in slot order j = 0..k-1
// then the shared term; the result is rounded to bf16 (round to nearest even).
#include "launch.cuh"
#include "moe_internal.h"

#include <cuda_bf16.h>

namespace moe {

namespace {

// grid (T, ceil(H/1024)), 256 threads: each thread owns 4 consecutive hidden features.  The
// token's k (row, weight) pairs are staged in shared memory once per block, so the k row loads
// of a thread do not each wait behind a load of their row index.
// With `check` set (checked mode), a permuted row index outside [0, rows) records
// MOE_ERR_BOUNDS in *check and the token's output is left unspecified (the row is not read).
__global__ void __launch_bounds__(256) combine_kernel(const float *__restrict__ y, const float *__restrict__ ysh,
                                                      const int32_t *__restrict__ pos,
                                                      const float *__restrict__ topk_w, int H, int k,
                                                      uint16_t *__restrict__ out, int rows, int *check)
{
    __shared__ int s_row[kMaxK];
    __shared__ float s_w[kMaxK];
    griddep_wait();
    griddep_launch_dependents();
    const int t = blockIdx.x;
    if (threadIdx.x < k) {
        int r = __ldg(pos + (size_t)t * k + threadIdx.x);
        if (check && (r < 0 || r >= rows)) {
            atomicCAS(check, 0, MOE_ERR_BOUNDS);
            r = 0;
        }
        s_row[threadIdx.x] = r;
        s_w[threadIdx.x] = __ldg(topk_w + (size_t)t * k + threadIdx.x);
    }
    __syncthreads();
    const int c = blockIdx.y * blockDim.x + threadIdx.x;  // float4 index within the row
    if (c >= H / 4) return;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int j = 0; j < k; ++j) {
        const int r = s_row[j];
        const float w = s_w[j];
        const float4 v = __ldg(reinterpret_cast<const float4 *>(y + (size_t)r * H) + c);
        acc.x = fmaf(w, v.x, acc.x);
        acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z);
        acc.w = fmaf(w, v.w, acc.w);
    }
    if (ysh) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(ysh + (size_t)t * H) + c);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
    }
    const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 o;
    o.x = *reinterpret_cast<const uint32_t *>(&lo);
    o.y = *reinterpret_cast<const uint32_t *>(&hi);
    reinterpret_cast<uint2 *>(out + (size_t)t * H)[c] = o;
}

}  // namespace

cudaError_t launch_combine(const float *y, const float *y_shared, const int32_t *pos, const float *topk_w, int T,
                           int H, int k, uint16_t *out, cudaStream_t s, int *check)
{
    if (T <= 0) return cudaSuccess;
    return launch_pdl(combine_kernel, dim3(T, (H / 4 + 255) / 256), dim3(256), 0, s, y, y_shared, pos, topk_w, H, k,
                      out, T * k, check);
}

}  // namespace moe
