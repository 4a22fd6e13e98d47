// quant.cu -- step A2: FP8 activation quantisation with 512-element sub-channels, and the
// gathers that place activation rows in permuted (per-expert) order.
//
// Page "把 397B MoE 榨進 TPU7x：Google 拿到 4.7 倍加速", section "Kernel 手術台": the expert FFN
// runs on FP8 with 512-element sub-channel quantisation.  Per (row, 512-block):
// s = amax / 448 in fp32 (1 when amax == 0) and q = e4m3(x / s), rounded to nearest even
// with saturation (cvt.rn.satfinite).  Both divisions are IEEE round-to-nearest; an all-zero
// block stores zero codes.
#include "launch.cuh"
#include "moe_internal.h"

#include <cuda_bf16.h>

namespace moe {

namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

// Quantise 16 values (one lane's share of a 512-block held by one warp); returns the 16
// codes as a uint4 and the block scale.
__device__ __forceinline__ uint4 quant16(const float (&f)[16], bool valid, float *scale_out)
{
    float amax = 0.0f;
    if (valid)
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, off));
    uint4 q = make_uint4(0, 0, 0, 0);
    float s = 1.0f;
    if (amax > 0.0f) {
        s = __fdiv_rn(amax, 448.0f);
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t lo = cvt_e4m3x2(__fdiv_rn(f[4 * i + 0], s), __fdiv_rn(f[4 * i + 1], s));
            const uint32_t hi = cvt_e4m3x2(__fdiv_rn(f[4 * i + 2], s), __fdiv_rn(f[4 * i + 3], s));
            w[i] = lo | (hi << 16);
        }
        q = make_uint4(w[0], w[1], w[2], w[3]);
    }
    *scale_out = s;
    return q;
}

// One warp per (token row t, 512-block kb), 8 warps per block over the flattened (t, kb)
// range: quantise the block and write it to the k permuted rows pos[t, :] and to shared row t.
__global__ void __launch_bounds__(256) quant_x_fp8_kernel(const uint16_t *__restrict__ x, int T, int H, int k,
                                                          const int32_t *__restrict__ pos, uint8_t *__restrict__ xq,
                                                          float *__restrict__ sx, uint8_t *__restrict__ xq_sh,
                                                          float *__restrict__ sx_sh)
{
    griddep_wait();
    griddep_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nb = (H + kBlockK - 1) / kBlockK;
    const long wid = (long)blockIdx.x * 8 + warp;
    if (wid >= (long)T * nb) return;
    const int t = (int)(wid / nb);
    const int kb = (int)(wid - (long)t * nb);
    const int i0 = kb * kBlockK + lane * 16;
    const bool valid = i0 < H;
    float f[16] = {};
    if (valid) {
        const uint4 *p = reinterpret_cast<const uint4 *>(x + (size_t)t * H + i0);
        const uint4 a = __ldg(p), b = __ldg(p + 1);
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            f[2 * i] = bf16_bits_to_float(w[i] & 0xffffu);
            f[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
        }
    }
    float s;
    const uint4 q = quant16(f, valid, &s);
    for (int j = 0; j < k; ++j) {
        const int r = __ldg(pos + (size_t)t * k + j);
        if (valid) *reinterpret_cast<uint4 *>(xq + (size_t)r * H + i0) = q;
        if (lane == 0) sx[(size_t)r * nb + kb] = s;
    }
    if (xq_sh) {
        if (valid) *reinterpret_cast<uint4 *>(xq_sh + (size_t)t * H + i0) = q;
        if (lane == 0) sx_sh[(size_t)t * nb + kb] = s;
    }
}

// One warp per (row, 512-block), 8 warps per block: fp32 rows -> e4m3 rows + scales.
struct RowsSeg {
    const float *h;
    int R, K;
    uint8_t *q;
    float *sq;
};

// Two row segments (the routed h and the shared expert's h) in one launch: warps
// [0, R0*nb0) quantise segment 0, the next R1*nb1 warps segment 1.
__global__ void __launch_bounds__(256) quant_rows_fp8_kernel(RowsSeg s0, RowsSeg s1)
{
    griddep_wait();
    griddep_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    long wid = (long)blockIdx.x * 8 + warp;
    const long n0 = (long)s0.R * ((s0.K + kBlockK - 1) / kBlockK);
    const RowsSeg &sg = wid < n0 ? s0 : s1;
    if (wid >= n0) wid -= n0;
    const float *h = sg.h;
    const int K = sg.K;
    uint8_t *q = sg.q;
    float *sq = sg.sq;
    const int nb = (K + kBlockK - 1) / kBlockK;
    if (wid >= (long)sg.R * nb) return;
    const int r = (int)(wid / nb);
    const int kb = (int)(wid - (long)r * nb);
    const int i0 = kb * kBlockK + lane * 16;
    const bool valid = i0 < K;
    float f[16] = {};
    if (valid) {
        const float4 *p = reinterpret_cast<const float4 *>(h + (size_t)r * K + i0);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 v = __ldg(p + i);
            f[4 * i] = v.x;
            f[4 * i + 1] = v.y;
            f[4 * i + 2] = v.z;
            f[4 * i + 3] = v.w;
        }
    }
    float s;
    const uint4 qq = quant16(f, valid, &s);
    if (valid) *reinterpret_cast<uint4 *>(q + (size_t)r * K + i0) = qq;
    if (lane == 0) sq[(size_t)r * nb + kb] = s;
}

// grid T: copy bf16 token row t to the permuted rows pos[t, :] and to shared row t.  With
// `interleave`, every aligned block of 8 elements is stored in the order 0, 4, 1, 5, 2, 6, 3, 7
// (the K order in which the int4 GEMM unpacks its weights), else as it is.
__global__ void __launch_bounds__(128) gather_x_bf16_kernel(const uint16_t *__restrict__ x, int H, int k,
                                                            const int32_t *__restrict__ pos, uint16_t *__restrict__ xp,
                                                            uint16_t *__restrict__ xp_sh, bool interleave)
{
    griddep_wait();
    griddep_launch_dependents();
    const int t = blockIdx.x;
    const int n16 = H / 8;  // uint4 chunks of 8 bf16
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t * H);
    for (int c = threadIdx.x; c < n16; c += blockDim.x) {
        uint4 v = __ldg(src + c);
        if (interleave) {
            // words hold elements (0, 1), (2, 3), (4, 5), (6, 7); make them (0, 4), (1, 5), ...
            uint4 u;
            asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(u.x) : "r"(v.x), "r"(v.z));
            asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(u.y) : "r"(v.x), "r"(v.z));
            asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(u.z) : "r"(v.y), "r"(v.w));
            asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(u.w) : "r"(v.y), "r"(v.w));
            v = u;
        }
        for (int j = 0; j < k; ++j) {
            const int r = pos[(size_t)t * k + j];
            reinterpret_cast<uint4 *>(xp + (size_t)r * H)[c] = v;
        }
        if (xp_sh) reinterpret_cast<uint4 *>(xp_sh + (size_t)t * H)[c] = v;
    }
}

}  // namespace

cudaError_t launch_quant_x_fp8(const uint16_t *x, int T, int H, int k, const int32_t *pos, uint8_t *xq, float *sx,
                               uint8_t *xq_shared, float *sx_shared, cudaStream_t s)
{
    if (T <= 0) return cudaSuccess;
    const long warps = (long)T * ((H + kBlockK - 1) / kBlockK);
    return launch_pdl(quant_x_fp8_kernel, dim3((unsigned)((warps + 7) / 8)), dim3(256), 0, s, x, T, H, k, pos, xq, sx,
                      xq_shared, sx_shared);
}

cudaError_t launch_quant_rows_fp8(const float *h, int R, int K, uint8_t *q, float *sq, const float *h1, int R1,
                                  int K1, uint8_t *q1, float *sq1, cudaStream_t s)
{
    const RowsSeg a{h, R > 0 ? R : 0, K, q, sq}, b{h1, h1 && R1 > 0 ? R1 : 0, K1, q1, sq1};
    const long warps = (long)a.R * ((a.K + kBlockK - 1) / kBlockK) + (long)b.R * ((b.K + kBlockK - 1) / kBlockK);
    if (warps == 0) return cudaSuccess;
    return launch_pdl(quant_rows_fp8_kernel, dim3((unsigned)((warps + 7) / 8)), dim3(256), 0, s, a, b);
}

cudaError_t launch_gather_x_bf16(const uint16_t *x, int T, int H, int k, const int32_t *pos, uint16_t *xp,
                                 uint16_t *xp_shared, bool interleave, cudaStream_t s)
{
    if (T <= 0) return cudaSuccess;
    return launch_pdl(gather_x_bf16_kernel, dim3(T), dim3(128), 0, s, x, H, k, pos, xp, xp_shared, interleave);
}

}  // namespace moe
