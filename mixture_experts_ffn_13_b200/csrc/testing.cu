// testing.cu -- test entry points (include/moe_b200_testing.h): the library's bounded mbarrier
// wait, run on a barrier that nothing arrives at, and the FP8 quantisers on caller buffers.
#include "../../include/moe_b200_testing.h"
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace {

__global__ void bounded_wait_kernel(int *status, uint64_t timeout_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    // phase 0 of a fresh barrier with one expected arrival: never completes here
    mbar_wait(&bar, 0, &abort_flag, status, timeout_ns);
}

// MMA issue-rate microbenchmark: one CTA (a 2-CTA cluster for the pair forms) issues `count`
// tcgen05.mma back to back on operands already resident in shared memory (zeros) or tensor
// memory, optionally committing to an mbarrier every `commit_every` MMAs as the pipelined
// kernels do per stage, and records the cycles spent issuing and until the last MMA completed.
enum { kRateF16SS = 0, kRateF16TS = 1, kRateF8SS = 2, kRateF16Pair = 3, kRateF8Pair = 4 };
constexpr int kRateA = 128 * 128, kRateB = 256 * 128;
constexpr int kRateSmem = 1024 + kRateA + kRateB + 64;  // + done, step[2], fin0, holder, abort flag

template <int FORM>
__global__ void __launch_bounds__(128, 1)
    mma_rate_kernel(int N, int count, int commit_every, int flags, long long *cycles, int *status,
                    uint64_t timeout_ns)
{
    constexpr bool kPair = FORM >= kRateF16Pair;
    constexpr bool kF8 = FORM == kRateF8SS || FORM == kRateF8Pair;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *A = smem, *B = smem + kRateA;
    uint64_t *done = reinterpret_cast<uint64_t *>(smem + kRateA + kRateB);
    uint64_t *step = done + 1;  // two barriers: step[0], step[1]
    uint64_t *fin0 = step + 2;  // completion of the second issuing thread (two-issuer variant)
    uint32_t *holder = reinterpret_cast<uint32_t *>(fin0 + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(holder + 1);
    const int warp = threadIdx.x >> 5;
    const uint32_t rank = kPair ? cluster_ctarank() : 0;
    for (int i = threadIdx.x; i < (kRateA + kRateB) / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (threadIdx.x == 0) {
        mbar_init(done, 1);
        mbar_init(&step[0], 1);
        mbar_init(&step[1], 1);
        mbar_init(fin0, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the zeros, for the tensor cores
    if (warp == 1) {
        if (kPair) {
            tmem_alloc_pair(holder, 512);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(holder, 512);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    if (kPair)
        cluster_sync();
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *holder;
    if ((flags & 4) && !kPair) {
        // two issuing threads in different warps, each with its own accumulator, commit
        // barrier and half of the MMAs: does one thread's commit hold up the other's issue?
        __shared__ long long t_end[2];
        const int who = threadIdx.x == 0 ? 0 : (threadIdx.x == 64 ? 1 : -1);
        const uint32_t idesc = instr_desc(128, N, kF8 ? 0 : 1, kF8 ? 0 : 1);
        const uint64_t da = smem_desc_sw128(A), db = smem_desc_sw128(B);
        __syncthreads();
        const long long t0 = clock64();
        if (who >= 0) {
            const uint32_t d = tmem + (who ? 256 : 0);
            uint64_t *b = &step[who];
            const int per = commit_every > 0 ? commit_every : count / 2;
            for (int i = 0; i < count / 2;) {
                for (int j = 0; j < per && i < count / 2; ++j, ++i) {
                    const uint32_t acc = i > 0 ? 1u : 0u;
                    if constexpr (FORM == kRateF16SS) mma_bf16(d, da, db, idesc, acc);
                    if constexpr (FORM == kRateF16TS) mma_bf16_ts(d, tmem + 384, db, idesc, acc);
                    if constexpr (FORM == kRateF8SS) mma_f8(d, da, db, idesc, acc);
                }
                if (commit_every > 0) mma_commit(b);
            }
            uint64_t *fin = who ? done : fin0;
            mma_commit(fin);
            mbar_wait(fin, 0, abort_flag, status, timeout_ns);
            t_end[who] = clock64();
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            cycles[0] = (t_end[0] > t_end[1] ? t_end[0] : t_end[1]) - t0;
            cycles[1] = cycles[0];
        }
    } else if (threadIdx.x == 0 && rank == 0) {
        const uint32_t idesc = instr_desc(kPair ? 256 : 128, N, kF8 ? 0 : 1, kF8 ? 0 : 1);
        const uint64_t da = smem_desc_sw128(A), db = smem_desc_sw128(B);
        const long long t0 = clock64();
        // flags bit 0: alternate the accumulator between two TMEM regions (columns 0 and 256;
        // the TS form's A then sits at column 384) every commit group; bit 1: alternate the
        // commit between two mbarriers
        const uint32_t ta = tmem + ((flags & 1) ? 384 : 256);
        const int per = commit_every > 0 ? commit_every : count;  // MMAs per commit group
        int i = 0;
        for (int grp = 0; i < count; ++grp) {
            const uint32_t d = tmem + (((flags & 1) && (grp & 1)) ? 256 : 0);
            for (int j = 0; j < per && i < count; ++j, ++i) {
                const uint32_t acc = (j > 0 || (i > 0 && !(flags & 1))) ? 1u : 0u;
                if constexpr (FORM == kRateF16SS) mma_bf16(d, da, db, idesc, acc);
                if constexpr (FORM == kRateF16TS) mma_bf16_ts(d, ta, db, idesc, acc);
                if constexpr (FORM == kRateF8SS) mma_f8(d, da, db, idesc, acc);
                if constexpr (FORM == kRateF16Pair) mma_bf16_pair(d, da, db, idesc, acc);
                if constexpr (FORM == kRateF8Pair) mma_f8_pair(d, da, db, idesc, acc);
            }
            if (commit_every > 0) {
                uint64_t *b = &step[(flags & 2) ? (grp & 1) : 0];
                if constexpr (kPair)
                    mma_commit_pair(b, 1);
                else
                    mma_commit(b);
            }
        }
        const long long t1 = clock64();
        if constexpr (kPair)
            mma_commit_pair(done, 3);
        else
            mma_commit(done);
        const bool ok = mbar_wait(done, 0, abort_flag, status, timeout_ns);
        const long long t2 = clock64();
        cycles[0] = t1 - t0;
        cycles[1] = ok ? t2 - t0 : -1;
    }
    // the odd CTA's tensor memory is written until the MMAs complete
    if (kPair && rank == 1 && threadIdx.x == 0) mbar_wait(done, 0, abort_flag, status, timeout_ns);
    tc_fence_before();
    if (kPair)
        cluster_sync();
    else
        __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        if (kPair)
            tmem_dealloc_pair(tmem, 512);
        else
            tmem_dealloc(tmem, 512);
    }
}

template <int FORM>
cudaError_t launch_rate(int N, int count, int commit_every, int flags, long long *cycles, int *status,
                        cudaStream_t s)
{
    constexpr bool kPair = FORM >= kRateF16Pair;
    auto kern = mma_rate_kernel<FORM>;
    cudaError_t e = set_smem_limit(reinterpret_cast<const void *>(kern), kRateSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kPair ? 2 : 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kPair ? 2 : 1);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = kRateSmem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, N, count, commit_every, flags, cycles, status, kDefaultTimeoutNs);
}

}  // namespace
}  // namespace moe

extern "C" int moe_test_mma_rate(int32_t form, int32_t N, int32_t count, int32_t commit_every, int32_t flags,
                                 long long *cycles, int32_t *status, moe_stream_t stream)
{
    using namespace moe;
    if (!cycles || !status || count < 2 || count > (1 << 20) || commit_every < 0 || flags < 0 || flags > 7)
        return MOE_ERR_INVALID_ARG;
    const bool pair = form == kRateF16Pair || form == kRateF8Pair;
    // MMA N: a multiple of 16 in [16, 256]; the pair forms split N over the two CTAs
    if (N < 16 || N > 256 || N % 16 || (pair && N < 32)) return MOE_ERR_INVALID_ARG;
    if (form == kRateF16TS && (flags & 5) && N > 128) return MOE_ERR_INVALID_ARG;  // A sits at column 384
    if ((flags & 4) && (pair || (flags & 3))) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    switch (form) {
        case kRateF16SS: e = launch_rate<kRateF16SS>(N, count, commit_every, flags, cycles, status, s); break;
        case kRateF16TS: e = launch_rate<kRateF16TS>(N, count, commit_every, flags, cycles, status, s); break;
        case kRateF8SS: e = launch_rate<kRateF8SS>(N, count, commit_every, flags, cycles, status, s); break;
        case kRateF16Pair: e = launch_rate<kRateF16Pair>(N, count, commit_every, flags, cycles, status, s); break;
        case kRateF8Pair: e = launch_rate<kRateF8Pair>(N, count, commit_every, flags, cycles, status, s); break;
        default: return MOE_ERR_INVALID_ARG;
    }
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_test_bounded_wait(int32_t *status, int32_t timeout_us, moe_stream_t stream)
{
    if (!status || timeout_us < 1 || timeout_us > 1000000) return MOE_ERR_INVALID_ARG;
    moe::bounded_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(status, (uint64_t)timeout_us * 1000ull);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_test_quant_x(int32_t T, int32_t H, int32_t k, const uint16_t *x, const int32_t *pos, uint8_t *xq,
                                float *sx, moe_stream_t stream)
{
    if (T < 0 || H < 16 || H % 16 || k < 1 || k > moe::kMaxK) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !pos || !xq || !sx)) return MOE_ERR_INVALID_ARG;
    const void *ptrs[] = {x, pos, xq, sx};
    for (const void *p : ptrs)
        if (reinterpret_cast<uintptr_t>(p) & 15) return MOE_ERR_INVALID_ARG;
    const cudaError_t e = moe::launch_quant_x_fp8(x, T, H, k, pos, xq, sx, nullptr, nullptr, (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_test_quant_rows(int32_t R, int32_t K, const float *h, uint8_t *q, float *sq, moe_stream_t stream)
{
    if (R < 0 || K < 16 || K % 16) return MOE_ERR_INVALID_ARG;
    if (R > 0 && (!h || !q || !sq)) return MOE_ERR_INVALID_ARG;
    const void *ptrs[] = {h, q, sq};
    for (const void *p : ptrs)
        if (reinterpret_cast<uintptr_t>(p) & 15) return MOE_ERR_INVALID_ARG;
    const cudaError_t e = moe::launch_quant_rows_fp8(h, R, K, q, sq, nullptr, 0, 0, nullptr, nullptr,
                                                     (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
