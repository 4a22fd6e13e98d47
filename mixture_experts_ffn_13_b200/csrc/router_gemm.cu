// router_gemm.cu -- the router's logits, the dense 16-bit layer that feeds step A1:
// logits[T, E] = x[T, H] . W_router[E, H]^T, bf16 inputs, fp32 accumulation and output.
//
// Page "Flash-Next 在 GPU 上到底在算什麼", section "② 密集 16-bit 層": the router is one of the
// small dense layers every token passes through; it stays in 16 bits and runs on the tensor
// cores.  Page "把 397B MoE 榨進 TPU7x", section "數值驗證": the gating path is checked against a
// high-precision reference because small drifts can reorder the top-k.
//
// Design (B200): the same operand roles as the expert GEMMs -- the MMA's 128-row M side is a
// tile of router weight rows (experts), the N side a BN-token tile -- with a persistent grid
// over (expert tile, token tile) pairs, warp 0 issuing TMA loads of 64-element K slices
// (128-byte swizzle) into an NS-deep ring, warp 1 issuing tcgen05.mma.kind::f16 from one
// thread into one of two TMEM accumulators, and warps 2-5 writing the finished tile as fp32
// (lane = expert, consecutive lanes store consecutive logits of one token).
#include "gemm_common.cuh"
#include "launch.cuh"
#include "sm100.cuh"

#include <mutex>

namespace moe {

namespace {

constexpr int kRKE = 64;  // K elements per stage (128 bytes of bf16)

template <int BN>
struct RCfg {
    static constexpr int A_BYTES = kTileM * kRKE * 2;  // 16 KB
    static constexpr int B_BYTES = BN * kRKE * 2;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int NS = (208 * 1024) / STAGE < 12 ? (208 * 1024) / STAGE : 12;
    static constexpr int THREADS = 64 + 128;
    static constexpr int SMEM = 1024 + NS * STAGE + 8 * (2 * NS + 4) + 16;
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "1024-byte aligned tiles");
};

struct RouterArgs {
    int T, H, E;
    float *logits;
    int *status;
    uint64_t timeout_ns;
};

template <int BN>
__global__ void __launch_bounds__(RCfg<BN>::THREADS, 1)
    router_gemm_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                       const __grid_constant__ RouterArgs a)
{
    using C = RCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::NS * C::STAGE);
    uint64_t *empty = full + C::NS;
    uint64_t *accf = empty + C::NS;  // 2
    uint64_t *acce = accf + 2;       // 2
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(acce + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    uint64_t *drain_bar = reinterpret_cast<uint64_t *>(tmem_holder + 2);  // MMA drain on exit
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&accf[s], 1);
            mbar_init(&acce[s], 4);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_w);
        tma_prefetch_desc(&map_x);
    }
    constexpr int kCols = 2 * BN < 32 ? 32 : 2 * BN;
    if (warp == 1) {
        tmem_alloc(tmem_holder, kCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    griddep_wait();
    griddep_launch_dependents();

    const int net = (a.E + kTileM - 1) / kTileM;  // the last expert tile may be partial
    const int ntt = (a.T + BN - 1) / BN;
    const int total = net * ntt;
    const int nkc = a.H / kRKE;
    uint32_t issued = 0;  // producer: stages whose copies have been issued
    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_x = l2_policy_evict_last();
            uint32_t it = 0;
            for (int w = blockIdx.x; w < total; w += gridDim.x) {
                const int et = w % net, tt = w / net;  // consecutive tiles share the token tile
                for (int kc = 0; kc < nkc; ++kc, ++it) {
                    const int s = it % C::NS;
                    if (!mbar_wait(&empty[s], ((it / C::NS) & 1) ^ 1, abort_flag, a.status, a.timeout_ns)) goto done;
                    uint8_t *st = smem + s * C::STAGE;
                    issued = it + 1;
                    mbar_arrive_expect_tx(&full[s], C::STAGE);
                    tma_load_2d(st, &map_w, &full[s], kc * kRKE, et * kTileM);
                    tma_load_2d_hint(st + C::A_BYTES, &map_x, &full[s], kc * kRKE, tt * BN, pol_x);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t kIdesc = instr_desc(kTileM, BN, 1, 1);
            uint32_t it = 0, ti = 0;
            for (int w = blockIdx.x; w < total; w += gridDim.x, ++ti) {
                const int slot = ti & 1;
                if (!mbar_wait(&acce[slot], ((ti >> 1) & 1) ^ 1, abort_flag, a.status, a.timeout_ns)) goto done;
                tc_fence_after();
                const uint32_t d = tmem_base + slot * BN;
                for (int kc = 0; kc < nkc; ++kc, ++it) {
                    const int s = it % C::NS;
                    if (!mbar_wait(&full[s], (it / C::NS) & 1, abort_flag, a.status, a.timeout_ns)) goto done;
                    tc_fence_after();
                    uint8_t *st = smem + s * C::STAGE;
                    const uint64_t da = smem_desc_sw128(st), db = smem_desc_sw128(st + C::A_BYTES);
#pragma unroll
                    for (int kk = 0; kk < kRKE / 16; ++kk)
                        mma_bf16(d, da + 2 * kk, db + 2 * kk, kIdesc, (kc > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&empty[s]);
                }
                mma_commit(&accf[slot]);
            }
        }
    } else {
        const int q = warp & 3;
        const int e_in = q * 32 + lane;
        uint32_t ti = 0;
        for (int w = blockIdx.x; w < total; w += gridDim.x, ++ti) {
            const int et = w % net, tt = w / net;
            const int slot = ti & 1;
            const bool ok = mbar_wait(&accf[slot], (ti >> 1) & 1, abort_flag, a.status, a.timeout_ns);
            if (!__all_sync(0xffffffffu, ok)) goto done;
            tc_fence_after();
            const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + slot * BN;
            const int e = et * kTileM + e_in;
            const int t0 = tt * BN;
#pragma unroll
            for (int c0 = 0; c0 < BN; c0 += 16) {
                float v[16];
                tmem_ld16(tb + c0, v);
                tmem_wait_ld(v);
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    if (t0 + c0 + c < a.T && e < a.E) a.logits[(size_t)(t0 + c0 + c) * a.E + e] = v[c];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce[slot]);
        }
    }
done:
    // own asynchronous work first (already finished unless a role gave up early)
    if (warp == 0 && lane == 0)
        for (uint32_t j = issued > (uint32_t)C::NS ? issued - C::NS : 0; j < issued; ++j)
            mbar_wait_drain(&full[j % C::NS], (j / C::NS) & 1, a.timeout_ns);
    if (warp == 1 && lane == 0) mma_drain(drain_bar, a.timeout_ns);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, kCols);
    }
}

// Split-K form for batches too small to give every SM a tile: a cluster of S CTAs shares one
// (expert tile, token tile); CTA r accumulates K slices [r*nkc/S, (r+1)*nkc/S) in its own
// TMEM, the S-1 other CTAs store their 128 x BN partial tile into the shared memory of CTA 0
// (distributed shared memory) and arrive on its mbarrier; CTA 0 adds the partials in rank
// order (a fixed summation order, so results do not depend on timing) and stores the logits.
// Each CTA reads 1/S of the router-weight and token rows of the tile, which is what bounds
// the one-CTA-per-tile form at small T (every token tile re-reads the expert tile's weights).
template <int BN>
struct SCfg {
    static constexpr int A_BYTES = kTileM * kRKE * 2;
    static constexpr int B_BYTES = BN * kRKE * 2;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int NS = 4;
    static constexpr int MAX_S = 4;
    static constexpr int RED_BYTES = (MAX_S - 1) * kTileM * BN * 4;  // partials of CTAs 1..S-1
    static constexpr int THREADS = 64 + 128;
    static constexpr int SMEM = 1024 + NS * STAGE + RED_BYTES + 8 * (2 * NS + 2) + 16;
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "1024-byte aligned tiles");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

template <int BN>
__global__ void __launch_bounds__(SCfg<BN>::THREADS, 1)
    router_splitk_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                         const __grid_constant__ RouterArgs a, int S)
{
    using C = SCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *red = reinterpret_cast<float *>(smem + C::NS * C::STAGE);  // [S-1][128][BN] in CTA 0
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::NS * C::STAGE + C::RED_BYTES);
    uint64_t *empty = full + C::NS;
    uint64_t *accf = empty + C::NS;
    uint64_t *redbar = accf + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(redbar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    uint64_t *drain_bar = reinterpret_cast<uint64_t *>(tmem_holder + 2);  // MMA drain on exit
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(drain_bar, 1);
        mbar_init(redbar, 128 * (S - 1));  // every epilogue thread of CTAs 1..S-1
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_w);
        tma_prefetch_desc(&map_x);
    }
    constexpr int kCols = BN < 32 ? 32 : BN;
    if (warp == 1) {
        tmem_alloc(tmem_holder, kCols);
        tmem_relinquish();
    }
    tc_fence_before();
    cluster_sync();  // barriers of every CTA initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    griddep_wait();
    griddep_launch_dependents();

    const int net = (a.E + kTileM - 1) / kTileM;
    const int tile = blockIdx.x / S;
    const int et = tile % net, tt = tile / net;
    const int nkc = a.H / kRKE;
    const int k0 = (int)(((long)nkc * rank) / S), k1 = (int)(((long)nkc * (rank + 1)) / S);
    uint32_t issued = 0;  // producer: stages whose copies have been issued
    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_x = l2_policy_evict_last();
            for (int kc = k0, it = 0; kc < k1; ++kc, ++it) {
                const int s = it % C::NS;
                if (!mbar_wait(&empty[s], ((it / C::NS) & 1) ^ 1, abort_flag, a.status, a.timeout_ns)) break;
                uint8_t *st = smem + s * C::STAGE;
                issued = it + 1;
                mbar_arrive_expect_tx(&full[s], C::STAGE);
                tma_load_2d(st, &map_w, &full[s], kc * kRKE, et * kTileM);
                tma_load_2d_hint(st + C::A_BYTES, &map_x, &full[s], kc * kRKE, tt * BN, pol_x);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t kIdesc = instr_desc(kTileM, BN, 1, 1);
            bool ok = true;
            for (int kc = k0, it = 0; kc < k1 && ok; ++kc, ++it) {
                const int s = it % C::NS;
                ok = mbar_wait(&full[s], (it / C::NS) & 1, abort_flag, a.status, a.timeout_ns);
                if (!ok) break;
                tc_fence_after();
                uint8_t *st = smem + s * C::STAGE;
                const uint64_t da = smem_desc_sw128(st), db = smem_desc_sw128(st + C::A_BYTES);
#pragma unroll
                for (int kk = 0; kk < kRKE / 16; ++kk)
                    mma_bf16(tmem_base, da + 2 * kk, db + 2 * kk, kIdesc, (it > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&empty[s]);
            }
            if (ok) mma_commit(accf);
        }
    } else {
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const int e = et * kTileM + row;
        const int t0 = tt * BN;
        const bool ok = mbar_wait(accf, 0, abort_flag, a.status, a.timeout_ns);
        if (__all_sync(0xffffffffu, ok)) {
            tc_fence_after();
            const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16);
            if (rank != 0) {
                // partial tile -> CTA 0's buffer slot rank-1, row `row`, then release it there
                const uint32_t dst = cluster_map(red + ((size_t)(rank - 1) * kTileM + row) * BN, 0);
#pragma unroll
                for (int c0 = 0; c0 < BN; c0 += 16) {
                    float v[16];
                    tmem_ld16(tb + c0, v);
                    tmem_wait_ld(v);
#pragma unroll
                    for (int c = 0; c < 16; c += 4)
                        st_cluster_v4(dst + 4u * (c0 + c), v[c], v[c + 1], v[c + 2], v[c + 3]);
                }
                mbar_arrive_cluster(cluster_map(redbar, 0));
            } else if (mbar_wait_cluster(redbar, 0, abort_flag, a.status, a.timeout_ns)) {
#pragma unroll
                for (int c0 = 0; c0 < BN; c0 += 16) {
                    float v[16];
                    tmem_ld16(tb + c0, v);
                    tmem_wait_ld(v);
                    for (int r = 1; r < S; ++r) {
                        const float *pr = red + ((size_t)(r - 1) * kTileM + row) * BN + c0;
#pragma unroll
                        for (int c = 0; c < 16; ++c) v[c] += pr[c];
                    }
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        if (t0 + c0 + c < a.T && e < a.E) a.logits[(size_t)(t0 + c0 + c) * a.E + e] = v[c];
                }
            }
        }
    }
    // own asynchronous work first (already finished unless a role gave up early)
    if (warp == 0 && lane == 0)
        for (uint32_t j = issued > (uint32_t)C::NS ? issued - C::NS : 0; j < issued; ++j)
            mbar_wait_drain(&full[j % C::NS], (j / C::NS) & 1, a.timeout_ns);
    if (warp == 1 && lane == 0) mma_drain(drain_bar, a.timeout_ns);
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // CTA 0 stays resident until every partial has been stored into it
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, kCols);
    }
}

template <int BN>
cudaError_t launch_sk(const CUtensorMap &mw, const CUtensorMap &mx, const RouterArgs &a, int S, int tiles,
                      cudaStream_t s)
{
    using C = SCfg<BN>;
    auto kern = router_splitk_kernel<BN>;  // shared-memory attribute set by resident_clusters()
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = S;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(tiles * S);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, mw, mx, a, S);
}

// Clusters of S CTAs of this kernel that can be resident at once (0 if the query fails);
// computed once per device and cluster size (host calls stay off the per-call path).
template <int BN>
int resident_clusters_query(int S)
{
    using C = SCfg<BN>;
    auto kern = router_splitk_kernel<BN>;
    if (set_smem_limit(reinterpret_cast<const void *>(kern), C::SMEM) != cudaSuccess) return 0;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(S);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

constexpr int kMaxDev = 64;

template <int BN>
int resident_clusters(int S)
{
    static std::mutex mu;
    static int cache[kMaxDev][5];  // [device][S]: 0 = not queried, else count + 1
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev || S < 1 || S > 4) return 0;
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev][S] == 0) cache[dev][S] = resident_clusters_query<BN>(S) + 1;
    return cache[dev][S] - 1;
}

template <int BN>
cudaError_t launch_rt(const CUtensorMap &mw, const CUtensorMap &mx, const RouterArgs &a, int num_sms, cudaStream_t s)
{
    using C = RCfg<BN>;
    auto kern = router_gemm_kernel<BN>;
    cudaError_t e = set_smem_limit(reinterpret_cast<const void *>(kern), C::SMEM);
    if (e != cudaSuccess) return e;
    const int tiles = ((a.E + kTileM - 1) / kTileM) * ((a.T + BN - 1) / BN);
    const int grid = tiles < num_sms ? tiles : num_sms;
    return launch_pdl(kern, dim3(grid), dim3(C::THREADS), C::SMEM, s, mw, mx, a);
}

}  // namespace

// Router logits for T tokens (H a multiple of 64; any E -- a partial last expert tile reads
// zeros past row E and stores nothing there).  The token tile is the widest of 16..256 rows
// that still gives about 0.8 work items per SM: wide tiles read each router-weight byte for
// more tokens, narrow ones spread small batches over more SMs.
cudaError_t launch_router_gemm(const uint16_t *x, const uint16_t *w, float *logits, int T, int H, int E, int *status,
                               int num_sms, cudaStream_t s)
{
    if (T <= 0) return cudaSuccess;
    const long net = (E + kTileM - 1) / kTileM;
    int bn = 256;
    while (bn > 16 && net * ((T + bn - 1) / bn) < (long)num_sms * 4 / 5) bn >>= 1;
    // Split-K when the one-CTA-per-tile form leaves each CTA streaming many weight bytes for
    // few tokens: compare the bytes a CTA reads per wave of resident CTAs (cost model; the
    // split form must fit all its clusters in one wave).
    const int nkc = H / kRKE;
    auto waves = [&](long ctas) { return (ctas + num_sms - 1) / num_sms; };
    double best = (double)waves(net * ((T + bn - 1) / bn)) * (kTileM + bn) * H;
    int sbn = 0, sS = 1;
    for (int cand : {64, 32}) {
        const long tiles = net * ((T + cand - 1) / cand);
        for (int S : {4, 2}) {
            if (nkc < S) continue;
            const int fit = cand == 64 ? resident_clusters<64>(S) : resident_clusters<32>(S);
            if (tiles > fit) continue;
            const double cost = (double)(kTileM + cand) * H / S * 1.1;  // 1.1: the reduction
            if (cost < best) {
                best = cost;
                sbn = cand;
                sS = S;
            }
        }
    }
    CUtensorMap mw, mx;
    if (sbn) {
        int rc = encode_map_2d(&mw, w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, E, kRKE, kTileM, true);
        rc |= encode_map_2d(&mx, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, T, kRKE, sbn, true);
        if (rc) return cudaErrorInvalidValue;
        RouterArgs a{T, H, E, logits, status, kDefaultTimeoutNs};
        const int tiles = (int)(net * ((T + sbn - 1) / sbn));
        return sbn == 64 ? launch_sk<64>(mw, mx, a, sS, tiles, s) : launch_sk<32>(mw, mx, a, sS, tiles, s);
    }
    int rc = encode_map_2d(&mw, w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, E, kRKE, kTileM, true);
    rc |= encode_map_2d(&mx, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, T, kRKE, bn, true);
    if (rc) return cudaErrorInvalidValue;
    RouterArgs a{T, H, E, logits, status, kDefaultTimeoutNs};
    switch (bn) {
        case 256: return launch_rt<256>(mw, mx, a, num_sms, s);
        case 128: return launch_rt<128>(mw, mx, a, num_sms, s);
        case 64: return launch_rt<64>(mw, mx, a, num_sms, s);
        case 32: return launch_rt<32>(mw, mx, a, num_sms, s);
        default: return launch_rt<16>(mw, mx, a, num_sms, s);
    }
}

}  // namespace moe

namespace moe {

// Router logits, then the route kernel's softmax top-k on them (PDL-chained, so the route
// kernel's prologue overlaps the GEMM's tail).
cudaError_t launch_router_topk(const uint16_t *x, const uint16_t *w, float *logits, int32_t *topk_idx, float *topk_w,
                               int T, int H, int E, int k, int *status, int num_sms, cudaStream_t s)
{
    if (T <= 0) return cudaSuccess;
    cudaError_t e = launch_router_gemm(x, w, logits, T, H, E, status, num_sms, s);
    if (e != cudaSuccess) return e;
    return launch_route(logits, T, E, k, topk_idx, topk_w, s);
}

}  // namespace moe
