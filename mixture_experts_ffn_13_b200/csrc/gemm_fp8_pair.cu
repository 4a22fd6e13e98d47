// gemm_fp8_pair.cu -- steps A4 and A5 for wide token tiles on CTA pairs: the FP8 grouped GEMMs of
// gemm_fp8.cu with each MMA spread over the tensor cores of two SMs (tcgen05 cta_group::2).
//
// Page "把 397B MoE 榨進 TPU7x：Google 拿到 4.7 倍加速", section "Kernel 手術台": the grouped GEMM
// fuses gate and up in one tile over 512-sub-channel FP8 and keeps its weight stream fed
// (triple-buffered weights on the TPU).  At prefill sizes the one-SM kernel is bound by how fast
// each SM can pull operand tiles into shared memory: every stage brings a 128-row weight slice
// and a 192-row activation slice for one 128 x 192 MMA tile.  Here two SMs (a 2-CTA cluster)
// share one 256 x 192 MMA: each CTA loads its own 128 weight rows but only HALF of the token
// rows, and the tensor cores of the pair read the other half from the peer's shared memory.  A
// stage then costs an SM 28 KB instead of 40 KB for the same MMA work, and seven stages fit in
// shared memory instead of five.
//
// Roles and synchronisation (both CTAs run every role except the MMA issuer):
//  * producer (warp 0): waits for its own stage to be free (the even CTA's MMA commits to the
//    `empty` barrier of BOTH CTAs), then loads its weight rows and its half of the token rows with
//    the cta_group::2 form of the TMA load, which signals the EVEN CTA's `full` barrier; the even
//    CTA's producer posts the byte count of both halves on that barrier.
//  * MMA issuer (warp 1, even CTA only): tcgen05.mma.cta_group::2.kind::f8f6f4, M = 256, N = the
//    tile's valid token rows rounded to 16; each 512-element K block into its own TMEM slot (two
//    slots of 192 columns), committed to the `accf` barrier of both CTAs.
//  * epilogue (12 warps per CTA): each CTA promotes its own 128 TMEM lanes (its weight rows) for
//    all N token columns, exactly as the one-SM kernel, and releases the slot on the even CTA's
//    `acce` barrier (remote arrive from the odd CTA), which counts the epilogue warps of both.
// Token split: for an MMA of N columns, column c < N/2 comes from the even CTA's shared memory
// row c and column c >= N/2 from the odd CTA's row c - N/2, so CTA r loads token rows
// row0 + r*N/2 .. + N/2 (in 32-row boxes) and column c always means token row0 + c.
// Every wait is bounded; a pair that gives up meets at the final cluster barrier, which both
// CTAs reach on every path, before tensor memory is released.
#include "moe_internal.h"
#include "gemm_common.cuh"
#include "launch.cuh"
#include "sm100.cuh"

#include <atomic>

namespace moe {

namespace {

constexpr int kKC = 128;  // K bytes per pipeline stage (one 128-byte swizzle row)
constexpr int kStagesPerBlock = kBlockK / kKC;
constexpr int kMaxKb = 16;
constexpr int kSmemLimit = 227 * 1024;

template <bool GATEUP>
struct PairCfg {
    static constexpr int BN = 192;                 // token rows of a pair tile (largest MMA N used)
    static constexpr int BH = BN / 2;              // token rows per CTA
    static constexpr int BOX = 32;                 // activation rows per TMA box
    static constexpr int EW = 12;                  // epilogue warps per CTA
    static constexpr int PARTS = EW / 4;
    static constexpr int CPW = BN / PARTS;         // token columns per epilogue thread
    static constexpr int THREADS = 64 + 32 * EW;
    static constexpr int RT_CTA = GATEUP ? kTileM / 2 : kTileM;  // output features per CTA
    static constexpr int RT = 2 * RT_CTA;          // output features per pair tile
    static constexpr int A_BYTES = kTileM * kKC;   // 16 KB
    static constexpr int B_BYTES = BH * kKC;       // 12 KB
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int SLOT_COLS = BN;
    static constexpr int NSLOT = 512 / SLOT_COLS;  // 2
    static constexpr int SX_BYTES = 2 * BN * kMaxKb * 4;  // activation scales, two tile buffers
    static constexpr int TT_BYTES = (4 * (kMaxE + 1) + 15) & ~15;
    static constexpr int BAR_BYTES = 8 * (2 * 16 + 2 * NSLOT) + 16 + 8;
    static constexpr int FIXED = 1024 + SX_BYTES + TT_BYTES + BAR_BYTES;
    static constexpr int NS_FIT = (kSmemLimit - FIXED) / STAGE_BYTES;
    static constexpr int NS = NS_FIT < 16 ? NS_FIT : 16;
    static constexpr int SMEM = FIXED + NS * STAGE_BYTES;
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "stage tiles must stay 1024-byte aligned");
    static_assert(CPW % 16 == 0 && CPW % 2 == 0, "epilogue split");
    static_assert(NS >= 4, "pipeline");
    static_assert((NS * STAGE_BYTES + SX_BYTES + TT_BYTES) % 16 == 0, "mbarriers must be 8-byte aligned");
    static_assert(BH % BOX == 0, "whole activation boxes per CTA");
};

__device__ __forceinline__ void epi_sync(int nthreads) { asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory"); }

// TMA loads whose completion is signalled on the even CTA's barrier (`bar_cluster` is a
// shared::cluster address); destination in this CTA's shared memory.
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, uint32_t bar_cluster, int x, int y,
                                                 uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_load_4d_pair(void *dst, const CUtensorMap *map, uint32_t bar_cluster, int c0,
                                                 int c1, int c2, int c3, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "l"(policy)
        : "memory");
}

template <bool GATEUP>
__global__ void __launch_bounds__(PairCfg<GATEUP>::THREADS, 1)
    gemm_fp8_pair_kernel(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmArgs args)
{
    using C = PairCfg<GATEUP>;
    constexpr int BN = C::BN, RT = C::RT, EW = C::EW;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *sxbuf = reinterpret_cast<float *>(smem + C::NS * C::STAGE_BYTES);  // [2][BN * kMaxKb]
    int *stt = reinterpret_cast<int *>(smem + C::NS * C::STAGE_BYTES + C::SX_BYTES);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::NS * C::STAGE_BYTES + C::SX_BYTES + C::TT_BYTES);
    uint64_t *empty = full + C::NS;
    uint64_t *accf = empty + C::NS;
    uint64_t *acce = accf + C::NSLOT;
    uint64_t *drain_bar = acce + C::NSLOT;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank() & 1u;
    const bool leader = rank == 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < C::NSLOT; ++s) {
            mbar_init(&accf[s], 1);
            mbar_init(&acce[s], 2 * EW);  // the epilogue warps of both CTAs
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < args.nseg; ++i) {
            tma_prefetch_desc(&maps.a0[i]);
            if (GATEUP) tma_prefetch_desc(&maps.a1[i]);
            tma_prefetch_desc(&maps.b[i]);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers initialised and tensor memory allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    griddep_wait();
    griddep_launch_dependents();
    load_ttile(args, stt);

    int tot0;
    const int total = total_tiles(args, BN, &tot0, RT);
    const int pair_id = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    int *status = args.status;
    const uint64_t tmo = args.timeout_ns;
    uint32_t issued = 0;  // producer: stages whose copies have been issued

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        const uint64_t pol_w = l2_policy_evict_first();
        const uint64_t pol_x = l2_policy_evict_last();
        uint32_t it = 0;
        for (int w = pair_id; w < total; w += npairs) {
            const TileInfo tl = decode_tile<BN, true, RT>(args, stt, w, tot0);
            const GemmSeg &sg = args.seg[tl.seg];
            const int nkc = sg.K / kKC;
            const int n_mma = min(BN, (tl.nrows + 15) & ~15);
            const int half = n_mma >> 1;                     // token rows this CTA holds
            const int nbox = (half + C::BOX - 1) / C::BOX;
            const int xrow0 = tl.row0 + (int)rank * half;
            const int wrow = tl.wrow + (int)rank * C::RT_CTA;
            const int nwa = GATEUP ? (sg.ilv4d ? 1 : 8) : 1;
            const uint32_t tx = 2u * (C::A_BYTES + nbox * C::BOX * kKC);  // both halves of the stage
            for (int kc = 0; kc < nkc; ++kc, ++it) {
                const int s = it % C::NS;
                const uint32_t ph = (it / C::NS) & 1;
                bool ok = true;
                if (lane == 0) {
                    ok = mbar_wait(&empty[s], ph ^ 1, abort_flag, status, tmo);
                    if (ok && leader) mbar_arrive_expect_tx(&full[s], tx);
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) goto done;
                issued = it + 1;
                uint8_t *st = smem + s * C::STAGE_BYTES;
                const uint32_t bar = cluster_map(&full[s], 0);
                const int x = kc * kKC;
                if (lane < nwa) {
                    if constexpr (GATEUP) {
                        if (sg.ilv4d) {
                            tma_load_4d_pair(st, &maps.a0[tl.seg], bar, x, 0, 0, wrow >> 4, pol_w);
                        } else {
                            const int q = lane >> 1, u = lane & 1;
                            tma_load_2d_pair(st + q * 4096 + u * 2048, u ? &maps.a1[tl.seg] : &maps.a0[tl.seg], bar,
                                             x, wrow + 16 * q, pol_w);
                        }
                    } else {
                        tma_load_2d_pair(st, &maps.a0[tl.seg], bar, x, wrow, pol_w);
                    }
                } else if (lane < nwa + nbox) {
                    const int j = lane - nwa;
                    tma_load_2d_pair(st + C::A_BYTES + j * C::BOX * kKC, &maps.b[tl.seg], bar, x, xrow0 + j * C::BOX,
                                     pol_x);
                }
                __syncwarp();
            }
        }
    } else if (warp == 1) {
        // ------------------------- MMA issuer (even CTA) --------------------------
        if (leader && lane == 0) {
            uint32_t it = 0, ai = 0;
            for (int w = pair_id; w < total; w += npairs) {
                const TileInfo tl = decode_tile<BN, true, RT>(args, stt, w, tot0);
                const int n_mma = min(BN, (tl.nrows + 15) & ~15);
                const uint32_t idesc = instr_desc(2 * kTileM, n_mma, 0, 0);
                const int K = args.seg[tl.seg].K;
                const int nkc = K / kKC;
                const int nkb = (K + kBlockK - 1) / kBlockK;
                for (int kb = 0; kb < nkb; ++kb, ++ai) {
                    const int slot = ai % C::NSLOT;
                    const uint32_t aph = (ai / C::NSLOT) & 1;
                    // released by both CTAs' epilogues (the odd CTA's arrive remotely, with
                    // release at cluster scope): acquire at cluster scope
                    if (!mbar_wait_cluster(&acce[slot], aph ^ 1, abort_flag, status, tmo)) goto done;
                    tc_fence_after();
                    const uint32_t d = tmem_base + slot * C::SLOT_COLS;
                    const int kc_end = min(nkc, (kb + 1) * kStagesPerBlock);
                    for (int kc = kb * kStagesPerBlock; kc < kc_end; ++kc, ++it) {
                        const int s = it % C::NS;
                        if (!mbar_wait(&full[s], (it / C::NS) & 1, abort_flag, status, tmo)) goto done;
                        tc_fence_after();
                        uint8_t *st = smem + s * C::STAGE_BYTES;
                        const uint64_t da = smem_desc_sw128(st);
                        const uint64_t db = smem_desc_sw128(st + C::A_BYTES);
#pragma unroll
                        for (int kk = 0; kk < kKC / 32; ++kk) {
                            const uint32_t acc = (kc > kb * kStagesPerBlock || kk > 0) ? 1u : 0u;
                            mma_f8_pair(d, da + 2 * kk, db + 2 * kk, idesc, acc);
                        }
                        mma_commit_pair(&empty[s], 3);
                    }
                    mma_commit_pair(&accf[slot], 3);
                }
            }
        }
    } else {
        // ------------------------------ epilogue ----------------------------------
        const int ew = warp - 2;
        const int q = warp & 3;
        const int cbase = (ew >> 2) * C::CPW;
        const int r = GATEUP ? q * 16 + (lane & 15) : q * 32 + lane;
        const int etid = ew * 32 + lane;
        const uint32_t acce_remote = leader ? 0u : cluster_map(&acce[0], 0);
        uint32_t ai = 0;
        int ti = 0;
        constexpr int NPF = (BN * kMaxKb) / (32 * EW);
        float pf[NPF];
        auto load_sx = [&](const TileInfo &t) {
            const GemmSeg &g = args.seg[t.seg];
            const int nk = (g.K + kBlockK - 1) / kBlockK;
#pragma unroll
            for (int j = 0; j < NPF; ++j) {
                const int i = etid + j * 32 * EW;
                if (i < BN * nk) {
                    const int c = i / nk, kb = i - c * nk;
                    const int row = min(t.row0 + c, g.rows - 1);
                    pf[j] = __ldg(g.sx + (size_t)row * nk + kb);
                }
            }
        };
        auto store_sx = [&](const TileInfo &t, float *dst) {
            const int nk = (args.seg[t.seg].K + kBlockK - 1) / kBlockK;
#pragma unroll
            for (int j = 0; j < NPF; ++j) {
                const int i = etid + j * 32 * EW;
                if (i < BN * nk) {
                    const int c = i / nk, kb = i - c * nk;
                    dst[kb * BN + c] = pf[j];
                }
            }
        };
        if (pair_id < total) {
            const TileInfo t0 = decode_tile<BN, true, RT>(args, stt, pair_id, tot0);
            load_sx(t0);
            store_sx(t0, sxbuf);
        }
        epi_sync(32 * EW);
        for (int w = pair_id; w < total; w += npairs, ++ti) {
            const TileInfo tl = decode_tile<BN, true, RT>(args, stt, w, tot0);
            const GemmSeg &sg = args.seg[tl.seg];
            const int nkb = (sg.K + kBlockK - 1) / kBlockK;
            const bool is_up = GATEUP && ((lane >= 16) != (sg.ilv4d && sg.up_lo));
            const float *sxs = sxbuf + (ti & 1) * (BN * kMaxKb);
            const int wn = w + npairs;
            TileInfo tn;
            if (wn < total) {
                tn = decode_tile<BN, true, RT>(args, stt, wn, tot0);
                load_sx(tn);
            }
            const int wrow = tl.wrow + (int)rank * C::RT_CTA;
            const float *sw0 = static_cast<const float *>(is_up ? sg.sw1 : sg.sw0) + (size_t)(wrow + r) * nkb;
            float acc[C::CPW];
#pragma unroll
            for (int c = 0; c < C::CPW; ++c) acc[c] = 0.0f;
            float s0n = __ldg(sw0);
            for (int kb = 0; kb < nkb; ++kb, ++ai) {
                const int slot = ai % C::NSLOT;
                const uint32_t aph = (ai / C::NSLOT) & 1;
                const float s0 = s0n;
                if (kb + 1 < nkb) s0n = __ldg(sw0 + kb + 1);
                const bool ok = mbar_wait(&accf[slot], aph, abort_flag, status, tmo);
                if (!__all_sync(0xffffffffu, ok)) goto done;
                tc_fence_after();
                const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + slot * C::SLOT_COLS + cbase;
                const float *sxk = sxs + kb * BN + cbase;
#pragma unroll
                for (int c0 = 0; c0 < C::CPW; c0 += 16) {
                    float v[16];
                    tmem_ld16(tb + c0, v);
                    tmem_wait_ld(v);
#pragma unroll
                    for (int c = 0; c < 16; ++c) acc[c0 + c] = fmaf(v[c], s0 * sxk[c0 + c], acc[c0 + c]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (leader)
                        mbar_arrive(&acce[slot]);
                    else
                        mbar_arrive_cluster(acce_remote + 8u * (uint32_t)slot);
                }
            }
            float *out = static_cast<float *>(sg.out);
            const int n = tl.nt * RT + (int)rank * C::RT_CTA + r;
            if constexpr (GATEUP) {
                // lane ^ 16 holds the other projection of feature n (as in the one-SM kernel)
                const bool odd = lane >= 16;
                float *orow = out + (size_t)(tl.row0 + cbase + (odd ? 1 : 0)) * sg.N + n;
#pragma unroll
                for (int c = 0; c < C::CPW; c += 2) {
                    const float other = __shfl_xor_sync(0xffffffffu, odd ? acc[c] : acc[c + 1], 16);
                    const float mine = odd ? acc[c + 1] : acc[c];
                    const float v = is_up ? silu_mul(other, mine) : silu_mul(mine, other);
                    if (cbase + c + (odd ? 1 : 0) < tl.nrows) orow[(size_t)c * sg.N] = v;
                }
            } else {
                constexpr int NREG = C::CPW / 32;
                int ctok[NREG];
                float cw[NREG];
                if (sg.accum) combine_cols(sg, tl.row0 + cbase, tl.nrows - cbase, lane, ctok, cw);
#pragma unroll
                for (int c = 0; c < C::CPW; ++c)
                    if (cbase + c < tl.nrows) down_out(sg, args, tl.row0 + cbase + c, c, n, acc[c], ctok, cw);
            }
            if (wn < total) store_sx(tn, sxbuf + ((ti + 1) & 1) * (BN * kMaxKb));
            epi_sync(32 * EW);
        }
    }
done:
    // own asynchronous work first: the even CTA's `full` barriers complete once both halves of
    // every issued stage have landed, and its MMAs have completed (already true unless a role
    // of either CTA gave up early); the cluster barrier keeps the odd CTA resident until then
    if (leader && warp == 0 && lane == 0)
        for (uint32_t j = issued > (uint32_t)C::NS ? issued - C::NS : 0; j < issued; ++j)
            mbar_wait_drain(&full[j % C::NS], (j / C::NS) & 1, tmo);
    if (leader && warp == 1 && lane == 0) {
        mma_commit_pair(drain_bar, 1);
        mbar_wait_drain(drain_bar, 0, tmo);
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, 512);
    }
}

// Pairs of CTAs that can be resident at once (one CTA per SM); cached per kernel and device.
template <bool GATEUP>
int resident_pairs(int num_sms)
{
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    int v = cached[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
    using C = PairCfg<GATEUP>;
    auto kern = gemm_fp8_pair_kernel<GATEUP>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess) return 0;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms & ~1);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess) return 0;
    v = clusters < num_sms / 2 ? clusters : num_sms / 2;
    cached[dev].store(v, std::memory_order_relaxed);
    return v;
}

template <bool GATEUP>
cudaError_t launch_pair(const GemmMaps &maps, const GemmArgs &args, int num_sms, cudaStream_t s)
{
    using C = PairCfg<GATEUP>;
    const int pairs = resident_pairs<GATEUP>(num_sms);  // also sets the shared-memory attribute
    if (pairs < 1) return cudaErrorInvalidConfiguration;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, gemm_fp8_pair_kernel<GATEUP>, maps, args);
}

}  // namespace

bool gemm_fp8_pair_fits(bool gateup, const GemmArgs &args)
{
    // pair tiles cover 128 features of gate|up (I a multiple of 128) or 256 rows of down
    // (H a multiple of 256), K <= 8192 for the staged activation scales
    for (int i = 0; i < args.nseg; ++i) {
        if (args.seg[i].N % (gateup ? 128 : 256)) return false;
        if (args.seg[i].K > kMaxKb * kBlockK) return false;
    }
    return true;
}

cudaError_t launch_gemm_fp8_pair(bool gateup, const GemmMaps &maps, const GemmArgs &args, int num_sms, cudaStream_t s)
{
    if (!gemm_fp8_pair_fits(gateup, args)) return cudaErrorInvalidValue;
    return gateup ? launch_pair<true>(maps, args, num_sms, s) : launch_pair<false>(maps, args, num_sms, s);
}

}  // namespace moe
