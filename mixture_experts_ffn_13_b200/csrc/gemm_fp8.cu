// gemm_fp8.cu -- steps A4 and A5: persistent grouped GEMMs over FP8 expert weights with
// 512-element sub-channel scales, on the 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
// Page "把 397B MoE 榨進 TPU7x：Google 拿到 4.7 倍加速", section "Kernel 手術台": the grouped GEMM
// fuses the gate and up projections in one tile, uses 512-sub-channel FP8, and sizes each
// expert's work by its real row count instead of a padded maximum.  Page "Flash-Next 在 GPU 上
// 到底在算什麼", section "① 專家 FFN": each expert is input x A -> activation -> x B.
//
// Design (B200):
//  * Operand roles are swapped: the MMA's M side (128 rows) is a tile of WEIGHT rows and its N
//    side is a tile of BN token rows of one expert group, so a decode-sized group (a handful
//    of tokens) still fills the 128-row MMA and the kernel streams weights at full width.
//  * One CTA per SM, persistent over a flat list of (group, weight-row tile, token tile)
//    work items; per group the list is built from the routed row counts, so empty experts
//    cost nothing and hot experts get many token tiles.
//  * Warp roles: warp 0 issues TMA loads of 128-byte-wide K slices (weights with an
//    evict-first L2 hint, activations evict-last) into an NS-deep ring of shared-memory
//    stages; warp 1 issues tcgen05.mma (E4M3 x E4M3 -> F32) from one thread; the remaining
//    EW warps are the epilogue (EW/4 warps per 32-lane TMEM quarter, each owning a slice of
//    the BN token columns so the fp32 accumulators stay in registers).
//  * Sub-channel promotion: the scales change every 512 elements of K for both operands, so
//    each 512-block gets its own TMEM accumulator slot (a ring of slots covering all 512
//    TMEM columns).  The epilogue reads a finished slot, multiplies it by
//    s_w[row, kb] * s_x[token, kb] and adds it into fp32 registers, then frees the slot, so
//    the MMAs of the next blocks overlap the promotion of the previous ones.  Wide tiles stage
//    the tile's activation scales s_x[row0 .. row0+BN, :] in shared memory once per tile
//    (double-buffered across tiles up to 128 rows, one buffer above) and prefetch the weight
//    scales a block ahead; narrow tiles read both through L1 in the promotion loop.
//  * gate|up, paired form (narrow token tiles): two 128-row weight tiles per stage (gate and
//    up) share one activation tile and accumulate into two TMEM regions; the epilogue computes
//    h = silu(G) * U in fp32 and stores it.
//  * gate|up, interleaved form (token tiles of up to 192 rows): one 128-row weight tile holds 64
//    gate rows and the matching 64 up rows, 16 of each per 32-lane TMEM quarter (gate rows at
//    lanes 0-15, up rows at lanes 16-31), so one MMA per K step covers both and each thread's
//    partner (lane ^ 16) holds the other projection of the same feature for the SwiGLU.  Each
//    weight byte then meets up to 192 tokens per pass through shared memory, which is what
//    bounds the narrow forms at prefill sizes (shared-memory bandwidth, not HBM).  The whole
//    interleaved weight tile is one 4-D TMA box: (128 K bytes, 16 rows, {gate, up}, 4 row
//    groups), the {gate, up} dimension's stride being the distance between the two arrays.
//  * down: one weight tile; y is stored in fp32.
//  * Every token tile loads its activations as one BN-row box (a TMA copy has a fixed cost of
//    the order of 0.1 us in the SM's copy engine, so a stage is as few copies as possible), and
//    wide tiles size the MMA's N to the tile's valid rows rounded up to 16.  The producer warp
//    issues a wide stage's copies from separate lanes, one copy each.
#include "moe_internal.h"
#include "gemm_common.cuh"
#include "launch.cuh"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int kKC = 128;     // K elements (bytes) per pipeline stage = one 128-byte swizzle row
constexpr int kStagesPerBlock = kBlockK / kKC;
constexpr int kMaxKb = 16;   // activation-scale staging holds up to 16 blocks (K <= 8192)
constexpr int kSmemLimit = 227 * 1024;

// Activation boxes: every tile loads its BN rows as one box.  A TMA copy costs the SM's copy
// engine on the order of a hundred nanoseconds whatever its size (measured: a wide stage of four
// copies took ~0.48 us to issue whether it held 40 KB or 28 KB), so a stage is as few copies as
// possible; rows past the tensor's end are zero-filled and rows past the tile's group are never
// used (the MMA's N covers the valid rows).
template <int BN>
struct BoxOf {
    static constexpr int ROWS = BN;
    static constexpr int BYTES = ROWS * kKC;
};

enum { kModeDown = 0, kModePair = 1, kModeInterleaved = 2 };

template <int BN, int MODE, int EW>
struct Fp8Cfg {
    static constexpr bool GATEUP = MODE != kModeDown;
    static constexpr bool PAIR = MODE == kModePair;
    static constexpr bool ILV = MODE == kModeInterleaved;
    static constexpr int RT = ILV ? kTileM / 2 : kTileM;  // output features per tile
    static constexpr int NA = PAIR ? 2 : 1;
    static constexpr int A_BYTES = kTileM * kKC;
    // activation rows a stage holds: the tile's box
    static constexpr int B_ROWS = BN;
    static constexpr int B_BYTES = B_ROWS * kKC;
    static constexpr int STAGE_BYTES = NA * A_BYTES + B_BYTES;
    static constexpr int SLOT_COLS = NA * BN;
    static constexpr int NSLOT = 512 / SLOT_COLS;
    static constexpr int EPI_WARPS = EW;
    static constexpr int PARTS = EW / 4;           // epilogue warps per TMEM lane quarter
    static constexpr int CPW = BN / PARTS;         // token columns per epilogue thread
    static constexpr int THREADS = 64 + 32 * EW;
    // Every tile keeps the block within 196 KB of shared memory, so that the shared-memory
    // carve-out leaves ~60 KB of L1 (the narrow tiles' inline scale loads, the epilogues' weight
    // scale loads).  That measured faster than a deeper ring in the largest carve-out, for the
    // narrow decode tiles and for the 192-row prefill tiles alike (four stages instead of five:
    // prefill 3.19 -> 3.03 ms on the same box).  Wide tiles (BN >= 64) stage activation scales
    // and the tile-prefix table in shared memory; tiles up to 128 rows double-buffer the scales
    // across tiles, wider tiles keep one buffer.
    static constexpr bool WIDE = BN >= 64;
    static constexpr int SX_BUFS = BN > 128 ? 1 : 2;
    static constexpr int SX_BYTES = WIDE ? SX_BUFS * BN * kMaxKb * 4 : 0;
    static constexpr int TT_BYTES = WIDE ? (4 * (kMaxE + 1) + 15) & ~15 : 0;  // keeps the mbarriers 8-byte aligned
    static constexpr int BAR_BYTES = 8 * (2 * 16 + 2 * NSLOT) + 16;
    static constexpr int FIXED = 1024 + SX_BYTES + TT_BYTES + BAR_BYTES;
    static constexpr int NS_FIT = (kSmemLimit - FIXED) / STAGE_BYTES;
    static constexpr int NS_L1 = (196 * 1024 - FIXED) / STAGE_BYTES;
    static constexpr int NS_CAP = NS_L1 < NS_FIT ? NS_L1 : NS_FIT;
    static constexpr int NS = NS_CAP < 16 ? NS_CAP : 16;
    static constexpr int SMEM = FIXED + NS * STAGE_BYTES;
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "stage tiles must stay 1024-byte aligned");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M=128 is a multiple of 16 in [16, 256]");
    static_assert(EW % 4 == 0 && CPW % 16 == 0, "epilogue split");
    static_assert(!ILV || CPW % 2 == 0, "interleaved stores pair columns");
    static_assert(NSLOT >= 1 && NS >= 2, "pipeline");
    static_assert((NS * STAGE_BYTES + SX_BYTES + TT_BYTES) % 16 == 0, "mbarriers must be 8-byte aligned");
};

// Named barrier among the EW epilogue warps (ids 2..2+EW-1); barrier 0 is __syncthreads.
__device__ __forceinline__ void epi_sync(int nthreads) { asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory"); }

template <int BN, int MODE, int EW>
__global__ void __launch_bounds__(Fp8Cfg<BN, MODE, EW>::THREADS, 1)
    gemm_fp8_kernel(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmArgs args)
{
    using C = Fp8Cfg<BN, MODE, EW>;
    constexpr bool GATEUP = C::GATEUP;
    constexpr int RT = C::RT;
    constexpr int kBoxRows = BoxOf<BN>::ROWS, kBoxB = BoxOf<BN>::BYTES;
    // Wide token tiles stage the tile's activation scales in shared memory; narrow (decode)
    // tiles read them straight from L2 in the promotion loop, which measured faster there.
    constexpr bool kStageSx = C::WIDE;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *sxbuf = reinterpret_cast<float *>(smem + C::NS * C::STAGE_BYTES);  // [SX_BUFS][BN * kMaxKb]
    int *stt = reinterpret_cast<int *>(smem + C::NS * C::STAGE_BYTES + C::SX_BYTES);  // [E + 1]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::NS * C::STAGE_BYTES + C::SX_BYTES + C::TT_BYTES);
    uint64_t *empty = full + C::NS;
    uint64_t *accf = empty + C::NS;
    uint64_t *acce = accf + C::NSLOT;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(acce + C::NSLOT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    uint64_t *drain_bar = reinterpret_cast<uint64_t *>(tmem_holder + 2);  // MMA drain on exit

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < C::NSLOT; ++s) {
            mbar_init(&accf[s], 1);
            mbar_init(&acce[s], C::EPI_WARPS);
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
        tmem_alloc(tmem_holder, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    // everything above overlaps the previous kernel's tail; activations, offsets and tile
    // prefixes are read only after it has completed
    griddep_wait();
    griddep_launch_dependents();
    if constexpr (kStageSx) load_ttile(args, stt);
    const int *ttab = kStageSx ? stt : args.ttile;

    int tot0;
    const int total = total_tiles(args, BN, &tot0, RT);
    int *status = args.status;
    const uint64_t tmo = args.timeout_ns;
    uint32_t issued = 0;  // producer: stages whose copies have been issued

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        // Wide tiles: lane 0 claims a free stage and posts its byte count; then each lane
        // issues at most one of the stage's TMA copies, so a stage of several boxes is issued
        // in parallel rather than one copy after another.  Narrow tiles (two copies a stage)
        // run the producer on lane 0 alone, which measured faster there.
        if (!C::WIDE && lane != 0) goto done;
        const uint64_t pol_w = l2_policy_evict_first();
        const uint64_t pol_x = l2_policy_evict_last();
        uint32_t it = 0;
        for (int w = blockIdx.x; w < total; w += gridDim.x) {
            const TileInfo tl = decode_tile<BN, kStageSx, RT>(args, ttab, w, tot0);
            const GemmSeg &sg = args.seg[tl.seg];
            const int nkc = sg.K / kKC;
            // activation copies: one box of the whole BN-row tile
            const int nbox = 1;
            // weight copies: the paired form loads two 128-row tiles; the interleaved form one
            // 4-D box or eight 16-row boxes
            const int nwa = C::ILV ? (sg.ilv4d ? 1 : 8) : C::NA;
            const uint32_t tx = C::NA * C::A_BYTES + nbox * kBoxB;
            for (int kc = 0; kc < nkc; ++kc, ++it) {
                const int s = it % C::NS;
                const uint32_t ph = (it / C::NS) & 1;
                bool ok = true;
                if (lane == 0) {
                    ok = mbar_wait(&empty[s], ph ^ 1, abort_flag, status, tmo);
                    if (ok) mbar_arrive_expect_tx(&full[s], tx);
                }
                if constexpr (C::WIDE) ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) goto done;
                issued = it + 1;
                uint8_t *st = smem + s * C::STAGE_BYTES;
                const int x = kc * kKC;
                if constexpr (!C::WIDE) {
                    tma_load_2d_hint(st, &maps.a0[tl.seg], &full[s], x, tl.wrow, pol_w);
                    if (C::PAIR) tma_load_2d_hint(st + C::A_BYTES, &maps.a1[tl.seg], &full[s], x, tl.wrow, pol_w);
                    tma_load_2d_hint(st + C::NA * C::A_BYTES, &maps.b[tl.seg], &full[s], x, tl.row0, pol_x);
                    continue;
                }
                if (lane < nwa) {
                    if constexpr (C::ILV) {
                        if (sg.ilv4d) {
                            tma_load_4d_hint(st, &maps.a0[tl.seg], &full[s], x, 0, 0, tl.wrow >> 4, pol_w);
                        } else {
                            // lane 2q loads gate rows wrow+16q.. to tile rows 32q.., lane 2q+1 the
                            // matching up rows to tile rows 32q+16..
                            const int q = lane >> 1, u = lane & 1;
                            tma_load_2d_hint(st + q * 4096 + u * 2048, u ? &maps.a1[tl.seg] : &maps.a0[tl.seg],
                                             &full[s], x, tl.wrow + 16 * q, pol_w);
                        }
                    } else {
                        tma_load_2d_hint(st + lane * C::A_BYTES, lane ? &maps.a1[tl.seg] : &maps.a0[tl.seg],
                                         &full[s], x, tl.wrow, pol_w);
                    }
                } else if (lane < nwa + nbox) {
                    const int j = lane - nwa;
                    tma_load_2d_hint(st + C::NA * C::A_BYTES + j * kBoxB, &maps.b[tl.seg], &full[s], x,
                                     tl.row0 + j * kBoxRows, pol_x);
                }
                __syncwarp();
            }
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0) {
            uint32_t it = 0, ai = 0;
            for (int w = blockIdx.x; w < total; w += gridDim.x) {
                const TileInfo tl = decode_tile<BN, kStageSx, RT>(args, ttab, w, tot0);
                // MMA N = the tile's valid rows rounded up to 16 for wide tiles (a group's last,
                // partial token tile costs no tensor-core work for absent rows); narrow
                // decode tiles keep N = BN, which measured faster
                const int n_mma = kStageSx ? min(BN, (tl.nrows + 15) & ~15) : BN;
                const uint32_t kIdesc = instr_desc(kTileM, n_mma, 0, 0);
                const int K = args.seg[tl.seg].K;
                const int nkc = K / kKC;
                const int nkb = (K + kBlockK - 1) / kBlockK;
                for (int kb = 0; kb < nkb; ++kb, ++ai) {
                    const int slot = ai % C::NSLOT;
                    const uint32_t aph = (ai / C::NSLOT) & 1;
                    if (!mbar_wait(&acce[slot], aph ^ 1, abort_flag, status, tmo)) goto done;
                    tc_fence_after();
                    const uint32_t d0 = tmem_base + slot * C::SLOT_COLS;
                    const uint32_t d1 = d0 + BN;
                    const int kc_end = min(nkc, (kb + 1) * kStagesPerBlock);
                    for (int kc = kb * kStagesPerBlock; kc < kc_end; ++kc, ++it) {
                        const int s = it % C::NS;
                        const uint32_t ph = (it / C::NS) & 1;
                        if (!mbar_wait(&full[s], ph, abort_flag, status, tmo)) goto done;
                        tc_fence_after();
                        uint8_t *st = smem + s * C::STAGE_BYTES;
                        const uint64_t da0 = smem_desc_sw128(st);
                        const uint64_t da1 = smem_desc_sw128(st + C::A_BYTES);
                        const uint64_t db = smem_desc_sw128(st + C::NA * C::A_BYTES);
#pragma unroll
                        for (int kk = 0; kk < kKC / 32; ++kk) {
                            const uint32_t acc = (kc > kb * kStagesPerBlock || kk > 0) ? 1u : 0u;
                            mma_f8(d0, da0 + 2 * kk, db + 2 * kk, kIdesc, acc);
                            if (C::PAIR) mma_f8(d1, da1 + 2 * kk, db + 2 * kk, kIdesc, acc);
                        }
                        mma_commit(&empty[s]);
                    }
                    mma_commit(&accf[slot]);
                }
            }
        }
    } else {
        // ------------------------------ epilogue ----------------------------------
        const int ew = warp - 2;
        const int q = warp & 3;               // TMEM lanes 32q..32q+31 are reachable from this warp
        const int cbase = (ew >> 2) * C::CPW; // this warp's first token column
        // weight row of this thread's TMEM lane: tile row q*32+lane, or for the interleaved
        // form feature 16q + (lane & 15) of the tile, gate for lanes < 16 and up above
        bool is_up = C::ILV && lane >= 16;  // refined per segment below (up rows may come first)
        const int r = C::ILV ? q * 16 + (lane & 15) : q * 32 + lane;
        const int etid = ew * 32 + lane;      // index among the epilogue threads
        uint32_t ai = 0;
        int ti = 0;
        // The tile's activation scales s_x[row0 + c, kb] live in shared memory (two buffers,
        // alternating by tile).  The next tile's values are loaded into registers while the
        // current tile is promoted, and stored at the end of it, so no tile waits on them.
        constexpr int NPF = C::SX_BUFS == 2 ? (BN * kMaxKb) / (32 * EW) : 1;
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
        constexpr bool kSxDouble = kStageSx && C::SX_BUFS == 2;
        if constexpr (kSxDouble) {
            if ((int)blockIdx.x < total) {
                const TileInfo t0 = decode_tile<BN, kStageSx, RT>(args, ttab, blockIdx.x, tot0);
                load_sx(t0);
                store_sx(t0, sxbuf);
            }
            epi_sync(32 * EW);
        }
        for (int w = blockIdx.x; w < total; w += gridDim.x, ++ti) {
            const TileInfo tl = decode_tile<BN, kStageSx, RT>(args, ttab, w, tot0);
            const GemmSeg &sg = args.seg[tl.seg];
            const int K = sg.K;
            const int nkb = (K + kBlockK - 1) / kBlockK;
            if constexpr (C::ILV) is_up = (lane >= 16) != (sg.ilv4d && sg.up_lo);
            const float *sxs = sxbuf + (kSxDouble ? (ti & 1) * (BN * kMaxKb) : 0);
            const int wn = w + gridDim.x;
            TileInfo tn;
            if constexpr (kStageSx && !kSxDouble) {  // one buffer: copy this tile's scales now
                for (int i = etid; i < BN * nkb; i += 32 * EW) {
                    const int c = i / nkb, kb = i - c * nkb;
                    const int row = min(tl.row0 + c, sg.rows - 1);
                    sxbuf[kb * BN + c] = __ldg(sg.sx + (size_t)row * nkb + kb);
                }
                epi_sync(32 * EW);
            }
            if (kSxDouble && wn < total) {
                tn = decode_tile<BN, kStageSx, RT>(args, ttab, wn, tot0);
                load_sx(tn);
            }
            // the interleaved form reads gate scales on lanes < 16 and up scales above; the
            // paired form reads both
            const float *sw0 = static_cast<const float *>(is_up ? sg.sw1 : sg.sw0) + (size_t)(tl.wrow + r) * nkb;
            const float *sw1 = C::PAIR ? static_cast<const float *>(sg.sw1) + (size_t)(tl.wrow + r) * nkb : nullptr;
            float acc0[C::CPW], acc1[C::PAIR ? C::CPW : 1];
#pragma unroll
            for (int c = 0; c < C::CPW; ++c) acc0[c] = 0.0f;
            if constexpr (C::PAIR) {
#pragma unroll
                for (int c = 0; c < C::CPW; ++c) acc1[c] = 0.0f;
            }
            float s0n = 0.0f, s1n = 0.0f;
            if constexpr (kStageSx) {
                s0n = __ldg(sw0);
                if (C::PAIR) s1n = __ldg(sw1);
            }
            for (int kb = 0; kb < nkb; ++kb, ++ai) {
                const int slot = ai % C::NSLOT;
                const uint32_t aph = (ai / C::NSLOT) & 1;
                float s0, s1;
                if constexpr (kStageSx) {  // wide tiles: weight scales prefetched a block ahead
                    s0 = s0n;
                    s1 = s1n;
                    if (kb + 1 < nkb) {
                        s0n = __ldg(sw0 + kb + 1);
                        if (C::PAIR) s1n = __ldg(sw1 + kb + 1);
                    }
                } else {
                    s0 = __ldg(sw0 + kb);
                    s1 = C::PAIR ? __ldg(sw1 + kb) : 0.0f;
                }
                const bool ok = mbar_wait(&accf[slot], aph, abort_flag, status, tmo);
                // wide tiles meet at named barriers between tiles: decide for all epilogue warps
                if (!(kStageSx ? bar_all(2, 32 * EW, ok) : __all_sync(0xffffffffu, ok))) goto done;
                tc_fence_after();
                const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + slot * C::SLOT_COLS + cbase;
                const float *sxk = sxs + kb * BN + cbase;
#pragma unroll
                for (int c0 = 0; c0 < C::CPW; c0 += 16) {
                    float v[16], u[16];
                    tmem_ld16(tb + c0, v);
                    if constexpr (C::PAIR) {
                        tmem_ld16(tb + BN + c0, u);
                        tmem_wait_ld2(v, u);
                    } else {
                        tmem_wait_ld(v);
                    }
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        float sx;
                        if constexpr (kStageSx) {
                            sx = sxk[c0 + c];
                        } else {
                            const int row = min(tl.row0 + cbase + c0 + c, sg.rows - 1);
                            sx = __ldg(sg.sx + (size_t)row * nkb + kb);
                        }
                        acc0[c0 + c] = fmaf(v[c], s0 * sx, acc0[c0 + c]);
                        if constexpr (C::PAIR) acc1[c0 + c] = fmaf(u[c], s1 * sx, acc1[c0 + c]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acce[slot]);
            }
            float *out = static_cast<float *>(sg.out);
            const int n = tl.nt * RT + r;
            if constexpr (C::ILV) {
                // partner lane (lane ^ 16) holds the other projection of feature n.  Of each
                // column pair the lower lane (odd = 0) finishes the even column and the upper lane
                // the odd one; each sends its partner the value for the partner's column.
                const bool odd = lane >= 16;
                float *orow = out + (size_t)(tl.row0 + cbase + (odd ? 1 : 0)) * sg.N + n;
#pragma unroll
                for (int c = 0; c < C::CPW; c += 2) {
                    const float other = __shfl_xor_sync(0xffffffffu, odd ? acc0[c] : acc0[c + 1], 16);
                    const float mine = odd ? acc0[c + 1] : acc0[c];
                    const float v = is_up ? silu_mul(other, mine) : silu_mul(mine, other);
                    if (cbase + c + (odd ? 1 : 0) < tl.nrows) orow[(size_t)c * sg.N] = v;
                }
            } else {
#pragma unroll
                for (int c = 0; c < C::CPW; ++c) {
                    if (cbase + c < tl.nrows) {
                        float v;
                        if constexpr (C::PAIR)
                            v = silu_mul(acc0[c], acc1[c]);
                        else
                            v = acc0[c];
                        out[(size_t)(tl.row0 + cbase + c) * sg.N + n] = v;
                    }
                }
            }
            if constexpr (kSxDouble) {
                if (wn < total) store_sx(tn, sxbuf + ((ti + 1) & 1) * (BN * kMaxKb));
                epi_sync(32 * EW);
            } else if constexpr (kStageSx) {
                epi_sync(32 * EW);  // every thread is done with the buffer before it is refilled
            }
        }
    }
done:
    // own asynchronous work first: the producer's copies of the last NS stages have landed and
    // the MMAs this CTA issued have completed (both already true unless a role gave up early)
    if (warp == 0 && lane == 0)
        for (uint32_t j = issued > (uint32_t)C::NS ? issued - C::NS : 0; j < issued; ++j)
            mbar_wait_drain(&full[j % C::NS], (j / C::NS) & 1, tmo);
    if (warp == 1 && lane == 0) mma_drain(drain_bar, tmo);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

template <int BN, int MODE, int EW>
cudaError_t launch_t(const GemmMaps &maps, const GemmArgs &args, int num_sms, cudaStream_t s)
{
    using C = Fp8Cfg<BN, MODE, EW>;
    auto kern = gemm_fp8_kernel<BN, MODE, EW>;
    cudaError_t e = set_smem_limit(reinterpret_cast<const void *>(kern), C::SMEM);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(num_sms), dim3(C::THREADS), C::SMEM, s, maps, args);
}

}  // namespace

cudaError_t launch_gemm_fp8(bool gateup, int bn, const GemmMaps &maps, const GemmArgs &args, int num_sms,
                            cudaStream_t s)
{
    if (args.seg[0].K > kMaxKb * kBlockK || (args.nseg > 1 && args.seg[1].K > kMaxKb * kBlockK))
        return cudaErrorInvalidValue;
    if (gateup) {
        switch (bn) {
            case 32: return launch_t<32, kModePair, 4>(maps, args, num_sms, s);
            case 64: return launch_t<64, kModePair, 8>(maps, args, num_sms, s);
            case 128: return launch_t<128, kModeInterleaved, 8>(maps, args, num_sms, s);
            case 160: return launch_t<160, kModeInterleaved, 8>(maps, args, num_sms, s);
            case 192: return launch_t<192, kModeInterleaved, 12>(maps, args, num_sms, s);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (bn) {
        case 32: return launch_t<32, kModeDown, 4>(maps, args, num_sms, s);
        case 64: return launch_t<64, kModeDown, 8>(maps, args, num_sms, s);
        case 128: return launch_t<128, kModeDown, 8>(maps, args, num_sms, s);
        case 160: return launch_t<160, kModeDown, 8>(maps, args, num_sms, s);
        case 192: return launch_t<192, kModeDown, 12>(maps, args, num_sms, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
