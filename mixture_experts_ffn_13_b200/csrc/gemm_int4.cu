// gemm_int4.cu -- steps A4/A5 for 4-bit expert weights: persistent grouped GEMMs that unpack
// int4, MXFP4 or NVFP4 weights into tensor memory and run bf16 x bf16 -> fp32 tcgen05 MMAs.
//
// Page "Flash-Next 在 GPU 上到底在算什麼", section "① 專家 FFN" (and its NVIDIA table): expert
// weights are stored in 4/8 bits and must be decompressed to 16-bit before the tensor units
// can use them; on consumer GPUs that decompress-then-FMA runs on the CUDA cores with the
// tensor cores idle.  Here the decompression feeds the tensor cores instead, and keeps the
// weights exact:
//  * warp 0 streams raw int4 weight tiles (128 rows x 128 bytes = 256 K-elements per matrix,
//    128-byte swizzle; narrower boxes make the TMA issue-bound) by TMA into a ring of raw
//    stages (evict-first), keeps an L2 prefetch of the raw tiles kPrefetch stages further
//    ahead, and streams the bf16 activation tiles through their own ring;
//  * warps 4-11 (two per TMEM lane quarter; a thread handles one weight row and one 32-element
//    half of every 64-K stage) turn the nibbles into the integers q as bf16 (exact: |q| <= 8):
//    flip each nibble's sign bit, place it in the mantissa of the bf16 value 128 (so it reads
//    128 + q + 8), subtract 136.  A 32-bit word of 8 nibbles holds elements i and i + 4 sixteen
//    bits apart, so each bf16 pair is one shift, one mask and one subtract when it pairs
//    element i with element i + 4: int4 tiles keep their K elements in that interleaved order
//    inside every aligned block of 8, and so do the activations and h they multiply (the
//    gather kernel and the int4 gate|up epilogue store them so); the products and their sums
//    are the same, only the order the MMA adds them in changes (11 instructions per 8 nibbles
//    instead of 16; the int4 layer went from 1.054 to 0.946 ms, since the conversion is what
//    the dequantisers spend their time on).  The result goes to TENSOR memory with tcgen05.st
//    (rows in lanes, two bf16 per 32-bit column): staging the 4x-expanded weights in shared
//    memory instead costs a write and a tensor-core read of them per stage, which made the
//    kernel shared-memory-bandwidth bound;
//  * warps 1 and 2 issue tcgen05.mma.kind::f16 (A from tensor memory, B from shared memory),
//    one thread each, 4 MMAs of K = 16 per 64-K stage and matrix: gate|up, one matrix each;
//    int4 down, alternate 128-element scale groups with the whole N; E2M1 down, issuer 0
//    alone with the whole N.  Each int4 K group (2 stages) accumulates into its own TMEM slot,
//    because the weight scale changes per (row, group);
//  * warps 12-19 (two per TMEM lane quarter, each owning half of the token columns) promote each
//    finished group, acc += D_g * s[row, g] in fp32 registers, and at the end of the tile write
//    gate|up h = silu(G) * U rounded to bf16 (the 4-bit layer keeps activations in bf16) or
//    down y in fp32;
//  * the five warpgroups (warp 3 idles) set their own register counts with setmaxnreg: 56 for
//    the producer and issuers, 80 for the dequantisers, 128 for the promotion's 96 sums.
// Multiplying the exact integers on the tensor cores and applying the bf16 scale to fp32
// partial sums reproduces sum_i x_i * q_i * s_i up to fp32 rounding; rounding q * s to bf16
// before the MMA would not (that costs ~2^-9 relative per weight and fails the layer's
// tolerance at these sizes).
//
// MXFP4 weights (page "设计 AI 芯片的硬件与软件", section "数值格式，或如何制造便宜的脉动阵列":
// 4-bit values plus an 8-bit scale per 32 of them, 4.25 bits per number) use the same
// pipeline with one change in the dequantisers and one in the MMA/epilogue split: an E2M1
// value (at most two significant bits) times its block's power-of-two E8M0 scale is exact in
// bf16, so the dequantisers write the scaled weights themselves, the whole K accumulates in
// one TMEM slot, and the epilogue has no promotion to do.  The warp roles shift with that:
// warps 3-10 dequantise (two per TMEM lane quarter, one 32-element block of each 64-K stage
// apiece, as for int4; the gate|up tiles take four per quarter, one half of one matrix apiece,
// warps 3-18) and one warp per quarter streams each finished tile out; at one register count
// for all warps nothing spills, so these formats need no register split.
//
// NVFP4 weights (the NVIDIA co-design commentary, section "讀的時候記得這是廠商文": two levels
// of scale factors) take the same path: an E2M1 value times its 16-block's E4M3 scale has at
// most six significant bits and stays within bf16's normal range, so it too is formed exactly
// in bf16 by the dequantisers; the matrix's fp32 tensor scale multiplies the accumulator in
// the epilogue.
#include "gemm_common.cuh"
#include "launch.cuh"
#include "sm100.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

namespace moe {

namespace {

constexpr int kKE = 64;                // K elements per MMA stage (one 128-byte bf16 swizzle row)
constexpr int kRawKE = 256;            // K elements per raw weight stage (128 bytes per row)
constexpr int kSubs = kRawKE / kKE;    // MMA stages per raw stage
constexpr int kPrefetch = 8;           // raw stages prefetched into L2 ahead of the loads

// Warp roles: 0 producer, 1 and 2 MMA issuers, then CONV dequantisers from warp D0 (two per TMEM
// lane quarter, each converting one 32-element half of every 64-K stage), then EW epilogue
// warps from warp E0.  int4 keeps two epilogue warps per quarter (each holds half the token
// columns' fp32 sums across the scale groups) and lays the roles out by warpgroup (warp 3
// idle, warpgroups 1-2 dequantise, 3-4 promote) so that each can set its own register count:
// the promotion needs ~128 per thread, the rest far fewer, and 20 warps at one count would
// leave the promotion 96.  MXFP4/NVFP4 have no promotion: one epilogue warp per quarter
// streams the accumulator out, and 15 warps fit without a split.
enum { kFmtInt4 = 0, kFmtMx = 1, kFmtNv = 2 };

template <int BN, bool GATEUP, bool FP4>
struct I4Cfg {
    // dequantiser warps: two per TMEM lane quarter (one 32-element half of each 64-K stage
    // apiece); the E2M1 gate|up tiles, whose conversion is the longest, take four (one half
    // of one matrix apiece)
    static constexpr int CONV = FP4 && GATEUP ? 16 : 8;
    static constexpr int MSPLIT = CONV / 8;                 // dequantiser sets sharing the matrices
    static constexpr int EW = FP4 ? 4 : 8;                  // epilogue warps
    static constexpr int D0 = FP4 ? 3 : 4;                  // first dequantiser warp
    static constexpr int E0 = D0 + CONV;                    // first epilogue warp
    static constexpr int CPW = BN / (EW / 4);               // token columns per epilogue thread
    static constexpr int THREADS = 32 * (E0 + EW);
    // int4 register split (per thread, multiples of 8): warpgroup 0 (producer, issuers),
    // warpgroups 1-2 (dequantisers), warpgroups 3-4 (promotion).  Their sum over the five
    // warpgroups must not exceed what the block is launched with (checked on the host before
    // every launch), or an increase would wait for registers that never come.
    static constexpr int REG_PI = 56, REG_D = 80, REG_E = 128;
    static constexpr int REG_SUM = REG_PI + 2 * REG_D + 2 * REG_E;  // x 128 threads
    static_assert(FP4 || THREADS == 640, "int4: five whole warpgroups");
    static constexpr int NA = GATEUP ? 2 : 1;
    static constexpr int RAW_BYTES = kTileM * (kRawKE / 2);  // 16 KB per matrix
    static constexpr int B_BYTES = BN * kKE * 2;
    // Converted weights live in tensor memory: NM stages x NA matrices x 32 columns (64 bf16
    // per row).  The accumulator slots take the remaining columns.
    static constexpr int NM = GATEUP ? 2 : 3;
    static constexpr int A_COLS = 32;
    static constexpr int A_TMEM = NM * NA * A_COLS;
    static constexpr int SLOT_COLS = NA * BN;  // one 128-element K group (int4) or a whole tile (E2M1)
    static constexpr int NSLOT = (512 - A_TMEM) / SLOT_COLS;
    static constexpr int STAGES_PER_GROUP = kGroupK / kKE;  // 2
    static constexpr int NR = GATEUP ? 3 : 5;               // raw weight stages (256 K each)
    // activation stages (64 K each).  int4 keeps the block within 196 KB of shared memory, so
    // that the carve-out leaves ~60 KB of L1 for its epilogue's scale loads (int4 layer 1.061
    // against 1.064 ms); the E2M1 formats have no such loads and keep the deeper ring (MXFP4
    // 1.185 against 1.206 ms with the int4 budget, NVFP4 even).
    static constexpr int SMEM_BUDGET = FP4 ? 212 * 1024 : 190 * 1024;
    static constexpr int NB_FIT = (SMEM_BUDGET - NR * NA * RAW_BYTES) / B_BYTES;
    static constexpr int NB = NB_FIT < 12 ? NB_FIT : 12;
    static constexpr int TT_BYTES = (4 * (kMaxE + 1) + 15) & ~15;  // keeps the mbarriers 8-byte aligned
    static constexpr int BAR_BYTES = 8 * (2 * NR + 2 * NB + NM + 2 * NSLOT) + 24;
    static constexpr int SMEM = 1024 + NB * B_BYTES + NR * NA * RAW_BYTES + TT_BYTES + BAR_BYTES;
    static_assert(B_BYTES % 1024 == 0, "1024-byte aligned tiles");
    static_assert(NSLOT >= 2, "TMEM slots");
    static_assert(NB > NM, "the weight stages' release is read from the deeper activation ring");
    static_assert(CONV % 4 == 0 && EW % 4 == 0, "whole TMEM lane quarters per role");
    static_assert(SMEM <= (FP4 ? 227 : 196) * 1024, "shared memory (int4: within the carve-out that leaves ~60 KB of L1)");
    static_assert((NR * NA * RAW_BYTES + NB * B_BYTES + TT_BYTES) % 16 == 0, "mbarriers must be 8-byte aligned");
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t bf2_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t *>(&v); }

__device__ __forceinline__ __nv_bfloat162 bits_bf2(uint32_t u) { return *reinterpret_cast<__nv_bfloat162 *>(&u); }

// 8 E2M1 nibbles (element 2i in the low nibble of byte i) times the block scale sc (2^x in both
// halves), as 4 words of bf16 pairs in element order.  Each 3-bit magnitude picks the low and
// the high byte of its bf16 value from two 8-entry byte tables with prmt (4 elements per prmt);
// the nibble's sign bit goes to bit 7 of the high byte; one bf16 multiply by 2^x scales a
// pair, exactly while the product stays a normal bf16 (E8M0 codes 2..252).
__device__ __forceinline__ uint4 unpack8_fp4(uint32_t w, __nv_bfloat162 sc)
{
    // bf16 of the magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6: 0000 3F00 3F80 3FC0 4000 4040 4080 40C0
    constexpr uint32_t kLo03 = 0xC0800000u, kLo47 = 0xC0804000u;  // low bytes, codes 0-3 | 4-7
    constexpr uint32_t kHi03 = 0x3F3F3F00u, kHi47 = 0x40404040u;  // high bytes
    const uint32_t mag = w & 0x77777777u;                          // prmt reads 4 selectors
    const uint32_t lo_a = prmt(kLo03, kLo47, mag), hi_a = prmt(kHi03, kHi47, mag);  // elements 0-3
    const uint32_t lo_b = prmt(kLo03, kLo47, mag >> 16), hi_b = prmt(kHi03, kHi47, mag >> 16);  // 4-7
    const uint32_t ev = (w << 4) & 0x80808080u;  // signs of elements 0, 2, 4, 6 at bit 7 of bytes 0-3
    const uint32_t od = w & 0x80808080u;         // signs of elements 1, 3, 5, 7
    const uint32_t ha = hi_a | prmt(ev, od, 0x5140u), hb = hi_b | prmt(ev, od, 0x7362u);
    const uint32_t r0 = prmt(lo_a, ha, 0x5140u), r1 = prmt(lo_a, ha, 0x7362u);
    const uint32_t r2 = prmt(lo_b, hb, 0x5140u), r3 = prmt(lo_b, hb, 0x7362u);
    return make_uint4(bf2_bits(__hmul2(bits_bf2(r0), sc)), bf2_bits(__hmul2(bits_bf2(r1), sc)),
                      bf2_bits(__hmul2(bits_bf2(r2), sc)), bf2_bits(__hmul2(bits_bf2(r3), sc)));
}

// The bf16 pair (2^(c-127), 2^(c-127)) of an E8M0 code c in 1..254.
__device__ __forceinline__ __nv_bfloat162 e8m0_pair(uint32_t c) { return bits_bf2((c << 7) | (c << 23)); }

// The bf16 pair (v, v) of the E4M3 byte c (every finite E4M3 value is exact in bf16).
__device__ __forceinline__ __nv_bfloat162 e4m3_pair(uint32_t c)
{
    const __half_raw hr = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3);
    const __nv_bfloat16 b = __float2bfloat16_rn(__half2float(__half(hr)));
    return __halves2bfloat162(b, b);
}

// 8 two's-complement nibbles (element 2i in the low nibble of byte i) -> the 8 integers as
// bf16 (exact), returned as 4 words of bf16 pairs in the interleaved K order: word i holds
// elements i (low half) and i + 4 (high half), the two nibbles 16 bits apart in w.
__device__ __forceinline__ uint4 unpack8(uint32_t w)
{
    const __nv_bfloat162 off = bits_bf2(0x43084308u);  // (136, 136)
    uint32_t r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        // q + 8 (sign bit flipped) in the low 4 mantissa bits of the bf16 pair (128, 128)
        const uint32_t v = (((w >> (4 * i)) ^ 0x00080008u) & 0x000F000Fu) | 0x43004300u;
        r[i] = bf2_bits(__hsub2(bits_bf2(v), off));
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}

// Position of K element j inside its aligned block of 8 in the interleaved order of unpack8:
// elements 0-3 go to the even positions, elements 4-7 to the odd ones.
__device__ __forceinline__ int k_interleave8(int j) { return (j & ~7) | ((j & 3) << 1) | ((j >> 2) & 1); }

// FMT: kFmtInt4 (bf16 scales per 128-group), kFmtMx (MXFP4) or kFmtNv (NVFP4).
template <int BN, bool GATEUP, int FMT>
__global__ void __launch_bounds__(I4Cfg<BN, GATEUP, FMT != kFmtInt4>::THREADS, 1)
    gemm_int4_kernel(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmArgs args)
{
    constexpr bool FP4 = FMT != kFmtInt4;  // E2M1 elements with exact bf16 scaling (MXFP4, NVFP4)
    constexpr bool NV = FMT == kFmtNv;
    constexpr bool DALT = !GATEUP;         // down: one issuer per group, with the whole N
    constexpr bool ONE = !GATEUP && FP4;   // E2M1 down: one tile = one group, so issuer 0 takes all
    using C = I4Cfg<BN, GATEUP, FP4>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *raw = smem;                                   // NR raw stages [raw0 | raw1]
    uint8_t *bst = raw + C::NR * C::NA * C::RAW_BYTES;     // NB activation stages
    int *stt = reinterpret_cast<int *>(bst + C::NB * C::B_BYTES);  // [E + 1]
    uint64_t *rfull = reinterpret_cast<uint64_t *>(bst + C::NB * C::B_BYTES + C::TT_BYTES);
    uint64_t *rempty = rfull + C::NR;
    uint64_t *bfull = rempty + C::NR;
    uint64_t *bempty = bfull + C::NB;
    uint64_t *mfull = bempty + C::NB;
    uint64_t *accf = mfull + C::NM;
    uint64_t *acce = accf + C::NSLOT;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(acce + C::NSLOT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    uint64_t *drain_bar = reinterpret_cast<uint64_t *>(tmem_holder + 2);  // MMA drain on exit, one per issuer

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NR; ++s) {
            mbar_init(&rfull[s], 1);
            mbar_init(&rempty[s], C::CONV);
        }
        // gate|up and the E2M1 down: both MMA issuers consume every stage and contribute to
        // every accumulator; int4 down: the issuers take alternate scale groups
        for (int s = 0; s < C::NB; ++s) {
            mbar_init(&bfull[s], 1);
            mbar_init(&bempty[s], DALT ? 1 : 2);
        }
        // a TMEM weight stage is free again once the MMAs of the stage that used it have
        // completed, which bempty of that stage records (the ring of activation stages is
        // deeper than the ring of weight stages, so the phase waited for is never overtaken)
        for (int s = 0; s < C::NM; ++s) mbar_init(&mfull[s], C::CONV);
        for (int s = 0; s < C::NSLOT; ++s) {
            mbar_init(&accf[s], DALT ? 1 : 2);
            mbar_init(&acce[s], C::EW);
        }
        mbar_init(&drain_bar[0], 1);
        mbar_init(&drain_bar[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
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
    load_ttile(args, stt);

    int tot0;
    const int total = total_tiles(args, BN, &tot0);
    int *status = args.status;
    const uint64_t tmo = args.timeout_ns;
    uint32_t issued_r = 0, issued_b = 0;  // producer: raw and activation stages issued

    if (warp < C::D0) {
        // int4: warpgroup 0 (producer, issuers and an idle warp) gives registers back; the
        // register counts are set at the top of each role's branch, where the compiler can
        // budget the role's code with them
        if constexpr (!FP4) regs_dec<C::REG_PI>();
        if (warp == 0) {
            // --------------------- raw weight + activation producer ---------------------
            if (lane == 0) {
                const uint64_t pol_w = l2_policy_evict_first();
                const uint64_t pol_x = l2_policy_evict_last();
                uint32_t it = 0, rt = 0;  // MMA-stage and raw-stage counters
                // L2 prefetch cursor: raw stage (pw tile, pk index) runs kPrefetch raw stages ahead
                // of the shared-memory loads, across tile boundaries
                int pw = blockIdx.x, pk = 0;
                TileInfo pt;
                if (pw < total) pt = decode_tile<BN, true>(args, stt, pw, tot0);
                auto prefetch_next = [&]() {
                    if (pw >= total) return;
                    const int x = pk * (kRawKE / 2);
                    tma_prefetch_l2_2d(&maps.a0[pt.seg], x, pt.wrow);
                    if (GATEUP) tma_prefetch_l2_2d(&maps.a1[pt.seg], x, pt.wrow);
                    if (++pk * kRawKE >= args.seg[pt.seg].K) {
                        pk = 0;
                        pw += gridDim.x;
                        if (pw < total) pt = decode_tile<BN, true>(args, stt, pw, tot0);
                    }
                };
                for (int i = 0; i < kPrefetch; ++i) prefetch_next();
                for (int w = blockIdx.x; w < total; w += gridDim.x) {
                    const TileInfo tl = decode_tile<BN, true>(args, stt, w, tot0);
                    const int nkc = args.seg[tl.seg].K / kKE;
                    for (int kc = 0; kc < nkc; ++kc, ++it) {
                        if (kc % kSubs == 0) {
                            prefetch_next();
                            // raw weights for the next 256 K-elements (the last stage of a K that is
                            // not a multiple of 256 reads zeros past the end)
                            const int s = rt % C::NR;
                            if (!mbar_wait(&rempty[s], ((rt / C::NR) & 1) ^ 1, abort_flag, status, tmo)) goto done;
                            uint8_t *rs = raw + s * C::NA * C::RAW_BYTES;
                            issued_r = rt + 1;
                            mbar_arrive_expect_tx(&rfull[s], C::NA * C::RAW_BYTES);
                            const int x = (kc / kSubs) * (kRawKE / 2);
                            tma_load_2d_hint(rs, &maps.a0[tl.seg], &rfull[s], x, tl.wrow, pol_w);
                            if (GATEUP) tma_load_2d_hint(rs + C::RAW_BYTES, &maps.a1[tl.seg], &rfull[s], x, tl.wrow, pol_w);
                            ++rt;
                        }
                        const int b = it % C::NB;
                        if (!mbar_wait(&bempty[b], ((it / C::NB) & 1) ^ 1, abort_flag, status, tmo)) goto done;
                        issued_b = it + 1;
                        mbar_arrive_expect_tx(&bfull[b], C::B_BYTES);
                        tma_load_2d_hint(bst + b * C::B_BYTES, &maps.b[tl.seg], &bfull[b], kc * kKE, tl.row0, pol_x);
                    }
                }
            }
        } else if (warp == 1 || warp == 2) {
            // ------------------------------ MMA issuers -------------------------------
            // Two threads in different warps share the MMAs: a tcgen05.commit holds up the
            // issuing thread, which one thread alone cannot hide behind the short N <= 96 MMAs.
            // gate|up: issuer 0 multiplies the gate weights and issuer 1 the up weights; both
            // wait for and release every stage.  int4 down: the issuers
            // take alternate 128-element scale groups (each its own TMEM slot) with the whole N,
            // so a stage costs four MMAs instead of eight; each waits for and releases the
            // stages of its groups only.  That is safe with parity waits because an issuer skips
            // only two stages at a time: the dequantisers cannot complete a stage more than NM
            // stages past an MMA stage that has not been issued, so no barrier an issuer waits
            // on is ever two phases ahead of it.  E2M1 down: a tile's whole K is one group, and
            // alternating whole tiles (24 stages and more apiece) lets the barriers run phases
            // ahead of the skipping issuer (the full-size MXFP4 layer timed out), so issuer 0
            // issues every stage with the whole N and issuer 1 idles.
            const int mt = warp - 1;
            if (lane == 0 && !(ONE && mt == 1)) {
                uint32_t it = 0, ai = 0;
                for (int w = blockIdx.x; w < total; w += gridDim.x) {
                    const TileInfo tl = decode_tile<BN, true>(args, stt, w, tot0);
                    // MMA N: the tile's valid rows rounded up to 16; partial tiles cost no work on
                    // absent rows
                    const int n_mma = min(BN, (tl.nrows + 15) & ~15);
                    const uint32_t kIdesc = instr_desc(kTileM, n_mma, 1, 1);
                    // int4: one TMEM slot per 128-element scale group; E2M1 formats: one for the K
                    const int ngrp = FP4 ? 1 : args.seg[tl.seg].K / kGroupK;
                    const int spg = FP4 ? args.seg[tl.seg].K / kKE : C::STAGES_PER_GROUP;
                    for (int g = 0; g < ngrp; ++g, ++ai) {
                        if (DALT && !ONE && (int)(ai & 1) != mt) {  // the other issuer's group
                            it += spg;
                            continue;
                        }
                        const int slot = ai % C::NSLOT;
                        if (!mbar_wait(&acce[slot], ((ai / C::NSLOT) & 1) ^ 1, abort_flag, status, tmo)) goto done;
                        tc_fence_after();
                        // gate|up: this issuer's matrix; down: the whole slot
                        const uint32_t d = tmem_base + C::A_TMEM + slot * C::SLOT_COLS + (GATEUP ? mt * BN : 0);
                        for (int sk = 0; sk < spg; ++sk, ++it) {
                            const int s = it % C::NM;
                            const int bs = it % C::NB;
                            if (!mbar_wait(&mfull[s], (it / C::NM) & 1, abort_flag, status, tmo)) goto done;
                            if (!mbar_wait(&bfull[bs], (it / C::NB) & 1, abort_flag, status, tmo)) goto done;
                            tc_fence_after();
                            const uint32_t a = tmem_base + s * C::NA * C::A_COLS + (GATEUP ? mt * C::A_COLS : 0);
                            // down: the second half's token rows start n_mma rows (n_mma * 128 bytes,
                            // whole 8-row swizzle atoms) into the activation stage
                            const uint64_t db = smem_desc_sw128(bst + bs * C::B_BYTES);
#pragma unroll
                            for (int kk = 0; kk < kKE / 16; ++kk)
                                mma_bf16_ts(d, a + 8 * kk, db + 2 * kk, kIdesc, (sk > 0 || kk > 0) ? 1u : 0u);
                            mma_commit(&bempty[bs]);  // frees the activation stage and the TMEM weight stage
                        }
                        mma_commit(&accf[slot]);
                    }
                }
            }
    }
    } else if (warp < C::E0) {
        if constexpr (!FP4) regs_dec<C::REG_D>();
        // ------------------------------ dequantisers ------------------------------
        const int q = warp & 3;        // TMEM lane quarter reachable from this warp
        const int r = q * 32 + lane;   // weight row of the tile handled by this thread
        uint32_t it = 0, rt = 0;
        // E2M1 formats: this row's block-scale bytes of the current raw stage (MXFP4: 8 E8M0
        // bytes, NVFP4: 16 E4M3 bytes per matrix) and those of the next raw stage in this
        // CTA's sequence (the next tile's first one at a tile's end), loaded a raw stage ahead
        // so that their latency overlaps the conversion
        constexpr int SBLK = NV ? 16 : 32;         // K elements per block scale
        constexpr int SW = kRawKE / SBLK / 4;      // scale words per raw stage: 2 (MX), 4 (NV)
        uint32_t scur[C::NA][SW] = {}, snxt[C::NA][SW] = {};
        const int unit = (warp - C::D0) >> 2;               // which share of each stage
        const int hx = C::MSPLIT == 2 ? (unit & 1) : unit;   // 32-element half of the 64-K stage
        const int mown = unit >> 1;                         // MSPLIT 2: the one matrix converted
        auto load_scales = [&](int wi, int kr, uint32_t (&dst)[C::NA][SW]) {
            const TileInfo t = decode_tile<BN, true>(args, stt, wi, tot0);
            const GemmSeg &s = args.seg[t.seg];
            const int nbk = s.K / SBLK;            // scale bytes per weight row: a multiple of 4
                                                   // (MX) or 8 (NV), so each load is aligned
            const int b0 = kr * (4 * SW);          // first byte of raw stage kr
            const int half = 2 * SW;               // bytes of the first 128 K of the raw stage
#pragma unroll
            for (int m = 0; m < C::NA / C::MSPLIT; ++m) {
                const int ms = C::MSPLIT == 2 ? mown : m;
                const uint8_t *base = static_cast<const uint8_t *>(ms == 0 ? s.sw0 : s.sw1);
                const uint8_t *p = base + (size_t)(t.wrow + r) * nbk + b0;
                // a last raw stage of 128 K has only its first half: b0 + half <= nbk always
                if constexpr (NV) {
                    const uint2 lo = __ldg(reinterpret_cast<const uint2 *>(p));
                    const uint2 hi =
                        b0 + half < nbk ? __ldg(reinterpret_cast<const uint2 *>(p + 8)) : make_uint2(0u, 0u);
                    dst[m][0] = lo.x;
                    dst[m][1] = lo.y;
                    dst[m][SW - 2] = hi.x;
                    dst[m][SW - 1] = hi.y;
                } else {
                    dst[m][0] = __ldg(reinterpret_cast<const uint32_t *>(p));
                    dst[m][SW - 1] = b0 + half < nbk ? __ldg(reinterpret_cast<const uint32_t *>(p + 4)) : 0u;
                }
            }
        };
        if (FP4 && (int)blockIdx.x < total) load_scales(blockIdx.x, 0, snxt);
        for (int w = blockIdx.x; w < total; w += gridDim.x) {
            const TileInfo tl = decode_tile<BN, true>(args, stt, w, tot0);
            const GemmSeg &sg = args.seg[tl.seg];
            const int nkc = sg.K / kKE;
            for (int kc = 0; kc < nkc; ++kc, ++it) {
                const int sub = kc % kSubs;
                if (FP4 && sub == 0) {
#pragma unroll
                    for (int m = 0; m < C::NA; ++m)
#pragma unroll
                        for (int j = 0; j < SW; ++j) scur[m][j] = snxt[m][j];
                    const int kr = kc / kSubs;
                    if ((kr + 1) * kRawKE < sg.K)
                        load_scales(w, kr + 1, snxt);
                    else if (w + (int)gridDim.x < total)
                        load_scales(w + gridDim.x, 0, snxt);
                }
                const int rs_i = rt % C::NR;
                const int ms_i = it % C::NM;
                bool ok = true;
                if (sub == 0) ok = mbar_wait(&rfull[rs_i], (rt / C::NR) & 1, abort_flag, status, tmo);
                if (!__all_sync(0xffffffffu, ok)) goto done;
                // TMEM stage ms_i was last read by the MMAs of stage it - NM
                if (it >= (uint32_t)C::NM) {
                    const uint32_t j = it - C::NM;
                    ok = mbar_wait(&bempty[j % C::NB], (j / C::NB) & 1, abort_flag, status, tmo);
                }
                if (!__all_sync(0xffffffffu, ok)) goto done;
                tc_fence_after();
                const uint8_t *rs = raw + rs_i * C::NA * C::RAW_BYTES + r * 128;
                const uint32_t ta = tmem_base + ((uint32_t)(q * 32) << 16) + ms_i * C::NA * C::A_COLS;
                if constexpr (FP4) {
                    // half hx of the stage: 16-byte chunk ch = 2*sub + hx of the row (the 128-byte
                    // swizzle stores chunk c at position c ^ (r & 7)), K elements 32*ch .. +31 of
                    // the raw stage, written to TMEM columns 16*hx .. 16*hx + 15; with MSPLIT 2
                    // only matrix mown, whose scale bytes sit in slot 0
                    const int cc = ((2 * sub + hx) ^ (r & 7)) << 4;
#pragma unroll
                    for (int mi = 0; mi < C::NA / C::MSPLIT; ++mi) {
                        const int m = C::MSPLIT == 2 ? mown : mi;
                        const uint4 qq = *reinterpret_cast<const uint4 *>(rs + m * C::RAW_BYTES + cc);
                        // scales of the chunk's elements 0-15 (sa) and 16-31 (sb)
                        __nv_bfloat162 sa, sb;
                        if constexpr (NV) {
                            // 16-blocks 2*ch and 2*ch + 1: bytes 2*ch, 2*ch + 1 = word sub, bytes
                            // 2*hx and 2*hx + 1 of it
                            const uint32_t sw = sub == 0   ? scur[mi][0]
                                                : sub == 1 ? scur[mi][1]
                                                : sub == 2 ? scur[mi][SW - 2]
                                                           : scur[mi][SW - 1];
                            sa = e4m3_pair((sw >> (hx * 16)) & 0xFFu);
                            sb = e4m3_pair((sw >> (hx * 16 + 8)) & 0xFFu);
                        } else {
                            // 32-block ch: byte ch = word sub >> 1, byte (sub & 1) * 2 + hx of it
                            const uint32_t sw = (sub >> 1) ? scur[mi][SW - 1] : scur[mi][0];
                            sa = sb = e8m0_pair((sw >> ((sub & 1) * 16 + hx * 8)) & 0xFFu);
                        }
                        const uint32_t words[4] = {qq.x, qq.y, qq.z, qq.w};
                        uint32_t v[16];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint4 u = unpack8_fp4(words[j], j < 2 ? sa : sb);
                            v[4 * j] = u.x;
                            v[4 * j + 1] = u.y;
                            v[4 * j + 2] = u.z;
                            v[4 * j + 3] = u.w;
                        }
                        tmem_st16(ta + m * C::A_COLS + 16 * hx, v);  // 32 bf16 = 16 packed columns
                    }
                } else {
                    // half hx of the sub-stage: 16-byte chunk 2*sub + hx of the row (the 128-byte
                    // swizzle stores chunk c at position c ^ (r & 7)), K elements 32*hx .. +31 of
                    // the 64, written to TMEM columns 16*hx .. 16*hx + 15
                    const int cc = ((2 * sub + hx) ^ (r & 7)) << 4;
#pragma unroll
                    for (int m = 0; m < C::NA; ++m) {
                        const uint4 qq = *reinterpret_cast<const uint4 *>(rs + m * C::RAW_BYTES + cc);
                        const uint32_t words[4] = {qq.x, qq.y, qq.z, qq.w};
                        uint32_t v[16];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint4 u = unpack8(words[j]);
                            v[4 * j] = u.x;
                            v[4 * j + 1] = u.y;
                            v[4 * j + 2] = u.z;
                            v[4 * j + 3] = u.w;
                        }
                        tmem_st16(ta + m * C::A_COLS + 16 * hx, v);  // 32 bf16 = 16 packed columns
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                const bool raw_done = (sub == kSubs - 1) || (kc == nkc - 1);
                if (lane == 0) {
                    mbar_arrive(&mfull[ms_i]);
                    if (raw_done) mbar_arrive(&rempty[rs_i]);
                }
                if (raw_done) ++rt;
            }
        }
    } else {
        if constexpr (!FP4) regs_inc<C::REG_E>();
        // ------------------------------ epilogue ----------------------------------
        const int q = warp & 3;                            // TMEM lane quarter
        const int cbase = ((warp - C::E0) >> 2) * C::CPW;  // first token column
        const int r = q * 32 + lane;
        uint32_t ai = 0;
        for (int w = blockIdx.x; w < total; w += gridDim.x) {
            const TileInfo tl = decode_tile<BN, true>(args, stt, w, tot0);
            const GemmSeg &sg = args.seg[tl.seg];
            if constexpr (FP4) {
                // E2M1 formats: the tile's whole K sits in one slot; stream it out 16 columns
                // at a time (NVFP4: times the matrices' tensor scales, expert wrow / N)
                float t0 = 1.0f, t1 = 1.0f;
                if constexpr (NV) {
                    const int g = tl.wrow / sg.N;
                    t0 = __ldg(sg.ts0 + g);
                    if (GATEUP) t1 = __ldg(sg.ts1 + g);
                }
                const int slot = ai % C::NSLOT;
                const bool ok = mbar_wait(&accf[slot], (ai / C::NSLOT) & 1, abort_flag, status, tmo);
                if (!__all_sync(0xffffffffu, ok)) goto done;
                tc_fence_after();
                const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + C::A_TMEM + slot * C::SLOT_COLS;
                const int n = tl.nt * kTileM + r;
                for (int c0 = 0; c0 < BN && c0 < tl.nrows; c0 += 16) {  // warp-uniform bounds
                    float v[16], u[16];
                    tmem_ld16(tb + c0, v);
                    if constexpr (GATEUP) {
                        tmem_ld16(tb + BN + c0, u);
                        tmem_wait_ld2(v, u);
                    } else {
                        tmem_wait_ld(v);
                    }
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        if (c0 + c < tl.nrows) {
                            const size_t o = (size_t)(tl.row0 + c0 + c) * sg.N + n;
                            if constexpr (GATEUP)
                                static_cast<__nv_bfloat16 *>(sg.out)[o] =
                                    __float2bfloat16_rn(NV ? silu_mul(v[c] * t0, u[c] * t1) : silu_mul(v[c], u[c]));
                            else
                                static_cast<float *>(sg.out)[o] = NV ? v[c] * t0 : v[c];
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acce[slot]);
                ++ai;
                continue;
            }
            // int4 only from here on (the E2M1 formats took the branch above)
            const int ngrp = sg.K / kGroupK;
            const __nv_bfloat16 *sw0 = static_cast<const __nv_bfloat16 *>(sg.sw0) + (size_t)(tl.wrow + r) * ngrp;
            const __nv_bfloat16 *sw1 =
                GATEUP ? static_cast<const __nv_bfloat16 *>(sg.sw1) + (size_t)(tl.wrow + r) * ngrp : nullptr;
            float acc0[C::CPW], acc1[GATEUP ? C::CPW : 1];
#pragma unroll
            for (int c = 0; c < C::CPW; ++c) acc0[c] = 0.0f;
            if constexpr (GATEUP) {
#pragma unroll
                for (int c = 0; c < C::CPW; ++c) acc1[c] = 0.0f;
            }
            float s0n = __bfloat162float(sw0[0]), s1n = GATEUP ? __bfloat162float(sw1[0]) : 0.0f;
            for (int g = 0; g < ngrp; ++g, ++ai) {
                const int slot = ai % C::NSLOT;
                const float s0 = s0n, s1 = s1n;
                if (g + 1 < ngrp) {
                    s0n = __bfloat162float(sw0[g + 1]);
                    if (GATEUP) s1n = __bfloat162float(sw1[g + 1]);
                }
                const bool ok = mbar_wait(&accf[slot], (ai / C::NSLOT) & 1, abort_flag, status, tmo);
                if (!__all_sync(0xffffffffu, ok)) goto done;
                tc_fence_after();
                const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + C::A_TMEM + slot * C::SLOT_COLS + cbase;
#pragma unroll
                for (int c0 = 0; c0 < C::CPW; c0 += 16) {
                    float v[16], u[16];
                    tmem_ld16(tb + c0, v);
                    if constexpr (GATEUP) {
                        tmem_ld16(tb + BN + c0, u);
                        tmem_wait_ld2(v, u);
                    } else {
                        tmem_wait_ld(v);
                    }
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        acc0[c0 + c] = fmaf(v[c], s0, acc0[c0 + c]);
                        if constexpr (GATEUP) acc1[c0 + c] = fmaf(u[c], s1, acc1[c0 + c]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acce[slot]);
            }
            // h is the down GEMM's K: stored in the interleaved order its int4 weights unpack to
            const int n = GATEUP ? k_interleave8(tl.nt * kTileM + r) : tl.nt * kTileM + r;
#pragma unroll
            for (int c = 0; c < C::CPW; ++c) {
                if (cbase + c < tl.nrows) {
                    const size_t o = (size_t)(tl.row0 + cbase + c) * sg.N + n;
                    if constexpr (GATEUP)
                        static_cast<__nv_bfloat16 *>(sg.out)[o] = __float2bfloat16_rn(silu_mul(acc0[c], acc1[c]));
                    else
                        static_cast<float *>(sg.out)[o] = acc0[c];
                }
            }
        }
    }
done:
    // own asynchronous work first: the producer's last copies of both rings have landed and
    // the MMAs this CTA issued have completed (both already true unless a role gave up early)
    if (warp == 0 && lane == 0) {
        for (uint32_t j = issued_r > (uint32_t)C::NR ? issued_r - C::NR : 0; j < issued_r; ++j)
            mbar_wait_drain(&rfull[j % C::NR], (j / C::NR) & 1, tmo);
        for (uint32_t j = issued_b > (uint32_t)C::NB ? issued_b - C::NB : 0; j < issued_b; ++j)
            mbar_wait_drain(&bfull[j % C::NB], (j / C::NB) & 1, tmo);
    }
    if ((warp == 1 || warp == 2) && lane == 0) mma_drain(&drain_bar[warp - 1], tmo);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

template <int BN, bool GATEUP, int FMT>
cudaError_t launch_t(const GemmMaps &maps, const GemmArgs &args, int num_sms, cudaStream_t s)
{
    using C = I4Cfg<BN, GATEUP, FMT != kFmtInt4>;
    auto kern = gemm_int4_kernel<BN, GATEUP, FMT>;
    cudaError_t e = set_smem_limit(reinterpret_cast<const void *>(kern), C::SMEM);
    if (e != cudaSuccess) return e;
    if constexpr (FMT == kFmtInt4) {
        // the register split must fit in what the block is launched with
        static const int launch_regs = [&] {
            cudaFuncAttributes fa{};
            return cudaFuncGetAttributes(&fa, reinterpret_cast<const void *>(kern)) == cudaSuccess ? fa.numRegs : 0;
        }();
        if (launch_regs * C::THREADS < 128 * C::REG_SUM || launch_regs < C::REG_D) return cudaErrorInvalidConfiguration;
    }
    return launch_pdl(kern, dim3(num_sms), dim3(C::THREADS), C::SMEM, s, maps, args);
}

template <int FMT>
cudaError_t launch_fmt(bool gateup, int bn, const GemmMaps &maps, const GemmArgs &args, int num_sms, cudaStream_t s)
{
    if (gateup) {
        switch (bn) {
            case 32: return launch_t<32, true, FMT>(maps, args, num_sms, s);
            case 64: return launch_t<64, true, FMT>(maps, args, num_sms, s);
            case 96: return launch_t<96, true, FMT>(maps, args, num_sms, s);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (bn) {
        case 32: return launch_t<32, false, FMT>(maps, args, num_sms, s);
        case 64: return launch_t<64, false, FMT>(maps, args, num_sms, s);
        case 96: return launch_t<96, false, FMT>(maps, args, num_sms, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_gemm_w4(bool gateup, int wfmt, int bn, const GemmMaps &maps, const GemmArgs &args, int num_sms,
                           cudaStream_t s)
{
    switch (wfmt) {
        case MOE_W_INT4_G128: return launch_fmt<kFmtInt4>(gateup, bn, maps, args, num_sms, s);
        case MOE_W_MXFP4_G32: return launch_fmt<kFmtMx>(gateup, bn, maps, args, num_sms, s);
        case MOE_W_NVFP4_G16: return launch_fmt<kFmtNv>(gateup, bn, maps, args, num_sms, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
