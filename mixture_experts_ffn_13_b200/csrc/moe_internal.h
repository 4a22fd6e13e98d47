// moe_internal.h -- declarations shared by the library's translation units (not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe_b200.h"

namespace moe {

constexpr int kMaxE = 1024;   // router: at most 32 logits per lane
constexpr int kMaxK = 32;     // router: one lane per selected expert
constexpr int kChunk = 256;   // permutation: tokens per chunk (8 warps x 32)
constexpr int kBlockK = 512;  // FP8 sub-channel block along K
constexpr int kGroupK = 128;  // int4 scale group along K
constexpr int kMxBlock = 32;  // MXFP4 scale block along K
constexpr uint64_t kDefaultTimeoutNs = 1000000000ull;  // device-side waits give up after 1 s

// ---- the current context (context.cu) -----------------------------------------------------

// Current device, context and the context's process-unique id; makes the device's primary
// context current if the thread has none.  MOE_OK or MOE_ERR_CUDA.
int current_context(int *dev, CUcontext *ctx, unsigned long long *id);
// MOE_OK if stream `s` belongs to context `ctx`, else MOE_ERR_INVALID_ARG.
int stream_in_context(cudaStream_t s, CUcontext ctx);
// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (context, kernel): later calls with
// the same or a smaller size return without a driver call.
cudaError_t set_smem_limit(const void *func, int smem);

// ---- routing / permutation (route.cu) ---------------------------------------------------

struct RouteBufs {
    int32_t *topk_idx;    // [T, k]
    float *topk_w;        // [T, k]
    int32_t *counts;      // [E]
    int32_t *offsets;     // [E + 1]
    int32_t *perm_tok;    // [T * k]
    int32_t *pos;         // [T, k]
    int32_t *chunk_hist;  // [nchunks, E]
    int32_t *ttile_a;     // [E + 1] token-tile prefix for the gate|up GEMM tile size
    int32_t *ttile_b;     // [E + 1] token-tile prefix for the down GEMM tile size
};

// An L2 prefetch the route kernel issues before it waits on the previous kernel: `chunks`
// blocks of kChunk bytes from each of a and b (16-byte aligned), or nothing (chunks = 0).
struct WeightPrefetch {
    static constexpr uint32_t kChunk = 64 * 1024;
    const uint8_t *a = nullptr, *b = nullptr;
    uint32_t chunks = 0;
};

// check != nullptr (checked mode): non-finite logits record MOE_ERR_BOUNDS in *check.
cudaError_t launch_route(const float *logits, int T, int E, int k, int32_t *topk_idx, float *topk_w,
                         cudaStream_t s, int *check = nullptr, WeightPrefetch pf = WeightPrefetch());
cudaError_t launch_permute(const RouteBufs &b, int T, int E, int k, int bn_a, int bn_b, cudaStream_t s);
// Permutation: one single-block kernel for small batches, else the three launches above.
cudaError_t launch_permute_any(const RouteBufs &b, int T, int E, int k, int bn_a, int bn_b, cudaStream_t s);
// Router followed by launch_permute_any, and the number of kernels the pair launches.
cudaError_t launch_route_permute(const float *logits, const RouteBufs &b, int T, int E, int k, int bn_a, int bn_b,
                                 cudaStream_t s, int *check = nullptr);
int route_permute_launches(int T, int E, int k);

// ---- activation quantisation and gathers (quant.cu) --------------------------------------

// FP8: quantise each bf16 token row of x (per 512-block) and write it to the permuted rows
// pos[t, 0..k) and, when shared_rows != nullptr, to shared row t.
cudaError_t launch_quant_x_fp8(const uint16_t *x, int T, int H, int k, const int32_t *pos, uint8_t *xq,
                               float *sx, uint8_t *xq_shared, float *sx_shared, cudaStream_t s);
// FP8: quantise fp32 rows (h) per 512-block.
// h -> e4m3 per (row, 512-block) for two row segments in one launch (segment 1 skipped when
// h1 is null or R1 == 0).
cudaError_t launch_quant_rows_fp8(const float *h, int R, int K, uint8_t *q, float *sq, const float *h1, int R1,
                                  int K1, uint8_t *q1, float *sq1, cudaStream_t s);
// 4-bit layers: copy bf16 token rows into the permuted rows (and the shared rows); with
// `interleave` (int4), each aligned block of 8 elements in the order 0, 4, 1, 5, 2, 6, 3, 7.
cudaError_t launch_gather_x_bf16(const uint16_t *x, int T, int H, int k, const int32_t *pos, uint16_t *xp,
                                 uint16_t *xp_shared, bool interleave, cudaStream_t s);

// ---- combine (combine.cu) ----------------------------------------------------------------

// check != nullptr (checked mode): a permuted row index outside [0, T*k) records
// MOE_ERR_BOUNDS in *check.
cudaError_t launch_combine(const float *y, const float *y_shared, const int32_t *pos, const float *topk_w,
                           int T, int H, int k, uint16_t *out, cudaStream_t s, int *check = nullptr);

// ---- grouped GEMMs (gemm_fp8.cu, gemm_int4.cu) -------------------------------------------

// One segment of a grouped GEMM: either the routed experts (E groups whose activation rows
// are given by offsets) or the shared expert (one group over T rows).
struct GemmSeg {
    int N;          // weight rows (output features) per group, multiple of 128
    int K;          // reduction length, multiple of 128
    int rows;       // activation rows of this segment
    const void *sw0;  // scales of the first weight matrix  (gate, or down)
    const void *sw1;  // scales of the second weight matrix (up), gate|up only
    const float *sx;  // activation scales [rows, ceil(K/512)] (FP8 only)
    void *out;        // gate|up: h [rows, N]; down: y [rows, N]
    int ilv4d;        // interleaved gate|up: a0 is one 4-D map that loads 16 gate + 16 up rows per quarter
    int up_lo;        // interleaved gate|up: the up rows come first in each 32-row quarter
    const float *ts0; // NVFP4: fp32 tensor scales of the first / second weight matrix, one per
    const float *ts1; //   group (routed: [E], shared: [1]); unused otherwise
};

struct GemmArgs {
    GemmSeg seg[2];
    int nseg;                // 1 (routed only) or 2 (routed + shared)
    int E;                   // routed groups
    int T;                   // shared-expert rows
    const int32_t *offsets;  // [E + 1] routed group row offsets
    const int32_t *ttile;    // [E + 1] routed token-tile prefix for this GEMM's tile size
    int *status;             // device status word
    uint64_t timeout_ns;
};

// Tensor maps of one GEMM launch: A (weights) 0 and 1 per segment, B (activations) per segment.
struct GemmMaps {
    CUtensorMap a0[2], a1[2], b[2];
};

// FP8 grouped GEMMs.  gateup: h = silu(x Wg^T) * (x Wu^T) in fp32; down: y = h Wd^T in fp32.
cudaError_t launch_gemm_fp8(bool gateup, int bn, const GemmMaps &maps, const GemmArgs &args, int num_sms,
                            cudaStream_t s);
// 4-bit grouped GEMMs over bf16 activations (wfmt: MOE_W_INT4_G128, MOE_W_MXFP4_G32 or
// MOE_W_NVFP4_G16): gate|up writes h as bf16, down writes y fp32.
cudaError_t launch_gemm_w4(bool gateup, int wfmt, int bn, const GemmMaps &maps, const GemmArgs &args,
                           int num_sms, cudaStream_t s);

// Small batches (2 <= T <= 16, FP8 weights): the whole layer in one cooperative persistent kernel
// (small_batch.cu).  small_batch_fits: shapes it takes (H a multiple of 2048 up to 4096, I and
// I_shared multiples of 512 up to 2048); small_batch_workspace: the bytes it needs in the
// workspace (partial sums, y rows, a grid-barrier counter).  launch_small_batch returns
// cudaErrorNotSupported, before any device work, when the gate and up weight arrays are too far
// apart for one tensor map (the caller then takes the regular path).
bool small_batch_fits(int T, const moe_dims &d);
size_t small_batch_workspace(const moe_dims &d);
cudaError_t launch_small_batch(const moe_dims &d, int T, const uint16_t *x, const float *logits,
                               const moe_weights *w, uint16_t *out, void *ws, int *status, int num_sms,
                               cudaStream_t s, int *launched);

// Router logits [T, E] (written) and their softmax top-k (step A1): the router GEMM, then the
// route kernel.
cudaError_t launch_router_topk(const uint16_t *x, const uint16_t *w, float *logits, int32_t *topk_idx, float *topk_w,
                               int T, int H, int E, int k, int *status, int num_sms, cudaStream_t s);
// Router logits: logits[T, E] = x[T, H] . W[E, H]^T (bf16 in, fp32 out) on the tensor cores.
cudaError_t launch_router_gemm(const uint16_t *x, const uint16_t *w, float *logits, int T, int H, int E, int *status,
                               int num_sms, cudaStream_t s);

// Tensor-map encoding through the driver entry point (host).
int encode_map_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes,
                  uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer, bool swizzle128);
// One 4-D map over two byte matrices gate, up [rows, K] (rows a multiple of 16) whose box of
// (128 bytes, 16 rows, 2 matrices, 4 row groups) lands in shared memory as 128 rows ordered
// [16 rows of the lower-addressed matrix, the same 16 rows of the other] x 4.  Sets *up_lo
// when the up matrix has the lower address.  Returns non-zero when the two matrices are too
// far apart (or misaligned) for one map.
int encode_map_gateup_ilv(CUtensorMap *map, const void *gate, const void *up, uint64_t K, uint64_t rows, int *up_lo);

}  // namespace moe
