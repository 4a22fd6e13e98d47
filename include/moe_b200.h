/*
 * moe_b200.h -- C ABI of the routed Mixture-of-Experts FFN layer on NVIDIA B200 (sm_100a).
 *
 * The layer (page "把 397B MoE 榨進 TPU7x：Google 拿到 4.7 倍加速", sections "稀疏在哪裡" and
 * "Kernel 手術台"; page "Flash-Next 在 GPU 上到底在算什麼", section "① 專家 FFN"):
 *
 *   route:    per token t, the k experts with the largest router logits (ties: lower index
 *             first), p_hat[t,j] = softmax over those k logits;
 *   permute:  the T*k (token, expert) assignments sorted by the key (expert, token) into
 *             contiguous per-expert groups (page "TPU推理外部化全面加速：InferenceX首份第三方性能
 *             數據發布", section "优化 MoE 路由与专家内核": packed expert/token sort key);
 *   experts:  h = silu(x Wg^T) * (x Wu^T),  y = h Wd^T  for each assignment, plus one shared
 *             expert of intermediate size I_shared that every token runs with weight 1;
 *   combine:  out[t] = sum_j p_hat[t,j] * y(t, e_j) + y_shared(t), rounded to bf16.
 *
 * Weight formats:
 *   MOE_W_FP8_SC512: e4m3 codes, row-major [out, in] (K-major), one fp32 scale per
 *     (row, 512-element block of K); activations (x and h) are quantised to e4m3 with one
 *     fp32 scale per (row, 512-block): s = amax/448 (1 when amax = 0), q = e4m3_rn_satfinite(v/s).
 *   MOE_W_INT4_G128: symmetric int4, two's-complement nibbles, two per byte with the even K
 *     index in the low nibble, [out, in/2] bytes; one bf16 scale per (row, 128-element
 *     K group); activations stay bf16 (h is rounded to bf16).
 *   MOE_W_MXFP4_G32: OCP Microscaling FP4 (page "设计 AI 芯片的硬件与软件", section "数值格式，
 *     或如何制造便宜的脉动阵列": 4-bit values plus an 8-bit scale per 32, 4.25 bits per number).
 *     E2M1 nibbles (sign, 2 exponent bits with bias 1, 1 mantissa bit: magnitudes 0, 0.5, 1,
 *     1.5, 2, 3, 4, 6), two per byte with the even K index in the low nibble, [out, in/2]
 *     bytes; one E8M0 byte c per (row, 32-element K block), the scale 2^(c-127).  The weight
 *     e2m1 * 2^(c-127) is formed exactly for c in 2..252 (other codes are outside the
 *     supported domain: the product may flush to zero or overflow).  Activations stay bf16
 *     (h is rounded to bf16), as for int4.
 *   MOE_W_NVFP4_G16: NVFP4 (the NVIDIA co-design commentary, section "讀的時候記得這是廠商文":
 *     two levels of scale factors).  E2M1 nibbles as for MXFP4; one E4M3 byte per (row,
 *     16-element K block), a positive finite value; one fp32 tensor scale per weight matrix
 *     (per expert and projection).  The weight is e2m1 * e4m3(s) * t: the first product is
 *     formed exactly in bf16, t multiplies the fp32 accumulator.  Activations stay bf16.
 *
 * Pointer conventions.  Every buffer passed to moe_router_logits / moe_route / moe_forward is
 * DEVICE memory that the caller allocates and owns; the library keeps no pointer to it after
 * the call returns.  All calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 * default stream) and never synchronise the host, except moe_get_status.  moe_forward
 * allocates nothing and only enqueues kernels on `stream`, so a call can be captured into a
 * CUDA graph and replayed (inputs updated in place between replays).  Rows are contiguous (stride = row
 * length).  Every pointer must be 16-byte aligned.  bf16 values are passed as uint16 bit
 * patterns.
 *
 * Errors.  Functions return MOE_OK (0) or a negative MOE_ERR_* code; on error the output
 * buffers hold unspecified values.  No function aborts the process.  Device-side waits are
 * bounded: a kernel that gives up records MOE_ERR_DEVICE_TIMEOUT in the plan's status word,
 * which moe_get_status reports.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* the same type as cudaStream_t */

enum moe_wfmt {
    MOE_W_FP8_SC512 = 1, /* e4m3 weights + fp32 scale per (row, 512-block of K) */
    MOE_W_INT4_G128 = 2, /* int4 weights + bf16 scale per (row, 128-group of K) */
    MOE_W_MXFP4_G32 = 3, /* E2M1 weights + E8M0 scale per (row, 32-block of K) */
    MOE_W_NVFP4_G16 = 4  /* E2M1 weights + E4M3 scale per (row, 16-block of K) + fp32 per matrix */
};

enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,    /* NULL / misaligned pointer, T > T_max, k outside [1, E] ... */
    MOE_ERR_UNSUPPORTED = -2,    /* shape the kernels do not handle (see moe_plan) */
    MOE_ERR_WORKSPACE = -3,      /* workspace NULL or smaller than moe_plan reported */
    MOE_ERR_CUDA = -4,           /* a CUDA runtime call or kernel launch failed */
    MOE_ERR_DEVICE_TIMEOUT = -5, /* a bounded device-side wait gave up (from moe_get_status) */
    MOE_ERR_BOUNDS = -6          /* a checked-mode device check failed: a non-finite router logit or a
                                    permuted row index out of range (from moe_get_status) */
};

typedef struct {
    int32_t T_max;    /* largest token count any later call will pass */
    int32_t H;        /* hidden size */
    int32_t E;        /* routed experts */
    int32_t I;        /* intermediate size of each routed expert */
    int32_t k;        /* experts per token, 1 <= k <= min(E, 32) */
    int32_t I_shared; /* intermediate size of the shared expert, 0 = no shared expert */
    int32_t wfmt;     /* enum moe_wfmt */
} moe_dims;

/* Expert weights and scales (device pointers, caller-owned).
 *   FP8:  w_gate, w_up [E, I, H] e4m3; w_down [E, H, I] e4m3;
 *         s_gate, s_up [E, I, ceil(H/512)] fp32; s_down [E, H, ceil(I/512)] fp32.
 *   int4: w_gate, w_up [E, I, H/2] bytes; w_down [E, H, I/2] bytes;
 *         s_gate, s_up [E, I, H/128] bf16; s_down [E, H, I/128] bf16.
 *   MXFP4: w_* as int4 (E2M1 nibbles); s_gate, s_up [E, I, H/32] bytes; s_down [E, H, I/32]
 *         bytes (E8M0).
 *   NVFP4: w_* as int4 (E2M1 nibbles); s_gate, s_up [E, I, H/16] bytes; s_down [E, H, I/16]
 *         bytes (E4M3); t_gate, t_up, t_down [E] fp32 tensor scales (ts_*: [1]).  The t_* and
 *         ts_* fields are read for NVFP4 only (NULL otherwise).
 *   ws_* / ss_*: the shared expert in the same format with E = 1 and I -> I_shared; NULL when
 *   I_shared == 0. */
typedef struct {
    const void *w_gate, *w_up, *w_down;
    const void *s_gate, *s_up, *s_down;
    const void *ws_gate, *ws_up, *ws_down;
    const void *ss_gate, *ss_up, *ss_down;
    const float *t_gate, *t_up, *t_down;
    const float *ts_gate, *ts_up, *ts_down;
} moe_weights;

typedef struct moe_plan_s moe_plan_t; /* opaque; owned by the library until moe_destroy */

/* Validate the dimensions, choose tile shapes and report the workspace size the later calls
 * need for any T <= T_max.  Launches no kernel.  Allocates one small device status word on
 * the current device (the plan is bound to that device).
 * Supported: 1 <= E <= 1024; 1 <= k <= min(E, 32); H, I, I_shared multiples of 128, <= 8192;
 * 1 <= T_max <= 2^20.  Returns MOE_ERR_INVALID_ARG for NULL outputs or non-positive sizes,
 * MOE_ERR_UNSUPPORTED for shapes outside that set. */
MOE_API int moe_plan(const moe_dims *dims, moe_plan_t **out_plan, size_t *workspace_bytes);

/* Router logits, the dense 16-bit layer that feeds step A1 (page "Flash-Next 在 GPU 上到底在算
 * 什麼", section "② 密集 16-bit 層": the router runs in 16 bits on the tensor cores):
 *   logits[T, E] (fp32, out) = x[T, H] (bf16) . w_router[E, H]^T (bf16, row-major [out, in]),
 * accumulated in fp32 on tcgen05 tensor cores.  Uses the plan's H and E; needs no workspace;
 * 0 <= T <= T_max.  The result can be passed to moe_route / moe_forward.  All pointers are
 * device pointers, 16-byte aligned, caller-owned.  Returns MOE_ERR_INVALID_ARG for a NULL plan,
 * T outside [0, T_max], NULL or misaligned buffers (T > 0); MOE_ERR_CUDA if the launch fails;
 * a device-side wait that runs out sets the plan's status (moe_get_status). */
MOE_API int moe_router_logits(moe_plan_t *plan, int32_t T, const uint16_t *x_bf16, const uint16_t *w_router_bf16,
                              float *logits, moe_stream_t stream);

/* Router logits and step A1 from hidden states (the pages' router as one dense 16-bit layer
 * followed by the softmax top-k, page "Flash-Next 在 GPU 上到底在算什麼", section "② 密集 16-bit
 * 層"): logits as moe_router_logits ([T, E] fp32, written), then topk_idx [T, k] int32 and
 * topk_w [T, k] fp32 with the conventions of moe_route, by the route kernel on those logits
 * (two launches, the second overlapping the first's tail).  Device pointers, 16-byte aligned,
 * caller-owned; 0 <= T <= T_max; no workspace.  Errors as moe_router_logits. */
MOE_API int moe_router_topk(moe_plan_t *plan, int32_t T, const uint16_t *x_bf16, const uint16_t *w_router_bf16,
                            float *logits, int32_t *topk_idx, float *topk_w, moe_stream_t stream);

/* Route and permute only (steps A1 and A3), for inspection and parity checks.
 *   logits   [T, E] fp32 (finite values; the caller guarantees it)
 *   topk_idx [T, k] int32 out: experts by (logit desc, index asc)
 *   topk_w   [T, k] fp32  out: p_hat, softmax over the k selected logits
 *   counts   [E] int32 out; offsets [E+1] int32 out (exclusive prefix sum of counts)
 *   perm_tok [T*k] int32 out: token of each permuted row, rows sorted by (expert, token)
 * 0 <= T <= T_max (T = 0 writes counts = offsets = 0). */
MOE_API int moe_route(moe_plan_t *plan, int32_t T, const float *logits, int32_t *topk_idx, float *topk_w,
              int32_t *counts, int32_t *offsets, int32_t *perm_tok, void *workspace,
              size_t ws_bytes, moe_stream_t stream);

/* Routing and permutation without any allocation, for callers that cannot call cudaMalloc
 * (code inside an allocator or pool callback, serving loops that forbid allocation after
 * start-up, embedders whose device memory another allocator has reserved).  The pages have no
 * counterpart: this is a library convenience.  Same outputs and argument rules as moe_route,
 * but no plan and no workspace: its scratch is one fixed 2 MiB __device__ array in the library
 * (held by every GPU that loads it until the process exits), so
 *   T*k + ceil(T/256)*E + 2*(E+1) <= 2^19 is required (else MOE_ERR_UNSUPPORTED, before any
 *   device work), with 1 <= k <= min(E, 32) and E <= 1024;
 *   the first call on a device looks up the array's address (cudaGetSymbolAddress, with the
 *   device current; again after the device's context is replaced, e.g. by cudaDeviceReset)
 *   -- make that first call before any stream capture;
 *   `stream` must belong to the current device (else MOE_ERR_INVALID_ARG) and the buffers must
 *   live on it;
 *   all calls share the array: calls whose kernels may overlap on the GPU race and must be
 *   serialised by the caller.
 * Returns MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED or MOE_ERR_CUDA. */
MOE_API int moe_route_static(int32_t T, int32_t E, int32_t k, const float *logits, int32_t *topk_idx,
                             float *topk_w, int32_t *counts, int32_t *offsets, int32_t *perm_tok,
                             moe_stream_t stream);

/* The whole layer: out[T, H] (bf16) from x[T, H] (bf16), logits[T, E] (fp32) and the
 * weights.  0 <= T <= T_max.  The workspace (>= the size moe_plan reported, 256-byte
 * aligned) holds every intermediate; its contents are undefined after the call. */
MOE_API int moe_forward(moe_plan_t *plan, int32_t T, const uint16_t *x_bf16, const float *logits,
                const moe_weights *weights, uint16_t *out_bf16, void *workspace, size_t ws_bytes,
                moe_stream_t stream);

/* The whole layer from hidden states: the router logits x . W_router^T (as moe_router_logits,
 * written into the workspace) and then exactly the work of moe_forward on them.  w_router is
 * bf16 [E, H] (device, 16-byte aligned).  Same workspace (moe_plan's size covers the logits),
 * outputs and errors as moe_forward; no argument error launches anything.  (The logits share
 * the workspace bytes of the down projection's output, which is written only after routing.) */
MOE_API int moe_forward_x(moe_plan_t *plan, int32_t T, const uint16_t *x_bf16, const uint16_t *w_router_bf16,
                          const moe_weights *weights, uint16_t *out_bf16, void *workspace, size_t workspace_bytes,
                          moe_stream_t stream);

/* Synchronise `stream`, read and clear the plan's device status word.  Returns MOE_OK,
 * MOE_ERR_DEVICE_TIMEOUT or MOE_ERR_BOUNDS (or MOE_ERR_CUDA if the copy itself fails). */
MOE_API int moe_get_status(moe_plan_t *plan, moe_stream_t stream);

/* The last CUDA error code seen by a call that returned MOE_ERR_CUDA (cudaError_t value). */
MOE_API int moe_last_cuda_error(const moe_plan_t *plan);

/* Release the plan and its status word.  NULL is accepted. */
MOE_API void moe_destroy(moe_plan_t *plan);

/* Tracing.  moe_profile_enable(plan, 1) creates one CUDA event per stage boundary (on the
 * plan's device); later moe_forward calls then record them on their stream around each stage:
 * 0 route, 1 permute, 2 quantise x, 3 gate|up GEMM, 4 quantise h, 5 down GEMM, 6 combine.
 * moe_profile_read waits for the events of the last call and writes each stage's device time
 * in milliseconds to ms[0..n) (n = min(max_stages, stage count)); it returns n, or a negative
 * MOE_ERR_* code (MOE_ERR_INVALID_ARG when profiling is off or no call was recorded).
 * moe_profile_enable(plan, 0) releases the events. */
MOE_API int moe_profile_enable(moe_plan_t *plan, int enable);
MOE_API int moe_profile_read(moe_plan_t *plan, float *ms, int max_stages);
MOE_API const char *moe_profile_stage_name(int stage);

/* Checked mode (off by default): with enable != 0, later moe_route / moe_forward /
 * moe_forward_x calls on this plan also verify on the device that every router logit is
 * finite (non-finite logits are caller error) and that every permuted row index the combine
 * reads is in range; a failed check records MOE_ERR_BOUNDS in the plan's status word
 * (moe_get_status) and the outputs of that call are unspecified.  Costs one extra read of the
 * logits.  Returns MOE_OK or MOE_ERR_INVALID_ARG (NULL plan). */
MOE_API int moe_set_checked(moe_plan_t *plan, int enable);

/* Number of kernels the last router / route / forward call on this plan launched. */
MOE_API int moe_launch_count(const moe_plan_t *plan);

/* A static, human-readable name of a status code. */
MOE_API const char *moe_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
