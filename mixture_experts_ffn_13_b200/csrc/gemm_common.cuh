// gemm_common.cuh -- the work decomposition shared by the grouped GEMMs: a flat list of
// (group, weight-row tile, token tile) items built from the per-expert row counts.
#pragma once

#include "moe_internal.h"

namespace moe {

constexpr int kTileM = 128;  // weight rows per tile (the MMA's M side)

struct TileInfo {
    int seg;    // 0 routed, 1 shared
    int nt;     // weight-row tile index within the group
    int row0;   // first activation row (segment-relative)
    int nrows;  // valid activation rows in this tile (<= BN)
    int wrow;   // first weight row in the segment's 2-D weight view
};

// Work item w -> tile.  Routed items come first: group g owns items
// [ttile[g]*nT, ttile[g+1]*nT), laid out n-tile major so consecutive items reuse the same
// weight tile across the group's token tiles.  Shared-expert items follow.  RT is the number
// of output features (weight rows of one matrix) a tile covers: 128, or 64 when a 128-row
// MMA tile holds 64 gate rows and the matching 64 up rows.
// `stt` is a.ttile itself (read through the read-only cache) or a shared-memory copy of it
// (E+1 entries; SMEM_TT), which keeps the binary search off global memory for kernels whose
// tiles are short enough for its latency to show.
template <int BN, bool SMEM_TT = false, int RT = kTileM>
__device__ __forceinline__ TileInfo decode_tile(const GemmArgs &a, const int *stt, int w, int tot0)
{
    auto tt = [&](int i) { return SMEM_TT ? stt[i] : __ldg(stt + i); };
    TileInfo t;
    if (w < tot0) {
        const int nT = a.seg[0].N / RT;
        int lo = 0, hi = a.E - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (tt(mid) * nT <= w)
                lo = mid;
            else
                hi = mid - 1;
        }
        const int g = lo;
        const int t0 = tt(g);
        const int ntt = tt(g + 1) - t0;
        const int local = w - t0 * nT;
        const int nt = local / ntt;
        const int tt = local - nt * ntt;
        const int rbeg = __ldg(a.offsets + g) + tt * BN;
        const int rend = __ldg(a.offsets + g + 1);
        t.seg = 0;
        t.nt = nt;
        t.row0 = rbeg;
        t.nrows = min(BN, rend - rbeg);
        t.wrow = g * a.seg[0].N + nt * RT;
    } else {
        const int ww = w - tot0;
        const int ntt = (a.T + BN - 1) / BN;
        const int nt = ww / ntt;
        const int tt = ww - nt * ntt;
        t.seg = 1;
        t.nt = nt;
        t.row0 = tt * BN;
        t.nrows = min(BN, a.T - t.row0);
        t.wrow = nt * RT;
    }
    return t;
}

// Copy a.ttile into shared memory (all threads of the CTA take part; call after griddep_wait).
__device__ __forceinline__ void load_ttile(const GemmArgs &a, int *stt)
{
    for (int i = threadIdx.x; i <= a.E; i += blockDim.x) stt[i] = __ldg(a.ttile + i);
    __syncthreads();
}

__device__ __forceinline__ int total_tiles(const GemmArgs &a, int BN, int *tot0, int RT = kTileM)
{
    *tot0 = __ldg(a.ttile + a.E) * (a.seg[0].N / RT);
    const int tot1 = a.nseg > 1 ? ((a.T + BN - 1) / BN) * (a.seg[1].N / RT) : 0;
    return *tot0 + tot1;
}

// Down GEMM epilogue with the combine fused: the token and p_hat of the `ncols` permuted rows
// row0 .. row0 + ncols - 1 that this warp's columns cover, one per lane (column j*32 + lane in
// register j), loaded before the epilogue's adds so that their latency is paid once per tile.
// Routed rows take them from the permutation; the shared segment's rows are their own tokens
// with weight 1.  Columns at or beyond `nvalid` get weight 0.
template <int NREG>
__device__ __forceinline__ void combine_cols(const GemmSeg &sg, int row0, int nvalid, int lane, int (&tok)[NREG],
                                             float (&w)[NREG])
{
#pragma unroll
    for (int j = 0; j < NREG; ++j) {
        const int c = j * 32 + lane;
        const bool ok = c < nvalid;
        tok[j] = ok ? (sg.tok ? __ldg(sg.tok + row0 + c) : row0 + c) : 0;
        w[j] = ok ? (sg.rw ? __ldg(sg.rw + row0 + c) : 1.0f) : 0.0f;
    }
}

// One output value v of feature n for column c of the tile: stored as y (plain mode) or, with
// the combine fused, w * v added into the fp32 accumulator row of the column's token (atomic add
// in L2; the summation order of a token's k+1 contributions is therefore unspecified).  Lanes of
// a warp hold consecutive n, so each add instruction of a warp covers 128 contiguous bytes.
template <int NREG>
__device__ __forceinline__ void down_out(const GemmSeg &sg, const GemmArgs &a, int row, int c, int n, float v,
                                         const int (&tok)[NREG], const float (&w)[NREG])
{
    if (!sg.accum) {
        static_cast<float *>(sg.out)[(size_t)row * sg.N + n] = v;
        return;
    }
    const int t = __shfl_sync(0xffffffffu, tok[c >> 5], c & 31);
    const float wt = __shfl_sync(0xffffffffu, w[c >> 5], c & 31);
    if (a.check && (unsigned)t >= (unsigned)a.T) {
        atomicCAS(a.check, 0, MOE_ERR_BOUNDS);
        return;
    }
    atomicAdd(sg.accum + (size_t)t * sg.N + n, wt * v);
}

// silu(g) * u = g / (1 + e^-g) * u with the hardware exponential and approximate division
// (a few ulp in fp32, far below the accumulation's own rounding).  For g below about -88 the
// denominator overflows to infinity and the approximate quotient is the exact limit 0.
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

}  // namespace moe
