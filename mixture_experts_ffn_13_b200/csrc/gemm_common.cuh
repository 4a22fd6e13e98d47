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

// silu(g) * u = g / (1 + e^-g) * u with the hardware exponential and approximate division
// (a few ulp in fp32, far below the accumulation's own rounding).  For g below about -88 the
// denominator overflows to infinity and the approximate quotient is the exact limit 0.
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

}  // namespace moe
