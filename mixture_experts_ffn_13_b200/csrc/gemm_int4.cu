// gemm_int4.cu -- steps A4/A5 for 4-bit weights (filled in below the FP8 path).
#include "moe_internal.h"

namespace moe {

cudaError_t launch_gemm_int4(bool, int, const GemmMaps &, const GemmArgs &, int, cudaStream_t)
{
    return cudaErrorNotSupported;
}

}  // namespace moe
