// FP8 grouped GEMM with per-128-K promotion (placeholder until the tcgen05
// kind::f8f6f4 kernel lands).
#include "launch.h"

namespace moe {

moe_status launch_fp8_gemm(const void*, const float*, const void*, const float*, int,
                           const int32_t*, int, int, int, int, bool, void*, float*, cudaStream_t) {
  return fail(MOE_ERR_UNSUPPORTED, "moe_expert_ffn: the e4m3 path is not built yet");
}

}  // namespace moe
