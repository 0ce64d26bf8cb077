// attn_fp4.cu -- fused FP4 (NVFP4-style) attention forward for sm_100a.
#include "sage_internal.h"

namespace sage {

cudaError_t launch_attn_fp4(const AttnArgs&, cudaStream_t, const char** detail) {
  if (detail) *detail = "the FP4 attention kernel is not built into this library yet";
  return cudaErrorNotSupported;
}

}  // namespace sage
