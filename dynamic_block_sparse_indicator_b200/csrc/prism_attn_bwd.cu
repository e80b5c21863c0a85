// prism_attn_bwd.cu -- gradients of the block-sparse attention (placeholder
// until the tensor-core backward lands).
#include "prism_internal.h"

int prism_launch_attn_bwd(prism_plan_s* P, const void* dO, const void* O, const float* lse,
                          void* dQ, void* dK, void* dV, void* stream) {
    (void)P; (void)dO; (void)O; (void)lse; (void)dQ; (void)dK; (void)dV; (void)stream;
    return PRISM_ERR_UNSUPPORTED;
}
