// Causal attention on the sm_100a tensor cores (tcgen05).  Until the
// tensor-core kernels are enabled, attn_tc_supported() reports false and the
// step runs the flash-style CUDA-core kernels of k_attn_simt.cu.
#include "kernels.cuh"

namespace gpt {

bool attn_tc_supported(const AttnDesc&) { return false; }
void attn_fwd_tc(Ctx&, const AttnDesc&) {}
void attn_bwd_tc(Ctx&, const AttnDesc&) {}

}  // namespace gpt
