// K2: tensor-core (tcgen05) prefill attention -- not yet built; the dispatcher never selects it.
#include "attention.cuh"

namespace spt {
bool attn_tc_supported(const spatten_attn_args&) { return false; }
int32_t attn_tc_launch(const AttnProblem&, cudaStream_t) { return SPATTEN_E_UNSUPPORTED; }
}  // namespace spt
