// Tensor-core (tcgen05) grouped expert FFN: placeholder until the kernel lands.
#include "moe_internal.cuh"

namespace moe {

bool ffn_tc_supported(const moe_shape&) { return false; }

cudaError_t launch_ffn_tc(const Ctx&, const moe_dispatch_bufs&, const moe_weights&, void*) {
  return cudaErrorNotSupported;
}

}  // namespace moe
