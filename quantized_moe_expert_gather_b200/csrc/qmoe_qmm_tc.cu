// Tensor-core (tcgen05 / TMEM) gathered quantised matmul for many rows per expert.
#include "qmoe_internal.h"

namespace qmoe {

bool qmm_tc_supported(const GemmArgs&) { return false; }

cudaError_t launch_qmm_tc(const GemmArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace qmoe
