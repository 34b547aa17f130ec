// Tensor-core kernel placeholder (filled in by the tcgen05 implementation).
#include "fq_internal.h"

namespace fq {
bool tc_supported(int64_t, int, int) { return false; }
cudaError_t launch_tc(const TcParams&, bool, int, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace fq
