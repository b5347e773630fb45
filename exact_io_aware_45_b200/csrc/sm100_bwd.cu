// Placeholder: the tcgen05 backward is not built yet.
#include "internal.h"
namespace fa {
bool sm100_bwd_supported(const Problem&) { return false; }
bool sm100_bwd_uses_dq_accumulator(const Problem&) { return false; }
cudaError_t sm100_bwd_main(const Problem&) { return cudaErrorNotSupported; }
}  // namespace fa
