// Placeholder: the tcgen05 forward is not enabled yet.
#include "internal.h"
namespace fa {
bool sm100_fwd_supported(const Problem&) { return false; }
cudaError_t sm100_fwd(const Problem&) { return cudaErrorNotSupported; }
}  // namespace fa
