// Causal tensor-core forward (filled in below; not yet available).
#include "internal.h"

namespace dark {
bool tc_causal_supported(const FwdArgs&) { return false; }
size_t tc_causal_workspace_bytes(int, int, int, int, int) { return 0; }
cudaError_t tc_causal_forward(const FwdArgs&) { return cudaErrorNotSupported; }
}  // namespace dark
