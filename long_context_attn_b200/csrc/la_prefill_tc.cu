// Placeholder: the tcgen05 prefill kernel is not built yet; every call takes the SIMT path.
#include "la_prefill_tc.h"

namespace la {
bool tc_eligible(const TcShape&, int) { return false; }
size_t tc_workspace_bytes(int, int, int64_t, int, int, int) { return 0; }
cudaError_t launch_tc_prefill(const TcArgs&, int, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace la
