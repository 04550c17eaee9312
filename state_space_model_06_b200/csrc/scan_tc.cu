// scan_tc.cu -- tcgen05 chunked prefill (placeholder until the kernel lands).
#include "m3_internal.h"

namespace m3 {

bool scan_tc_supported(int, int, int, int) { return false; }
size_t scan_tc_workspace_bytes(int, int, int, int, int, long long, int) { return 0; }
cudaError_t launch_scan_tc(const ScanArgs&, int, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace m3
