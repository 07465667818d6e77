// scan_tc.cu -- tcgen05 tensor-core scan (not built yet: no shape selects it).
#include "ssd_internal.cuh"

namespace ssd {
bool tc_supported(int, int, int) { return false; }
size_t tc_workspace_bytes(int, int, int, int, int, int) { return 0; }
cudaError_t launch_tc_scan(const ScanArgs &, void *, cudaStream_t) { return cudaErrorNotSupported; }
int tc_kernel_launches() { return 1; }
}  // namespace ssd
