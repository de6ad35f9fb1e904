// scan_tc.cu -- tensor-core chunked scan (placeholder until the tcgen05 kernel lands).
#include "ssm_internal.h"

namespace ssm {

bool scan_tc_supports(const ScanArgs &) { return false; }

cudaError_t launch_scan_tc(const ScanArgs &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace ssm
