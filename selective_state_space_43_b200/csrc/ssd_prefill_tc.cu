// ssd_prefill_tc.cu -- tcgen05 tensor-core chunked SSD prefill (in progress).
#include "ssd_common.cuh"
#include "ssd_internal.h"

namespace ssd {

bool prefill_tc_supported(int, int, int, bool) { return false; }
size_t prefill_tc_workspace_bytes(int64_t, int64_t, int, int) { return 0; }
cudaError_t launch_prefill_tc(const PrefillArgs&, ActKind, cudaStream_t, const TimingHook&) { return cudaErrorNotSupported; }

}  // namespace ssd
