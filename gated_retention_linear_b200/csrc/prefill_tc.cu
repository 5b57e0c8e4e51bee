// prefill_tc.cu -- tensor-core chunkwise prefill (placeholder until the tcgen05 kernel lands).
#include "prefill_tc.cuh"

namespace gret {

size_t tc_workspace_size(int64_t, int, int) { return 256; }
gret_status_t launch_prefill_tc(const PrefillArgs&) { return GRET_ERR_UNSUPPORTED; }

}  // namespace gret
