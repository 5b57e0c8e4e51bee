// prefill_tc.cuh -- host interface of the tensor-core (tcgen05) chunkwise prefill.
#pragma once
#include "common.cuh"

namespace gret {

constexpr int TC_CHUNK = 128;  // tokens per chunk: one 128-row tcgen05 tile

size_t tc_workspace_size(int64_t total_tokens, int n_units, int H);
gret_status_t launch_prefill_tc(const PrefillArgs& a);

}  // namespace gret
