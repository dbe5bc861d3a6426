// Data-parallel gradient exchange: internal entry points of gpt2_dp.cu.
#pragma once

#include <cstdint>
#include <utility>
#include <vector>

#include "common.cuh"

namespace gpt2_internal {
// NCCL communicator over `world` ranks from a unique id (GPT2_DP_ID_BYTES)
int dp_comm_init(void** comm, const char* id, int rank, int world);
void dp_comm_destroy(void* comm);
// in-place average over the ranks of grad[off .. off + n) for each (off, n), on st
int dp_allreduce_ranges(void* comm, const std::vector<std::pair<int64_t, int64_t>>& ranges,
                        float* grad, cudaStream_t st);
}  // namespace gpt2_internal
