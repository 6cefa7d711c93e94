// Mamba-2 SSD chunked scan (sm_100a, tcgen05) -- under construction.
#include "common.cuh"
#include "internal.h"

namespace ssmq {

size_t ssd_workspace_bytes(const ssmq_ssd_args&) { return 0; }

cudaError_t launch_ssd(const ssmq_ssd_args&, void*, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace ssmq
