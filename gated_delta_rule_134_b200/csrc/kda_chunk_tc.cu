// Fused tensor-core prefill: placeholder until the tcgen05 kernel lands.
#include "kda_internal.h"

namespace kda {
bool chunk_tc_supported(const ChunkArgs&) { return false; }
size_t chunk_tc_workspace_bytes(int, int, int, int, int) { return 0; }
cudaError_t launch_chunk_tc(const ChunkArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace kda
