// Internal launch interface between the C-ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "kda.h"

namespace kda {

struct ChunkArgs {
    const void *q, *k, *v, *log_alpha, *beta;
    const float* S0;
    void* o;
    float* ST;
    int B, T, H, dk, dv, chunk;
    int bf16;
    int erase;  // 1: delta-rule family (I - beta k k^T), 0: additive write beta k v^T
    int gate;   // 0: log_alpha per key channel [.., dk]; 1: one per token and head [B, T, H]; 2: none
    // Packed variable-length sequences (NULL: dense [B, T, H, .] batch). When
    // set, B is the number of sequences, T the packed token count, and
    // sequence b owns tokens [cu_seqlens[b], cu_seqlens[b+1]) of the [1, T, H, .]
    // tensors; kernels clamp the offsets into [0, T].
    const int* cu_seqlens;
    void* workspace;
    size_t workspace_bytes;
    // Fault injection for the timeout test (tensor-core prefill only): withhold
    // the first k/q load of every CTA and bound each wait by this many SM
    // cycles, so the first wait expires. Zero in every other call.
    int test_withhold_first_load = 0;
    long long test_wait_budget = 0;
};

// Synchronous argument validation shared by every prefill entry point
// (sizes, dtype, head and chunk sizes, variant switches, required pointers
// and their 16-byte alignment). Launches nothing.
kda_status_t check_chunk_args(const ChunkArgs& a, kda_dtype_t dtype);

cudaError_t launch_decode(const void* q, const void* k, const void* v, const void* la, const void* beta,
                          const float* S_in, float* S_out, void* o, int N, int H, int dk, int dv, int bf16,
                          int erase, int gate, cudaStream_t stream);

cudaError_t launch_chunk_simt(const ChunkArgs& a, cudaStream_t stream);

// Fused tensor-core prefill (bf16, dk = dv = 128, chunk = 64).
bool chunk_tc_supported(const ChunkArgs& a);
// scan_mode: 0 one pass per sequence; 1 the chunk-parallel segment scan where
// it pays (dense batch, few heads, long T); 2 the scan whenever T has 3 chunks.
size_t chunk_tc_workspace_bytes(const ChunkArgs& a, int scan_mode);
cudaError_t launch_chunk_tc(const ChunkArgs& a, int scan_mode, cudaStream_t stream);

// Backward of the chunkwise prefill (SIMT fp32, any variant, dk = dv = d in {64, 128}).
struct BwdArgs {
    const void *q, *k, *v, *log_alpha, *beta, *dO;
    const float *S0, *dST;
    void *g_q, *g_k, *g_v, *g_log_alpha, *g_beta;  // gradients (input dtype)
    float* g_S0;
    int B, T, H, d, bf16, erase, gate;
    int mode;  // 0: keep every chunk's state while that fits 16 GB; 1: always; 2: one per 64 tokens
    void* workspace;
    size_t workspace_bytes;
};
size_t chunk_bwd_workspace_bytes(int B, int T, int H, int d, int mode);
cudaError_t launch_chunk_bwd(const BwdArgs& a, cudaStream_t stream);

}  // namespace kda
