// C-ABI layer of libkda.so: argument validation, workspace sizing and
// dispatch to the kernels. Declarations and contracts are in include/kda.h.
#include <stdint.h>

#include "kda.h"
#include "kda_internal.h"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool head_dims_ok(int dk, int dv) { return dk == dv && (dk == 64 || dk == 128); }

// 0: one pass per sequence; 1: the segment scan where it pays; 2: the scan forced.
int scan_mode_of(kda_algo_t algo) { return algo == KDA_ALGO_TC_SCAN ? 2 : (algo == KDA_ALGO_AUTO ? 1 : 0); }

kda_status_t run_chunk(const kda::ChunkArgs& a, kda_dtype_t dtype, kda_algo_t algo, void* stream);

}  // namespace

kda_status_t kda::check_chunk_args(const kda::ChunkArgs& a, kda_dtype_t dtype) {
    if (a.B < 0 || a.T < 0 || a.H < 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (!head_dims_ok(a.dk, a.dv)) return KDA_ERR_UNSUPPORTED;
    if (a.chunk != 16 && a.chunk != 32 && a.chunk != 64) return KDA_ERR_UNSUPPORTED;
    if ((long long)a.B * a.H > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    if (a.erase != 0 && a.erase != 1) return KDA_ERR_INVALID_ARG;
    if (a.gate < KDA_GATE_CHANNEL || a.gate > KDA_GATE_NONE) return KDA_ERR_INVALID_ARG;
    const bool has_tokens = (long long)a.B * a.T * a.H > 0;
    if (has_tokens) {
        const void* req[] = {a.q, a.k, a.v, a.beta, a.o};
        for (const void* p : req)
            if (p == nullptr || !aligned16(p)) return KDA_ERR_INVALID_ARG;
        if (a.gate != KDA_GATE_NONE && (a.log_alpha == nullptr || !aligned16(a.log_alpha)))
            return KDA_ERR_INVALID_ARG;
    }
    if (a.S0 && !aligned16(a.S0)) return KDA_ERR_INVALID_ARG;
    if (a.ST && !aligned16(a.ST)) return KDA_ERR_INVALID_ARG;
    return KDA_OK;
}

extern "C" {

const char* kda_status_string(kda_status_t s) {
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: null/misaligned pointer, bad size or workspace too small";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: head size, chunk size or algorithm not implemented";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA: CUDA launch or query failed";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: a bounded device-side wait expired";
    }
    return "KDA: unknown status";
}

size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int chunk, kda_dtype_t dtype,
                                    kda_algo_t algo) {
    kda::ChunkArgs a{};
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv; a.chunk = chunk; a.bf16 = dtype == KDA_BF16;
    a.erase = 1; a.gate = KDA_GATE_CHANNEL; a.cu_seqlens = nullptr;
    if (B < 0 || T < 0 || H < 0 || !head_dims_ok(dk, dv)) return 0;
    const bool tc = (algo == KDA_ALGO_TC) || (algo == KDA_ALGO_TC_SCAN) ||
                    (algo == KDA_ALGO_AUTO && kda::chunk_tc_supported(a));
    return tc ? kda::chunk_tc_workspace_bytes(a, scan_mode_of(algo)) : 0;
}

kda_status_t kda_chunk_fwd_v(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                             const float* S0, void* o, float* S_T, int B, int T, int H, int dk, int dv, int chunk,
                             kda_dtype_t dtype, int erase, kda_gate_t gate, void* workspace, size_t workspace_bytes,
                             kda_algo_t algo, void* stream) {
    kda::ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.S0 = S0; a.o = o; a.ST = S_T;
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv; a.chunk = chunk; a.bf16 = dtype == KDA_BF16;
    a.erase = erase; a.gate = (int)gate;
    a.cu_seqlens = nullptr;
    a.workspace = workspace; a.workspace_bytes = workspace_bytes;
    return run_chunk(a, dtype, algo, stream);
}

kda_status_t kda_chunk_fwd_varlen(const void* q, const void* k, const void* v, const void* log_alpha,
                                  const void* beta, const float* S0, void* o, float* S_T, const int* cu_seqlens,
                                  int N, int total_T, int H, int dk, int dv, int chunk, kda_dtype_t dtype, int erase,
                                  kda_gate_t gate, void* workspace, size_t workspace_bytes, kda_algo_t algo,
                                  void* stream) {
    if (N < 0 || total_T < 0) return KDA_ERR_INVALID_ARG;
    if (N > 0 && (cu_seqlens == nullptr || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0))
        return KDA_ERR_INVALID_ARG;
    kda::ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.S0 = S0; a.o = o; a.ST = S_T;
    a.B = N; a.T = total_T; a.H = H; a.dk = dk; a.dv = dv; a.chunk = chunk; a.bf16 = dtype == KDA_BF16;
    a.erase = erase; a.gate = (int)gate;
    a.cu_seqlens = cu_seqlens;
    a.workspace = workspace; a.workspace_bytes = workspace_bytes;
    return run_chunk(a, dtype, algo, stream);
}

}  // extern "C"

namespace {

kda_status_t run_chunk(const kda::ChunkArgs& a, kda_dtype_t dtype, kda_algo_t algo, void* stream) {
    const int B = a.B, T = a.T, H = a.H, dk = a.dk, dv = a.dv;
    void* workspace = a.workspace;
    const size_t workspace_bytes = a.workspace_bytes;
    kda_status_t st = kda::check_chunk_args(a, dtype);
    if (st != KDA_OK) return st;
    if (algo != KDA_ALGO_AUTO && algo != KDA_ALGO_SIMT && algo != KDA_ALGO_TC && algo != KDA_ALGO_TC_SCAN)
        return KDA_ERR_INVALID_ARG;
    const bool tc = (algo == KDA_ALGO_TC) || (algo == KDA_ALGO_TC_SCAN) ||
                    (algo == KDA_ALGO_AUTO && kda::chunk_tc_supported(a));
    if (tc && !kda::chunk_tc_supported(a)) return KDA_ERR_UNSUPPORTED;
    if (algo == KDA_ALGO_TC_SCAN && a.cu_seqlens) return KDA_ERR_UNSUPPORTED;
    if (tc) {
        const size_t need = kda::chunk_tc_workspace_bytes(a, scan_mode_of(algo));
        if (need > 0 && (workspace == nullptr || workspace_bytes < need ||
                         (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0))
            return KDA_ERR_INVALID_ARG;
    }
    if ((long long)B * H == 0) return KDA_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t err = tc ? kda::launch_chunk_tc(a, scan_mode_of(algo), s) : kda::launch_chunk_simt(a, s);
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace

extern "C" {

kda_status_t kda_chunk_fwd_ex(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                              const float* S0, void* o, float* S_T, int B, int T, int H, int dk, int dv, int chunk,
                              kda_dtype_t dtype, void* workspace, size_t workspace_bytes, kda_algo_t algo,
                              void* stream) {
    return kda_chunk_fwd_v(q, k, v, log_alpha, beta, S0, o, S_T, B, T, H, dk, dv, chunk, dtype, 1, KDA_GATE_CHANNEL,
                           workspace, workspace_bytes, algo, stream);
}

kda_status_t kda_chunk_fwd(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                           const float* S0, void* o, float* S_T, int B, int T, int H, int dk, int dv, int chunk,
                           kda_dtype_t dtype, void* workspace, size_t workspace_bytes, void* stream) {
    return kda_chunk_fwd_ex(q, k, v, log_alpha, beta, S0, o, S_T, B, T, H, dk, dv, chunk, dtype, workspace,
                            workspace_bytes, KDA_ALGO_AUTO, stream);
}

kda_status_t kda_chunk_fwd_timeout_test(const void* q, const void* k, const void* v, const void* log_alpha,
                                       const void* beta, const float* S0, void* o, float* S_T, int B, int T, int H,
                                       int dk, int dv, int chunk, kda_dtype_t dtype, void* workspace,
                                       size_t workspace_bytes, long long wait_budget_cycles, void* stream) {
    if (wait_budget_cycles <= 0 || wait_budget_cycles > (1ll << 31)) return KDA_ERR_INVALID_ARG;
    kda::ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.S0 = S0; a.o = o; a.ST = S_T;
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv; a.chunk = chunk; a.bf16 = dtype == KDA_BF16;
    a.erase = 1;
    a.gate = KDA_GATE_CHANNEL;
    a.cu_seqlens = nullptr;
    a.workspace = workspace; a.workspace_bytes = workspace_bytes;
    a.test_withhold_first_load = 1;
    a.test_wait_budget = wait_budget_cycles;
    // Only the single-pass tensor-core kernel has the waits this exercises.
    if (T == 0) return KDA_ERR_INVALID_ARG;
    return run_chunk(a, dtype, KDA_ALGO_TC, stream);
}

kda_status_t kda_workspace_status(const void* workspace, size_t workspace_bytes, void* stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_CUDA;
    if (workspace == nullptr || workspace_bytes < sizeof(unsigned)) return KDA_OK;
    unsigned flag = 0;
    if (cudaMemcpy(&flag, workspace, sizeof(flag), cudaMemcpyDeviceToHost) != cudaSuccess) return KDA_ERR_CUDA;
    return flag ? KDA_ERR_TIMEOUT : KDA_OK;
}

kda_status_t kda_decode_step_v(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                               const float* S_in, float* S_out, void* o, int N, int H, int dk, int dv,
                               kda_dtype_t dtype, int erase, kda_gate_t gate, void* stream) {
    if (N < 0 || H < 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (erase != 0 && erase != 1) return KDA_ERR_INVALID_ARG;
    if (gate < KDA_GATE_CHANNEL || gate > KDA_GATE_NONE) return KDA_ERR_INVALID_ARG;
    if (!head_dims_ok(dk, dv)) return KDA_ERR_UNSUPPORTED;
    if ((long long)N * H * (dv / 32) > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    if ((long long)N * H == 0) return KDA_OK;
    const void* req[] = {q, k, v, beta, S_in, S_out, o};
    for (const void* p : req)
        if (p == nullptr || !aligned16(p)) return KDA_ERR_INVALID_ARG;
    if (gate != KDA_GATE_NONE && (log_alpha == nullptr || !aligned16(log_alpha))) return KDA_ERR_INVALID_ARG;
    const cudaError_t err = kda::launch_decode(q, k, v, log_alpha, beta, S_in, S_out, o, N, H, dk, dv,
                                               dtype == KDA_BF16, erase, (int)gate, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status_t kda_decode_step(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                             const float* S_in, float* S_out, void* o, int N, int H, int dk, int dv,
                             kda_dtype_t dtype, void* stream) {
    return kda_decode_step_v(q, k, v, log_alpha, beta, S_in, S_out, o, N, H, dk, dv, dtype, 1, KDA_GATE_CHANNEL,
                             stream);
}

size_t kda_chunk_bwd_workspace_size_ex(int B, int T, int H, int dk, int dv, kda_bwd_mode_t mode) {
    if (B < 0 || T < 0 || H < 0 || !head_dims_ok(dk, dv)) return 0;
    if (mode < KDA_BWD_AUTO || mode > KDA_BWD_LOW_MEMORY) return 0;
    return kda::chunk_bwd_workspace_bytes(B, T, H, dk, (int)mode);
}

size_t kda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv) {
    return kda_chunk_bwd_workspace_size_ex(B, T, H, dk, dv, KDA_BWD_AUTO);
}

kda_status_t kda_chunk_bwd(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                           const float* S0, const void* dO, const float* dS_T, void* d_q, void* d_k, void* d_v,
                           void* d_log_alpha, void* d_beta, float* d_S0, int B, int T, int H, int dk, int dv,
                           kda_dtype_t dtype, int erase, kda_gate_t gate, void* workspace, size_t workspace_bytes,
                           void* stream) {
    return kda_chunk_bwd_ex(q, k, v, log_alpha, beta, S0, dO, dS_T, d_q, d_k, d_v, d_log_alpha, d_beta, d_S0, B, T,
                            H, dk, dv, dtype, erase, gate, KDA_BWD_AUTO, workspace, workspace_bytes, stream);
}

kda_status_t kda_chunk_bwd_ex(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                              const float* S0, const void* dO, const float* dS_T, void* d_q, void* d_k, void* d_v,
                              void* d_log_alpha, void* d_beta, float* d_S0, int B, int T, int H, int dk, int dv,
                              kda_dtype_t dtype, int erase, kda_gate_t gate, kda_bwd_mode_t mode, void* workspace,
                              size_t workspace_bytes, void* stream) {
    if (B < 0 || T < 0 || H < 0) return KDA_ERR_INVALID_ARG;
    if (mode < KDA_BWD_AUTO || mode > KDA_BWD_LOW_MEMORY) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (!head_dims_ok(dk, dv)) return KDA_ERR_UNSUPPORTED;
    if ((long long)B * H > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    if (erase != 0 && erase != 1) return KDA_ERR_INVALID_ARG;
    if (gate < KDA_GATE_CHANNEL || gate > KDA_GATE_NONE) return KDA_ERR_INVALID_ARG;
    if ((long long)B * T * H > 0) {
        const void* req[] = {q, k, v, beta, dO, d_q, d_k, d_v, d_beta};
        for (const void* p : req)
            if (p == nullptr || !aligned16(p)) return KDA_ERR_INVALID_ARG;
        if (gate != KDA_GATE_NONE &&
            (log_alpha == nullptr || !aligned16(log_alpha) || d_log_alpha == nullptr || !aligned16(d_log_alpha)))
            return KDA_ERR_INVALID_ARG;
    }
    const float* opt[] = {S0, dS_T, d_S0};
    for (const float* p : opt)
        if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
    const size_t need = kda::chunk_bwd_workspace_bytes(B, T, H, dk, (int)mode);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
        return KDA_ERR_INVALID_ARG;
    if ((long long)B * H == 0) return KDA_OK;
    kda::BwdArgs a{};
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.dO = dO; a.S0 = S0; a.dST = dS_T;
    a.g_q = d_q; a.g_k = d_k; a.g_v = d_v; a.g_log_alpha = d_log_alpha; a.g_beta = d_beta; a.g_S0 = d_S0;
    a.B = B; a.T = T; a.H = H; a.d = dk; a.bf16 = dtype == KDA_BF16; a.erase = erase; a.gate = (int)gate;
    a.mode = (int)mode;
    a.workspace = workspace; a.workspace_bytes = workspace_bytes;
    const cudaError_t err = kda::launch_chunk_bwd(a, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // extern "C"
