// KDA chunkwise prefill, fp32 SIMT kernel (any dtype, dk = dv in {64,128},
// chunk in {16,32,64}). It is the exact-arithmetic path: fp32 everywhere,
// per-pair decay exponentials (exponent always <= 0), no tensor cores. It
// serves fp32 inputs, shapes the tensor-core kernel does not cover, and as a
// second GPU formulation for tests.
//
// Chunkwise form ("Decoding Hybrid Attention Architectures", section 4;
// "Technical Analysis ... Novel Hybrid Linear Attention", sections 3.1-3.2),
// with the decay placement derived from the recurrence. In a chunk of C tokens
// with local cumulative log-decay G_r = sum_{s<=r} log_alpha_s (per key
// channel) and chunk-start state S:
//   A_rs = beta_r sum_c k_rc k_sc e^{G_rc - G_sc}   (s < r)   strictly lower
//   P_rs = sum_c q_rc k_sc e^{G_rc - G_sc}          (s <= r)  lower incl. diag
//   T = (I + A)^{-1}  (forward substitution)
//   W = T (beta k e^{G}),  U = T (beta v)   -- the "precomputed" U and W
//   D = U - W S                              -- per-token corrected write
//   O = (q e^{G}) S + P D
//   S <- Diag(e^{G_last}) S + (k e^{G_last - G})^T D
// One CTA owns one (batch, head) and a 32-wide slice of the value channels;
// the slice's state stays in shared memory across all chunks.
// Variants (variant table of section 3.4): the gate switch selects a
// per-channel, per-token-scalar or absent log_alpha; without the erase term
// (additive write) A = 0 and W = 0, so T = I and D = beta v.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

constexpr int kSimtThreads = 256;
constexpr int kSimtDVT = 32;

template <int DK, int C>
constexpr size_t simt_smem_floats() {
    return 4 * C * DK + 2 * C * C + 3 * C * kSimtDVT + DK * kSimtDVT + C + DK;
}

template <typename T, int DK, int C>
__global__ void __launch_bounds__(kSimtThreads)
chunk_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const T* __restrict__ log_alpha, const T* __restrict__ beta, const float* S0,
                  T* __restrict__ o, float* ST, int Tlen, int H, int dv, int erase, int gate,
                  const int* __restrict__ cu_seqlens) {
    constexpr int NT = kSimtThreads, DVT = kSimtDVT;
    extern __shared__ float smem[];
    float* sQ = smem;             // q, then q e^G
    float* sK = sQ + C * DK;      // k, then k e^{G_last - G}
    float* sG = sK + C * DK;      // log_alpha, then G, then W
    float* sX = sG + C * DK;      // beta k e^G
    float* sA = sX + C * DK;      // A, then strictly-lower part of T
    float* sP = sA + C * C;
    float* sV = sP + C * C;       // v slice
    float* sU = sV + C * DVT;
    float* sD = sU + C * DVT;
    float* sS = sD + C * DVT;     // state slice [DK][DVT]
    float* sB = sS + DK * DVT;    // beta
    float* sGam = sB + C;         // e^{G_last}

    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int j0 = blockIdx.y * DVT;
    const int tid = threadIdx.x;
    // this sequence's tokens: [tok0, tok0 + len) of the token-major layout
    // (dense: sequence b of a [B, T] batch; packed: offsets clamped into [0, T])
    size_t tok0;
    int len_seq;
    if (cu_seqlens) {
        const int s0 = min(max(cu_seqlens[b], 0), Tlen), s1 = min(max(cu_seqlens[b + 1], s0), Tlen);
        tok0 = (size_t)s0;
        len_seq = s1 - s0;
    } else {
        tok0 = (size_t)b * Tlen;
        len_seq = Tlen;
    }

    for (int e = tid; e < DK * DVT; e += NT) {
        const int c = e / DVT, j = e % DVT;
        sS[e] = S0 ? S0[((size_t)bh * DK + c) * dv + j0 + j] : 0.f;
    }

    const int NC = (len_seq + C - 1) / C;
    for (int n = 0; n < NC; ++n) {
        const int t0 = n * C;
        const int len = min(C, len_seq - t0);
        __syncthreads();
        for (int e = tid; e < C * DK; e += NT) {
            const int r = e / DK, c = e % DK;
            float qv = 0.f, kv = 0.f, lv = 0.f;
            if (r < len) {
                const size_t tok = (tok0 + t0 + r) * H + h;
                const size_t off = tok * DK + c;
                qv = to_f32(q[off]);
                kv = to_f32(k[off]);
                lv = gate == 0 ? to_f32(log_alpha[off]) : (gate == 1 ? to_f32(log_alpha[tok]) : 0.f);
            }
            sQ[e] = qv;
            sK[e] = kv;
            sG[e] = lv;
        }
        for (int e = tid; e < C * DVT; e += NT) {
            const int r = e / DVT, j = e % DVT;
            sV[e] = r < len ? to_f32(v[((tok0 + t0 + r) * H + h) * dv + j0 + j]) : 0.f;
        }
        for (int r = tid; r < C; r += NT) sB[r] = r < len ? to_f32(beta[(tok0 + t0 + r) * H + h]) : 0.f;
        __syncthreads();

        // G: inclusive prefix sum over the chunk's tokens, per key channel.
        for (int c = tid; c < DK; c += NT) {
            float acc = 0.f;
            for (int r = 0; r < C; ++r) {
                acc += sG[r * DK + c];
                sG[r * DK + c] = acc;
            }
            sGam[c] = expf(acc);
        }
        __syncthreads();

        // A and P over the lower triangle, one (r, s) pair per thread; the
        // channel loop is rotated by the pair index so a warp's lanes hit
        // distinct banks.
        for (int p = tid; p < C * (C + 1) / 2; p += NT) {
            int r = (int)((sqrtf(8.f * (float)p + 1.f) - 1.f) * 0.5f);
            while ((r + 1) * (r + 2) / 2 <= p) ++r;
            while (r * (r + 1) / 2 > p) --r;
            const int s = p - r * (r + 1) / 2;
            float a = 0.f, pp = 0.f;
            for (int i = 0; i < DK; ++i) {
                const int c = (i + p) & (DK - 1);
                const float ks = sK[s * DK + c] * expf(sG[r * DK + c] - sG[s * DK + c]);
                a = fmaf(sK[r * DK + c], ks, a);
                pp = fmaf(sQ[r * DK + c], ks, pp);
            }
            sA[r * C + s] = (s < r && erase) ? sB[r] * a : 0.f;
            sP[r * C + s] = pp;
            if (s < r) {
                sA[s * C + r] = 0.f;
                sP[s * C + r] = 0.f;
            }
        }
        __syncthreads();

        // T = (I + A)^{-1} by forward substitution, row by row, in place
        // (strictly lower part; the unit diagonal is implicit):
        //   T_rj = -A_rj - sum_{j<s<r} A_rs T_sj.
        for (int r = 1; r < C; ++r) {
            float tv = 0.f;
            if (tid < r) {
                tv = -sA[r * C + tid];
                for (int s = tid + 1; s < r; ++s) tv = fmaf(-sA[r * C + s], sA[s * C + tid], tv);
            }
            __syncthreads();
            if (tid < r) sA[r * C + tid] = tv;
            __syncthreads();
        }

        for (int e = tid; e < C * DK; e += NT) {
            const int r = e / DK, c = e % DK;
            const float g = sG[e], eg = expf(g), kv = sK[e];
            sX[e] = erase ? sB[r] * kv * eg : 0.f;  // W = 0 without the erase term
            sQ[e] *= eg;
            sK[e] = kv * expf(sG[(C - 1) * DK + c] - g);
        }
        __syncthreads();

        // W = T X (into sG), U = T (beta v)
        for (int e = tid; e < C * DK; e += NT) {
            const int r = e / DK, c = e % DK;
            float acc = sX[e];
            for (int s = 0; s < r; ++s) acc = fmaf(sA[r * C + s], sX[s * DK + c], acc);
            sG[e] = acc;
        }
        for (int e = tid; e < C * DVT; e += NT) {
            const int r = e / DVT, j = e % DVT;
            float acc = sB[r] * sV[e];
            for (int s = 0; s < r; ++s) acc = fmaf(sA[r * C + s], sB[s] * sV[s * DVT + j], acc);
            sU[e] = acc;
        }
        __syncthreads();

        // D = U - W S
        for (int e = tid; e < C * DVT; e += NT) {
            const int r = e / DVT, j = e % DVT;
            float acc = sU[e];
            for (int c = 0; c < DK; ++c) acc = fmaf(-sG[r * DK + c], sS[c * DVT + j], acc);
            sD[e] = acc;
        }
        __syncthreads();

        // O = (q e^G) S + P D
        for (int e = tid; e < C * DVT; e += NT) {
            const int r = e / DVT, j = e % DVT;
            float acc = 0.f;
            for (int c = 0; c < DK; ++c) acc = fmaf(sQ[r * DK + c], sS[c * DVT + j], acc);
            for (int s = 0; s <= r; ++s) acc = fmaf(sP[r * C + s], sD[s * DVT + j], acc);
            if (r < len) o[((tok0 + t0 + r) * H + h) * dv + j0 + j] = from_f32<T>(acc);
        }
        __syncthreads();

        // S <- Diag(gamma) S + Ktilde^T D
        for (int e = tid; e < DK * DVT; e += NT) {
            const int c = e / DVT, j = e % DVT;
            float acc = sGam[c] * sS[e];
            for (int r = 0; r < C; ++r) acc = fmaf(sK[r * DK + c], sD[r * DVT + j], acc);
            sS[e] = acc;
        }
    }
    __syncthreads();
    if (ST) {
        for (int e = tid; e < DK * DVT; e += NT) {
            const int c = e / DVT, j = e % DVT;
            ST[((size_t)bh * DK + c) * dv + j0 + j] = sS[e];
        }
    }
}

template <typename T, int DK, int C>
static cudaError_t launch_simt_t(const ChunkArgs& a, cudaStream_t stream) {
    constexpr size_t smem = simt_smem_floats<DK, C>() * sizeof(float);
    auto kern = chunk_simt_kernel<T, DK, C>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    dim3 grid((unsigned)(a.B * a.H), (unsigned)(a.dv / kSimtDVT));
    kern<<<grid, kSimtThreads, smem, stream>>>((const T*)a.q, (const T*)a.k, (const T*)a.v, (const T*)a.log_alpha,
                                               (const T*)a.beta, a.S0, (T*)a.o, a.ST, a.T, a.H, a.dv, a.erase,
                                               a.gate, a.cu_seqlens);
    return cudaGetLastError();
}

template <typename T, int DK>
static cudaError_t launch_simt_dk(const ChunkArgs& a, cudaStream_t s) {
    switch (a.chunk) {
        case 16: return launch_simt_t<T, DK, 16>(a, s);
        case 32: return launch_simt_t<T, DK, 32>(a, s);
        default: return launch_simt_t<T, DK, 64>(a, s);
    }
}

cudaError_t launch_chunk_simt(const ChunkArgs& a, cudaStream_t stream) {
    if (a.bf16) return a.dk == 64 ? launch_simt_dk<__nv_bfloat16, 64>(a, stream)
                                  : launch_simt_dk<__nv_bfloat16, 128>(a, stream);
    return a.dk == 64 ? launch_simt_dk<float, 64>(a, stream) : launch_simt_dk<float, 128>(a, stream);
}

}  // namespace kda
