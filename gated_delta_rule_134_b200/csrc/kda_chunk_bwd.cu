// Backward of the KDA chunkwise prefill: given dL/do and dL/dS_T, the
// gradients with respect to q, k, v, log_alpha, beta and S0.
//
// The pages give no backward pass ("Decoding Hybrid Attention Architectures",
// section 5, names training throughput as a goal only); what follows is the
// chain rule applied to the update of section 3.4,
//     S_t = S~_t + k_t delta_t^T,  S~_t = Diag(a_t) S_{t-1},
//     delta_t = b_t (v_t - S~_t^T k_t)          (additive write: b_t v_t)
// organised by chunks like the forward pass. With Lam_t = dL/dS_t the
// adjoint runs backwards as Lam_{t-1} = Diag(a_t)(I - b_t k_t k_t^T) Lam_t
// + q_{t-1} dO_{t-1}^T, and in a chunk of C tokens with entry state S,
// local prefix sums G_r of log a (per channel), Gamma_r = e^{G_r},
// E_rs = e^{G_r - G_s} (s <= r, exponent <= 0) and F = the adjoint flowing
// in from the chunk's end:
//   A0_rs = sum_c k_rc k_sc E_rs,c (s < r),  A = Diag(b) A0,  T = (I + A)^{-1}
//   P_rs  = sum_c q_rc k_sc E_rs,c (s <= r)
//   delta = T(b v) - T(b k Gamma) S,   R = v - (k Gamma) S - A0 delta
//   X = (k e^{G_last - G}) F + P^T dO,   d(delta) = T^T X,   dv = b d(delta)
//   db_r = d(delta)_r . R_r
//   dq_r  = Gamma_r (S dO_r) + sum_{s<=r} E_rs k_s (delta_s . dO_r)
//   dkr_r = -b_r [Gamma_r (S d(delta)_r) + sum_{s<r} E_rs k_s (delta_s . d(delta)_r)]
//   dkw_r = e^{G_last - G_r} (F delta_r) + sum_{s>=r} E_sr q_s (dO_s . delta_r)
//           - sum_{s>r} E_sr k_s (dv_s . delta_r),          dk = dkw + dkr
//   F <- Gamma_last F + (q Gamma)^T dO - (k Gamma)^T dv
// (without the erase term: A = 0, T = I, R = v, dkr = 0 and the dv terms of
// dkw and F drop). The decay gradient uses an identity of the update:
// raising log a_tau by eps equals moving e^{eps} onto the write-side key,
// e^{-eps} onto the read-side key and the query of every later token, so
//   dlog_a_tau = sum_{t >= tau} (q dq - k dkw + k dkr)_t + rowsum(dS_T * S_T),
// one reverse running sum per channel (a scalar gate sums it over channels).
//
// Design: one CTA per (batch, head), fp32 throughout, the state S and the
// adjoint F ([dk][dv], rows padded by one float against bank conflicts) in
// shared memory, chunks of 8 tokens with every decay factor an exact
// exponential of a non-positive exponent. A forward sweep stores the state
// every 8 chunks (64 tokens); the backward sweep recomputes the 8 entry
// states of each such block into a per-CTA ring in global memory (L2) and
// then walks the block in reverse.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int kBT = 512;                      // threads per CTA
constexpr int kBC = 8;                        // tokens per backward chunk
constexpr int kBlk = 8;                       // chunks per stored state
constexpr int kPairs = kBC * (kBC + 1) / 2;   // (r, s) pairs with s <= r

__host__ __device__ constexpr int pidx(int r, int s) { return r * (r + 1) / 2 + s; }

template <int D>
struct BwdLayout {  // offsets in floats
    static constexpr int LD = D + 1;
    static constexpr int S = 0;
    static constexpr int F = S + D * LD;
    static constexpr int Q = F + D * LD;
    static constexpr int K = Q + kBC * D;
    static constexpr int G = K + kBC * D;     // log a, then inclusive prefix sums
    static constexpr int GAM = G + kBC * D;   // e^{G}
    static constexpr int V = GAM + kBC * D;
    static constexpr int DO = V + kBC * D;
    static constexpr int DL = DO + kBC * D;   // U, then delta
    static constexpr int R = DL + kBC * D;    // W, then R, then S dO
    static constexpr int X = R + kBC * D;     // k e^G / k e^{G_last-G}, X, then F delta
    static constexpr int DD = X + kBC * D;    // d(delta)
    static constexpr int DG = DD + kBC * D;   // S d(delta), then q dq - k dkw + k dkr
    static constexpr int E = DG + kBC * D;    // [pair][D]: e^{G_r - G_s}
    static constexpr int RED = E + kPairs * D;  // [kBT / D groups][8][D] partial sums
    static constexpr int A0 = RED + kBT * kBC;
    static constexpr int P = A0 + 64;
    static constexpr int TM = P + 64;
    static constexpr int C1 = TM + 64;        // [r][s] delta_s . dO_r
    static constexpr int C2 = C1 + 64;        // [r][s] delta_s . d(delta)_r
    static constexpr int C3 = C2 + 64;        // [r][s] delta_r . dv_s
    static constexpr int BETA = C3 + 64;
    static constexpr int CARRY = BETA + kBC;  // running reverse sum of the decay gradient
    static constexpr int TOTAL = CARRY + D;
    static constexpr size_t BYTES = (size_t)TOTAL * sizeof(float);
};

__device__ __forceinline__ void pair_rs(int p, int& r, int& s) {
    r = 0;
    while (pidx(r + 1, 0) <= p) ++r;
    s = p - pidx(r, 0);
}

template <typename T, int D>
__global__ void __launch_bounds__(kBT, 1)
chunk_bwd_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                 const T* __restrict__ log_alpha, const T* __restrict__ beta, const float* __restrict__ S0,
                 const T* __restrict__ dO, const float* __restrict__ dST, T* __restrict__ dq, T* __restrict__ dk,
                 T* __restrict__ dv, T* __restrict__ dla, T* __restrict__ dbeta, float* __restrict__ dS0,
                 float* __restrict__ ckpt, float* __restrict__ ring, int Tlen, int H, int erase, int gate) {
    using L = BwdLayout<D>;
    constexpr int LD = L::LD;
    constexpr int NG = kBT / D;   // thread groups in the matrix-vector products
    constexpr int RW = D / NG;    // rows (or columns) per group
    extern __shared__ float sm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const size_t tok0 = (size_t)b * Tlen;
    const int NB = (Tlen + kBC - 1) / kBC;
    const int NBLK = (NB + kBlk - 1) / kBlk;
    constexpr size_t kMat = (size_t)D * D;
    float* ck = ckpt + (size_t)bh * NBLK * kMat;
    float* rg = ring + (size_t)bh * kBlk * kMat;
    float* sS = sm + L::S;
    float* sF = sm + L::F;

    auto load_mat = [&](float* dst, const float* src) {
        for (int e = tid; e < D * D; e += kBT) dst[(e / D) * LD + e % D] = src ? src[e] : 0.f;
    };
    auto store_mat = [&](const float* src, float* dst) {
        for (int e = tid; e < D * D; e += kBT) dst[e] = src[(e / D) * LD + e % D];
    };
    // out_v = sum_i x_v[i] M[i][.] (x from the left), 8 vectors; partials to RED
    auto left_partials = [&](const float* M, const float* x) {
        const int j = tid % D, g = tid / D;
        float acc[kBC];
#pragma unroll
        for (int u = 0; u < kBC; ++u) acc[u] = 0.f;
        for (int ii = 0; ii < RW; ++ii) {
            const int i = g * RW + ii;
            const float m = M[i * LD + j];
#pragma unroll
            for (int u = 0; u < kBC; ++u) acc[u] = fmaf(x[u * D + i], m, acc[u]);
        }
#pragma unroll
        for (int u = 0; u < kBC; ++u) sm[L::RED + (g * kBC + u) * D + j] = acc[u];
    };
    // out_v = M x_v (x from the right), 8 vectors; partials to RED
    auto right_partials = [&](const float* M, const float* x) {
        const int i = tid % D, g = tid / D;
        float acc[kBC];
#pragma unroll
        for (int u = 0; u < kBC; ++u) acc[u] = 0.f;
        for (int jj = 0; jj < RW; ++jj) {
            const int j = g * RW + jj;
            const float m = M[i * LD + j];
#pragma unroll
            for (int u = 0; u < kBC; ++u) acc[u] = fmaf(m, x[u * D + j], acc[u]);
        }
#pragma unroll
        for (int u = 0; u < kBC; ++u) sm[L::RED + (g * kBC + u) * D + i] = acc[u];
    };
    auto red_sum = [&](int u, int c) -> float {
        float s = 0.f;
#pragma unroll
        for (int g = 0; g < NG; ++g) s += sm[L::RED + (g * kBC + u) * D + c];
        return s;
    };

    // inputs of chunk n (rows past T are zero: identity steps)
    auto load_chunk = [&](int n, bool full) -> int {
        const int len = min(kBC, Tlen - n * kBC);
        for (int e = tid; e < kBC * D; e += kBT) {
            const int r = e / D, c = e % D;
            float qv = 0.f, kv = 0.f, gv = 0.f, vv = 0.f, ov = 0.f;
            if (r < len) {
                const size_t tok = (tok0 + (size_t)n * kBC + r) * H + h;
                kv = to_f32(k[tok * D + c]);
                vv = to_f32(v[tok * D + c]);
                gv = gate == 0 ? to_f32(log_alpha[tok * D + c]) : (gate == 1 ? to_f32(log_alpha[tok]) : 0.f);
                if (full) {
                    qv = to_f32(q[tok * D + c]);
                    ov = to_f32(dO[tok * D + c]);
                }
            }
            sm[L::Q + e] = qv;
            sm[L::K + e] = kv;
            sm[L::G + e] = gv;
            sm[L::V + e] = vv;
            sm[L::DO + e] = ov;
        }
        if (tid < kBC) sm[L::BETA + tid] = tid < len ? to_f32(beta[(tok0 + (size_t)n * kBC + tid) * H + h]) : 0.f;
        __syncthreads();
        return len;
    };
    // prefix sums, e^G, the pair table, A0 (and P), T
    auto prep = [&](bool want_p) {
        for (int c = tid; c < D; c += kBT) {
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < kBC; ++r) {
                acc += sm[L::G + r * D + c];
                sm[L::G + r * D + c] = acc;
                sm[L::GAM + r * D + c] = expf(acc);
            }
        }
        __syncthreads();
        for (int e = tid; e < kPairs * D; e += kBT) {
            const int p = e / D, c = e % D;
            int r, s;
            pair_rs(p, r, s);
            sm[L::E + e] = expf(sm[L::G + r * D + c] - sm[L::G + s * D + c]);
        }
        __syncthreads();
        for (int p = warp; p < kPairs; p += kBT / 32) {
            int r, s;
            pair_rs(p, r, s);
            float a = 0.f, pp = 0.f;
            for (int c = lane; c < D; c += 32) {
                const float ks = sm[L::K + s * D + c] * sm[L::E + p * D + c];
                a = fmaf(sm[L::K + r * D + c], ks, a);
                if (want_p) pp = fmaf(sm[L::Q + r * D + c], ks, pp);
            }
            a = warp_sum(a);
            pp = warp_sum(pp);
            if (lane == 0) {
                sm[L::A0 + r * kBC + s] = s < r ? a : 0.f;
                sm[L::P + r * kBC + s] = pp;
            }
        }
        __syncthreads();
        if (tid < kBC) {  // column j of T = (I + Diag(b) A0)^{-1}: unit lower triangular
            const int j = tid;
            for (int r = 0; r < kBC; ++r) sm[L::TM + r * kBC + j] = r == j ? 1.f : 0.f;
            if (erase)
                for (int r = j + 1; r < kBC; ++r) {
                    float acc = 0.f;
                    for (int s = j; s < r; ++s) acc = fmaf(sm[L::A0 + r * kBC + s], sm[L::TM + s * kBC + j], acc);
                    sm[L::TM + r * kBC + j] = -sm[L::BETA + r] * acc;
                }
        }
        __syncthreads();
    };
    // delta = T(b v) - T(b k e^G) S into DL (W staged in R)
    auto make_delta = [&]() {
        for (int e = tid; e < kBC * D; e += kBT) {
            const int r = e / D, c = e % D;
            float w = 0.f, u = 0.f;
            for (int s = 0; s <= r; ++s) {
                const float ts = sm[L::TM + r * kBC + s] * sm[L::BETA + s];
                w = fmaf(ts, sm[L::K + s * D + c] * sm[L::GAM + s * D + c], w);
                u = fmaf(ts, sm[L::V + s * D + c], u);
            }
            sm[L::R + e] = erase ? w : 0.f;
            sm[L::DL + e] = u;
        }
        __syncthreads();
        if (erase) {
            left_partials(sS, sm + L::R);
            __syncthreads();
            for (int e = tid; e < kBC * D; e += kBT) sm[L::DL + e] -= red_sum(e / D, e % D);
            __syncthreads();
        }
    };
    // one chunk forward: S <- Gamma_last S + (k e^{G_last - G})^T delta
    auto fwd_step = [&](int n) {
        load_chunk(n, false);
        prep(false);
        make_delta();
        for (int e = tid; e < kBC * D; e += kBT) {
            const int r = e / D, c = e % D;
            sm[L::X + e] = sm[L::K + e] * expf(sm[L::G + (kBC - 1) * D + c] - sm[L::G + r * D + c]);
        }
        __syncthreads();
        for (int e = tid; e < D * D; e += kBT) {
            const int i = e / D, j = e % D;
            float acc = sm[L::GAM + (kBC - 1) * D + i] * sS[i * LD + j];
#pragma unroll
            for (int r = 0; r < kBC; ++r) acc = fmaf(sm[L::X + r * D + i], sm[L::DL + r * D + j], acc);
            sS[i * LD + j] = acc;
        }
        __syncthreads();
    };

    auto bwd_step = [&](int n) {
        const int len = load_chunk(n, true);
        prep(true);
        make_delta();
        // R = v - (k e^G) S - A0 delta  (additive write: R = v)
        if (erase) {
            for (int e = tid; e < kBC * D; e += kBT) sm[L::X + e] = sm[L::K + e] * sm[L::GAM + e];
            __syncthreads();
            left_partials(sS, sm + L::X);
            __syncthreads();
            for (int e = tid; e < kBC * D; e += kBT) {
                const int r = e / D, c = e % D;
                float acc = sm[L::V + e] - red_sum(r, c);
                for (int s = 0; s < r; ++s) acc = fmaf(-sm[L::A0 + r * kBC + s], sm[L::DL + s * D + c], acc);
                sm[L::R + e] = acc;
            }
        } else {
            for (int e = tid; e < kBC * D; e += kBT) sm[L::R + e] = sm[L::V + e];
        }
        // X = (k e^{G_last - G}) F + P^T dO
        for (int e = tid; e < kBC * D; e += kBT) {
            const int r = e / D, c = e % D;
            sm[L::X + e] = sm[L::K + e] * expf(sm[L::G + (kBC - 1) * D + c] - sm[L::G + r * D + c]);
        }
        __syncthreads();
        left_partials(sF, sm + L::X);
        __syncthreads();
        for (int e = tid; e < kBC * D; e += kBT) {
            const int r = e / D, c = e % D;
            float acc = red_sum(r, c);
            for (int s = r; s < kBC; ++s) acc = fmaf(sm[L::P + s * kBC + r], sm[L::DO + s * D + c], acc);
            sm[L::X + e] = acc;
        }
        __syncthreads();
        // d(delta) = T^T X; dv = b d(delta)
        for (int e = tid; e < kBC * D; e += kBT) {
            const int r = e / D, c = e % D;
            float acc = 0.f;
            for (int s = r; s < kBC; ++s) acc = fmaf(sm[L::TM + s * kBC + r], sm[L::X + s * D + c], acc);
            sm[L::DD + e] = acc;
            if (r < len) dv[((tok0 + (size_t)n * kBC + r) * H + h) * D + c] = from_f32<T>(sm[L::BETA + r] * acc);
        }
        __syncthreads();
        // db_r = d(delta)_r . R_r (warps 0-7), and the three dot tables (all warps)
        if (warp < kBC) {
            const int r = warp;
            float acc = 0.f;
            for (int c = lane; c < D; c += 32) acc = fmaf(sm[L::DD + r * D + c], sm[L::R + r * D + c], acc);
            acc = warp_sum(acc);
            if (lane == 0 && r < len) dbeta[(tok0 + (size_t)n * kBC + r) * H + h] = from_f32<T>(acc);
        }
        for (int d = warp; d < 3 * kBC * kBC; d += kBT / 32) {
            const int tbl = d / (kBC * kBC), r = (d / kBC) % kBC, s = d % kBC;
            // C1: delta_s . dO_r;  C2: delta_s . d(delta)_r;  C3: delta_r . d(delta)_s (times b_s)
            const float* x = sm + L::DL + (tbl == 2 ? r : s) * D;
            const float* y = tbl == 0 ? sm + L::DO + r * D : sm + L::DD + (tbl == 1 ? r : s) * D;
            float acc = 0.f;
            for (int c = lane; c < D; c += 32) acc = fmaf(x[c], y[c], acc);
            acc = warp_sum(acc);
            if (lane == 0) {
                if (tbl == 0) sm[L::C1 + r * kBC + s] = acc;
                else if (tbl == 1) sm[L::C2 + r * kBC + s] = acc;
                else sm[L::C3 + r * kBC + s] = sm[L::BETA + s] * acc;  // delta_r . dv_s
            }
        }
        __syncthreads();
        // right products: S dO -> R, S d(delta) -> DG, F delta -> X
        right_partials(sS, sm + L::DO);
        __syncthreads();
        for (int e = tid; e < kBC * D; e += kBT) sm[L::R + e] = red_sum(e / D, e % D);
        __syncthreads();
        right_partials(sS, sm + L::DD);
        __syncthreads();
        for (int e = tid; e < kBC * D; e += kBT) sm[L::DG + e] = red_sum(e / D, e % D);
        __syncthreads();
        right_partials(sF, sm + L::DL);
        __syncthreads();
        for (int e = tid; e < kBC * D; e += kBT) sm[L::X + e] = red_sum(e / D, e % D);
        __syncthreads();
        // per (token, channel): dq, dk, and q dq - k dkw + k dkr
        for (int e = tid; e < kBC * D; e += kBT) {
            const int r = e / D, c = e % D;
            const float gam = sm[L::GAM + e], kr = sm[L::K + e], qr = sm[L::Q + e];
            float gq = gam * sm[L::R + e];
            for (int s = 0; s <= r; ++s)
                gq = fmaf(sm[L::E + pidx(r, s) * D + c] * sm[L::K + s * D + c], sm[L::C1 + r * kBC + s], gq);
            float gkr = 0.f;
            if (erase) {
                gkr = gam * sm[L::DG + e];
                for (int s = 0; s < r; ++s)
                    gkr = fmaf(sm[L::E + pidx(r, s) * D + c] * sm[L::K + s * D + c], sm[L::C2 + r * kBC + s], gkr);
                gkr *= -sm[L::BETA + r];
            }
            float gkw = expf(sm[L::G + (kBC - 1) * D + c] - sm[L::G + e]) * sm[L::X + e];
            for (int s = r; s < kBC; ++s) {
                const float es = sm[L::E + pidx(s, r) * D + c];
                gkw = fmaf(es * sm[L::Q + s * D + c], sm[L::C1 + s * kBC + r], gkw);
                if (erase && s > r) gkw = fmaf(-es * sm[L::K + s * D + c], sm[L::C3 + r * kBC + s], gkw);
            }
            if (r < len) {
                const size_t off = ((tok0 + (size_t)n * kBC + r) * H + h) * D + c;
                dq[off] = from_f32<T>(gq);
                dk[off] = from_f32<T>(gkw + gkr);
            }
            sm[L::DG + e] = qr * gq - kr * gkw + kr * gkr;
        }
        __syncthreads();
        // decay gradient: reverse running sum per channel
        if (gate != 2) {
            for (int c = tid; c < D; c += kBT) {
                float acc = sm[L::CARRY + c];
                for (int r = kBC - 1; r >= 0; --r) {
                    acc += sm[L::DG + r * D + c];
                    if (gate == 0) {
                        if (r < len) dla[((tok0 + (size_t)n * kBC + r) * H + h) * D + c] = from_f32<T>(acc);
                    } else {
                        sm[L::DG + r * D + c] = acc;
                    }
                }
                sm[L::CARRY + c] = acc;
            }
            if (gate == 1) {
                __syncthreads();
                if (warp < kBC) {
                    const int r = warp;
                    float acc = 0.f;
                    for (int c = lane; c < D; c += 32) acc += sm[L::DG + r * D + c];
                    acc = warp_sum(acc);
                    if (lane == 0 && r < len) dla[(tok0 + (size_t)n * kBC + r) * H + h] = from_f32<T>(acc);
                }
            }
        }
        // F <- Gamma_last F + (q e^G)^T dO - (k e^G)^T dv
        for (int e = tid; e < D * D; e += kBT) {
            const int i = e / D, j = e % D;
            float acc = sm[L::GAM + (kBC - 1) * D + i] * sF[i * LD + j];
#pragma unroll
            for (int r = 0; r < kBC; ++r) {
                const float gr = sm[L::GAM + r * D + i];
                acc = fmaf(sm[L::Q + r * D + i] * gr, sm[L::DO + r * D + j], acc);
                if (erase) acc = fmaf(-sm[L::K + r * D + i] * gr, sm[L::BETA + r] * sm[L::DD + r * D + j], acc);
            }
            sF[i * LD + j] = acc;
        }
        __syncthreads();
    };

    // ---- forward sweep: the state every kBlk chunks, and S_T
    load_mat(sS, S0 ? S0 + (size_t)bh * kMat : nullptr);
    __syncthreads();
    for (int n = 0; n < NB; ++n) {
        if (n % kBlk == 0) {
            store_mat(sS, ck + (size_t)(n / kBlk) * kMat);
            __syncthreads();
        }
        fwd_step(n);
    }
    // ---- F = dS_T; carry = rowsum(dS_T * S_T)
    const float* dst_h = dST ? dST + (size_t)bh * kMat : nullptr;
    load_mat(sF, dst_h);
    __syncthreads();
    for (int c = warp; c < D; c += kBT / 32) {
        float acc = 0.f;
        for (int j = lane; j < D; j += 32) acc = fmaf(sF[c * LD + j], sS[c * LD + j], acc);
        acc = warp_sum(acc);
        if (lane == 0) sm[L::CARRY + c] = acc;
    }
    __syncthreads();
    // ---- backward sweep, one block of kBlk chunks at a time
    for (int blk = NBLK - 1; blk >= 0; --blk) {
        const int n0 = blk * kBlk, n1 = min(n0 + kBlk, NB);
        load_mat(sS, ck + (size_t)blk * kMat);
        __syncthreads();
        for (int n = n0; n < n1; ++n) {
            store_mat(sS, rg + (size_t)(n - n0) * kMat);
            __syncthreads();
            if (n + 1 < n1) fwd_step(n);
        }
        for (int n = n1 - 1; n >= n0; --n) {
            load_mat(sS, rg + (size_t)(n - n0) * kMat);
            __syncthreads();
            bwd_step(n);
        }
    }
    if (dS0) store_mat(sF, dS0 + (size_t)bh * kMat);
}

template <typename T, int D>
cudaError_t launch_bwd_t(const BwdArgs& a, cudaStream_t stream) {
    using L = BwdLayout<D>;
    auto kern = chunk_bwd_kernel<T, D>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::BYTES);
    if (err != cudaSuccess) return err;
    const size_t NBLK = ((size_t)(a.T + kBC - 1) / kBC + kBlk - 1) / kBlk;
    float* ckpt = static_cast<float*>(a.workspace);
    float* ring = ckpt + (size_t)a.B * a.H * NBLK * D * D;
    kern<<<(unsigned)(a.B * a.H), kBT, L::BYTES, stream>>>(
        (const T*)a.q, (const T*)a.k, (const T*)a.v, (const T*)a.log_alpha, (const T*)a.beta, a.S0, (const T*)a.dO,
        a.dST, (T*)a.g_q, (T*)a.g_k, (T*)a.g_v, (T*)a.g_log_alpha, (T*)a.g_beta, a.g_S0, ckpt, ring, a.T, a.H,
        a.erase, a.gate);
    return cudaGetLastError();
}

}  // namespace

size_t chunk_bwd_workspace_bytes(int B, int T, int H, int d) {
    const size_t NBLK = ((size_t)(T + kBC - 1) / kBC + kBlk - 1) / kBlk;
    return (size_t)B * H * (NBLK + kBlk) * d * d * sizeof(float);
}

cudaError_t launch_chunk_bwd(const BwdArgs& a, cudaStream_t stream) {
    if (a.bf16) return a.d == 64 ? launch_bwd_t<__nv_bfloat16, 64>(a, stream) : launch_bwd_t<__nv_bfloat16, 128>(a, stream);
    return a.d == 64 ? launch_bwd_t<float, 64>(a, stream) : launch_bwd_t<float, 128>(a, stream);
}

}  // namespace kda
