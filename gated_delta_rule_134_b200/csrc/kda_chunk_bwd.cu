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
// Design: one CTA per (batch, head), the state S and the adjoint F
// ([dk][dv] fp32, rows padded by 4 floats) in shared memory, chunks of 8
// tokens with every decay factor an exact exponential of a non-positive
// exponent. The six [8 x d] x [d x d] products per chunk run on warp-level
// tensor-core MMAs (m16n8k8) with each fp32 operand split into a tf32 high
// part and a tf32 remainder: hi*hi + hi*lo + lo*hi keeps the product at about
// fp32 accuracy. A forward sweep keeps every chunk's entry state and delta
// in the workspace (up to 16 GB of it), and the backward sweep walks the
// chunks in reverse from there. Beyond that size the forward sweep keeps the
// state every 8 chunks (64 tokens), and the backward sweep recomputes the 8
// entry states and deltas of each such block into a per-CTA ring in global
// memory, then walks the block in reverse.
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
    static constexpr int LD = D + 4;          // row stride of S and F
    static constexpr int TD = D + 4;          // row stride of the [8][D] tiles
    static constexpr int TILE = kBC * TD;
    static constexpr int S = 0;
    static constexpr int F = S + D * LD;
    static constexpr int Q = F + D * LD;
    static constexpr int K = Q + TILE;
    static constexpr int G = K + TILE;        // log a, then inclusive prefix sums
    static constexpr int GAM = G + TILE;      // e^{G}
    static constexpr int V = GAM + TILE;
    static constexpr int DO = V + TILE;
    static constexpr int DL = DO + TILE;      // U, then delta
    static constexpr int R = DL + TILE;       // W, then R, then S dO
    static constexpr int X = R + TILE;        // k e^G / k e^{G_last-G}, X, then F delta
    static constexpr int DD = X + TILE;       // d(delta)
    static constexpr int DG = DD + TILE;      // S d(delta), then q dq - k dkw + k dkr
    static constexpr int E = DG + TILE;       // [pair][D]: e^{G_r - G_s}
    static constexpr int RED = E + kPairs * D;  // [k-splits][8][D] partial sums
    static constexpr int NKS = 256 / D;         // k-splits of a product over 16 warps
    static constexpr int A0 = RED + NKS * kBC * D;
    static constexpr int P = A0 + 64;
    static constexpr int TM = P + 64;
    static constexpr int C1 = TM + 64;        // [r][s] delta_s . dO_r
    static constexpr int C2 = C1 + 64;        // [r][s] delta_s . d(delta)_r
    static constexpr int C3 = C2 + 64;        // [r][s] delta_r . dv_s
    static constexpr int BETA = C3 + 64;
    static constexpr int CARRY = BETA + kBC;  // running reverse sum of the decay gradient
    static constexpr int TOTAL = CARRY + D;
    static constexpr size_t BYTES = (size_t)TOTAL * sizeof(float);
    static_assert(BYTES <= 232448, "shared memory budget");
};

__device__ __forceinline__ void pair_rs(int p, int& r, int& s) {
    r = 0;
    while (pidx(r + 1, 0) <= p) ++r;
    s = p - pidx(r, 0);
}

// fp32 -> (tf32 high part, tf32 remainder)
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(x));
    const float rem = x - __uint_as_float(hi);
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(lo) : "f"(rem));
}

__device__ __forceinline__ void mma_16x8x8(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// One 16 x 8 x 8 step at fp32 accuracy: A given by its four fp32 fragment
// values, B by two.
__device__ __forceinline__ void mma3_step(float (&d)[4], const float (&af)[4], float b0f, float b1f) {
    uint32_t ah[4], al[4], bh0, bl0, bh1, bl1;
#pragma unroll
    for (int e = 0; e < 4; ++e) split_tf32(af[e], ah[e], al[e]);
    split_tf32(b0f, bh0, bl0);
    split_tf32(b1f, bh1, bl1);
    mma_16x8x8(d, al, bh0, bh1);
    mma_16x8x8(d, ah, bl0, bl1);
    mma_16x8x8(d, ah, bh0, bh1);
}

template <typename T, int D>
__global__ void __launch_bounds__(kBT, 1)
chunk_bwd_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                 const T* __restrict__ log_alpha, const T* __restrict__ beta, const float* __restrict__ S0,
                 const T* __restrict__ dO, const float* __restrict__ dST, T* __restrict__ dq, T* __restrict__ dk,
                 T* __restrict__ dv, T* __restrict__ dla, T* __restrict__ dbeta, float* __restrict__ dS0,
                 float* __restrict__ ckpt, float* __restrict__ ring, int Tlen, int H, int erase, int gate,
                 int store_all) {
    using L = BwdLayout<D>;
    constexpr int LD = L::LD, TD = L::TD, NKS = L::NKS;
    constexpr int MT = D / 16;              // 16-row tiles of a product's output
    constexpr int KSTEPS = D / 8 / NKS;     // 8-deep k steps per warp
    extern __shared__ float sm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g8 = lane >> 2, t4 = lane & 3;  // mma fragment coordinates
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const size_t tok0 = (size_t)b * Tlen;
    const int NB = (Tlen + kBC - 1) / kBC;
    const int NBLK = (NB + kBlk - 1) / kBlk;
    constexpr size_t kMat = (size_t)D * D;
    constexpr size_t kRing = kMat + (size_t)kBC * D;  // ring slot: entry state, then delta
    float* ck = ckpt + (size_t)bh * NBLK * kMat;
    float* rg = ring + (size_t)bh * kBlk * kRing;
    float* sS = sm + L::S;
    float* sF = sm + L::F;
    auto tl = [&](int base, int r, int c) -> float& { return sm[base + r * TD + c]; };

    auto load_mat = [&](float* dst, const float* src) {
        for (int e = tid; e < D * D; e += kBT) dst[(e / D) * LD + e % D] = src ? src[e] : 0.f;
    };
    auto store_mat = [&](const float* src, float* dst) {
        for (int e = tid; e < D * D; e += kBT) dst[e] = src[(e / D) * LD + e % D];
    };
    // out_u[j] = sum_i x_u[i] M[i][j]  (x from the left), as out^T = M^T x^T:
    // m = j, n = u, k = i. Warp w: output rows 16 (w % MT).., k split w / MT.
    auto left_partials = [&](const float* M, int xb) {
        const int j0 = 16 * (warp % MT), ks = warp / MT;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
        for (int st = 0; st < KSTEPS; ++st) {
            const int i0 = 8 * (ks * KSTEPS + st);
            const float af[4] = {M[(i0 + t4) * LD + j0 + g8], M[(i0 + t4) * LD + j0 + g8 + 8],
                                 M[(i0 + t4 + 4) * LD + j0 + g8], M[(i0 + t4 + 4) * LD + j0 + g8 + 8]};
            mma3_step(d, af, sm[xb + g8 * TD + i0 + t4], sm[xb + g8 * TD + i0 + t4 + 4]);
        }
        float* red = sm + L::RED + ks * kBC * D;
        red[(2 * t4) * D + j0 + g8] = d[0];
        red[(2 * t4 + 1) * D + j0 + g8] = d[1];
        red[(2 * t4) * D + j0 + g8 + 8] = d[2];
        red[(2 * t4 + 1) * D + j0 + g8 + 8] = d[3];
    };
    // out_u[i] = sum_j M[i][j] x_u[j]  (x from the right): m = i, n = u, k = j
    auto right_partials = [&](const float* M, int xb) {
        const int i0 = 16 * (warp % MT), ks = warp / MT;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
        for (int st = 0; st < KSTEPS; ++st) {
            const int j0 = 8 * (ks * KSTEPS + st);
            const float af[4] = {M[(i0 + g8) * LD + j0 + t4], M[(i0 + g8 + 8) * LD + j0 + t4],
                                 M[(i0 + g8) * LD + j0 + t4 + 4], M[(i0 + g8 + 8) * LD + j0 + t4 + 4]};
            mma3_step(d, af, sm[xb + g8 * TD + j0 + t4], sm[xb + g8 * TD + j0 + t4 + 4]);
        }
        float* red = sm + L::RED + ks * kBC * D;
        red[(2 * t4) * D + i0 + g8] = d[0];
        red[(2 * t4 + 1) * D + i0 + g8] = d[1];
        red[(2 * t4) * D + i0 + g8 + 8] = d[2];
        red[(2 * t4 + 1) * D + i0 + g8 + 8] = d[3];
    };
    // M[i][j] = rowscale[i] M[i][j] + sum_r a_r[i] b_r[j] over one or two 8-deep
    // k steps: (a0, b0) with sign +1 and, if two, (a1, b1) with sign sgn1. a_r[i]
    // is tile(a, r, i) times tile(am, r, i) when am >= 0; b_r[j] is tile(b, r, j)
    // times beta_r when bb is set. Warp w owns the 16 x 8 output tiles w, w+16, ...
    auto rank_update = [&](float* M, int rs, int a0b, int am0, int b0b, bool two, int a1b, int am1, int b1b,
                           float sgn1, bool bb1) {
        for (int tile = warp; tile < (D / 16) * (D / 8); tile += kBT / 32) {
            const int i0 = 16 * (tile / (D / 8)), j0 = 8 * (tile % (D / 8));
            float d[4];
            const float sc0 = tl(rs, kBC - 1, i0 + g8), sc1 = tl(rs, kBC - 1, i0 + g8 + 8);
            d[0] = sc0 * M[(i0 + g8) * LD + j0 + 2 * t4];
            d[1] = sc0 * M[(i0 + g8) * LD + j0 + 2 * t4 + 1];
            d[2] = sc1 * M[(i0 + g8 + 8) * LD + j0 + 2 * t4];
            d[3] = sc1 * M[(i0 + g8 + 8) * LD + j0 + 2 * t4 + 1];
            auto av = [&](int ab, int am, int r, int i) { return am >= 0 ? tl(ab, r, i) * tl(am, r, i) : tl(ab, r, i); };
            {
                const float af[4] = {av(a0b, am0, t4, i0 + g8), av(a0b, am0, t4, i0 + g8 + 8),
                                     av(a0b, am0, t4 + 4, i0 + g8), av(a0b, am0, t4 + 4, i0 + g8 + 8)};
                mma3_step(d, af, tl(b0b, t4, j0 + g8), tl(b0b, t4 + 4, j0 + g8));
            }
            if (two) {
                const float af[4] = {sgn1 * av(a1b, am1, t4, i0 + g8), sgn1 * av(a1b, am1, t4, i0 + g8 + 8),
                                     sgn1 * av(a1b, am1, t4 + 4, i0 + g8), sgn1 * av(a1b, am1, t4 + 4, i0 + g8 + 8)};
                const float bf0 = tl(b1b, t4, j0 + g8) * (bb1 ? sm[L::BETA + t4] : 1.f);
                const float bf1 = tl(b1b, t4 + 4, j0 + g8) * (bb1 ? sm[L::BETA + t4 + 4] : 1.f);
                mma3_step(d, af, bf0, bf1);
            }
            M[(i0 + g8) * LD + j0 + 2 * t4] = d[0];
            M[(i0 + g8) * LD + j0 + 2 * t4 + 1] = d[1];
            M[(i0 + g8 + 8) * LD + j0 + 2 * t4] = d[2];
            M[(i0 + g8 + 8) * LD + j0 + 2 * t4 + 1] = d[3];
        }
    };
    auto red_sum = [&](int u, int c) -> float {
        float s = 0.f;
#pragma unroll
        for (int g = 0; g < NKS; ++g) s += sm[L::RED + (g * kBC + u) * D + c];
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
            tl(L::Q, r, c) = qv;
            tl(L::K, r, c) = kv;
            tl(L::G, r, c) = gv;
            tl(L::V, r, c) = vv;
            tl(L::DO, r, c) = ov;
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
                acc += tl(L::G, r, c);
                tl(L::G, r, c) = acc;
                tl(L::GAM, r, c) = expf(acc);
            }
        }
        __syncthreads();
        for (int e = tid; e < kPairs * D; e += kBT) {
            const int p = e / D, c = e % D;
            int r, s;
            pair_rs(p, r, s);
            sm[L::E + e] = expf(tl(L::G, r, c) - tl(L::G, s, c));
        }
        __syncthreads();
        for (int p = warp; p < kPairs; p += kBT / 32) {
            int r, s;
            pair_rs(p, r, s);
            float a = 0.f, pp = 0.f;
            for (int c = lane; c < D; c += 32) {
                const float ks = tl(L::K, s, c) * sm[L::E + p * D + c];
                a = fmaf(tl(L::K, r, c), ks, a);
                if (want_p) pp = fmaf(tl(L::Q, r, c), ks, pp);
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
                w = fmaf(ts, tl(L::K, s, c) * tl(L::GAM, s, c), w);
                u = fmaf(ts, tl(L::V, s, c), u);
            }
            tl(L::R, r, c) = erase ? w : 0.f;
            tl(L::DL, r, c) = u;
        }
        __syncthreads();
        if (erase) {
            left_partials(sS, L::R);
            __syncthreads();
            for (int e = tid; e < kBC * D; e += kBT) tl(L::DL, e / D, e % D) -= red_sum(e / D, e % D);
            __syncthreads();
        }
    };
    // S <- Gamma_last S + (k e^{G_last - G})^T delta
    auto state_update = [&]() {
        for (int e = tid; e < kBC * D; e += kBT) {
            const int r = e / D, c = e % D;
            tl(L::X, r, c) = tl(L::K, r, c) * expf(tl(L::G, kBC - 1, c) - tl(L::G, r, c));
        }
        __syncthreads();
        rank_update(sS, L::GAM, L::X, -1, L::DL, false, 0, -1, 0, 0.f, false);
        __syncthreads();
    };
    // one chunk forward; its delta also goes to dslot when given, and the state
    // update is skipped when the next entry state is not needed
    auto fwd_step = [&](int n, float* dslot, bool update) {
        load_chunk(n, false);
        prep(false);
        make_delta();
        if (dslot)
            for (int e = tid; e < kBC * D; e += kBT) dslot[e] = tl(L::DL, e / D, e % D);
        if (update) state_update();
        __syncthreads();
    };

    auto bwd_step = [&](int n, const float* delta_g) {
        const int len = load_chunk(n, true);
        prep(true);
        for (int e = tid; e < kBC * D; e += kBT) tl(L::DL, e / D, e % D) = delta_g[e];  // delta of the recompute
        // R = v - (k e^G) S - A0 delta  (additive write: R = v)
        for (int e = tid; e < kBC * D; e += kBT) {
            const int r = e / D, c = e % D;
            tl(L::X, r, c) = tl(L::K, r, c) * tl(L::GAM, r, c);
        }
        __syncthreads();
        if (erase) {
            left_partials(sS, L::X);
            __syncthreads();
            for (int e = tid; e < kBC * D; e += kBT) {
                const int r = e / D, c = e % D;
                float acc = tl(L::V, r, c) - red_sum(r, c);
                for (int s = 0; s < r; ++s) acc = fmaf(-sm[L::A0 + r * kBC + s], tl(L::DL, s, c), acc);
                tl(L::R, r, c) = acc;
            }
        } else {
            for (int e = tid; e < kBC * D; e += kBT) tl(L::R, e / D, e % D) = tl(L::V, e / D, e % D);
        }
        __syncthreads();
        // X = (k e^{G_last - G}) F + P^T dO
        for (int e = tid; e < kBC * D; e += kBT) {
            const int r = e / D, c = e % D;
            tl(L::X, r, c) = tl(L::K, r, c) * expf(tl(L::G, kBC - 1, c) - tl(L::G, r, c));
        }
        __syncthreads();
        left_partials(sF, L::X);
        __syncthreads();
        for (int e = tid; e < kBC * D; e += kBT) {
            const int r = e / D, c = e % D;
            float acc = red_sum(r, c);
            for (int s = r; s < kBC; ++s) acc = fmaf(sm[L::P + s * kBC + r], tl(L::DO, s, c), acc);
            tl(L::X, r, c) = acc;
        }
        __syncthreads();
        // d(delta) = T^T X; dv = b d(delta)
        for (int e = tid; e < kBC * D; e += kBT) {
            const int r = e / D, c = e % D;
            float acc = 0.f;
            for (int s = r; s < kBC; ++s) acc = fmaf(sm[L::TM + s * kBC + r], tl(L::X, s, c), acc);
            tl(L::DD, r, c) = acc;
            if (r < len) dv[((tok0 + (size_t)n * kBC + r) * H + h) * D + c] = from_f32<T>(sm[L::BETA + r] * acc);
        }
        __syncthreads();
        // db_r = d(delta)_r . R_r (warps 0-7), and the three dot tables (all warps)
        if (warp < kBC) {
            const int r = warp;
            float acc = 0.f;
            for (int c = lane; c < D; c += 32) acc = fmaf(tl(L::DD, r, c), tl(L::R, r, c), acc);
            acc = warp_sum(acc);
            if (lane == 0 && r < len) dbeta[(tok0 + (size_t)n * kBC + r) * H + h] = from_f32<T>(acc);
        }
        for (int dd = warp; dd < 3 * kBC * kBC; dd += kBT / 32) {
            const int tbl = dd / (kBC * kBC), r = (dd / kBC) % kBC, s = dd % kBC;
            // C1: delta_s . dO_r;  C2: delta_s . d(delta)_r;  C3: delta_r . d(delta)_s (times b_s)
            const int xb = L::DL + (tbl == 2 ? r : s) * TD;
            const int yb = tbl == 0 ? L::DO + r * TD : L::DD + (tbl == 1 ? r : s) * TD;
            float acc = 0.f;
            for (int c = lane; c < D; c += 32) acc = fmaf(sm[xb + c], sm[yb + c], acc);
            acc = warp_sum(acc);
            if (lane == 0) {
                if (tbl == 0) sm[L::C1 + r * kBC + s] = acc;
                else if (tbl == 1) sm[L::C2 + r * kBC + s] = acc;
                else sm[L::C3 + r * kBC + s] = sm[L::BETA + s] * acc;  // delta_r . dv_s
            }
        }
        __syncthreads();
        // right products: S dO -> R, S d(delta) -> DG, F delta -> X
        right_partials(sS, L::DO);
        __syncthreads();
        for (int e = tid; e < kBC * D; e += kBT) tl(L::R, e / D, e % D) = red_sum(e / D, e % D);
        __syncthreads();
        right_partials(sS, L::DD);
        __syncthreads();
        for (int e = tid; e < kBC * D; e += kBT) tl(L::DG, e / D, e % D) = red_sum(e / D, e % D);
        __syncthreads();
        right_partials(sF, L::DL);
        __syncthreads();
        for (int e = tid; e < kBC * D; e += kBT) tl(L::X, e / D, e % D) = red_sum(e / D, e % D);
        __syncthreads();
        // per (token, channel): dq, dk, and q dq - k dkw + k dkr
        for (int e = tid; e < kBC * D; e += kBT) {
            const int r = e / D, c = e % D;
            const float gam = tl(L::GAM, r, c), kr = tl(L::K, r, c), qr = tl(L::Q, r, c);
            float gq = gam * tl(L::R, r, c);
            for (int s = 0; s <= r; ++s)
                gq = fmaf(sm[L::E + pidx(r, s) * D + c] * tl(L::K, s, c), sm[L::C1 + r * kBC + s], gq);
            float gkr = 0.f;
            if (erase) {
                gkr = gam * tl(L::DG, r, c);
                for (int s = 0; s < r; ++s)
                    gkr = fmaf(sm[L::E + pidx(r, s) * D + c] * tl(L::K, s, c), sm[L::C2 + r * kBC + s], gkr);
                gkr *= -sm[L::BETA + r];
            }
            float gkw = expf(tl(L::G, kBC - 1, c) - tl(L::G, r, c)) * tl(L::X, r, c);
            for (int s = r; s < kBC; ++s) {
                const float es = sm[L::E + pidx(s, r) * D + c];
                gkw = fmaf(es * tl(L::Q, s, c), sm[L::C1 + s * kBC + r], gkw);
                if (erase && s > r) gkw = fmaf(-es * tl(L::K, s, c), sm[L::C3 + r * kBC + s], gkw);
            }
            if (r < len) {
                const size_t off = ((tok0 + (size_t)n * kBC + r) * H + h) * D + c;
                dq[off] = from_f32<T>(gq);
                dk[off] = from_f32<T>(gkw + gkr);
            }
            tl(L::DG, r, c) = qr * gq - kr * gkw + kr * gkr;
        }
        __syncthreads();
        // decay gradient: reverse running sum per channel
        if (gate != 2) {
            for (int c = tid; c < D; c += kBT) {
                float acc = sm[L::CARRY + c];
                for (int r = kBC - 1; r >= 0; --r) {
                    acc += tl(L::DG, r, c);
                    if (gate == 0) {
                        if (r < len) dla[((tok0 + (size_t)n * kBC + r) * H + h) * D + c] = from_f32<T>(acc);
                    } else {
                        tl(L::DG, r, c) = acc;
                    }
                }
                sm[L::CARRY + c] = acc;
            }
            if (gate == 1) {
                __syncthreads();
                if (warp < kBC) {
                    const int r = warp;
                    float acc = 0.f;
                    for (int c = lane; c < D; c += 32) acc += tl(L::DG, r, c);
                    acc = warp_sum(acc);
                    if (lane == 0 && r < len) dla[(tok0 + (size_t)n * kBC + r) * H + h] = from_f32<T>(acc);
                }
            }
        }
        // F <- Gamma_last F + (q e^G)^T dO - (k e^G)^T dv
        rank_update(sF, L::GAM, L::Q, L::GAM, L::DO, erase != 0, L::K, L::GAM, L::DD, -1.f, true);
        __syncthreads();
    };

    // the (entry state, delta) slot of every chunk, when they are all kept
    float* all = ckpt + (size_t)bh * NB * kRing;
    // ---- forward sweep: every chunk's entry state and delta, or the state
    // every kBlk chunks; and S_T
    load_mat(sS, S0 ? S0 + (size_t)bh * kMat : nullptr);
    __syncthreads();
    for (int n = 0; n < NB; ++n) {
        float* dslot = nullptr;
        if (store_all) {
            store_mat(sS, all + (size_t)n * kRing);
            dslot = all + (size_t)n * kRing + kMat;
        } else if (n % kBlk == 0) {
            store_mat(sS, ck + (size_t)(n / kBlk) * kMat);
        }
        __syncthreads();
        fwd_step(n, dslot, true);
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
    // ---- backward sweep over the chunks in reverse. Without every slot kept,
    // the top chunk of each block of kBlk first recomputes the block's entry
    // states and deltas into the ring.
    int n0 = 0;
    for (int n = NB - 1; n >= 0; --n) {
        const float* slot;
        if (store_all) {
            slot = all + (size_t)n * kRing;
        } else {
            if (n == NB - 1 || n % kBlk == kBlk - 1) {
                n0 = n - n % kBlk;
                load_mat(sS, ck + (size_t)(n0 / kBlk) * kMat);
                __syncthreads();
                for (int r = n0; r <= n; ++r) {
                    float* rs = rg + (size_t)(r - n0) * kRing;
                    store_mat(sS, rs);
                    __syncthreads();
                    fwd_step(r, rs + kMat, r < n);
                }
            }
            slot = rg + (size_t)(n - n0) * kRing;
        }
        load_mat(sS, slot);
        __syncthreads();
        bwd_step(n, slot + kMat);
    }
    if (dS0) store_mat(sF, dS0 + (size_t)bh * kMat);
}

// Keep every chunk's entry state and delta (no recompute sweep) while that
// takes at most this much workspace; beyond it, one state per 64 tokens and a
// per-CTA ring of recomputed ones.
constexpr size_t kStoreAllCap = (size_t)16 << 30;

size_t bwd_bytes_all(int B, int T, int H, int d) {
    const size_t NB = (size_t)(T + kBC - 1) / kBC;
    return (size_t)B * H * NB * ((size_t)d * d + (size_t)kBC * d) * sizeof(float);
}

bool bwd_store_all(int B, int T, int H, int d, int mode) {
    return mode == 1 || (mode == 0 && bwd_bytes_all(B, T, H, d) <= kStoreAllCap);
}

template <typename T, int D>
cudaError_t launch_bwd_t(const BwdArgs& a, cudaStream_t stream) {
    using L = BwdLayout<D>;
    auto kern = chunk_bwd_kernel<T, D>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::BYTES);
    if (err != cudaSuccess) return err;
    const size_t NBLK = ((size_t)(a.T + kBC - 1) / kBC + kBlk - 1) / kBlk;
    const int store_all = bwd_store_all(a.B, a.T, a.H, D, a.mode) ? 1 : 0;
    float* ckpt = static_cast<float*>(a.workspace);
    float* ring = ckpt + (size_t)a.B * a.H * NBLK * D * D;  // then B*H*kBlk slots of (state, delta)
    kern<<<(unsigned)(a.B * a.H), kBT, L::BYTES, stream>>>(
        (const T*)a.q, (const T*)a.k, (const T*)a.v, (const T*)a.log_alpha, (const T*)a.beta, a.S0, (const T*)a.dO,
        a.dST, (T*)a.g_q, (T*)a.g_k, (T*)a.g_v, (T*)a.g_log_alpha, (T*)a.g_beta, a.g_S0, ckpt, ring, a.T, a.H,
        a.erase, a.gate, store_all);
    return cudaGetLastError();
}

}  // namespace

size_t chunk_bwd_workspace_bytes(int B, int T, int H, int d, int mode) {
    if (bwd_store_all(B, T, H, d, mode)) return bwd_bytes_all(B, T, H, d);
    const size_t NBLK = ((size_t)(T + kBC - 1) / kBC + kBlk - 1) / kBlk;
    return (size_t)B * H * (NBLK * d * d + kBlk * ((size_t)d * d + (size_t)kBC * d)) * sizeof(float);
}

cudaError_t launch_chunk_bwd(const BwdArgs& a, cudaStream_t stream) {
    if (a.bf16) return a.d == 64 ? launch_bwd_t<__nv_bfloat16, 64>(a, stream) : launch_bwd_t<__nv_bfloat16, 128>(a, stream);
    return a.d == 64 ? launch_bwd_t<float, 64>(a, stream) : launch_bwd_t<float, 128>(a, stream);
}

}  // namespace kda
