// Fused KDA chunkwise prefill on sm_100a: tcgen05 tensor cores, TMEM-resident
// state, TMA-fed inputs. bf16 q, k, v, log_alpha, beta, o; fp32 state and
// accumulation; dk = dv = 128; chunk C = 64.
//
// Chunkwise form ("Decoding Hybrid Attention Architectures", section 4;
// "Technical Analysis ... Novel Hybrid Linear Attention", sections 3.1-3.2),
// decay placement derived from the recurrence. For a chunk with local
// cumulative log-decay G_r (per key channel) and chunk-start state S:
//   A = StrictTril(beta_r * sum_c k_rc k_sc e^{G_rc - G_sc})
//   P = Tril     (         sum_c q_rc k_sc e^{G_rc - G_sc})
//   T = (I + A)^{-1},  T' = T Diag(beta)
//   W = T' (k e^G),    U = T' v                 (precomputed per chunk)
//   delta = U - W S                              (per-token corrected write)
//   O     = (q e^G) S + P delta
//   S    <- Diag(e^{G_last}) S + (k e^{G_last - G})^T delta
//
// One CTA owns one (batch, head) and a DVT-wide slice of value channels. The
// slice's state S (dk x DVT fp32) lives in tensor memory for the whole
// sequence. Per chunk, all on one SM:
//   TMA      : k, q, log_alpha tiles (64 x 128 bf16) and the v slice land in
//              shared memory (128-byte swizzle); the next chunk's tiles are
//              requested as soon as the current ones are consumed.
//   SIMT     : cumulative gate G and the decay-scaled MMA operands.
//   tcgen05  : [K e^{G-G_m}; Q e^{G-G_m}] (K e^{G_m-G})^T  -> A and P   (M=128)
//   SIMT     : (I + A)^{-1} by blocked forward substitution (16x16 blocks)
//   tcgen05  : U = [T'; 0] V  straight into the output accumulator D1,
//              W^T = (K e^G)^T T'^T
//   tcgen05  : D1 += [-W; Q e^G] S          -> rows 0-63 delta, 64-127 Q~S
//   tcgen05  : S  += (K e^{G_last-G})^T delta,  D1 += [0; P] delta  -> O
//
// Overflow safety of the decay exponentials: the intra-chunk products use the
// factorisation e^{G_r - G_s} = e^{G_r - G_m} e^{G_m - G_s} with G_m the
// gate at the middle of the chunk, so each factor is a single exponential
// that fits bf16/fp32 as long as |G_r - G_m| <= 80 for every token and
// channel. A block-wide guard checks that bound per chunk; a chunk that
// violates it is handled with exact per-pair exponentials e^{G_r - G_s}
// (exponent <= 0, never overflows) on the SIMT pipes instead.
//
// Every wait on an mbarrier is bounded; on expiry the kernel records
// status 1 in the caller's workspace word, stops, frees its tensor memory
// and returns.
#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_sm100.cuh"

namespace kda {

using namespace sm100;

namespace {

constexpr int kThreads = 256;
constexpr int kC = 64;    // chunk
constexpr int kD = 128;   // dk = dv
constexpr int kLDA = 68;  // fp32 row stride of the A / T scratch (bank spread)
constexpr float kGuard = 80.f;
constexpr long long kWaitBudget = 1ll << 31;  // SM cycles (~1 s)

template <int DVT>
struct Layout {
    // bytes, relative to a 1024-aligned base
    static constexpr uint32_t RAWK = 0;                    // 2 boxes [64 tok][64 ch] bf16, swizzled
    static constexpr uint32_t RAWQ = RAWK + 16384;
    static constexpr uint32_t RAWG = RAWQ + 16384;
    static constexpr uint32_t RAWV = RAWG + 16384;         // DVT/64 boxes [64 tok][64 ch]
    static constexpr uint32_t R48 = RAWV + DVT * 128;      // 48 KB, reused within a chunk:
    static constexpr uint32_t ROWOP = R48;                 //   [K e^{G-Gm}; Q e^{G-Gm}]  MN-major 128x128
    static constexpr uint32_t COLOP = R48 + 32768;         //   K e^{Gm-G}               MN-major  64x128
    static constexpr uint32_t SA = R48;                    //   A  fp32 [64][68]
    static constexpr uint32_t ST = R48 + 64 * kLDA * 4;    //   T  fp32 [64][68]
    static constexpr uint32_t SY = ST + 64 * kLDA * 4;     //   block products fp32 [3][16][16]
    static constexpr uint32_t SOP = R48;                   //   S bf16, MN-major (K = dk) x DVT
    static constexpr uint32_t DOP = R48 + 32768;           //   delta bf16, MN-major (K = 64) x DVT
    static constexpr uint32_t XOP = R48 + 49152;           // (K e^G)^T  K-major 128 x 64
    static constexpr uint32_t WQ = XOP + 16384;            // [-W; Q e^G] MN-major 128x128 (also G fp32, exact path)
    static constexpr uint32_t KT = WQ + 32768;             // (K e^{G_last-G})^T  K-major 128 x 64
    static constexpr uint32_t TZP = KT + 16384;            // T' (64x64) | zeros (64x64) | P (64x64), K-major
    static constexpr uint32_t SMALL = TZP + 24576;
    static constexpr uint32_t SBETA = SMALL;               // 64 f32
    static constexpr uint32_t SGAM = SBETA + 256;          // 128 f32
    static constexpr uint32_t SPART = SGAM + 512;          // 2 x 128 f32
    static constexpr uint32_t SRED = SPART + 1024;         // 8 f32
    static constexpr uint32_t BARS = SRED + 32;            // 3 mbarriers
    static constexpr uint32_t MISC = BARS + 32;            // tmem base, abort flag
    static constexpr uint32_t END = MISC + 16;
    static constexpr uint32_t SMEM_BYTES = END + 1024;     // + alignment slack
    static constexpr uint32_t SBO_V = 1024 * (DVT / 64);   // K-group stride of S / delta operands
    // tensor memory columns
    static constexpr uint32_t S_COL = 0;
    static constexpr uint32_t D1_COL = DVT;
    static constexpr uint32_t AP_COL = 2 * DVT;
    static constexpr uint32_t WT_COL = 2 * DVT + 64;
    static constexpr uint32_t TMEM_COLS = (2 * DVT + 128 <= 256) ? 256 : 512;
    static_assert(SY + 3 * 256 * 4 <= R48 + 49152, "R48 overflow");
    static_assert(SOP + 128 * DVT * 2 <= DOP && DOP + 64 * DVT * 2 <= R48 + 49152, "R48 overflow");
};

__device__ __forceinline__ float ld_bf16(const uint8_t* base, uint32_t off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + off));
}

// offset of element (token r, channel c) in a [64 tok][128 ch] tile stored as
// two TMA boxes of [64][64] with the 128-byte swizzle
__device__ __forceinline__ uint32_t raw_off(int r, int c) {
    return (uint32_t)((c >> 6) * 8192 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1));
}

template <int DVT>
__global__ void __launch_bounds__(kThreads, 1)
kda_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_v,
                    const __nv_bfloat16* __restrict__ beta, const float* S0, __nv_bfloat16* __restrict__ o,
                    float* ST, int Tlen, int H, unsigned* status) {
    using L = Layout<DVT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nslices = kD / DVT;
    const int bh = blockIdx.x / nslices;
    const int b = bh / H, h = bh % H;
    const int j0 = (blockIdx.x % nslices) * DVT;
    const int NC = (Tlen + kC - 1) / kC;

    float* sBeta = reinterpret_cast<float*>(sm + L::SBETA);
    float* sGam = reinterpret_cast<float*>(sm + L::SGAM);
    float* sPart = reinterpret_cast<float*>(sm + L::SPART);
    float* sRed = reinterpret_cast<float*>(sm + L::SRED);
    uint64_t* bar_kqg = reinterpret_cast<uint64_t*>(sm + L::BARS);
    uint64_t* bar_v = bar_kqg + 1;
    uint64_t* bar_mma = bar_kqg + 2;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + L::MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(sm + L::MISC + 4);
    float* sA = reinterpret_cast<float*>(sm + L::SA);
    float* sT = reinterpret_cast<float*>(sm + L::ST);
    float* sY = reinterpret_cast<float*>(sm + L::SY);

    // ---- setup
    if (tid == 0) {
        mbar_init(bar_kqg, 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_mma, 1);
        *s_abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_g);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, L::TMEM_COLS);
        tmem_relinquish();
    }
    {  // zero block between T' and P (rows 0-63 of the [0; P] operand, rows 64-127 of [T'; 0])
        uint4* z = reinterpret_cast<uint4*>(sm + L::TZP + 8192);
        for (int i = tid; i < 8192 / 16; i += kThreads) z[i] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    constexpr uint32_t KQG_BYTES = 3 * 2 * 8192;
    constexpr uint32_t V_BYTES = (DVT / 64) * 8192;
    auto issue_kqg = [&](int n) {
        mbar_arrive_expect_tx(bar_kqg, KQG_BYTES);
        for (int x = 0; x < 2; ++x) {
            tma_load_4d(sm + L::RAWK + x * 8192, &tm_k, bar_kqg, 64 * x, h, n * kC, b);
            tma_load_4d(sm + L::RAWQ + x * 8192, &tm_q, bar_kqg, 64 * x, h, n * kC, b);
            tma_load_4d(sm + L::RAWG + x * 8192, &tm_g, bar_kqg, 64 * x, h, n * kC, b);
        }
    };
    auto issue_v = [&](int n) {
        mbar_arrive_expect_tx(bar_v, V_BYTES);
        for (int x = 0; x < DVT / 64; ++x)
            tma_load_4d(sm + L::RAWV + x * 8192, &tm_v, bar_v, j0 + 64 * x, h, n * kC, b);
    };
    if (tid == 0 && NC > 0) {
        issue_kqg(0);
        issue_v(0);
    }

    // Thread <-> tensor-memory lane mapping for whole-tile readouts: warp w
    // reads lanes 32*(w%4) .. +31 and half `hf` of the columns.
    const int quad = warp & 3, hf = warp >> 2;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * quad) << 16);
    constexpr int NJ = DVT / 2;  // state / output columns per thread

    // ---- initial state into TMEM (fp32, lane = key channel)
    {
        const int c = 32 * quad + lane;
#pragma unroll
        for (int g = 0; g < NJ / 32; ++g) {
            uint32_t r[32];
            const int jb = hf * NJ + 32 * g;
            if (S0) {
                const float4* src = reinterpret_cast<const float4*>(S0 + ((size_t)bh * kD + c) * kD + j0 + jb);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const float4 v = src[u];
                    r[4 * u] = __float_as_uint(v.x); r[4 * u + 1] = __float_as_uint(v.y);
                    r[4 * u + 2] = __float_as_uint(v.z); r[4 * u + 3] = __float_as_uint(v.w);
                }
            } else {
#pragma unroll
                for (int u = 0; u < 32; ++u) r[u] = 0u;
            }
            tmem_st32(lane_addr + L::S_COL + jb, r);
        }
        tmem_st_wait();
    }

    uint32_t mma_phase = 0;
    auto wait_mma = [&]() {
        if (!*s_abort && !mbar_wait_bounded(bar_mma, mma_phase & 1, kWaitBudget)) {
            atomicExch(status, 1u);
            *s_abort = 1;
        }
        ++mma_phase;
        tc_fence_after();
    };

    constexpr uint32_t ID_AP = idesc_bf16(128, 64, 1, 1);
    constexpr uint32_t ID_U = idesc_bf16(128, DVT, 0, 1);
    constexpr uint32_t ID_WT = idesc_bf16(128, 64, 0, 0);
    constexpr uint32_t ID_M1 = idesc_bf16(128, DVT, 1, 1);
    constexpr uint32_t ID_M2 = idesc_bf16(128, DVT, 0, 1);

    for (int n = 0; n < NC; ++n) {
        const int t0 = n * kC;
        const int len = min(kC, Tlen - t0);
        tc_fence_before();
        __syncthreads();
        if (*s_abort) break;

        // ---- P1: inputs of this chunk
        if (tid < kC) sBeta[tid] = tid < len ? __bfloat162float(beta[((size_t)b * Tlen + t0 + tid) * H + h]) : 0.f;
        if (!mbar_wait_bounded(bar_kqg, n & 1, kWaitBudget)) {
            atomicExch(status, 1u);
            *s_abort = 1;
        }
        __syncthreads();
        if (*s_abort) break;

        // ---- P2: cumulative gate, guard, decay-scaled operands.
        // thread <-> (channel c, token half hh)
        const int c = tid & 127, hh = tid >> 7, r0 = 32 * hh;
        float g[32];
        {
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                acc += ld_bf16(sm + L::RAWG, raw_off(r0 + i, c));
                g[i] = acc;
            }
            sPart[hh * 128 + c] = acc;
        }
        __syncthreads();
        const float G31 = sPart[c];
        const float G63 = sPart[c] + sPart[128 + c];
        if (hh) {
#pragma unroll
            for (int i = 0; i < 32; ++i) g[i] += G31;
        }
        float dev = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) dev = fmaxf(dev, fabsf(g[i] - G31));
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) dev = fmaxf(dev, __shfl_xor_sync(0xffffffffu, dev, o2));
        if (lane == 0) sRed[warp] = dev;
        if (hh == 0) sGam[c] = __expf(G63);
        __syncthreads();
        float devmax = sRed[0];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) devmax = fmaxf(devmax, sRed[w]);
        const bool exact = !(devmax <= kGuard);  // also catches NaN

        if (exact) {
            // Exact path: per-pair exponentials with exponent G_r - G_s <= 0.
            float* sG = reinterpret_cast<float*>(sm + L::WQ);  // [64][128] fp32
#pragma unroll
            for (int i = 0; i < 32; ++i) sG[(r0 + i) * 128 + c] = g[i];
            for (int i = tid; i < 64 * kLDA; i += kThreads) sA[i] = 0.f;
            for (int i = tid; i < 8192 / 16; i += kThreads)
                reinterpret_cast<uint4*>(sm + L::TZP + 16384)[i] = make_uint4(0, 0, 0, 0);
            __syncthreads();
            for (int p = tid; p < kC * (kC + 1) / 2; p += kThreads) {
                int r = (int)((sqrtf(8.f * (float)p + 1.f) - 1.f) * 0.5f);
                while ((r + 1) * (r + 2) / 2 <= p) ++r;
                while (r * (r + 1) / 2 > p) --r;
                const int s = p - r * (r + 1) / 2;
                float a = 0.f, pp = 0.f;
                for (int i = 0; i < kD; ++i) {
                    const int cc = (i + p) & (kD - 1);
                    const float ks = ld_bf16(sm + L::RAWK, raw_off(s, cc)) * __expf(sG[r * 128 + cc] - sG[s * 128 + cc]);
                    a = fmaf(ld_bf16(sm + L::RAWK, raw_off(r, cc)), ks, a);
                    pp = fmaf(ld_bf16(sm + L::RAWQ, raw_off(r, cc)), ks, pp);
                }
                if (s < r) sA[r * kLDA + s] = sBeta[r] * a;
                *reinterpret_cast<__nv_bfloat16*>(sm + L::TZP + 16384 + r * 128 + ((((s >> 3) ^ (r & 7))) << 4) +
                                                  ((s & 7) << 1)) = __float2bfloat16_rn(pp);
            }
            __syncthreads();
        }

        {
            // operands built from this thread's 32 tokens, 8 tokens (16 bytes) at a time
            // e^{G_r} as e^{G_r - G_m} e^{G_m} unless e^{G_m} is below the
            // normal range; e^{G_last - G_r} = e^{G_m - G_r} e^{G_last - G_m}
            // (the guard keeps the second factor >= e^-80).
            const float eGm = __expf(G31), eKm = __expf(G63 - G31);
            const bool direct_eg = exact || G31 < -kGuard;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t ke[4], qe[4], kf[4], xx[4], qt[4], kt[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int i = 8 * j + 2 * u;
                    const int r = r0 + i;
                    const float k0 = ld_bf16(sm + L::RAWK, raw_off(r, c)), k1 = ld_bf16(sm + L::RAWK, raw_off(r + 1, c));
                    const float q0 = ld_bf16(sm + L::RAWQ, raw_off(r, c)), q1 = ld_bf16(sm + L::RAWQ, raw_off(r + 1, c));
                    float eg0, eg1, ek0, ek1;
                    if (!exact) {
                        const float E0 = __expf(g[i] - G31), E1 = __expf(g[i + 1] - G31);
                        const float F0 = __expf(G31 - g[i]), F1 = __expf(G31 - g[i + 1]);
                        ke[u] = pack_bf16x2(k0 * E0, k1 * E1);
                        qe[u] = pack_bf16x2(q0 * E0, q1 * E1);
                        kf[u] = pack_bf16x2(k0 * F0, k1 * F1);
                        if (direct_eg) {
                            eg0 = __expf(g[i]); eg1 = __expf(g[i + 1]);
                        } else {
                            eg0 = E0 * eGm; eg1 = E1 * eGm;
                        }
                        ek0 = F0 * eKm; ek1 = F1 * eKm;
                    } else {
                        eg0 = __expf(g[i]); eg1 = __expf(g[i + 1]);
                        ek0 = __expf(G63 - g[i]); ek1 = __expf(G63 - g[i + 1]);
                    }
                    xx[u] = pack_bf16x2(k0 * eg0, k1 * eg1);
                    qt[u] = pack_bf16x2(q0 * eg0, q1 * eg1);
                    kt[u] = pack_bf16x2(k0 * ek0, k1 * ek1);
                }
                const uint32_t chunk = (uint32_t)(((r0 >> 3) + j) ^ (c & 7)) << 4;
                const uint32_t mn = (uint32_t)(c >> 3) * 2048 + (uint32_t)(c & 7) * 128 + chunk;  // 128-row MN-major
                const uint32_t km = (uint32_t)c * 128 + chunk;                                     // K-major rows c
                if (!exact) {
                    st_shared_v4(sb + L::ROWOP + mn, ke[0], ke[1], ke[2], ke[3]);
                    st_shared_v4(sb + L::ROWOP + mn + 1024, qe[0], qe[1], qe[2], qe[3]);
                    st_shared_v4(sb + L::COLOP + (uint32_t)(c >> 3) * 1024 + (uint32_t)(c & 7) * 128 + chunk,
                                 kf[0], kf[1], kf[2], kf[3]);
                }
                st_shared_v4(sb + L::XOP + km, xx[0], xx[1], xx[2], xx[3]);
                st_shared_v4(sb + L::KT + km, kt[0], kt[1], kt[2], kt[3]);
                st_shared_v4(sb + L::WQ + mn + 1024, qt[0], qt[1], qt[2], qt[3]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // raw k, q, log_alpha consumed: fetch the next chunk's
        if (tid == 0 && n + 1 < NC) issue_kqg(n + 1);

        if (!exact) {
            // ---- P3: A and P on the tensor cores
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ss(tmem + L::AP_COL, sdesc_sw128(sb + L::ROWOP + kk * 4096, 1024, 2048),
                                sdesc_sw128(sb + L::COLOP + kk * 2048, 1024, 1024), ID_AP, kk > 0);
                mma_commit(bar_mma);
            }
            wait_mma();
            // ---- P4: A (lanes 0-63) -> fp32 scratch; P (lanes 64-127) -> bf16 operand
            {
                uint32_t v[32];
                tmem_ld32(lane_addr + L::AP_COL + 32 * hf, v);
                tmem_ld_wait(v);
                if (quad < 2) {
                    const int r = 32 * quad + lane;
                    const float br = sBeta[r];
                    float* dst = sA + r * kLDA + 32 * hf;
#pragma unroll
                    for (int u = 0; u < 32; u += 4) {
                        float4 f;
                        f.x = (32 * hf + u + 0 < r) ? br * __uint_as_float(v[u + 0]) : 0.f;
                        f.y = (32 * hf + u + 1 < r) ? br * __uint_as_float(v[u + 1]) : 0.f;
                        f.z = (32 * hf + u + 2 < r) ? br * __uint_as_float(v[u + 2]) : 0.f;
                        f.w = (32 * hf + u + 3 < r) ? br * __uint_as_float(v[u + 3]) : 0.f;
                        *reinterpret_cast<float4*>(dst + u) = f;
                    }
                } else {
                    const int r = 32 * (quad - 2) + lane;
#pragma unroll
                    for (int jc = 0; jc < 4; ++jc) {
                        uint32_t w[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int s = 32 * hf + 8 * jc + 2 * u;
                            const float p0 = (s <= r) ? __uint_as_float(v[8 * jc + 2 * u]) : 0.f;
                            const float p1 = (s + 1 <= r) ? __uint_as_float(v[8 * jc + 2 * u + 1]) : 0.f;
                            w[u] = pack_bf16x2(p0, p1);
                        }
                        st_shared_v4(sb + L::TZP + 16384 + r * 128 + ((((4 * hf + jc) ^ (r & 7))) << 4), w[0], w[1],
                                     w[2], w[3]);
                    }
                }
            }
            __syncthreads();
        }

        // ---- P5: T = (I + A)^{-1}. Diagonal 16x16 blocks by forward
        // substitution (one column per thread), then the blocks below the
        // diagonal level by level: T_ab = -T_aa * sum_{b<=k<a} A_ak T_kb.
        if (tid < 64) {
            const int a = tid >> 4, jc = tid & 15;
            const float* Ab = sA + (16 * a) * kLDA + 16 * a;
            float col[16], acc[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[i] = 0.f;
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const float t = (r == jc) ? 1.f : (r > jc ? -acc[r] : 0.f);
                col[r] = t;
#pragma unroll
                for (int r2 = r + 1; r2 < 16; ++r2) acc[r2] = fmaf(Ab[r2 * kLDA + r], t, acc[r2]);
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) sT[(16 * a + r) * kLDA + 16 * a + jc] = col[r];
        }
        __syncthreads();
#pragma unroll 1
        for (int d = 1; d < 4; ++d) {
            const int nblk = 4 - d;
            for (int e = tid; e < nblk * 256; e += kThreads) {
                const int bb = e >> 8, i = (e >> 4) & 15, jj = e & 15, aa = bb + d;
                float y = 0.f;
                for (int kb = bb; kb < aa; ++kb) {
                    const float* arow = sA + (16 * aa + i) * kLDA + 16 * kb;
                    const float* tcol = sT + (16 * kb) * kLDA + 16 * bb + jj;
#pragma unroll
                    for (int m = 0; m < 16; ++m) y = fmaf(arow[m], tcol[m * kLDA], y);
                }
                sY[e] = y;
            }
            __syncthreads();
            for (int e = tid; e < nblk * 256; e += kThreads) {
                const int bb = e >> 8, i = (e >> 4) & 15, jj = e & 15, aa = bb + d;
                const float* trow = sT + (16 * aa + i) * kLDA + 16 * aa;
                const float* ycol = sY + bb * 256 + jj;
                float t = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m) t = fmaf(trow[m], ycol[m * 16], t);
                sT[(16 * aa + i) * kLDA + 16 * bb + jj] = -t;
            }
            __syncthreads();
        }
        // T' = T Diag(beta) -> bf16, K-major rows r (s contiguous)
        for (int e = tid; e < 64 * 8; e += kThreads) {
            const int r = e >> 3, ch = e & 7;
            uint32_t w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int s = 8 * ch + 2 * u;
                const float t0v = (s <= r) ? sT[r * kLDA + s] * sBeta[s] : 0.f;
                const float t1v = (s + 1 <= r) ? sT[r * kLDA + s + 1] * sBeta[s + 1] : 0.f;
                w[u] = pack_bf16x2(t0v, t1v);
            }
            st_shared_v4(sb + L::TZP + r * 128 + (((ch ^ (r & 7))) << 4), w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- P6: U = [T'; 0] V into D1, W^T = X^T T'^T into WT
        if (tid == 0) {
            if (!mbar_wait_bounded(bar_v, n & 1, kWaitBudget)) {
                atomicExch(status, 1u);
                *s_abort = 1;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + L::D1_COL, sdesc_sw128(sb + L::TZP + kk * 32, 16, 1024),
                            sdesc_sw128(sb + L::RAWV + kk * 2048, 8192, 1024), ID_U, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + L::WT_COL, sdesc_sw128(sb + L::XOP + kk * 32, 16, 1024),
                            sdesc_sw128(sb + L::TZP + kk * 32, 16, 1024), ID_WT, kk > 0);
            mma_commit(bar_mma);
        }
        wait_mma();
        if (tid == 0 && n + 1 < NC) issue_v(n + 1);

        // ---- P7: -W from W^T (lane c, columns r) -> rows 0-63 of [-W; Q e^G]
        {
            const int cc = 32 * quad + lane;
            uint32_t v[32];
            tmem_ld32(lane_addr + L::WT_COL + 32 * hf, v);
            tmem_ld_wait(v);
#pragma unroll
            for (int jc = 0; jc < 4; ++jc) {
                uint32_t w[4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    w[u] = pack_bf16x2(-__uint_as_float(v[8 * jc + 2 * u]), -__uint_as_float(v[8 * jc + 2 * u + 1]));
                const uint32_t off = (uint32_t)(cc >> 3) * 2048 + (uint32_t)(cc & 7) * 128 +
                                     ((uint32_t)((4 * hf + jc) ^ (cc & 7)) << 4);
                st_shared_v4(sb + L::WQ + off, w[0], w[1], w[2], w[3]);
            }
        }

        // ---- S1: state -> bf16 operand; state *= gamma in place
        {
            const int cc = 32 * quad + lane;
            const float gam = sGam[cc];
#pragma unroll
            for (int gq = 0; gq < NJ / 32; ++gq) {
                const int jb = hf * NJ + 32 * gq;
                uint32_t v[32];
                tmem_ld32(lane_addr + L::S_COL + jb, v);
                tmem_ld_wait(v);
#pragma unroll
                for (int jc = 0; jc < 4; ++jc) {
                    uint32_t w[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        w[u] = pack_bf16x2(__uint_as_float(v[8 * jc + 2 * u]), __uint_as_float(v[8 * jc + 2 * u + 1]));
                    const int j = jb + 8 * jc;
                    const uint32_t off = (uint32_t)(cc >> 3) * L::SBO_V + (uint32_t)(j >> 6) * 1024 +
                                         (uint32_t)(cc & 7) * 128 + ((uint32_t)(((j & 63) >> 3) ^ (cc & 7)) << 4);
                    st_shared_v4(sb + L::SOP + off, w[0], w[1], w[2], w[3]);
                }
#pragma unroll
                for (int u = 0; u < 32; ++u) v[u] = __float_as_uint(__uint_as_float(v[u]) * gam);
                tmem_st32(lane_addr + L::S_COL + jb, v);
            }
            tmem_st_wait();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- S2: D1 += [-W; Q e^G] S   (rows 0-63 become delta = U - W S)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16_ss(tmem + L::D1_COL, sdesc_sw128(sb + L::WQ + kk * 4096, 1024, 2048),
                            sdesc_sw128(sb + L::SOP + kk * 2 * L::SBO_V, 1024, L::SBO_V), ID_M1, 1);
            mma_commit(bar_mma);
        }
        wait_mma();

        // ---- S3: delta (lanes 0-63) -> bf16 operand, MN-major (K = token)
        if (quad < 2) {
            const int r = 32 * quad + lane;
#pragma unroll
            for (int gq = 0; gq < NJ / 32; ++gq) {
                const int jb = hf * NJ + 32 * gq;
                uint32_t v[32];
                tmem_ld32(lane_addr + L::D1_COL + jb, v);
                tmem_ld_wait(v);
#pragma unroll
                for (int jc = 0; jc < 4; ++jc) {
                    uint32_t w[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        w[u] = pack_bf16x2(__uint_as_float(v[8 * jc + 2 * u]), __uint_as_float(v[8 * jc + 2 * u + 1]));
                    const int j = jb + 8 * jc;
                    const uint32_t off = (uint32_t)(r >> 3) * L::SBO_V + (uint32_t)(j >> 6) * 1024 +
                                         (uint32_t)(r & 7) * 128 + ((uint32_t)(((j & 63) >> 3) ^ (r & 7)) << 4);
                    st_shared_v4(sb + L::DOP + off, w[0], w[1], w[2], w[3]);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- S4: S += Ktilde^T delta ; D1 += [0; P] delta   (rows 64-127 become O)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + L::S_COL, sdesc_sw128(sb + L::KT + kk * 32, 16, 1024),
                            sdesc_sw128(sb + L::DOP + kk * 2 * L::SBO_V, 1024, L::SBO_V), ID_M2, 1);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + L::D1_COL, sdesc_sw128(sb + L::TZP + 8192 + kk * 32, 16, 1024),
                            sdesc_sw128(sb + L::DOP + kk * 2 * L::SBO_V, 1024, L::SBO_V), ID_M2, 1);
            mma_commit(bar_mma);
        }
        wait_mma();

        // ---- S5: O (lanes 64-127) -> global bf16
        if (quad >= 2) {
            const int r = 32 * (quad - 2) + lane;
#pragma unroll
            for (int gq = 0; gq < NJ / 32; ++gq) {
                const int jb = hf * NJ + 32 * gq;
                uint32_t v[32];
                tmem_ld32(lane_addr + L::D1_COL + jb, v);
                tmem_ld_wait(v);
                if (r < len) {
                    uint4* dst = reinterpret_cast<uint4*>(o + (((size_t)b * Tlen + t0 + r) * H + h) * kD + j0 + jb);
#pragma unroll
                    for (int jc = 0; jc < 4; ++jc) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(v[8 * jc + 0]), __uint_as_float(v[8 * jc + 1]));
                        w.y = pack_bf16x2(__uint_as_float(v[8 * jc + 2]), __uint_as_float(v[8 * jc + 3]));
                        w.z = pack_bf16x2(__uint_as_float(v[8 * jc + 4]), __uint_as_float(v[8 * jc + 5]));
                        w.w = pack_bf16x2(__uint_as_float(v[8 * jc + 6]), __uint_as_float(v[8 * jc + 7]));
                        dst[jc] = w;
                    }
                }
            }
        }
    }

    // ---- final state
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (ST && !*s_abort) {
        const int c = 32 * quad + lane;
#pragma unroll
        for (int gq = 0; gq < NJ / 32; ++gq) {
            const int jb = hf * NJ + 32 * gq;
            uint32_t v[32];
            tmem_ld32(lane_addr + L::S_COL + jb, v);
            tmem_ld_wait(v);
            float4* dst = reinterpret_cast<float4*>(ST + ((size_t)bh * kD + c) * kD + j0 + jb);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                dst[u] = make_float4(__uint_as_float(v[4 * u]), __uint_as_float(v[4 * u + 1]),
                                     __uint_as_float(v[4 * u + 2]), __uint_as_float(v[4 * u + 3]));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [B, T, H, 128] bf16 viewed as a 4-D tensor (channel, head, token, batch);
// box = 64 channels x 1 head x 64 tokens x 1 batch, 128-byte swizzle. Tokens
// past T read as zero.
bool make_map(CUtensorMap* m, const void* base, int B, int T, int H) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)T * H * kD * 2};
    const cuuint32_t box[4] = {64, 1, 64, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DVT>
cudaError_t launch_dvt(const ChunkArgs& a, cudaStream_t stream) {
    using L = Layout<DVT>;
    CUtensorMap mk, mq, mg, mv;
    if (!make_map(&mk, a.k, a.B, a.T, a.H) || !make_map(&mq, a.q, a.B, a.T, a.H) ||
        !make_map(&mg, a.log_alpha, a.B, a.T, a.H) || !make_map(&mv, a.v, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    auto kern = kda_chunk_tc_kernel<DVT>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::SMEM_BYTES);
    if (err != cudaSuccess) return err;
    unsigned* status = static_cast<unsigned*>(a.workspace);
    err = cudaMemsetAsync(status, 0, sizeof(unsigned), stream);
    if (err != cudaSuccess) return err;
    const unsigned grid = (unsigned)(a.B * a.H * (kD / DVT));
    kern<<<grid, kThreads, L::SMEM_BYTES, stream>>>(mk, mq, mg, mv, (const __nv_bfloat16*)a.beta, a.S0,
                                                    (__nv_bfloat16*)a.o, a.ST, a.T, a.H, status);
    return cudaGetLastError();
}

}  // namespace

bool chunk_tc_supported(const ChunkArgs& a) {
    return a.bf16 && a.dk == kD && a.dv == kD && a.chunk == kC;
}

size_t chunk_tc_workspace_bytes(int, int, int, int, int) { return 256; }

cudaError_t launch_chunk_tc(const ChunkArgs& a, cudaStream_t stream) {
    // An empty sequence has no chunk to load (and no tensor map can describe
    // it): the result is S_T = S0, which the SIMT kernel writes.
    if (a.T == 0) {
        cudaError_t err = cudaMemsetAsync(a.workspace, 0, sizeof(unsigned), stream);
        return err != cudaSuccess ? err : launch_chunk_simt(a, stream);
    }
    // One CTA per (batch, head) when there are enough heads to fill the
    // GPU; otherwise split the value channels in two.
    if ((long)a.B * a.H >= 96) return launch_dvt<128>(a, stream);
    return launch_dvt<64>(a, stream);
}

}  // namespace kda

// ---------------------------------------------------------------- allocation-free variant
//
// kda_chunk_fwd_noalloc runs the same tensor-core prefill as kda_chunk_fwd
// but keeps the kernel's scratch (its device status word, padded to 256
// bytes) in a fixed array that lives inside this library, so the caller
// passes only inputs and outputs. It exists for callers that must not
// allocate device memory at the point where they run a prefill, for example
// code running inside a memory allocator's own callbacks, host applications
// that forbid cudaMalloc on their worker threads, or runtimes that expose
// only the tensors they already own.
#include <mutex>

#include "kda.h"

// Scratch of the allocation-free entry point; every GPU that loads this
// library holds these bytes until the process exits. In host code this name
// is only a stand-in for the symbol: its device address comes from
// cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_kda_noalloc_scratch[256];

namespace {

constexpr int kNoAllocMaxDevices = 128;
std::mutex g_noalloc_mutex;
void* g_noalloc_scratch_addr[kNoAllocMaxDevices] = {};

// Device address of the scratch array on the current device, looked up on
// the first call made with that device current.
cudaError_t noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_kda_noalloc_scratch);
        if (err != cudaSuccess) return err;
        g_noalloc_scratch_addr[dev] = p;
    }
    *out = g_noalloc_scratch_addr[dev];
    return cudaSuccess;
}

bool noalloc_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" kda_status_t kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const void* log_alpha,
                                              const void* beta, const float* S0, void* o, float* S_T, int B,
                                              int T, int H, int dk, int dv, int chunk, kda_dtype_t dtype,
                                              void* stream) {
    if (B < 0 || T < 0 || H < 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if ((long long)B * H > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    kda::ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.S0 = S0; a.o = o; a.ST = S_T;
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv; a.chunk = chunk; a.bf16 = dtype == KDA_BF16;
    if (!kda::chunk_tc_supported(a)) return KDA_ERR_UNSUPPORTED;
    if ((long long)B * T * H > 0) {
        const void* req[] = {q, k, v, log_alpha, beta, o};
        for (const void* p : req)
            if (p == nullptr || !noalloc_aligned16(p)) return KDA_ERR_INVALID_ARG;
    }
    if ((S0 && !noalloc_aligned16(S0)) || (S_T && !noalloc_aligned16(S_T))) return KDA_ERR_INVALID_ARG;
    // The kernel's scratch must fit the fixed array.
    if (kda::chunk_tc_workspace_bytes(B, T, H, dk, dv) > sizeof(g_kda_noalloc_scratch)) return KDA_ERR_INVALID_ARG;
    if ((long long)B * H == 0) return KDA_OK;
    void* scratch = nullptr;
    if (noalloc_scratch(&scratch) != cudaSuccess) return KDA_ERR_CUDA;
    a.workspace = scratch;
    a.workspace_bytes = sizeof(g_kda_noalloc_scratch);
    // launch_chunk_tc clears the status word before the kernel runs.
    const cudaError_t err = kda::launch_chunk_tc(a, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
