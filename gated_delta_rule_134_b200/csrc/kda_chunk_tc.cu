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
// Reference-point factorisation. With G_m the gate at the chunk's middle token
// and E_r = e^{G_r - G_m}, F_r = e^{G_m - G_r} (per channel):
//   e^{G_r - G_s} = E_r F_s,  k e^G = (k E) e^{G_m},  k e^{G_last-G} = (k F) e^{G_last-G_m}.
// So three bf16 tiles, KE = k E, QE = q E and KF = k F, feed every MMA:
//   [KE; QE] KF^T           -> A and P (one M=128 MMA)
//   W' = T' KE              -> W = W' Diag(e^{G_m})
//   D1 += [-W'; QE] (e^{G_m} S)   -> rows 0-63: U - W S = delta, rows 64-127: (q e^G) S
//   R  = e^{G_m} S + KF^T delta   -> S_next = Diag(e^{G_last-G_m}) R
// The tensor memory therefore holds R, and the next chunk rescales it per
// channel while it copies the state into the bf16 MMA operand. Each factor is
// a single exponential, finite as long as |G_r - G_m| <= 80 and G_m >= -80;
// a block-wide guard checks that per chunk. A chunk that fails the guard uses
// exact per-pair exponentials e^{G_r - G_s} (exponent <= 0) for A and P and the
// plain tiles k e^G, q e^G, k e^{G_last-G} (with G_m := 0); the same MMAs then
// produce the same quantities.
//
// Schedule. One CTA owns one (batch, head) and a DVT-wide slice of value
// channels; its state stays in tensor memory for the whole sequence. Chunk n's
// state-dependent MMAs overlap the state-independent preparation of chunk n+1
// on the same warps:
//   S1(n)  state -> bf16 operand            | cumsum MMA(n+1) issued, then MMA1(n)
//   P2(n+1) gate, guard, KE/QE/KF in regs   | while MMA1(n) runs
//   S3(n)  delta -> bf16; P2(n+1) stores    | then AP(n+1), MMA2(n) issued
//   P4/P5(n+1) A, P readout; (I+A)^{-1}     | while MMA2(n) runs
//   U(n+1), W'(n+1) issued; S5(n) O out; P7(n+1) -W' stored
// The cumulative gate itself is an MMA with a lower-triangular ones matrix.
// (I + A)^{-1}: 16x16 diagonal blocks by forward substitution (four threads per
// column), N = T_diag A_offdiag, then the blocks below the diagonal level by
// level, T_ab = -sum_k N_ak T_kb; T' = T Diag(beta) is written as bf16 by the
// thread that finalises each entry.
//
// Every wait on an mbarrier is bounded; on expiry the kernel records status 1
// in the caller's workspace word, stops, frees its tensor memory and returns.
#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_sm100.cuh"

namespace kda {

using namespace sm100;

namespace {

constexpr int kCompute = 256;             // 8 compute warps
constexpr int kCtrlWarp = kCompute / 32;  // warp 8 issues TMA loads and MMAs
constexpr int kThreads = kCompute + 32;
// named barriers (0 is __syncthreads)
constexpr int NB_SIMT = 1;  // compute warps only
constexpr int NB_OR = 2;    // compute warps only, OR-reduction
constexpr int NB_S1 = 3;    // compute -> control: state operand ready
constexpr int NB_K = 4;     // compute -> control: k, q tiles consumed
constexpr int NB_S3 = 5;    // compute -> control: delta / next-chunk operands ready
constexpr int NB_P5 = 6;    // compute -> control: T' ready
constexpr int kC = 64;    // chunk
constexpr int kD = 128;   // dk = dv
constexpr int kLDA = 68;  // fp32 row stride of the A / T scratch (bank spread)
constexpr float kGuard = 80.f;
constexpr long long kWaitBudget = 1ll << 31;  // SM cycles (~1 s)

template <int DVT>
struct Layout {
    // shared memory, bytes from a 1024-aligned base
    static constexpr uint32_t RAWK = 0;                  // k tile: 2 TMA boxes [64 tok][64 ch], swizzled
    static constexpr uint32_t RAWQ = RAWK + 16384;       // q tile
    static constexpr uint32_t RAWG = RAWQ + 16384;       // log_alpha tile
    static constexpr uint32_t RAWV = RAWG + 16384;       // v slice: DVT/64 boxes; then the delta operand
    static constexpr uint32_t DOP = RAWV;                //   delta bf16, MN-major (K = 64 tokens) x DVT
    static constexpr uint32_t LMAT = RAWV + DVT * 128;   // lower-triangular ones, K-major 64 x 64
    static constexpr uint32_t ROWOP = LMAT + 8192;       // [KE|X|-W'; QE|Q~] MN-major 128 x 128
    static constexpr uint32_t COLOP = ROWOP + 32768;     // 2 x (KF|K~) MN-major 64 x 128
    static constexpr uint32_t TZP = COLOP + 32768;       // T' | Z | P0 | Z | P1 (8 KB each), K-major
    static constexpr uint32_t SCR = TZP + 40960;         // A, T fp32 [64][68] (also the S operand)
    static constexpr uint32_t SA = SCR;
    static constexpr uint32_t ST = SCR + 64 * kLDA * 4;
    static constexpr uint32_t SOP = SCR;                 //   S bf16, MN-major (K = dk) x DVT
    static constexpr uint32_t SMALL = SCR + 2 * 64 * kLDA * 4;
    static constexpr uint32_t SBETA = SMALL;             // 64 f32
    static constexpr uint32_t SOPS = SBETA + 256;        // 128 f32: operand scale per channel
    static constexpr uint32_t STMS = SOPS + 512;         // 128 f32: tensor-memory scale per channel
    static constexpr uint32_t SEK = STMS + 512;          // 128 f32: e^{G_last - G_m} of the last prepared chunk
    static constexpr uint32_t SEX = SEK + 512;           // 2 x 128 f32: G_m, G_last exchange
    static constexpr uint32_t BARS = SEX + 1024;         // 9 mbarriers
    static constexpr uint32_t MISC = BARS + 72;          // tmem base, abort flag
    static constexpr uint32_t END = MISC + 16;
    static constexpr uint32_t SMEM_BYTES = END + 1024;   // + alignment slack
    static constexpr uint32_t SBO_V = 1024 * (DVT / 64); // K-group stride of the S / delta operands
    static_assert(SOP + 128 * DVT * 2 <= SMALL, "S operand overflows the scratch");
    static_assert(DOP + 64 * DVT * 2 <= RAWV + DVT * 128, "delta operand overflows the v tile");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    // tensor memory columns
    static constexpr uint32_t S_COL = 0;                 // R (fp32, lane = key channel)
    static constexpr uint32_t D1_COL = DVT;              // 2 x DVT: U / delta / O accumulators
    static constexpr uint32_t G_COL = 3 * DVT;           // 64: cumulative gate of the chunk being prepared
    static constexpr uint32_t APW_COL = 3 * DVT + 64;    // 64: A (lanes 0-63) and P (lanes 64-127), then W'^T
    static constexpr uint32_t TMEM_COLS = 512;
};

__device__ __forceinline__ float ld_bf16(const uint8_t* base, uint32_t off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + off));
}

// offset of element (token r, channel c) in a [64 tok][128 ch] tile stored as
// two TMA boxes of [64][64] with the 128-byte swizzle
__device__ __forceinline__ uint32_t raw_off(int r, int c) {
    return (uint32_t)((c >> 6) * 8192 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1));
}

// byte offset of element (row r, col s) of a K-major swizzled 64-wide tile
__device__ __forceinline__ uint32_t km_off(int r, int s) {
    return (uint32_t)(r * 128 + ((((s >> 3) ^ (r & 7))) << 4) + ((s & 7) << 1));
}

// 1/x for normal positive x, accurate to ~2.4e-4 relative (enough for a bf16
// result): seed 2^-e (2 - f)/2 for x = 2^e (1 + f), obtained by subtracting
// the bit pattern from 254 << 23 (seed error <= 12.5%), then two Newton steps
// r <- r (2 - x r), each squaring the relative error. Runs on the FMA pipe.
__device__ __forceinline__ float recip_bf16(float x) {
    float r = __int_as_float(0x7F000000 - __float_as_int(x));
    r = r * fmaf(-x, r, 2.f);
    r = r * fmaf(-x, r, 2.f);
    return r;
}

// fp32 -> tf32 (round to nearest) for the warp-level MMAs of the UT inverse
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// acc += X Y restricted to columns [8*nt, 8*nt+8) of the 16x16 product; X and
// Y are 16x16 fp32 tiles (row stride kLDA) in shared memory, rounded to tf32
// (the resulting T' is stored as bf16, which dominates its rounding error).
// Fragment mapping of m16n8k8 (g = lane/4, t = lane%4): A (g|g+8, t|t+4),
// B (t|t+4, g), C (g|g+8, 2t|2t+1).
__device__ __forceinline__ void mm16_ntile(float (&acc)[4], const float* X, const float* Y, int nt, int lane) {
    const int g = lane >> 2, t = lane & 3;
    float part[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const uint32_t a[4] = {to_tf32(X[g * kLDA + 8 * ks + t]), to_tf32(X[(g + 8) * kLDA + 8 * ks + t]),
                               to_tf32(X[g * kLDA + 8 * ks + t + 4]), to_tf32(X[(g + 8) * kLDA + 8 * ks + t + 4])};
        const uint32_t bq[2] = {to_tf32(Y[(8 * ks + t) * kLDA + 8 * nt + g]),
                                to_tf32(Y[(8 * ks + t + 4) * kLDA + 8 * nt + g])};
        mma_tf32_16x8x8(part[ks], a, bq);  // two independent accumulators
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] += part[0][e] + part[1][e];
}

__device__ __forceinline__ void nb_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void nb_arrive(int id, int nthreads) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ bool nb_or(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

struct Bars {
    uint64_t *k, *q, *g, *v, *cs, *ap, *uw, *m1, *m2;
};

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
    // thread <-> tensor-memory lane: warp w reads lanes 32*(w%4).. and column half w/4
    const int quad = warp & 3, hf = warp >> 2;
    const int trow = 32 * quad + lane;
    constexpr int NJ = DVT / 2;

    float* sBeta = reinterpret_cast<float*>(sm + L::SBETA);
    float* sOpS = reinterpret_cast<float*>(sm + L::SOPS);
    float* sTmS = reinterpret_cast<float*>(sm + L::STMS);
    float* sEK = reinterpret_cast<float*>(sm + L::SEK);
    float* sEx = reinterpret_cast<float*>(sm + L::SEX);
    float* sA = reinterpret_cast<float*>(sm + L::SA);
    float* sT = reinterpret_cast<float*>(sm + L::ST);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BARS);
    const Bars bar{bars, bars + 1, bars + 2, bars + 3, bars + 4, bars + 5, bars + 6, bars + 7, bars + 8};
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + L::MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(sm + L::MISC + 4);
    volatile int* s_exact = reinterpret_cast<volatile int*>(sm + L::MISC + 8);  // guard verdict of the chunk being prepared

    // ---------------------------------------------------------------- setup
    if (tid == 0) {
        for (int i = 0; i < 9; ++i) mbar_init(bars + i, 1);
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
    {
        // T' (upper part stays zero), both zero blocks; L = lower-triangular ones
        uint4* z = reinterpret_cast<uint4*>(sm + L::TZP);
        for (int i = tid; i < 40960 / 16; i += kThreads) z[i] = make_uint4(0, 0, 0, 0);
        for (int e = tid; e < 64 * 8; e += kThreads) {
            const int r = e >> 3, ch = e & 7;
            uint32_t w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int s = 8 * ch + 2 * u;
                w[u] = (s <= r ? 0x3F80u : 0u) | ((s + 1 <= r) ? 0x3F800000u : 0u);
            }
            *reinterpret_cast<uint4*>(sm + L::LMAT + r * 128 + ((ch ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        for (int c = tid; c < kD; c += kThreads) sEK[c] = 1.f;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * quad) << 16);

    auto fail = [&]() {
        atomicExch(status, 1u);
        *s_abort = 1;
    };
    // Waits are executed by whole warps; __syncwarp reconverges the lanes
    // before the warp-collective instructions (tcgen05.ld, bar) that follow.
    auto wait_all = [&](uint64_t* bar_, int chunk) {  // compute warps; MMA results then readable
        if (!*s_abort && !mbar_wait_bounded(bar_, (uint32_t)chunk & 1u, kWaitBudget)) fail();
        __syncwarp();
        tc_fence_after();
    };
    auto wait_one = [&](uint64_t* bar_, int chunk) {  // control warp (before issuing dependent work)
        if (!*s_abort && !mbar_wait_bounded(bar_, (uint32_t)chunk & 1u, kWaitBudget)) fail();
        __syncwarp();
    };
    auto issue_k = [&](int n) {
        mbar_arrive_expect_tx(bar.k, 2 * 8192);
        for (int x = 0; x < 2; ++x) tma_load_4d(sm + L::RAWK + x * 8192, &tm_k, bar.k, 64 * x, h, n * kC, b);
    };
    auto issue_q = [&](int n) {
        mbar_arrive_expect_tx(bar.q, 2 * 8192);
        for (int x = 0; x < 2; ++x) tma_load_4d(sm + L::RAWQ + x * 8192, &tm_q, bar.q, 64 * x, h, n * kC, b);
    };
    auto issue_g = [&](int n) {
        mbar_arrive_expect_tx(bar.g, 2 * 8192);
        for (int x = 0; x < 2; ++x) tma_load_4d(sm + L::RAWG + x * 8192, &tm_g, bar.g, 64 * x, h, n * kC, b);
    };
    auto issue_v = [&](int n) {
        mbar_arrive_expect_tx(bar.v, (DVT / 64) * 8192);
        for (int x = 0; x < DVT / 64; ++x)
            tma_load_4d(sm + L::RAWV + x * 8192, &tm_v, bar.v, j0 + 64 * x, h, n * kC, b);
    };
    auto load_beta = [&](int n) -> float {
        const int t = n * kC + tid;
        return (tid < kC && n < NC && t < Tlen) ? __bfloat162float(beta[((size_t)b * Tlen + t) * H + h]) : 0.f;
    };

    constexpr uint32_t ID_CS = idesc_bf16(128, 64, 1, 0);
    constexpr uint32_t ID_AP = idesc_bf16(128, 64, 1, 1);
    constexpr uint32_t ID_U = idesc_bf16(128, DVT, 0, 1);
    constexpr uint32_t ID_WT = idesc_bf16(128, 64, 0, 0);
    constexpr uint32_t ID_M1 = idesc_bf16(128, DVT, 1, 1);
    constexpr uint32_t ID_M2 = idesc_bf16(128, DVT, 0, 1);

    // ---- MMA issue helpers (thread 0)
    auto mma_cumsum = [&]() {  // G^T[c][r] = sum_s la[s][c] * L[r][s]
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem + L::G_COL, sdesc_sw128(sb + L::RAWG + kk * 2048, 8192, 1024),
                        sdesc_sw128(sb + L::LMAT + kk * 32, 16, 1024), ID_CS, kk > 0);
        mma_commit(bar.cs);
    };
    auto mma_ap = [&](int m, bool exact) {  // [KE; QE] KF^T
        tc_fence_after();
        if (!exact) {
            const uint32_t col = sb + L::COLOP + (m & 1) * 16384;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16_ss(tmem + L::APW_COL, sdesc_sw128(sb + L::ROWOP + kk * 4096, 1024, 2048),
                            sdesc_sw128(col + kk * 2048, 1024, 1024), ID_AP, kk > 0);
        }
        mma_commit(bar.ap);
    };
    auto mma_uw = [&](int m) {  // U = [T'; 0] V into D1[m%2];  W'^T = KE^T T'^T (over A/P, already read)
        tc_fence_after();
        const uint32_t d1 = tmem + L::D1_COL + (m & 1) * DVT;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(d1, sdesc_sw128(sb + L::TZP + kk * 32, 16, 1024),
                        sdesc_sw128(sb + L::RAWV + kk * 2048, 8192, 1024), ID_U, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem + L::APW_COL, sdesc_sw128(sb + L::ROWOP + kk * 32, 16, 2048),
                        sdesc_sw128(sb + L::TZP + kk * 32, 16, 1024), ID_WT, kk > 0);
        mma_commit(bar.uw);
    };
    auto mma_1 = [&](int n) {  // D1[n%2] += [-W'; QE] (scaled S)
        tc_fence_after();
        const uint32_t d1 = tmem + L::D1_COL + (n & 1) * DVT;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ss(d1, sdesc_sw128(sb + L::ROWOP + kk * 4096, 1024, 2048),
                        sdesc_sw128(sb + L::SOP + kk * 2 * L::SBO_V, 1024, L::SBO_V), ID_M1, 1);
        mma_commit(bar.m1);
    };
    auto mma_2 = [&](int n) {  // R += KF^T delta ; D1[n%2] += [0; P] delta
        tc_fence_after();
        const uint32_t d1 = tmem + L::D1_COL + (n & 1) * DVT;
        const uint32_t col = sb + L::COLOP + (n & 1) * 16384;
        const uint32_t zp = sb + L::TZP + 8192 + (n & 1) * 16384;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem + L::S_COL, sdesc_sw128(col + kk * 32, 16, 1024),
                        sdesc_sw128(sb + L::DOP + kk * 2 * L::SBO_V, 1024, L::SBO_V), ID_M2, 1);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(d1, sdesc_sw128(zp + kk * 32, 16, 1024),
                        sdesc_sw128(sb + L::DOP + kk * 2 * L::SBO_V, 1024, L::SBO_V), ID_M2, 1);
        mma_commit(bar.m2);
    };

    // ---- P2 of chunk m (after its cumulative gate is in TMEM and its k, q tiles are in smem):
    // thread <-> (channel c = trow, token half hf). Computes the three operand
    // tiles into registers and the per-channel scales; returns the block-wide
    // guard verdict. In the exact case it also builds A and P.
    uint32_t opk[16], opq[16], opf[16];  // packed bf16 pairs along tokens
    auto p2_compute = [&](int m) -> bool {
        const int c = trow, r0 = 32 * hf;
        uint32_t gv[32];
        tmem_ld32(lane_addr + L::G_COL + 32 * hf, gv);
        tmem_ld_wait(gv);
        sEx[hf * 128 + c] = __uint_as_float(gv[31]);  // G_31 (hf = 0) / G_63 (hf = 1)
        tc_fence_before();
        nb_sync(NB_SIMT, kCompute);
        const float Gm = sEx[c], Gl = sEx[128 + c];
        float dev = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) dev = fmaxf(dev, fabsf(__uint_as_float(gv[i]) - Gm));
        const bool bad = !(dev <= kGuard) || !(Gm >= -kGuard);
        const bool exact = nb_or(NB_OR, kCompute, bad);
        if (hf == 0) {
            const float ek_prev = sEK[c];
            if (!exact) {
                const float s = __expf(Gm) * ek_prev;
                sOpS[c] = s;
                sTmS[c] = s;
                sEK[c] = __expf(Gl - Gm);
            } else {
                sOpS[c] = ek_prev;
                sTmS[c] = __expf(Gl) * ek_prev;
                sEK[c] = 1.f;
            }
        }
        if (exact) {
            // exact A and P with per-pair exponentials; G staged as fp32 in the
            // row-operand tile (free once MMA1 of the previous chunk completed)
            if (m > 0) wait_all(bar.m1, m - 1);
            float* sG = reinterpret_cast<float*>(sm + L::ROWOP);  // [64][128]
#pragma unroll
            for (int i = 0; i < 32; ++i) sG[(r0 + i) * 128 + c] = __uint_as_float(gv[i]);
            for (int i = tid; i < 64 * kLDA; i += kCompute) sA[i] = 0.f;
            uint4* pz = reinterpret_cast<uint4*>(sm + L::TZP + 16384 + (m & 1) * 16384);
            for (int i = tid; i < 8192 / 16; i += kCompute) pz[i] = make_uint4(0, 0, 0, 0);
            nb_sync(NB_SIMT, kCompute);
            uint8_t* pb = sm + L::TZP + 16384 + (m & 1) * 16384;
            for (int p = tid; p < kC * (kC + 1) / 2; p += kCompute) {
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
                *reinterpret_cast<__nv_bfloat16*>(pb + km_off(r, s)) = __float2bfloat16_rn(pp);
            }
        }
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
            const int r = r0 + i;
            const float k0 = ld_bf16(sm + L::RAWK, raw_off(r, c)), k1 = ld_bf16(sm + L::RAWK, raw_off(r + 1, c));
            const float q0 = ld_bf16(sm + L::RAWQ, raw_off(r, c)), q1 = ld_bf16(sm + L::RAWQ, raw_off(r + 1, c));
            const float g0 = __uint_as_float(gv[i]), g1 = __uint_as_float(gv[i + 1]);
            float e0, e1, f0, f1;
            if (!exact) {
                e0 = __expf(g0 - Gm); e1 = __expf(g1 - Gm);
                f0 = recip_bf16(e0); f1 = recip_bf16(e1);
            } else {
                e0 = __expf(g0); e1 = __expf(g1);
                f0 = __expf(Gl - g0); f1 = __expf(Gl - g1);
            }
            opk[i / 2] = pack_bf16x2(k0 * e0, k1 * e1);
            opq[i / 2] = pack_bf16x2(q0 * e0, q1 * e1);
            opf[i / 2] = pack_bf16x2(k0 * f0, k1 * f1);
        }
        return exact;
    };
    auto p2_store = [&](int m) {
        const int c = trow;
        const uint32_t col = sb + L::COLOP + (m & 1) * 16384;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t chunk = (uint32_t)((4 * hf + j) ^ (c & 7)) << 4;
            const uint32_t mn = (uint32_t)(c >> 3) * 2048 + (uint32_t)(c & 7) * 128 + chunk;
            st_shared_v4(sb + L::ROWOP + mn, opk[4 * j], opk[4 * j + 1], opk[4 * j + 2], opk[4 * j + 3]);
            st_shared_v4(sb + L::ROWOP + mn + 1024, opq[4 * j], opq[4 * j + 1], opq[4 * j + 2], opq[4 * j + 3]);
            st_shared_v4(col + (uint32_t)(c >> 3) * 1024 + (uint32_t)(c & 7) * 128 + chunk, opf[4 * j], opf[4 * j + 1],
                         opf[4 * j + 2], opf[4 * j + 3]);
        }
    };
    // ---- P4 of chunk m: A (lanes 0-63) -> fp32 scratch; P (lanes 64-127) -> bf16 operand
    auto p4 = [&](int m) {
        uint32_t v[32];
        tmem_ld32(lane_addr + L::APW_COL + 32 * hf, v);
        tmem_ld_wait(v);
        if (quad < 2) {
            const int r = trow;
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
            const int r = trow - 64;
            const uint32_t pbase = sb + L::TZP + 16384 + (m & 1) * 16384;
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
                st_shared_v4(pbase + r * 128 + ((((4 * hf + jc) ^ (r & 7))) << 4), w[0], w[1], w[2], w[3]);
            }
        }
    };
    // ---- P5: T = (I + A)^{-1}, written as T' = T Diag(beta) in bf16
    auto store_tprime = [&](int r, int s, float t) {
        *reinterpret_cast<__nv_bfloat16*>(sm + L::TZP + km_off(r, s)) = __float2bfloat16_rn(t * sBeta[s]);
    };
    auto p5 = [&]() {
        {   // diagonal 16x16 blocks: four threads per column, rows q, q+4, q+8, q+12
            const int a = tid >> 6, jc = (tid >> 2) & 15, q = tid & 3;
            const float* Ab = sA + (16 * a) * kLDA + 16 * a;
            float acc[4] = {0.f, 0.f, 0.f, 0.f}, colv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const float mine = (r == jc) ? 1.f : ((r > jc) ? -acc[r >> 2] : 0.f);
                const float t = __shfl_sync(0xffffffffu, mine, (lane & ~3) | (r & 3));
                if (q == (r & 3)) colv[r >> 2] = t;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (q + 4 * i > r) acc[i] = fmaf(Ab[(q + 4 * i) * kLDA + r], t, acc[i]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = 16 * a + q + 4 * i, s = 16 * a + jc;
                sT[r * kLDA + s] = colv[i];
                store_tprime(r, s, colv[i]);
            }
        }
        nb_sync(NB_SIMT, kCompute);
        // Blocks below the diagonal on the tensor cores (m16n8k8, tf32): one
        // warp per (block, 8-column half). N_ak = T_aa A_ak replaces A_ak.
        auto put_t = [&](int a, int bb, int nt, const float (&acc)[4]) {  // T_ab = -acc
            const int g = lane >> 2, t = lane & 3;
            const int s = 16 * bb + 8 * nt + 2 * t;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = 16 * a + g + 8 * hh;
                const float v0 = -acc[2 * hh], v1 = -acc[2 * hh + 1];
                *reinterpret_cast<float2*>(sT + r * kLDA + s) = make_float2(v0, v1);
                *reinterpret_cast<uint32_t*>(sm + L::TZP + km_off(r, s)) =
                    pack_bf16x2(v0 * sBeta[s], v1 * sBeta[s + 1]);
            }
        };
        for (int task = warp; task < 12; task += kCompute / 32) {
            const int blk = task >> 1, nt = task & 1;
            const int a = (blk == 0) ? 1 : (blk <= 2 ? 2 : 3);
            const int k = (blk == 0) ? 0 : (blk == 1 ? 0 : (blk == 2 ? 1 : blk - 3));
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            mm16_ntile(acc, sT + (16 * a) * kLDA + 16 * a, sA + (16 * a) * kLDA + 16 * k, nt, lane);
            __syncwarp();
            const int g = lane >> 2, t = lane & 3;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                *reinterpret_cast<float2*>(sA + (16 * a + g + 8 * hh) * kLDA + 16 * k + 8 * nt + 2 * t) =
                    make_float2(acc[2 * hh], acc[2 * hh + 1]);
        }
        nb_sync(NB_SIMT, kCompute);
        // level d: T_ab = -sum_{k=b}^{a-1} N_ak T_kb, a - b = d
#pragma unroll 1
        for (int d = 1; d < 4; ++d) {
            if (warp < 2 * (4 - d)) {
                const int bb = warp >> 1, nt = warp & 1, a = bb + d;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                for (int kb = bb; kb < a; ++kb)
                    mm16_ntile(acc, sA + (16 * a) * kLDA + 16 * kb, sT + (16 * kb) * kLDA + 16 * bb, nt, lane);
                put_t(a, bb, nt, acc);
            }
            nb_sync(NB_SIMT, kCompute);
        }
    };
    // ---- P7 of chunk m: -W' (W'^T in TMEM, lane c, columns r) -> rows 0-63 of the row operand
    auto p7 = [&]() {
        const int cc = trow;
        uint32_t v[32];
        tmem_ld32(lane_addr + L::APW_COL + 32 * hf, v);
        tmem_ld_wait(v);
#pragma unroll
        for (int jc = 0; jc < 4; ++jc) {
            uint32_t w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                w[u] = pack_bf16x2(-__uint_as_float(v[8 * jc + 2 * u]), -__uint_as_float(v[8 * jc + 2 * u + 1]));
            const uint32_t off = (uint32_t)(cc >> 3) * 2048 + (uint32_t)(cc & 7) * 128 +
                                 ((uint32_t)((4 * hf + jc) ^ (cc & 7)) << 4);
            st_shared_v4(sb + L::ROWOP + off, w[0], w[1], w[2], w[3]);
        }
    };
    // ---- S1 of chunk n: R -> bf16 operand (times the operand scale); R *= tensor-memory scale
    auto s1 = [&]() {
        const int cc = trow;
        const float os = sOpS[cc], ts = sTmS[cc];
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
                    w[u] = pack_bf16x2(__uint_as_float(v[8 * jc + 2 * u]) * os, __uint_as_float(v[8 * jc + 2 * u + 1]) * os);
                const int j = jb + 8 * jc;
                const uint32_t off = (uint32_t)(cc >> 3) * L::SBO_V + (uint32_t)(j >> 6) * 1024 +
                                     (uint32_t)(cc & 7) * 128 + ((uint32_t)(((j & 63) >> 3) ^ (cc & 7)) << 4);
                st_shared_v4(sb + L::SOP + off, w[0], w[1], w[2], w[3]);
            }
#pragma unroll
            for (int u = 0; u < 32; ++u) v[u] = __float_as_uint(__uint_as_float(v[u]) * ts);
            tmem_st32(lane_addr + L::S_COL + jb, v);
        }
        tmem_st_wait();
    };
    // ---- S3 of chunk n: delta (D1 lanes 0-63) -> bf16 operand, MN-major (K = token)
    auto s3 = [&](int n) {
        if (quad < 2) {
            const int r = trow;
            const uint32_t d1 = L::D1_COL + (n & 1) * DVT;
#pragma unroll
            for (int gq = 0; gq < NJ / 32; ++gq) {
                const int jb = hf * NJ + 32 * gq;
                uint32_t v[32];
                tmem_ld32(lane_addr + d1 + jb, v);
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
    };
    // ---- S5 of chunk n: O (D1 lanes 64-127) -> global bf16
    auto s5 = [&](int n) {
        if (quad >= 2) {
            const int r = trow - 64;
            const int t0 = n * kC;
            const uint32_t d1 = L::D1_COL + (n & 1) * DVT;
#pragma unroll
            for (int gq = 0; gq < NJ / 32; ++gq) {
                const int jb = hf * NJ + 32 * gq;
                uint32_t v[32];
                tmem_ld32(lane_addr + d1 + jb, v);
                tmem_ld_wait(v);
                if (t0 + r < Tlen) {
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
                __syncwarp();  // (ragged tail) reconverge before the next tcgen05.ld
            }
        }
    };
    // compute warps: operands written -> visible to the control warp's next MMA
    auto signal = [&](int id) {
        fence_proxy_async_smem();
        tc_fence_before();
        nb_arrive(id, kThreads);
    };

    if (warp == kCtrlWarp) {
        // ============================================================ control warp
        // Issues every TMA load and MMA (lane 0), in the order the compute
        // warps signal that operands are ready. Never blocks the compute warps.
        const bool leader = lane == 0;
        if (NC > 0) {
            if (leader) {
                issue_k(0);
                issue_q(0);
                issue_g(0);
                issue_v(0);
            }
            __syncwarp();
            wait_one(bar.g, 0);
            if (leader) mma_cumsum();
            __syncwarp();
            wait_one(bar.cs, 0);
            if (leader && NC > 1) issue_g(1);       // log_alpha tile consumed
            __syncwarp();
            nb_sync(NB_K, kThreads);                 // gate and k, q tiles of chunk 0 read
            if (leader && NC > 1) {
                issue_k(1);
                issue_q(1);
            }
            __syncwarp();
            nb_sync(NB_S3, kThreads);                // operands of chunk 0 stored
            if (leader) mma_ap(0, *s_exact != 0);
            __syncwarp();
            if (NC > 1) {                            // gate of chunk 1, ready long before it is needed
                wait_one(bar.g, 1);
                if (leader) mma_cumsum();
                __syncwarp();
            }
            nb_sync(NB_P5, kThreads);                // T' of chunk 0 stored
            wait_one(bar.v, 0);
            if (leader) mma_uw(0);
            __syncwarp();
        }
        for (int n = 0; n < NC; ++n) {
            const bool more = n + 1 < NC;
            if (__syncthreads_or(*s_abort)) break;
            nb_sync(NB_S1, kThreads);                // state operand of chunk n stored
            if (leader) mma_1(n);
            __syncwarp();
            if (more) {
                wait_one(bar.cs, n + 1);             // (issued one iteration earlier)
                if (leader && n + 2 < NC) issue_g(n + 2);  // log_alpha tile consumed
                __syncwarp();
                nb_sync(NB_K, kThreads);             // gate and k, q tiles of chunk n+1 read
                if (leader && n + 2 < NC) {
                    issue_k(n + 2);
                    issue_q(n + 2);
                }
                __syncwarp();
            }
            nb_sync(NB_S3, kThreads);                // delta(n) and operands of chunk n+1 stored
            if (leader) {
                if (more) mma_ap(n + 1, *s_exact != 0);
                mma_2(n);
            }
            __syncwarp();
            if (n + 2 < NC) {                        // gate of chunk n+2 (the gate TMEM columns are free)
                wait_one(bar.g, n + 2);
                if (leader) mma_cumsum();
                __syncwarp();
            }
            wait_one(bar.m2, n);
            if (leader && more) issue_v(n + 1);      // delta operand (on the v tile) consumed
            __syncwarp();
            if (more) {
                nb_sync(NB_P5, kThreads);            // T' of chunk n+1 stored
                wait_one(bar.v, n + 1);
                if (leader) mma_uw(n + 1);
                __syncwarp();
            }
        }
        __syncthreads();
    } else {
        // ============================================================ compute warps
        {   // initial state into TMEM (fp32, lane = key channel)
            const int c = trow;
#pragma unroll
            for (int gq = 0; gq < NJ / 32; ++gq) {
                uint32_t r[32];
                const int jb = hf * NJ + 32 * gq;
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
        float beta_next = 0.f;
        if (NC > 0) {
            if (tid < kC) sBeta[tid] = load_beta(0);
            beta_next = load_beta(1);
            wait_all(bar.cs, 0);
            wait_all(bar.k, 0);
            wait_all(bar.q, 0);
            nb_sync(NB_SIMT, kCompute);  // sBeta visible
            const bool exact0 = p2_compute(0);
            if (tid == 0) *s_exact = exact0;
            __syncwarp();
            nb_sync(NB_SIMT, kCompute);  // (exact path) staged gate values read before the tiles are overwritten
            nb_arrive(NB_K, kThreads);
            p2_store(0);
            signal(NB_S3);
            wait_all(bar.ap, 0);
            if (!exact0) p4(0);
            nb_sync(NB_SIMT, kCompute);
            p5();
            signal(NB_P5);
            wait_all(bar.uw, 0);
            p7();
        }
        for (int n = 0; n < NC; ++n) {
            const bool more = n + 1 < NC;
            tc_fence_before();
            if (__syncthreads_or(*s_abort)) break;
            s1();
            signal(NB_S1);
            bool exact_next = false;
            if (more) {
                if (tid < kC) sBeta[tid] = beta_next;
                beta_next = load_beta(n + 2);
                wait_all(bar.cs, n + 1);
                wait_all(bar.k, n + 1);
                wait_all(bar.q, n + 1);
                nb_sync(NB_SIMT, kCompute);  // sBeta(n+1) visible
                exact_next = p2_compute(n + 1);
                if (tid == 0) *s_exact = exact_next;
                __syncwarp();
                nb_sync(NB_SIMT, kCompute);  // k, q tiles (and the exact path's staged gate) read
                nb_arrive(NB_K, kThreads);
            }
            wait_all(bar.m1, n);
            s3(n);
            if (more) p2_store(n + 1);
            signal(NB_S3);
            if (more) {
                wait_all(bar.ap, n + 1);
                if (!exact_next) p4(n + 1);
                nb_sync(NB_SIMT, kCompute);
                p5();
                signal(NB_P5);
            }
            wait_all(bar.m2, n);
            s5(n);
            if (more) {
                wait_all(bar.uw, n + 1);
                p7();
            }
        }
        // ------------------------------------------------------------ final state S = e^{G_last - G_m} R
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (ST && !*s_abort) {
            const int c = trow;
            const float ek = sEK[c];
#pragma unroll
            for (int gq = 0; gq < NJ / 32; ++gq) {
                const int jb = hf * NJ + 32 * gq;
                uint32_t v[32];
                tmem_ld32(lane_addr + L::S_COL + jb, v);
                tmem_ld_wait(v);
                float4* dst = reinterpret_cast<float4*>(ST + ((size_t)bh * kD + c) * kD + j0 + jb);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    dst[u] = make_float4(__uint_as_float(v[4 * u]) * ek, __uint_as_float(v[4 * u + 1]) * ek,
                                         __uint_as_float(v[4 * u + 2]) * ek, __uint_as_float(v[4 * u + 3]) * ek);
            }
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
