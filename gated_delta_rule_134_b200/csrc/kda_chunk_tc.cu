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
// Reference-point factorisation. G_r is counted from the chunk's entry, so
// with E_r = e^{G_r} and F_r = e^{-G_r} (per channel):
//   e^{G_r - G_s} = E_r F_s,  k e^G = k E,  k e^{G_last-G} = (k F) e^{G_last}.
// Three bf16 tiles, KE = k E, QE = q E and KF = k F, feed every MMA. The
// output is regrouped so that P never meets the state: with PT = P T',
//   O = QE S + P (U - W' S) = (QE - P W') S + P T' v,   W' = T' KE,
// so per chunk the state-independent MMAs are
//   G = [L; L] g                  -> gate prefix sums (L: lower-triangular ones)
//   [A; P] = [KE; QE] KF^T        (one M=128 MMA)
//   PT = P T'
//   [W'; P W'] = [T'; PT] KE      -> row operand [-W'; QE - P W']
//   [U; P T' v] = [T'; PT] v      -> the chunk's accumulator
// and the state chain needs only two:
//   D += [-W'; QE - P W'] S       -> rows 0-63: delta, rows 64-127: O
//   R  = S + KF^T delta           -> S_next = Diag(e^{G_last}) R
// The tensor memory holds R; the per-channel factor e^{G_last} is applied
// lazily, when the next chunk copies the state into the bf16 MMA operand (and
// when the final state is written). Each factor is a single exponential,
// finite as long as |G_r| <= 80; a vote of the tile warps checks that per
// chunk. A chunk that fails it tries the reference point G_m = G_last / 2
// (E = e^{G - G_m}, F = e^{G_m - G}, the state operand e^{G_m} S), which holds
// while |G_r - G_m| <= 80, i.e. a decay of up to 160 over the chunk: the raw
// k/q rows are reloaded and the tiles rebuilt. A chunk that fails that too
// uses exact per-pair exponentials e^{G_r - G_s} (exponent <= 0) for A and P
// and the plain tiles k e^G, q e^G, k e^{G_last-G}; the same MMAs then produce
// the same quantities.
//
// Schedule. One CTA owns one (batch, head) and a DVT-wide slice of value
// channels; its state stays in tensor memory for the whole sequence. Each
// chunk m lives in one of three tensor-memory slots (m mod 3) from its prefix
// sums to its output, so the state-independent work of chunks m+1 and m+2
// runs while the chain works on chunk m. Three warp groups hand work over
// through mbarriers:
//   chain (warps 0-3)   state -> bf16 operand (one channel row per thread);
//                       the U MMA that starts the chunk's accumulator, then
//                       MMA1 over all 128 key channels, delta -> bf16, MMA2,
//                       O -> global; it also issues the TMA loads of k/q and
//                       log_alpha into the buffers its MMAs free.
//   tile  (warps 4-7)   prefix sums out of tensor memory, KE/QE in place over
//                       the raw k/q rows, KF over the log_alpha tile, the
//                       overflow vote, per-channel scales; issues the [A; P]
//                       MMA, reads A (beta-scaled, fp32) and P (bf16) out of
//                       tensor memory, then issues the next chunk's prefix-sum
//                       MMA.
//   inverse (warps 8-15) (I + A)^{-1} -> T', the PT and W MMAs and their
//                       readouts into the row operand; issues the v loads and
//                       stores beta a chunk ahead.
// k/q tiles are double-buffered, the log_alpha/KF tiles triple-buffered, the
// per-channel scales kept by chunk mod 3. The A scratch of the inverse is fp16
// (the tf32 MMAs of the inverse read it through the same 10-bit mantissa).
// (I + A)^{-1}: 16x16 diagonal blocks by forward substitution (four threads per
// column), then one column chain per warp, T_ab = -T_aa sum_k A_ak T_kb, on
// m16n8k8 tf32 MMAs; T' = T Diag(beta) is written as bf16 by the thread that
// finalises each entry.
//
// Every wait on an mbarrier is bounded; on expiry the kernel records status 1
// in the caller's workspace word and stops waiting (later waits are skipped,
// so every role reaches the end), waits for its copies and MMAs in flight,
// frees its tensor memory and returns.
#include <algorithm>
#include <type_traits>

#include <cuda_fp16.h>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_sm100.cuh"

namespace kda {

using namespace sm100;

namespace {

constexpr int kTileWarp0 = 4;   // warps 0-3: chain; 4-7: tiles; 8-15: inverse and W/U side
constexpr int kInvWarp0 = 8;
constexpr int kThreads = 512;
// named barriers (0 is __syncthreads)
constexpr int NB_TILE = 1;  // tile warps
constexpr int NB_TOR = 2;   // tile warps, OR-vote
constexpr int NB_INV = 3;   // inverse warps
constexpr int NB_CHLO = 4;  // chain warps 0-1
constexpr int NB_CHHI = 6;  // chain warps 2-3
constexpr int NB_CH = 7;    // all chain warps
constexpr int kC = 64;    // chunk
constexpr int kD = 128;   // dk = dv
constexpr int kLDA = 72;  // fp16 row stride of the A scratch (16-byte rows, bank spread)
constexpr int kLDT = 20;  // fp32 row stride of the diagonal blocks of T (bank spread)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kGuardL = 80.f * kLog2e;      // |G_r| <= 80, in log2 units
constexpr long long kWaitBudget = 1ll << 31;  // SM cycles (~1 s)
constexpr long long kDrainBudget = 1ll << 24;

template <int DVT>
struct Layout {
    // shared memory, bytes from a 1024-aligned base
    static constexpr uint32_t ROW = 0;          // 2 x 32 KB, K-major: per 64-channel box x (x * 16 KB)
                                                //   rows 0-63: k -> KE -> -W', rows 64-127: q -> QE -> QE - P W'
    static constexpr uint32_t COL = 65536;      // 3 x 16 KB: log_alpha tile, then KF (box x at x * 8 KB)
    static constexpr uint32_t RAWV = 114688;    // v slice: DVT/64 boxes of [64 tok][64 ch]
    static constexpr uint32_t LMAT = 131072;    // [L; L] K-major 128 x 64
    static constexpr uint32_t TP = 147456;      // [T'; PT] K-major 128 x 64
    static constexpr uint32_t SP = TP + 16384;  // P, K-major 64 x 64 bf16 (rows 64-127 of [Y; P], Y = TP rows 64-127)
    static constexpr uint32_t SOP = SP + 8192;  // S (128 channels) x DVT, bf16 MN-major, then delta (64 tokens)
    static constexpr uint32_t OST = SOP + 128 * DVT * 2;  // 2 x [32 tok][32 ch] bf16 (64-byte swizzle): O stores
    static constexpr uint32_t SCR = OST + 4096;          // A fp16 [64][kLDA], T diagonal blocks fp32 [4][16][kLDT]
    static constexpr uint32_t SA = SCR;                  //   (exact path: 8 KB fp32 staging)
    static constexpr uint32_t STD = SCR + 64 * kLDA * 2;
    static constexpr uint32_t SCR_BYTES = 64 * kLDA * 2 + 4 * 16 * kLDT * 4;
    static constexpr uint32_t SMALL = SCR + SCR_BYTES;
    static constexpr uint32_t SBETA = SMALL;        // 2 x 64 f32: beta of the chunk (by parity)
    static constexpr uint32_t SOPS = SBETA + 512;   // 3 x 128 f32: operand scale per channel (by chunk mod 3)
    static constexpr uint32_t STMS = SOPS + 1536;   // 3 x 128 f32: tensor-memory scale per channel
    static constexpr uint32_t SMDS = STMS + 1536;   // 3 x 128 f32: second factor of both (middle tier, else 1)
    static constexpr uint32_t SEK = SMDS + 1536;    // 128 f32: pending state factor after the last prepared chunk
    static constexpr uint32_t SGL = SEK + 512;      // 128 f32: G_last
    static constexpr uint32_t BARS = SGL + 512;     // mbarriers
    static constexpr uint32_t MISC = BARS + 512;    // tmem base, abort flag, copies issued, wait budget
    static constexpr uint32_t END = MISC + 64;
    static constexpr uint32_t SMEM_BYTES = END + 1024;   // + alignment slack
    static constexpr uint32_t SBO_V = 1024 * (DVT / 64); // K-group stride of the S / delta operands
    static_assert(SOP % 1024 == 0 && TP % 1024 == 0 && LMAT % 1024 == 0 && OST % 1024 == 0, "operand alignment");
    static_assert(32 * 64 * 4 <= SCR_BYTES, "exact-path staging overflows the scratch");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    // tensor memory columns: R (fp32, lane = key channel) and three chunk slots
    static constexpr uint32_t S_COL = 0;
    static constexpr uint32_t SLOT0 = 128;
    static constexpr uint32_t TMEM_COLS = 512;
};

// mbarrier slots
enum : int {
    B_KQ = 0,     // 2: k/q tiles landed (by chunk parity)
    B_G = 2,      // 3: log_alpha tile (or per-token gate row) of the chunk (mod 3) in place
    B_V = 5,      // v tile landed
    B_CS = 6,     // 3: prefix-sum MMA of the slot's chunk done
    B_AP = 9,     // 3: [A; P] of the slot's chunk in tensor memory
    B_PT = 12,    // PT MMA done
    B_WB = 13,    // [W'; P W'] MMA done
    B_UO = 14,    // 3: [U; P T' v] MMA of the slot's chunk done (also frees [T'; PT] and the v tile)
    B_RR = 17,    // 2: row operand [-W'; QE - P W'] of the chunk of this parity stored
    B_SC = 19,    // 3 (of 4): per-channel scales of the chunk (mod 3) stored
    B_M1A = 23,   // (unused)
    B_M1 = 24,    // MMA1 done (row operand free)
    B_M2 = 25,    // MMA2 done (KF and delta operand free, R updated)
    B_SF = 28,    // 3: the slot's chunk read out by the chain (count 2)
    B_SCRF = 31,  // A/T scratch of the inverse warps' chunk free
    B_EXKQ = 32,  // k/q reloaded for an exact chunk
    B_FIN = 33,   // 3: final drain of each MMA-issuing thread
    B_AR = 36,    // A (fp32 scratch) and P (bf16 tile) of the chunk read out of tensor memory
    NUM_BARS = 37
};

// offset of element (row R, channel c) of a row-operand buffer (K-major, two
// 64-channel boxes of 128 rows, 128-byte swizzle)
__device__ __forceinline__ uint32_t rop_off(int R, int c) {
    return (uint32_t)((c >> 6) * 16384 + R * 128 + ((((c & 63) >> 3) ^ (R & 7)) << 4) + ((c & 7) << 1));
}

// byte offset of element (row r, col s) of a K-major swizzled 64-wide tile
__device__ __forceinline__ uint32_t km_off(int r, int s) {
    return (uint32_t)(r * 128 + ((((s >> 3) ^ (r & 7))) << 4) + ((s & 7) << 1));
}

// 2^x by the hardware approximation (one MUFU operation)
__device__ __forceinline__ float ex2(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
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

__device__ __forceinline__ void nb_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
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

// 32 lanes x 1 column (the x1 form of tmem_ld32)
__device__ __forceinline__ void tmem_ld1(uint32_t taddr, uint32_t& r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait1(uint32_t& r) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(r) : : "memory");
}

// Chunk-parallel scan over segments of each sequence (few heads, long T).
// The update is affine in the state, so a segment maps its entry state S_in
// to M S_in + C. Phase 1 runs segment 0 in full and, for each middle segment
// j = 1..P-2, its transition M_j (entry state I, v = 0) and offset C_j (entry
// state 0); a scan then chains S_in of segments 1..P-1; phase 3 runs those
// segments in full from their entry states. P = 0: whole sequences.
struct SegJobs {
    int P;       // segments per sequence (0: no scan)
    int L;       // tokens per segment, a multiple of the chunk
    int phase;   // 1 or 3
    float* M;    // [B*H][P-2][dk][dv]
    float* C;    // [B*H][P-2][dk][dv]
    float* Sin;  // [B*H][P-1][dk][dv]: state entering segment j at [j-1]
    // Fault injection for the timeout test only (zero in every other launch):
    // withhold the first k/q load, and give every wait this budget in SM cycles.
    int withhold_first_load;
    long long wait_budget;
};

// ERASE: 1 delta-rule family, 0 additive write. GATE: 0 per-channel log_alpha,
// 1 one per token and head, 2 none. Compile-time, so each variant is its own
// kernel and the KDA instance carries no variant branches.
template <int DVT, int ERASE, int GATE>
__global__ void __launch_bounds__(kThreads, 1)
kda_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_o, const __nv_bfloat16* __restrict__ beta, const float* S0, __nv_bfloat16* __restrict__ o,
                    float* ST, int Tlen, int H, unsigned* status, const __nv_bfloat16* __restrict__ gate_tok,
                    const int* __restrict__ cu_seqlens, const SegJobs sj) {
    constexpr int erase = ERASE;
    using L = Layout<DVT>;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base (the 128-byte swizzle repeats every 1024 bytes);
    // offsetting the array itself keeps the pointer in the shared window, so
    // accesses through it compile to shared-memory instructions
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(sm);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3;  // tensor-memory lane quadrant this warp may access
    const int nslices = kD / DVT;
    const int unit = blockIdx.x / nslices;  // the (sequence-head, piece) of this CTA
    const int per = sj.P == 0 ? 1 : (sj.phase == 1 ? 2 * sj.P - 3 : sj.P - 1);
    const int bh = unit / per, piece = unit % per;
    const int b = bh / H, h = bh % H;
    constexpr size_t kMat = (size_t)kD * kD;
    // This piece's tokens: [tok0, tok0 + seq_len) of the token-major layout.
    // Dense batch: sequence b of [B, T]; packed: offsets clamped into [0, T], and
    // the tensor maps then describe one [1, T] sequence (tile origin tma_t0).
    size_t tok0;
    int seq_len, tma_t0, tma_b;
    const float* s0m = S0 ? S0 + bh * kMat : nullptr;  // entry state [dk][dv] (NULL: zero)
    float* stm = ST ? ST + bh * kMat : nullptr;        // final state destination (NULL: none)
    bool s0_ident = false, v_zero = false, o_on = true;
    if (cu_seqlens) {
        const int s0 = min(max(cu_seqlens[b], 0), Tlen), s1 = min(max(cu_seqlens[b + 1], s0), Tlen);
        tok0 = (size_t)s0;
        seq_len = s1 - s0;
        tma_t0 = s0;
        tma_b = 0;
    } else {
        tok0 = (size_t)b * Tlen;
        seq_len = Tlen;
        tma_t0 = 0;
        tma_b = b;
        if (sj.P > 0) {
            // phase 1: piece 0 = segment 0 in full, then (M_j, C_j) pairs; phase 3: segments 1..P-1
            const int j = sj.phase == 3 ? piece + 1 : (piece == 0 ? 0 : 1 + (piece - 1) / 2);
            const int t_begin = j * sj.L;
            seq_len = max(0, min(sj.L, Tlen - t_begin));
            tok0 += (size_t)t_begin;
            tma_t0 = t_begin;
            if (sj.phase == 3) {
                s0m = sj.Sin + ((size_t)bh * (sj.P - 1) + (j - 1)) * kMat;
                if (j != sj.P - 1) stm = nullptr;
            } else if (piece == 0) {
                stm = sj.Sin + (size_t)bh * (sj.P - 1) * kMat;
            } else {
                const size_t off = ((size_t)bh * (sj.P - 2) + (j - 1)) * kMat;
                const bool is_m = ((piece - 1) & 1) == 0;
                o_on = false;
                s0m = nullptr;
                s0_ident = is_m;
                v_zero = is_m;
                stm = (is_m ? sj.M : sj.C) + off;
            }
        }
    }
    const int j0 = (blockIdx.x % nslices) * DVT;
    const int NC = (seq_len + kC - 1) / kC;

    float* sBeta = reinterpret_cast<float*>(sm + L::SBETA);
    float* sOpS = reinterpret_cast<float*>(sm + L::SOPS);
    float* sTmS = reinterpret_cast<float*>(sm + L::STMS);
    float* sMdS = reinterpret_cast<float*>(sm + L::SMDS);
    float* sEK = reinterpret_cast<float*>(sm + L::SEK);
    float* sGl = reinterpret_cast<float*>(sm + L::SGL);
    __half* sA = reinterpret_cast<__half*>(sm + L::SA);
    float* sTd = reinterpret_cast<float*>(sm + L::STD);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BARS);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + L::MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(sm + L::MISC + 4);
    // Copies issued so far, for the final drain after an abort: the last chunk
    // whose k/q, log_alpha and v tiles were loaded (-1: none; each kind is loaded
    // in chunk order), and the number of exact-path k/q reloads.
    int* s_issued = reinterpret_cast<int*>(sm + L::MISC + 8);
    // SM cycles a wait may take before it gives up (read only when a wait blocks)
    volatile long long* s_budget = reinterpret_cast<volatile long long*>(sm + L::MISC + 40);

    // ---------------------------------------------------------------- setup
    if (tid == 0) {
        for (int i = 0; i < NUM_BARS; ++i) mbar_init(bars + i, (i >= B_SF && i < B_SF + 3) ? 2u : 1u);
        *s_abort = 0;
        s_issued[0] = s_issued[1] = s_issued[2] = -1;
        s_issued[3] = 0;
        *s_budget = sj.wait_budget > 0 ? sj.wait_budget : kWaitBudget;
        fence_mbar_init();
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_g);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_o);
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, L::TMEM_COLS);
        tmem_relinquish();
    }
    {   // constants: [L; L] (row R: ones in columns 0..R%64) and the T' half of
        // [T'; PT], whose blocks above the diagonal are never written again
        for (int i = tid; i < 128 * 8; i += kThreads) {
            const int R = i >> 3, j = i & 7, r = R & 63;
            uint32_t w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int s = 8 * j + 2 * u;
                w[u] = pack_bf16x2(s <= r ? 1.f : 0.f, s + 1 <= r ? 1.f : 0.f);
            }
            st_shared_v4(sb + L::LMAT + R * 128 + ((j ^ (R & 7)) << 4), w[0], w[1], w[2], w[3]);
            if (R < 64) st_shared_v4(sb + L::TP + R * 128 + (j << 4), 0u, 0u, 0u, 0u);
        }
        for (int c = tid; c < kD; c += kThreads) sEK[c] = 1.f;
        if (v_zero)  // transition run: v = 0 stays in the v tile, which is never loaded
            for (int i = tid; i < (DVT / 64) * 8192 / 16; i += kThreads) st_shared_v4(sb + L::RAWV + 16 * i, 0u, 0u, 0u, 0u);
    }
    if (tid < kC)  // beta of chunk 0 (later chunks: the inverse warps, a chunk ahead)
        sBeta[tid] = tid < seq_len ? __bfloat162float(beta[(tok0 + tid) * H + h]) : 0.f;
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
    // Bounded wait by one thread; after a timeout every later wait is skipped.
    // True when the phase completed and no thread had aborted by then (a copy
    // issued on that condition cannot race a phase another wait skipped).
    auto wait1 = [&](int slot, uint32_t parity) -> bool {
        if (*s_abort) return false;
        if (mbar_wait_bounded(bars + slot, parity & 1u, s_budget)) return !*s_abort;
        fail();
        return false;
    };
    // Bounded wait by a whole warp, then reconverge; MMA results readable after.
    auto waitw = [&](int slot, uint32_t parity) -> bool {
        const bool ok = wait1(slot, parity);
        __syncwarp();
        tc_fence_after();
        return ok;
    };

    constexpr uint32_t ID_CS = idesc_bf16(128, 128, 0, 1);   // [L; L] x g (MN-major)
    constexpr uint32_t ID_CS1 = idesc_bf16(128, 16, 0, 0);   // [L; L] x per-token gate row (K-major)
    constexpr uint32_t ID_AP = idesc_bf16(128, 64, 0, 0);
    constexpr uint32_t ID_PT = idesc_bf16(128, 64, 0, 1);    // [Y; P] x T' (MN-major)
    constexpr uint32_t ID_W = idesc_bf16(128, 128, 0, 1);
    constexpr uint32_t ID_U = idesc_bf16(128, DVT, 0, 1);
    constexpr uint32_t ID_M1 = idesc_bf16(128, DVT, 0, 1);
    constexpr uint32_t ID_M2 = idesc_bf16(128, DVT, 1, 1);
    // Shared-memory descriptors, built once: the address field holds addr >> 4,
    // so an offset of x bytes inside a tile is a plain add of x >> 4.
    auto dadd = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
    const uint64_t dLMAT = sdesc_sw128(sb + L::LMAT, 16, 1024);          // K-major A
    const uint64_t dTP = sdesc_sw128(sb + L::TP, 16, 1024);              // [T'; PT] as K-major A
    const uint64_t dTPN = sdesc_sw128(sb + L::TP, 8192, 1024);           // T' as MN-major B
    const uint64_t dYP = sdesc_sw128(sb + L::SP - 8192, 16, 1024);       // [Y; P] as K-major A
    const uint64_t dROWK = sdesc_sw128(sb + L::ROW, 16, 1024);           // row operand as K-major A
    const uint64_t dROWN = sdesc_sw128(sb + L::ROW, 16384, 1024);        // its KE rows as MN-major B
    const uint64_t dCOLK = sdesc_sw128(sb + L::COL, 16, 1024);           // KF / gate row as K-major B
    const uint64_t dCOLN = sdesc_sw128(sb + L::COL, 8192, 1024);         // g as MN-major B, KF^T as MN-major A
    const uint64_t dV = sdesc_sw128(sb + L::RAWV, 8192, 1024);           // MN-major B
    const uint64_t dSOP = sdesc_sw128(sb + L::SOP, 1024, L::SBO_V);      // MN-major B (S, then delta)

    // TMA issue helpers (one thread). A copy that reuses a barrier is issued only
    // after a wait that completed for real (not one skipped after an abort):
    // arming a barrier again while its previous phase still waits for bytes
    // would over-arrive on that phase.
    auto load_kq = [&](int m, int bar) {  // k/q tiles of chunk m into the row buffer of its parity
        uint8_t* dst = sm + L::ROW + (m & 1) * 32768;
        if (bar == B_EXKQ) ++s_issued[3];
        else s_issued[0] = m;
        mbar_arrive_expect_tx(bars + bar, 4 * 8192);
        for (int x = 0; x < 2; ++x) {
            tma_load_4d(dst + x * 16384, &tm_k, bars + bar, 64 * x, h, tma_t0 + m * kC, tma_b);
            tma_load_4d(dst + x * 16384 + 8192, &tm_q, bars + bar, 64 * x, h, tma_t0 + m * kC, tma_b);
        }
    };
    auto pf_kq = [&](int m) {  // into L2: the load itself waits for a free buffer
        if (m < NC)
            for (int x = 0; x < 2; ++x) {
                tma_prefetch_l2_4d(&tm_k, 64 * x, h, tma_t0 + m * kC, tma_b);
                tma_prefetch_l2_4d(&tm_q, 64 * x, h, tma_t0 + m * kC, tma_b);
            }
    };
    auto load_g = [&](int m) {
        s_issued[1] = m;
        mbar_arrive_expect_tx(bars + B_G + m % 3, 2 * 8192);
        for (int x = 0; x < 2; ++x)
            tma_load_4d(sm + L::COL + (m % 3) * 16384 + x * 8192, &tm_g, bars + B_G + m % 3, 64 * x, h,
                        tma_t0 + m * kC, tma_b);
    };
    auto pf_g = [&](int m) {
        if (m < NC)
            for (int x = 0; x < 2; ++x) tma_prefetch_l2_4d(&tm_g, 64 * x, h, tma_t0 + m * kC, tma_b);
    };
    auto load_v = [&](int m) {
        if (v_zero) {  // the zero tile is already in place
            mbar_arrive(bars + B_V);
            return;
        }
        s_issued[2] = m;
        mbar_arrive_expect_tx(bars + B_V, (DVT / 64) * 8192);
        for (int x = 0; x < DVT / 64; ++x)
            tma_load_4d(sm + L::RAWV + x * 8192, &tm_v, bars + B_V, j0 + 64 * x, h, tma_t0 + m * kC, tma_b);
    };
    auto pf_v = [&](int m) {
        if (m < NC && !v_zero)
            for (int x = 0; x < DVT / 64; ++x) tma_prefetch_l2_4d(&tm_v, j0 + 64 * x, h, tma_t0 + m * kC, tma_b);
    };
    // per-token gate (GATE == 1): the chunk's 64 gates as row 0 of a K-major
    // B tile at the start of its log_alpha/KF buffer (rows 1-15 feed prefix-sum
    // columns that are never read). Lane l holds tokens 2l, 2l+1.
    auto gate_row_load = [&](int m) -> uint32_t {
        const int t = m * kC + 2 * lane;
        const float a = (m < NC && t < seq_len) ? __bfloat162float(gate_tok[(tok0 + t) * H + h]) : 0.f;
        const float c = (m < NC && t + 1 < seq_len) ? __bfloat162float(gate_tok[(tok0 + t + 1) * H + h]) : 0.f;
        return pack_bf16x2(a, c);
    };
    auto gate_row_store = [&](int m, uint32_t w) {  // warp-collective
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sb + L::COL + (uint32_t)(m % 3) * 16384 + 4u * lane), "r"(w)
                     : "memory");
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + B_G + m % 3);
    };
    auto cumsum_mma = [&](int m) {  // prefix sums of chunk m into its slot (one thread)
        const int s = m % 3;
        if (GATE == 0) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + L::SLOT0 + 128 * s, dadd(dLMAT, kk * 32), dadd(dCOLN, s * 16384 + kk * 2048),
                            ID_CS, kk > 0);
        } else if (GATE == 1) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + L::SLOT0 + 128 * s, dadd(dLMAT, kk * 32), dadd(dCOLK, s * 16384 + kk * 32),
                            ID_CS1, kk > 0);
        }
        mma_commit(bars + B_CS + s);  // (no gate: an empty commit completes the phase)
    };

    if (warp < kTileWarp0) {
        // ============================================================ chain warps
        // lane row = 32 * quad + lane: a key channel of the state, a token row of the slot
        const int row = 32 * quad + lane;
        const bool issuer = warp == 0 && lane == 0;
        {   // initial state into TMEM (fp32, lane = key channel)
#pragma unroll 1
            for (int gq = 0; gq < DVT / 32; ++gq) {
                uint32_t r[32];
                if (s0m) {
                    const float4* src = reinterpret_cast<const float4*>(s0m + (size_t)row * kD + j0 + 32 * gq);
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float4 v = src[u];
                        r[4 * u] = __float_as_uint(v.x); r[4 * u + 1] = __float_as_uint(v.y);
                        r[4 * u + 2] = __float_as_uint(v.z); r[4 * u + 3] = __float_as_uint(v.w);
                    }
                } else {
#pragma unroll
                    for (int u = 0; u < 32; ++u) r[u] = (s0_ident && row == j0 + 32 * gq + u) ? __float_as_uint(1.f) : 0u;
                }
                tmem_st32(lane_addr + L::S_COL + 32 * gq, r);
            }
            tmem_st_wait();
            tc_fence_before();
            nb_sync(NB_CH, 128);
            tc_fence_after();
        }
        uint32_t gnext = 0;  // per-token gate row of the next chunk to place (warp 0)
        if (NC > 0) {
            if (issuer) {
                if (!sj.withhold_first_load) load_kq(0, B_KQ);
                if (NC > 1) load_kq(1, B_KQ + 1);
                pf_kq(2);
                if (GATE == 0) {
                    for (int j = 0; j < 3 && j < NC; ++j) load_g(j);
                    pf_g(3);
                }
            }
            if (GATE == 1 && warp == 3) {
                for (int j = 0; j < 3 && j < NC; ++j) gate_row_store(j, gate_row_load(j));
                gnext = gate_row_load(3);
            }
        }
        // s1 body for one 32-column group: state rows -> bf16 operand words (times
        // the operand scale), R *= tensor-memory scale
        auto s1_group = [&](int gq, float os, float ts, float ms, uint32_t (&pk)[16]) {
            uint32_t v[32];
            tmem_ld32(lane_addr + L::S_COL + 32 * gq, v);
            tmem_ld_wait(v);
            if (os == ts) {  // (every factored chunk) the operand is the rescaled state itself;
                             // two factors, so that their product may lie below the fp32 range
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    float x0, x1;
                    mul_f32x2(x0, x1, __uint_as_float(v[2 * u]), __uint_as_float(v[2 * u + 1]), ts, ts);
                    mul_f32x2(x0, x1, x0, x1, ms, ms);
                    v[2 * u] = __float_as_uint(x0);
                    v[2 * u + 1] = __float_as_uint(x1);
                    pk[u] = pack_bf16x2(x0, x1);
                }
            } else {
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    float x0, x1, y0, y1;
                    mul_f32x2(x0, x1, __uint_as_float(v[2 * u]), __uint_as_float(v[2 * u + 1]), os, os);
                    mul_f32x2(y0, y1, __uint_as_float(v[2 * u]), __uint_as_float(v[2 * u + 1]), ts, ts);
                    pk[u] = pack_bf16x2(x0, x1);
                    v[2 * u] = __float_as_uint(y0);
                    v[2 * u + 1] = __float_as_uint(y1);
                }
            }
            tmem_st32(lane_addr + L::S_COL + 32 * gq, v);
        };
        // operand words of one 32-column group of channel row i -> the S/delta operand
        auto sop_store = [&](int i, int gq, const uint32_t (&pk)[16]) {
#pragma unroll
            for (int jc = 0; jc < 4; ++jc) {
                const int j = 32 * gq + 8 * jc;
                const uint32_t off = (uint32_t)(i >> 3) * L::SBO_V + (uint32_t)(j >> 6) * 1024 + (uint32_t)(i & 7) * 128 +
                                     ((uint32_t)(((j & 63) >> 3) ^ (i & 7)) << 4);
                st_shared_v4(sb + L::SOP + off, pk[4 * jc], pk[4 * jc + 1], pk[4 * jc + 2], pk[4 * jc + 3]);
            }
        };
        for (int n = 0; n < NC; ++n) {
            const int s = n % 3, rb = n & 1;
            const uint32_t slot = lane_addr + L::SLOT0 + 128 * s;
            if (n > 0) {
                const bool m2 = waitw(B_M2, (uint32_t)(n - 1));  // state update of the previous chunk done
                if (n + 2 < NC) {  // its log_alpha/KF buffer is free: the gate tile of chunk n+2 (warp 3)
                    if (GATE == 0 && warp == 3 && lane == 0 && m2) {
                        load_g(n + 2);
                        pf_g(n + 3);
                    }
                    if (GATE == 1 && warp == 3) {
                        gate_row_store(n + 2, gnext);
                        gnext = gate_row_load(n + 3);
                    }
                }
            }
            waitw(B_SC + s, (uint32_t)(n / 3));
            const float os = sOpS[s * 128 + row], ts = sTmS[s * 128 + row], ms = sMdS[s * 128 + row];
            // the whole state (channel row `row` per thread) -> the bf16 operand of MMA1
#pragma unroll 1
            for (int gq = 0; gq < DVT / 32; ++gq) {
                uint32_t pk[16];
                s1_group(gq, os, ts, ms, pk);
                sop_store(row, gq, pk);
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            nb_sync(NB_CH, 128);
            if (issuer) {
                wait1(B_RR + rb, (uint32_t)(n >> 1));  // row operand (and [T'; PT]) of chunk n stored
                wait1(B_V, (uint32_t)n);                // its v tile landed
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)  // [U; P T' v] = [T'; PT] v starts the accumulator
                    mma_bf16_ss(tmem + L::SLOT0 + 128 * s, dadd(dTP, kk * 32), dadd(dV, kk * 2048), ID_U, kk > 0);
                mma_commit(bars + B_UO + s);  // [T'; PT] and the v tile read
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)  // + [-W'; QE - P W'] S^ over all 128 key channels
                    mma_bf16_ss(tmem + L::SLOT0 + 128 * s, dadd(dROWK, rb * 32768 + (kk >> 2) * 16384 + (kk & 3) * 32),
                                dadd(dSOP, kk * 2 * L::SBO_V), ID_M1, 1);
                mma_commit(bars + B_M1);
            }
            __syncwarp();
            const bool m1 = waitw(B_M1, (uint32_t)n);
            if (quad < 2) {
                {   // delta (slot rows 0-63) -> bf16 operand over the state operand
#pragma unroll 1
                    for (int gq = 0; gq < DVT / 32; ++gq) {
                        uint32_t v[32];
                        tmem_ld32(slot + 32 * gq, v);
                        tmem_ld_wait(v);
                        uint32_t pk[16];
#pragma unroll
                        for (int u = 0; u < 16; ++u)
                            pk[u] = pack_bf16x2(__uint_as_float(v[2 * u]), __uint_as_float(v[2 * u + 1]));
                        sop_store(row, gq, pk);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                nb_sync(NB_CHLO, 64);
                if (issuer) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)  // R += KF^T delta
                        mma_bf16_ss(tmem + L::S_COL, dadd(dCOLN, s * 16384 + kk * 2048), dadd(dSOP, kk * 2 * L::SBO_V),
                                    ID_M2, 1);
                    mma_commit(bars + B_M2);
                    mbar_arrive(bars + B_SF + s);  // slot rows 0-63 read
                }
                __syncwarp();
            } else {
                if (warp == 2 && lane == 0 && n + 2 < NC && m1) {  // the row buffer of this parity is free
                    load_kq(n + 2, B_KQ + rb);
                    pf_kq(n + 3);
                }
                {   // O (slot rows 64-127) -> global bf16: a full chunk through a swizzled
                    // [32 tok][32 ch] stage and a tensor store per 32 columns (coalesced,
                    // asynchronous); a partial chunk by plain stores (rows past a packed
                    // sequence belong to the next one)
                    const int r = row - 64;
                    const int t0 = n * kC;
                    const bool full = t0 + kC <= seq_len;
                    uint8_t* stg = sm + L::OST + (quad - 2) * 2048;
#pragma unroll 1
                    for (int gq = 0; gq < DVT / 32; ++gq) {
                        uint32_t v[32];
                        tmem_ld32(slot + 32 * gq, v);
                        tmem_ld_wait(v);
                        if (o_on && full) {
                            if (lane == 0) bulk_wait_read0();  // the stage's previous store has read it
                            __syncwarp();
#pragma unroll
                            for (int jc = 0; jc < 4; ++jc)
                                st_shared_v4(smem_u32(stg) + lane * 64 + ((jc ^ ((lane >> 1) & 3)) << 4),
                                             pack_bf16x2(__uint_as_float(v[8 * jc + 0]), __uint_as_float(v[8 * jc + 1])),
                                             pack_bf16x2(__uint_as_float(v[8 * jc + 2]), __uint_as_float(v[8 * jc + 3])),
                                             pack_bf16x2(__uint_as_float(v[8 * jc + 4]), __uint_as_float(v[8 * jc + 5])),
                                             pack_bf16x2(__uint_as_float(v[8 * jc + 6]), __uint_as_float(v[8 * jc + 7])));
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                tma_store_4d(&tm_o, stg, j0 + 32 * gq, h, tma_t0 + t0 + 32 * (quad - 2), tma_b);
                                bulk_commit();
                            }
                        } else if (o_on && t0 + r < seq_len) {
                            uint4* dst = reinterpret_cast<uint4*>(o + ((tok0 + t0 + r) * H + h) * kD + j0 + 32 * gq);
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
                tc_fence_before();
                nb_sync(NB_CHHI, 64);
                if (warp == 2 && lane == 0) mbar_arrive(bars + B_SF + s);  // slot rows 64-127 read
                __syncwarp();
            }
        }
        // ------------------------------------------------------------ final state S = Diag(ek) R
        if (NC > 0) waitw(B_M2, (uint32_t)(NC - 1));
        // one decision per warp: the tensor-memory loads below are warp-collective
        if (__shfl_sync(0xffffffffu, (stm && !*s_abort) ? 1 : 0, 0)) {
            const float ek = sEK[row];
#pragma unroll 1
            for (int gq = 0; gq < DVT / 32; ++gq) {
                uint32_t v[32];
                tmem_ld32(lane_addr + L::S_COL + 32 * gq, v);
                tmem_ld_wait(v);
                float4* dst = reinterpret_cast<float4*>(stm + (size_t)row * kD + j0 + 32 * gq);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    dst[u] = make_float4(__uint_as_float(v[4 * u]) * ek, __uint_as_float(v[4 * u + 1]) * ek,
                                         __uint_as_float(v[4 * u + 2]) * ek, __uint_as_float(v[4 * u + 3]) * ek);
            }
        }
        if (quad >= 2 && lane == 0) bulk_wait0();  // every tensor store of O complete
        if (issuer) {  // after an abort: wait (bounded) for this thread's MMAs
            if (*s_abort) {
                mma_commit(bars + B_FIN);
                mbar_wait_bounded(bars + B_FIN, 0u, kDrainBudget);
            }
        }
    } else if (warp < kInvWarp0) {
        // ============================================================ tile warps
        // thread: token tok (lanes of its quadrant, both halves of [L; L] hold the
        // chunk's 64 tokens), 64 channels from ch0
        const int ttid = tid - 32 * kTileWarp0;
        const int tok = 32 * (quad & 1) + lane, ch0 = 64 * (quad >> 1);
        int nex = 0;
        if (NC > 0 && ttid == 0) {
            if (GATE != 2) wait1(B_G, 0u);
            tc_fence_after();
            cumsum_mma(0);
        }
        // Exact path of a chunk that fails the vote: reload the raw k/q rows, per-pair
        // exponentials for A and P (raw sums, staged and stored into the slot where
        // the [A; P] MMA would have put them), plain tiles k e^G, q e^G, k e^{G_last-G}.
        // Middle tier for a chunk whose decay is too strong for the chunk-start
        // reference (some |G_r| > 80): reference point G_m = G_last / 2 per channel,
        // E = e^{G - G_m}, F = e^{G_m - G}. With a decay (G falling from 0 to G_last)
        // every exponent is within |G_last| / 2, so it holds up to |G_last| = 160;
        // the vote checks it. Returns false (nothing changed) when it does not
        // hold; otherwise the raw k/q rows are reloaded and the tiles rebuilt.
        auto mid_chunk = [&](int m, int s, int rb, int cb, int lim) -> bool {
            const uint32_t slotq = lane_addr + L::SLOT0 + 128 * s;
            const bool live = tok < lim;
            float amax = 0.f;
            if (GATE == 0) {
#pragma unroll 1
                for (int u8 = 0; u8 < 8; ++u8) {
                    const int c0 = ch0 + 8 * u8;
                    uint32_t g8[8];
                    tmem_ld8(slotq + c0, g8);
                    tmem_ld_wait(g8);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        amax = fmaxf(amax, fabsf((__uint_as_float(g8[e]) - 0.5f * sGl[c0 + e]) * kLog2e));
                }
            } else {
                uint32_t g1;
                tmem_ld1(slotq, g1);
                tmem_ld_wait1(g1);
                amax = fabsf((__uint_as_float(g1) - 0.5f * sGl[0]) * kLog2e);
            }
            if (nb_or(NB_TOR, 128, live && !(amax <= kGuardL))) return false;
            // reload the raw k/q rows over the tiles just written (their stores are
            // ordered before the copy by the proxy fence and the barrier)
            fence_proxy_async_smem();
            nb_sync(NB_TILE, 128);
            if (ttid == 0 && !*s_abort) load_kq(m, B_EXKQ);
            waitw(B_EXKQ, (uint32_t)nex);
            ++nex;
            const uint32_t rop = sb + L::ROW + rb * 32768;
            const uint32_t colp = sb + L::COL + cb * 16384;
            const uint32_t km = live ? 0xFFFFFFFFu : 0u;
            uint32_t ep1 = 0, fp1 = 0;
            if (GATE == 1) {
                uint32_t g1;
                tmem_ld1(slotq, g1);
                tmem_ld_wait1(g1);
                const float a = (__uint_as_float(g1) - 0.5f * sGl[0]) * kLog2e;
                ep1 = pack_bf16x2(ex2(a), ex2(a));
                fp1 = pack_bf16x2(ex2(-a), ex2(-a));
            }
#pragma unroll 1
            for (int u8 = 0; u8 < 8; ++u8) {
                const int c0 = ch0 + 8 * u8;
                const uint32_t ko = rop_off(tok, c0);
                const uint32_t fo = (uint32_t)((c0 >> 6) * 8192 + tok * 128 + ((((c0 & 63) >> 3) ^ (tok & 7)) << 4));
                const uint4 kv = ld_shared_v4(rop + ko);
                const uint4 qv = ld_shared_v4(rop + ko + 8192);
                const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
                const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
                uint32_t ke[4], qe[4], kf[4];
                if (GATE == 0) {
                    uint32_t g8[8];
                    tmem_ld8(slotq + c0, g8);
                    tmem_ld_wait(g8);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float a0 = (__uint_as_float(g8[2 * u]) - 0.5f * sGl[c0 + 2 * u]) * kLog2e;
                        const float a1 = (__uint_as_float(g8[2 * u + 1]) - 0.5f * sGl[c0 + 2 * u + 1]) * kLog2e;
                        const uint32_t ep = pack_bf16x2(ex2(a0), ex2(a1));
                        const uint32_t fp = pack_bf16x2(ex2(-a0), ex2(-a1));
                        ke[u] = hmul2_bf16(kw[u], ep) & km;
                        qe[u] = hmul2_bf16(qw[u], ep) & km;
                        kf[u] = hmul2_bf16(kw[u], fp) & km;
                    }
                } else {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        ke[u] = hmul2_bf16(kw[u], ep1) & km;
                        qe[u] = hmul2_bf16(qw[u], ep1) & km;
                        kf[u] = hmul2_bf16(kw[u], fp1) & km;
                    }
                }
                st_shared_v4(rop + ko, ke[0], ke[1], ke[2], ke[3]);
                st_shared_v4(rop + ko + 8192, qe[0], qe[1], qe[2], qe[3]);
                st_shared_v4(colp + fo, kf[0], kf[1], kf[2], kf[3]);
            }
            return true;
        };
        auto exact_chunk = [&](int m, int s, int rb, int cb, int lim) {
            const uint32_t slotq = lane_addr + L::SLOT0 + 128 * s;
            fence_proxy_async_smem();  // (as in the middle tier: tile stores before the copy)
            nb_sync(NB_TILE, 128);
            if (ttid == 0 && !*s_abort) load_kq(m, B_EXKQ);
            waitw(B_EXKQ, (uint32_t)nex);
            if (m > 0) waitw(B_SCRF, (uint32_t)(m - 1));  // the inverse warps are done with the scratch
            float* stg = reinterpret_cast<float*>(sm + L::SCR);  // 8 KB: G of 32 channels, then half of A or P
            const bool live = tok < lim;
            const uint8_t* rk = sm + L::ROW + rb * 32768;
            constexpr int kPairs = kC * (kC + 1) / 2, kPer = (kPairs + 127) / 128;
            float av[kPer], pv[kPer];
#pragma unroll
            for (int i = 0; i < kPer; ++i) {
                av[i] = 0.f;
                pv[i] = 0.f;
            }
            auto pair_rs = [](int p, int& r, int& s2) {
                r = (int)((sqrtf(8.f * (float)p + 1.f) - 1.f) * 0.5f);
                while ((r + 1) * (r + 2) / 2 <= p) ++r;
                while (r * (r + 1) / 2 > p) --r;
                s2 = p - r * (r + 1) / 2;
            };
#pragma unroll 1
            for (int hq = 0; hq < 4; ++hq) {     // channels [32 hq, 32 hq + 32)
                if ((ch0 >> 6) == (hq >> 1)) {  // this thread's channels: G -> fp32 [64 tok][32 ch]
#pragma unroll 1
                    for (int u4 = 0; u4 < 4; ++u4) {
                        const int u8 = 4 * (hq & 1) + u4;
                        uint32_t g8[8];
                        if (GATE == 0) {
                            tmem_ld8(slotq + ch0 + 8 * u8, g8);
                            tmem_ld_wait(g8);
                        } else {
                            uint32_t g1;
                            tmem_ld1(slotq, g1);
                            tmem_ld_wait1(g1);
#pragma unroll
                            for (int e = 0; e < 8; ++e) g8[e] = g1;
                        }
                        float* dst = stg + tok * 32 + 8 * u4;
                        *reinterpret_cast<float4*>(dst) = make_float4(__uint_as_float(g8[0]), __uint_as_float(g8[1]),
                                                                      __uint_as_float(g8[2]), __uint_as_float(g8[3]));
                        *reinterpret_cast<float4*>(dst + 4) = make_float4(__uint_as_float(g8[4]), __uint_as_float(g8[5]),
                                                                          __uint_as_float(g8[6]), __uint_as_float(g8[7]));
                    }
                }
                nb_sync(NB_TILE, 128);
#pragma unroll
                for (int i = 0; i < kPer; ++i) {
                    const int p = ttid + 128 * i;
                    if (p < kPairs) {
                        int r, s2;
                        pair_rs(p, r, s2);
                        float a = av[i], pp = pv[i];
                        // rows past the sequence stay 0 (their gates may be another
                        // sequence's and overflow the exponential)
                        for (int i2 = 0; i2 < (r < lim ? 32 : 0); ++i2) {
                            const int c = (i2 + p) & 31, cc = 32 * hq + c;
                            const float ks =
                                __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(rk + rop_off(s2, cc))) *
                                ex2((stg[r * 32 + c] - stg[s2 * 32 + c]) * kLog2e);
                            a = fmaf(__bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(rk + rop_off(r, cc))), ks, a);
                            pp = fmaf(__bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(rk + rop_off(64 + r, cc))),
                                      ks, pp);
                        }
                        av[i] = a;
                        pv[i] = pp;
                    }
                }
                nb_sync(NB_TILE, 128);  // staging read
            }
            {   // plain tiles in place (the raw rows are no longer needed)
                const uint32_t rop = sb + L::ROW + rb * 32768;
                const uint32_t colp = sb + L::COL + cb * 16384;
#pragma unroll 1
                for (int u8 = 0; u8 < 8; ++u8) {
                    const int c0 = ch0 + 8 * u8;
                    uint32_t g8[8];
                    if (GATE == 0) {
                        tmem_ld8(slotq + c0, g8);
                        tmem_ld_wait(g8);
                    } else {
                        uint32_t g1;
                        tmem_ld1(slotq, g1);
                        tmem_ld_wait1(g1);
#pragma unroll
                        for (int e = 0; e < 8; ++e) g8[e] = g1;
                    }
                    const uint32_t ko = rop_off(tok, c0);
                    const uint32_t fo = (uint32_t)((c0 >> 6) * 8192 + tok * 128 + ((((c0 & 63) >> 3) ^ (tok & 7)) << 4));
                    const uint4 kv = ld_shared_v4(rop + ko);
                    const uint4 qv = ld_shared_v4(rop + ko + 8192);
                    const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
                    const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
                    uint32_t ke[4], qe[4], kf[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float g0 = __uint_as_float(g8[2 * u]), g1 = __uint_as_float(g8[2 * u + 1]);
                        const float gl0 = GATE == 0 ? sGl[c0 + 2 * u] : sGl[0];
                        const float gl1 = GATE == 0 ? sGl[c0 + 2 * u + 1] : sGl[0];
                        const uint32_t ep = pack_bf16x2(ex2(g0 * kLog2e), ex2(g1 * kLog2e));
                        const uint32_t fp = pack_bf16x2(ex2((gl0 - g0) * kLog2e), ex2((gl1 - g1) * kLog2e));
                        ke[u] = live ? hmul2_bf16(kw[u], ep) : 0u;
                        qe[u] = live ? hmul2_bf16(qw[u], ep) : 0u;
                        kf[u] = live ? hmul2_bf16(kw[u], fp) : 0u;
                    }
                    st_shared_v4(rop + ko, ke[0], ke[1], ke[2], ke[3]);
                    st_shared_v4(rop + ko + 8192, qe[0], qe[1], qe[2], qe[3]);
                    st_shared_v4(colp + fo, kf[0], kf[1], kf[2], kf[3]);
                }
            }
            // raw A sums, then raw P sums -> fp32 [32][64] staging, 32 rows at a time
            // -> the slot (quadrants 0/1 hold the A rows, 2/3 the P rows)
#pragma unroll 1
            for (int wh = 0; wh < 4; ++wh) {
                const int w = wh >> 1, rh = wh & 1;  // A or P; rows [32 rh, 32 rh + 32)
                for (int i = ttid; i < 32 * 64 / 4; i += 128)
                    reinterpret_cast<float4*>(stg)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                nb_sync(NB_TILE, 128);
#pragma unroll
                for (int i = 0; i < kPer; ++i) {
                    const int p = ttid + 128 * i;
                    if (p < kPairs) {
                        int r, s2;
                        pair_rs(p, r, s2);
                        if ((r >> 5) == rh) stg[(r & 31) * 64 + s2] = w == 0 ? av[i] : pv[i];
                    }
                }
                nb_sync(NB_TILE, 128);
                if (quad == wh) {
                    const float* src = stg + lane * 64;
#pragma unroll 1
                    for (int h2 = 0; h2 < 2; ++h2) {
                        uint32_t r32[32];
#pragma unroll
                        for (int u = 0; u < 32; ++u) r32[u] = __float_as_uint(src[32 * h2 + u]);
                        tmem_st32(slotq + 32 * h2, r32);
                    }
                    tmem_st_wait();
                }
                nb_sync(NB_TILE, 128);  // staging read before the next pass overwrites it
            }
            ++nex;
        };
        // A/P of chunk m out of the slot: A (rows 0-63, scaled by beta_r, strictly
        // lower) into the fp32 scratch, P (rows 64-127, lower incl.) into the bf16
        // K-major tile. The scratch is free once the inverse warps finished the
        // previous chunk's inverse, the P tile once its PT MMA completed.
        auto readout_ap = [&](int m, int s) {
            const uint32_t slotq = lane_addr + L::SLOT0 + 128 * s;
            if (m > 0) waitw(quad < 2 ? B_SCRF : B_PT, (uint32_t)(m - 1));
            waitw(B_AP + s, (uint32_t)(m / 3));
            if (quad < 2) {
                if (erase) {
                    const int r = 32 * quad + lane;
                    // (the inverse warps stored this chunk's beta before the scratch-free arrive)
                    const float br = sBeta[(m & 1) * 64 + r];
#pragma unroll 1
                    for (int e8 = 0; e8 < 8; ++e8) {
                        uint32_t v[8];
                        tmem_ld8(slotq + 8 * e8, v);
                        tmem_ld_wait(v);
                        uint32_t w[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int c = 8 * e8 + 2 * u;
                            const float a0 = (c < r) ? br * __uint_as_float(v[2 * u]) : 0.f;
                            const float a1 = (c + 1 < r) ? br * __uint_as_float(v[2 * u + 1]) : 0.f;
                            const __half2 h = __floats2half2_rn(a0, a1);
                            w[u] = *reinterpret_cast<const uint32_t*>(&h);
                        }
                        st_shared_v4(smem_u32(sA + r * kLDA + 8 * e8), w[0], w[1], w[2], w[3]);
                    }
                }
            } else {
                const int r = 32 * (quad - 2) + lane;
#pragma unroll 1
                for (int jc = 0; jc < 8; ++jc) {
                    uint32_t v[8];
                    tmem_ld8(slotq + 8 * jc, v);
                    tmem_ld_wait(v);
                    uint32_t w[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int c = 8 * jc + 2 * u;
                        const float p0 = (c <= r) ? __uint_as_float(v[2 * u]) : 0.f;
                        const float p1 = (c + 1 <= r) ? __uint_as_float(v[2 * u + 1]) : 0.f;
                        w[u] = pack_bf16x2(p0, p1);
                    }
                    st_shared_v4(sb + L::SP + r * 128 + ((jc ^ (r & 7)) << 4), w[0], w[1], w[2], w[3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            nb_sync(NB_TILE, 128);
            if (ttid == 0) mbar_arrive(bars + B_AR);
        };
        for (int m = 0; m < NC; ++m) {
            const int s = m % 3, rb = m & 1, cb = m % 3;
            const uint32_t slotq = lane_addr + L::SLOT0 + 128 * s;
            waitw(B_CS + s, (uint32_t)(m / 3));
            waitw(B_KQ + rb, (uint32_t)(m >> 1));
            // Tokens of this chunk that belong to the sequence: [0, lim). Rows past
            // it are zero (past the tensor) or the next packed sequence's.
            const int lim = min(seq_len - m * kC, kC);
            const bool live = tok < lim;
            const int tl_tok = lim - 1;  // last token: publishes G_last for the scales
            // operand tiles, in place: 8 groups of 8 channels of this thread's row;
            // amax tracks the largest |exponent| for the vote
            float amax = 0.f;
            {
                const uint32_t rop = sb + L::ROW + rb * 32768;
                const uint32_t colp = sb + L::COL + cb * 16384;
                uint32_t ep1 = 0, fp1 = 0;
                if (GATE == 1) {  // per-token gate: one factor pair per token
                    uint32_t g1;
                    tmem_ld1(slotq, g1);
                    tmem_ld_wait1(g1);
                    if (tok == tl_tok) sGl[0] = __uint_as_float(g1);
                    const float a = __uint_as_float(g1) * kLog2e;
                    amax = fabsf(a);
                    const float e = ex2(a), f = ex2(-a);
                    ep1 = pack_bf16x2(e, e);
                    fp1 = pack_bf16x2(f, f);
                }
                const uint32_t km = live ? 0xFFFFFFFFu : 0u;  // rows past the sequence: k = q = 0
                const bool masked = !__all_sync(0xffffffffu, live);
#pragma unroll 1
                for (int u8 = 0; u8 < 8; ++u8) {
                    const int c0 = ch0 + 8 * u8;
                    const uint32_t ko = rop_off(tok, c0);
                    const uint32_t fo = (uint32_t)((c0 >> 6) * 8192 + tok * 128 + ((((c0 & 63) >> 3) ^ (tok & 7)) << 4));
                    const uint4 kv = ld_shared_v4(rop + ko);
                    const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
                    uint32_t ke[4], qe[4], kf[4];
                    if (GATE == 2) {  // no decay: KE = k, QE = q, KF = k
                        if (!live) {
                            st_shared_v4(rop + ko, 0u, 0u, 0u, 0u);
                            st_shared_v4(rop + ko + 8192, 0u, 0u, 0u, 0u);
                        }
                        st_shared_v4(colp + fo, kw[0] & km, kw[1] & km, kw[2] & km, kw[3] & km);
                        continue;
                    }
                    const uint4 qv = ld_shared_v4(rop + ko + 8192);
                    const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
                    if (GATE == 0) {
                        uint32_t g8[8];
                        tmem_ld8(slotq + c0, g8);
                        tmem_ld_wait(g8);
                        if (tok == tl_tok) {
                            *reinterpret_cast<float4*>(sGl + c0) = make_float4(
                                __uint_as_float(g8[0]), __uint_as_float(g8[1]), __uint_as_float(g8[2]), __uint_as_float(g8[3]));
                            *reinterpret_cast<float4*>(sGl + c0 + 4) = make_float4(
                                __uint_as_float(g8[4]), __uint_as_float(g8[5]), __uint_as_float(g8[6]), __uint_as_float(g8[7]));
                        }
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            // E = e^G = 2^{G log2 e}, F = 1/E
                            float a0, a1;
                            mul_f32x2(a0, a1, __uint_as_float(g8[2 * u]), __uint_as_float(g8[2 * u + 1]), kLog2e, kLog2e);
                            amax = fmaxf(amax, fmaxf(fabsf(a0), fabsf(a1)));
                            // packed bf16 products: the factor pairs are rounded to bf16
                            // first, the products once more (both well inside the bf16
                            // rounding of the MMA operands)
                            const uint32_t ep = pack_bf16x2(ex2(a0), ex2(a1));
                            const uint32_t fp = pack_bf16x2(ex2(-a0), ex2(-a1));
                            ke[u] = hmul2_bf16(kw[u], ep);
                            qe[u] = hmul2_bf16(qw[u], ep);
                            kf[u] = hmul2_bf16(kw[u], fp);
                        }
                    } else {
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            ke[u] = hmul2_bf16(kw[u], ep1);
                            qe[u] = hmul2_bf16(qw[u], ep1);
                            kf[u] = hmul2_bf16(kw[u], fp1);
                        }
                    }
                    if (masked) {
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            ke[u] &= km;
                            qe[u] &= km;
                            kf[u] &= km;
                        }
                    }
                    st_shared_v4(rop + ko, ke[0], ke[1], ke[2], ke[3]);
                    st_shared_v4(rop + ko + 8192, qe[0], qe[1], qe[2], qe[3]);
                    st_shared_v4(colp + fo, kf[0], kf[1], kf[2], kf[3]);
                }
            }
            // every factor finite and normal? (NaN counts as a failure); the vote also
            // makes G_last visible to every tile thread
            const bool failed = GATE != 2 && nb_or(NB_TOR, 128, live && !(amax <= kGuardL));
            // 0: reference at the chunk start, 1: at G_last / 2, 2: exact per-pair path
            const int tier = !failed ? 0 : (mid_chunk(m, s, rb, cb, lim) ? 1 : 2);
            const bool exact = tier == 2;
            if (exact) exact_chunk(m, s, rb, cb, lim);
            {   // per-channel scales of this chunk. The tensor memory holds R with
                // S = Diag(ek) R; the chain feeds S^ = Diag(os) Diag(ms) R to MMA1 and
                // keeps Diag(ts) Diag(ms) R + KF^T delta (ms = 1 unless os = ts), whose
                // true state is Diag(ek_new) times it.
                const int c = ttid;
                const float g_l = GATE == 0 ? sGl[c] : (GATE == 1 ? sGl[0] : 0.f);
                const float ek_prev = sEK[c];
                const int slot4 = m % 3;  // (the tile warps reach chunk m + 3 only after the chain read chunk m)
                if (tier == 0) {         // reference at the chunk start: S^ = S, KF = k e^{-G}
                    sOpS[slot4 * 128 + c] = ek_prev;
                    sTmS[slot4 * 128 + c] = ek_prev;
                    sMdS[slot4 * 128 + c] = 1.f;
                    sEK[c] = __expf(g_l);
                } else if (tier == 1) {  // S^ = e^{G_m} S, KF = k e^{G_m - G}, G_m = G_last / 2
                    // (ek_prev e^{G_m} can lie below the fp32 range while the state it
                    // scales does not: the chain applies the two factors one after the other)
                    const float em = __expf(0.5f * g_l);
                    sOpS[slot4 * 128 + c] = ek_prev;
                    sTmS[slot4 * 128 + c] = ek_prev;
                    sMdS[slot4 * 128 + c] = em;
                    sEK[c] = em;
                } else {                 // exact: KF = k e^{G_last - G}
                    sOpS[slot4 * 128 + c] = ek_prev;
                    sTmS[slot4 * 128 + c] = __expf(g_l) * ek_prev;
                    sMdS[slot4 * 128 + c] = 1.f;
                    sEK[c] = 1.f;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            nb_sync(NB_TILE, 128);
            if (ttid == 0) {
                mbar_arrive(bars + B_SC + m % 3);
                tc_fence_after();
                if (!exact) {  // [A; P] = [KE; QE] KF^T over the prefix-sum columns (read)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ss(tmem + L::SLOT0 + 128 * s, dadd(dROWK, rb * 32768 + (kk >> 2) * 16384 + (kk & 3) * 32),
                                    dadd(dCOLK, cb * 16384 + (kk >> 2) * 8192 + (kk & 3) * 32), ID_AP, kk > 0);
                }
                mma_commit(bars + B_AP + s);
            }
            __syncwarp();
            readout_ap(m, s);
            if (ttid == 0 && m + 1 < NC) {  // next chunk's prefix sums, once its slot is read out and its gate is in place
                const int s1 = (m + 1) % 3;
                if (m + 1 >= 3) wait1(B_SF + s1, (uint32_t)((m + 1) / 3 - 1));
                if (GATE != 2) wait1(B_G + s1, (uint32_t)((m + 1) / 3));
                tc_fence_after();
                cumsum_mma(m + 1);
            }
            __syncwarp();
        }
        if (ttid == 0) {  // after an abort: wait (bounded) for this thread's MMAs
            if (*s_abort) {
                mma_commit(bars + B_FIN + 1);
                mbar_wait_bounded(bars + B_FIN + 1, 0u, kDrainBudget);
            }
        }
    } else {
        // ============================================================ inverse warps
        // Per chunk m: (I + A)^{-1} -> T', then the PT and W MMAs with the readouts
        // after them (PT -> [T'; PT], [W'; P W'] -> row operand); the v loads.
        const int iw = warp - kInvWarp0;  // 0..7
        const int hf = iw >> 2;           // which 32-column half of a readout this warp takes
        const int itid = tid - 32 * kInvWarp0;
        auto load_beta = [&](int m) -> float {
            const int t = m * kC + itid;
            return (itid < kC && m < NC && t < seq_len) ? __bfloat162float(beta[(tok0 + t) * H + h]) : 0.f;
        };
        const float* sBm = sBeta;  // beta of the chunk in work (parity buffer)
        // [T'; PT] and the v tile are free once the previous chunk's U MMA (issued by
        // the chain) completed; then the v tile of chunk m is loaded (one thread)
        auto tp_free = [&](int m) {
            if (m > 0) {
                if (wait1(B_UO + (m - 1) % 3, (uint32_t)((m - 1) / 3))) load_v(m);
                pf_v(m + 1);
            }
        };
        // ---- P5: T = (I + A)^{-1} -> T' = T Diag(beta), bf16, rows 0-63 of [T'; PT]
        auto store_tprime = [&](int r, int s, float t) {
            *reinterpret_cast<__nv_bfloat16*>(sm + L::TP + km_off(r, s)) = __float2bfloat16_rn(t * sBm[s]);
        };
        auto p5 = [&](int m) {
            if (!erase) {  // A = 0: T = I, T' = Diag(beta); thread: row itid/4, 16 columns
                const int r = itid >> 2, j0c = 2 * (itid & 3);
#pragma unroll
                for (int jc = 0; jc < 2; ++jc) {
                    const int j = j0c + jc;  // 8-column chunk
                    uint32_t w[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int s0 = 8 * j + 2 * u;
                        w[u] = pack_bf16x2(s0 == r ? sBm[r] : 0.f, s0 + 1 == r ? sBm[r] : 0.f);
                    }
                    st_shared_v4(sb + L::TP + r * 128 + ((j ^ (r & 7)) << 4), w[0], w[1], w[2], w[3]);
                }
                return;
            }
            // diagonal 16x16 blocks: four threads per column, rows q, q+4, q+8, q+12
            const int a = itid >> 6, jc = (itid >> 2) & 15, q = itid & 3;
            float colv[4] = {0.f, 0.f, 0.f, 0.f};
            {
                const __half* Ab = sA + (16 * a) * kLDA + 16 * a;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    const float mine = (r == jc) ? 1.f : ((r > jc) ? -acc[r >> 2] : 0.f);
                    const float t = __shfl_sync(0xffffffffu, mine, (lane & ~3) | (r & 3));
                    if (q == (r & 3)) colv[r >> 2] = t;
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if (q + 4 * i > r) acc[i] = fmaf(__half2float(Ab[(q + 4 * i) * kLDA + r]), t, acc[i]);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) sTd[(a * 16 + q + 4 * i) * kLDT + jc] = colv[i];
            }
            // [T'; PT] is free once the previous chunk's U MMA has read it (waited
            // here, after the diagonal blocks, which do not touch it)
            if (itid == 0) tp_free(m);
            nb_sync(NB_INV, 256);
#pragma unroll
            for (int i = 0; i < 4; ++i) store_tprime(16 * a + q + 4 * i, 16 * a + jc, colv[i]);
            // Blocks below the diagonal, one column chain per warp (block column
            // bb, 8-column half nt), held in registers: for a = bb+1..3,
            // X = sum_{k=bb}^{a-1} A_ak T_kb, then T_ab = -T_aa X, on m16n8k8 tf32
            // MMAs. A product's accumulator fragment becomes the right-hand operand
            // of the next product by shuffles; A and the diagonal blocks come from
            // shared memory.
            const int bb = iw >> 1, nt = iw & 1;
            if (bb < 3) {
                const int g = lane >> 2, t = lane & 3;
                const int sc = 16 * bb + 8 * nt;  // first column of this warp's half
                // accumulator (rows g | g+8, columns 2t | 2t+1) -> right operand
                // fragments of the two 8-row k-steps (rows t | t+4, column g)
                auto c2b = [&](const float (&c)[4], uint32_t (&bf)[2][2]) {
                    const int src0 = 4 * t + (g >> 1), src1 = 4 * (t + 4) + (g >> 1);
                    const bool odd = (g & 1) != 0;
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const float e0 = __shfl_sync(0xffffffffu, c[2 * j], src0);
                        const float o0 = __shfl_sync(0xffffffffu, c[2 * j + 1], src0);
                        const float e1 = __shfl_sync(0xffffffffu, c[2 * j], src1);
                        const float o1 = __shfl_sync(0xffffffffu, c[2 * j + 1], src1);
                        bf[j][0] = to_tf32(odd ? o0 : e0);
                        bf[j][1] = to_tf32(odd ? o1 : e1);
                    }
                };
                uint32_t tb[3][2][2];  // right operand fragments of T_kb, k = bb..2
                {
                    const float* D = sTd + bb * 16 * kLDT + 8 * nt;
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        tb[0][j][0] = to_tf32(D[(8 * j + t) * kLDT + g]);
                        tb[0][j][1] = to_tf32(D[(8 * j + t + 4) * kLDT + g]);
                    }
                }
                // da = a - bb and dk = k - bb run over compile-time ranges, so the
                // fragment array stays in registers
#pragma unroll
                for (int da = 1; da < 4; ++da) {
                    const int a = bb + da;
                    if (a > 3) break;
                    float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int dk = 0; dk < da; ++dk) {
                        const int k = bb + dk;
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const __half* Ar = sA + (16 * a) * kLDA + 16 * k + 8 * j;
                            const uint32_t af[4] = {to_tf32(__half2float(Ar[g * kLDA + t])),
                                                    to_tf32(__half2float(Ar[(g + 8) * kLDA + t])),
                                                    to_tf32(__half2float(Ar[g * kLDA + t + 4])),
                                                    to_tf32(__half2float(Ar[(g + 8) * kLDA + t + 4]))};
                            mma_tf32_16x8x8(x, af, tb[dk][j]);
                        }
                    }
                    uint32_t xb[2][2];
                    c2b(x, xb);
                    float y[4] = {0.f, 0.f, 0.f, 0.f};
                    const float* D = sTd + a * 16 * kLDT;
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const uint32_t af[4] = {to_tf32(D[g * kLDT + 8 * j + t]), to_tf32(D[(g + 8) * kLDT + 8 * j + t]),
                                                to_tf32(D[g * kLDT + 8 * j + t + 4]),
                                                to_tf32(D[(g + 8) * kLDT + 8 * j + t + 4])};
                        mma_tf32_16x8x8(y, af, xb[j]);
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) y[e] = -y[e];
                    const int s0 = sc + 2 * t;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
                        *reinterpret_cast<uint32_t*>(sm + L::TP + km_off(16 * a + g + 8 * hh, s0)) =
                            pack_bf16x2(y[2 * hh] * sBm[s0], y[2 * hh + 1] * sBm[s0 + 1]);
                    if (da < 3 && a < 3) c2b(y, tb[da]);
                }
            }
        };
        // ---- PT (slot rows 64-127, columns 64-127) -> bf16 rows 64-127 of [T'; PT]
        auto p6 = [&](uint32_t slot) {
            if (quad < 2) return;
            const int r = 32 * (quad - 2) + lane;
            uint32_t v[32];
            tmem_ld32(slot + 64 + 32 * hf, v);
            tmem_ld_wait(v);
#pragma unroll
            for (int jc = 0; jc < 4; ++jc) {
                uint32_t w[4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    w[u] = pack_bf16x2(__uint_as_float(v[8 * jc + 2 * u]), __uint_as_float(v[8 * jc + 2 * u + 1]));
                const int R = 64 + r;
                st_shared_v4(sb + L::TP + R * 128 + (((4 * hf + jc) ^ (R & 7)) << 4), w[0], w[1], w[2], w[3]);
            }
        };
        // ---- P7: [W'; P W'] -> row operand: rows 0-63 -W' over KE, rows 64-127 QE - P W'
        auto p7 = [&](uint32_t slot, int rb) {
            const uint32_t rop = sb + L::ROW + rb * 32768;
            if (quad < 2) {
                const int r = 32 * quad + lane;
                if (!erase) {  // additive write: delta = U, the W S term is zero
#pragma unroll
                    for (int jc = 0; jc < 8; ++jc)
                        st_shared_v4(rop + hf * 16384 + r * 128 + ((jc ^ (r & 7)) << 4), 0u, 0u, 0u, 0u);
                    return;
                }
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t v[32];
                    tmem_ld32(slot + 64 * hf + 32 * hh, v);
                    tmem_ld_wait(v);
#pragma unroll
                    for (int jc = 0; jc < 4; ++jc) {
                        uint32_t w[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            w[u] = pack_bf16x2(__uint_as_float(v[8 * jc + 2 * u]), __uint_as_float(v[8 * jc + 2 * u + 1])) ^
                                   0x80008000u;
                        st_shared_v4(rop + hf * 16384 + r * 128 + (((4 * hh + jc) ^ (r & 7)) << 4), w[0], w[1], w[2], w[3]);
                    }
                }
            } else {
                if (!erase) return;  // W = 0: the rows keep QE
                const int r = 32 * (quad - 2) + lane, R = 64 + r;
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t v[32];
                    tmem_ld32(slot + 64 * hf + 32 * hh, v);
                    tmem_ld_wait(v);
#pragma unroll
                    for (int jc = 0; jc < 4; ++jc) {
                        const uint32_t addr = rop + hf * 16384 + R * 128 + (((4 * hh + jc) ^ (R & 7)) << 4);
                        const uint4 qv = ld_shared_v4(addr);
                        const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
                        uint32_t w[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            w[u] = hsub2_bf16(qw[u], pack_bf16x2(__uint_as_float(v[8 * jc + 2 * u]),
                                                                 __uint_as_float(v[8 * jc + 2 * u + 1])));
                        st_shared_v4(addr, w[0], w[1], w[2], w[3]);
                    }
                }
            }
        };
        if (NC > 0 && itid == 0) {
            load_v(0);
            pf_v(1);
        }
        // beta of chunk m + 1 goes into its parity buffer at the start of chunk m:
        // the tile warps read it for their A readout after the scratch-free
        // arrive of chunk m (chunk 0's was stored during setup)
        float beta_next = load_beta(1);
        for (int m = 0; m < NC; ++m) {
            const int s = m % 3, rb = m & 1;
            const uint32_t slot = lane_addr + L::SLOT0 + 128 * s;
            sBm = sBeta + (m & 1) * 64;
            if (itid < kC) sBeta[((m + 1) & 1) * 64 + itid] = beta_next;
            beta_next = load_beta(m + 2);
            waitw(B_AR, (uint32_t)m);  // A and P of chunk m in shared memory
            if (!erase) {  // T' = Diag(beta) goes straight into [T'; PT]
                if (itid == 0) tp_free(m);
                nb_sync(NB_INV, 256);
            }
            p5(m);
            fence_proxy_async_smem();
            tc_fence_before();
            nb_sync(NB_INV, 256);
            if (itid == 0) {
                mbar_arrive(bars + B_SCRF);  // A/T scratch free
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)  // PT = P T' into columns 64-127 (rows 0-63 take junk)
                    mma_bf16_ss(tmem + L::SLOT0 + 128 * s + 64, dadd(dYP, kk * 32), dadd(dTPN, kk * 2048), ID_PT, kk > 0);
                mma_commit(bars + B_PT);
            }
            waitw(B_PT, (uint32_t)m);
            p6(slot);
            fence_proxy_async_smem();
            tc_fence_before();
            nb_sync(NB_INV, 256);
            if (erase) {
                if (itid == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)  // [W'; P W'] = [T'; PT] KE
                        mma_bf16_ss(tmem + L::SLOT0 + 128 * s, dadd(dTP, kk * 32), dadd(dROWN, rb * 32768 + kk * 2048),
                                    ID_W, kk > 0);
                    mma_commit(bars + B_WB);
                }
                waitw(B_WB, (uint32_t)m);
            }
            p7(slot, rb);
            fence_proxy_async_smem();
            tc_fence_before();
            nb_sync(NB_INV, 256);
            if (itid == 0) mbar_arrive(bars + B_RR + rb);  // row operand of chunk m stored (the chain issues its U MMA)
            __syncwarp();
        }
        if (itid == 0) {  // after an abort: wait (bounded) for this thread's MMAs
            if (*s_abort) {
                mma_commit(bars + B_FIN + 2);
                mbar_wait_bounded(bars + B_FIN + 2, 0u, kDrainBudget);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        // After an abort: wait (bounded) for the last phase armed on each copy
        // barrier, so no tensor copy still writes shared memory when the CTA exits.
        if (lane == 0 && *s_abort) {
            // phases armed on each copy barrier: k/q of chunk j on B_KQ + j % 2,
            // log_alpha on B_G + j % 3, v on B_V, exact-path reloads on B_EXKQ
            int armed[7];
#pragma unroll
            for (int x = 0; x < 2; ++x) armed[x] = s_issued[0] >= x ? (s_issued[0] - x) / 2 + 1 : 0;
            if (sj.withhold_first_load && armed[0] > 0) --armed[0];
#pragma unroll
            for (int x = 0; x < 3; ++x) armed[2 + x] = s_issued[1] >= x ? (s_issued[1] - x) / 3 + 1 : 0;
            armed[5] = s_issued[2] + 1;
            armed[6] = s_issued[3];
#pragma unroll
            for (int i = 0; i < 7; ++i) {
                const int bar = i < 5 ? B_KQ + i : (i == 5 ? B_V : B_EXKQ);
                if (armed[i] > 0) mbar_wait_bounded(bars + bar, (uint32_t)(armed[i] - 1) & 1u, kDrainBudget);
            }
        }
        __syncwarp();
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

// [B, T, H, 128] bf16 viewed as a 4-D tensor (channel, head, token, batch).
// Loads: box = 64 channels x 1 head x 64 tokens x 1 batch, 128-byte swizzle;
// tokens past T read as zero. Output stores (out = true): box = 32 channels
// x 1 x 32 tokens x 1, 64-byte swizzle; tokens past T are not written.
bool make_map(CUtensorMap* m, const void* base, int B, int T, int H, bool out = false) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)T * H * kD * 2};
    const cuuint32_t box_in[4] = {64, 1, 64, 1}, box_out[4] = {32, 1, 32, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, out ? box_out : box_in,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, out ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Chains the entry states of the segments: S_in[j+1] = M_j S_in[j] + C_j for
// j = 1..P-2 (S_in[1] is segment 0's final state). The columns of a state are
// independent, so each CTA carries 8 value columns of one sequence-head
// through every segment, in fp32.
__global__ void __launch_bounds__(256) segment_scan_kernel(const float* __restrict__ M, const float* __restrict__ C,
                                                           float* Sin, int P) {
    constexpr size_t kMat = (size_t)kD * kD;
    const int bh = blockIdx.x, c0 = blockIdx.y * 8, tid = threadIdx.x;
    const int i = tid >> 1, cc = (tid & 1) * 4;  // output row, first of 4 columns
    __shared__ float s[kD][8];
    const float* S1 = Sin + (size_t)bh * (P - 1) * kMat;
    for (int e = tid; e < kD * 8; e += 256) s[e >> 3][e & 7] = S1[(size_t)(e >> 3) * kD + c0 + (e & 7)];
    __syncthreads();
    for (int j = 1; j <= P - 2; ++j) {
        const size_t mj = ((size_t)bh * (P - 2) + (j - 1)) * kMat + (size_t)i * kD;
        const float4 cv = *reinterpret_cast<const float4*>(C + mj + c0 + cc);
        float a0 = cv.x, a1 = cv.y, a2 = cv.z, a3 = cv.w;
        const float4* mrow = reinterpret_cast<const float4*>(M + mj);
#pragma unroll 4
        for (int k4 = 0; k4 < kD / 4; ++k4) {
            const float4 m = mrow[k4];
            const float mk[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float* sr = s[4 * k4 + u] + cc;
                a0 = fmaf(mk[u], sr[0], a0);
                a1 = fmaf(mk[u], sr[1], a1);
                a2 = fmaf(mk[u], sr[2], a2);
                a3 = fmaf(mk[u], sr[3], a3);
            }
        }
        __syncthreads();  // every read of the previous state is done
        s[i][cc] = a0; s[i][cc + 1] = a1; s[i][cc + 2] = a2; s[i][cc + 3] = a3;
        *reinterpret_cast<float4*>(Sin + ((size_t)bh * (P - 1) + j) * kMat + (size_t)i * kD + c0 + cc) =
            make_float4(a0, a1, a2, a3);
        __syncthreads();
    }
}

template <int DVT, int ERASE, int GATE>
cudaError_t launch_dvt(const ChunkArgs& a, cudaStream_t stream, const SegJobs& sj, long units) {
    using L = Layout<DVT>;
    CUtensorMap mk, mq, mg, mv, mo;
    const int mb = a.cu_seqlens ? 1 : a.B;  // packed sequences: one [1, T] token range
    if (!make_map(&mk, a.k, mb, a.T, a.H) || !make_map(&mq, a.q, mb, a.T, a.H) ||
        (a.gate == 0 && !make_map(&mg, a.log_alpha, mb, a.T, a.H)) || !make_map(&mv, a.v, mb, a.T, a.H) ||
        !make_map(&mo, a.o, mb, a.T, a.H, true))
        return cudaErrorInvalidValue;
    if (a.gate != 0) mg = mk;  // no log_alpha tile is loaded; any valid map fills the parameter
    auto kern = kda_chunk_tc_kernel<DVT, ERASE, GATE>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::SMEM_BYTES);
    if (err != cudaSuccess) return err;
    unsigned* status = static_cast<unsigned*>(a.workspace);
    const unsigned grid = (unsigned)(units * (kD / DVT));
    kern<<<grid, kThreads, L::SMEM_BYTES, stream>>>(mk, mq, mg, mv, mo, (const __nv_bfloat16*)a.beta, a.S0,
                                                    (__nv_bfloat16*)a.o, a.ST, a.T, a.H, status,
                                                    GATE == 1 ? (const __nv_bfloat16*)a.log_alpha : nullptr,
                                                    a.cu_seqlens, sj);
    return cudaGetLastError();
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess || n <= 0) {
        cudaGetLastError();  // (no device: plan for a B200)
        return 148;
    }
    return n;
}

// Segments for the chunk-parallel scan, or 0 when it does not pay.
// Every CTA runs its chunks at about the same period, so a plan's time is its
// depth in chunk periods: each phase takes ceil(CTAs / SMs) waves of L chunks
// plus kFillChunks for filling and draining a CTA's pipeline (fitted to
// measurements: B1 H32 T131072 runs P = 5 at 0.95x the time of P = 3, while
// B2 H16 T4096, 13-chunk segments, runs P = 5 at 1.13x). Phase 1 holds
// B*H*(2P-3) CTAs, phase 3 B*H*(P-1) units (two CTAs each when that fits one
// wave). P runs over 3 .. NC / kMinSegChunks (forced: up to NC / 2, and P >= 3
// whenever T has 3 chunks); L is rounded to whole chunks and P recounted so
// no segment is empty. AUTO takes the scan only when it is shallower than one
// pass over the whole sequence; ties go to fewer segments.
constexpr int kMinSegChunks = 8;
constexpr int kFillChunks = 8;
void scan_plan(const ChunkArgs& a, int mode, int* P_out, int* L_out) {
    *P_out = 0;
    *L_out = 0;
    if (mode == 0 || a.cu_seqlens || a.T <= 0) return;
    const long bh = (long)a.B * a.H;
    const long NC = (a.T + kC - 1) / kC;
    if (bh <= 0 || NC < 3) return;
    const long sms = sm_count();
    auto waves = [&](long ctas) { return (ctas + sms - 1) / sms; };
    const long one_pass = waves(bh) * (NC + kFillChunks);
    const long pmax = mode == 2 ? std::max<long>(3, NC / 2) : NC / kMinSegChunks;
    long best_P = 0, best_L = 0, best_cost = 0;
    for (long P = 3; P <= pmax; ++P) {
        const long Lc = (NC + P - 1) / P;
        const long Pn = (NC + Lc - 1) / Lc;
        if (Pn < 3 || Pn != P) continue;  // (a recounted P is visited on its own)
        const long units3 = bh * (Pn - 1);
        const long cost = (waves(bh * (2 * Pn - 3)) + waves(2 * units3 <= sms ? 2 * units3 : units3)) * (Lc + kFillChunks);
        if (best_P == 0 || cost < best_cost) {
            best_P = Pn;
            best_L = Lc;
            best_cost = cost;
        }
    }
    if (best_P == 0 || (mode == 1 && best_cost >= one_pass)) return;
    *P_out = (int)best_P;
    *L_out = (int)(best_L * kC);
}

}  // namespace

bool chunk_tc_supported(const ChunkArgs& a) {
    return a.bf16 && a.dk == kD && a.dv == kD && a.chunk == kC;
}

size_t chunk_tc_workspace_bytes(const ChunkArgs& a, int scan_mode) {
    int P, L;
    scan_plan(a, scan_mode, &P, &L);
    if (P == 0) return 256;
    const size_t mat = (size_t)kD * kD * sizeof(float), bh = (size_t)a.B * a.H;
    return 256 + bh * mat * (size_t)(2 * (P - 2) + (P - 1));
}

cudaError_t launch_chunk_tc(const ChunkArgs& a, int scan_mode, cudaStream_t stream) {
    cudaError_t err = cudaMemsetAsync(a.workspace, 0, sizeof(unsigned), stream);
    if (err != cudaSuccess) return err;
    // An empty sequence has no chunk to load (and no tensor map can describe
    // it): the result is S_T = S0, which the SIMT kernel writes.
    if (a.T == 0) return launch_chunk_simt(a, stream);
    const long bh = (long)a.B * a.H;
    const int sms = sm_count();
    int P, L;
    scan_plan(a, scan_mode, &P, &L);
    SegJobs one{};
    one.withhold_first_load = a.test_withhold_first_load;
    one.wait_budget = a.test_wait_budget;
    auto pick = [&](auto erase_c, auto gate_c) -> cudaError_t {
        constexpr int E = decltype(erase_c)::value, G = decltype(gate_c)::value;
        if (P == 0) {
            // One CTA per (batch, head) when there are enough heads to fill the
            // GPU; otherwise split the value channels in two.
            const bool wide = bh >= 96;
            return wide ? launch_dvt<128, E, G>(a, stream, one, bh) : launch_dvt<64, E, G>(a, stream, one, bh);
        }
        const size_t mat = (size_t)kD * kD;
        float* Mb = reinterpret_cast<float*>(static_cast<uint8_t*>(a.workspace) + 256);
        float* Cb = Mb + (size_t)bh * (P - 2) * mat;
        float* Sin = Cb + (size_t)bh * (P - 2) * mat;
        SegJobs sj{P, L, 1, Mb, Cb, Sin, one.withhold_first_load, one.wait_budget};
        cudaError_t e = launch_dvt<128, E, G>(a, stream, sj, bh * (2 * P - 3));
        if (e != cudaSuccess) return e;
        if (P > 2) {
            segment_scan_kernel<<<dim3((unsigned)bh, kD / 8), 256, 0, stream>>>(Mb, Cb, Sin, P);
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
        sj.phase = 3;
        const long units3 = bh * (P - 1);
        return 2 * units3 <= sms ? launch_dvt<64, E, G>(a, stream, sj, units3) : launch_dvt<128, E, G>(a, stream, sj, units3);
    };
    using I0 = std::integral_constant<int, 0>;
    using I1 = std::integral_constant<int, 1>;
    using I2 = std::integral_constant<int, 2>;
    if (a.erase) {
        if (a.gate == 0) return pick(I1{}, I0{});
        if (a.gate == 1) return pick(I1{}, I1{});
        return pick(I1{}, I2{});
    }
    if (a.gate == 0) return pick(I0{}, I0{});
    if (a.gate == 1) return pick(I0{}, I1{});
    return pick(I0{}, I2{});
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
#include "kda.h"

// Scratch of the allocation-free entry point; every GPU that loads this
// library holds these bytes until the process exits. In host code this name
// is only a stand-in for the symbol: its device address comes from
// cudaGetSymbolAddress, looked up on every call with the caller's device
// current (a host-side query, so a device reset cannot leave a stale address
// behind).
static __device__ __align__(256) unsigned char g_kda_noalloc_scratch[256];

namespace {

// Device address of the scratch array on the current device.
cudaError_t noalloc_scratch(void** out) {
    void* p = nullptr;
    const cudaError_t err = cudaGetSymbolAddress(&p, g_kda_noalloc_scratch);
    if (err != cudaSuccess) return err;
    *out = p;
    return cudaSuccess;
}

}  // namespace

extern "C" kda_status_t kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const void* log_alpha,
                                              const void* beta, const float* S0, void* o, float* S_T, int B,
                                              int T, int H, int dk, int dv, int chunk, kda_dtype_t dtype,
                                              void* stream) {
    kda::ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.S0 = S0; a.o = o; a.ST = S_T;
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv; a.chunk = chunk; a.bf16 = dtype == KDA_BF16;
    a.erase = 1;  // KDA: erase with a per-channel gate
    a.gate = KDA_GATE_CHANNEL;
    a.cu_seqlens = nullptr;
    const kda_status_t st = kda::check_chunk_args(a, dtype);
    if (st != KDA_OK) return st;
    if (!kda::chunk_tc_supported(a)) return KDA_ERR_UNSUPPORTED;
    // The kernel's scratch must fit the fixed array.
    if (kda::chunk_tc_workspace_bytes(a, 0) > sizeof(g_kda_noalloc_scratch)) return KDA_ERR_INVALID_ARG;
    if ((long long)B * H == 0) return KDA_OK;
    void* scratch = nullptr;
    if (noalloc_scratch(&scratch) != cudaSuccess) return KDA_ERR_CUDA;
    a.workspace = scratch;
    a.workspace_bytes = sizeof(g_kda_noalloc_scratch);
    // launch_chunk_tc clears the status word before the kernel runs.
    const cudaError_t err = kda::launch_chunk_tc(a, 0, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

extern "C" kda_status_t kda_noalloc_status(void* stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_CUDA;
    void* scratch = nullptr;
    if (noalloc_scratch(&scratch) != cudaSuccess) return KDA_ERR_CUDA;
    unsigned flag = 0;
    if (cudaMemcpy(&flag, scratch, sizeof(flag), cudaMemcpyDeviceToHost) != cudaSuccess) return KDA_ERR_CUDA;
    return flag ? KDA_ERR_TIMEOUT : KDA_OK;
}
