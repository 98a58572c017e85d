// Single-token KDA decode step (memory bound).
//
// "Decoding Hybrid Attention Architectures", sections 1 and 5: at inference
// the recurrent state has a fixed size, so one step costs the same whatever
// the context length. Per (sequence, head), with S in R^{dk x dv}:
//     S' = Diag(alpha) S,   delta = beta (v - S'^T k),
//     S_out = S' + k delta^T,   o = S_out^T q = S'^T q + delta (k . q).
// Variants (variant table of section 3.4): log_alpha per key channel, one per
// head, or none; without the erase term delta = beta v.
// The state is read once and written once: each CTA owns a 32-column slice of
// one head's state, keeps it in registers between the two reductions
// (S'^T k and S'^T q) and the rank-one update, and streams it with 16-byte
// evict-first loads/stores. S_out may alias S_in: every element is read by
// the thread that later writes it, before it writes.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

constexpr int kDecodeThreads = 128;
constexpr int kDecodeCols = 32;  // value columns per CTA (8 threads x float4)

// ERASE / GATE: the variant switches, compile-time so each variant is its own
// kernel and the KDA instance carries no variant branches.
template <typename T, int DK, int ERASE, int GATE>
__global__ void __launch_bounds__(kDecodeThreads, 8)
decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   const T* __restrict__ log_alpha, const T* __restrict__ beta, const float* S_in,
                   float* S_out, T* __restrict__ o, int dv) {
    constexpr int erase = ERASE, gate = GATE;
    constexpr int RG = kDecodeThreads / 8;  // 16 row groups
    constexpr int ROWS = DK / RG;           // rows per thread
    const int nslices = dv / kDecodeCols;
    const long head = blockIdx.x / nslices;  // n * H + h
    const int col0 = (blockIdx.x % nslices) * kDecodeCols;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int c4 = t & 7, rg = t >> 3;

    __shared__ float sk[DK], sq[DK], sa[DK];
    __shared__ float4 red_k[kDecodeThreads / 32][8], red_q[kDecodeThreads / 32][8];
    __shared__ float s_kq;

    const float* Sh = S_in + head * DK * dv + col0 + c4 * 4;
    float4 s[ROWS];
#pragma unroll
    for (int i = 0; i < ROWS; ++i) s[i] = __ldcs(reinterpret_cast<const float4*>(Sh + (size_t)(rg + RG * i) * dv));

    for (int i = t; i < DK; i += kDecodeThreads) {
        sk[i] = to_f32(k[head * DK + i]);
        sq[i] = to_f32(q[head * DK + i]);
        sa[i] = gate == 0 ? expf(to_f32(log_alpha[head * DK + i])) : (gate == 1 ? expf(to_f32(log_alpha[head])) : 1.f);
    }
    __syncthreads();
    if (warp == 0) {
        float acc = 0.f;
        for (int i = lane; i < DK; i += 32) acc = fmaf(sk[i], sq[i], acc);
        acc = warp_sum(acc);
        if (lane == 0) s_kq = acc;
    }

    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
        const int r = rg + RG * i;
        const float a = sa[r], kr = sk[r], qr = sq[r];
        s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
        pk.x = fmaf(kr, s[i].x, pk.x); pk.y = fmaf(kr, s[i].y, pk.y);
        pk.z = fmaf(kr, s[i].z, pk.z); pk.w = fmaf(kr, s[i].w, pk.w);
        pq.x = fmaf(qr, s[i].x, pq.x); pq.y = fmaf(qr, s[i].y, pq.y);
        pq.z = fmaf(qr, s[i].z, pq.z); pq.w = fmaf(qr, s[i].w, pq.w);
    }
    // lanes l, l^8, l^16, l^24 share a column group
#pragma unroll
    for (int off = 8; off < 32; off <<= 1) {
        pk.x += __shfl_xor_sync(0xffffffffu, pk.x, off); pk.y += __shfl_xor_sync(0xffffffffu, pk.y, off);
        pk.z += __shfl_xor_sync(0xffffffffu, pk.z, off); pk.w += __shfl_xor_sync(0xffffffffu, pk.w, off);
        pq.x += __shfl_xor_sync(0xffffffffu, pq.x, off); pq.y += __shfl_xor_sync(0xffffffffu, pq.y, off);
        pq.z += __shfl_xor_sync(0xffffffffu, pq.z, off); pq.w += __shfl_xor_sync(0xffffffffu, pq.w, off);
    }
    if (lane < 8) {
        red_k[warp][lane] = pk;
        red_q[warp][lane] = pq;
    }
    __syncthreads();
    float4 u = red_k[0][c4], sq4 = red_q[0][c4];
#pragma unroll
    for (int w = 1; w < kDecodeThreads / 32; ++w) {
        const float4 a = red_k[w][c4], b = red_q[w][c4];
        u.x += a.x; u.y += a.y; u.z += a.z; u.w += a.w;
        sq4.x += b.x; sq4.y += b.y; sq4.z += b.z; sq4.w += b.w;
    }
    const float b = to_f32(beta[head]);
    const T* vh = v + head * dv + col0 + c4 * 4;
    float4 d;
    const float er = erase ? 1.f : 0.f;  // no erase: delta = beta v
    d.x = b * (to_f32(vh[0]) - er * u.x);
    d.y = b * (to_f32(vh[1]) - er * u.y);
    d.z = b * (to_f32(vh[2]) - er * u.z);
    d.w = b * (to_f32(vh[3]) - er * u.w);

    float* Sout = S_out + head * DK * dv + col0 + c4 * 4;
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
        const float kr = sk[rg + RG * i];
        float4 x = s[i];
        x.x = fmaf(kr, d.x, x.x); x.y = fmaf(kr, d.y, x.y);
        x.z = fmaf(kr, d.z, x.z); x.w = fmaf(kr, d.w, x.w);
        __stcs(reinterpret_cast<float4*>(Sout + (size_t)(rg + RG * i) * dv), x);
    }
    if (rg == 0) {
        const float kq = s_kq;
        T* oh = o + head * dv + col0 + c4 * 4;
        oh[0] = from_f32<T>(fmaf(d.x, kq, sq4.x));
        oh[1] = from_f32<T>(fmaf(d.y, kq, sq4.y));
        oh[2] = from_f32<T>(fmaf(d.z, kq, sq4.z));
        oh[3] = from_f32<T>(fmaf(d.w, kq, sq4.w));
    }
}

template <typename T, int DK>
static cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const void* la, const void* beta,
                                   const float* S_in, float* S_out, void* o, int N, int H, int dv, int erase,
                                   int gate, cudaStream_t stream) {
    const unsigned blocks = (unsigned)((long)N * H * (dv / kDecodeCols));
    auto go = [&](auto kern) {
        kern<<<blocks, kDecodeThreads, 0, stream>>>((const T*)q, (const T*)k, (const T*)v, (const T*)la,
                                                    (const T*)beta, S_in, S_out, (T*)o, dv);
        return cudaGetLastError();
    };
    if (erase) {
        if (gate == 0) return go(decode_step_kernel<T, DK, 1, 0>);
        if (gate == 1) return go(decode_step_kernel<T, DK, 1, 1>);
        return go(decode_step_kernel<T, DK, 1, 2>);
    }
    if (gate == 0) return go(decode_step_kernel<T, DK, 0, 0>);
    if (gate == 1) return go(decode_step_kernel<T, DK, 0, 1>);
    return go(decode_step_kernel<T, DK, 0, 2>);
}

cudaError_t launch_decode(const void* q, const void* k, const void* v, const void* la, const void* beta,
                          const float* S_in, float* S_out, void* o, int N, int H, int dk, int dv, int bf16,
                          int erase, int gate, cudaStream_t stream) {
    if (bf16) {
        if (dk == 64)
            return launch_decode_t<__nv_bfloat16, 64>(q, k, v, la, beta, S_in, S_out, o, N, H, dv, erase, gate, stream);
        return launch_decode_t<__nv_bfloat16, 128>(q, k, v, la, beta, S_in, S_out, o, N, H, dv, erase, gate, stream);
    }
    if (dk == 64) return launch_decode_t<float, 64>(q, k, v, la, beta, S_in, S_out, o, N, H, dv, erase, gate, stream);
    return launch_decode_t<float, 128>(q, k, v, la, beta, S_in, S_out, o, N, H, dv, erase, gate, stream);
}

}  // namespace kda
