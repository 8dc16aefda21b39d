// attn_bwd_kernel.cuh -- backward of the exact attention forward: dQ, dK, dV.
//
// Gradients of O = softmax(scale Q K^T [causal]) V for an upstream dO
// (aiinarabic.com "flash-attention", Equation (1) and its recomputation
// section: S and P are rebuilt tile by tile from Q, K and the forward's saved
// logsumexp instead of being stored):
//
//     P  = exp(scale S - lse)            S = Q K^T, masked
//     dV = P^T dO
//     dP = dO V^T
//     dS = P * (dP - D),  D_i = sum_c dO_ic O_ic   (= rowsum(P * dP))
//     dQ = scale dS K,    dK = scale dS^T Q
//
// Two kernels, no atomics and no scratch memory: one CTA per 64-key block
// accumulates dK and dV over the query blocks that see it; one CTA per
// 64-query block accumulates dQ over the key blocks it sees.  Both recompute
// S and dP.  This version runs on the FP32 pipes (CUDA cores): every tile is
// staged in shared memory and each thread computes 4 x 4 register blocks, so
// that a shared-memory load feeds several FMAs; the tensor-core version is
// future work.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace attn {
namespace bwd {

constexpr int kRows = 64;       // query rows and key rows per block
constexpr int kThreads = 256;

struct BwdParams {
    int B, H, N, Nk;            // N query rows, Nk key rows
    int causal_off;             // Nk - N: query i sees key j iff j <= i + causal_off (causal)
    float scale;
    const void *q, *k, *v, *o, *dout;
    int64_t q_sb, q_sh, q_si, k_sb, k_sh, k_si, v_sb, v_sh, v_si, o_sb, o_sh, o_si, do_sb, do_sh, do_si;
    const float* lse;           // [B*H*N]
    void *dq, *dk, *dv;
    int64_t dq_sb, dq_sh, dq_si, dk_sb, dk_sh, dk_si, dv_sb, dv_sh, dv_si;
};

template <typename T>
__device__ __forceinline__ float ld(const T* p) {
    return static_cast<float>(*p);
}
template <>
__device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
}
template <>
__device__ __forceinline__ float ld<__half>(const __half* p) {
    return __half2float(*p);
}
template <typename T>
__device__ __forceinline__ T cvt(float x);
template <>
__device__ __forceinline__ __half cvt<__half>(float x) {
    return __float2half_rn(x);
}
template <>
__device__ __forceinline__ __nv_bfloat16 cvt<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Shared-memory tiles (floats).  Row-major tiles R[r][c] have row stride D + 4
// (the two row groups a warp reads in the S/dP loop fall in different banks);
// transposed tiles T[c][r] have row stride 68 (staging writes them column by
// column; 68 spreads those stores over eight banks) and are read as float4
// along r; P and dS are [64][68].
template <int D>
struct BwdSmem {
    static constexpr int kLdr = D + 4;
    static constexpr int kRow = kRows * kLdr;       // a row-major tile
    static constexpr int kLdt = kRows + 4;
    static constexpr int kTr = D * kLdt;            // a transposed tile
    static constexpr int kLdp = kRows + 4;
    static constexpr int kSq = kRows * kLdp;
    // dK/dV kernel: K^T, V^T, Q, dO, P, dS, D, lse; dQ kernel: Q, dO, K^T, V^T, K, dS^T, D, lse
    static constexpr int kFloats = 2 * kTr + 2 * kRow + 2 * kSq + 2 * kRows;
    static constexpr int kFloatsDq = 2 * kRow + 2 * kTr + kRow + kSq + 2 * kRows;
    static constexpr int kBytes = (kFloats > kFloatsDq ? kFloats : kFloatsDq) * 4;
};

// rows [r0, r0 + 64) of a [rows, D] matrix (row stride `si`) into a row-major
// tile; rows past `nrows` are 0
template <typename T, int D>
__device__ __forceinline__ void stage_rows(float* dst, const T* src, int64_t si, int r0, int nrows) {
    for (int e = threadIdx.x; e < kRows * D; e += kThreads) {
        const int r = e / D, c = e % D;
        dst[r * (D + 4) + c] = (r0 + r < nrows) ? ld<T>(src + static_cast<int64_t>(r0 + r) * si + c) : 0.f;
    }
}

// the same rows into a transposed tile [c][r]
template <typename T, int D>
__device__ __forceinline__ void stage_cols(float* dst, const T* src, int64_t si, int r0, int nrows) {
    for (int e = threadIdx.x; e < kRows * D; e += kThreads) {
        const int r = e / D, c = e % D;
        dst[c * (kRows + 4) + r] = (r0 + r < nrows) ? ld<T>(src + static_cast<int64_t>(r0 + r) * si + c) : 0.f;
    }
}

// Phase A, shared by both kernels: the 64 x 64 tile of query rows q0.. and keys
// k0..  Thread t owns the 4 x 4 block rows 4 (t / 16).., keys 4 (t % 16)..;
// per column c it reads 4 Q and 4 dO values (row-major tiles) and one float4
// each of K^T and V^T, for 32 FMAs.  Returns P and dS of its block.
template <int D, bool CAUSAL>
__device__ __forceinline__ void tile_p_ds(const float* sQ, const float* sdO, const float* sKT, const float* sVT,
                                          const float* sD, const float* sL, float (&pv)[4][4], float (&ds)[4][4],
                                          int q0, int k0, const BwdParams& p) {
    const int ti = threadIdx.x >> 4, tj = threadIdx.x & 15;
    float s[4][4], dp[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) s[a][b] = dp[a][b] = 0.f;
#pragma unroll 4
    for (int c = 0; c < D; ++c) {
        float qv[4], dov[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            qv[a] = sQ[(4 * ti + a) * (D + 4) + c];
            dov[a] = sdO[(4 * ti + a) * (D + 4) + c];
        }
        const float4 kv = *reinterpret_cast<const float4*>(sKT + c * (kRows + 4) + 4 * tj);
        const float4 vv = *reinterpret_cast<const float4*>(sVT + c * (kRows + 4) + 4 * tj);
        const float kk[4] = {kv.x, kv.y, kv.z, kv.w}, vk[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                s[a][b] = fmaf(qv[a], kk[b], s[a][b]);
                dp[a][b] = fmaf(dov[a], vk[b], dp[a][b]);
            }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int i = 4 * ti + a, gi = q0 + i;
        const float lse = sL[i], Di = sD[i];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int gj = k0 + 4 * tj + b;
            bool ok = gi < p.N && gj < p.Nk;
            if (CAUSAL) ok = ok && gj <= gi + p.causal_off;
            pv[a][b] = ok ? expf(p.scale * s[a][b] - lse) : 0.f;
            ds[a][b] = pv[a][b] * (dp[a][b] - Di);
        }
    }
}

// D_i = sum_c dO_ic O_ic and lse_i for query rows q0.. into shared memory
// (dO from the row-major tile)
template <typename T, int D>
__device__ __forceinline__ void row_stats(float* sD, float* sL, const float* sdO, const T* o, int64_t o_si,
                                          const float* lse, int q0, int nrows) {
    const int i = threadIdx.x >> 2, part = threadIdx.x & 3;
    float acc = 0.f;
    if (q0 + i < nrows) {
        const T* orow = o + static_cast<int64_t>(q0 + i) * o_si;
        for (int c = part; c < D; c += 4) acc = fmaf(sdO[i * (D + 4) + c], ld<T>(orow + c), acc);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (part == 0) {
        sD[i] = acc;
        sL[i] = (q0 + i < nrows) ? lse[q0 + i] : 0.f;
    }
}

// ----------------------------------------------------------------------------- dK, dV
template <typename T, int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1) attn_bwd_dkdv_kernel(const BwdParams p) {
    extern __shared__ __align__(16) float smem[];
    using S = BwdSmem<D>;
    float *sKT = smem, *sVT = sKT + S::kTr, *sQ = sVT + S::kTr, *sdO = sQ + S::kRow;
    float *sP = sdO + S::kRow, *sdS = sP + S::kSq, *sD = sdS + S::kSq, *sL = sD + kRows;
    const int k0 = blockIdx.x * kRows;
    const int bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
    const T* q = static_cast<const T*>(p.q) + b * p.q_sb + h * p.q_sh;
    const T* k = static_cast<const T*>(p.k) + b * p.k_sb + h * p.k_sh;
    const T* v = static_cast<const T*>(p.v) + b * p.v_sb + h * p.v_sh;
    const T* o = static_cast<const T*>(p.o) + b * p.o_sb + h * p.o_sh;
    const T* dout = static_cast<const T*>(p.dout) + b * p.do_sb + h * p.do_sh;
    const float* lse = p.lse + static_cast<int64_t>(bh) * p.N;
    stage_cols<T, D>(sKT, k, p.k_si, k0, p.Nk);
    stage_cols<T, D>(sVT, v, p.v_si, k0, p.Nk);
    // phase B: thread t accumulates keys 4 (t / 16).. and columns t % 16 + 16 m
    constexpr int kC = D / 16;
    const int tj = threadIdx.x >> 4, tc = threadIdx.x & 15;
    const int ti = tj;                                   // phase A block row (same t / 16)
    float dk[4][kC], dv[4][kC];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int m = 0; m < kC; ++m) dk[a][m] = dv[a][m] = 0.f;
    // queries that see at least one of these keys: i >= k0 - causal_off
    int q_first = 0;
    if (CAUSAL) q_first = max(0, k0 - p.causal_off) / kRows * kRows;
    for (int q0 = q_first; q0 < p.N; q0 += kRows) {
        __syncthreads();   // previous tile's readers are done with sQ, sdO, sP, sdS
        stage_rows<T, D>(sQ, q, p.q_si, q0, p.N);
        stage_rows<T, D>(sdO, dout, p.do_si, q0, p.N);
        __syncthreads();
        row_stats<T, D>(sD, sL, sdO, o, p.o_si, lse, q0, p.N);
        __syncthreads();
        float pv[4][4], dsv[4][4];
        tile_p_ds<D, CAUSAL>(sQ, sdO, sKT, sVT, sD, sL, pv, dsv, q0, k0, p);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            *reinterpret_cast<float4*>(sP + (4 * ti + a) * S::kLdp + 4 * (threadIdx.x & 15)) =
                make_float4(pv[a][0], pv[a][1], pv[a][2], pv[a][3]);
            *reinterpret_cast<float4*>(sdS + (4 * ti + a) * S::kLdp + 4 * (threadIdx.x & 15)) =
                make_float4(dsv[a][0], dsv[a][1], dsv[a][2], dsv[a][3]);
        }
        __syncthreads();
        // dV += P^T dO, dK += dS^T Q over the 64 rows of the tile
#pragma unroll 2
        for (int i = 0; i < kRows; ++i) {
            const float4 p4 = *reinterpret_cast<const float4*>(sP + i * S::kLdp + 4 * tj);
            const float4 s4 = *reinterpret_cast<const float4*>(sdS + i * S::kLdp + 4 * tj);
            const float pp[4] = {p4.x, p4.y, p4.z, p4.w}, ss[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
            for (int m = 0; m < kC; ++m) {
                const float dov = sdO[i * (D + 4) + tc + 16 * m], qv = sQ[i * (D + 4) + tc + 16 * m];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    dv[a][m] = fmaf(pp[a], dov, dv[a][m]);
                    dk[a][m] = fmaf(ss[a], qv, dk[a][m]);
                }
            }
        }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int j = 4 * tj + a;
        if (k0 + j >= p.Nk) continue;
        T* dkr = static_cast<T*>(p.dk) + b * p.dk_sb + h * p.dk_sh + static_cast<int64_t>(k0 + j) * p.dk_si;
        T* dvr = static_cast<T*>(p.dv) + b * p.dv_sb + h * p.dv_sh + static_cast<int64_t>(k0 + j) * p.dv_si;
#pragma unroll
        for (int m = 0; m < kC; ++m) {
            dkr[tc + 16 * m] = cvt<T>(p.scale * dk[a][m]);
            dvr[tc + 16 * m] = cvt<T>(dv[a][m]);
        }
    }
}

// ----------------------------------------------------------------------------- dQ
template <typename T, int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1) attn_bwd_dq_kernel(const BwdParams p) {
    extern __shared__ __align__(16) float smem[];
    using S = BwdSmem<D>;
    float *sQ = smem, *sdO = sQ + S::kRow, *sKT = sdO + S::kRow, *sVT = sKT + S::kTr, *sK = sVT + S::kTr;
    float *sdST = sK + S::kRow, *sD = sdST + S::kSq, *sL = sD + kRows;
    const int q0 = blockIdx.x * kRows;
    const int bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
    const T* q = static_cast<const T*>(p.q) + b * p.q_sb + h * p.q_sh;
    const T* k = static_cast<const T*>(p.k) + b * p.k_sb + h * p.k_sh;
    const T* v = static_cast<const T*>(p.v) + b * p.v_sb + h * p.v_sh;
    const T* o = static_cast<const T*>(p.o) + b * p.o_sb + h * p.o_sh;
    const T* dout = static_cast<const T*>(p.dout) + b * p.do_sb + h * p.do_sh;
    const float* lse = p.lse + static_cast<int64_t>(bh) * p.N;
    stage_rows<T, D>(sQ, q, p.q_si, q0, p.N);
    stage_rows<T, D>(sdO, dout, p.do_si, q0, p.N);
    __syncthreads();
    row_stats<T, D>(sD, sL, sdO, o, p.o_si, lse, q0, p.N);
    // phase B: thread t accumulates rows 4 (t / 16).. and columns t % 16 + 16 m
    constexpr int kC = D / 16;
    const int ti = threadIdx.x >> 4, tc = threadIdx.x & 15;
    float dq[4][kC];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int m = 0; m < kC; ++m) dq[a][m] = 0.f;
    // keys seen by at least one of these rows: j <= q0 + 63 + causal_off
    int k_end = p.Nk;
    if (CAUSAL) k_end = min(p.Nk, max(0, q0 + kRows + p.causal_off));
    for (int k0 = 0; k0 < k_end; k0 += kRows) {
        __syncthreads();   // previous tile's readers are done with sKT, sVT, sK, sdST
        stage_cols<T, D>(sKT, k, p.k_si, k0, p.Nk);
        stage_cols<T, D>(sVT, v, p.v_si, k0, p.Nk);
        stage_rows<T, D>(sK, k, p.k_si, k0, p.Nk);
        __syncthreads();
        float pv[4][4], dsv[4][4];
        tile_p_ds<D, CAUSAL>(sQ, sdO, sKT, sVT, sD, sL, pv, dsv, q0, k0, p);
        // dS transposed, so that phase B reads four rows of one key as a float4
        const int tj = threadIdx.x & 15;
#pragma unroll
        for (int bb = 0; bb < 4; ++bb)
            *reinterpret_cast<float4*>(sdST + (4 * tj + bb) * S::kLdp + 4 * ti) =
                make_float4(dsv[0][bb], dsv[1][bb], dsv[2][bb], dsv[3][bb]);
        __syncthreads();
#pragma unroll 2
        for (int j = 0; j < kRows; ++j) {
            const float4 d4 = *reinterpret_cast<const float4*>(sdST + j * S::kLdp + 4 * ti);
            const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
            for (int m = 0; m < kC; ++m) {
                const float kv = sK[j * (D + 4) + tc + 16 * m];
#pragma unroll
                for (int a = 0; a < 4; ++a) dq[a][m] = fmaf(dd[a], kv, dq[a][m]);
            }
        }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int i = 4 * ti + a;
        if (q0 + i >= p.N) continue;
        T* dqr = static_cast<T*>(p.dq) + b * p.dq_sb + h * p.dq_sh + static_cast<int64_t>(q0 + i) * p.dq_si;
#pragma unroll
        for (int m = 0; m < kC; ++m) dqr[tc + 16 * m] = cvt<T>(p.scale * dq[a][m]);
    }
}

}  // namespace bwd
}  // namespace attn
