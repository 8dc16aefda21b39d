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
// S and dP.  This first version runs on the FP32 pipes (CUDA cores), with
// every tile staged in shared memory; the tensor-core version is future work.
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

// rows [r0, r0 + 64) of a [rows, D] matrix (row stride `si`) into shared memory
// with row stride D + 1 (conflict-free column walks); rows past `nrows` are 0
template <typename T, int D>
__device__ __forceinline__ void stage(float* dst, const T* src, int64_t si, int r0, int nrows) {
    for (int e = threadIdx.x; e < kRows * D; e += kThreads) {
        const int r = e / D, c = e % D;
        dst[r * (D + 1) + c] = (r0 + r < nrows) ? ld<T>(src + static_cast<int64_t>(r0 + r) * si + c) : 0.f;
    }
}

// Shared-memory layout of both kernels (floats): A, B, C, E as 64 x (D+1)
// tiles, P and dS as 64 x 65, then D (row dot products) and lse, 64 each.
template <int D>
struct BwdSmem {
    static constexpr int kTile = kRows * (D + 1);
    static constexpr int kSq = kRows * (kRows + 1);
    static constexpr int kFloats = 4 * kTile + 2 * kSq + 2 * kRows;
    static constexpr int kBytes = kFloats * 4;
};

// Phase A, shared by both kernels: for the 64 x 64 tile of query rows q0.. and
// keys k0.., P and dS into shared memory.  Thread t owns row i = t / 4 and keys
// j = 4 jj + t % 4 (interleaved, so the four threads of a row read four rows
// of K and V in four different banks).
template <int D, bool CAUSAL>
__device__ __forceinline__ void tile_p_ds(const float* sQ, const float* sK, const float* sV, const float* sdO,
                                          const float* sD, const float* sL, float* sP, float* sdS, int q0,
                                          int k0, const BwdParams& p) {
    const int i = threadIdx.x >> 2, jg = threadIdx.x & 3;
    float s[16], dp[16];
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) s[jj] = dp[jj] = 0.f;
    for (int c = 0; c < D; ++c) {
        const float qv = sQ[i * (D + 1) + c], dov = sdO[i * (D + 1) + c];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
            const int j = 4 * jj + jg;
            s[jj] = fmaf(qv, sK[j * (D + 1) + c], s[jj]);
            dp[jj] = fmaf(dov, sV[j * (D + 1) + c], dp[jj]);
        }
    }
    const int gi = q0 + i;
    const float lse = sL[i], Di = sD[i];
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) {
        const int j = 4 * jj + jg, gj = k0 + j;
        bool ok = gi < p.N && gj < p.Nk;
        if (CAUSAL) ok = ok && gj <= gi + p.causal_off;
        const float pv = ok ? expf(p.scale * s[jj] - lse) : 0.f;
        sP[i * (kRows + 1) + j] = pv;
        sdS[i * (kRows + 1) + j] = pv * (dp[jj] - Di);
    }
}

// D_i = sum_c dO_ic O_ic and lse_i for query rows q0.. into shared memory.
template <typename T, int D>
__device__ __forceinline__ void row_stats(float* sD, float* sL, const float* sdO, const T* o, int64_t o_si,
                                          const float* lse, int q0, int nrows) {
    const int i = threadIdx.x >> 2, part = threadIdx.x & 3;
    float acc = 0.f;
    if (q0 + i < nrows) {
        const T* orow = o + static_cast<int64_t>(q0 + i) * o_si;
        for (int c = part; c < D; c += 4) acc = fmaf(sdO[i * (D + 1) + c], ld<T>(orow + c), acc);
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
    extern __shared__ float smem[];
    using S = BwdSmem<D>;
    float *sK = smem, *sV = sK + S::kTile, *sQ = sV + S::kTile, *sdO = sQ + S::kTile;
    float *sP = sdO + S::kTile, *sdS = sP + S::kSq, *sD = sdS + S::kSq, *sL = sD + kRows;
    const int k0 = blockIdx.x * kRows;
    const int bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
    const T* q = static_cast<const T*>(p.q) + b * p.q_sb + h * p.q_sh;
    const T* k = static_cast<const T*>(p.k) + b * p.k_sb + h * p.k_sh;
    const T* v = static_cast<const T*>(p.v) + b * p.v_sb + h * p.v_sh;
    const T* o = static_cast<const T*>(p.o) + b * p.o_sb + h * p.o_sh;
    const T* dout = static_cast<const T*>(p.dout) + b * p.do_sb + h * p.do_sh;
    const float* lse = p.lse + static_cast<int64_t>(bh) * p.N;
    stage<T, D>(sK, k, p.k_si, k0, p.Nk);
    stage<T, D>(sV, v, p.v_si, k0, p.Nk);
    // thread t accumulates key row j = t / 4, columns c = t % 4 + 4 cc
    const int j = threadIdx.x >> 2, cg = threadIdx.x & 3;
    float dk[D / 4], dv[D / 4];
#pragma unroll
    for (int cc = 0; cc < D / 4; ++cc) dk[cc] = dv[cc] = 0.f;
    // queries that see at least one of these keys: i >= k0 - causal_off
    int q_first = 0;
    if (CAUSAL) q_first = max(0, k0 - p.causal_off) / kRows * kRows;
    for (int q0 = q_first; q0 < p.N; q0 += kRows) {
        __syncthreads();   // previous tile's readers are done with sQ, sdO, sP, sdS
        stage<T, D>(sQ, q, p.q_si, q0, p.N);
        stage<T, D>(sdO, dout, p.do_si, q0, p.N);
        __syncthreads();
        row_stats<T, D>(sD, sL, sdO, o, p.o_si, lse, q0, p.N);
        __syncthreads();
        tile_p_ds<D, CAUSAL>(sQ, sK, sV, sdO, sD, sL, sP, sdS, q0, k0, p);
        __syncthreads();
        for (int i = 0; i < kRows; ++i) {
            const float pv = sP[i * (kRows + 1) + j], dsv = sdS[i * (kRows + 1) + j];
#pragma unroll
            for (int cc = 0; cc < D / 4; ++cc) {
                const int c = cg + 4 * cc;
                dv[cc] = fmaf(pv, sdO[i * (D + 1) + c], dv[cc]);
                dk[cc] = fmaf(dsv, sQ[i * (D + 1) + c], dk[cc]);
            }
        }
    }
    if (k0 + j < p.Nk) {
        T* dkr = static_cast<T*>(p.dk) + b * p.dk_sb + h * p.dk_sh + static_cast<int64_t>(k0 + j) * p.dk_si;
        T* dvr = static_cast<T*>(p.dv) + b * p.dv_sb + h * p.dv_sh + static_cast<int64_t>(k0 + j) * p.dv_si;
#pragma unroll
        for (int cc = 0; cc < D / 4; ++cc) {
            dkr[cg + 4 * cc] = cvt<T>(p.scale * dk[cc]);
            dvr[cg + 4 * cc] = cvt<T>(dv[cc]);
        }
    }
}

// ----------------------------------------------------------------------------- dQ
template <typename T, int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1) attn_bwd_dq_kernel(const BwdParams p) {
    extern __shared__ float smem[];
    using S = BwdSmem<D>;
    float *sQ = smem, *sdO = sQ + S::kTile, *sK = sdO + S::kTile, *sV = sK + S::kTile;
    float *sP = sV + S::kTile, *sdS = sP + S::kSq, *sD = sdS + S::kSq, *sL = sD + kRows;
    const int q0 = blockIdx.x * kRows;
    const int bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
    const T* q = static_cast<const T*>(p.q) + b * p.q_sb + h * p.q_sh;
    const T* k = static_cast<const T*>(p.k) + b * p.k_sb + h * p.k_sh;
    const T* v = static_cast<const T*>(p.v) + b * p.v_sb + h * p.v_sh;
    const T* o = static_cast<const T*>(p.o) + b * p.o_sb + h * p.o_sh;
    const T* dout = static_cast<const T*>(p.dout) + b * p.do_sb + h * p.do_sh;
    const float* lse = p.lse + static_cast<int64_t>(bh) * p.N;
    stage<T, D>(sQ, q, p.q_si, q0, p.N);
    stage<T, D>(sdO, dout, p.do_si, q0, p.N);
    __syncthreads();
    row_stats<T, D>(sD, sL, sdO, o, p.o_si, lse, q0, p.N);
    // thread t accumulates query row i = t / 4, columns c = t % 4 + 4 cc
    const int i = threadIdx.x >> 2, cg = threadIdx.x & 3;
    float dq[D / 4];
#pragma unroll
    for (int cc = 0; cc < D / 4; ++cc) dq[cc] = 0.f;
    // keys seen by at least one of these rows: j <= q0 + 63 + causal_off
    int k_end = p.Nk;
    if (CAUSAL) k_end = min(p.Nk, max(0, q0 + kRows + p.causal_off));
    for (int k0 = 0; k0 < k_end; k0 += kRows) {
        __syncthreads();   // previous tile's readers are done with sK, sV, sdS
        stage<T, D>(sK, k, p.k_si, k0, p.Nk);
        stage<T, D>(sV, v, p.v_si, k0, p.Nk);
        __syncthreads();
        tile_p_ds<D, CAUSAL>(sQ, sK, sV, sdO, sD, sL, sP, sdS, q0, k0, p);
        __syncthreads();
        for (int jj = 0; jj < kRows; ++jj) {
            const float dsv = sdS[i * (kRows + 1) + jj];
#pragma unroll
            for (int cc = 0; cc < D / 4; ++cc) dq[cc] = fmaf(dsv, sK[jj * (D + 1) + cg + 4 * cc], dq[cc]);
        }
    }
    if (q0 + i < p.N) {
        T* dqr = static_cast<T*>(p.dq) + b * p.dq_sb + h * p.dq_sh + static_cast<int64_t>(q0 + i) * p.dq_si;
#pragma unroll
        for (int cc = 0; cc < D / 4; ++cc) dqr[cg + 4 * cc] = cvt<T>(p.scale * dq[cc]);
    }
}

}  // namespace bwd
}  // namespace attn
