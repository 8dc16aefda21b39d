// attn_bwd_tc.cuh -- tensor-core backward of the exact attention forward (sm_100a).
//
// Gradients of O = softmax(scale Q K^T [causal]) V for an upstream dO, with S and P rebuilt
// tile by tile from Q, K and the forward's logsumexp (aiinarabic.com "flash-attention",
// Equation (1) and its recomputation section):
//
//     P  = exp(scale S - lse),  S = Q K^T masked
//     dV = P^T dO,   dP = dO V^T,   dS = P * (dP - D),  D_i = sum_c dO_ic O_ic
//     dQ = scale dS K,   dK = scale dS^T Q
//
// Three launches, no atomics:
//   bwd_prep_kernel   D_i for every query row, written as an fp32 at the start of dQ's row i
//                     (dQ's storage carries D until the dQ kernel overwrites that row);
//   bwd_dkdv_kernel   one CTA per 128-key block: for each 64-query block that sees it,
//                     S^T = K Q^T and dP^T = V dO^T on the tensor core into tensor memory
//                     (128 lanes = keys), P^T and dS^T by the four warps (thread = key row),
//                     stored back as 16-bit A operands over S^T and dP^T, then
//                     dV += P^T dO and dK += dS^T Q accumulate in tensor memory;
//   bwd_dq_kernel     one CTA per 128-query block: for each 64-key block it sees, S = Q K^T and
//                     dP = dO V^T, dS by the warps (thread = query row), dQ += dS K.
// Each CTA takes 256 tensor-memory columns (512 for the dK/dV kernel at d = 128), so two CTAs
// share an SM and one's elementwise phase overlaps the other's MMAs.  Every mbarrier wait is
// bounded; a timeout sets the status word, every thread leaves at the next block barrier, and
// the CTA drains its TMA loads and MMAs before it frees tensor memory.
#pragma once

#include <type_traits>

#include "sm100.cuh"

namespace attn {
namespace bwdtc {

constexpr int kThreads = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusCheck = 2u;     // debug builds: an index or range check failed (ATTN_CHECK)
constexpr unsigned long long kDrainLimit = 1ull << 32;

struct Params {
    int B, H, N, Nk;
    int causal_off;              // Nk - N: query i sees key j iff j <= i + causal_off (causal)
    float scale, scale_log2;
    const void* o;
    int64_t o_sb, o_sh, o_si;
    const void* dout;
    int64_t do_sb, do_sh, do_si;
    const float* lse;            // [B*H*N]
    void* dq;                    // also carries D_i (fp32 at each row's start) between launches
    int64_t dq_sb, dq_sh, dq_si;
    void* dk;
    int64_t dk_sb, dk_sh, dk_si;
    void* dv;
    int64_t dv_sb, dv_sh, dv_si;
    unsigned long long wait_limit;
    unsigned int* status;
    // score modifications (MODS builds): s <- scale s - slope_h |i + causal_off - j|, then
    // softcap c tanh(s / c) (dS picks up its derivative 1 - tanh^2), then keys
    // j < i + causal_off - window_left masked
    const float* alibi;          // nullable [H]
    float softcap;               // > 0: on
    int window_left;             // >= 0: on
};

// One score with the modifications: returns the modified score (natural units) and the
// softcap's derivative in *deriv (1 when off).
__device__ __forceinline__ float mod_score(float s_scaled, float slope, float dist, float cap, float* deriv) {
    float x = fmaf(-slope, fabsf(dist), s_scaled);
    if (cap > 0.f) {
        const float t = tanhf(x / cap);
        *deriv = 1.f - t * t;
        return cap * t;
    }
    *deriv = 1.f;
    return x;
}

// A tile of R rows x D 16-bit columns in the layout TMA writes: D/64 atoms of R rows x 128 bytes
// (128-byte swizzle), or for D = 32 one atom of R rows x 64 bytes (64-byte swizzle).
template <int D, int R>
struct Tile {
    static constexpr int kAtomCols = (D >= 64) ? 64 : 32;
    static constexpr int kNumAtoms = D / kAtomCols;
    static constexpr int kRowBytes = kAtomCols * 2;
    static constexpr int kAtomBytes = R * kRowBytes;
    static constexpr int kBytes = kNumAtoms * kAtomBytes;
    static constexpr uint32_t kLayout = (D >= 64) ? 2u : 4u;
    static constexpr uint32_t kSBO = 8 * kRowBytes;
    // operand whose reduction dimension is the column (K-major): offset of the kk-th 16-column step
    static __device__ __forceinline__ uint32_t kstep(int kk) {
        return static_cast<uint32_t>((((kk * 16) / kAtomCols) * kAtomBytes + ((kk * 16) % kAtomCols) * 2) >> 4);
    }
    // operand whose reduction dimension is the row (N-major): offset of the kk-th 16-row step
    static __device__ __forceinline__ uint32_t rstep(int kk) {
        return static_cast<uint32_t>((kk * 16 * kRowBytes) >> 4);
    }
    static __device__ __forceinline__ uint64_t desc_k(const void* p) {
        return sm100::smem_desc(sm100::smem_u32(p), 16, kSBO, kLayout);
    }
    static __device__ __forceinline__ uint64_t desc_n(const void* p) {
        return sm100::smem_desc(sm100::smem_u32(p), kAtomBytes, kSBO, kLayout);
    }
    static __device__ __forceinline__ void load(void* dst, const CUtensorMap* map, uint64_t* bar, int row0, int h,
                                                int b, uint64_t pol) {
#pragma unroll
        for (int a = 0; a < kNumAtoms; ++a)
            sm100::tma_load_4d(static_cast<uint8_t*>(dst) + a * kAtomBytes, map, bar, a * kAtomCols, row0, h, b, pol);
    }
};

// Bounded wait: false after `limit` cycles (status word + abort flag) or once another thread aborted.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, int* abort_flag, const Params& p) {
    const uint32_t a = sm100::smem_u32(bar);
    if (sm100::mbar_try_wait(a, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (sm100::mbar_try_wait(a, parity)) return true;
        if (*reinterpret_cast<volatile int*>(abort_flag)) return false;
        if (static_cast<unsigned long long>(clock64() - t0) > p.wait_limit) {
            atomicOr(p.status, kStatusTimeout);
            *reinterpret_cast<volatile int*>(abort_flag) = 1;
            return false;
        }
    }
}

// Bounded wait used only while draining on exit.
__device__ __forceinline__ void drain_bar(uint64_t* bar, uint32_t parity, const Params& p) {
    const uint32_t a = sm100::smem_u32(bar);
    const long long t0 = clock64();
    while (!sm100::mbar_try_wait(a, parity)) {
        if (static_cast<unsigned long long>(clock64() - t0) > kDrainLimit) {
            atomicOr(p.status, kStatusTimeout);
            return;
        }
    }
}

template <typename T>
__device__ __forceinline__ const uint8_t* row_ptr(const void* base, int64_t sb, int64_t sh, int64_t si, int b, int h,
                                                  int64_t i) {
    return static_cast<const uint8_t*>(base) + (b * sb + h * sh + i * si) * static_cast<int64_t>(sizeof(T));
}

// D_i = sum_c dO_ic O_ic in fp32, one group of D/8 threads per row (16 bytes each), written as an
// fp32 at the start of dQ's row i.
template <typename T, int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const Params p) {
    constexpr int G = D / 8;                                   // threads per row
    const int64_t rows = static_cast<int64_t>(p.B) * p.H * p.N;
    const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / G;
    const int c = threadIdx.x % G;
    float acc = 0.f;
    int b = 0, h = 0;
    int64_t i = 0;
    if (r < rows) {
        i = r % p.N;
        h = static_cast<int>((r / p.N) % p.H);
        b = static_cast<int>(r / (static_cast<int64_t>(p.N) * p.H));
        const uint4 ov = *reinterpret_cast<const uint4*>(row_ptr<T>(p.o, p.o_sb, p.o_sh, p.o_si, b, h, i) + c * 16);
        const uint4 dv = *reinterpret_cast<const uint4*>(row_ptr<T>(p.dout, p.do_sb, p.do_sh, p.do_si, b, h, i) + c * 16);
        const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w}, dw[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float o0, o1, d0, d1;
            sm100::unpack2<T>(ow[q], o0, o1);
            sm100::unpack2<T>(dw[q], d0, d1);
            acc = fmaf(o0, d0, fmaf(o1, d1, acc));
        }
    }
#pragma unroll
    for (int off = G / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (r < rows && c == 0)
        *reinterpret_cast<float*>(const_cast<uint8_t*>(row_ptr<T>(p.dq, p.dq_sb, p.dq_sh, p.dq_si, b, h, i))) = acc;
}

// Rounds a row of `n` fp32 accumulators (times `mul`) to T and stores it (16 bytes at a time).
template <typename T, int N>
__device__ __forceinline__ void store_row(uint8_t* dst, const uint32_t (&r)[N], float mul) {
#pragma unroll
    for (int v = 0; v < N / 8; ++v) {
        uint4 w;
        w.x = sm100::pack2<T>(__uint_as_float(r[8 * v + 0]) * mul, __uint_as_float(r[8 * v + 1]) * mul);
        w.y = sm100::pack2<T>(__uint_as_float(r[8 * v + 2]) * mul, __uint_as_float(r[8 * v + 3]) * mul);
        w.z = sm100::pack2<T>(__uint_as_float(r[8 * v + 4]) * mul, __uint_as_float(r[8 * v + 5]) * mul);
        w.w = sm100::pack2<T>(__uint_as_float(r[8 * v + 6]) * mul, __uint_as_float(r[8 * v + 7]) * mul);
        *reinterpret_cast<uint4*>(dst + v * 16) = w;
    }
}

// Reads D fp32 columns of this warp's lanes starting at column `col` and stores them as a row.
template <typename T, int D>
__device__ __forceinline__ void tmem_row_to_global(uint32_t taddr, uint8_t* dst, bool store, float mul) {
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        sm100::tmem_ld32(taddr + c * 32, r);
        sm100::tmem_wait_ld(r);
        if (store) store_row<T, 32>(dst + c * 64, r, mul);
    }
}

template <typename T, int D>
__device__ __forceinline__ void zero_row(uint8_t* dst) {
#pragma unroll
    for (int v = 0; v < D / 8; ++v) *reinterpret_cast<uint4*>(dst + v * 16) = make_uint4(0u, 0u, 0u, 0u);
}

// ------------------------------------------------------------------------------------ dK, dV
template <int D>
struct DkdvCfg {
    using TK = Tile<D, 128>;       // K, V: the CTA's 128 keys
    using TQ = Tile<D, 64>;        // Q, dO: one 64-query block, two stages
    static constexpr uint32_t kCols = (D == 128) ? 512u : 256u;
    static constexpr uint32_t kColS = 0, kColDP = 64, kColDV = 128, kColDK = 128 + D;
    static constexpr int kOffK = 0, kOffV = TK::kBytes, kOffQ = 2 * TK::kBytes, kOffDO = kOffQ + 2 * TQ::kBytes;
    static constexpr int kBytes = kOffDO + 2 * TQ::kBytes;
    // at least 80 KB so that no more than two CTAs (2 x 256 columns of tensor memory) share an SM
    static constexpr int kDynBytes = (kBytes + 1024 > 80 * 1024) ? kBytes + 1024 : 80 * 1024;
};

template <typename T, int D, bool CAUSAL, bool MODS = false>
__global__ void __launch_bounds__(kThreads, 2)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const Params p) {
    using namespace sm100;
    using C = DkdvCfg<D>;
    using TK = typename C::TK;
    using TQ = typename C::TQ;
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;

    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bar_kv, bar_qdo[2], bar_s, bar_free[2], bar_end;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    __shared__ float sL[64], sDr[64];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sdO = smem + C::kOffDO;

    const int t = threadIdx.x, warp = t >> 5;
    const int bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
    const int k0 = blockIdx.x * 128;
    const int nqb = (p.N + 63) / 64;
    int m0 = 0;                    // first query block with a row that sees a key of this block
    if (CAUSAL) {
        const int first = k0 - p.causal_off;
        m0 = first <= 0 ? 0 : min(nqb, first / 64);
    }
    int m_end = nqb;               // a left window hides these keys from queries far below them
    if (MODS && p.window_left >= 0) {
        const int last_q = k0 + 127 - p.causal_off + p.window_left;
        m_end = last_q < 0 ? 0 : min(nqb, last_q / 64 + 1);
    }
    const int nit = m_end > m0 ? m_end - m0 : 0;
    ATTN_CHECK(p.status, m0 >= 0 && m0 <= nqb && m_end >= 0 && m_end <= nqb && k0 < p.Nk && b < p.B);

    if (t == 0) {
        mbar_init(&bar_kv, 1);
        mbar_init(&bar_s, 1);
        mbar_init(&bar_end, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar_qdo[s], 1);
            mbar_init(&bar_free[s], 1);
        }
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, C::kCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    ATTN_CHECK(p.status, (tmem >> 16) == 0u && (tmem & 0xFFFFu) + C::kCols <= 512u);
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    int* abort_p = &abort_flag;

    // loads issued / waited per barrier (thread 0), for the drain on exit
    int qdo_issued[2] = {0, 0}, qdo_waited[2] = {0, 0};
    bool kv_issued = false, kv_waited = false;
    const uint64_t pol_once = policy_evict_first();   // K, V: read by this CTA only
    const uint64_t pol_many = policy_evict_last();    // Q, dO: read by every key block of the head
    auto load_qdo = [&](int it) {
        const int s = it & 1;
        mbar_arrive_expect_tx(&bar_qdo[s], 2 * TQ::kBytes);
        TQ::load(sQ + s * TQ::kBytes, &tm_q, &bar_qdo[s], (m0 + it) * 64, h, b, pol_many);
        TQ::load(sdO + s * TQ::kBytes, &tm_do, &bar_qdo[s], (m0 + it) * 64, h, b, pol_many);
        ++qdo_issued[s];
    };
    if (t == 0 && nit > 0) {
        mbar_arrive_expect_tx(&bar_kv, 2 * TK::kBytes);
        TK::load(sK, &tm_k, &bar_kv, k0, h, b, pol_once);
        TK::load(sV, &tm_v, &bar_kv, k0, h, b, pol_once);
        kv_issued = true;
        load_qdo(0);
    }

    constexpr uint32_t idesc_s = instr_desc_f16(kBF16, 128, 64, false);
    constexpr uint32_t idesc_o = instr_desc_f16(kBF16, 128, D, true);
    const float* lse_bh = p.lse + static_cast<int64_t>(bh) * p.N;
    const int kr = k0 + t;                          // this thread's key row
    bool ok = true;
    int it = 0;
    for (; it < nit; ++it) {
        const int s = it & 1, q0 = (m0 + it) * 64;
        if (t == 0 && ok) {
            if (it == 0) {
                ok = wait_bar(&bar_kv, 0, abort_p, p);
                kv_waited = ok;
            }
            if (ok) ok = wait_bar(&bar_qdo[s], (it >> 1) & 1, abort_p, p);
            if (ok) {
                ++qdo_waited[s];
                tc_fence_after();
                const uint64_t dk_ = TK::desc_k(sK), dv_ = TK::desc_k(sV);
                const uint64_t dq_ = TQ::desc_k(sQ + s * TQ::kBytes), ddo = TQ::desc_k(sdO + s * TQ::kBytes);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem + C::kColS, dk_ + TK::kstep(kk), dq_ + TQ::kstep(kk), idesc_s, kk > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem + C::kColDP, dv_ + TK::kstep(kk), ddo + TQ::kstep(kk), idesc_s, kk > 0 ? 1u : 0u);
                mma_commit(&bar_s);
            }
            // the next query block into the other stage, once dV/dK of the block before released it
            if (ok && it + 1 < nit) {
                if (it >= 1) ok = wait_bar(&bar_free[(it + 1) & 1], ((it - 1) >> 1) & 1, abort_p, p);
                if (ok) load_qdo(it + 1);
            }
        }
        __syncwarp();
        // lse (log2 units) and D of the block's 64 queries; columns past N are masked below
        if (t < 64) {
            const int qi = q0 + t;
            float l = 0.f, dd = 0.f;
            if (qi < p.N) {
                l = lse_bh[qi] * kLog2e;
                dd = *reinterpret_cast<const float*>(row_ptr<T>(p.dq, p.dq_sb, p.dq_sh, p.dq_si, b, h, qi));
            }
            sL[t] = l;
            sDr[t] = dd;
        }
        ok = __syncthreads_and(ok) != 0;
        if (!ok) break;
        ok = wait_bar(&bar_s, it & 1, abort_p, p);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc_fence_after();
            uint32_t rs[2][32], rd[2][32];
            tmem_ld32(tmem + lane_off + C::kColS, rs[0]);
            tmem_ld32(tmem + lane_off + C::kColS + 32, rs[1]);
            tmem_ld32(tmem + lane_off + C::kColDP, rd[0]);
            tmem_ld32(tmem + lane_off + C::kColDP + 32, rd[1]);
            tmem_wait_ld(rs[0]);
            tmem_wait_ld(rs[1]);
            tmem_wait_ld(rd[0]);
            tmem_wait_ld(rd[1]);
            // key kr is seen by query q iff q < N and (causal) kr <= q + causal_off
            int qlim = min(p.N - q0, 64);
            const int qmin = CAUSAL ? kr - p.causal_off - q0 : -1;     // first column that sees key kr
            if (MODS && p.window_left >= 0) qlim = min(qlim, kr - p.causal_off + p.window_left - q0 + 1);
            const float slope = (MODS && p.alibi != nullptr) ? p.alibi[h] : 0.f;
            uint32_t pk[32], dk2[32];
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
                const int hh = c >> 5, cc = c & 31;
                float x0, x1, d0 = 1.f, d1 = 1.f;
                if constexpr (MODS) {
                    const float dist = static_cast<float>(q0 + c + p.causal_off - kr);
                    x0 = fmaf(mod_score(__uint_as_float(rs[hh][cc]) * p.scale, slope, dist, p.softcap, &d0), kLog2e, -sL[c]);
                    x1 = fmaf(mod_score(__uint_as_float(rs[hh][cc + 1]) * p.scale, slope, dist + 1.f, p.softcap, &d1),
                              kLog2e, -sL[c + 1]);
                } else {
                    x0 = fmaf(__uint_as_float(rs[hh][cc]), p.scale_log2, -sL[c]);
                    x1 = fmaf(__uint_as_float(rs[hh][cc + 1]), p.scale_log2, -sL[c + 1]);
                }
                const bool v0 = c < qlim && c >= qmin, v1 = c + 1 < qlim && c + 1 >= qmin;
                const float p0 = v0 ? ex2_approx(x0) : 0.f, p1 = v1 ? ex2_approx(x1) : 0.f;
                const float g0 = p0 * (__uint_as_float(rd[hh][cc]) - sDr[c]) * d0;
                const float g1 = p1 * (__uint_as_float(rd[hh][cc + 1]) - sDr[c + 1]) * d1;
                pk[c >> 1] = pack2<T>(p0, p1);
                dk2[c >> 1] = pack2<T>(g0, g1);
            }
            tmem_st32(tmem + lane_off + C::kColS, pk);       // P^T over S^T
            tmem_st32(tmem + lane_off + C::kColDP, dk2);     // dS^T over dP^T
            tmem_wait_st();
        }
        tc_fence_before();
        ok = __syncthreads_and(ok) != 0;
        if (!ok) break;
        if (t == 0) {
            tc_fence_after();
            const uint64_t qn = TQ::desc_n(sQ + s * TQ::kBytes), don = TQ::desc_n(sdO + s * TQ::kBytes);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_ts(tmem + C::kColDV, tmem + C::kColS + kk * 8, don + TQ::rstep(kk), idesc_o,
                       (it > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_ts(tmem + C::kColDK, tmem + C::kColDP + kk * 8, qn + TQ::rstep(kk), idesc_o,
                       (it > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&bar_free[s]);
        }
        __syncwarp();
    }

    // every MMA and load completes before the accumulators are read and tensor memory is freed
    if (t == 0) {
        mma_commit(&bar_end);
        drain_bar(&bar_end, 0, p);
        if (kv_issued && !kv_waited) drain_bar(&bar_kv, 0, p);
        for (int s = 0; s < 2; ++s)
            if (qdo_issued[s] > qdo_waited[s]) drain_bar(&bar_qdo[s], (qdo_issued[s] - 1) & 1, p);
    }
    tc_fence_before();
    ok = __syncthreads_and(ok) != 0;
    tc_fence_after();
    if (ok) {
        const bool row_ok = kr < p.Nk;
        uint8_t* dvrow = const_cast<uint8_t*>(row_ptr<T>(p.dv, p.dv_sb, p.dv_sh, p.dv_si, b, h, row_ok ? kr : 0));
        uint8_t* dkrow = const_cast<uint8_t*>(row_ptr<T>(p.dk, p.dk_sb, p.dk_sh, p.dk_si, b, h, row_ok ? kr : 0));
        if (nit > 0) {
            tmem_row_to_global<T, D>(tmem + lane_off + C::kColDV, dvrow, row_ok, 1.f);
            tmem_row_to_global<T, D>(tmem + lane_off + C::kColDK, dkrow, row_ok, p.scale);
        } else if (row_ok) {
            zero_row<T, D>(dvrow);
            zero_row<T, D>(dkrow);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kCols);
    }
}

// ------------------------------------------------------------------------------------ dQ
template <int D>
struct DqCfg {
    using TQ = Tile<D, 128>;       // Q, dO: the CTA's 128 queries
    using TK = Tile<D, 64>;        // K, V: one 64-key block, two stages
    static constexpr uint32_t kCols = 256u;
    static constexpr uint32_t kColS = 0, kColDP = 64, kColDQ = 128;
    static_assert(kColDQ + D <= kCols, "tensor memory budget");
    static constexpr int kOffQ = 0, kOffDO = TQ::kBytes, kOffK = 2 * TQ::kBytes, kOffV = kOffK + 2 * TK::kBytes;
    static constexpr int kBytes = kOffV + 2 * TK::kBytes;
    static constexpr int kDynBytes = (kBytes + 1024 > 80 * 1024) ? kBytes + 1024 : 80 * 1024;
};

template <typename T, int D, bool CAUSAL, bool MODS = false>
__global__ void __launch_bounds__(kThreads, 2)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const Params p) {
    using namespace sm100;
    using C = DqCfg<D>;
    using TK = typename C::TK;
    using TQ = typename C::TQ;
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;

    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bar_q, bar_kv[2], bar_s, bar_free[2], bar_end;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sdO = smem + C::kOffDO;
    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;

    const int t = threadIdx.x, warp = t >> 5;
    const int bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
    // causal: later query blocks see more keys; launch them first
    const int q0 = (CAUSAL ? gridDim.x - 1 - blockIdx.x : blockIdx.x) * 128;
    const int qi = q0 + t;                          // this thread's query row
    const int nkb_all = (p.Nk + 63) / 64;
    int nkb = nkb_all;                              // key blocks with a key some row of the block sees
    if (CAUSAL) {
        const int last = q0 + 127 + p.causal_off;
        nkb = last < 0 ? 0 : min(nkb_all, last / 64 + 1);
    }
    int kb_first = 0;              // a left window hides the key blocks before the first row's window
    if (MODS && p.window_left >= 0) {
        const int lo_key = q0 + p.causal_off - p.window_left;
        kb_first = lo_key > 0 ? min(nkb, lo_key / 64) : 0;
    }
    ATTN_CHECK(p.status, kb_first >= 0 && kb_first <= nkb && nkb <= nkb_all && q0 < p.N + 127 && b < p.B);

    if (t == 0) {
        mbar_init(&bar_q, 1);
        mbar_init(&bar_s, 1);
        mbar_init(&bar_end, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar_kv[s], 1);
            mbar_init(&bar_free[s], 1);
        }
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, C::kCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    ATTN_CHECK(p.status, (tmem >> 16) == 0u && (tmem & 0xFFFFu) + C::kCols <= 512u);
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    int* abort_p = &abort_flag;

    // this row's lse (log2 units) and D, read before the row of dQ's storage is overwritten
    const bool row_ok = qi < p.N;
    uint8_t* dqrow = const_cast<uint8_t*>(row_ptr<T>(p.dq, p.dq_sb, p.dq_sh, p.dq_si, b, h, row_ok ? qi : 0));
    float lse2 = 0.f, drow = 0.f;
    if (row_ok) {
        lse2 = p.lse[static_cast<int64_t>(bh) * p.N + qi] * kLog2e;
        drow = *reinterpret_cast<const float*>(dqrow);
    }

    int kv_issued[2] = {0, 0}, kv_waited[2] = {0, 0};
    bool q_issued = false, q_waited = false;
    const uint64_t pol_once = policy_evict_first();
    const uint64_t pol_many = policy_evict_last();
    const int nkv = nkb - kb_first;                 // key blocks this CTA visits
    auto load_kv = [&](int it) {
        const int s = it & 1;
        mbar_arrive_expect_tx(&bar_kv[s], 2 * TK::kBytes);
        TK::load(sK + s * TK::kBytes, &tm_k, &bar_kv[s], (kb_first + it) * 64, h, b, pol_many);
        TK::load(sV + s * TK::kBytes, &tm_v, &bar_kv[s], (kb_first + it) * 64, h, b, pol_many);
        ++kv_issued[s];
    };
    if (t == 0 && nkv > 0) {
        mbar_arrive_expect_tx(&bar_q, 2 * TQ::kBytes);
        TQ::load(sQ, &tm_q, &bar_q, q0, h, b, pol_once);
        TQ::load(sdO, &tm_do, &bar_q, q0, h, b, pol_once);
        q_issued = true;
        load_kv(0);
    }

    constexpr uint32_t idesc_s = instr_desc_f16(kBF16, 128, 64, false);
    constexpr uint32_t idesc_o = instr_desc_f16(kBF16, 128, D, true);
    bool ok = true;
    for (int it = 0; it < nkv; ++it) {
        const int s = it & 1, kb0 = (kb_first + it) * 64;
        if (t == 0 && ok) {
            if (it == 0) {
                ok = wait_bar(&bar_q, 0, abort_p, p);
                q_waited = ok;
            }
            if (ok) ok = wait_bar(&bar_kv[s], (it >> 1) & 1, abort_p, p);
            if (ok) {
                ++kv_waited[s];
                tc_fence_after();
                const uint64_t dq_ = TQ::desc_k(sQ), ddo = TQ::desc_k(sdO);
                const uint64_t dk_ = TK::desc_k(sK + s * TK::kBytes), dv_ = TK::desc_k(sV + s * TK::kBytes);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem + C::kColS, dq_ + TQ::kstep(kk), dk_ + TK::kstep(kk), idesc_s, kk > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem + C::kColDP, ddo + TQ::kstep(kk), dv_ + TK::kstep(kk), idesc_s, kk > 0 ? 1u : 0u);
                mma_commit(&bar_s);
            }
            if (ok && it + 1 < nkv) {
                if (it >= 1) ok = wait_bar(&bar_free[(it + 1) & 1], ((it - 1) >> 1) & 1, abort_p, p);
                if (ok) load_kv(it + 1);
            }
        }
        __syncwarp();
        ok = wait_bar(&bar_s, it & 1, abort_p, p);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc_fence_after();
            uint32_t rs[2][32], rd[2][32];
            tmem_ld32(tmem + lane_off + C::kColS, rs[0]);
            tmem_ld32(tmem + lane_off + C::kColS + 32, rs[1]);
            tmem_ld32(tmem + lane_off + C::kColDP, rd[0]);
            tmem_ld32(tmem + lane_off + C::kColDP + 32, rd[1]);
            tmem_wait_ld(rs[0]);
            tmem_wait_ld(rs[1]);
            tmem_wait_ld(rd[0]);
            tmem_wait_ld(rd[1]);
            // key kb0 + c is seen iff it is < Nk and (causal) <= qi + causal_off; rows past N are
            // never stored, and their zero Q and dO rows contribute nothing to other rows
            int lim = min(p.Nk - kb0, 64);
            if (CAUSAL) lim = min(lim, qi + p.causal_off - kb0 + 1);
            const int lo = (MODS && p.window_left >= 0) ? qi + p.causal_off - p.window_left - kb0 : 0;
            const float slope = (MODS && p.alibi != nullptr) ? p.alibi[h] : 0.f;
            uint32_t pk[32];
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
                const int hh = c >> 5, cc = c & 31;
                float x0, x1, d0 = 1.f, d1 = 1.f;
                if constexpr (MODS) {
                    const float dist = static_cast<float>(qi + p.causal_off - kb0 - c);
                    x0 = fmaf(mod_score(__uint_as_float(rs[hh][cc]) * p.scale, slope, dist, p.softcap, &d0), kLog2e, -lse2);
                    x1 = fmaf(mod_score(__uint_as_float(rs[hh][cc + 1]) * p.scale, slope, dist - 1.f, p.softcap, &d1),
                              kLog2e, -lse2);
                } else {
                    x0 = fmaf(__uint_as_float(rs[hh][cc]), p.scale_log2, -lse2);
                    x1 = fmaf(__uint_as_float(rs[hh][cc + 1]), p.scale_log2, -lse2);
                }
                const float p0 = (c < lim && c >= lo) ? ex2_approx(x0) : 0.f;
                const float p1 = (c + 1 < lim && c + 1 >= lo) ? ex2_approx(x1) : 0.f;
                pk[c >> 1] = pack2<T>(p0 * (__uint_as_float(rd[hh][cc]) - drow) * d0,
                                      p1 * (__uint_as_float(rd[hh][cc + 1]) - drow) * d1);
            }
            tmem_st32(tmem + lane_off + C::kColS, pk);       // dS over S
            tmem_wait_st();
        }
        tc_fence_before();
        ok = __syncthreads_and(ok) != 0;
        if (!ok) break;
        if (t == 0) {
            tc_fence_after();
            const uint64_t kn = TK::desc_n(sK + s * TK::kBytes);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_ts(tmem + C::kColDQ, tmem + C::kColS + kk * 8, kn + TK::rstep(kk), idesc_o,
                       (it > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&bar_free[s]);
        }
        __syncwarp();
    }

    if (t == 0) {
        mma_commit(&bar_end);
        drain_bar(&bar_end, 0, p);
        if (q_issued && !q_waited) drain_bar(&bar_q, 0, p);
        for (int s = 0; s < 2; ++s)
            if (kv_issued[s] > kv_waited[s]) drain_bar(&bar_kv[s], (kv_issued[s] - 1) & 1, p);
    }
    tc_fence_before();
    ok = __syncthreads_and(ok) != 0;
    tc_fence_after();
    if (ok) {
        if (nkv > 0) tmem_row_to_global<T, D>(tmem + lane_off + C::kColDQ, dqrow, row_ok, p.scale);
        else if (row_ok) zero_row<T, D>(dqrow);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kCols);
    }
}

}  // namespace bwdtc
}  // namespace attn
