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
//                     (128 lanes = keys), P^T and dS^T by an elementwise group (thread = key
//                     row), stored back as 16-bit A operands over S^T and dP^T, then
//                     dV += P^T dO and dK += dS^T Q accumulate in tensor memory;
//   bwd_dq_kernel     one CTA per 128-query block: for each 64-key block it sees, S = Q K^T and
//                     dP = dO V^T, dS by an elementwise group (thread = query row), dQ += dS K.
// In both, two elementwise groups take alternate column blocks, a TMA warp streams the column
// blocks' operands through a ring of stages and one thread issues the tensor-core work, so one
// group's products run while the other group works (roles below).  A CTA takes all 512
// tensor-memory columns, one CTA per SM.  Every mbarrier wait is bounded; a timeout sets the
// status word, the groups stop at their next group barrier, and the CTA drains its TMA loads
// and tensor-core work before it frees tensor memory.
#pragma once

#include <type_traits>

#include "sm100.cuh"

namespace attn {
namespace bwdtc {

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

// ------------------------------------------------------------------------------------ roles
// Both gradient kernels take a CTA's 128-row block (keys for dK/dV, queries for dQ) against a
// sequence of 64-wide blocks of the other side, with the warps split by role:
//   warps 0-3 (group 0), 4-7 (group 1)   elementwise work of the even / odd column blocks,
//                                        thread = row of the 128-row block (= tensor-memory lane)
//   warp 8                               tensor-core issuer (one thread)
//   warp 9                               TMA producer (one thread), a ring of kStages stages
//   warps 10-11                          idle (they complete warpgroup 2, whose registers
//                                        setmaxnreg hands to the elementwise groups)
// Column block m's two products (64 columns each) go into column set m % kSets (128 columns;
// 3 sets where the tensor memory holds them beside the accumulators, else 2), where group m % 2
// overwrites them with the 16-bit operands of the accumulating products.  The issuer's order
// is: the products of blocks 0 .. kSets-1, then per block m the accumulating products of block
// m (once group m % 2 stored its operands in the set) followed by the products of block m + kSets into
// the set just read, so that a group finds its next block's products ready (3 sets) or the
// tensor core runs one group's products while the other group works (2 sets).  Tensor-core
// operations of one thread execute in issue order, so block m + kSets's products overwrite
// the set only after block m's accumulating products have read it.
constexpr int kWarps = 12;
constexpr int kThreadsPP = 32 * kWarps;
constexpr int kMmaWarp = 8, kTmaWarp = 9;
// Register split (launch: 65536 / 384 threads = 168 each): warpgroup 2 gives up to 56, the two
// elementwise groups take 224 (128 x 56 + 256 x 224 = 384 x 168).
constexpr int kRegsGroup = 224, kRegsOther = 56;

// Named barrier `id` over the 128 threads of one elementwise group; returns the AND of `pred`
// over them, so that a timeout seen by one thread stops the whole group at the same block.
__device__ __forceinline__ bool group_sync_and(uint32_t id, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred)), "r"(id)
        : "memory");
    return r != 0;
}

// Shared-memory operand ring and the barriers of one CTA.
template <int ST>
struct PipeBars {
    uint64_t row_full;             // the CTA's own 128-row operands (K, V or Q, dO) in shared memory
    uint64_t row_tmem;             // dQ: Q and dO copied into tensor memory (both groups, 256 arrivals)
    uint64_t full[ST], empty[ST];  // column-block operand stages
    uint64_t s_full[3];            // column set c holds its block's two products (issuer commit)
    uint64_t p_ready[3];           // set c holds its block's 16-bit operands (the group's 128
                                   // arrivals; per set, not per group: with 3 sets a group can
                                   // finish its next block before the issuer read this one)
    uint64_t acc_done;             // every product issued has completed
};

template <int ST>
__device__ __forceinline__ void init_pipe(PipeBars<ST>& br) {
    sm100::mbar_init(&br.row_full, 1);
    sm100::mbar_init(&br.row_tmem, 256);
    for (int s = 0; s < ST; ++s) {
        sm100::mbar_init(&br.full[s], 1);
        sm100::mbar_init(&br.empty[s], 1);
    }
    for (int c = 0; c < 3; ++c) {
        sm100::mbar_init(&br.s_full[c], 1);
        sm100::mbar_init(&br.p_ready[c], 128);
    }
    sm100::mbar_init(&br.acc_done, 1);
    sm100::fence_barrier_init();
}

// TMA producer (one thread): the row block's two operands, then the column blocks' two operands
// through the ring; before returning it waits for every load it issued (a timeout elsewhere may
// have stopped the consumer).
template <int ST, typename TR, typename TC, typename RowLoad, typename ColLoad>
__device__ __forceinline__ void produce(PipeBars<ST>& br, int nit, int* abort_p, const Params& p, RowLoad row_load,
                                        ColLoad col_load) {
    sm100::mbar_arrive_expect_tx(&br.row_full, 2 * TR::kBytes);
    row_load(&br.row_full);
    int issued[ST];
    for (int s = 0; s < ST; ++s) issued[s] = 0;
    for (int m = 0; m < nit; ++m) {
        const int s = m % ST, use = m / ST;
        if (use > 0 && !wait_bar(&br.empty[s], (use - 1) & 1, abort_p, p)) break;
        sm100::mbar_arrive_expect_tx(&br.full[s], 2 * TC::kBytes);
        col_load(m, s, &br.full[s]);
        issued[s] = use + 1;
    }
    drain_bar(&br.row_full, 0, p);
    for (int s = 0; s < ST; ++s)
        if (issued[s] > 0) drain_bar(&br.full[s], (issued[s] - 1) & 1, p);
}

// Tensor-core issuer: the whole warp runs the loop, so that its waits and descriptor arithmetic
// are warp-uniform, and the elected lane `leader` issues.  It starts once `row_ready` completed
// (the row block's operands are in place).  products(s, col) fills the column set
// at `col` from stage s, accumulate(m, s, col) consumes it; the final commit on acc_done covers
// every product, and the warp waits for it before returning (the CTA frees tensor memory after).
template <int ST, int SETS, typename Products, typename Accumulate>
__device__ __forceinline__ void issue(PipeBars<ST>& br, uint64_t* row_ready, int nit, int* abort_p, const Params& p,
                                      bool leader, Products products, Accumulate accumulate) {
    auto W = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, wait_bar(bar, parity, abort_p, p));
    };
    bool ok = W(row_ready, 0);        // the row block's operands (row_full, or row_tmem for dQ)
    auto prod = [&](int m) -> bool {
        if (!W(&br.full[m % ST], (m / ST) & 1)) return false;
        sm100::tc_fence_after();
        products(m % ST, static_cast<uint32_t>(128 * (m % SETS)));
        if (leader) sm100::mma_commit(&br.s_full[m % SETS]);
        return true;
    };
    for (int m = 0; ok && m < SETS && m < nit; ++m) ok = prod(m);
    for (int m = 0; ok && m < nit; ++m) {
        if (!W(&br.p_ready[m % SETS], (m / SETS) & 1)) break;
        sm100::tc_fence_after();
        accumulate(m, m % ST, static_cast<uint32_t>(128 * (m % SETS)));
        if (leader) sm100::mma_commit(&br.empty[m % ST]);
        if (m + SETS < nit) ok = prod(m + SETS);
    }
    if (leader) sm100::mma_commit(&br.acc_done);
    drain_bar(&br.acc_done, 0, p);
}

// A shared-memory descriptor from its two 32-bit halves.  Offsets are added to the low half,
// whose address field (bits 0-13, address / 16) cannot carry out below 256 KB.
__device__ __forceinline__ uint64_t desc_at(uint32_t lo, uint32_t hi) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "r"(lo), "r"(hi));
    return d;
}
__device__ __forceinline__ uint32_t lo32(uint64_t d) { return static_cast<uint32_t>(d); }
__device__ __forceinline__ uint32_t hi32(uint64_t d) { return static_cast<uint32_t>(d >> 32); }

// ------------------------------------------------------------------------------------ dK, dV
template <int D>
struct DkdvCfg {
    using TK = Tile<D, 128>;       // K, V: the CTA's 128 keys
    using TQ = Tile<D, 64>;        // Q, dO: one 64-query block per stage
    static constexpr int kStages = (D == 128) ? 3 : 6;
    // three sets where tensor memory holds them beside dK and dV and the ring keeps loads two
    // blocks ahead of the products that read them
    static constexpr int kSets = (3 * 128 + 2 * D <= 512 && kStages >= 5) ? 3 : 2;
    static constexpr uint32_t kCols = 512u;
    static constexpr uint32_t kColDV = 128 * kSets, kColDK = 128 * kSets + D;   // after the sets
    static constexpr int kOffK = 0, kOffV = TK::kBytes, kOffQ = 2 * TK::kBytes;
    static constexpr int kOffDO = kOffQ + kStages * TQ::kBytes;
    static constexpr int kBytes = kOffDO + kStages * TQ::kBytes;
    // above half of an SM's shared memory: one CTA per SM, which takes all 512 columns
    static constexpr int kDynBytes = (kBytes + 1024 > 120 * 1024) ? kBytes + 1024 : 120 * 1024;
};

template <typename T, int D, bool CAUSAL, bool MODS = false>
__global__ void __launch_bounds__(kThreadsPP, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const Params p) {
    using namespace sm100;
    using C = DkdvCfg<D>;
    using TK = typename C::TK;
    using TQ = typename C::TQ;
    constexpr int ST = C::kStages;
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;

    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) PipeBars<ST> br;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    __shared__ __align__(16) float sL[2][2][64];     // -lse (log2 units) [group][buffer][query]
    __shared__ __align__(16) float sDr[2][2][64];    // -D
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sdO = smem + C::kOffDO;

    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
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
        init_pipe(br);
        abort_flag = 0;
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
    int* abort_p = &abort_flag;

    if (warp >= 8) {
        regs_dec<kRegsOther>();
        if (warp == kTmaWarp) {
            if (lane == 0 && nit > 0) {
                const uint64_t pol_once = policy_evict_first();   // K, V: read by this CTA only
                const uint64_t pol_many = policy_evict_last();    // Q, dO: read by every key block of the head
                produce<ST, TK, TQ>(
                    br, nit, abort_p, p,
                    [&](uint64_t* bar) {
                        TK::load(sK, &tm_k, bar, k0, h, b, pol_once);
                        TK::load(sV, &tm_v, bar, k0, h, b, pol_once);
                    },
                    [&](int m, int s, uint64_t* bar) {
                        TQ::load(sQ + s * TQ::kBytes, &tm_q, bar, (m0 + m) * 64, h, b, pol_many);
                        TQ::load(sdO + s * TQ::kBytes, &tm_do, bar, (m0 + m) * 64, h, b, pol_many);
                    });
            }
            __syncwarp();
        } else if (warp == kMmaWarp) {
            if (nit > 0) {
                constexpr uint32_t idesc_s = instr_desc_f16(kBF16, 128, 64, false);
                constexpr uint32_t idesc_o = instr_desc_f16(kBF16, 128, D, true);
                const uint64_t dk_ = TK::desc_k(sK), dv_ = TK::desc_k(sV);
                const uint64_t dq_ = TQ::desc_k(sQ), ddo = TQ::desc_k(sdO);     // stage 0
                const uint64_t qn = TQ::desc_n(sQ), don = TQ::desc_n(sdO);
                const bool leader = elect_one();
                issue<ST, C::kSets>(
                    br, &br.row_full, nit, abort_p, p, leader,
                    [&](int s, uint32_t col) {             // S^T = K Q^T, dP^T = V dO^T
                        const uint32_t so = (s * TQ::kBytes) >> 4;
                        if (leader) {
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk)
                                mma_ss(tmem + col, desc_at(lo32(dk_) + TK::kstep(kk), hi32(dk_)),
                                       desc_at(lo32(dq_) + so + TQ::kstep(kk), hi32(dq_)), idesc_s, kk > 0 ? 1u : 0u);
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk)
                                mma_ss(tmem + col + 64, desc_at(lo32(dv_) + TK::kstep(kk), hi32(dv_)),
                                       desc_at(lo32(ddo) + so + TQ::kstep(kk), hi32(ddo)), idesc_s, kk > 0 ? 1u : 0u);
                        }
                    },
                    [&](int m, int s, uint32_t col) {      // dV += P^T dO, dK += dS^T Q
                        const uint32_t so = (s * TQ::kBytes) >> 4;
                        if (leader) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_ts(tmem + C::kColDV, tmem + col + kk * 8,
                                       desc_at(lo32(don) + so + TQ::rstep(kk), hi32(don)), idesc_o,
                                       (m > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_ts(tmem + C::kColDK, tmem + col + 64 + kk * 8,
                                       desc_at(lo32(qn) + so + TQ::rstep(kk), hi32(qn)), idesc_o,
                                       (m > 0 || kk > 0) ? 1u : 0u);
                        }
                    });
            }
            __syncwarp();
        }
    } else {
        regs_inc<kRegsGroup>();
        // ------------------------------------------------------------ elementwise groups
        const int g = warp >> 2, tw = t & 127;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const int kr = k0 + tw;                      // this thread's key row
        const float* lse_bh = p.lse + static_cast<int64_t>(bh) * p.N;
        // lse and D of a block's queries, fetched one of the group's blocks ahead and stored
        // (as -lse in log2 units and -D) only when that block starts, so that no instruction
        // waits for the loads before then
        float l_nx = 0.f, d_nx = 0.f;
        auto fetch = [&](int m) {
            l_nx = 0.f;
            d_nx = 0.f;
            const int qi = (m0 + m) * 64 + tw;
            if (tw < 64 && m < nit && qi < p.N) {
                l_nx = lse_bh[qi];
                d_nx = *reinterpret_cast<const float*>(row_ptr<T>(p.dq, p.dq_sb, p.dq_sh, p.dq_si, b, h, qi));
            }
        };
        fetch(g);
        bool ok = true;
        int it = 0;
        for (int m = g; m < nit; m += 2, ++it) {
            const int buf = it & 1;
            if (tw < 64) {
                sL[g][buf][tw] = -l_nx * kLog2e;
                sDr[g][buf][tw] = -d_nx;
            }
            ok = group_sync_and(1 + g, ok);
            if (!ok) break;
            fetch(m + 2);
            ok = wait_bar(&br.s_full[m % C::kSets], (m / C::kSets) & 1, abort_p, p);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) continue;                       // the next group barrier stops the group
            tc_fence_after();
            const uint32_t col_s = tmem + lane_off + 128 * (m % C::kSets), col_dp = col_s + 64;
            const int q0 = (m0 + m) * 64;
            // key kr is seen by query q iff q < N and (causal) kr <= q + causal_off
            int qlim = min(p.N - q0, 64);
            const int qmin = CAUSAL ? kr - p.causal_off - q0 : -1;   // first column that sees key kr
            if (MODS && p.window_left >= 0) qlim = min(qlim, kr - p.causal_off + p.window_left - q0 + 1);
            uint32_t rs[2][32], rd[2][32];           // S^T and dP^T of the block's 64 queries
            tmem_ld32(col_s, rs[0]);
            tmem_ld32(col_s + 32, rs[1]);
            tmem_ld32(col_dp, rd[0]);
            tmem_ld32(col_dp + 32, rd[1]);
            tmem_wait_ld(rs[0]);
            tmem_wait_ld(rs[1]);
            tmem_wait_ld(rd[0]);
            tmem_wait_ld(rd[1]);
            const float4* nl4 = reinterpret_cast<const float4*>(sL[g][buf]);
            const float4* nd4 = reinterpret_cast<const float4*>(sDr[g][buf]);
            uint32_t pk[32], dk2[32];                // 16-bit P^T and dS^T, two queries per word
            if (!MODS && __all_sync(0xffffffffu, qmin <= 0 && qlim >= 64)) {
                // every query of the block sees every key of the warp: no masks, two lanes per op
                const float sl = p.scale_log2;
#pragma unroll
                for (int c4 = 0; c4 < 16; ++c4) {
                    const int hh = c4 >> 3, cc = (c4 & 7) * 4;
                    const float4 nl = nl4[c4], nd = nd4[c4];
                    float x0, x1, x2, x3, t0, t1, t2, t3;
                    ffma2(x0, x1, __uint_as_float(rs[hh][cc]), __uint_as_float(rs[hh][cc + 1]), sl, sl, nl.x, nl.y);
                    ffma2(x2, x3, __uint_as_float(rs[hh][cc + 2]), __uint_as_float(rs[hh][cc + 3]), sl, sl, nl.z, nl.w);
                    const float p0 = ex2_approx(x0), p1 = ex2_approx(x1), p2 = ex2_approx(x2), p3 = ex2_approx(x3);
                    fadd2(t0, t1, __uint_as_float(rd[hh][cc]), __uint_as_float(rd[hh][cc + 1]), nd.x, nd.y);
                    fadd2(t2, t3, __uint_as_float(rd[hh][cc + 2]), __uint_as_float(rd[hh][cc + 3]), nd.z, nd.w);
                    fmul2(t0, t1, t0, t1, p0, p1);
                    fmul2(t2, t3, t2, t3, p2, p3);
                    pk[2 * c4] = pack2<T>(p0, p1);
                    pk[2 * c4 + 1] = pack2<T>(p2, p3);
                    dk2[2 * c4] = pack2<T>(t0, t1);
                    dk2[2 * c4 + 1] = pack2<T>(t2, t3);
                }
            } else {
                const float slope = (MODS && p.alibi != nullptr) ? p.alibi[h] : 0.f;
                const float* nl = sL[g][buf];
                const float* nd = sDr[g][buf];
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    const int hh = c >> 5, cc = c & 31;
                    float x0, x1, d0 = 1.f, d1 = 1.f;
                    if constexpr (MODS) {
                        const float dist = static_cast<float>(q0 + c + p.causal_off - kr);
                        x0 = fmaf(mod_score(__uint_as_float(rs[hh][cc]) * p.scale, slope, dist, p.softcap, &d0), kLog2e,
                                  nl[c]);
                        x1 = fmaf(mod_score(__uint_as_float(rs[hh][cc + 1]) * p.scale, slope, dist + 1.f, p.softcap, &d1),
                                  kLog2e, nl[c + 1]);
                    } else {
                        x0 = fmaf(__uint_as_float(rs[hh][cc]), p.scale_log2, nl[c]);
                        x1 = fmaf(__uint_as_float(rs[hh][cc + 1]), p.scale_log2, nl[c + 1]);
                    }
                    const bool v0 = c < qlim && c >= qmin, v1 = c + 1 < qlim && c + 1 >= qmin;
                    const float p0 = v0 ? ex2_approx(x0) : 0.f, p1 = v1 ? ex2_approx(x1) : 0.f;
                    const float g0 = p0 * (__uint_as_float(rd[hh][cc]) + nd[c]) * d0;
                    const float g1 = p1 * (__uint_as_float(rd[hh][cc + 1]) + nd[c + 1]) * d1;
                    pk[c >> 1] = pack2<T>(p0, p1);
                    dk2[c >> 1] = pack2<T>(g0, g1);
                }
            }
            // 16-bit P^T over S^T and dS^T over dP^T (all of both were read above)
            tmem_st32(col_s, pk);
            tmem_st32(col_dp, dk2);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&br.p_ready[m % C::kSets]);
        }
        // group 0 writes dV, group 1 dK (one row per thread)
        bool store = ok && (nit == 0 || wait_bar(&br.acc_done, 0, abort_p, p));
        store = __all_sync(0xffffffffu, store);
        tc_fence_after();
        if (store) {
            const bool row_ok = kr < p.Nk;
            uint8_t* dst = g == 0 ? const_cast<uint8_t*>(row_ptr<T>(p.dv, p.dv_sb, p.dv_sh, p.dv_si, b, h, row_ok ? kr : 0))
                                  : const_cast<uint8_t*>(row_ptr<T>(p.dk, p.dk_sb, p.dk_sh, p.dk_si, b, h, row_ok ? kr : 0));
            if (nit > 0)
                tmem_row_to_global<T, D>(tmem + lane_off + (g == 0 ? C::kColDV : C::kColDK), dst, row_ok,
                                         g == 0 ? 1.f : p.scale);
            else if (row_ok)
                zero_row<T, D>(dst);
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
    using TK = Tile<D, 64>;        // K, V: one 64-key block per stage
    static constexpr int kStages = (D == 128) ? 4 : 6;
    static constexpr int kSets = (kStages >= 5) ? 3 : 2;
    static constexpr uint32_t kCols = 512u;
    static constexpr uint32_t kColDQ = 128 * kSets;              // after the sets
    // Q and dO, 16-bit pairs per column: the A operands of the products (TS form, whose only
    // shared-memory operand is the key block: SS products at N = 64 are bound by their operand reads)
    static constexpr uint32_t kColQ = kColDQ + D, kColDO = kColQ + D / 2;
    static_assert(kColDO + D / 2 <= kCols, "tensor memory budget");
    static constexpr int kOffQ = 0, kOffDO = TQ::kBytes, kOffK = 2 * TQ::kBytes;
    static constexpr int kOffV = kOffK + kStages * TK::kBytes;
    static constexpr int kBytes = kOffV + kStages * TK::kBytes;
    static constexpr int kDynBytes = (kBytes + 1024 > 120 * 1024) ? kBytes + 1024 : 120 * 1024;
};

template <typename T, int D, bool CAUSAL, bool MODS = false>
__global__ void __launch_bounds__(kThreadsPP, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const Params p) {
    using namespace sm100;
    using C = DqCfg<D>;
    using TK = typename C::TK;
    using TQ = typename C::TQ;
    constexpr int ST = C::kStages;
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;

    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) PipeBars<ST> br;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sdO = smem + C::kOffDO;
    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;

    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
    // causal: later query blocks see more keys; launch them first
    const int q0 = (CAUSAL ? gridDim.x - 1 - blockIdx.x : blockIdx.x) * 128;
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
    const int nit = nkb - kb_first;                 // key blocks this CTA visits
    ATTN_CHECK(p.status, kb_first >= 0 && kb_first <= nkb && nkb <= nkb_all && q0 < p.N + 127 && b < p.B);

    if (t == 0) {
        init_pipe(br);
        abort_flag = 0;
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
    int* abort_p = &abort_flag;

    if (warp >= 8) {
        regs_dec<kRegsOther>();
        if (warp == kTmaWarp) {
            if (lane == 0 && nit > 0) {
                const uint64_t pol_once = policy_evict_first();
                const uint64_t pol_many = policy_evict_last();
                produce<ST, TQ, TK>(
                    br, nit, abort_p, p,
                    [&](uint64_t* bar) {
                        TQ::load(sQ, &tm_q, bar, q0, h, b, pol_once);
                        TQ::load(sdO, &tm_do, bar, q0, h, b, pol_once);
                    },
                    [&](int m, int s, uint64_t* bar) {
                        TK::load(sK + s * TK::kBytes, &tm_k, bar, (kb_first + m) * 64, h, b, pol_many);
                        TK::load(sV + s * TK::kBytes, &tm_v, bar, (kb_first + m) * 64, h, b, pol_many);
                    });
            }
            __syncwarp();
        } else if (warp == kMmaWarp) {
            if (nit > 0) {
                constexpr uint32_t idesc_s = instr_desc_f16(kBF16, 128, 64, false);
                constexpr uint32_t idesc_o = instr_desc_f16(kBF16, 128, D, true);
                const uint64_t dk_ = TK::desc_k(sK), dv_ = TK::desc_k(sV);     // stage 0
                const uint64_t kn = TK::desc_n(sK);
                const bool leader = elect_one();
                issue<ST, C::kSets>(
                    br, &br.row_tmem, nit, abort_p, p, leader,
                    [&](int s, uint32_t col) {             // S = Q K^T, dP = dO V^T (Q, dO in TMEM)
                        const uint32_t so = (s * TK::kBytes) >> 4;
                        if (leader) {
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk)
                                mma_ts(tmem + col, tmem + C::kColQ + kk * 8,
                                       desc_at(lo32(dk_) + so + TK::kstep(kk), hi32(dk_)), idesc_s, kk > 0 ? 1u : 0u);
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk)
                                mma_ts(tmem + col + 64, tmem + C::kColDO + kk * 8,
                                       desc_at(lo32(dv_) + so + TK::kstep(kk), hi32(dv_)), idesc_s, kk > 0 ? 1u : 0u);
                        }
                    },
                    [&](int m, int s, uint32_t col) {      // dQ += dS K
                        const uint32_t so = (s * TK::kBytes) >> 4;
                        if (leader) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_ts(tmem + C::kColDQ, tmem + col + kk * 8,
                                       desc_at(lo32(kn) + so + TK::rstep(kk), hi32(kn)), idesc_o,
                                       (m > 0 || kk > 0) ? 1u : 0u);
                        }
                    });
            }
            __syncwarp();
        }
    } else {
        regs_inc<kRegsGroup>();
        // ------------------------------------------------------------ elementwise groups
        const int g = warp >> 2, tw = t & 127;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const int qi = q0 + tw;                      // this thread's query row
        const bool row_ok = qi < p.N;
        uint8_t* dqrow = const_cast<uint8_t*>(row_ptr<T>(p.dq, p.dq_sb, p.dq_sh, p.dq_si, b, h, row_ok ? qi : 0));
        // this row's lse (log2 units) and D, read only by a group with a block: it arrives on
        // p_ready after the read, and the dQ stores below (chunk 0 holds D) follow acc_done,
        // which follows every p_ready phase
        float nlse2 = 0.f, ndrow = 0.f;              // -lse (log2 units), -D
        if (row_ok && nit > g) {
            nlse2 = -p.lse[static_cast<int64_t>(bh) * p.N + qi] * kLog2e;
            ndrow = -*reinterpret_cast<const float*>(dqrow);
        }
        bool ok = true;
        if (nit > 0) {
            // this thread's row of Q (group 0) or dO (group 1) from the TMA-written tile (128- or,
            // at d = 32, 64-byte swizzle) into tensor memory, the A operand of the products
            ok = __all_sync(0xffffffffu, wait_bar(&br.row_full, 0, abort_p, p));
            if (ok) {
                tc_fence_after();
                const uint8_t* row = (g == 0 ? sQ : sdO) + tw * TQ::kRowBytes;
                constexpr int kChunks = TQ::kRowBytes / 16;            // 16-byte chunks per atom row
                const int swz = (kChunks == 8) ? (tw & 7) : ((tw >> 1) & 3);
                uint32_t w[D / 2];
#pragma unroll
                for (int a = 0; a < TQ::kNumAtoms; ++a)
#pragma unroll
                    for (int c = 0; c < kChunks; ++c) {
                        const uint4 v = *reinterpret_cast<const uint4*>(row + a * TQ::kAtomBytes + ((c ^ swz) << 4));
                        const int o = (a * kChunks + c) * 4;
                        w[o] = v.x;
                        w[o + 1] = v.y;
                        w[o + 2] = v.z;
                        w[o + 3] = v.w;
                    }
                const uint32_t dst = tmem + lane_off + (g == 0 ? C::kColQ : C::kColDO);
                if constexpr (D == 32) {
                    tmem_st16(dst, w);
                } else {
#pragma unroll
                    for (int c = 0; c < D / 64; ++c)
                        tmem_st32(dst + c * 32, *reinterpret_cast<const uint32_t(*)[32]>(&w[c * 32]));
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&br.row_tmem);
            }
        }
        const float slope = (MODS && p.alibi != nullptr) ? p.alibi[h] : 0.f;
        for (int m = g; m < nit; m += 2) {
            ok = group_sync_and(1 + g, ok);
            if (!ok) break;
            ok = wait_bar(&br.s_full[m % C::kSets], (m / C::kSets) & 1, abort_p, p);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) continue;                       // the next group barrier stops the group
            tc_fence_after();
            const uint32_t col_s = tmem + lane_off + 128 * (m % C::kSets), col_dp = col_s + 64;
            const int kb0 = (kb_first + m) * 64;
            // key kb0 + c is seen iff it is < Nk and (causal) <= qi + causal_off; rows past N are
            // never stored, and their zero Q and dO rows contribute nothing to other rows
            int lim = min(p.Nk - kb0, 64);
            if (CAUSAL) lim = min(lim, qi + p.causal_off - kb0 + 1);
            const int lo = (MODS && p.window_left >= 0) ? qi + p.causal_off - p.window_left - kb0 : 0;
            uint32_t rs[2][32], rd[2][32];           // S and dP of the block's 64 keys
            tmem_ld32(col_s, rs[0]);
            tmem_ld32(col_s + 32, rs[1]);
            tmem_ld32(col_dp, rd[0]);
            tmem_ld32(col_dp + 32, rd[1]);
            tmem_wait_ld(rs[0]);
            tmem_wait_ld(rs[1]);
            tmem_wait_ld(rd[0]);
            tmem_wait_ld(rd[1]);
            uint32_t pk[32];                         // 16-bit dS, two keys per word
            if (!MODS && __all_sync(0xffffffffu, lim >= 64)) {
                // every key of the block is seen by every row of the warp: no masks, two lanes per op
                const float sl = p.scale_log2;
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    const int hh = c >> 5, cc = c & 31;
                    float x0, x1, t0, t1;
                    ffma2(x0, x1, __uint_as_float(rs[hh][cc]), __uint_as_float(rs[hh][cc + 1]), sl, sl, nlse2, nlse2);
                    const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                    fadd2(t0, t1, __uint_as_float(rd[hh][cc]), __uint_as_float(rd[hh][cc + 1]), ndrow, ndrow);
                    fmul2(t0, t1, t0, t1, p0, p1);
                    pk[c >> 1] = pack2<T>(t0, t1);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    const int hh = c >> 5, cc = c & 31;
                    float x0, x1, d0 = 1.f, d1 = 1.f;
                    if constexpr (MODS) {
                        const float dist = static_cast<float>(qi + p.causal_off - kb0 - c);
                        x0 = fmaf(mod_score(__uint_as_float(rs[hh][cc]) * p.scale, slope, dist, p.softcap, &d0), kLog2e,
                                  nlse2);
                        x1 = fmaf(mod_score(__uint_as_float(rs[hh][cc + 1]) * p.scale, slope, dist - 1.f, p.softcap, &d1),
                                  kLog2e, nlse2);
                    } else {
                        x0 = fmaf(__uint_as_float(rs[hh][cc]), p.scale_log2, nlse2);
                        x1 = fmaf(__uint_as_float(rs[hh][cc + 1]), p.scale_log2, nlse2);
                    }
                    const float p0 = (c < lim && c >= lo) ? ex2_approx(x0) : 0.f;
                    const float p1 = (c + 1 < lim && c + 1 >= lo) ? ex2_approx(x1) : 0.f;
                    pk[c >> 1] = pack2<T>(p0 * (__uint_as_float(rd[hh][cc]) + ndrow) * d0,
                                          p1 * (__uint_as_float(rd[hh][cc + 1]) + ndrow) * d1);
                }
            }
            tmem_st32(col_s, pk);                    // dS over S (all of S was read above)
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&br.p_ready[m % C::kSets]);
        }
        // the row's dQ: group g writes its 32-column chunks c = g, g + 2, ...
        bool store = ok && (nit == 0 || wait_bar(&br.acc_done, 0, abort_p, p));
        store = __all_sync(0xffffffffu, store);
        tc_fence_after();
        if (store) {
#pragma unroll
            for (int c = g; c < D / 32; c += 2) {
                if (nit > 0) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_off + C::kColDQ + c * 32, r);
                    tmem_wait_ld(r);
                    if (row_ok) store_row<T, 32>(dqrow + c * 64, r, p.scale);
                } else if (row_ok) {
                    zero_row<T, 32>(dqrow + c * 64);
                }
            }
        }
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
