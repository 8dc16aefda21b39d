// attn_fwd_kernel.cuh -- fused exact attention forward for sm_100a.
//
// What it computes (aiinarabic.com "flash-attention", Equation (1), plus the
// optional additive bias and sigmoid gate of the gated Evoformer variant named
// in the gist.science FLASHLIGHT summary):
//     O = softmax(scale * Q K^T [+ bias]) V [* sigmoid(G)],  lse = m + ln(l).
// How: block by block (aiinarabic.com "flash-attention", the per-block order:
// load a block of Q, K, V on chip, QK^T of the block, softmax of the block,
// multiply by V, merge with the previous blocks and move on), merging with the
// online softmax of the gist.science FLASHLIGHT summary (Methodology, item 3):
// a running row maximum m and running sum l; whenever m grows, l and the
// output accumulator are rescaled by 2^(m_old - m_new).  No score or
// probability tile ever leaves the SM.
//
// Work unit: 256 query rows (two 128-row tiles Q0, Q1) of one (batch, head).
// The kernel is persistent (one CTA per SM) and walks the units with a static
// heaviest-first order.  Within a unit the two query tiles ping-pong through
// the tensor core so that the softmax of one overlaps the MMAs of the other
// (the B200 counterpart of the matmul / softmax interleave of hamidun.com's
// FlashAttention-3 article):
//     tensor core:  S0(j) | PV1(j-1) | S1(j) | PV0(j) | S0(j+1) | PV1(j) | ...
//     softmax WG0:        [ softmax S0(j) ]          [ softmax S0(j+1) ] ...
//     softmax WG1:                        [ softmax S1(j) ]          ...
//
// Warp roles (16 warps):
//   WG0 (warps 0-3)   softmax of Q0: thread t owns query row t; reads its score
//                     row from tensor memory, masks/scales, updates m and l,
//                     writes P (fp16/bf16) back to tensor memory.  When m grew by
//                     more than 2^8 the O accumulator row is rescaled (otherwise
//                     the stale maximum is kept: the final O/l and lse use the
//                     same reference, so the result is unchanged): at d <= 64 by
//                     the softmax thread itself, at d = 128 by WG2.
//   WG1 (warps 4-7)   the same for Q1.
//   WG2 (warps 8-11)  epilogue: O/l, gate, rounding, stores of O and lse; at
//                     d = 128 also the correction (the O rescale above).
//   warp 12           tcgen05.mma issuer (one elected lane); allocates tensor memory.
//                     Without causal masking at d <= 64 it issues only Q0's MMAs and
//                     warp 14 those of Q1 (one issuer per query tile).
//   warp 13           TMA producer: Q0, Q1 per unit, K and V tiles into rings.
//   warps 14-15       otherwise idle (they complete warpgroup 3's register hand-back).
//
// Tensor memory (128 lanes = query rows, 512 columns):
//   d <= 64:  S0 [0,128) S1 [128,256) P0 [256,320) P1 [320,384) O0 [384,384+d) O1 [384+d, 384+2d)
//   d = 128:  S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512), P_i in the first 64 columns of S_i
//             (S_i(j+1) overwrites P_i(j) after PV_i(j), which the single MMA thread issued
//             earlier; tcgen05.mma operations from one thread execute in issue order).
//
// Every mbarrier wait is bounded: a wait that gives up records a timeout in
// the device status word and raises a CTA-wide abort flag; every role then
// stops, drains what it has in flight, and the CTA exits without hanging.
#pragma once

#include <type_traits>

#include "sm100.cuh"

namespace attn {

constexpr int kBlockM = 128;              // rows per query tile (one TMEM lane per row)
constexpr int kBlockN = 128;              // keys per key/value tile
constexpr int kRowsPerUnit = 2 * kBlockM;
constexpr int kThreads = 512;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f; // log2 domain: rescale only when m grows by > 2^8
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusCheck = 2u;     // debug builds: an index or range check failed

constexpr unsigned long long kDrainLimit = 1ull << 32;
constexpr int kMaxSeq = 64;    // sequences of a ragged batch handled by one launch

struct FwdParams {
    int B, H, N;               // N: query rows
    int Nk;                    // key rows
    int causal_off;            // Nk - N: query i sees key j iff j <= i + causal_off (causal)
    int num_q_pairs;           // ceil(N / 256)
    int num_units;             // num_q_pairs * B * H
    int n_kv_tiles;            // ceil(Nk / 128)
    int head_group;            // heads per scheduling group (see decode_unit)
    float scale;               // multiplies Q K^T
    float scale_log2;          // scale * log2(e)
    const void* bias;          // nullable
    int64_t bias_sb, bias_sh, bias_si;   // element strides (bias_sb = 0 when shared over B)
    const void* gate;          // nullable
    int64_t gate_sb, gate_sh, gate_si;
    void* out;
    int64_t out_sb, out_sh, out_si;
    float* lse;                // nullable; row (b, h, i) at b * lse_sb + h * lse_sh + i
    int64_t lse_sb, lse_sh;
    // score modifications (generic path only), applied after scale and bias in this order:
    const float* alibi;        // nullable [H]: s -= slope_h * |i + causal_off - j|
    float softcap;             // > 0: s <- softcap * tanh(s / softcap)
    int window_left;           // >= 0: keys j < i + causal_off - window_left are masked
    int has_mods;              // any of the three is on
    unsigned long long wait_limit;
    unsigned int* status;
    int inject_stall;          // test hook: the MMA warp first waits on a barrier nothing arrives on
    float v_scale;             // e4m3 inputs: the value tensor's scale (the query and key scales are in scale)
    // ragged batch in one launch (n_seq > 0; B = 1 and the tensors are packed [1, H, T, d] views):
    // sequence s owns query rows seq_q0[s] .. + seq_nq[s] and key rows seq_k0[s] .. + seq_nk[s].
    // level_order == 0: units seq_units[s] .. seq_units[s + 1] are sequence s's query pairs x H,
    // heaviest pairs first.  level_order == 1 (causal, N_q = N_k in every sequence, sequences
    // sorted by query pairs, most first): the units of all sequences ordered by query pair,
    // highest first, which is heaviest first (a causal pair's key tiles depend on its index
    // only); segment i, units seq_units[i] .. seq_units[i + 1], holds the pairs only sequences
    // 0..i have, (i + 1) x H units per pair.
    int n_seq;
    int level_order;
    int seq_units[kMaxSeq + 1];
    int seq_q0[kMaxSeq], seq_k0[kMaxSeq], seq_nq[kMaxSeq], seq_nk[kMaxSeq];
};

template <int D, bool FP8 = false>
struct Cfg {
    static_assert(D == 32 || D == 64 || D == 128, "head dim");
    static_assert(!FP8 || D >= 64, "e4m3 inputs: d = 64 or 128");
    // A 128-row tile of D 16-bit elements is stored as D/64 "atoms" of 128 rows
    // x 128 bytes (128-byte swizzle), or for D = 32 one atom of 128 rows x 64
    // bytes (64-byte swizzle): exactly the layout TMA writes.  With e4m3 inputs a
    // row of D bytes is one atom: 64 bytes (64-byte swizzle) or 128 bytes (128-byte).
    static constexpr int kElemBytes = FP8 ? 1 : 2;
    static constexpr int kRowBytes = FP8 ? D : ((D >= 64) ? 128 : 64);
    static constexpr int kAtomCols = kRowBytes / kElemBytes;
    static constexpr int kNumAtoms = D / kAtomCols;
    static constexpr int kAtomBytes = 128 * kRowBytes;
    static constexpr int kTileBytes = kNumAtoms * kAtomBytes;     // 128 * D * element bytes
    static constexpr uint32_t kLayout = (kRowBytes == 128) ? 2u : 4u;   // SW128 : SW64
    // reduction elements per MMA instruction: always 32 bytes (16 halves or 32 e4m3 values)
    static constexpr int kK = 32 / kElemBytes;
    // offset (16-byte units) of the kk-th reduction step in a K-major tile
    static __host__ __device__ constexpr uint32_t kstep(int kk) {
        return static_cast<uint32_t>((((kk * 32) / kRowBytes) * kAtomBytes + (kk * 32) % kRowBytes) >> 4);
    }
    // tensor-memory columns of one tile's P: 128 keys packed into 32-bit columns
    static constexpr uint32_t kColsP = 128 * kElemBytes / 4;
    static constexpr uint32_t kSBO = 8 * kRowBytes;               // 8-row group stride
    static constexpr int kStages = (D == 128) ? 2 : (D == 64 ? 3 : 4);
    // tensor memory columns
    // d <= 64: P has columns of its own, so S_i(j+1) may be computed while the
    // softmax of S_i(j) runs; d = 128: P lives inside S_i (no room otherwise).
    static constexpr bool kSeparateP = (D <= 64);
    // Who rescales O when a row maximum moves.  With separate P columns the softmax warps do it
    // themselves, after waiting for the previous PV (which they wait for anyway before P is
    // overwritten), so PV_i(j) waits only for the softmax.  At d = 128 (P inside S) the softmax
    // has no such wait and no registers to spare: the correction warpgroup rescales O between
    // PV_i(j-1) and PV_i(j) and PV_i(j) waits for both (measured on B200: each choice is the
    // faster one for its head dim).
    static constexpr bool kInlineRescale = kSeparateP;
    static constexpr uint32_t kPvArrivals = kInlineRescale ? kBlockM : 2 * kBlockM;
    // One exponential pair in kEmuPeriod goes through the FMA-pipe 2^x (0: none).  Measured
    // on B200: at d=64 one in four beats one in three and none; at d=128 (MMA-bound) and
    // d=32 (short units) the extra FMA-pipe work costs more than the MUFU time it saves.
    static constexpr int kEmuPeriod = (D == 64) ? 4 : 0;
    static constexpr uint32_t kColS0 = 0, kColS1 = 128;
    static constexpr uint32_t kColP0 = (D == 128) ? 0 : 256;
    static constexpr uint32_t kColP1 = (D == 128) ? 128 : 256 + kColsP;
    static constexpr uint32_t kColO0 = (D == 128) ? 256 : 256 + 2 * kColsP;
    static constexpr uint32_t kColO1 = kColO0 + ((D == 128) ? 128 : D);
    static_assert(kColO1 + D <= kTmemCols, "tensor memory budget");
    // shared memory (dynamic, 1024-byte aligned)
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + 2 * kTileBytes;
    static constexpr int kOffV = kOffK + kStages * kTileBytes;
    static constexpr int kBytes = kOffV + kStages * kTileBytes;
    static constexpr int kDynBytes = kBytes + 1024;
    static_assert(kDynBytes <= 227 * 1024, "shared memory budget");
    // per-thread registers after setmaxnreg: 256 softmax + 128 epilogue + 128 other
    // threads must fit the 65536 the CTA was launched with (512 threads x 128)
    // (d=64: the MMA issuer and TMA producer get 96, the epilogue 64 - fewer spills in the
    // issuer's loop, measured 2-3 % faster than 80 / 80 at N=8192)
    static constexpr int kRegsSoftmax = 176;
    static constexpr int kRegsEpilogue = (D == 64) ? 64 : 80;
    static constexpr int kRegsOther = (D == 64) ? 96 : 80;
    static_assert(256 * kRegsSoftmax + 128 * kRegsEpilogue + 128 * kRegsOther <= 65536, "register budget");
};

// Additive bias staged through shared memory by TMA (d <= 64; at d = 128 the K/V rings
// leave no room and each softmax thread reads its bias row from global memory).  A bias
// tile is 128 query rows x 128 keys of 16-bit values, stored as two 128 x 64 boxes with
// the 128-byte swizzle, so that thread t reading 16-byte chunk k of its row touches
// chunk position k ^ (t & 7): conflict-free.
template <int D, bool HAS_BIAS>
struct BiasCfg {
    static constexpr bool kTma = HAS_BIAS && D <= 64;
    static constexpr int kStages = (D == 32) ? 2 : 1;
    static constexpr int kBoxBytes = kBlockM * 64 * 2;            // 16 KB
    static constexpr int kTileBytes = 2 * kBoxBytes;               // 32 KB
    static constexpr int kOff = Cfg<D>::kBytes;
    static constexpr int kBytes = kTma ? 2 * kStages * kTileBytes : 0;
    static constexpr int kDynBytes = Cfg<D>::kBytes + kBytes + 1024;
    static_assert(kDynBytes <= 214 * 1024, "shared memory budget (dynamic + static)");
};

template <int ST>
struct __align__(8) FwdShared {
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[ST], k_empty[ST], v_full[ST], v_empty[ST];
    uint64_t s_full[2];      // MMA -> softmax i: S_i(j) in tensor memory
    uint64_t s_free[2];      // softmax i -> MMA: S_i(j) read into registers (d <= 64 only)
    uint64_t pv_ready[2];    // softmax i (P_i(j) written) [+ correction (O_i rescaled), d = 128] -> MMA
    uint64_t o_done[2];      // MMA -> softmax i (d <= 64) or correction (d = 128): PV_i(j) complete
    uint64_t o_final[2];     // MMA -> epilogue (d <= 64): the unit's last PV_i complete
    uint64_t sm2corr[2];     // softmax i -> correction (d = 128): alpha(j), j >= 1
    uint64_t o_free[2];      // epilogue -> MMA and softmax i: epilogue has read O_i and m, l
    uint64_t stats_full[2];  // softmax i -> epilogue: final m, l of the unit
    uint64_t drain;
    uint64_t never;          // no arrivals: target of the injected stall
    uint64_t bias_full[2][2], bias_empty[2][2];   // [tile][stage], staged bias tiles
    uint32_t tmem_base;
    int abort_flag;
    float alpha[2][2][kBlockM];    // [iteration parity][tile][row] (d = 128)
    float stat_m[2][2][kBlockM];   // [unit parity][tile][row]
    float stat_l[2][2][kBlockM];
};

// Bounded wait.  Returns false (and raises the abort flag) if the phase did
// not complete within `limit` cycles or another role aborted first.
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, int* abort_flag,
                                           unsigned long long limit, unsigned int* status) {
    const uint32_t a = sm100::smem_u32(bar);
    if (sm100::mbar_try_wait(a, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (sm100::mbar_try_wait(a, parity)) return true;
        if (*reinterpret_cast<volatile int*>(abort_flag)) return false;
        if (static_cast<unsigned long long>(clock64() - t0) > limit) {
            atomicOr(status, kStatusTimeout);
            *reinterpret_cast<volatile int*>(abort_flag) = 1;
            return false;
        }
    }
}

// Bounded wait used only while draining on exit (ignores the abort flag).
__device__ __forceinline__ void drain_phase(uint64_t* bar, uint32_t parity, unsigned int* status) {
    const uint32_t a = sm100::smem_u32(bar);
    const long long t0 = clock64();
    while (!sm100::mbar_try_wait(a, parity)) {
        if (static_cast<unsigned long long>(clock64() - t0) > kDrainLimit) {
            atomicOr(status, kStatusTimeout);
            return;
        }
    }
}

// Maximum of a 128-entry row: eight independent chains of three-input max
// instructions (dependency depth 10 instead of 43), then a small tree.
__device__ __forceinline__ float row_max(const float (&s)[kBlockN]) {
    float m[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        float a = fmaxf(s[16 * q], s[16 * q + 1]);
#pragma unroll
        for (int c = 2; c < 16; c += 2) a = sm100::max3(a, s[16 * q + c], s[16 * q + c + 1]);
        m[q] = a;
    }
    return sm100::max3(sm100::max3(m[0], m[1], m[2]), sm100::max3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// Keeps the scores of keys lo <= c < lim of a row's tile and sets the others to -inf: per
// 32-key chunk a word with the chunk's visible keys as set bits, then one bit test and one
// select per key rather than two compares and a select (with one bound, the plain compare
// is cheaper).
__device__ __forceinline__ void mask_keys(float (&s)[kBlockN], int lo, int lim) {
#pragma unroll
    for (int k = 0; k < kBlockN / 32; ++k) {
        const int a = min(max(lo - 32 * k, 0), 32), b = min(max(lim - 32 * k, 0), 32);
        const uint32_t below_b = b >= 32 ? 0xffffffffu : ((1u << b) - 1u);
        const uint32_t below_a = a >= 32 ? 0xffffffffu : ((1u << a) - 1u);
        const uint32_t keep = below_b & ~below_a;
#pragma unroll
        for (int c = 0; c < 32; ++c) s[32 * k + c] = ((keep >> c) & 1u) ? s[32 * k + c] : -INFINITY;
    }
}

// 2^x for two lanes on the FMA and integer pipes instead of the MUFU unit.
// Range reduction in the style of Cody and Waite: n = floor(x) by a
// round-toward-minus-infinity add of 1.5 * 2^23 (n then sits in the low
// mantissa bits of t), f = x - n in [0, 1); 2^f by a cubic whose
// coefficients we fitted for minimum relative error on [0, 1) (max relative
// error 7.5e-5, below the half-ulp of the fp16/bf16 P it feeds); finally n is
// added to the exponent field.  Inputs below -126 are clamped there, which
// yields at most a denormal that the fp16 rounding and the flushed row sum
// discard.
__device__ __forceinline__ void ex2_emu2(float& y0, float& y1, float x0, float x1) {
    constexpr float kShift = 12582912.f;                     // 1.5 * 2^23
    constexpr float c0 = 0.9999251814280168f, c1 = 0.6958336953498905f;
    constexpr float c2 = 0.2260672333620784f, c3 = 0.07802422535748339f;
    x0 = fmaxf(x0, -126.f);
    x1 = fmaxf(x1, -126.f);
    float t0, t1, r0, r1, f0, f1, p0, p1;
    sm100::fadd2_rm(t0, t1, x0, x1, kShift, kShift);        // kShift + floor(x)
    sm100::fadd2(r0, r1, t0, t1, -kShift, -kShift);          // floor(x), exact
    sm100::fsub2(f0, f1, x0, x1, r0, r1);                    // f in [0, 1)
    sm100::ffma2(p0, p1, f0, f1, c3, c3, c2, c2);
    sm100::ffma2(p0, p1, p0, p1, f0, f1, c1, c1);
    sm100::ffma2(p0, p1, p0, p1, f0, f1, c0, c0);
    y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
    y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

// One work unit: query rows [q0, q0 + 256) of (b, h); tile i processes key tiles
// [kv_lo, kv_lo + nkv_i) (kv_lo > 0 only when a left window skips whole tiles).  The problem's
// sizes travel with the unit (a ragged batch mixes sequences): N query rows, Nk key rows,
// off = Nk - N, and the first query / key row of the sequence in the packed tensors.
struct Unit {
    int b, h, bh, qp, q0, nkv0, nkv1, kv_lo;
    int N, Nk, off, q_base, k_base;
};

// The k-th unit a CTA processes.  Wave k (the k-th unit of every CTA) takes units
// [k G, (k+1) G) of the heaviest-first order, G = gridDim.x, forwards for even k and
// backwards for odd k: the CTA that drew the heaviest unit of one wave draws the
// lightest of the next, which evens out the per-CTA totals of causal workloads.
__device__ __forceinline__ int unit_at(int k) {
    const int G = static_cast<int>(gridDim.x), b = static_cast<int>(blockIdx.x);
    return k * G + ((k & 1) ? (G - 1 - b) : b);
}

template <bool CAUSAL, bool MODS = false>
__device__ __forceinline__ Unit decode_unit(int u, const FwdParams& p) {
    Unit U;
    if (p.n_seq > 0) {
        // ragged batch: the sequence holding unit u is the last s with seq_units[s] <= u
        int lo = 0, hi = p.n_seq - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.seq_units[mid] <= u) lo = mid;
            else hi = mid - 1;
        }
        const int r = u - p.seq_units[lo];
        int s = lo;
        if (p.level_order) {
            // segment lo: (lo + 1) sequences x H units per query pair, pairs from nqp(lo) - 1 down
            const int per_pair = (lo + 1) * p.H;
            const int t = r / per_pair, w = r - t * per_pair;
            s = w / p.H;
            U.qp = (p.seq_nq[lo] + kRowsPerUnit - 1) / kRowsPerUnit - 1 - t;
            U.h = w % p.H;
        } else {
            const int nqp = (p.seq_nq[lo] + kRowsPerUnit - 1) / kRowsPerUnit;
            U.qp = nqp - 1 - r / p.H;
            U.h = r % p.H;
        }
        U.N = p.seq_nq[s];
        U.Nk = p.seq_nk[s];
        U.q_base = p.seq_q0[s];
        U.k_base = p.seq_k0[s];
        U.b = 0;
        U.bh = U.h;
    } else {
        // Units are taken in groups of `head_group` heads; inside a group the heaviest query
        // pairs come first (causal load balance).  With head_group = B*H (the default) this is
        // one group: heaviest pairs of all heads first.  For long sequences whose K/V do not
        // fit in L2 the host picks a small group, so that the CTAs running at the same time
        // share the K/V of a few heads in L2 instead of streaming all of them from DRAM.
        const int BH = p.B * p.H;
        const int G = p.head_group;
        const int per = G * p.num_q_pairs;
        const int g = u / per, r = u % per;
        const int gsize = min(G, BH - g * G);       // the last group may be partial
        U.qp = p.num_q_pairs - 1 - r / gsize;
        U.bh = g * G + r % gsize;
        U.b = U.bh / p.H;
        U.h = U.bh % p.H;
        U.N = p.N;
        U.Nk = p.Nk;
        U.q_base = 0;
        U.k_base = 0;
    }
    U.off = U.Nk - U.N;
    const int n_kv_tiles = (U.Nk + kBlockN - 1) / kBlockN;
    U.q0 = U.qp * kRowsPerUnit;
    if (CAUSAL) {
        // key tiles up to the one holding the last visible key of the tile's last row; at
        // least one (a tile whose rows all precede every key is processed once, fully masked)
        const int last0 = U.q0 + kBlockM - 1 + U.off, last1 = last0 + kBlockM;
        U.nkv0 = last0 < 0 ? 1 : min(n_kv_tiles, last0 / kBlockN + 1);
        U.nkv1 = last1 < 0 ? 1 : min(n_kv_tiles, last1 / kBlockN + 1);
    } else {
        U.nkv0 = U.nkv1 = n_kv_tiles;
    }
    U.kv_lo = 0;
    if (MODS && p.window_left >= 0) {
        // left window: key tiles wholly left of the first row's window are skipped.  The unit's
        // first row has the leftmost window, so both query tiles start at its first key tile (the
        // second tile may process one tile it masks completely).  kv_lo < nkv_i: the first row's
        // own diagonal key (or, without causal masking, key Nk - 1) lies at or after it.
        const int lo_key = U.q0 + U.off - p.window_left;
        U.kv_lo = lo_key > 0 ? lo_key / kBlockN : 0;
        U.nkv0 -= U.kv_lo;
        U.nkv1 -= U.kv_lo;
    }
    ATTN_CHECK(p.status, U.b >= 0 && U.b < p.B && U.h >= 0 && U.h < p.H && U.qp >= 0 && U.q0 < U.N);
    ATTN_CHECK(p.status, U.kv_lo >= 0 && U.nkv0 >= 1 && U.nkv1 >= U.nkv0 && U.nkv1 <= U.nkv0 + 1);
    ATTN_CHECK(p.status, (U.kv_lo + U.nkv1 - 1) * kBlockN < U.Nk || U.nkv1 == 1);
    ATTN_CHECK(p.status, U.q_base >= 0 && U.k_base >= 0 && U.q_base + U.N <= (p.n_seq > 0 ? p.N : U.N) &&
                             U.k_base + U.Nk <= (p.n_seq > 0 ? p.Nk : U.Nk));
    return U;
}

// MODS: score modifications compiled in (only without bias and gate); other builds carry none of it.
// FP8: Q, K and V (transposed) are e4m3 codes and T is the output type; the plain path only.
template <typename T, int D, bool CAUSAL, bool HAS_BIAS, bool HAS_GATE, bool MODS = false, bool FP8 = false>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_bias,
                    const __grid_constant__ FwdParams p) {
    using namespace sm100;
    using C = Cfg<D, FP8>;
    static_assert(!FP8 || (!HAS_BIAS && !HAS_GATE && !MODS), "e4m3 inputs: plain path only");
    constexpr int ST = C::kStages;
    // Non-causal with P in its own columns (d <= 64): one MMA issuer per query tile (warps 12 and
    // 14), each releasing every K / V stage and the drain once.  Both tiles take the same key
    // tiles there.  (Causal units, where tile 1 takes one more key tile, keep one issuer: the
    // per-tile form measured slower on them.)
    constexpr bool kTileIssuers = C::kSeparateP && !CAUSAL;
    constexpr uint32_t kReleases = kTileIssuers ? 2 : 1;
    // operand format bits of the instruction descriptor: 1 selects bf16 (kind::f16); e4m3 is 0
    constexpr bool kBF16 = !FP8 && std::is_same<T, __nv_bfloat16>::value;

    extern __shared__ uint8_t smem_raw[];
    __shared__ FwdShared<ST> sh;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;
    using BC = BiasCfg<D, HAS_BIAS>;
    uint8_t* sBias = smem + BC::kOff;      // [tile][stage][2 boxes]

    const int warp = warp_id();
    const int lane = lane_id();
    const int wg = warp >> 2;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh.q_full[i], 1);
            mbar_init(&sh.q_empty[i], 1);
            mbar_init(&sh.s_full[i], 1);
            mbar_init(&sh.s_free[i], kBlockM);
            mbar_init(&sh.pv_ready[i], C::kPvArrivals);
            mbar_init(&sh.o_done[i], 1);
            mbar_init(&sh.o_final[i], 1);
            mbar_init(&sh.sm2corr[i], kBlockM);
            mbar_init(&sh.o_free[i], kBlockM);
            mbar_init(&sh.stats_full[i], kBlockM);
        }
        for (int s = 0; s < ST; ++s) {
            mbar_init(&sh.k_full[s], 1);
            mbar_init(&sh.k_empty[s], kReleases);
            mbar_init(&sh.v_full[s], 1);
            mbar_init(&sh.v_empty[s], kReleases);
        }
        mbar_init(&sh.drain, kReleases);
        mbar_init(&sh.never, 1);
        for (int i = 0; i < 2; ++i)
            for (int b = 0; b < 2; ++b) {
                mbar_init(&sh.bias_full[i][b], 1);
                mbar_init(&sh.bias_empty[i][b], kBlockM);
            }
        sh.abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 12) {
        tmem_alloc(&sh.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    int* abort_flag = &sh.abort_flag;
    ATTN_CHECK(p.status, tmem == 0u);      // all 512 columns, from lane 0 column 0

    if (wg == 3) {
        regs_dec<C::kRegsOther>();
        if (warp == 13) {
            // ============================================================ TMA producer
            // The whole warp runs this loop (uniform control flow); one elected lane issues.
            if (elect_one()) {
                tma_prefetch_desc(&tm_q);
                tma_prefetch_desc(&tm_k);
                tma_prefetch_desc(&tm_v);
            }
            const uint64_t pol_q = policy_evict_first();
            const uint64_t pol_kv = policy_evict_last();
            uint32_t kc = 0, vc = 0;            // tiles loaded into the K / V rings
            uint32_t qc[2] = {0, 0};            // Q tiles loaded per slot (one per unit)
            bool ok = true;
            auto WU = [&](uint64_t* bar, uint32_t parity) {
                if (ok) ok = wait_phase(bar, parity, abort_flag, p.wait_limit, p.status);
                ok = __all_sync(0xffffffffu, ok);
                return ok;
            };
            auto load_q = [&](int i, const Unit& U) {
                if (qc[i] > 0 && !WU(&sh.q_empty[i], (qc[i] - 1) & 1)) return;
                if (elect_one()) {
                    mbar_arrive_expect_tx(&sh.q_full[i], C::kTileBytes);
                    for (int a = 0; a < C::kNumAtoms; ++a)
                        tma_load_4d(sQ + (i * C::kNumAtoms + a) * C::kAtomBytes, &tm_q, &sh.q_full[i],
                                    a * C::kAtomCols, U.q_base + U.q0 + i * kBlockM, U.h, U.b, pol_q);
                }
                __syncwarp();
                ++qc[i];
            };
            uint32_t bc[2] = {0, 0};            // bias tiles loaded per query tile
            auto load_bias = [&](int i, int j, const Unit& U) {
                const uint32_t st = bc[i] % BC::kStages;
                if (bc[i] >= BC::kStages &&
                    !WU(&sh.bias_empty[i][st], ((bc[i] / BC::kStages) - 1) & 1))
                    return;
                if (elect_one()) {
                    mbar_arrive_expect_tx(&sh.bias_full[i][st], BC::kTileBytes);
                    uint8_t* dst = sBias + (i * BC::kStages + st) * BC::kTileBytes;
                    const int bb = p.bias_sb != 0 ? U.b : 0;
                    for (int half = 0; half < 2; ++half)
                        tma_load_4d(dst + half * BC::kBoxBytes, &tm_bias, &sh.bias_full[i][st],
                                    (U.kv_lo + j) * kBlockN + half * 64, U.q0 + i * kBlockM, U.h, bb, pol_kv);
                }
                __syncwarp();
                ++bc[i];
            };
            auto load_kv = [&](uint64_t* full, uint64_t* empty, uint8_t* ring, const CUtensorMap* map, uint32_t& cnt,
                               int j, const Unit& U) {
                const uint32_t st = cnt % ST;
                if (cnt >= ST && !WU(&empty[st], ((cnt / ST) - 1) & 1)) return;
                const int key0 = U.k_base + (U.kv_lo + j) * kBlockN;
                ATTN_CHECK(p.status, key0 >= 0 && (C::kAtomCols * C::kElemBytes) % 16 == 0 && (!FP8 || key0 % 16 == 0));
                if (elect_one()) {
                    mbar_arrive_expect_tx(&full[st], C::kTileBytes);
                    if (FP8 && ring == sV) {
                        // e4m3: V arrives transposed ([B, H, d, Nk]); one box of 128 keys x d rows,
                        // one 128-byte swizzle atom per row, which the PV MMA reads K-major
                        tma_load_4d(ring + st * C::kTileBytes, map, &full[st], key0, 0, U.h, U.b, pol_kv);
                    } else {
                        for (int a = 0; a < C::kNumAtoms; ++a)
                            tma_load_4d(ring + (st * C::kNumAtoms + a) * C::kAtomBytes, map, &full[st],
                                        a * C::kAtomCols, key0, U.h, U.b, pol_kv);
                    }
                }
                __syncwarp();
                ++cnt;
            };
            for (int k = 0, u = unit_at(0); ok && u < p.num_units; u = unit_at(++k)) {
                const Unit U = decode_unit<CAUSAL, MODS>(u, p);
                // the unit's first bias tiles go first: their stages free up as soon as the
                // softmax has read the previous unit's first tiles, long before the Q slots do
                // (each Q_i waits for the previous unit's last S_i)
                if constexpr (BC::kTma) {
                    load_bias(0, 0, U);
                    if (ok) load_bias(1, 0, U);
                }
                if (ok) load_q(0, U);
                if (ok) load_kv(sh.k_full, sh.k_empty, sK, &tm_k, kc, 0, U);
                if (ok) load_q(1, U);
                if (ok) load_kv(sh.v_full, sh.v_empty, sV, &tm_v, vc, 0, U);
                for (int j = 1; ok && j < U.nkv1; ++j) {
                    load_kv(sh.k_full, sh.k_empty, sK, &tm_k, kc, j, U);
                    if (ok) load_kv(sh.v_full, sh.v_empty, sV, &tm_v, vc, j, U);
                    if constexpr (BC::kTma) {
                        if (ok && j < U.nkv0) load_bias(0, j, U);
                        if (ok) load_bias(1, j, U);
                    }
                }
            }
            // drain: every load issued into shared memory lands before the CTA exits
            for (int i = 0; i < 2; ++i)
                if (qc[i] > 0) drain_phase(&sh.q_full[i], (qc[i] - 1) & 1, p.status);
            for (uint32_t s = 0; s < ST; ++s) {
                if (kc > s) drain_phase(&sh.k_full[s], ((kc - 1 - s) / ST) & 1, p.status);
                if (vc > s) drain_phase(&sh.v_full[s], ((vc - 1 - s) / ST) & 1, p.status);
            }
            if constexpr (BC::kTma) {
                for (int i = 0; i < 2; ++i)
                    for (uint32_t s = 0; s < (uint32_t)BC::kStages; ++s)
                        if (bc[i] > s)
                            drain_phase(&sh.bias_full[i][s], ((bc[i] - 1 - s) / BC::kStages) & 1, p.status);
            }
        } else if (warp == 12 || (kTileIssuers && warp == 14)) {
            // ============================================================ MMA issuer(s)
            constexpr uint32_t idesc_s = instr_desc_f16(kBF16, kBlockM, kBlockN, false);
            // (e4m3: V^T is K-major, like K in S; 16-bit V is N-major)
            constexpr uint32_t idesc_o = instr_desc_f16(kBF16, kBlockM, D, !FP8);
            const uint32_t q_addr = smem_u32(sQ);
            const uint32_t k_addr = smem_u32(sK);
            const uint32_t v_addr = smem_u32(sV);
            // (columns by select, not by indexing a local array with a runtime tile index)
            auto col_s = [](int i) { return i ? C::kColS1 : C::kColS0; };
            auto col_p = [](int i) { return i ? C::kColP1 : C::kColP0; };
            auto col_o = [](int i) { return i ? C::kColO1 : C::kColO0; };
            // Descriptors are affine in the start address (bits [0,14) hold address / 16 and
            // shared addresses stay below 256 KB), so each step adds a constant to a base.
            const uint64_t dq = smem_desc(q_addr, 16, C::kSBO, C::kLayout);
            const uint64_t dk = smem_desc(k_addr, 16, C::kSBO, C::kLayout);
            // e4m3 V^T: rows of 128 keys (128 bytes, 128-byte swizzle), K-major
            const uint64_t dv = FP8 ? smem_desc(v_addr, 16, 8 * 128, 2u)
                                    : smem_desc(v_addr, C::kAtomBytes, C::kSBO, C::kLayout);
            // S_i = Q_i K^T: both operands K-major, 32 bytes of the head dim per step
            // Descriptor offsets never carry out of the low word (shared addresses < 256 KB): the
            // low words are advanced with 32-bit adds and the high words are constants.
            const uint32_t dq_lo = static_cast<uint32_t>(dq), dq_hi = static_cast<uint32_t>(dq >> 32);
            const uint32_t dk_lo = static_cast<uint32_t>(dk), dk_hi = static_cast<uint32_t>(dk >> 32);
            const uint32_t dv_lo = static_cast<uint32_t>(dv), dv_hi = static_cast<uint32_t>(dv >> 32);
            auto desc = [](uint32_t lo, uint32_t hi) {
                uint64_t d;
                asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "r"(lo), "r"(hi));
                return d;
            };
            const bool leader = elect_one();     // the lane that issues (elected once)
            auto issue_s = [&](int i, uint32_t kst) {
                const uint32_t qb = dq_lo + ((i * C::kTileBytes) >> 4);
                const uint32_t kb = dk_lo + ((kst * C::kTileBytes) >> 4);
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < D / C::kK; ++kk) {
                        const uint32_t off = C::kstep(kk);
                        if constexpr (FP8)
                            mma_ss_f8(tmem + col_s(i), desc(qb + off, dq_hi), desc(kb + off, dk_hi), idesc_s, kk > 0 ? 1u : 0u);
                        else
                            mma_ss(tmem + col_s(i), desc(qb + off, dq_hi), desc(kb + off, dk_hi), idesc_s, kk > 0 ? 1u : 0u);
                    }
                }
            };
            // O_i += P_i V: P from tensor memory (8 columns per step), kK keys per step of V: kK rows
            // of the N(=d)-major 16-bit V, or 32 bytes along each row of the e4m3 V^T
            auto issue_pv = [&](int i, uint32_t vst, bool acc) {
                const uint32_t vb = dv_lo + ((vst * C::kTileBytes) >> 4);
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < kBlockN / C::kK; ++kk) {
                        const uint64_t vk = desc(vb + (FP8 ? ((kk * 32) >> 4) : ((kk * C::kK * C::kRowBytes) >> 4)), dv_hi);
                        if constexpr (FP8)
                            mma_ts_f8(tmem + col_o(i), tmem + col_p(i) + kk * 8, vk, idesc_o, (acc || kk > 0) ? 1u : 0u);
                        else
                            mma_ts(tmem + col_o(i), tmem + col_p(i) + kk * 8, vk, idesc_o, (acc || kk > 0) ? 1u : 0u);
                    }
                }
            };
            auto commit = [&](uint64_t* bar) {
                if (leader) mma_commit(bar);
            };
            uint32_t kc = 0, vc = 0, uit = 0;
            uint32_t pv_cnt[2] = {0, 0}, sf_cnt[2] = {0, 0};
            bool ok = true;
            auto W = [&](uint64_t* bar, uint32_t parity) {
                if (ok) ok = wait_phase(bar, parity, abort_flag, p.wait_limit, p.status);
                ok = __all_sync(0xffffffffu, ok);
                return ok;
            };
            if (p.inject_stall) W(&sh.never, 0);   // gives up after wait_limit cycles: exercises the abort path
            // S_i(0) of a unit: Q_i of that unit and its first key tile (ring position kpos)
            auto issue_first_s = [&](int i, int nkv_i, uint32_t kpos, uint32_t qpar) -> bool {
                if (!W(&sh.q_full[i], qpar) || !W(&sh.k_full[kpos % ST], (kpos / ST) & 1)) return false;
                tc_fence_after();
                issue_s(i, kpos % ST);
                commit(&sh.s_full[i]);
                if (kTileIssuers || i == 1) commit(&sh.k_empty[kpos % ST]);
                if (nkv_i == 1) commit(&sh.q_empty[i]);
                return true;
            };
            if constexpr (kTileIssuers) {
                // One query tile per issuing warp: S_ti(j+1) as soon as the softmax has read
                // S_ti(j), then PV_ti(j); the next unit's S_ti(0) right behind the unit's last PV_ti.
                const int ti = warp == 12 ? 0 : 1;
                uint32_t pv_n = 0, sf_n = 0;
                bool early_t = false;
                for (int u = unit_at(0); ok && u < p.num_units; u = unit_at(++uit)) {
                    const Unit U = decode_unit<CAUSAL, MODS>(u, p);
                    const int nkv = U.nkv1;          // == nkv0 without causal masking
                    const int u_next = unit_at(uit + 1);
                    const int nkv_next = u_next < p.num_units ? decode_unit<CAUSAL, MODS>(u_next, p).nkv1 : 0;
                    if (!early_t && !issue_first_s(ti, nkv, kc, uit & 1)) break;
                    early_t = false;
                    for (int j = 0; j < nkv; ++j) {
                        const uint32_t vst = (vc + j) % ST, vph = ((vc + j) / ST) & 1;
                        const uint32_t kn = kc + j + 1, kst = kn % ST, kph = (kn / ST) & 1;
                        if (j + 1 < nkv) {
                            if (!W(&sh.s_free[ti], sf_n & 1)) break;
                            ++sf_n;
                            if (!W(&sh.k_full[kst], kph)) break;
                            tc_fence_after();
                            issue_s(ti, kst);
                            commit(&sh.s_full[ti]);
                            commit(&sh.k_empty[kst]);
                            if (j + 2 == nkv) commit(&sh.q_empty[ti]);
                        }
                        if (!W(&sh.pv_ready[ti], pv_n & 1)) break;
                        ++pv_n;
                        if (j == 0 && uit > 0 && !W(&sh.o_free[ti], (uit - 1) & 1)) break;
                        if (!W(&sh.v_full[vst], vph)) break;
                        tc_fence_after();
                        issue_pv(ti, vst, j > 0);
                        commit(&sh.o_done[ti]);
                        commit(&sh.v_empty[vst]);
                        if (j + 1 == nkv) {
                            commit(&sh.o_final[ti]);
                            if (nkv_next > 0) {
                                if (!issue_first_s(ti, nkv_next, kc + nkv, (uit + 1) & 1)) break;
                                early_t = true;
                            }
                        }
                    }
                    kc += nkv;
                    vc += nkv;
                }
            } else {
                // d <= 64 issues S_i(0) of the next unit right after this unit's last PV_i rather than
                // after both tiles' last PVs, so tile 0's softmax restarts one PV group earlier.
                // Issued after that PV, S_i(0) needs no further ordering: its commit covers the PV.
                bool early[2] = {false, false};
                for (int u = unit_at(0); ok && u < p.num_units; u = unit_at(++uit)) {
                    const Unit U = decode_unit<CAUSAL, MODS>(u, p);
                    const int u_next = unit_at(uit + 1);
                    int nkv_next[2] = {0, 0};      // 0: no next unit
                    if (C::kSeparateP && u_next < p.num_units) {
                        const Unit Un = decode_unit<CAUSAL, MODS>(u_next, p);
                        nkv_next[0] = Un.nkv0;
                        nkv_next[1] = Un.nkv1;
                    }
                    // S0(0), S1(0), unless issued at the end of the previous unit
                    if (!early[0] && !issue_first_s(0, U.nkv0, kc, uit & 1)) break;
                    if (!early[1] && !issue_first_s(1, U.nkv1, kc, uit & 1)) break;
                    early[0] = early[1] = false;
                    for (int j = 0; j < U.nkv1; ++j) {
                        const uint32_t vst = (vc + j) % ST, vph = ((vc + j) / ST) & 1;
                        const uint32_t kn = kc + j + 1, kst = kn % ST, kph = (kn / ST) & 1;
                        if constexpr (C::kSeparateP) {
                            // S0(j+1), S1(j+1) as soon as the softmax has read S(j); then PV0(j), PV1(j)
                            if (j + 1 < U.nkv0) {
                                if (!W(&sh.s_free[0], sf_cnt[0] & 1)) break;
                                ++sf_cnt[0];
                                if (!W(&sh.k_full[kst], kph)) break;
                                tc_fence_after();
                                issue_s(0, kst);
                                commit(&sh.s_full[0]);
                                if (j + 2 == U.nkv0) commit(&sh.q_empty[0]);
                            }
                            if (j + 1 < U.nkv1) {
                                if (!W(&sh.s_free[1], sf_cnt[1] & 1)) break;
                                ++sf_cnt[1];
                                // (K(j+1) has been waited for by S0(j+1) unless tile 0 ends at j: only
                                // causal units give tile 1 one more key tile)
                                if (j + 1 >= U.nkv0 && !W(&sh.k_full[kst], kph)) break;
                                tc_fence_after();
                                issue_s(1, kst);
                                commit(&sh.s_full[1]);
                                commit(&sh.k_empty[kst]);
                                if (j + 2 == U.nkv1) commit(&sh.q_empty[1]);
                            }
                            if (j < U.nkv0) {
                                if (!W(&sh.pv_ready[0], pv_cnt[0] & 1)) break;
                                ++pv_cnt[0];
                                if (j == 0 && uit > 0 && !W(&sh.o_free[0], (uit - 1) & 1)) break;
                                if (!W(&sh.v_full[vst], vph)) break;
                                tc_fence_after();
                                issue_pv(0, vst, j > 0);
                                commit(&sh.o_done[0]);
                                if (j + 1 == U.nkv0) commit(&sh.o_final[0]);
                                if (j + 1 == U.nkv0 && nkv_next[0] > 0) {
                                    if (!issue_first_s(0, nkv_next[0], kc + U.nkv1, (uit + 1) & 1))
                                        break;
                                    early[0] = true;
                                }
                            }
                            if (!W(&sh.pv_ready[1], pv_cnt[1] & 1)) break;
                            ++pv_cnt[1];
                            if (j == 0 && uit > 0 && !W(&sh.o_free[1], (uit - 1) & 1)) break;
                            if (j >= U.nkv0 && !W(&sh.v_full[vst], vph)) break;   // else seen by PV0(j)
                            tc_fence_after();
                            issue_pv(1, vst, j > 0);
                            commit(&sh.o_done[1]);
                            commit(&sh.v_empty[vst]);
                            if (j + 1 == U.nkv1) commit(&sh.o_final[1]);
                            if (j + 1 == U.nkv1 && nkv_next[1] > 0) {
                                if (!issue_first_s(1, nkv_next[1], kc + U.nkv1, (uit + 1) & 1))
                                    break;
                                early[1] = true;
                            }
                            continue;
                        }
                        if (j < U.nkv0) {   // PV0(j)
                            if (!W(&sh.pv_ready[0], pv_cnt[0] & 1)) break;
                            ++pv_cnt[0];
                            if (j == 0 && uit > 0 && !W(&sh.o_free[0], (uit - 1) & 1)) break;
                            if (!W(&sh.v_full[vst], vph)) break;
                            tc_fence_after();
                            issue_pv(0, vst, j > 0);
                            commit(&sh.o_done[0]);
                        }
                        if (j + 1 < U.nkv0) {   // S0(j+1)
                            if (!W(&sh.k_full[kst], kph)) break;
                            tc_fence_after();
                            issue_s(0, kst);
                            commit(&sh.s_full[0]);
                            if (j + 2 == U.nkv0) commit(&sh.q_empty[0]);
                        }
                        // PV1(j)
                        if (!W(&sh.pv_ready[1], pv_cnt[1] & 1)) break;
                        ++pv_cnt[1];
                        if (j == 0 && uit > 0 && !W(&sh.o_free[1], (uit - 1) & 1)) break;
                        if (!W(&sh.v_full[vst], vph)) break;
                        tc_fence_after();
                        issue_pv(1, vst, j > 0);
                        commit(&sh.o_done[1]);
                        commit(&sh.v_empty[vst]);
                        if (j + 1 < U.nkv1) {   // S1(j+1)
                            if (!W(&sh.k_full[kst], kph)) break;
                            tc_fence_after();
                            issue_s(1, kst);
                            commit(&sh.s_full[1]);
                            commit(&sh.k_empty[kst]);
                            if (j + 2 == U.nkv1) commit(&sh.q_empty[1]);
                        }
                    }
                    kc += U.nkv1;
                    vc += U.nkv1;
                }
            }
            // drain: all MMAs complete before tensor memory is released
            commit(&sh.drain);
            drain_phase(&sh.drain, 0, p.status);
        }
        __syncwarp();
    } else if (wg < 2) {
        // ================================================================ softmax of tile i = wg
        regs_inc<C::kRegsSoftmax>();
        const int i = wg;
        const int t = threadIdx.x & 127;          // row within the tile
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t col_s = i ? C::kColS1 : C::kColS0;
        const uint32_t col_p = i ? C::kColP1 : C::kColP0;
        const uint32_t col_o = i ? C::kColO1 : C::kColO0;
        const float scale_log2 = p.scale_log2;
        // fast path: the row maximum over raw scores and the scale fused into the exponent's FMA
        // (no bias; of the score modifications only the left window, which only masks)
        const bool win = MODS && p.window_left >= 0;
        const bool fast = !HAS_BIAS && scale_log2 > 0.f && (!MODS || (p.alibi == nullptr && p.softcap <= 0.f));
        uint32_t s_cnt = 0, od_cnt = 0, bcnt = 0, uit = 0;
        bool ok = true;
        for (int u = unit_at(0); ok && u < p.num_units; u = unit_at(++uit)) {
            const Unit U = decode_unit<CAUSAL, MODS>(u, p);
            const int nkv = i ? U.nkv1 : U.nkv0;
            const int row = U.q0 + i * kBlockM + t;
            const int first_row = U.q0 + i * kBlockM;
            const T* bias_row = nullptr;
            if constexpr (HAS_BIAS)
                bias_row = reinterpret_cast<const T*>(p.bias) + U.b * p.bias_sb + U.h * p.bias_sh +
                           static_cast<int64_t>(row < U.N ? row : 0) * p.bias_si;
            float m_ref = -INFINITY;                // reference maximum (log2 domain)
            float l = 0.f;
            for (int j = 0; j < nkv; ++j) {
                ok = wait_phase(&sh.s_full[i], s_cnt & 1, abort_flag, p.wait_limit, p.status);
                ++s_cnt;
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
                float s[kBlockN];
                {
                    uint32_t r[kBlockN];
#pragma unroll
                    for (int c = 0; c < kBlockN / 32; ++c)
                        tmem_ld32(tmem + lane_off + col_s + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
                    tmem_wait_ld128(r);
#pragma unroll
                    for (int c = 0; c < kBlockN; ++c) s[c] = __uint_as_float(r[c]);
                }
                if constexpr (C::kSeparateP) {
                    // S_i may now be overwritten by S_i(j+1) (S_i(0) of the next unit is issued
                    // only after this unit's last PV_i, which needs this softmax to finish)
                    if (j + 1 < nkv) {
                        tc_fence_before();
                        mbar_arrive(&sh.s_free[i]);
                    }
                }
                const int kv0 = (U.kv_lo + j) * kBlockN;
                // key tiles past the end, and (causal) tiles reaching past the first row's last key
                const bool need_mask =
                    (kv0 + kBlockN > U.Nk) || (CAUSAL && kv0 + kBlockN - 1 > first_row + U.off);
                // left window: only a tile that starts before the window of its last row masks
                const bool need_win = win && kv0 < first_row + kBlockM - 1 + U.off - p.window_left;
                float m_tile;   // tile maximum, log2 domain
                if (fast) {
                    if (need_mask || need_win) {
                        const int lim = CAUSAL ? min(U.Nk - kv0, row + U.off - kv0 + 1) : (U.Nk - kv0);
                        if (win) {
                            mask_keys(s, row + U.off - p.window_left - kv0, lim);
                        } else {
#pragma unroll
                            for (int c = 0; c < kBlockN; ++c) s[c] = c < lim ? s[c] : -INFINITY;
                        }
                    }
                    m_tile = row_max(s) * scale_log2;
                } else {
                    const uint8_t* brow = nullptr;
                    uint32_t bst = 0;
                    if constexpr (BC::kTma) {
                        bst = bcnt % BC::kStages;
                        ok = wait_phase(&sh.bias_full[i][bst], (bcnt / BC::kStages) & 1, abort_flag, p.wait_limit,
                                        p.status);
                        ok = __all_sync(0xffffffffu, ok);
                        if (!ok) break;
                        brow = sBias + (i * BC::kStages + bst) * BC::kTileBytes + t * 128;
                    }
                    // y = scale * s + bias in natural units, one packed FMA per pair; the
                    // conversion to log2 units rides on the exponent's FMA below
                    const float sc = p.scale;
#pragma unroll
                    for (int c = 0; c < kBlockN; c += 8) {
                        if constexpr (HAS_BIAS) {
                            uint4 raw;
                            if constexpr (BC::kTma) {
                                // chunk (c % 64) / 8 of box c / 64, 128-byte swizzle
                                raw = *reinterpret_cast<const uint4*>(
                                    brow + (c / 64) * BC::kBoxBytes + ((((c % 64) / 8) ^ (t & 7)) << 4));
                            } else if (row < U.N && kv0 + c + 8 <= U.Nk) {
                                raw = __ldg(reinterpret_cast<const uint4*>(bias_row + kv0 + c));
                            } else {
                                T e[8];
#pragma unroll
                                for (int q = 0; q < 8; ++q)
                                    e[q] = (row < U.N && kv0 + c + q < U.Nk) ? bias_row[kv0 + c + q] : T(0.f);
                                raw = *reinterpret_cast<const uint4*>(e);
                            }
                            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                float b0, b1;
                                unpack2<T>(w[q], b0, b1);
                                ffma2(s[c + 2 * q], s[c + 2 * q + 1], s[c + 2 * q], s[c + 2 * q + 1], sc, sc, b0, b1);
                            }
                        } else {
#pragma unroll
                            for (int q = 0; q < 8; q += 2)
                                fmul2(s[c + q], s[c + q + 1], s[c + q], s[c + q + 1], sc, sc);
                        }
                    }
                    if constexpr (BC::kTma) {          // the staged bias tile may be refilled
                        mbar_arrive(&sh.bias_empty[i][bst]);
                        ++bcnt;
                    }
                    int lo = 0;                        // first visible key of the tile (left window)
                    if constexpr (MODS) {
                        if (p.alibi != nullptr) {      // linear distance penalty of this head
                            const float slope = p.alibi[U.h];
                            const float dist0 = static_cast<float>(row + U.off - kv0);   // exact below 2^24
#pragma unroll
                            for (int c = 0; c < kBlockN; ++c) s[c] = fmaf(-slope, fabsf(dist0 - c), s[c]);
                        }
                        if (p.softcap > 0.f) {         // c tanh(s / c): one MUFU operation per score
                            const float cap = p.softcap, inv = 1.f / p.softcap;
#pragma unroll
                            for (int c = 0; c < kBlockN; ++c) s[c] = cap * tanh_approx(s[c] * inv);
                        }
                        if (p.window_left >= 0) lo = row + U.off - p.window_left - kv0;
                    }
                    if (need_mask || need_win) {
                        const int lim = CAUSAL ? min(U.Nk - kv0, row + U.off - kv0 + 1) : (U.Nk - kv0);
                        if (win) {
                            mask_keys(s, lo, lim);
                        } else {
#pragma unroll
                            for (int c = 0; c < kBlockN; ++c) s[c] = c < lim ? s[c] : -INFINITY;
                        }
                    }
                    m_tile = row_max(s) * kLog2e;
                }
                // reference maximum: move it only when the row maximum grew by more than the threshold
                float m_new = m_ref, alpha = 1.f;
                if (m_ref == -INFINITY) {
                    m_new = m_tile;
                    alpha = 0.f;
                } else if (m_tile > m_ref + kRescaleThreshold) {
                    m_new = m_tile;
                    alpha = ex2_approx(m_ref - m_new);
                }
                if (!C::kInlineRescale && j > 0) {
                    // d = 128: S_i(j) was issued after PV_i(j-1), so the correction has consumed
                    // alpha(j-1); it rescales O_i while the exponentials below run
                    sh.alpha[j & 1][i][t] = alpha;
                    mbar_arrive(&sh.sm2corr[i]);
                }
                const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
                // p = 2^(x - m): x = s * scale_log2 on the fast path (s raw), x = y * log2(e) otherwise.
                // At d=64 one pair in four goes through the FMA-pipe exponential so that the
                // MUFU unit (16 lanes per clock per SM) is not the only exp resource.
                const float xa = fast ? scale_log2 : kLog2e;
                const float xb = -m_use;
                float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                // With separate P columns (d <= 64) all of P is formed first, packed in registers
                // (s dies as P is formed), so that the wait for the previous PV_i below comes after
                // the exponentials, not between them.  At d = 128 P goes into S_i's own columns,
                // which nothing else reads now: each half is stored as soon as it is formed.
                constexpr int kWords = FP8 ? 32 : 64;      // 32-bit words of this row's packed P
                uint32_t pk[kWords];
                auto store_p_half = [&](int half) {
                    if constexpr (FP8)
                        tmem_st16(tmem + lane_off + col_p + half * 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[half * 16]));
                    else
                        tmem_st32(tmem + lane_off + col_p + half * 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[half * 32]));
                };
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float ep0 = 0.f, ep1 = 0.f;            // e4m3: the even pair of the current word
#pragma unroll
                    for (int q2 = 0; q2 < 32; ++q2) {
                        const int pp = half * 32 + q2;
                        float x0, x1, e0, e1;
                        ffma2(x0, x1, s[2 * pp], s[2 * pp + 1], xa, xa, xb, xb);
                        constexpr int kEmu = C::kEmuPeriod;
                        if (kEmu > 0 && pp % (kEmu > 0 ? kEmu : 1) == kEmu - 1) {
                            ex2_emu2(e0, e1, x0, x1);
                        } else {
                            e0 = ex2_approx(x0);
                            e1 = ex2_approx(x1);
                        }
                        const int q = (pp & 3) * 2;
                        fadd2_ftz(acc[q], acc[q + 1], acc[q], acc[q + 1], e0, e1);
                        if constexpr (FP8) {
                            // four keys per 32-bit word: the even pair waits for the odd one
                            if (pp & 1) pk[pp >> 1] = pack4_e4m3(ep0, ep1, e0, e1);
                            else { ep0 = e0; ep1 = e1; }
                        } else {
                            pk[pp] = pack2<T>(e0, e1);
                        }
                    }
                    if constexpr (!C::kSeparateP) store_p_half(half);
                }
                if constexpr (C::kSeparateP) {
                    // P_i(j) overwrites P_i(j-1), and O_i may be rescaled below: PV_i(j-1) must
                    // have completed.  (Iteration 0 needs no wait: S_i(0) was issued after the
                    // previous unit's last PV_i, and its commit covers that PV.)  At d = 128
                    // S_i(j) was issued after PV_i(j-1) by the same thread, so the completion of
                    // S_i(j), awaited above, already covers that PV.
                    if (j > 0) {
                        ok = wait_phase(&sh.o_done[i], od_cnt & 1, abort_flag, p.wait_limit, p.status);
                        ++od_cnt;
                        ok = __all_sync(0xffffffffu, ok);
                        if (!ok) break;
                        tc_fence_after();
                    }
                }
                // O_i *= alpha when the reference maximum moved (rare with the threshold): each
                // warp rescales its own 32 rows in tensor memory before releasing PV_i(j)
                if (C::kInlineRescale && j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                    uint32_t r[16];               // (16-column chunks: few registers live here)
#pragma unroll 1
                    for (int c = 0; c < D / 16; ++c) {
                        tmem_ld16(tmem + lane_off + col_o + c * 16, r);
                        tmem_wait_ld16(r);
#pragma unroll
                        for (int q = 0; q < 16; q += 2) {
                            float y0, y1;
                            fmul2(y0, y1, __uint_as_float(r[q]), __uint_as_float(r[q + 1]), alpha, alpha);
                            r[q] = __float_as_uint(y0);
                            r[q + 1] = __float_as_uint(y1);
                        }
                        tmem_st16(tmem + lane_off + col_o + c * 16, r);
                    }
                }
                if constexpr (C::kSeparateP) {
                    store_p_half(0);
                    store_p_half(1);
                }
                tmem_wait_st();
                const float rsum = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
                l = fmaf(l, alpha, rsum);
                m_ref = m_new;
                tc_fence_before();
                mbar_arrive(&sh.pv_ready[i]);
            }
            if (!ok) break;
            // The epilogue must have consumed the previous unit's statistics before this unit's
            // are published: a unit with a single key tile can otherwise finish before the
            // epilogue reaches the previous unit, running stats_full two phases ahead.
            if constexpr (C::kSeparateP) ++od_cnt;   // the unit's last PV_i is not waited for here
            if (uit > 0) {
                ok = wait_phase(&sh.o_free[i], (uit - 1) & 1, abort_flag, p.wait_limit, p.status);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
            }
            sh.stat_m[uit & 1][i][t] = m_ref;
            sh.stat_l[uit & 1][i][t] = l;
            mbar_arrive(&sh.stats_full[i]);
        }
    } else {
        // ================================================================ (correction +) epilogue
        regs_dec<C::kRegsEpilogue>();
        const int t = threadIdx.x & 127;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        constexpr uint32_t kColO[2] = {C::kColO0, C::kColO1};
        uint32_t st_cnt[2] = {0, 0}, of_cnt[2] = {0, 0}, c_cnt[2] = {0, 0}, uit = 0;
        bool ok = true;
        auto WS = [&](uint64_t* bar, uint32_t& cnt) {
            if (ok) ok = wait_phase(bar, cnt & 1, abort_flag, p.wait_limit, p.status);
            ++cnt;
            ok = __all_sync(0xffffffffu, ok);
            return ok;
        };
        const bool has_next_unit_pv_arrival = !C::kInlineRescale;
        for (int u = unit_at(0); ok && u < p.num_units; u = unit_at(++uit)) {
            const Unit U = decode_unit<CAUSAL, MODS>(u, p);
            if constexpr (!C::kInlineRescale) {
                // d = 128, the correction: O_i *= alpha(j) between PV_i(j-1) and PV_i(j) (only when
                // some row of the warp moved its reference maximum), then its pv_ready arrival.
                // Its o_done waits use the of_cnt counters: every PV_i phase, the last one in the
                // epilogue below.
                for (int j = 0; ok && j < U.nkv1; ++j) {
                    for (int i = 0; i < 2; ++i) {
                        if (j >= (i ? U.nkv1 : U.nkv0)) continue;
                        if (j > 0) {
                            if (!WS(&sh.sm2corr[i], c_cnt[i])) break;
                            const float alpha = sh.alpha[j & 1][i][t];
                            if (!WS(&sh.o_done[i], of_cnt[i])) break;   // PV_i(j-1) complete
                            tc_fence_after();
                            if (__any_sync(0xffffffffu, alpha != 1.f)) {
                                uint32_t r[32];
#pragma unroll
                                for (int c = 0; c < D / 32; ++c) {
                                    tmem_ld32(tmem + lane_off + kColO[i] + c * 32, r);
                                    tmem_wait_ld(r);
#pragma unroll
                                    for (int q = 0; q < 32; q += 2) {
                                        float x0, x1;
                                        fmul2(x0, x1, __uint_as_float(r[q]), __uint_as_float(r[q + 1]), alpha, alpha);
                                        r[q] = __float_as_uint(x0);
                                        r[q + 1] = __float_as_uint(x1);
                                    }
                                    tmem_st32(tmem + lane_off + kColO[i] + c * 32, r);
                                }
                                tmem_wait_st();
                            }
                            tc_fence_before();
                            mbar_arrive(&sh.pv_ready[i]);
                        } else if (uit == 0) {
                            mbar_arrive(&sh.pv_ready[i]);   // later units: arrived by the previous epilogue
                        }
                    }
                }
                if (!ok) break;
            }
            // O = O_acc / l (* sigmoid(G)), lse = (m + log2 l) * ln 2.  O_i is released as soon as
            // its last chunk is in registers (at d = 128 together with the next unit's first
            // pv_ready arrival: iteration 0 needs no rescale), so the next unit's PV_i(0) does not
            // wait for the gate arithmetic and the global stores.
            const bool has_next = has_next_unit_pv_arrival && unit_at(uit + 1) < p.num_units;
            for (int i = 0; i < 2; ++i) {
                const int row = U.q0 + i * kBlockM + t;
                const bool row_ok = row < U.N;
                T* orow = reinterpret_cast<T*>(p.out) + U.b * p.out_sb + U.h * p.out_sh +
                          static_cast<int64_t>(U.q_base + (row_ok ? row : 0)) * p.out_si;
                const T* grow = nullptr;
                if constexpr (HAS_GATE)
                    grow = reinterpret_cast<const T*>(p.gate) + U.b * p.gate_sb + U.h * p.gate_sh +
                           static_cast<int64_t>(U.q_base + (row_ok ? row : 0)) * p.gate_si;
                constexpr int kPre = (HAS_GATE && D == 32) ? D / 8 : 1;   // gate row prefetched (d = 32)
                uint4 graw[kPre];
                if constexpr (HAS_GATE && D == 32) {
                    if (row_ok) {
#pragma unroll
                        for (int v8 = 0; v8 < D / 8; ++v8) graw[v8] = __ldg(reinterpret_cast<const uint4*>(grow + v8 * 8));
                    }
                }
                if (!WS(&sh.stats_full[i], st_cnt[i])) break;  // final m, l
                // the unit's last PV_i complete (d = 128: the last phase of o_done)
                if (!WS(C::kInlineRescale ? &sh.o_final[i] : &sh.o_done[i], of_cnt[i])) break;
                tc_fence_after();
                const float m = sh.stat_m[uit & 1][i][t];
                const float l = sh.stat_l[uit & 1][i][t];
                // (e4m3 inputs: the value tensor's scale comes in here)
                const float inv_l = (l > 0.f) ? (FP8 ? p.v_scale / l : 1.f / l) : 0.f;
                // one 32-column chunk of O: normalise, gate, round, store
                auto finish_chunk = [&](const uint32_t (&r)[32], int c) {
                    if (!row_ok) return;
#pragma unroll
                    for (int v8 = 0; v8 < 4; ++v8) {
                        float o[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q) o[q] = __uint_as_float(r[v8 * 8 + q]) * inv_l;
                        if constexpr (HAS_GATE) {
                            uint4 raw;
                            if constexpr (D == 32) raw = graw[v8];
                            else raw = __ldg(reinterpret_cast<const uint4*>(grow + c * 32 + v8 * 8));
                            const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
                            // sigmoid(g) = (1 + tanh(g / 2)) / 2: one MUFU operation per element
                            for (int q = 0; q < 8; ++q) o[q] *= fmaf(0.5f, tanh_approx(0.5f * to_f32<T>(e[q])), 0.5f);
                        }
                        uint4 w;
                        w.x = pack2<T>(o[0], o[1]);
                        w.y = pack2<T>(o[2], o[3]);
                        w.z = pack2<T>(o[4], o[5]);
                        w.w = pack2<T>(o[6], o[7]);
                        *reinterpret_cast<uint4*>(orow + c * 32 + v8 * 8) = w;
                    }
                };
                uint32_t r[32];
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    tmem_ld32(tmem + lane_off + kColO[i] + c * 32, r);
                    tmem_wait_ld(r);
                    if (c == D / 32 - 1) {        // O_i fully read: release it
                        tc_fence_before();
                        mbar_arrive(&sh.o_free[i]);
                        if (has_next) mbar_arrive(&sh.pv_ready[i]);
                    }
                    finish_chunk(r, c);
                }
                ATTN_CHECK(p.status, !row_ok || (U.q_base + row >= 0 && U.q_base + row < (p.n_seq > 0 ? p.N : U.N)));
                if (p.lse != nullptr && row_ok)
                    p.lse[U.b * p.lse_sb + U.h * p.lse_sh + U.q_base + row] =
                        (l > 0.f) ? (m + lg2_approx(l)) * kLn2 : -INFINITY;
            }
        }
    }

    // ---------------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 12) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace attn
