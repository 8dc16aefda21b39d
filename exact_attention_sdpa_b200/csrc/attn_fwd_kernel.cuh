// attn_fwd_kernel.cuh -- fused exact attention forward for sm_100a.
//
// One CTA owns one 128-row query tile of one (batch, head) and walks its key /
// value tiles of 128 rows (aiinarabic.com "flash-attention", the per-block
// order: load a block of Q, K, V on chip, QK^T for the block, softmax of the
// block, multiply by V, merge with what came before, advance).  The merge is
// the online softmax of the gist.science FLASHLIGHT summary (Methodology,
// item 3): a running row maximum m and running sum l, with l and the output
// accumulator rescaled by e^(m_old - m_new) whenever the maximum grows, so no
// score or probability tile ever leaves the chip.
//
// Roles (warp specialisation):
//   warps 0-3  softmax: thread t owns query row t of the tile.  It reads its
//              score row from tensor memory, masks / scales / biases it, updates
//              m and l, writes the probabilities P (fp16/bf16) back to tensor
//              memory, rescales its output row when m grew, and finally
//              normalises, gates and stores O and lse.
//   warp 4     TMA producer: Q once, then K_j and V_j into a 2-stage ring.
//   warp 5     MMA issuer (one thread): S_j = Q K_j^T (both operands in shared
//              memory) into one of two S buffers, and O += P_j V_j with P read
//              from tensor memory.  S_{j+1} is issued before waiting for P_j so
//              the next score tile is computed while row softmax runs.
//
// Tensor memory (512 columns x 128 lanes, lane = query row):
//   [0,128)   S buffer 0 (fp32)      [128,256) S buffer 1 (fp32)
//   [256,320) P buffer 0 (2 x 16-bit per column)
//   [320,384) P buffer 1             [384,384+d) O accumulator (fp32)
//
// Every mbarrier wait is bounded; a wait that gives up records a timeout in
// the device status word, raises a CTA-wide abort flag, and every role then
// drains what it has in flight and the CTA exits normally.
#pragma once

#include "sm100.cuh"

namespace attn {

constexpr int kBlockM = 128;
constexpr int kBlockN = 128;
constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColP0 = 256, kColP1 = 320, kColO = 384;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned long long kDrainLimit = 1ull << 32;

struct FwdParams {
    int B, H, N;
    int num_q_tiles;
    int num_units;             // num_q_tiles * B * H
    float scale_log2;          // scale * log2(e)
    const void* bias;          // nullable
    int64_t bias_sb, bias_sh, bias_si;   // element strides (bias_sb = 0 when shared over B)
    const void* gate;          // nullable
    int64_t gate_sb, gate_sh, gate_si;
    void* out;
    int64_t out_sb, out_sh, out_si;
    float* lse;                // nullable, [B*H*N]
    unsigned long long wait_limit;
    unsigned int* status;
};

struct __align__(8) FwdBarriers {
    uint64_t q_full;
    uint64_t k_full[kStages];
    uint64_t v_full[kStages];
    uint64_t kv_empty[kStages];
    uint64_t s_full[2];
    uint64_t p_full;
    uint64_t o_done;
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

// Bounded wait.  Returns false (and raises the abort flag) if the phase did
// not complete within `limit` cycles or another role aborted first.
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, FwdBarriers* sb,
                                           unsigned long long limit, unsigned int* status) {
    const uint32_t a = sm100::smem_u32(bar);
    if (sm100::mbar_try_wait(a, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (sm100::mbar_try_wait(a, parity)) return true;
        if (*reinterpret_cast<volatile int*>(&sb->abort_flag)) return false;
        if (static_cast<unsigned long long>(clock64() - t0) > limit) {
            atomicOr(status, kStatusTimeout);
            *reinterpret_cast<volatile int*>(&sb->abort_flag) = 1;
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

template <int D>
struct TileGeom {
    static_assert(D == 32 || D == 64 || D == 128, "head dim");
    // a tile of 128 rows x D 16-bit elements is stored as D/64 "atoms" of
    // 128 rows x 128 bytes (128-byte swizzle), or for D = 32 one atom of
    // 128 rows x 64 bytes (64-byte swizzle), exactly as TMA writes it.
    static constexpr int kAtomCols = (D >= 64) ? 64 : 32;       // elements per row per atom
    static constexpr int kNumAtoms = D / kAtomCols;
    static constexpr int kRowBytes = kAtomCols * 2;               // 128 or 64
    static constexpr int kAtomBytes = 128 * kRowBytes;
    static constexpr int kTileBytes = kNumAtoms * kAtomBytes;     // 128 * D * 2
    static constexpr uint32_t kLayout = (D >= 64) ? 2u : 4u;      // SW128 : SW64
    static constexpr uint32_t kSBO = 8 * kRowBytes;               // 8-row group stride
};

template <int D>
struct FwdSmem {
    static constexpr int kTile = TileGeom<D>::kTileBytes;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kTile;
    static constexpr int kOffV = kOffK + kStages * kTile;
    static constexpr int kBytes = kOffV + kStages * kTile;
    // pad so that at most one CTA is resident per SM (it allocates all 512 TMEM columns)
    static constexpr int kDynBytes = (kBytes + 1024 > 120 * 1024) ? (kBytes + 1024) : (120 * 1024);
};

template <typename T, int D, bool CAUSAL, bool HAS_BIAS, bool HAS_GATE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using namespace sm100;
    using G = TileGeom<D>;
    using L = FwdSmem<D>;
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;

    extern __shared__ uint8_t smem_raw[];
    __shared__ FwdBarriers sbar;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + L::kOffQ;
    uint8_t* sK = smem + L::kOffK;
    uint8_t* sV = smem + L::kOffV;

    const int warp = warp_id();
    const int lane = lane_id();

    // work unit: heaviest query tiles first (causal), then (b, h)
    const int BH = p.B * p.H;
    const int unit = blockIdx.x;
    const int qt = p.num_q_tiles - 1 - unit / BH;
    const int bh = unit % BH;
    const int b = bh / p.H;
    const int h = bh % p.H;
    const int q0 = qt * kBlockM;
    const int n_kv_all = (p.N + kBlockN - 1) / kBlockN;
    const int nkv = CAUSAL ? min(n_kv_all, qt + 1) : n_kv_all;

    if (threadIdx.x == 0) {
        mbar_init(&sbar.q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sbar.k_full[s], 1);
            mbar_init(&sbar.v_full[s], 1);
            mbar_init(&sbar.kv_empty[s], 1);
        }
        mbar_init(&sbar.s_full[0], 1);
        mbar_init(&sbar.s_full[1], 1);
        mbar_init(&sbar.p_full, kBlockM);
        mbar_init(&sbar.o_done, 1);
        mbar_init(&sbar.drain, 1);
        sbar.abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 4) {
        tmem_alloc(&sbar.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sbar.tmem_base;

    if (warp == 4) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            const uint64_t pol_q = policy_evict_first();
            const uint64_t pol_kv = policy_evict_last();
            mbar_arrive_expect_tx(&sbar.q_full, G::kTileBytes);
            for (int a = 0; a < G::kNumAtoms; ++a)
                tma_load_4d(sQ + a * G::kAtomBytes, &tm_q, &sbar.q_full, a * G::kAtomCols, q0, h, b, pol_q);
            int issued[kStages] = {0, 0};
            for (int j = 0; j < nkv; ++j) {
                const int st = j % kStages;
                if (j >= kStages) {
                    if (!wait_phase(&sbar.kv_empty[st], ((j / kStages) - 1) & 1, &sbar, p.wait_limit, p.status))
                        break;
                }
                uint8_t* dk = sK + st * G::kTileBytes;
                uint8_t* dv = sV + st * G::kTileBytes;
                mbar_arrive_expect_tx(&sbar.k_full[st], G::kTileBytes);
                for (int a = 0; a < G::kNumAtoms; ++a)
                    tma_load_4d(dk + a * G::kAtomBytes, &tm_k, &sbar.k_full[st], a * G::kAtomCols, j * kBlockN,
                                h, b, pol_kv);
                mbar_arrive_expect_tx(&sbar.v_full[st], G::kTileBytes);
                for (int a = 0; a < G::kNumAtoms; ++a)
                    tma_load_4d(dv + a * G::kAtomBytes, &tm_v, &sbar.v_full[st], a * G::kAtomCols, j * kBlockN,
                                h, b, pol_kv);
                ++issued[st];
            }
            // drain: every load issued into this CTA's shared memory has landed before exit
            drain_phase(&sbar.q_full, 0, p.status);
            for (int st = 0; st < kStages; ++st) {
                if (issued[st] > 0) {
                    drain_phase(&sbar.k_full[st], (issued[st] - 1) & 1, p.status);
                    drain_phase(&sbar.v_full[st], (issued[st] - 1) & 1, p.status);
                }
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = instr_desc_f16(kBF16, kBlockM, kBlockN, false);
            constexpr uint32_t idesc_o = instr_desc_f16(kBF16, kBlockM, D, true);
            const uint32_t q_addr = smem_u32(sQ);
            const uint32_t k_addr = smem_u32(sK);
            const uint32_t v_addr = smem_u32(sV);
            auto issue_s = [&](int j) {
                const int st = j % kStages;
                const uint32_t kb = k_addr + st * G::kTileBytes;
                const uint32_t dst = tmem + ((j & 1) ? kColS1 : kColS0);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    // K-major operands: 16 elements (32 bytes) per step inside an atom
                    const int atom = (kk * 16) / G::kAtomCols;
                    const uint32_t off = atom * G::kAtomBytes + ((kk * 16) % G::kAtomCols) * 2;
                    const uint64_t da = smem_desc(q_addr + off, 16, G::kSBO, G::kLayout);
                    const uint64_t db = smem_desc(kb + off, 16, G::kSBO, G::kLayout);
                    mma_ss(dst, da, db, idesc_s, kk > 0 ? 1u : 0u);
                }
            };
            bool ok = wait_phase(&sbar.q_full, 0, &sbar, p.wait_limit, p.status);
            if (ok) ok = wait_phase(&sbar.k_full[0], 0, &sbar, p.wait_limit, p.status);
            if (ok) {
                tc_fence_after();
                issue_s(0);
                mma_commit(&sbar.s_full[0]);
            }
            for (int j = 0; ok && j < nkv; ++j) {
                if (j + 1 < nkv) {
                    const int st1 = (j + 1) % kStages;
                    if (!wait_phase(&sbar.k_full[st1], ((j + 1) / kStages) & 1, &sbar, p.wait_limit, p.status))
                        break;
                    tc_fence_after();
                    issue_s(j + 1);
                    mma_commit(&sbar.s_full[(j + 1) & 1]);
                }
                if (!wait_phase(&sbar.p_full, j & 1, &sbar, p.wait_limit, p.status)) break;
                const int st = j % kStages;
                if (!wait_phase(&sbar.v_full[st], (j / kStages) & 1, &sbar, p.wait_limit, p.status)) break;
                tc_fence_after();
                const uint32_t vb = v_addr + st * G::kTileBytes;
                const uint32_t pcol = tmem + ((j & 1) ? kColP1 : kColP0);
#pragma unroll
                for (int kk = 0; kk < kBlockN / 16; ++kk) {
                    // V is N(=d)-major: 16 keys per step = 16 rows of the tile
                    const uint64_t dv = smem_desc(vb + kk * 16 * G::kRowBytes, G::kAtomBytes, G::kSBO, G::kLayout);
                    mma_ts(tmem + kColO, pcol + kk * 8, dv, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&sbar.o_done);
                mma_commit(&sbar.kv_empty[st]);
            }
            // drain: all MMAs complete before tensor memory is released
            mma_commit(&sbar.drain);
            drain_phase(&sbar.drain, 0, p.status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ softmax / epilogue
        const int t = threadIdx.x;              // 0..127, the query row within the tile
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const int row = q0 + t;
        const bool row_ok = row < p.N;
        float m_run = -INFINITY;                // running max, log2 domain
        float l_run = 0.f;                      // running sum
        bool ok = true;
        const T* bias_row = nullptr;
        if constexpr (HAS_BIAS) {
            bias_row = reinterpret_cast<const T*>(p.bias) + b * p.bias_sb + h * p.bias_sh +
                       static_cast<int64_t>(row_ok ? row : 0) * p.bias_si;
        }

        for (int j = 0; j < nkv; ++j) {
            const int sbuf = j & 1;
            ok = wait_phase(&sbar.s_full[sbuf], (j >> 1) & 1, &sbar, p.wait_limit, p.status);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();

            float s[kBlockN];
            {
                uint32_t r[32];
#pragma unroll
                for (int c = 0; c < kBlockN / 32; ++c) {
                    tmem_ld32(tmem + lane_off + (sbuf ? kColS1 : kColS0) + c * 32, r);
                    tmem_wait_ld(r);
#pragma unroll
                    for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(r[i]);
                }
            }
            const int kv0 = j * kBlockN;
            const bool need_mask = (kv0 + kBlockN > p.N) || (CAUSAL && j == qt);
            float mx = m_run;
#pragma unroll
            for (int c = 0; c < kBlockN; c += 8) {
                float bv[8];
                if constexpr (HAS_BIAS) {
                    if (row_ok && kv0 + c + 8 <= p.N) {
                        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(bias_row + kv0 + c));
                        const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
                        for (int i = 0; i < 8; ++i) bv[i] = to_f32<T>(e[i]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            bv[i] = (row_ok && kv0 + c + i < p.N) ? to_f32<T>(bias_row[kv0 + c + i]) : 0.f;
                    }
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float x = s[c + i] * p.scale_log2;
                    if constexpr (HAS_BIAS) x = fmaf(bv[i], kLog2e, x);
                    if (need_mask) {
                        const int key = kv0 + c + i;
                        if (key >= p.N || (CAUSAL && key > row)) x = -INFINITY;
                    }
                    s[c + i] = x;
                    mx = fmaxf(mx, x);
                }
            }
            const float alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - mx);
            const float m_use = (mx == -INFINITY) ? 0.f : mx;
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < kBlockN; ++c) {
                const float e = ex2_approx(s[c] - m_use);
                s[c] = e;
                sum += e;
            }
            l_run = fmaf(l_run, alpha, sum);
            m_run = mx;

            // O_{j-1} must be complete before rescaling O (and before P_{j} overwrites P_{j-2}'s buffer)
            if (j > 0) {
                ok = wait_phase(&sbar.o_done, (j - 1) & 1, &sbar, p.wait_limit, p.status);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
            }
            {
                uint32_t pk[32];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) pk[i] = pack2<T>(s[half * 64 + 2 * i], s[half * 64 + 2 * i + 1]);
                    tmem_st32(tmem + lane_off + (sbuf ? kColP1 : kColP0) + half * 32, pk);
                }
            }
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                uint32_t r[32];
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    tmem_ld32(tmem + lane_off + kColO + c * 32, r);
                    tmem_wait_ld(r);
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                    tmem_st32(tmem + lane_off + kColO + c * 32, r);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sbar.p_full);
        }

        if (ok) {
            ok = wait_phase(&sbar.o_done, (nkv - 1) & 1, &sbar, p.wait_limit, p.status);
            ok = __all_sync(0xffffffffu, ok);
        }
        if (ok) {
            tc_fence_after();
            const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
            T* orow = reinterpret_cast<T*>(p.out) + b * p.out_sb + h * p.out_sh +
                      static_cast<int64_t>(row_ok ? row : 0) * p.out_si;
            const T* grow = nullptr;
            if constexpr (HAS_GATE)
                grow = reinterpret_cast<const T*>(p.gate) + b * p.gate_sb + h * p.gate_sh +
                       static_cast<int64_t>(row_ok ? row : 0) * p.gate_si;
            uint32_t r[32];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                tmem_ld32(tmem + lane_off + kColO + c * 32, r);
                tmem_wait_ld(r);
                float o[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = __uint_as_float(r[i]) * inv_l;
                if constexpr (HAS_GATE) {
                    if (row_ok) {
#pragma unroll
                        for (int v8 = 0; v8 < 4; ++v8) {
                            const uint4 raw = __ldg(reinterpret_cast<const uint4*>(grow + c * 32 + v8 * 8));
                            const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const float g = to_f32<T>(e[i]);
                                o[v8 * 8 + i] *= 1.f / (1.f + ex2_approx(-g * kLog2e));
                            }
                        }
                    }
                }
                if (row_ok) {
#pragma unroll
                    for (int v8 = 0; v8 < 4; ++v8) {
                        uint4 w;
                        w.x = pack2<T>(o[v8 * 8 + 0], o[v8 * 8 + 1]);
                        w.y = pack2<T>(o[v8 * 8 + 2], o[v8 * 8 + 3]);
                        w.z = pack2<T>(o[v8 * 8 + 4], o[v8 * 8 + 5]);
                        w.w = pack2<T>(o[v8 * 8 + 6], o[v8 * 8 + 7]);
                        *reinterpret_cast<uint4*>(orow + c * 32 + v8 * 8) = w;
                    }
                }
            }
            if (p.lse != nullptr && row_ok) {
                const float lse = (l_run > 0.f) ? (m_run + lg2_approx(l_run)) * kLn2 : -INFINITY;
                p.lse[static_cast<int64_t>(bh) * p.N + row] = lse;
            }
        }
    }

    // ---------------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace attn
