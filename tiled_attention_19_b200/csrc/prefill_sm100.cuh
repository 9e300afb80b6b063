// prefill_sm100.cuh -- exact attention forward on B200 tensor cores (tcgen05 + TMEM + TMA).
//
// Computes O = softmax(Q K^T * scale [+ causal mask]) V per head, tile by tile, with
// an online softmax, writing only O and the per-row log-sum-exp ("Self-attention,
// CUDA kernels and FlashAttention", section 3: tiling, the online-softmax trick that
// tracks the running maximum and normaliser and rescales partial outputs, and the
// saved normalisation statistics). The score matrix lives only in tensor memory.
//
// One CTA owns one 128-row query tile of one (batch, head) and walks its 128-key
// tiles. Roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t, which is TMEM lane t. It loads a
//              row of S from TMEM, masks, updates the running max (log2 domain,
//              scale folded into the exponent), forms P = 2^(S*c - m) in f16/bf16
//              and stores it back into the same TMEM columns, corrects O when the
//              reference max moved, and finally writes O / l and the lse.
//   warp 4     producer: one lane issues TMA loads of Q once and of K_j, V_j into a
//              ring of shared-memory stages (128-byte swizzle).
//   warp 5     MMA issuer: one lane issues S_j = Q K_j^T (both operands in smem) and
//              O += P_j V_j (P from TMEM, V from smem); it also owns TMEM allocation.
// S/P use three 128-column TMEM buffers so S_{j+1} is computed while row j's
// softmax runs; O uses 128 columns after them (512 columns in total).
//
// Causal masking (the "Flash Attention" skill page, Scenario 2 step 2: causal=True
// for autoregressive models): key j is visible to query i iff j <= i + (Lk - Lq).
// Key tiles entirely above the diagonal of the tile's last row are never loaded or
// multiplied; the mask itself is applied only on tiles that cross the diagonal or
// the ragged end of the keys.
//
// Lazy rescaling: the reference max m of a row moves only when a tile's maximum
// exceeds it by more than 8 (log2 units). Until then p = 2^(s*c - m) <= 2^8, which
// f16/bf16 and fp32 hold without loss, and O and l keep a common reference, so the
// final O / l is unchanged; O in TMEM is rescaled only when m moves.
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace attn {

constexpr int kBM = 128;          // query rows per tile
constexpr int kBN = 128;          // keys per tile
constexpr int kSBufs = 3;         // S/P buffers in TMEM
constexpr int kPrefillThreads = 192;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct PrefillCfg {
    static constexpr int kChunks = D / 64;             // 64-element (128-byte) column chunks
    static constexpr int kChunkBytes = kBM * 128;      // one chunk of a 128-row tile
    static constexpr int kTileBytes = kBM * D * 2;     // a whole Q, K or V tile
    static constexpr int kStages = (D == 64) ? 4 : 3;  // K/V ring depth
    static constexpr int kOCol = kSBufs * kBN;         // first TMEM column of O
    static constexpr int kTmemCols = 512;
    static constexpr int kNumBars = 1 + 3 * kStages + 3 * kSBufs + 2;
    static constexpr int kTileRegion = kTileBytes * (1 + 2 * kStages);
    static constexpr int kSmemBytes = 1024 /*alignment slack*/ + kTileRegion + kNumBars * 8 + 16;
    static_assert(kOCol + D <= kTmemCols, "TMEM budget");
    static_assert(kSmemBytes <= 232448, "shared-memory budget");
};

struct PrefillArgs {
    void* out;
    float* lse;
    int Hq, Hkv, group, Lq, Lk;
    int n_q_tiles;
    float scale_log2;  // scale * log2(e)
};

template <int D, bool BF16, bool CAUSAL>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    prefill_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const PrefillArgs args) {
    using Cfg = PrefillCfg<D>;
    constexpr int NS = Cfg::kStages;
    // barrier slots
    constexpr int Q_FULL = 0;
    constexpr int K_FULL = 1;
    constexpr int V_FULL = K_FULL + NS;
    constexpr int KV_EMPTY = V_FULL + NS;
    constexpr int S_FULL = KV_EMPTY + NS;
    constexpr int P_FULL = S_FULL + kSBufs;
    constexpr int PV_BUF = P_FULL + kSBufs;
    constexpr int PV_DONE = PV_BUF + kSBufs;
    constexpr int DRAIN = PV_DONE + 1;
    static_assert(DRAIN + 1 == Cfg::kNumBars, "barrier count");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t sQ = s_base;
    const uint32_t sK0 = s_base + Cfg::kTileBytes;
    const uint32_t sV0 = sK0 + NS * Cfg::kTileBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kTileRegion);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const uint32_t bar0 = smem_u32(bars);
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int bh = blockIdx.x;                          // b * Hq + h
    const int qt = args.n_q_tiles - 1 - blockIdx.y;     // longest causal tiles first
    const int h = bh % args.Hq;
    const int b = bh / args.Hq;
    const int kv_plane = b * args.Hkv + h / args.group;  // grouped-query head mapping
    const int q0 = qt * kBM;
    const int diag = args.Lk - args.Lq;                  // causal: key j visible iff j <= i + diag

    int n_kv = (args.Lk + kBN - 1) / kBN;
    if (CAUSAL) {
        const int last_row = min(q0 + kBM - 1, args.Lq - 1);
        const int max_key = last_row + diag;
        n_kv = max_key < 0 ? 0 : min(n_kv, max_key / kBN + 1);
    }

    if (threadIdx.x == 0) {
        mbar_init(bar(Q_FULL), 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar(K_FULL + s), 1);
            mbar_init(bar(V_FULL + s), 1);
            mbar_init(bar(KV_EMPTY + s), 1);
        }
        for (int s = 0; s < kSBufs; ++s) {
            mbar_init(bar(S_FULL + s), 1);
            mbar_init(bar(P_FULL + s), kBM);
            mbar_init(bar(PV_BUF + s), 1);
        }
        mbar_init(bar(PV_DONE), 1);
        mbar_init(bar(DRAIN), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 5) {
        tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
        tmem_relinquish();
    }
    if (warp == 4 && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    int loads_issued = 0;  // producer: K/V tiles issued (for the abort drain)
    bool mma_started = false;

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && n_kv > 0) {
            mbar_arrive_expect_tx(bar(Q_FULL), Cfg::kTileBytes);
#pragma unroll
            for (int c = 0; c < Cfg::kChunks; ++c)
                tma_load_3d(sQ + c * Cfg::kChunkBytes, &tm_q, bar(Q_FULL), c * 64, q0, bh);
            for (int j = 0; j < n_kv; ++j) {
                const int s = j % NS;
                if (j >= NS && !wait_phase(bar(KV_EMPTY + s), ((j / NS) - 1) & 1, abort_flag))
                    break;
                mbar_arrive_expect_tx(bar(K_FULL + s), Cfg::kTileBytes);
#pragma unroll
                for (int c = 0; c < Cfg::kChunks; ++c)
                    tma_load_3d(sK0 + s * Cfg::kTileBytes + c * Cfg::kChunkBytes, &tm_k,
                                bar(K_FULL + s), c * 64, j * kBN, kv_plane);
                mbar_arrive_expect_tx(bar(V_FULL + s), Cfg::kTileBytes);
#pragma unroll
                for (int c = 0; c < Cfg::kChunks; ++c)
                    tma_load_3d(sV0 + s * Cfg::kTileBytes + c * Cfg::kChunkBytes, &tm_v,
                                bar(V_FULL + s), c * 64, j * kBN, kv_plane);
                loads_issued = j + 1;
            }
        }
    } else if (warp == 5) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0 && n_kv > 0) {
            constexpr uint32_t kIdescQK = idesc_f16(BF16, kBM, kBN, false, false);
            constexpr uint32_t kIdescPV = idesc_f16(BF16, kBM, D, false, true);
            mma_started = true;
            if (wait_phase(bar(Q_FULL), 0, abort_flag)) {
                tc_fence_after();
                for (int j = 0; j <= n_kv; ++j) {
                    if (j < n_kv) {
                        const int s = j % NS, sb = j % kSBufs;
                        if (!wait_phase(bar(K_FULL + s), (j / NS) & 1, abort_flag)) break;
                        // The S buffer is free once the P·V that read it has completed.
                        if (j >= kSBufs &&
                            !wait_phase(bar(PV_BUF + sb), ((j / kSBufs) - 1) & 1, abort_flag))
                            break;
                        tc_fence_after();
                        const uint32_t sK = sK0 + s * Cfg::kTileBytes;
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            // K-major operands: 16 elements (32 bytes) per step inside a
                            // 128-byte swizzle row, then the next 64-column chunk.
                            const uint32_t koff = (kk >> 2) * Cfg::kChunkBytes + (kk & 3) * 32;
                            mma_ss(tmem + sb * kBN, sdesc_sw128(sQ + koff, 16, 1024),
                                   sdesc_sw128(sK + koff, 16, 1024), kIdescQK, kk > 0 ? 1u : 0u);
                        }
                        mma_commit(bar(S_FULL + sb));
                    }
                    if (j >= 1) {
                        const int i = j - 1, s = i % NS, sb = i % kSBufs;
                        if (!wait_phase(bar(P_FULL + sb), (i / kSBufs) & 1, abort_flag)) break;
                        if (!wait_phase(bar(V_FULL + s), (i / NS) & 1, abort_flag)) break;
                        tc_fence_after();
                        const uint32_t sV = sV0 + s * Cfg::kTileBytes;
#pragma unroll
                        for (int ks = 0; ks < kBN / 16; ++ks) {
                            // V is MN-major: 16 keys = two 8-row swizzle atoms (2048 bytes);
                            // the 64-column chunks of D sit 16 KiB apart (leading offset).
                            mma_ts(tmem + Cfg::kOCol, tmem + sb * kBN + ks * 8,
                                   sdesc_sw128(sV + ks * 2048, Cfg::kChunkBytes, 1024), kIdescPV,
                                   (i > 0 || ks > 0) ? 1u : 0u);
                        }
                        mma_commit(bar(PV_DONE));
                        mma_commit(bar(PV_BUF + sb));
                        mma_commit(bar(KV_EMPTY + s));
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------------------- softmax
        const int t = threadIdx.x;  // 0..127: query row within the tile == TMEM lane
        const int row = q0 + t;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const float c = args.scale_log2;
        const int row_limit = CAUSAL ? min(args.Lk, row + diag + 1) : args.Lk;
        float m_ref = -INFINITY;  // reference max, log2 units
        float l = 0.f;            // running sum of 2^(s*c - m_ref)
        bool ok = true;

        for (int j = 0; j < n_kv; ++j) {
            const int sb = j % kSBufs;
            const bool w = wait_phase(bar(S_FULL + sb), (j / kSBufs) & 1, abort_flag);
            if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[kBN];
            tmem_ld32(lane_base + sb * kBN + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
            tmem_ld32(lane_base + sb * kBN + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
            tmem_ld32(lane_base + sb * kBN + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
            tmem_ld32(lane_base + sb * kBN + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
            tmem_wait_ld();
            float s[kBN];
#pragma unroll
            for (int x = 0; x < kBN; ++x) s[x] = __uint_as_float(sr[x]);

            const int kbase = j * kBN;
            const bool need_mask =
                (kbase + kBN > args.Lk) || (CAUSAL && kbase + kBN - 1 > q0 + diag);
            if (need_mask) {
                const int lim = row_limit - kbase;
#pragma unroll
                for (int x = 0; x < kBN; ++x) s[x] = (x < lim) ? s[x] : -INFINITY;
            }
            float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
            for (int x = 4; x < kBN; x += 4) {
                mx0 = fmaxf(mx0, s[x]);
                mx1 = fmaxf(mx1, s[x + 1]);
                mx2 = fmaxf(mx2, s[x + 2]);
                mx3 = fmaxf(mx3, s[x + 3]);
            }
            const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * c;
            const float m_new = (m_tile > m_ref + kRescaleThreshold) ? m_tile : m_ref;
            const float alpha = (m_new == m_ref) ? 1.f : ex2_approx(m_ref - m_new);
            const float neg_m = (m_new == -INFINITY) ? 0.f : -m_new;

            uint32_t pk[kBN / 2];
            float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
            for (int x = 0; x < kBN; x += 2) {
                const float p0 = ex2_approx(fmaf(s[x], c, neg_m));
                const float p1 = ex2_approx(fmaf(s[x + 1], c, neg_m));
                rs0 += p0;
                rs1 += p1;
                pk[x / 2] = pack2<BF16>(p0, p1);
            }

            // Correct O when the reference max moved; the previous P·V must be done.
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                const bool w2 = wait_phase(bar(PV_DONE), (j - 1) & 1, abort_flag);
                if (!__all_sync(0xffffffffu, w2)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int d0 = 0; d0 < D; d0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + Cfg::kOCol + d0, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
                    tmem_st32(lane_base + Cfg::kOCol + d0, o);
                }
            }
            // P overwrites the first 64 columns of this S buffer (16-bit pairs).
            tmem_st32(lane_base + sb * kBN + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
            tmem_st32(lane_base + sb * kBN + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(P_FULL + sb));
            l = l * alpha + (rs0 + rs1);
            m_ref = m_new;
        }

        if (ok && n_kv > 0) {
            const bool w = wait_phase(bar(PV_DONE), (n_kv - 1) & 1, abort_flag);
            ok = __all_sync(0xffffffffu, w);
            if (ok) tc_fence_after();
        }
        if (ok) {
            // ------------------------------------------------------------ epilogue
            const bool has = l > 0.f;
            const float inv_l = has ? 1.f / l : 0.f;
            using T = uint16_t;
            T* out_row = reinterpret_cast<T*>(args.out) +
                         (static_cast<size_t>(bh) * args.Lq + row) * D;
#pragma unroll
            for (int d0 = 0; d0 < D; d0 += 32) {
                uint32_t o[32];
                if (n_kv > 0) {
                    tmem_ld32(lane_base + Cfg::kOCol + d0, o);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int x = 0; x < 32; ++x) o[x] = 0u;
                }
                uint32_t pkd[16];
#pragma unroll
                for (int x = 0; x < 16; ++x)
                    pkd[x] = pack2<BF16>(__uint_as_float(o[2 * x]) * inv_l,
                                         __uint_as_float(o[2 * x + 1]) * inv_l);
                if (row < args.Lq) {
                    uint4* dst = reinterpret_cast<uint4*>(out_row + d0);
#pragma unroll
                    for (int x = 0; x < 4; ++x)
                        dst[x] = make_uint4(pkd[4 * x], pkd[4 * x + 1], pkd[4 * x + 2], pkd[4 * x + 3]);
                }
            }
            if (args.lse != nullptr && row < args.Lq)
                args.lse[static_cast<size_t>(bh) * args.Lq + row] =
                    has ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
        }
    }

    // ----------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // Nothing may still be writing into this CTA's shared or tensor memory when
        // it exits: wait for the loads already issued and for every MMA issued.
        if (warp == 4 && lane == 0 && n_kv > 0) {
            drain_phase(bar(Q_FULL), 0);
            for (int j = max(0, loads_issued - NS); j < loads_issued; ++j) {
                drain_phase(bar(K_FULL + j % NS), (j / NS) & 1);
                drain_phase(bar(V_FULL + j % NS), (j / NS) & 1);
            }
        }
        if (warp == 5 && lane == 0 && mma_started) {
            mma_commit(bar(DRAIN));
            drain_phase(bar(DRAIN), 0);
        }
        __syncthreads();
    }
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::kTmemCols);
    }
}

// Writes O = 0 and lse = -inf (a problem with no keys at all).
template <bool BF16>
__global__ void fill_empty_kernel(uint16_t* out, float* lse, size_t n_out, size_t n_rows) {
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n_out; i += stride)
        out[i] = 0;  // +0.0 in both f16 and bf16
    if (lse != nullptr)
        for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n_rows;
             i += stride)
            lse[i] = -INFINITY;
}

}  // namespace attn
