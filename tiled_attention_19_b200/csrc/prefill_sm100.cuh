// prefill_sm100.cuh -- exact attention forward on B200 tensor cores (tcgen05 + TMEM + TMA).
//
// Computes O = softmax(Q K^T * scale [+ causal mask]) V per head, tile by tile, with
// an online softmax, writing only O and the per-row log-sum-exp ("Self-attention,
// CUDA kernels and FlashAttention", section 3: tiling, the online-softmax trick that
// tracks the running maximum and normaliser and rescales partial outputs, and the
// saved normalisation statistics). The score matrix lives only in tensor memory.
//
// One CTA owns two 128-row query tiles (Q0, Q1: 256 consecutive rows) of one
// (batch, head); both walk the same 128-key tiles, so each K/V tile is loaded once
// for 256 rows. Roles (384 threads, three warpgroups):
//   warps 0-3  softmax of Q0, warps 4-7 softmax of Q1: thread t of a warpgroup owns
//              query row t of its tile, which is TMEM lane t. Per key tile it loads its
//              row of S from TMEM, masks, updates the running max (log2 domain, scale
//              folded into the exponent), writes P = 2^(S*c - m) in f16/bf16 back over
//              the same TMEM columns, corrects O when the reference max moved, and at
//              the end writes O / l and the lse.
//   warp 8     producer: one lane issues TMA loads of Q0, Q1 once and of K_j, V_j into
//              two rings of shared-memory stages (128-byte swizzle).
//   warp 9     MMA issuer: one lane issues, per key tile j,
//                 PV0_{j-1}: O0 += P0_{j-1} V_{j-1}   (P from TMEM, V from smem)
//                 S0_j     : S0  = Q0 K_j^T           (both from smem)
//                 PV1_{j-1}, S1_j likewise,
//              so each warpgroup's softmax of tile j overlaps the tensor core working
//              for the other warpgroup. tcgen05 MMAs of one thread execute in issue
//              order, so S0_j may overwrite the columns P0_{j-1} occupied once PV0_{j-1}
//              was issued, and the commit that signals S0_j also covers PV0_{j-1}: the
//              softmax may rescale O0 as soon as S0_j is ready.
//   warps 10-11 idle.
// Registers: the third warpgroup releases registers (setmaxnreg.dec to 72) and the two
// softmax warpgroups take them (setmaxnreg.inc to 216): 2x128x216 + 128x72 = 64,512, all
// of the 384 x 168 the CTA is launched with.
// TMEM (512 columns): S0/P0 at 0, S1/P1 at 128, O0 at 256, O1 at 384.
//
// Band masks (the "Flash Attention" skill page, Scenario 2: causal=True for
// autoregressive models, step 2, and sliding-window attention window_size=(left,
// right), step 3): with i' = i + (Lk - Lq), key j is visible to query i iff
// i' - left <= j <= i' + right (a negative bound is unbounded; causal is right = 0).
// Each query tile walks only the key tiles that hold a visible key of one of its rows;
// the element mask is applied only on tiles that cross a band edge or the ragged end
// of the keys. Without a band (kMaskNone) only the ragged end is masked; causal and
// general windows are separate instantiations (kMaskCausal, kMaskWindow).
//
// Lazy rescaling: the reference max m of a row moves only when a tile's maximum
// exceeds it by more than 8 (log2 units). Until then p = 2^(s*c - m) <= 2^8, which
// f16/bf16 and fp32 hold without loss, and O and l keep a common reference, so the
// final O / l is unchanged; O in TMEM is rescaled only when m moves.
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace attn {

constexpr int kBM = 128;          // query rows per tile (two tiles per CTA)
constexpr int kBN = 128;          // keys per tile
constexpr int kPrefillThreads = 384;
// Register split between warpgroups (setmaxnreg). It only works if the registers the
// CTA was launched with cover it; the launcher checks 384 x (registers per thread at
// launch) >= kRegBudget before the first launch and refuses otherwise, because a
// setmaxnreg.inc that cannot be satisfied waits forever.
// ptxas allocates each region for the count its setmaxnreg sets, so these are also the
// registers the softmax and the other roles are compiled for (216 leaves the softmax
// without spills; the producer and MMA roles fit in 72).
constexpr int kSoftmaxRegs = 216;
constexpr int kOtherRegs = 72;
constexpr int kRegBudget = 2 * 128 * kSoftmaxRegs + 128 * kOtherRegs;  // 64,512
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D, bool FP8 = false>
struct PrefillCfg {
    static constexpr int kElem = FP8 ? 1 : 2;           // bytes per Q/K/V element
    static constexpr int kRowBytes = D * kElem;
    static constexpr int kChunks = kRowBytes / 128;    // 128-byte column chunks
    static constexpr int kChunkElems = 128 / kElem;    // elements per chunk row
    static constexpr int kChunkBytes = kBM * 128;      // one chunk of a 128-row tile
    static constexpr int kTileBytes = kBM * kRowBytes; // a whole Q, K or V tile
    static constexpr int kKSteps = kRowBytes / 32;     // S = Q K^T: 32 bytes of K per MMA
    static constexpr int kPVKeys = FP8 ? 32 : 16;      // keys per P.V MMA
    static constexpr int kPCols = kBN * kElem / 4;     // TMEM columns P takes
    static constexpr int kKStages = (kTileBytes == 16384) ? 5 : 3;
    static constexpr int kVStages = (kTileBytes == 16384) ? 5 : 2;
    // At D = 64 the O accumulators take 64 columns each, which leaves room for a third
    // S buffer (kSCol2). The split-KV form rotates S through all three (kTriS) while a
    // warpgroup has at most kTriMaxTiles key tiles: S issued ahead shortens the start of
    // short loops; in long ones the two-buffer order measured faster.
    static constexpr int kSCol0 = 0, kSCol1 = 128, kSCol2 = 256;
    static constexpr int kOCol0 = D == 64 ? 384 : 256, kOCol1 = D == 64 ? 448 : 384;
    static constexpr bool kTriS = D == 64;
    static constexpr int kTriMaxTiles = 4;
    static constexpr int kTmemCols = 512;
    // P is handed to the MMA warp in two parts: the first kPSplit keys, then the rest
    // (kPSplit is a multiple of kPVKeys, so each part is whole P.V instructions).
    static constexpr int kPSplit = 96;  // the softmax's stores below are laid out for 96
    static constexpr bool kSplitP = D == 64;  // the MMA warp takes the first part early
    static_assert(kPSplit == 96 && kBN == 128, "P hand-off layout");
    // barriers: Q_FULL, K_FULL/K_EMPTY per K stage, V_FULL/V_EMPTY per V stage,
    // S_FULL[3], P_FULL[2] (first part of P), P_REST[2] (the rest), O_READY[2],
    // O_DONE[2], DRAIN
    static constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 12;
    static constexpr int kTileRegion = kTileBytes * (2 + kKStages + kVStages);
    static constexpr int kSmemBytes = 1024 /*alignment slack*/ + kTileRegion + kNumBars * 8 + 16;
    static_assert(kSmemBytes <= 232448, "shared-memory budget");
};

struct PrefillArgs {
    void* out;
    long long out_sb, out_sh, out_sl;  // element strides of out over (batch, head, row)
    float* lse;
    int Hq, Hkv, group, Lq, Lk;
    int n_q_blocks;    // CTAs along the query axis: ceil(Lq / 256), or ceil(Lq / 128) with split_kv
    int split_kv;      // one query tile per CTA whose key tiles are split between the two
                       // softmax warpgroups (the first half and the rest), merged at the end
    int win_left;      // band: keys >= i' - win_left visible (-1: unbounded)
    int win_right;     // band: keys <= i' + win_right visible (-1: unbounded; causal: 0)
    float scale_log2;  // scale * log2(e) (8-bit inputs: times the q and k descale factors)
    float o_scale;     // 8-bit inputs: the v descale factor, applied to O (else unused)
    // Paged keys (prefill over a paged cache): K and V of sequence b are rows
    // (block_table[b][t / 16] * Hkv + h_kv) * 16 + t % 16 of the caches, seq_lens[b] keys;
    // its chunk of queries is the first q_lens[b] rows (all Lq if q_lens is NULL).
    const int32_t* block_table;
    const int32_t* seq_lens;
    const int32_t* q_lens;
    int max_blocks, num_blocks;
};

// First and one-past-last visible key of query row i (empty if hi <= lo).
template <int MASK>
__device__ __forceinline__ void row_keys(int i, const PrefillArgs& a, int& lo, int& hi) {
    lo = 0;
    hi = a.Lk;
    if (MASK == kMaskCausal) {
        hi = min(a.Lk, i + (a.Lk - a.Lq) + 1);
    } else if (MASK == kMaskWindow) {
        const int ii = i + (a.Lk - a.Lq);
        if (a.win_left >= 0) lo = max(0, ii - a.win_left);
        if (a.win_right >= 0) hi = min(a.Lk, ii + a.win_right + 1);
    }
}

// Key tiles [t0, t1) holding a visible key of some row in [row0, row0 + 128). Without
// a window a tile past Lq takes the tiles of the last real row (t0 = 0 and t1 never
// below the previous tile's), which the two-tile issue loop relies on; with a window it
// is empty.
template <int MASK>
__device__ __forceinline__ void key_tiles_for(int row0, const PrefillArgs& a, int& t0, int& t1) {
    const int r1 = min(row0 + kBM - 1, a.Lq - 1);
    if (MASK != kMaskWindow) {
        int lo, hi;
        row_keys<MASK>(r1, a, lo, hi);
        t0 = 0;
        t1 = hi <= 0 ? 0 : (hi - 1) / kBN + 1;
        return;
    }
    if (r1 < row0) {  // no real rows (past Lq)
        t0 = t1 = 0;
        return;
    }
    int lo0, hi0, lo1, hi1;
    row_keys<MASK>(row0, a, lo0, hi0);  // band edges grow with the row
    row_keys<MASK>(r1, a, lo1, hi1);
    const int first = lo0, last = hi1 - 1;
    if (last < first || last < 0 || first >= a.Lk) {
        t0 = t1 = 0;
        return;
    }
    t0 = first / kBN;
    t1 = last / kBN + 1;
}

template <int D, bool BF16, int MASK, bool PAGED, bool FP8 = false>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    prefill_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const PrefillArgs args) {
    static_assert(!FP8 || (BF16 && !PAGED), "8-bit inputs: bf16 output, dense keys");
    using Cfg = PrefillCfg<D, FP8>;
    constexpr int NK = Cfg::kKStages;
    constexpr int NV = Cfg::kVStages;
    constexpr int Q_FULL = 0;
    constexpr int K_FULL = 1;
    constexpr int K_EMPTY = K_FULL + NK;
    constexpr int V_FULL = K_EMPTY + NK;
    constexpr int V_EMPTY = V_FULL + NV;
    constexpr int S_FULL = V_EMPTY + NV;  // [3] per S buffer (the third only with kTriS)
    constexpr int P_FULL = S_FULL + 3;    // [2] the first kPSplit keys of P are in TMEM
    constexpr int P_REST = P_FULL + 2;    // [2] the rest of P is in TMEM
    constexpr int O_READY = P_REST + 2;   // [2] a P.V into O_t completed (kTriS)
    constexpr int O_DONE = O_READY + 2;   // [2]
    constexpr int DRAIN = O_DONE + 2;
    static_assert(DRAIN + 1 == Cfg::kNumBars, "barrier count");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t sQ0 = s_base;
    const uint32_t sQ1 = s_base + Cfg::kTileBytes;
    const uint32_t sK0 = s_base + 2 * Cfg::kTileBytes;
    const uint32_t sV0 = sK0 + NK * Cfg::kTileBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kTileRegion);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const uint32_t bar0 = smem_u32(bars);
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Barrier initialisation (by the producer lane, which then issues the first loads)
    // and the TMEM allocation (warp 9). With kEarlySetup they run before the wait for the
    // previous kernel of the stream (programmatic stream serialisation), while that
    // kernel finishes; otherwise after the wait, where at D = 128 the registers come out
    // without spills (ptxas spilled with the early form there, and the e4m3 kernel ran
    // 6 % slower).
    constexpr bool kEarlySetup = D == 64;
    auto init_barriers = [&] {
        mbar_init(bar(Q_FULL), 1);
        for (int s = 0; s < NK; ++s) {
            mbar_init(bar(K_FULL + s), 1);
            mbar_init(bar(K_EMPTY + s), 1);
        }
        for (int s = 0; s < NV; ++s) {
            mbar_init(bar(V_FULL + s), 1);
            mbar_init(bar(V_EMPTY + s), 1);
        }
        for (int t = 0; t < 3; ++t) mbar_init(bar(S_FULL + t), 1);
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(P_FULL + t), kBM);
            mbar_init(bar(P_REST + t), kBM);
            mbar_init(bar(O_READY + t), 1);
            mbar_init(bar(O_DONE + t), 1);
        }
        mbar_init(bar(DRAIN), 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    };
    auto alloc_tmem = [&] {
        tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
        tmem_relinquish();
    };
    if constexpr (kEarlySetup) {
        if (warp == 8 && lane == 0) init_barriers();
        if (warp == 9) alloc_tmem();
    }
    // Wait for the previous kernel of the stream (its writes visible) before any global
    // memory is touched.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int bh = blockIdx.x;                           // b * Hq + h
    const int h = bh % args.Hq;
    const int b = bh / args.Hq;
    const int hkv = h / args.group;  // grouped-query head mapping
    // First rows of the CTA's two query tiles, the CTAs with the most key tiles first:
    // two consecutive tiles, or with split_kv one tile that both softmax warpgroups
    // work on (each over its share of the key tiles).
    const bool split = !PAGED && args.split_kv != 0;
    const int qb = args.n_q_blocks - 1 - blockIdx.y;
    const int qrow0 = split ? qb * kBM : qb * 2 * kBM;
    const int qrow1 = split ? qrow0 : qrow0 + kBM;
    // The lengths the masks see: the problem's, or with paged keys the sequence's own
    // (seq_lens[b] keys, q_lens[b] queries at its last positions). Out-of-range values
    // are clamped and reported.
    PrefillArgs a = args;
    if constexpr (PAGED) {
        int len = args.seq_lens[b];
        const int cap = args.max_blocks * kPageSize;
        int ql = args.q_lens != nullptr ? args.q_lens[b] : args.Lq;
        if (len < 0 || len > cap || ql < 0 || ql > args.Lq) {
            if (threadIdx.x == 0) report_status(ATTN_ERR_BAD_INDEX);
            len = min(max(len, 0), cap);
            ql = min(max(ql, 0), args.Lq);
        }
        a.Lk = len;
        a.Lq = ql;
    }
    // key-tile ranges of the two query tiles and of the CTA (their union, no gaps:
    // the band edges are monotone in the row)
    int a0 = 0, b0, a1 = 0, b1;
    if constexpr (MASK == kMaskWindow) {
        key_tiles_for<MASK>(qrow0, a, a0, b0);
        key_tiles_for<MASK>(qrow1, a, a1, b1);
    } else {  // every query tile starts at key tile 0
        int unused;
        key_tiles_for<MASK>(qrow0, a, unused, b0);
        key_tiles_for<MASK>(qrow1, a, unused, b1);
    }
    if (PAGED && qrow0 >= a.Lq) a0 = b0 = a1 = b1 = 0;  // every row past the sequence's chunk
    if (split) {  // warpgroup 0 takes the first half of the tile's key tiles, 1 the rest
        const int t0 = (MASK == kMaskWindow) ? a0 : 0, t1 = b0;
        a0 = t0;
        b0 = t1 > t0 ? t0 + (t1 - t0 + 1) / 2 : t0;
        a1 = b0;
        b1 = t1 > b0 ? t1 : b0;
    }
    const int jlo = (MASK != kMaskWindow) ? 0 : ((b0 > a0) ? a0 : a1);
    const int jhi = max(b0, b1);
    // key tiles this CTA loads (with split_kv each is used by one warpgroup)
    const int n_all = split ? (b0 - a0) + (b1 - a1)
                            : ((b1 > a1 || b0 > a0) ? jhi - jlo : 0);
    // Both query tiles walking key tiles 0 .. jhi-1 together (no window, no split): one
    // full barrier per key tile j counts K_j and V_{j-1}, and one empty barrier per key
    // tile, committed after S1_j, releases both K_j's and V_{j-1}'s ring slots (the K
    // ring's barriers serve as both; the V ring's are unused). The MMA warp then waits and
    // commits once per key tile for the ring instead of twice.
    const bool paired = MASK != kMaskWindow && !split;
    static_assert(NK >= NV, "the empty barrier of a key tile is looked up in the K ring");
    // split_kv ring order: the two warpgroups' tiles alternate, (a0, a1, a0+1, a1+1, ...),
    // then the rest of warpgroup 0's (it has at least as many)
    const int ns0 = b0 - a0, ns1 = b1 - a1;
    auto split_tile = [&](int n) -> int {
        return n < 2 * ns1 ? ((n & 1) ? a1 : a0) + (n >> 1) : a0 + (n - ns1);
    };

    // The producer lane issues the query tile(s) at once, so their load overlaps the
    // start-up barrier, on which it only arrives (the other warps wait there for the
    // barriers and the TMEM address).
    if (warp == 8 && lane == 0) {
        if constexpr (!kEarlySetup) init_barriers();
        if (n_all > 0) {
            mbar_arrive_expect_tx(bar(Q_FULL), (split ? 1 : 2) * Cfg::kTileBytes);
#pragma unroll
            for (int c = 0; c < Cfg::kChunks; ++c) {
                tma_load_4d(sQ0 + c * Cfg::kChunkBytes, &tm_q, bar(Q_FULL), c * Cfg::kChunkElems, qrow0,
                            h, b);
                if (!split)
                    tma_load_4d(sQ1 + c * Cfg::kChunkBytes, &tm_q, bar(Q_FULL), c * Cfg::kChunkElems,
                                qrow1, h, b);
            }
        }
    }
    if constexpr (!kEarlySetup) {
        if (warp == 9) alloc_tmem();
    }
    if (warp == 8) {
        __syncwarp();
        named_barrier_arrive(2, kPrefillThreads);
    } else {
        tc_fence_before();
        named_barrier_sync(2, kPrefillThreads);
        tc_fence_after();
    }
    const uint32_t tmem = *tmem_slot;  // (not read by the producer warp, which did not wait)

    int k_issued = 0, v_issued = 0;  // producer: tiles issued per ring (for the abort drain)
    bool mma_started = false;

    if (warp >= 10) {
        regs_decrease<kOtherRegs>();  // idle warps of the third warpgroup
    } else if (warp == 8) {
        // ------------------------------------------------------------ producer
        regs_decrease<kOtherRegs>();
        if (lane == 0 && n_all > 0) {
            // (the query tiles were issued before the start-up barrier)
            constexpr int kBlocks = kBN / kPageSize;  // cache blocks per key tile
            // Paged keys: a tile's rows come from kBlocks cache blocks; a block past the
            // sequence loads its first block instead (finite rows, masked), and an entry
            // outside the pool is reported and replaced by block 0.
            auto block_rows = [&](int j, int (&rows)[PAGED ? kBlocks : 1]) {
                if constexpr (PAGED) {
                    const int32_t* tbl = args.block_table + static_cast<size_t>(b) * args.max_blocks;
                    const int nblk = (a.Lk + kPageSize - 1) / kPageSize;
#pragma unroll
                    for (int k = 0; k < kBlocks; ++k) {
                        const int bi = j * kBlocks + k;
                        int e = __ldg(tbl + (bi < nblk ? bi : 0));
                        if (e < 0 || e >= args.num_blocks) {
                            report_status(ATTN_ERR_BAD_INDEX);
                            e = 0;
                        }
                        rows[k] = (e * args.Hkv + hkv) * kPageSize;
                    }
                }
            };
            // K or V of key tile j into the 128-byte-swizzled tile at dst, counted on fb
            auto load_tile = [&](const CUtensorMap* tm, uint32_t dst, uint32_t fb, int j,
                                 const int (&rows)[PAGED ? kBlocks : 1]) {
#pragma unroll
                for (int c = 0; c < Cfg::kChunks; ++c) {
                    if constexpr (PAGED) {
#pragma unroll
                        for (int k = 0; k < kBlocks; ++k)
                            tma_load_2d(dst + c * Cfg::kChunkBytes + k * kPageSize * 128, tm, fb,
                                        c * 64, rows[k]);
                    } else {
                        tma_load_4d(dst + c * Cfg::kChunkBytes, tm, fb, c * Cfg::kChunkElems, j * kBN,
                                    hkv, b);
                    }
                }
            };
            if (paired) {
                // iteration j: K_j (if j < n_all) and V_{j-1} (if j >= 1) on full barrier j
                int rows_k[PAGED ? kBlocks : 1], rows_v[PAGED ? kBlocks : 1];
                for (int j = 0; j <= n_all; ++j) {
                    const bool has_k = j < n_all, has_v = j >= 1;
                    const int sf = j % NK;
                    if (has_k) block_rows(j, rows_k);
                    // Full barrier j % NK was last armed for j-NK, and K_j takes the slot of
                    // K_{j-NK}: both are free once the empty barrier of j-NK completes (the
                    // MMA warp waited on that full barrier before committing it). V_{j-1}
                    // takes the slot of V_{j-1-NV}, freed by the empty barrier of j-NV, a
                    // later one when NV < NK.
                    if (j >= NK && !wait_phase(bar(K_EMPTY + sf), ((j / NK) - 1) & 1, abort_flag))
                        break;
                    if (NV < NK && has_v && j - 1 >= NV &&
                        !wait_phase(bar(K_EMPTY + (j - NV) % NK), ((j - NV) / NK) & 1, abort_flag))
                        break;
                    mbar_arrive_expect_tx(bar(K_FULL + sf), (has_k ? Cfg::kTileBytes : 0) +
                                                                 (has_v ? Cfg::kTileBytes : 0));
                    if (has_k) load_tile(&tm_k, sK0 + sf * Cfg::kTileBytes, bar(K_FULL + sf), j, rows_k);
                    if (has_v)
                        load_tile(&tm_v, sV0 + ((j - 1) % NV) * Cfg::kTileBytes, bar(K_FULL + sf), j - 1,
                                  rows_v);
                    k_issued = j + 1;  // full barriers armed (drained after an abort)
                    if constexpr (PAGED) {
#pragma unroll
                        for (int k = 0; k < kBlocks; ++k) rows_v[k] = rows_k[k];
                    }
                }
            } else
            for (int n = 0; n < n_all; ++n) {  // ring sequence n holds key tile j
                const int j = split ? split_tile(n) : jlo + n;
                const int sk = n % NK, sv = n % NV;
                int rows[PAGED ? kBlocks : 1];
                block_rows(j, rows);
                if (n >= NK && !wait_phase(bar(K_EMPTY + sk), ((n / NK) - 1) & 1, abort_flag)) break;
                mbar_arrive_expect_tx(bar(K_FULL + sk), Cfg::kTileBytes);
                load_tile(&tm_k, sK0 + sk * Cfg::kTileBytes, bar(K_FULL + sk), j, rows);
                k_issued = n + 1;
                if (n >= NV && !wait_phase(bar(V_EMPTY + sv), ((n / NV) - 1) & 1, abort_flag)) break;
                mbar_arrive_expect_tx(bar(V_FULL + sv), Cfg::kTileBytes);
                load_tile(&tm_v, sV0 + sv * Cfg::kTileBytes, bar(V_FULL + sv), j, rows);
                v_issued = n + 1;
            }
        }
    } else if (warp == 9) {
        // ---------------------------------------------------------- MMA issuer
        regs_decrease<kOtherRegs>();
        if (lane == 0 && n_all > 0) {
            // 8-bit inputs: format code 0 is E4M3 under kind::f8f6f4
            constexpr uint32_t kIdescQK = idesc_f16(BF16 && !FP8, kBM, kBN, false, false);
            constexpr uint32_t kIdescPV = idesc_f16(BF16 && !FP8, kBM, D, false, true);
            mma_started = true;
            // The issue of a tcgen05.mma blocks while the tensor core's queue is full, so
            // this thread's own work between products is tensor-core idle time: the shared
            // memory descriptors are built once and offset per product (the start address
            // is the descriptor's low field, in 16-byte units, and never carries out of it).
            const uint64_t dq0 = sdesc_sw128(sQ0, 16, 1024), dq1 = sdesc_sw128(sQ1, 16, 1024);
            const uint64_t dk0 = sdesc_sw128(sK0, 16, 1024);
            const uint64_t dv0 = sdesc_sw128(sV0, Cfg::kChunkBytes, 1024);
            constexpr uint32_t kTileUnits = Cfg::kTileBytes >> 4;
            // S_t = Q_t K^T into TMEM columns s_col, K from ring stage sk (K-major operands:
            // 16 elements = 32 bytes per step inside a 128-byte swizzle row, then the next
            // chunk).
            auto issue_s = [&](uint64_t dq, uint32_t s_col, int sk) {
                const uint64_t dk = dk0 + static_cast<uint32_t>(sk) * kTileUnits;
#pragma unroll
                for (int kk = 0; kk < Cfg::kKSteps; ++kk) {
                    constexpr uint32_t kChunkUnits = Cfg::kChunkBytes >> 4;
                    const uint32_t off = (kk >> 2) * kChunkUnits + (kk & 3) * 2;
                    if constexpr (FP8)
                        mma_ss_f8(tmem + s_col, dq + off, dk + off, kIdescQK, kk > 0 ? 1u : 0u);
                    else
                        mma_ss(tmem + s_col, dq + off, dk + off, kIdescQK, kk > 0 ? 1u : 0u);
                }
            };
            // O_t += P_t V: P from TMEM (kPVKeys keys = 8 columns per step), V from ring
            // stage sv, MN-major (kPVKeys keys = 8-row swizzle atoms of 128 bytes,
            // kPVKeys * 128 bytes per step; D chunks 16 KiB apart). Keys [k0, k1) of the tile
            // (whole instructions); `first` starts the accumulator (the query tile's first
            // key tile).
            auto issue_pv = [&](uint32_t p_col, uint32_t o_col, int sv, bool first, int k0, int k1) {
                const uint64_t dv = dv0 + static_cast<uint32_t>(sv) * kTileUnits;
#pragma unroll
                for (int ks = k0 / Cfg::kPVKeys; ks < k1 / Cfg::kPVKeys; ++ks) {
                    const uint32_t off = ks * Cfg::kPVKeys * 8;  // kPVKeys * 128 bytes
                    if constexpr (FP8)
                        mma_ts_f8(tmem + o_col, tmem + p_col + ks * 8, dv + off, kIdescPV,
                                  (!first || ks > 0) ? 1u : 0u);
                    else
                        mma_ts(tmem + o_col, tmem + p_col + ks * 8, dv + off, kIdescPV,
                               (!first || ks > 0) ? 1u : 0u);
                }
            };
            // O_t += P_t V. At D = 64 the first part of P goes as soon as it is in TMEM
            // and the rest after it (there the products wait for the softmax); at D = 128,
            // where P is always ready first, all of it after the one arrival that follows
            // both parts (fewer waits on the issuing thread). V is already known to be in
            // stage sv. Returns false if a wait gave up.
            auto pv_parts = [&](int t, uint32_t p_col, uint32_t o_col, int sv, bool first,
                                uint32_t parity) -> bool {
                if constexpr (Cfg::kSplitP) {
                    if (!wait_phase(bar(P_FULL + t), parity, abort_flag)) return false;
                    tc_fence_after();
                    issue_pv(p_col, o_col, sv, first, 0, Cfg::kPSplit);
                    if (!wait_phase(bar(P_REST + t), parity, abort_flag)) return false;
                    tc_fence_after();
                    issue_pv(p_col, o_col, sv, first, Cfg::kPSplit, kBN);
                } else {
                    if (!wait_phase(bar(P_FULL + t), parity, abort_flag)) return false;
                    tc_fence_after();
                    issue_pv(p_col, o_col, sv, first, 0, kBN);
                }
                return true;
            };
            bool ok = wait_phase(bar(Q_FULL), 0, abort_flag);
            // ring positions: K of the tile whose S is due, V of the tile whose P.V is due
            int sk = 0, sv = 0;
            uint32_t kpar = 0, vpar = 0;
            if (split && Cfg::kTriS && ns0 <= Cfg::kTriMaxTiles) {
                // Three S buffers (D = 64): ring sequence g (the alternating order below)
                // is S product g, in buffer g % 3, for warpgroup owner(g). S(g + 3) is
                // issued right after P.V(g), which frees its buffer (MMAs of one thread run
                // in issue order), so each warpgroup finds its next S computed while its
                // softmax ran. O_READY(t) signals each P.V into O_t: with S issued ahead,
                // S completing no longer implies the warpgroup's previous P.V did, so the
                // softmax waits for it before an O correction and before announcing P
                // (which keeps P_FULL(t) within one phase of this warp's wait on it).
                auto owner = [&](int g) { return g < 2 * ns1 ? (g & 1) : 0; };
                auto local = [&](int g) { return g < 2 * ns1 ? (g >> 1) : g - ns1; };
                auto issue_s_seq = [&](int g) -> bool {
                    const int skg = g % NK;
                    if (!wait_phase(bar(K_FULL + skg), static_cast<uint32_t>(g / NK) & 1u, abort_flag))
                        return false;
                    tc_fence_after();
                    const int buf = g % 3;
                    issue_s(dq0, static_cast<uint32_t>(buf) * 128u, skg);
                    mma_commit(bar(S_FULL + buf));
                    mma_commit(bar(K_EMPTY + skg));
                    return true;
                };
                for (int g = 0; ok && g < min(3, n_all); ++g) ok = issue_s_seq(g);
                for (int g = 0; ok && g < n_all; ++g) {
                    const int t = owner(g), m = local(g);
                    const int svg = g % NV;
                    ok = wait_phase(bar(V_FULL + svg), static_cast<uint32_t>(g / NV) & 1u, abort_flag) &&
                         pv_parts(t, static_cast<uint32_t>(g % 3) * 128u,
                                  t == 0 ? Cfg::kOCol0 : Cfg::kOCol1, svg, m == 0, m & 1);
                    if (!ok) break;
                    mma_commit(bar(O_READY + t));
                    if (m == (t == 0 ? ns0 : ns1) - 1) mma_commit(bar(O_DONE + t));
                    mma_commit(bar(V_EMPTY + svg));
                    if (g + 3 < n_all) ok = issue_s_seq(g + 3);
                }
            } else if (split) {
                // Both warpgroups work on Q0 (the only query tile), warpgroup t over its own
                // key tiles, which sit at ring sequence seq(t, m) in the alternating order.
                // Per step m: PV0 of its tile m-1, S0 of tile m, then the same for
                // warpgroup 1. Every ring slot is read by one product only.
                auto seq0 = [&](int m) { return m + min(m, ns1); };
                auto ring = [&](int q, int nst, int& st, uint32_t& par) {
                    st = q % nst;
                    par = static_cast<uint32_t>(q / nst) & 1u;
                };
                for (int m = 0; ok && m <= ns0; ++m) {
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        const int nt = t == 0 ? ns0 : ns1;
                        const uint32_t s_col = t == 0 ? Cfg::kSCol0 : Cfg::kSCol1;
                        const uint32_t o_col = t == 0 ? Cfg::kOCol0 : Cfg::kOCol1;
                        if (m >= 1 && m - 1 < nt) {  // P.V of this warpgroup's tile m-1
                            const int q = t == 0 ? seq0(m - 1) : 2 * (m - 1) + 1;
                            ring(q, NV, sv, vpar);
                            ok = wait_phase(bar(V_FULL + sv), vpar, abort_flag) &&
                                 pv_parts(t, s_col, o_col, sv, m == 1, (m - 1) & 1);
                            if (!ok) break;
                            if (m - 1 == nt - 1) mma_commit(bar(O_DONE + t));
                            mma_commit(bar(V_EMPTY + sv));
                        }
                        if (m < nt) {  // S of its tile m
                            const int q = t == 0 ? seq0(m) : 2 * m + 1;
                            ring(q, NK, sk, kpar);
                            ok = wait_phase(bar(K_FULL + sk), kpar, abort_flag);
                            if (!ok) break;
                            tc_fence_after();
                            issue_s(dq0, s_col, sk);
                            mma_commit(bar(S_FULL + t));
                            mma_commit(bar(K_EMPTY + sk));
                        }
                    }
                }
            } else
            if constexpr (MASK != kMaskWindow) {
                // Query tiles both start at key tile 0: n0 = b0 <= n1 = b1 = n_all. Full
                // barrier j (entry j % NK) covers K_j and V_{j-1}; the empty barrier of j,
                // committed after S1_j (so after PV1_{j-1} too), frees both their slots.
                const int n0 = b0, n1 = b1;
                for (int j = 0; ok && j <= n1; ++j) {
                    const int i = j - 1;  // the key tile whose P·V is due
                    ok = wait_phase(bar(K_FULL + sk), kpar, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    // PV0_{j-1}
                    if (i >= 0 && i < n0) {
                        ok = pv_parts(0, Cfg::kSCol0, Cfg::kOCol0, sv, i == 0, i & 1);
                        if (!ok) break;
                        if (i == n0 - 1) mma_commit(bar(O_DONE + 0));
                    }
                    if (j < n0) {
                        issue_s(dq0, Cfg::kSCol0, sk);
                        mma_commit(bar(S_FULL + 0));
                    }
                    // PV1_{j-1}
                    if (i >= 0) {
                        ok = pv_parts(1, Cfg::kSCol1, Cfg::kOCol1, sv, i == 0, i & 1);
                        if (!ok) break;
                        if (i == n1 - 1) mma_commit(bar(O_DONE + 1));
                        if (++sv == NV) sv = 0;
                    }
                    if (j < n1) {
                        issue_s(dq1, Cfg::kSCol1, sk);
                        mma_commit(bar(S_FULL + 1));
                        mma_commit(bar(K_EMPTY + sk));
                    }
                    if (++sk == NK) sk = 0, kpar ^= 1u;
                }
            } else {
                for (int n = 0; ok && n <= n_all; ++n) {
                    const int j = jlo + n;  // the key tile whose S is due
                    const int i = j - 1;    // the key tile whose P·V is due
                    if (n >= 1) {
                        ok = wait_phase(bar(V_FULL + sv), vpar, abort_flag);
                        if (!ok) break;
                    }
                    // PV0_{j-1}
                    if (n >= 1 && i >= a0 && i < b0) {
                        ok = pv_parts(0, Cfg::kSCol0, Cfg::kOCol0, sv, i == a0, (i - a0) & 1);
                        if (!ok) break;
                        if (i == b0 - 1) mma_commit(bar(O_DONE + 0));
                    }
                    if (n < n_all) {
                        ok = wait_phase(bar(K_FULL + sk), kpar, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
                        if (j >= a0 && j < b0) {
                            issue_s(dq0, Cfg::kSCol0, sk);
                            mma_commit(bar(S_FULL + 0));
                        }
                    }
                    // PV1_{j-1}
                    if (n >= 1) {
                        if (i >= a1 && i < b1) {
                            ok = pv_parts(1, Cfg::kSCol1, Cfg::kOCol1, sv, i == a1, (i - a1) & 1);
                            if (!ok) break;
                            if (i == b1 - 1) mma_commit(bar(O_DONE + 1));
                        }
                        mma_commit(bar(V_EMPTY + sv));  // V_{j-1} is no longer needed
                        if (++sv == NV) sv = 0, vpar ^= 1u;
                    }
                    if (n < n_all) {
                        if (j >= a1 && j < b1) {
                            issue_s(dq1, Cfg::kSCol1, sk);
                            mma_commit(bar(S_FULL + 1));
                        }
                        mma_commit(bar(K_EMPTY + sk));  // K_j is no longer needed
                        if (++sk == NK) sk = 0, kpar ^= 1u;
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------------------- softmax
        regs_increase<kSoftmaxRegs>();
        const int tile = warp >> 2;          // 0: Q0 (warps 0-3), 1: Q1 (warps 4-7)
        const int t = threadIdx.x & 127;     // query row within the tile == TMEM lane
        const int tile_row0 = tile == 0 ? qrow0 : qrow1;
        const int row = tile_row0 + t;
        const int ta = tile == 0 ? a0 : a1;  // this query tile's key tiles [ta, tb)
        const int tb = tile == 0 ? b0 : b1;
        const int n_kv = tb > ta ? tb - ta : 0;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const uint32_t s_col_t = tile == 0 ? Cfg::kSCol0 : Cfg::kSCol1;
        const uint32_t o_col = tile == 0 ? Cfg::kOCol0 : Cfg::kOCol1;
        const float c = args.scale_log2;
        int row_lo, row_hi;  // this row's visible keys [row_lo, row_hi)
        row_keys<MASK>(row, a, row_lo, row_hi);
        // band edges of the tile: the largest first key and the smallest end
        int edge_lo, edge_hi, unused;
        row_keys<MASK>(min(tile_row0 + kBM - 1, a.Lq - 1), a, edge_lo, unused);
        row_keys<MASK>(tile_row0, a, unused, edge_hi);
        float m_ref = -INFINITY;  // reference max, log2 units
        float l = 0.f;            // running sum of 2^(s*c - m_ref)
        bool ok = true;

        const bool tri = Cfg::kTriS && split && ns0 <= Cfg::kTriMaxTiles;  // three S buffers
        for (int jj = 0; jj < n_kv; ++jj) {
            const int j = ta + jj;  // key tile
            // S buffer and barrier phase of this tile: its own buffer, or with three
            // buffers those of S product g (the ring sequence of the split order)
            uint32_t s_col = s_col_t;
            int s_bar = S_FULL + tile;
            uint32_t s_par = jj & 1;
            if (tri) {
                const int g = tile == 0 ? jj + min(jj, ns1) : 2 * jj + 1;
                s_col = static_cast<uint32_t>(g % 3) * 128u;
                s_bar = S_FULL + g % 3;
                s_par = static_cast<uint32_t>(g / 3) & 1u;
            }
            const bool w = wait_phase(bar(s_bar), s_par, abort_flag);
            if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[kBN];
            tmem_ld32(lane_base + s_col + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
            tmem_ld32(lane_base + s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
            tmem_ld32(lane_base + s_col + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
            tmem_ld32(lane_base + s_col + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
            tmem_wait_ld();
            float s[kBN];
#pragma unroll
            for (int x = 0; x < kBN; ++x) s[x] = __uint_as_float(sr[x]);

            const int kbase = j * kBN;
            const bool need_mask = (kbase + kBN > a.Lk) ||
                                   (MASK != kMaskNone && (kbase < edge_lo || kbase + kBN > edge_hi));
            if (need_mask) {
                const int lo = row_lo - kbase, hi = row_hi - kbase;
                if (MASK == kMaskWindow) {
#pragma unroll
                    for (int x = 0; x < kBN; ++x) s[x] = (x >= lo && x < hi) ? s[x] : -INFINITY;
                } else {
#pragma unroll
                    for (int x = 0; x < kBN; ++x) s[x] = (x < hi) ? s[x] : -INFINITY;
                }
            }
            // row maximum: four chains of three-input maxima over 32 scores each
            float mx[4];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                float m = fmaxf(s[32 * q4], s[32 * q4 + 1]);
#pragma unroll
                for (int x = 2; x < 32; x += 2) m = max3(m, s[32 * q4 + x], s[32 * q4 + x + 1]);
                mx[q4] = m;
            }
            const float m_tile = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * c;
            const float m_new = (m_tile > m_ref + kRescaleThreshold) ? m_tile : m_ref;
            const float alpha = (m_new == m_ref) ? 1.f : ex2_approx(m_ref - m_new);
            const float neg_m = (m_new == -INFINITY) ? 0.f : -m_new;

            // Correct O when the reference max moved, before any part of this tile's P
            // is handed over. S_t(j) completing implies the P.V of tile j-1 (issued
            // before it) has completed too; with three S buffers S runs ahead, so the
            // P.V of tile j-1 is waited for here. (P.V of tile j-2 completed before this
            // S was issued, so the barrier is at most one phase behind.)
            if (jj > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                if (tri) {
                    if (!__all_sync(0xffffffffu,
                                    wait_phase(bar(O_READY + tile), (jj - 1) & 1, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
#pragma unroll
                for (int d0 = 0; d0 < D; d0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + o_col + d0, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
                    tmem_st32(lane_base + o_col + d0, o);
                }
            }

            // P = 2^(s*c - m), stored in two parts. At D = 64 the first kPSplit keys are
            // handed to the MMA warp (P_FULL) while the rest are still being exponentiated
            // (P_REST); at D = 128 the MMA warp only ever needs all of P, so one arrival
            // (P_FULL) after both parts spares it a wait.
            float rs0 = 0.f, rs1 = 0.f;
            const uint64_t c2 = f2pack(c, c), nm2 = f2pack(neg_m, neg_m);
            uint64_t rs2 = f2pack(0.f, 0.f);
            if constexpr (FP8) {
                // P in e4m3, four keys per column (the lowest key in the lowest byte);
                // p <= 2^8 < 448 under the lazy rescale, so it never saturates
                uint32_t pk[kBN / 4];
#pragma unroll
                for (int x = 0; x < kBN; x += 4) {
                    float t0, t1, t2, t3;
                    f2unpack(fma2(f2pack(s[x], s[x + 1]), c2, nm2), t0, t1);
                    f2unpack(fma2(f2pack(s[x + 2], s[x + 3]), c2, nm2), t2, t3);
                    // an eighth of the exponentials (two of every sixteen) on the FMA pipe: the
                    // e4m3 path has half the tensor time per exponential of the 16-bit one, so
                    // the MUFU sets its pace; an eighth moved over balanced the two pipes best
                    float p0, p1;
                    if ((x / 4) % 4 == 3) {
                        ex2_fma2(t0, t1, p0, p1);
                    } else {
                        p0 = ex2_approx(t0);
                        p1 = ex2_approx(t1);
                    }
                    const float p2 = ex2_approx(t2), p3 = ex2_approx(t3);
                    rs2 = add2(rs2, add2(f2pack(p0, p1), f2pack(p2, p3)));
                    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(p0, p1), __NV_SATFINITE, __NV_E4M3);
                    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(p2, p3), __NV_SATFINITE, __NV_E4M3);
                    pk[x / 4] = lo | (hi << 16);
                    if (x + 4 == Cfg::kPSplit) {
                        // columns [0, 24): keys [0, 96)
                        tmem_st16(lane_base + s_col, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
                        tmem_st8(lane_base + s_col + 16, *reinterpret_cast<uint32_t(*)[8]>(&pk[16]));
                        if constexpr (Cfg::kSplitP) {
                            tmem_wait_st();
                            tc_fence_before();
                            mbar_arrive(bar(P_FULL + tile));
                        }
                    }
                }
                tmem_st8(lane_base + s_col + 24, *reinterpret_cast<uint32_t(*)[8]>(&pk[24]));
            } else {
                // exponent arguments and row sums two at a time (f32x2 instructions)
                uint32_t pk[kBN / 2];
#pragma unroll
                for (int x = 0; x < kBN; x += 2) {
                    float t0, t1;
                    f2unpack(fma2(f2pack(s[x], s[x + 1]), c2, nm2), t0, t1);
                    const float p0 = ex2_approx(t0);
                    const float p1 = ex2_approx(t1);
                    rs2 = add2(rs2, f2pack(p0, p1));
                    pk[x / 2] = pack2<BF16>(p0, p1);
                    if (x + 2 == Cfg::kPSplit) {
                        // 16-bit pairs: columns [0, 48) hold keys [0, 96)
                        tmem_st32(lane_base + s_col, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
                        tmem_st16(lane_base + s_col + 32, *reinterpret_cast<uint32_t(*)[16]>(&pk[32]));
                        if constexpr (Cfg::kSplitP) {
                            tmem_wait_st();
                            // With three S buffers this tile's S can be ready before the
                            // MMA warp has taken the previous tile's P (it may still be
                            // waiting for that tile's V). P is announced only once the
                            // previous P.V has completed, so P_FULL never runs two phases
                            // ahead of the MMA warp's wait on it.
                            if (tri && jj > 0)
                                ok = __all_sync(0xffffffffu, wait_phase(bar(O_READY + tile),
                                                                        (jj - 1) & 1, abort_flag));
                            tc_fence_before();
                            if (ok) mbar_arrive(bar(P_FULL + tile));
                        }
                    }
                }
                tmem_st16(lane_base + s_col + 48, *reinterpret_cast<uint32_t(*)[16]>(&pk[48]));
            }
            if (!ok) break;  // a wait gave up (the abort flag is set)
            f2unpack(rs2, rs0, rs1);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar((Cfg::kSplitP ? P_REST : P_FULL) + tile));
            l = l * alpha + (rs0 + rs1);
            m_ref = m_new;
        }

        // This CTA's key tiles are done: once every CTA of the grid is this far, the next
        // kernel of the stream may launch and take the places of CTAs that exit.
        if (tile == 1 && t == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        if (ok && n_kv > 0) {
            const bool w = wait_phase(bar(O_DONE + tile), 0, abort_flag);
            ok = __all_sync(0xffffffffu, w);
            if (ok) tc_fence_after();
        }
        if (split) {
            // ------------------------------------------------ split_kv merge epilogue
            // Each warpgroup holds the row's partial (O_t, m_t, l_t) over its share of
            // the key tiles: O = (O_0 2^(m_0 - M) + O_1 2^(m_1 - M)) / L with M the larger
            // reference max and L = l_0 2^(m_0 - M) + l_1 2^(m_1 - M) (the same
            // log-sum-exp combine as split-KV decoding). The statistics meet in shared
            // memory (the unused second Q buffer); every softmax thread reaches the
            // barrier, also after a wait gave up, so it cannot hang.
            float* stat = reinterpret_cast<float*>(smem + Cfg::kTileBytes);  // [2][2][128]
            stat[tile * 256 + t] = m_ref;
            stat[tile * 256 + 128 + t] = l;
            tc_fence_before();
            named_barrier_sync(1, 256);
            tc_fence_after();
            if (!*abort_flag) {
                const float m0 = stat[t], l0 = stat[128 + t];
                const float m1 = stat[256 + t], l1 = stat[384 + t];
                const float M = fmaxf(m0, m1);
                const float f0 = m0 == -INFINITY ? 0.f : ex2_approx(m0 - M);
                const float f1 = m1 == -INFINITY ? 0.f : ex2_approx(m1 - M);
                const float L = l0 * f0 + l1 * f1;
                const bool has = L > 0.f;
                const float inv_l = has ? (FP8 ? args.o_scale : 1.f) / L : 0.f;
                const float g0 = f0 * inv_l, g1 = f1 * inv_l;
                uint16_t* out_row = reinterpret_cast<uint16_t*>(args.out) + b * args.out_sb +
                                    h * args.out_sh + static_cast<long long>(row) * args.out_sl;
                // warpgroup t writes the columns [t D / 2, (t + 1) D / 2)
#pragma unroll
                for (int d0 = tile * (D / 2); d0 < (tile + 1) * (D / 2); d0 += 32) {
                    uint32_t o0[32], o1[32];
                    tmem_ld32(lane_base + Cfg::kOCol0 + d0, o0);
                    if (ns1 > 0) tmem_ld32(lane_base + Cfg::kOCol1 + d0, o1);
                    tmem_wait_ld();
                    uint32_t pkd[16];
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        float v0 = __uint_as_float(o0[2 * x]) * g0;
                        float v1 = __uint_as_float(o0[2 * x + 1]) * g0;
                        if (ns1 > 0) {
                            v0 = fmaf(__uint_as_float(o1[2 * x]), g1, v0);
                            v1 = fmaf(__uint_as_float(o1[2 * x + 1]), g1, v1);
                        }
                        pkd[x] = has ? pack2<BF16>(v0, v1) : 0u;
                    }
                    if (row < args.Lq) {
                        uint4* dst = reinterpret_cast<uint4*>(out_row + d0);
#pragma unroll
                        for (int x = 0; x < 4; ++x)
                            dst[x] = make_uint4(pkd[4 * x], pkd[4 * x + 1], pkd[4 * x + 2], pkd[4 * x + 3]);
                    }
                }
                if (tile == 0 && args.lse != nullptr && row < args.Lq)
                    args.lse[static_cast<size_t>(bh) * args.Lq + row] =
                        has ? (M + log2f(L)) * kLn2 : -INFINITY;
            }
        } else if (ok) {
            // ------------------------------------------------------------ epilogue
            // rows past a paged sequence's chunk are written as rows with no key
            const bool real = !PAGED || row < a.Lq;
            const bool has = real && l > 0.f;
            const float inv_l = has ? (FP8 ? args.o_scale : 1.f) / l : 0.f;
            uint16_t* out_row = reinterpret_cast<uint16_t*>(args.out) + b * args.out_sb +
                                h * args.out_sh + static_cast<long long>(row) * args.out_sl;
#pragma unroll
            for (int d0 = 0; d0 < D; d0 += 32) {
                uint32_t o[32];
                if (n_kv > 0) {
                    tmem_ld32(lane_base + o_col + d0, o);
                    tmem_wait_ld();
                    if (!has) {
#pragma unroll
                        for (int x = 0; x < 32; ++x) o[x] = 0u;
                    }
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
        if (warp == 8 && lane == 0 && n_all > 0) {
            // the K ring's full barriers (in the paired scheme they also count V) and the
            // V ring's (the other schemes)
            drain_phase(bar(Q_FULL), 0);
            for (int j = max(0, k_issued - NK); j < k_issued; ++j)
                drain_phase(bar(K_FULL + j % NK), (j / NK) & 1);
            for (int j = max(0, v_issued - NV); j < v_issued; ++j)
                drain_phase(bar(V_FULL + j % NV), (j / NV) & 1);
        }
        if (warp == 9 && lane == 0 && mma_started) {
            mma_commit(bar(DRAIN));
            drain_phase(bar(DRAIN), 0);
        }
        __syncthreads();
    }
    if (warp == 9) {
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
