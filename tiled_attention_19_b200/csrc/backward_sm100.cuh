// backward_sm100.cuh -- attention backward pass on B200 tensor cores (tcgen05 + TMEM + TMA).
//
// The forward pass keeps only O and the per-row log-sum-exp; the backward pass
// recomputes the attention tiles from them ("Self-attention, CUDA kernels and
// FlashAttention", section 3: recomputation during backpropagation, only the small
// normalisation statistics are saved). With c = scale * log2(e), lse2 = lse * log2(e)
// and delta_i = dO_i . O_i, for every visible (query i, key j):
//   P_ij  = 2^(c * q_i.k_j - lse2_i)
//   dP_ij = dO_i . v_j
//   dS_ij = P_ij (dP_ij - delta_i)
//   dV_j += P_ij dO_i,  dK_j += scale dS_ij q_i,  dQ_i += scale dS_ij k_j.
// (delta_i = sum_j P_ij dP_ij = dO_i . sum_j P_ij v_j = dO_i . O_i.)
//
// Three launches, no atomics, so the result does not depend on scheduling:
//   bwd_prep_kernel  lse2 and delta per query row, into a caller workspace whose rows
//                    are padded to a multiple of 128 (padding: lse2 = +inf, delta = 0,
//                    so padded and fully masked rows give P = 0).
//   bwd_kernel<kDKDV> one CTA per 128-key tile of one (batch, K/V head): K and V stay in
//                    shared memory while 64-row sub-tiles of Q and dO (of every query head
//                    of the group) stream through a ring; dV and dK accumulate in TMEM.
//   bwd_kernel<kDQ>  one CTA per 128-row query tile of one (batch, head): Q and dO stay,
//                    64-key sub-tiles of K and V stream; dQ accumulates in TMEM.
// Both kinds run the same pipeline. Call the fixed pair (X, W) and a streamed pair
// (Y, Z): (K, V) and (Q, dO) for kDKDV, (Q, dO) and (K, V) for kDQ. Per sub-tile n:
//   S  = X Y^T, dP = W Z^T            (M = 128 fixed rows, N = 64, K = D; both operands
//                                      K-major from shared memory), into TMEM buffer n & 1
//   softmax warps: P and dS from S, dP and the row statistics, written back over the
//                 first half of their own S / dP columns in f16/bf16
//   kDKDV: dV += P Z, dK += dS Y;  kDQ: dQ += dS Y   (A from TMEM, B MN-major from
//                                      shared memory; M = 128, N = D, K = 64)
// For kDKDV the TMEM rows are keys and S is the transpose of the forward's scores; for
// kDQ the rows are queries. The S and dP buffers are double-buffered, so the MMAs of
// sub-tile n+1 run while the softmax warps work on sub-tile n.
//
// Roles (320 threads): warps 0-7 softmax (warp w reads TMEM lanes 32 (w % 4) .. +32 and
// the sub-tile's columns 32 (w / 4) .. +32), warp 8 TMA producer, warp 9 MMA issuer and
// TMEM owner. TMEM (512 columns): S0 at 0, S1 at 64, dP0 at 128, dP1 at 192, then the
// accumulators (kDKDV: dV at 256, dK at 256 + D; kDQ: dQ at 256).
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace attn {

constexpr int kBwdThreads = 320;
constexpr int kBwdFix = 128;  // rows of the fixed tiles (TMEM lanes)
constexpr int kBwdSub = 64;   // rows of a streamed sub-tile
enum : int { kDKDV = 0, kDQ = 1 };

template <int D>
struct BwdCfg {
    static constexpr int kChunks = D / 64;                 // 128-byte column chunks
    static constexpr int kFixChunk = kBwdFix * 128;        // one chunk of a fixed tile
    static constexpr int kSubChunk = kBwdSub * 128;        // one chunk of a sub-tile
    static constexpr int kFixBytes = kBwdFix * D * 2;
    static constexpr int kSubBytes = kBwdSub * D * 2;
    static constexpr int kStages = (D == 64) ? 8 : 4;
    static constexpr int kTileRegion = 2 * kFixBytes + kStages * 2 * kSubBytes;
    static constexpr int kStatBytes = kStages * 2 * kBwdSub * 4;  // lse2 + delta per stage
    // barriers: FIX_FULL, FULL/EMPTY per stage, ST_FULL[2], P_FULL[2], DONE, DRAIN
    static constexpr int kNumBars = 1 + 2 * kStages + 6;
    static constexpr int kSmemBytes = 1024 + kTileRegion + kStatBytes + kNumBars * 8 + 16;
    static_assert(kSmemBytes <= 232448, "shared-memory budget");
    static constexpr int kSCol0 = 0, kSCol1 = 64, kDPCol0 = 128, kDPCol1 = 192, kGCol = 256;
    static constexpr int kTmemCols = 512;
};

struct BwdArgs {
    const float* lse2;   // [B*Hq][Lq_pad] log2-domain lse (+inf: row sees no key / padding)
    const float* delta;  // [B*Hq][Lq_pad] dO . O
    void* dq;            // [B, Hq, Lq, D]
    void* dk;            // [B, Hkv, Lk, D]
    void* dv;            // [B, Hkv, Lk, D]
    int Hq, Hkv, group, Lq, Lk, Lq_pad;
    int win_left, win_right;  // band as in the forward pass (-1: unbounded; causal: right 0)
    float scale;              // applied to dQ and dK
    float scale_log2;         // scale * log2(e)
};

// Key j visible to query i (the forward pass's band, with i' = i + Lk - Lq).
template <int MASK>
__device__ __forceinline__ bool bwd_visible(int i, int j, const BwdArgs& a) {
    const int ii = i + (a.Lk - a.Lq);
    if (MASK == kMaskCausal) return j <= ii;
    if (MASK == kMaskWindow)
        return (a.win_left < 0 || j >= ii - a.win_left) && (a.win_right < 0 || j <= ii + a.win_right);
    return true;
}

// Streamed sub-tiles [lo, hi) a CTA walks. kDKDV: 64-row query sub-tiles with a query
// that sees a key of [k0, k0 + 128); kDQ: 64-key sub-tiles holding a key visible to a
// row of [r0, r0 + 128).
template <int KIND, int MASK>
__device__ __forceinline__ void bwd_range(int base, const BwdArgs& a, int& lo, int& hi) {
    const int off = a.Lk - a.Lq;
    const int right = (MASK == kMaskCausal) ? 0 : (MASK == kMaskWindow ? a.win_right : -1);
    const int left = (MASK == kMaskWindow) ? a.win_left : -1;
    if (KIND == kDKDV) {
        const int k0 = base, k1 = min(base + kBwdFix, a.Lk) - 1;
        long long i0 = 0, i1 = a.Lq - 1;
        if (right >= 0) i0 = max(i0, static_cast<long long>(k0) - right - off);
        if (left >= 0) i1 = min(i1, static_cast<long long>(k1) + left - off);
        if (k1 < k0 || i1 < i0) { lo = hi = 0; return; }
        lo = static_cast<int>(i0 / kBwdSub);
        hi = static_cast<int>(i1 / kBwdSub) + 1;
    } else {
        const int r0 = base, r1 = min(base + kBwdFix, a.Lq) - 1;
        long long j0 = 0, j1 = a.Lk - 1;
        if (left >= 0) j0 = max(j0, static_cast<long long>(r0) + off - left);
        if (right >= 0) j1 = min(j1, static_cast<long long>(r1) + off + right);
        if (r1 < r0 || j1 < j0) { lo = hi = 0; return; }
        lo = static_cast<int>(j0 / kBwdSub);
        hi = static_cast<int>(j1 / kBwdSub) + 1;
    }
}

// lse2 = lse * log2(e) (+inf where lse = -inf) and delta = dO . O per query row, into
// rows padded to Lq_pad (padding: +inf and 0). Eight threads per row.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const uint16_t* __restrict__ out,
                                                       const uint16_t* __restrict__ dout,
                                                       const float* __restrict__ lse,
                                                       float* __restrict__ lse2,
                                                       float* __restrict__ delta, int Lq,
                                                       int Lq_pad, long long rows_pad) {
    constexpr int kPer = D / 8;  // elements per thread: 16 (D = 128) or 8 (D = 64)
    const long long r = (blockIdx.x * 256LL + threadIdx.x) >> 3;
    const int sub = threadIdx.x & 7;
    if (r >= rows_pad) return;  // whole groups of 8 leave together
    const long long plane = r / Lq_pad;
    const int i = static_cast<int>(r % Lq_pad);
    float acc = 0.f;
    if (i < Lq) {
        const size_t e = (static_cast<size_t>(plane) * Lq + i) * D + sub * kPer;
        const uint4* po = reinterpret_cast<const uint4*>(out + e);
        const uint4* pd = reinterpret_cast<const uint4*>(dout + e);
#pragma unroll
        for (int c = 0; c < kPer / 8; ++c) {
            const uint4 a = po[c], b = pd[c];
            const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const float2 fa = unpack2<BF16>(aw[x]), fb = unpack2<BF16>(bw[x]);
                acc = fmaf(fa.x, fb.x, acc);
                acc = fmaf(fa.y, fb.y, acc);
            }
        }
    }
#pragma unroll
    for (int o = 4; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (sub == 0) {
        float l2 = INFINITY;
        if (i < Lq) {
            const float l = lse[static_cast<size_t>(plane) * Lq + i];
            l2 = (l == -INFINITY) ? INFINITY : l * kLog2e;
        }
        lse2[r] = l2;
        delta[r] = (i < Lq) ? acc : 0.f;
    }
}

template <int D, bool BF16, int MASK, int KIND>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
               const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_z,
               const BwdArgs args) {
    using Cfg = BwdCfg<D>;
    constexpr int NS = Cfg::kStages;
    constexpr int FIX_FULL = 0;
    constexpr int FULL = 1;
    constexpr int EMPTY = FULL + NS;
    constexpr int ST_FULL = EMPTY + NS;  // [2]
    constexpr int P_FULL = ST_FULL + 2;  // [2]
    constexpr int DONE = P_FULL + 2;
    constexpr int DRAIN = DONE + 1;
    static_assert(DRAIN + 1 == Cfg::kNumBars, "barrier count");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t sX = s_base;
    const uint32_t sW = s_base + Cfg::kFixBytes;
    const uint32_t sStage0 = s_base + 2 * Cfg::kFixBytes;  // stage s: Y at +2s*Sub, Z after it
    float* stats = reinterpret_cast<float*>(smem + Cfg::kTileRegion);  // [NS][2][64]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kTileRegion + Cfg::kStatBytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const uint32_t bar0 = smem_u32(bars);
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
    auto sY = [&](int st) -> uint32_t { return sStage0 + 2u * st * Cfg::kSubBytes; };
    auto sZ = [&](int st) -> uint32_t { return sStage0 + (2u * st + 1) * Cfg::kSubBytes; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // The fixed tile: kDKDV (b, h_kv, key tile), longest causal work (key tile 0) first;
    // kDQ (b, h_q, query tile), longest causal work (last query tile) first.
    const int plane = blockIdx.x;
    const int tile = (KIND == kDKDV) ? static_cast<int>(blockIdx.y)
                                     : static_cast<int>(gridDim.y - 1 - blockIdx.y);
    const int base = tile * kBwdFix;
    int s_lo, s_hi;
    bwd_range<KIND, MASK>(base, args, s_lo, s_hi);
    const int n_sub = s_hi - s_lo;
    const int n_all = (KIND == kDKDV) ? n_sub * args.group : n_sub;
    const int b = (KIND == kDKDV) ? plane / args.Hkv : plane / args.Hq;
    const int kv_plane = (KIND == kDKDV) ? plane : b * args.Hkv + (plane % args.Hq) / args.group;

    if (threadIdx.x == 0) {
        mbar_init(bar(FIX_FULL), 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar(FULL + s), 1);
            mbar_init(bar(EMPTY + s), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(ST_FULL + t), 1);
            mbar_init(bar(P_FULL + t), 256);
        }
        mbar_init(bar(DONE), 1);
        mbar_init(bar(DRAIN), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 9) {
        tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
        tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_w);
        prefetch_tmap(&tm_y);
        prefetch_tmap(&tm_z);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    int issued = 0;  // producer: sub-tiles issued (for the abort drain)
    bool mma_started = false;

    if (warp == 8) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && n_all > 0) {
            const int fix_plane = (KIND == kDKDV) ? kv_plane : plane;
            mbar_arrive_expect_tx(bar(FIX_FULL), 2 * Cfg::kFixBytes);
#pragma unroll
            for (int c = 0; c < Cfg::kChunks; ++c) {
                tma_load_3d(sX + c * Cfg::kFixChunk, &tm_x, bar(FIX_FULL), c * 64, base, fix_plane);
                tma_load_3d(sW + c * Cfg::kFixChunk, &tm_w, bar(FIX_FULL), c * 64, base, fix_plane);
            }
            for (int n = 0; n < n_all; ++n) {
                const int st = n % NS;
                if (n >= NS && !wait_phase(bar(EMPTY + st), ((n / NS) - 1) & 1, abort_flag)) break;
                int sub, y_plane;
                if (KIND == kDKDV) {
                    const int g = n / n_sub;
                    sub = s_lo + n % n_sub;
                    y_plane = b * args.Hq + (kv_plane % args.Hkv) * args.group + g;
                } else {
                    sub = s_lo + n;
                    y_plane = kv_plane;
                }
                const int row = sub * kBwdSub;
                mbar_arrive_expect_tx(bar(FULL + st), 2 * Cfg::kSubBytes +
                                                          (KIND == kDKDV ? 2 * kBwdSub * 4 : 0));
#pragma unroll
                for (int c = 0; c < Cfg::kChunks; ++c) {
                    tma_load_3d(sY(st) + c * Cfg::kSubChunk, &tm_y, bar(FULL + st), c * 64, row, y_plane);
                    tma_load_3d(sZ(st) + c * Cfg::kSubChunk, &tm_z, bar(FULL + st), c * 64, row, y_plane);
                }
                if (KIND == kDKDV) {
                    const size_t so = static_cast<size_t>(y_plane) * args.Lq_pad + row;
                    bulk_load(smem_u32(stats + st * 2 * kBwdSub), args.lse2 + so, kBwdSub * 4,
                              bar(FULL + st));
                    bulk_load(smem_u32(stats + st * 2 * kBwdSub + kBwdSub), args.delta + so,
                              kBwdSub * 4, bar(FULL + st));
                }
                issued = n + 1;
            }
        }
    } else if (warp == 9) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0 && n_all > 0) {
            constexpr uint32_t kIdescSD = idesc_f16(BF16, kBwdFix, kBwdSub, false, false);
            constexpr uint32_t kIdescG = idesc_f16(BF16, kBwdFix, D, false, true);
            mma_started = true;
            // S = X Y^T and dP = W Z^T into buffer n & 1 (K-major: 16 elements = 32 bytes
            // per step inside a 128-byte swizzle row, then the next chunk).
            auto issue_sd = [&](int n) {
                const int st = n % NS;
                const uint32_t s_col = (n & 1) ? Cfg::kSCol1 : Cfg::kSCol0;
                const uint32_t dp_col = (n & 1) ? Cfg::kDPCol1 : Cfg::kDPCol0;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t fa = (kk >> 2) * Cfg::kFixChunk + (kk & 3) * 32;
                    const uint32_t fb = (kk >> 2) * Cfg::kSubChunk + (kk & 3) * 32;
                    mma_ss(tmem + s_col, sdesc_sw128(sX + fa, 16, 1024),
                           sdesc_sw128(sY(st) + fb, 16, 1024), kIdescSD, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t fa = (kk >> 2) * Cfg::kFixChunk + (kk & 3) * 32;
                    const uint32_t fb = (kk >> 2) * Cfg::kSubChunk + (kk & 3) * 32;
                    mma_ss(tmem + dp_col, sdesc_sw128(sW + fa, 16, 1024),
                           sdesc_sw128(sZ(st) + fb, 16, 1024), kIdescSD, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(ST_FULL + (n & 1)));
            };
            // Gradient MMAs: A from TMEM (the f16/bf16 P or dS; rows 16ks..16ks+15 of the
            // sub-tile sit in the columns of the softmax warpgroup ks / 2 that wrote them),
            // B MN-major from the sub-tile (16 rows = two 8-row swizzle atoms, 2048 bytes;
            // D chunks kSubChunk apart).
            auto issue_grad = [&](int n) {
                const int st = n % NS;
                const uint32_t s_col = (n & 1) ? Cfg::kSCol1 : Cfg::kSCol0;
                const uint32_t dp_col = (n & 1) ? Cfg::kDPCol1 : Cfg::kDPCol0;
#pragma unroll
                for (int ks = 0; ks < kBwdSub / 16; ++ks) {
                    const uint32_t a_off = (ks >> 1) * 32 + (ks & 1) * 8;
                    const uint32_t acc = (n > 0 || ks > 0) ? 1u : 0u;
                    if (KIND == kDKDV)  // dV += P dO
                        mma_ts(tmem + Cfg::kGCol, tmem + s_col + a_off,
                               sdesc_sw128(sZ(st) + ks * 2048, Cfg::kSubChunk, 1024), kIdescG, acc);
                    // kDKDV: dK += dS Q;  kDQ: dQ += dS K
                    mma_ts(tmem + Cfg::kGCol + (KIND == kDKDV ? D : 0), tmem + dp_col + a_off,
                           sdesc_sw128(sY(st) + ks * 2048, Cfg::kSubChunk, 1024), kIdescG, acc);
                }
                mma_commit(bar(EMPTY + st));
            };
            bool ok = wait_phase(bar(FIX_FULL), 0, abort_flag) &&
                      wait_phase(bar(FULL + 0), 0, abort_flag);
            if (ok) {
                tc_fence_after();
                issue_sd(0);
            }
            for (int n = 0; ok && n < n_all; ++n) {
                if (n + 1 < n_all) {
                    // Buffer (n+1) & 1 was last read by the softmax of n-1 (done: its
                    // P_FULL was awaited) and by the gradient MMAs of n-1 (issued earlier,
                    // so they execute first).
                    ok = wait_phase(bar(FULL + (n + 1) % NS), ((n + 1) / NS) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    issue_sd(n + 1);
                }
                ok = wait_phase(bar(P_FULL + (n & 1)), (n >> 1) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                issue_grad(n);
            }
            if (ok) mma_commit(bar(DONE));
        }
    } else {
        // ------------------------------------------------------------- softmax
        const int wg = warp >> 2;  // which 32 columns of the 64-wide sub-tile
        const int quad = warp & 3;
        const int r = base + quad * 32 + lane;  // this thread's fixed row (key or query)
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const float c = args.scale_log2;
        float row_lse2 = 0.f, row_delta = 0.f;
        if (KIND == kDQ) {  // padded rows exist up to Lq_pad > r
            row_lse2 = args.lse2[static_cast<size_t>(plane) * args.Lq_pad + r];
            row_delta = args.delta[static_cast<size_t>(plane) * args.Lq_pad + r];
        }
        bool ok = true;
        for (int n = 0; n < n_all; ++n) {
            const int buf = n & 1;
            const int st = n % NS;
            const int sub = (KIND == kDKDV) ? s_lo + n % n_sub : s_lo + n;
            bool w = wait_phase(bar(ST_FULL + buf), (n >> 1) & 1, abort_flag);
            if (KIND == kDKDV) w = w && wait_phase(bar(FULL + st), (n / NS) & 1, abort_flag);
            if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
            tc_fence_after();
            const uint32_t s_col = (buf ? Cfg::kSCol1 : Cfg::kSCol0) + wg * 32;
            const uint32_t dp_col = (buf ? Cfg::kDPCol1 : Cfg::kDPCol0) + wg * 32;
            uint32_t sr[32], dr[32];
            tmem_ld32(lane_base + s_col, sr);
            tmem_ld32(lane_base + dp_col, dr);
            tmem_wait_ld();
            const int cbase = sub * kBwdSub + wg * 32;  // first column index (query or key)
            uint32_t pk[16], dk[16];
            if (KIND == kDKDV) {
                const float* L = stats + st * 2 * kBwdSub + wg * 32;
                const float* Dl = L + kBwdSub;
#pragma unroll
                for (int x = 0; x < 32; x += 2) {
                    float p0 = ex2_approx(fmaf(__uint_as_float(sr[x]), c, -L[x]));
                    float p1 = ex2_approx(fmaf(__uint_as_float(sr[x + 1]), c, -L[x + 1]));
                    if (MASK != kMaskNone) {
                        if (!bwd_visible<MASK>(cbase + x, r, args)) p0 = 0.f;
                        if (!bwd_visible<MASK>(cbase + x + 1, r, args)) p1 = 0.f;
                    }
                    const float d0 = p0 * (__uint_as_float(dr[x]) - Dl[x]);
                    const float d1 = p1 * (__uint_as_float(dr[x + 1]) - Dl[x + 1]);
                    pk[x / 2] = pack2<BF16>(p0, p1);
                    dk[x / 2] = pack2<BF16>(d0, d1);
                }
                tmem_st16(lane_base + s_col, pk);
            } else {
                const bool edge = (MASK != kMaskNone) || (cbase + 32 > args.Lk);
#pragma unroll
                for (int x = 0; x < 32; x += 2) {
                    float p0 = ex2_approx(fmaf(__uint_as_float(sr[x]), c, -row_lse2));
                    float p1 = ex2_approx(fmaf(__uint_as_float(sr[x + 1]), c, -row_lse2));
                    if (edge) {
                        if (cbase + x >= args.Lk || !bwd_visible<MASK>(r, cbase + x, args)) p0 = 0.f;
                        if (cbase + x + 1 >= args.Lk || !bwd_visible<MASK>(r, cbase + x + 1, args))
                            p1 = 0.f;
                    }
                    dk[x / 2] = pack2<BF16>(p0 * (__uint_as_float(dr[x]) - row_delta),
                                            p1 * (__uint_as_float(dr[x + 1]) - row_delta));
                }
            }
            tmem_st16(lane_base + dp_col, dk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(P_FULL + buf));
        }
        if (ok && n_all > 0) {
            const bool w = wait_phase(bar(DONE), 0, abort_flag);
            ok = __all_sync(0xffffffffu, w);
            if (ok) tc_fence_after();
        }
        if (ok) {
            // ------------------------------------------------------------ epilogue
            // kDKDV: warpgroup 0 writes the dV row, warpgroup 1 the dK row (times scale);
            // kDQ: each warpgroup writes half of the dQ row (times scale).
            uint16_t* dst;
            int col0, ncols, valid;
            uint32_t g_col;
            float mul;
            if (KIND == kDKDV) {
                dst = static_cast<uint16_t*>(wg == 0 ? args.dv : args.dk) +
                      (static_cast<size_t>(plane) * args.Lk + r) * D;
                col0 = 0;
                ncols = D;
                g_col = Cfg::kGCol + wg * D;
                mul = wg == 0 ? 1.f : args.scale;
                valid = r < args.Lk;
            } else {
                dst = static_cast<uint16_t*>(args.dq) + (static_cast<size_t>(plane) * args.Lq + r) * D;
                col0 = wg * (D / 2);
                ncols = D / 2;
                g_col = Cfg::kGCol + col0;
                mul = args.scale;
                valid = r < args.Lq;
            }
            for (int d0 = 0; d0 < ncols; d0 += 32) {
                uint32_t o[32];
                if (n_all > 0) {
                    tmem_ld32(lane_base + g_col + d0, o);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int x = 0; x < 32; ++x) o[x] = 0u;
                }
                uint32_t pkd[16];
#pragma unroll
                for (int x = 0; x < 16; ++x)
                    pkd[x] = pack2<BF16>(__uint_as_float(o[2 * x]) * mul,
                                         __uint_as_float(o[2 * x + 1]) * mul);
                if (valid) {
                    uint4* p = reinterpret_cast<uint4*>(dst + col0 + d0);
#pragma unroll
                    for (int x = 0; x < 4; ++x)
                        p[x] = make_uint4(pkd[4 * x], pkd[4 * x + 1], pkd[4 * x + 2], pkd[4 * x + 3]);
                }
            }
        }
    }

    // ----------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // Nothing may still be writing into this CTA's shared or tensor memory when it
        // exits: wait for the loads already issued and for every MMA issued.
        if (warp == 8 && lane == 0 && n_all > 0) {
            drain_phase(bar(FIX_FULL), 0);
            for (int n = max(0, issued - NS); n < issued; ++n)
                drain_phase(bar(FULL + n % NS), (n / NS) & 1);
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

}  // namespace attn
