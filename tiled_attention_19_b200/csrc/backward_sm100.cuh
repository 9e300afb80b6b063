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
//                    shared memory while 128-row sub-tiles of Q and dO (of every query
//                    head of the group) stream through a ring; dV and dK accumulate in TMEM.
//   bwd_kernel<kDQ>  one CTA per 128-row query tile of one (batch, head): Q and dO stay,
//                    128-key sub-tiles of K and V stream; dQ accumulates in TMEM.
// Both kinds run the same pipeline. Call the fixed pair (X, W) and a streamed pair
// (Y, Z): (K, V) and (Q, dO) for kDKDV, (Q, dO) and (K, V) for kDQ. Per sub-tile n:
//   S  = X Y^T, dP = W Z^T     (M = N = 128, K = D; both operands K-major from shared
//                               memory; fp32 in TMEM)
//   softmax warps: copy S and dP to registers, release the dP columns (DP_FREE) and
//                 form P and dS; kDKDV does it in two phases (P from S as soon as S is
//                 there, dS once dP is); write P (kDKDV only) and dS in f16/bf16 over
//                 their own S columns
//   kDKDV: dK += dS Y, dV += P Z;  kDQ: dQ += dS Y   (A from TMEM, B MN-major from
//                               shared memory; M = 128, N = D, K = 128)
// For kDKDV the TMEM rows are keys and S is the transpose of the forward's scores. Its
// two 128-column regions swap roles every sub-tile: S(n+1) goes where dP(n) was as soon
// as the softmax warps hold dP(n), so their exponentials for n+1 overlap the gradient
// MMAs of n; dP(n+1) then takes the region of S(n) behind those MMAs. kDQ keeps two S
// buffers and one dP buffer and computes S and dP of n+1 while the softmax works on n.
// Every product is 128 wide: a 64-wide product of the same work runs at a fraction of the
// tensor core's rate.
//
// Roles (384 threads): warps 0-7 softmax (warp w reads TMEM lanes 32 (w % 4) .. +32 and
// the sub-tile's columns 64 (w / 4) .. +64), warp 8 TMA producer, warp 9 MMA issuer and
// TMEM owner, warps 10-11 idle (they complete the third warpgroup for setmaxnreg).
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace attn {

constexpr int kBwdThreads = 384;
// Register split between warpgroups (setmaxnreg), as in the forward kernel: the two
// softmax warpgroups take 192 registers, the third (producer, MMA issuer, two idle warps)
// keeps 104. The launcher checks that the CTA's launch registers (384 x registers per
// thread) cover 2 x 128 x 192 + 128 x 104 before the first launch: an unsatisfiable
// setmaxnreg.inc would wait forever.
constexpr int kBwdSoftmaxRegs = 192;
constexpr int kBwdOtherRegs = 104;
constexpr int kBwdRegBudget = 2 * 128 * kBwdSoftmaxRegs + 128 * kBwdOtherRegs;  // 62,464
constexpr int kBwdFix = 128;  // rows of the fixed tiles (TMEM lanes)
constexpr int kBwdSub = 128;  // rows of a streamed sub-tile
enum : int { kDKDV = 0, kDQ = 1 };

template <int D, int KIND>
struct BwdCfg {
    static constexpr int kChunks = D / 64;                 // 128-byte column chunks
    static constexpr int kFixChunk = kBwdFix * 128;        // one chunk of a fixed tile
    static constexpr int kSubChunk = kBwdSub * 128;        // one chunk of a sub-tile
    static constexpr int kFixBytes = kBwdFix * D * 2;
    static constexpr int kSubBytes = kBwdSub * D * 2;
    // Separate rings for the two streamed tiles. kDQ frees V (Z) after dP and K (Y) only
    // after dQ += dS K, so K gets the extra stage.
    static constexpr int kYStages = (D == 64) ? 4 : (KIND == kDQ ? 3 : 2);
    static constexpr int kZStages = (D == 64) ? 4 : 2;
    static constexpr int kTileRegion = 2 * kFixBytes + (kYStages + kZStages) * kSubBytes;
    // kDKDV: -lse*log2(e) and delta of the 128 query rows of each Y stage
    static constexpr int kStatBytes = (KIND == kDKDV) ? kYStages * 2 * kBwdSub * 4 : 0;
    // barriers: FIX_FULL, FULL/EMPTY per Y and per Z stage, S_FULL, DP_FULL, DP_FREE, two
    // P_FULL, DONE, DRAIN
    static constexpr int kNumBars = 1 + 2 * (kYStages + kZStages) + 7;
    static constexpr int kSmemBytes = 1024 + kTileRegion + kStatBytes + kNumBars * 8 + 16;
    static_assert(kSmemBytes <= 232448, "shared-memory budget");
    // TMEM: kDQ: S of even / odd sub-tiles at 0 / 128, dP at 256, dQ at 384;
    //       kDKDV: two regions at 0 and 128 that swap roles every sub-tile (S of sub-tile n
    //       in region n & 1, its dP in the other), dV at 256, dK at 256 + D.
    static constexpr int kTmemCols = 512;
};

struct BwdArgs {
    const float* nlse2;  // [B*Hq][Lq_pad] -lse * log2(e) (-inf: row sees no key / padding)
    const float* delta;  // [B*Hq][Lq_pad] dO . O
    void* dq;            // [B, Hq, Lq, D] through dq_s
    void* dk;            // [B, Hkv, Lk, D] through dk_s
    void* dv;            // [B, Hkv, Lk, D] through dv_s
    long long dq_s[3], dk_s[3], dv_s[3];  // element strides over (batch, head, row)
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

// True if every query of [i0, i0 + ni) sees every key of [j0, j0 + nj) (no element mask
// needed; rows past Lq are zeroed through their -inf statistics instead).
template <int MASK>
__device__ __forceinline__ bool bwd_all_visible(int i0, int ni, int j0, int nj, const BwdArgs& a) {
    const int off = a.Lk - a.Lq;
    if (MASK == kMaskCausal) return j0 + nj - 1 <= i0 + off;
    if (MASK == kMaskWindow)
        return (a.win_left < 0 || j0 >= i0 + ni - 1 + off - a.win_left) &&
               (a.win_right < 0 || j0 + nj - 1 <= i0 + off + a.win_right);
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

// nlse2 = -lse * log2(e) (-inf where lse = -inf) and delta = dO . O per query row, into
// rows padded to Lq_pad (padding: -inf and 0). Eight threads per row.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const uint16_t* __restrict__ out,
                                                       const uint16_t* __restrict__ dout,
                                                       const float* __restrict__ lse,
                                                       float* __restrict__ nlse2,
                                                       float* __restrict__ delta, int Lq,
                                                       int Lq_pad, long long rows_pad, int Hq,
                                                       long long o_sb, long long o_sh,
                                                       long long o_sl, long long d_sb,
                                                       long long d_sh, long long d_sl) {
    constexpr int kPer = D / 8;  // elements per thread: 16 (D = 128) or 8 (D = 64)
    const long long r = (blockIdx.x * 256LL + threadIdx.x) >> 3;
    const int sub = threadIdx.x & 7;
    if (r >= rows_pad) return;  // whole groups of 8 leave together
    const long long plane = r / Lq_pad;
    const int i = static_cast<int>(r % Lq_pad);
    float acc = 0.f;
    if (i < Lq) {
        const long long bb = plane / Hq, hh = plane % Hq;
        const uint4* po = reinterpret_cast<const uint4*>(out + bb * o_sb + hh * o_sh + i * o_sl + sub * kPer);
        const uint4* pd = reinterpret_cast<const uint4*>(dout + bb * d_sb + hh * d_sh + i * d_sl + sub * kPer);
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
        float nl2 = -INFINITY;
        if (i < Lq) {
            const float l = lse[static_cast<size_t>(plane) * Lq + i];
            nl2 = (l == -INFINITY) ? -INFINITY : -l * kLog2e;
        }
        nlse2[r] = nl2;
        delta[r] = (i < Lq) ? acc : 0.f;
    }
}

template <int D, bool BF16, int MASK, int KIND>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
               const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_z,
               const BwdArgs args) {
    using Cfg = BwdCfg<D, KIND>;
    constexpr int NY = Cfg::kYStages;
    constexpr int NZ = Cfg::kZStages;
    constexpr int FIX_FULL = 0;
    constexpr int Y_FULL = 1;
    constexpr int Y_EMPTY = Y_FULL + NY;
    constexpr int Z_FULL = Y_EMPTY + NY;
    constexpr int Z_EMPTY = Z_FULL + NZ;
    constexpr int S_FULL = Z_EMPTY + NZ;   // S of the next sub-tile is in TMEM
    constexpr int DP_FULL = S_FULL + 1;    // dP of the next sub-tile is in TMEM
    constexpr int DP_FREE = DP_FULL + 1;   // the softmax warps hold S and dP in registers
    // P / dS of sub-tile n are in TMEM: barrier P_FULL + (n & 1). The 256 softmax threads
    // arrive once per sub-tile, and for kDQ a fast warp can arrive for n + 1 (S and dP of
    // n + 1 are issued as soon as every warp holds those of n) while a slow one is still
    // writing dS(n); on a single barrier that early arrival would complete phase n before
    // dS(n) is whole. Alternating barriers keep each phase's arrivals apart: no warp can
    // reach n + 2 before every warp has finished n, since S(n + 2) waits for DP_FREE(n + 1).
    constexpr int P_FULL = DP_FREE + 1;
    constexpr int DONE = P_FULL + 2;
    constexpr int DRAIN = DONE + 1;
    static_assert(DRAIN + 1 == Cfg::kNumBars, "barrier count");
    constexpr uint32_t G_COL = (KIND == kDKDV) ? 256 : 384;
    static_assert(G_COL + (KIND == kDKDV ? 2 * D : D) <= Cfg::kTmemCols, "TMEM budget");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t sX = s_base;
    const uint32_t sW = s_base + Cfg::kFixBytes;
    const uint32_t sY0 = s_base + 2 * Cfg::kFixBytes;
    const uint32_t sZ0 = sY0 + NY * Cfg::kSubBytes;
    float* stats = reinterpret_cast<float*>(smem + Cfg::kTileRegion);  // kDKDV: [NY][2][128]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kTileRegion + Cfg::kStatBytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const uint32_t bar0 = smem_u32(bars);
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
    auto sY = [&](int n) -> uint32_t { return sY0 + (n % NY) * Cfg::kSubBytes; };
    auto sZ = [&](int n) -> uint32_t { return sZ0 + (n % NZ) * Cfg::kSubBytes; };
    // TMEM columns of S and dP of sub-tile n (P and dS are written over S)
    auto s_col_of = [&](int n) -> uint32_t { return (n & 1) ? 128u : 0u; };
    auto dp_col_of = [&](int n) -> uint32_t {
        return (KIND == kDQ) ? 256u : ((n & 1) ? 0u : 128u);
    };

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
    const int h_fix = (KIND == kDKDV) ? plane % args.Hkv : plane % args.Hq;  // head of the fixed pair

    if (threadIdx.x == 0) {
        mbar_init(bar(FIX_FULL), 1);
        for (int s = 0; s < NY; ++s) {
            mbar_init(bar(Y_FULL + s), 1);
            mbar_init(bar(Y_EMPTY + s), 1);
        }
        for (int s = 0; s < NZ; ++s) {
            mbar_init(bar(Z_FULL + s), 1);
            mbar_init(bar(Z_EMPTY + s), 1);
        }
        mbar_init(bar(S_FULL), 1);
        mbar_init(bar(DP_FULL), 1);
        mbar_init(bar(DP_FREE), 256);
        mbar_init(bar(P_FULL), 256);
        mbar_init(bar(P_FULL + 1), 256);
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

    int y_issued = 0, z_issued = 0;  // producer: sub-tiles issued per ring (abort drain)
    bool mma_started = false;

    if (warp >= 10) {
        regs_decrease<kBwdOtherRegs>();  // idle warps of the third warpgroup
    } else if (warp == 8) {
        // ------------------------------------------------------------ producer
        regs_decrease<kBwdOtherRegs>();
        if (lane == 0 && n_all > 0) {
            mbar_arrive_expect_tx(bar(FIX_FULL), 2 * Cfg::kFixBytes);
#pragma unroll
            for (int c = 0; c < Cfg::kChunks; ++c) {
                tma_load_4d(sX + c * Cfg::kFixChunk, &tm_x, bar(FIX_FULL), c * 64, base, h_fix, b);
                tma_load_4d(sW + c * Cfg::kFixChunk, &tm_w, bar(FIX_FULL), c * 64, base, h_fix, b);
            }
            for (int n = 0; n < n_all; ++n) {
                int sub, y_plane, h_y;  // the streamed pair's (batch * heads + head) and head
                if (KIND == kDKDV) {
                    const int g = n / n_sub;
                    sub = s_lo + n % n_sub;
                    h_y = (kv_plane % args.Hkv) * args.group + g;
                    y_plane = b * args.Hq + h_y;
                } else {
                    sub = s_lo + n;
                    h_y = kv_plane % args.Hkv;
                    y_plane = kv_plane;
                }
                const int row = sub * kBwdSub;
                // Load first the tile whose slot frees first and is needed first: kDQ
                // frees V (Z) after dP; kDKDV needs Q (Y) early, for S of the next sub-tile.
                const int zs = n % NZ, ys = n % NY;
                auto load_z = [&]() -> bool {
                    if (n >= NZ && !wait_phase(bar(Z_EMPTY + zs), ((n / NZ) - 1) & 1, abort_flag))
                        return false;
                    mbar_arrive_expect_tx(bar(Z_FULL + zs), Cfg::kSubBytes);
#pragma unroll
                    for (int c = 0; c < Cfg::kChunks; ++c)
                        tma_load_4d(sZ(n) + c * Cfg::kSubChunk, &tm_z, bar(Z_FULL + zs), c * 64, row,
                                    h_y, b);
                    z_issued = n + 1;
                    return true;
                };
                auto load_y = [&]() -> bool {
                    if (n >= NY && !wait_phase(bar(Y_EMPTY + ys), ((n / NY) - 1) & 1, abort_flag))
                        return false;
                    mbar_arrive_expect_tx(bar(Y_FULL + ys),
                                          Cfg::kSubBytes + (KIND == kDKDV ? 2 * kBwdSub * 4 : 0));
#pragma unroll
                    for (int c = 0; c < Cfg::kChunks; ++c)
                        tma_load_4d(sY(n) + c * Cfg::kSubChunk, &tm_y, bar(Y_FULL + ys), c * 64, row,
                                    h_y, b);
                    if (KIND == kDKDV) {
                        const size_t so = static_cast<size_t>(y_plane) * args.Lq_pad + row;
                        bulk_load(smem_u32(stats + ys * 2 * kBwdSub), args.nlse2 + so, kBwdSub * 4,
                                  bar(Y_FULL + ys));
                        bulk_load(smem_u32(stats + ys * 2 * kBwdSub + kBwdSub), args.delta + so,
                                  kBwdSub * 4, bar(Y_FULL + ys));
                    }
                    y_issued = n + 1;
                    return true;
                };
                if (KIND == kDQ) {
                    if (!load_z() || !load_y()) break;
                } else {
                    if (!load_y() || !load_z()) break;
                }
            }
        }
    } else if (warp == 9) {
        // ---------------------------------------------------------- MMA issuer
        regs_decrease<kBwdOtherRegs>();
        if (lane == 0 && n_all > 0) {
            constexpr uint32_t kIdescSD = idesc_f16(BF16, kBwdFix, kBwdSub, false, false);
            constexpr uint32_t kIdescG = idesc_f16(BF16, kBwdFix, D, false, true);
            mma_started = true;
            // S = X Y^T into column s_col, or dP = W Z^T into DP_COL (K-major operands: 16
            // elements = 32 bytes per step inside a 128-byte swizzle row, then the next chunk).
            // The issue of a tcgen05.mma blocks while the tensor core's queue is full, so
            // work between products idles it: each operand's descriptor is built once per
            // call and offset per step (the start address is the descriptor's low field, in
            // 16-byte units, and never carries out of it).
            auto issue_prod = [&](uint32_t a_tile, uint32_t b_tile, uint32_t d_col) {
                const uint64_t da = sdesc_sw128(a_tile, 16, 1024), db = sdesc_sw128(b_tile, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t fa = ((kk >> 2) * Cfg::kFixChunk + (kk & 3) * 32) >> 4;
                    const uint32_t fb = ((kk >> 2) * Cfg::kSubChunk + (kk & 3) * 32) >> 4;
                    mma_ss(tmem + d_col, da + fa, db + fb, kIdescSD, kk > 0 ? 1u : 0u);
                }
            };
            // acc += A B with A the f16/bf16 tile the softmax warps packed into TMEM at
            // a_col (sub-tile rows 64w .. 64w+63 sit at columns 64w .. 64w+31 of it), B
            // MN-major from a sub-tile (16 rows = two 8-row swizzle atoms, 2048 bytes;
            // D chunks kSubChunk apart).
            auto issue_grad = [&](uint32_t acc_col, uint32_t a_col, uint32_t b_tile, bool first) {
                const uint64_t db = sdesc_sw128(b_tile, Cfg::kSubChunk, 1024);
#pragma unroll
                for (int ks = 0; ks < kBwdSub / 16; ++ks)
                    mma_ts(tmem + acc_col, tmem + a_col + (ks >> 2) * 64 + (ks & 3) * 8,
                           db + ks * (2048 >> 4), kIdescG, (!first || ks > 0) ? 1u : 0u);
            };
            bool ok = wait_phase(bar(FIX_FULL), 0, abort_flag) &&
                      wait_phase(bar(Y_FULL + 0), 0, abort_flag) &&
                      wait_phase(bar(Z_FULL + 0), 0, abort_flag);
            if (ok) {
                tc_fence_after();
                issue_prod(sX, sY(0), s_col_of(0));
                mma_commit(bar(S_FULL));
                issue_prod(sW, sZ(0), dp_col_of(0));
                mma_commit(bar(DP_FULL));
                if (KIND == kDQ) mma_commit(bar(Z_EMPTY + 0));  // V(0) was needed by dP only
            }
            for (int n = 0; ok && n < n_all; ++n) {
                const int m = n + 1;
                const bool more = m < n_all;
                if (more) {
                    // The softmax warps copied S(n) and dP(n) to registers. S(n+1) takes
                    // the region dP(n) used (kDKDV) or the S buffer of n-1, whose dS the
                    // gradient MMA of n-1 (issued earlier) reads first (kDQ); kDQ's dP(n+1)
                    // takes the dP columns.
                    ok = wait_phase(bar(Y_FULL + m % NY), (m / NY) & 1, abort_flag) &&
                         (KIND == kDKDV || wait_phase(bar(Z_FULL + m % NZ), (m / NZ) & 1, abort_flag)) &&
                         wait_phase(bar(DP_FREE), n & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    issue_prod(sX, sY(m), s_col_of(m));
                    mma_commit(bar(S_FULL));
                    if (KIND == kDQ) {
                        issue_prod(sW, sZ(m), dp_col_of(m));
                        mma_commit(bar(DP_FULL));
                        mma_commit(bar(Z_EMPTY + m % NZ));
                    }
                }
                ok = wait_phase(bar(P_FULL + (n & 1)), (n >> 1) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                if (KIND == kDKDV) {
                    // dK += dS Q, then dV += P dO; P and dS sit in the S region of n
                    issue_grad(G_COL + D, s_col_of(n) + 32, sY(n), n == 0);
                    mma_commit(bar(Y_EMPTY + n % NY));
                    issue_grad(G_COL, s_col_of(n), sZ(n), n == 0);
                    mma_commit(bar(Z_EMPTY + n % NZ));
                    if (more) {
                        // dP(n+1) takes the S region of n, read by the MMAs just issued
                        ok = wait_phase(bar(Z_FULL + m % NZ), (m / NZ) & 1, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
                        issue_prod(sW, sZ(m), dp_col_of(m));
                        mma_commit(bar(DP_FULL));
                    }
                } else {
                    issue_grad(G_COL, s_col_of(n), sY(n), n == 0);  // dQ += dS K
                    mma_commit(bar(Y_EMPTY + n % NY));
                }
            }
            if (ok) mma_commit(bar(DONE));
        }
    } else {
        // ------------------------------------------------------------- softmax
        regs_increase<kBwdSoftmaxRegs>();
        const int wg = warp >> 2;  // which 64 columns of the 128-wide sub-tile
        const int quad = warp & 3;
        const int r = base + quad * 32 + lane;  // this thread's fixed row (key or query)
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const uint64_t c2 = f2pack(args.scale_log2, args.scale_log2);
        uint64_t nl2_row = 0, dl2_row = 0;
        if (KIND == kDQ) {  // padded rows exist up to Lq_pad > r
            const float nl = args.nlse2[static_cast<size_t>(plane) * args.Lq_pad + r];
            const float dl = args.delta[static_cast<size_t>(plane) * args.Lq_pad + r];
            nl2_row = f2pack(nl, nl);
            dl2_row = f2pack(dl, dl);
        }
        bool ok = true;
        for (int n = 0; n < n_all; ++n) {
            const int sub = (KIND == kDKDV) ? s_lo + n % n_sub : s_lo + n;
            // kDKDV, phase 1: P from S (and the statistics) alone; dP comes later.
            // kDQ: S and dP arrive together; both are copied and released at once.
            bool w = wait_phase(bar(S_FULL), n & 1, abort_flag);
            if (KIND == kDKDV) w = w && wait_phase(bar(Y_FULL + n % NY), (n / NY) & 1, abort_flag);
            else w = w && wait_phase(bar(DP_FULL), n & 1, abort_flag);
            if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
            tc_fence_after();
            const uint32_t s_col = s_col_of(n) + wg * 64;
            const uint32_t dp_col = dp_col_of(n) + wg * 64;
            uint32_t sr[64], dr[64];
            tmem_ld32(lane_base + s_col, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
            tmem_ld32(lane_base + s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
            if (KIND == kDQ) {
                tmem_ld32(lane_base + dp_col, *reinterpret_cast<uint32_t(*)[32]>(&dr[0]));
                tmem_ld32(lane_base + dp_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&dr[32]));
            }
            tmem_wait_ld();
            if (KIND == kDQ) {
                tc_fence_before();
                mbar_arrive(bar(DP_FREE));  // S and dP of n are in registers
            }
            const int cbase = sub * kBwdSub + wg * 64;  // first column index (query or key)
            const float* st = stats + (n % NY) * 2 * kBwdSub + wg * 64;
            uint64_t p2[32];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int c0 = cbase + h * 32;  // first column of this half
                bool full;
                if (KIND == kDKDV) full = bwd_all_visible<MASK>(c0, 32, r, 1, args);
                else full = c0 + 32 <= args.Lk && bwd_all_visible<MASK>(r, 1, c0, 32, args);
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int x = h * 32 + 2 * q;
                    uint64_t nl2;
                    if (KIND == kDKDV) {
                        const float2 nl = reinterpret_cast<const float2*>(st + h * 32)[q];
                        nl2 = f2pack(nl.x, nl.y);
                    } else {
                        nl2 = nl2_row;
                    }
                    float t0, t1;
                    f2unpack(fma2(f2pack(__uint_as_float(sr[x]), __uint_as_float(sr[x + 1])), c2, nl2),
                             t0, t1);
                    float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
                    if (!full) {
                        if (KIND == kDKDV) {
                            if (!bwd_visible<MASK>(c0 + 2 * q, r, args)) p0 = 0.f;
                            if (!bwd_visible<MASK>(c0 + 2 * q + 1, r, args)) p1 = 0.f;
                        } else {
                            if (c0 + 2 * q >= args.Lk || !bwd_visible<MASK>(r, c0 + 2 * q, args)) p0 = 0.f;
                            if (c0 + 2 * q + 1 >= args.Lk || !bwd_visible<MASK>(r, c0 + 2 * q + 1, args))
                                p1 = 0.f;
                        }
                    }
                    p2[h * 16 + q] = f2pack(p0, p1);
                }
            }
            if (KIND == kDKDV) {
                // Phase 2: dS = P (dP - delta) once dP is there.
                w = wait_phase(bar(DP_FULL), n & 1, abort_flag);
                if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
                tc_fence_after();
                tmem_ld32(lane_base + dp_col, *reinterpret_cast<uint32_t(*)[32]>(&dr[0]));
                tmem_ld32(lane_base + dp_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&dr[32]));
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(bar(DP_FREE));  // S and dP of n are in registers
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t pk[16], dk[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int x = h * 32 + 2 * q;
                    uint64_t dl2;
                    if (KIND == kDKDV) {
                        const float2 dl = reinterpret_cast<const float2*>(st + kBwdSub + h * 32)[q];
                        dl2 = f2pack(dl.x, dl.y);
                    } else {
                        dl2 = dl2_row;
                    }
                    float p0, p1, d0, d1;
                    f2unpack(p2[h * 16 + q], p0, p1);
                    if (KIND == kDKDV) pk[q] = pack2<BF16>(p0, p1);
                    f2unpack(mul2(p2[h * 16 + q],
                                  sub2(f2pack(__uint_as_float(dr[x]), __uint_as_float(dr[x + 1])), dl2)),
                             d0, d1);
                    dk[q] = pack2<BF16>(d0, d1);
                }
                if (KIND == kDKDV) {
                    // P at columns 64w + [0, 32), dS at 64w + [32, 64) of the S region: this
                    // warpgroup's own S columns, already copied to registers
                    tmem_st16(lane_base + s_col + h * 16, pk);
                    tmem_st16(lane_base + s_col + 32 + h * 16, dk);
                } else {
                    tmem_st16(lane_base + s_col + h * 16, dk);  // dS at 64w + [0, 32)
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(P_FULL + (n & 1)));
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
                const long long* st = wg == 0 ? args.dv_s : args.dk_s;
                dst = static_cast<uint16_t*>(wg == 0 ? args.dv : args.dk) + b * st[0] + h_fix * st[1] +
                      static_cast<long long>(r) * st[2];
                col0 = 0;
                ncols = D;
                g_col = G_COL + wg * D;
                mul = wg == 0 ? 1.f : args.scale;
                valid = r < args.Lk;
            } else {
                dst = static_cast<uint16_t*>(args.dq) + b * args.dq_s[0] + h_fix * args.dq_s[1] +
                      static_cast<long long>(r) * args.dq_s[2];
                col0 = wg * (D / 2);
                ncols = D / 2;
                g_col = G_COL + col0;
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
            for (int n = max(0, y_issued - NY); n < y_issued; ++n)
                drain_phase(bar(Y_FULL + n % NY), (n / NY) & 1);
            for (int n = max(0, z_issued - NZ); n < z_issued; ++n)
                drain_phase(bar(Z_FULL + n % NZ), (n / NZ) & 1);
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
