// paged_decode.cuh -- decode attention over a paged KV cache (one query token per
// sequence), memory-bound.
//
// The cache is stored in fixed-size blocks of 16 tokens and a block table maps each
// sequence's logical block to a physical one; the kernel resolves every position
// through the table ("Fast attention kernels and operator fusion", the-ai.news,
// section on FlashAttention-style and paged attention; block_size = 16 as in its
// vLLM example). The softmax is exact: an online softmax per chunk of blocks, then the
// chunks of a sequence are merged with log-sum-exp weights.
//
// Work split. A unit is one (sequence, K/V head); its G = H_q / H_kv query heads are
// the rows of one m16n8k16 tensor-core tile (rows >= G are zero), so every K/V byte is
// read once. The grid has P = max(kDecCtas, 2U) CTAs for U units. Every CTA reads the
// sequence lengths and derives the same schedule: each unit is cut into
// max(1, ceil(blocks / C)) near-equal chunks, with C the smallest chunk size whose
// chunk count over all units fits P (a binary search between ceil(T / P) and
// ceil(T / (P - U)), which always fits; T = all units' blocks) while P is one wave of
// kDecCtas, else ceil(T / (P - U)); CTA c takes chunk c.
// One wave of CTAs with near-equal shares of the bytes: the kernel is bound by HBM
// bandwidth, not by its longest sequence. (With more than kDecMaxUnits units each CTA
// takes one whole unit instead.)
//
// Per CTA: a producer warp reads the chunk's block-table entries and issues 2-D TMA
// loads (128-byte swizzle) of each block's K and V rows into a ring of shared-memory
// stages; four consumer warps take the blocks in turn and read their fragments with
// ldmatrix (.trans for V), so the swizzle keeps the reads free of bank conflicts. Each
// warp keeps its own running max, sum and output; the CTA merges its warps in shared
// memory. A unit with one chunk writes O and lse directly; otherwise every chunk writes
// its normalised output and log2-sum-exp to the workspace and bumps the unit's counter
// with an acquire-release atomic, and the CTA that completes the count merges the
// chunks and resets the counter to zero.
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace attn {

constexpr int kMaxGroup = 16;
constexpr int kDecConsumers = 4;                      // consumer warps
constexpr int kDecThreads = (kDecConsumers + 1) * 32;  // + the producer warp
constexpr int kDecStages = 12;                        // blocks in flight per CTA
constexpr int kDecCtas = 296;                         // two per SM on a 148-SM B200
constexpr int kDecMaxUnits = 1024;                    // balanced schedule up to this many units

template <int D>
struct DecodeCfg {
    static constexpr int kTileBytes = kPageSize * 128;          // one 16-row x 64-column swizzled tile
    static constexpr int kKBytes = kPageSize * D * 2;           // one block's K rows (D/64 tiles)
    static constexpr int kStageBytes = 2 * kKBytes;             // K and V
    // merge buffers, reusing the ring: per-warp O with padded rows; the chunk weights of
    // one unit (a unit has at most (P - U) + 1 <= kDecMaxUnits + 1 chunks, since
    // P = max(kDecCtas, 2U) and U <= kDecMaxUnits); and, when they fit, a unit's partial
    // outputs staged for its merge, with their weights.
    static constexpr int kMergeBytes = kDecConsumers * kMaxGroup * (D + 8) * 4;
    static constexpr int kWeightBytes = (kDecMaxUnits + 1) * kMaxGroup * 4;
    static constexpr int kRingBytes = kDecStages * kStageBytes;
    static constexpr int kBufBytes = kRingBytes > kMergeBytes
                                         ? (kRingBytes > kWeightBytes ? kRingBytes : kWeightBytes)
                                         : (kMergeBytes > kWeightBytes ? kMergeBytes : kWeightBytes);
    static_assert(kDecCtas - 1 <= kDecMaxUnits, "chunks of one unit bounded by kDecMaxUnits + 1");
    static constexpr int kSmemBytes = 1024 + kBufBytes;         // + alignment slack
};

struct PagedArgs {
    const uint16_t* q;
    const int32_t* block_table;
    const int32_t* seq_lens;
    uint16_t* out;
    float* lse;
    float* ws_o;      // [P][G][D]   normalised chunk outputs
    float* ws_lse;    // [P][G]      chunk log2-sum-exp
    int* ws_count;    // [U]         completed chunks per unit
    int num_seqs, Hq, Hkv, G, max_blocks, num_blocks;
    int balanced;     // 1: chunked schedule over P CTAs; 0: one CTA per unit
    float scale_log2;
};

// Grid and workspace layout, shared by the size query and the launcher.
struct PagedLayout {
    int grid;
    int balanced;
    size_t count_off, lse_off, o_off, total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline PagedLayout paged_layout(int num_seqs, int Hq, int Hkv, int D, int max_blocks) {
    PagedLayout L{};
    const long long U = static_cast<long long>(num_seqs) * Hkv;
    if (U <= 0) return L;
    if (U > kDecMaxUnits) {  // one CTA per unit, no split, no workspace
        L.grid = static_cast<int>(U);
        L.balanced = 0;
        return L;
    }
    L.balanced = 1;
    L.grid = static_cast<int>(U * 2 > kDecCtas ? U * 2 : kDecCtas);
    if (max_blocks <= 1) return L;  // every unit fits one chunk: nothing is ever merged
    const size_t G = Hq / Hkv;
    L.count_off = 0;
    L.lse_off = align_up(static_cast<size_t>(U) * sizeof(int), 256);
    L.o_off = L.lse_off + align_up(static_cast<size_t>(L.grid) * G * sizeof(float), 256);
    L.total = L.o_off + align_up(static_cast<size_t>(L.grid) * G * D * sizeof(float), 256);
    return L;
}

// ldmatrix of four 8x8 16-bit matrices from shared memory (and the transposing form).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

template <bool BF16>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    if constexpr (BF16) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
            "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    } else {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
            "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
}

// Byte offset of 16-byte chunk `ch` (of the row's D/8) of token row `row` in a block
// stored as D/64 swizzled 16 x 64 tiles (the chunk index is XORed with row % 8).
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int ch) {
    return (ch >> 3) * DecodeCfg<D>::kTileBytes + row * 128 + (((ch & 7) ^ (row & 7)) << 4);
}

template <bool BF16>
__device__ __forceinline__ uint16_t to_bits(float x) {
    if constexpr (BF16) return __bfloat16_as_ushort(__float2bfloat16_rn(x));
    else return __half_as_ushort(__float2half_rn(x));
}

template <int D, bool BF16>
__global__ void __launch_bounds__(kDecThreads, 2)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const PagedArgs a) {
    using Cfg = DecodeCfg<D>;
    constexpr int SL = D / 16;  // score k-slabs
    constexpr int NT = D / 8;   // output n-tiles
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full_bar[kDecStages], empty_bar[kDecStages];
    __shared__ uint64_t merge_bar;  // the bulk copy of a unit's partials (last chunk only)
    __shared__ int stage_skip[kDecStages];
    __shared__ int s_nb[kDecMaxUnits];   // blocks per unit
    __shared__ int s_pre[kDecMaxUnits];  // first chunk index of each unit
    __shared__ int s_red[8];
    __shared__ float sm_m[kDecConsumers][kMaxGroup], sm_l[kDecConsumers][kMaxGroup];
    __shared__ int s_last;
    __shared__ int s_abort;  // raised by a bounded wait that ran out
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t ring = smem_u32(smem);

    const int tid = threadIdx.x;
    // Barriers first: this needs no global memory, so under programmatic stream
    // serialisation it overlaps the previous kernel's tail.
    if (tid == 0) {
        for (int s = 0; s < kDecStages; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1);
        }
        mbar_init(smem_u32(&merge_bar), 1);
        s_abort = 0;
        fence_barrier_init();
    }
    // Launched with programmatic stream serialisation: wait for the previous kernel of the
    // stream before touching global memory, and let the next one launch at once (its CTAs
    // take this grid's places as they free up and wait here in turn).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int Hkv = a.Hkv, G = a.G;
    const int U = a.num_seqs * Hkv;
    const int cap = a.max_blocks * kPageSize;

    // The block table is read only after the schedule is known: start pulling it into
    // L2 now (the CTAs split its 128-byte lines between them).
    {
        const size_t tbl_bytes = static_cast<size_t>(a.num_seqs) * a.max_blocks * sizeof(int32_t);
        const char* tbl = reinterpret_cast<const char*>(a.block_table);
        for (size_t off = (static_cast<size_t>(blockIdx.x) * blockDim.x + tid) * 128; off < tbl_bytes;
             off += static_cast<size_t>(gridDim.x) * blockDim.x * 128)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(tbl + off));
    }
    // ------------------------------------------------------------ the schedule
    int unit = -1, b0 = 0, b1 = 0, chunk0 = 0, nchunk = 1;
    int raw_len = -1;  // the unit's seq_lens entry, when the schedule already read it
    if (a.balanced && U <= 32) {
        // One warp derives the schedule for up to 32 units with shuffles only.
        if (warp == 0) {
            int nbu = 0, raw = 0;
            if (lane < U) {
                raw = a.seq_lens[lane / Hkv];
                int len = raw;
                if (len < 0 || len > cap) len = len < 0 ? 0 : cap;
                nbu = (len + kPageSize - 1) / kPageSize;
            }
            int T = nbu;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) T += __shfl_xor_sync(0xffffffffu, T, o);
            const int P = gridDim.x;
            // The smallest chunk size C whose chunk count sum_u max(1, ceil(blocks_u / C))
            // fits the P CTAs: a binary search between ceil(T / P), below which the count
            // exceeds P, and ceil(T / (P - U)), which always fits. (Here P is one wave.)
            int C = max(1, (T + (P - U) - 1) / (P - U));
            for (int lo = max(1, (T + P - 1) / P); lo < C;) {
                const int mid = (lo + C) >> 1;
                int cnt = lane < U ? max(1, (nbu + mid - 1) / mid) : 0;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
                if (cnt <= P) C = mid;
                else lo = mid + 1;
            }
            const int v = lane < U ? max(1, (nbu + C - 1) / C) : 0;
            int x = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            const int start = x - v;  // exclusive prefix
            const int cta = blockIdx.x;
            const bool mine = lane < U && cta >= start && cta < start + v;
            const unsigned who = __ballot_sync(0xffffffffu, mine);
            if (lane == 0) s_red[0] = who ? (__ffs(who) - 1) : -1;
            if (mine) {
                const int k = cta - start;
                s_red[1] = static_cast<int>(static_cast<long long>(k) * nbu / v);
                s_red[2] = static_cast<int>(static_cast<long long>(k + 1) * nbu / v);
                s_red[3] = start;
                s_red[4] = v;
                s_red[5] = raw;  // the unit's sequence length as read
            }
        }
        __syncthreads();
        unit = s_red[0];
        if (unit < 0) return;  // more CTAs than chunks (CTA-uniform)
        b0 = s_red[1];
        b1 = s_red[2];
        chunk0 = s_red[3];
        nchunk = s_red[4];
        raw_len = s_red[5];
    } else if (a.balanced) {
        // pass 1: blocks per unit, and their total T
        int part = 0;
        for (int u = tid; u < U; u += blockDim.x) {
            int len = a.seq_lens[u / Hkv];
            if (len < 0 || len > cap) len = len < 0 ? 0 : cap;  // reported by the unit's CTA
            const int nbu = (len + kPageSize - 1) / kPageSize;
            s_nb[u] = nbu;
            part += nbu;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (lane == 0) s_red[warp] = part;
        __syncthreads();
        long long T = 0;
#pragma unroll
        for (int w = 0; w < kDecThreads / 32; ++w) T += s_red[w];
        __syncthreads();
        const int P = gridDim.x;  // P >= 2U, so P - U >= U >= 1
        // the smallest feasible chunk size, as in the one-warp schedule above (every
        // thread takes the same branches: the counts are CTA-wide sums), while the grid
        // is one wave; a grid of several waves balances itself, and there fewer, larger
        // chunks cost less
        int C = static_cast<int>(max(1LL, (T + (P - U) - 1) / (P - U)));
        for (int lo = P == kDecCtas ? static_cast<int>(max(1LL, (T + P - 1) / P)) : C; lo < C;) {
            const int mid = (lo + C) >> 1;
            int cnt = 0;
            for (int u = tid; u < U; u += blockDim.x) cnt += max(1, (s_nb[u] + mid - 1) / mid);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
            if (lane == 0) s_red[warp] = cnt;
            __syncthreads();
            long long total = 0;
#pragma unroll
            for (int w = 0; w < kDecThreads / 32; ++w) total += s_red[w];
            __syncthreads();
            if (total <= P) C = mid;
            else lo = mid + 1;
        }
        // pass 2: exclusive prefix over units of the chunk counts max(1, ceil(blocks / C))
        int carry = 0;
        for (int base = 0; base < U; base += blockDim.x) {
            const int u = base + tid;
            const int v = (u < U) ? max(1, (s_nb[u] + C - 1) / C) : 0;
            int x = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (lane == 31) s_red[warp] = x;
            __syncthreads();
            int before = carry, total = 0;
#pragma unroll
            for (int w = 0; w < kDecThreads / 32; ++w) {
                if (w < warp) before += s_red[w];
                total += s_red[w];
            }
            if (u < U) s_pre[u] = before + x - v;
            carry += total;
            __syncthreads();
        }
        // this CTA's chunk: the last unit whose prefix is <= blockIdx.x
        const int cta = blockIdx.x;
        int lo = 0, hi = U - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_pre[mid] <= cta) lo = mid;
            else hi = mid - 1;
        }
        const int nbu = s_nb[lo];
        const int n = max(1, (nbu + C - 1) / C);
        if (cta >= s_pre[lo] + n) return;  // more CTAs than chunks (CTA-uniform)
        unit = lo;
        const int k = cta - s_pre[lo];
        b0 = static_cast<int>(static_cast<long long>(k) * nbu / n);
        b1 = static_cast<int>(static_cast<long long>(k + 1) * nbu / n);
        chunk0 = s_pre[lo];
        nchunk = n;
    } else {
        unit = blockIdx.x;
        int len = a.seq_lens[unit / Hkv];
        if (len < 0 || len > cap) len = len < 0 ? 0 : cap;
        b1 = (len + kPageSize - 1) / kPageSize;
    }
    const int sq = unit / Hkv;
    const int hkv = unit % Hkv;
    int len = (a.balanced && U <= 32) ? raw_len : a.seq_lens[sq];
    if (len < 0 || len > cap) {
        if (tid == 0 && b0 == 0) report_status(ATTN_ERR_BAD_INDEX);
        len = len < 0 ? 0 : cap;
    }
    const int nb = b1 - b0;

    __syncthreads();  // the barriers are initialised

    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // rows g and g + 8
    float oacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) oacc[nt][0] = oacc[nt][1] = oacc[nt][2] = oacc[nt][3] = 0.f;
    const int g = lane >> 2, t = lane & 3;
    volatile int* abort_flag = &s_abort;
    int issued = 0;  // producer: blocks whose loads were issued

    if (warp == kDecConsumers) {
        // ---------------------------------------------------------------- producer
        for (int base = 0; base < nb; base += 32) {
            int phys = -1;
            if (base + lane < nb) {
                phys = a.block_table[static_cast<size_t>(sq) * a.max_blocks + b0 + base + lane];
                if (phys < 0 || phys >= a.num_blocks) {
                    report_status(ATTN_ERR_BAD_INDEX);
                    phys = -1;
                }
            }
            const int n_here = min(32, nb - base);
            bool ok = true;
            for (int k = 0; k < n_here; ++k) {
                const int i = base + k;
                const int p = __shfl_sync(0xffffffffu, phys, k);
                if (lane == 0) {
                    const int s = i % kDecStages;
                    if (i >= kDecStages &&
                        !wait_phase(smem_u32(&empty_bar[s]), ((i / kDecStages) - 1) & 1, abort_flag))
                        ok = false;
                    const uint32_t fb = smem_u32(&full_bar[s]);
                    if (!ok) {
                        // gave up: issue nothing more
                    } else
                    if (p < 0) {
                        stage_skip[s] = 1;
                        mbar_arrive(fb);
                    } else {
                        stage_skip[s] = 0;
                        mbar_arrive_expect_tx(fb, Cfg::kStageBytes);
                        const int row = (p * Hkv + hkv) * kPageSize;
                        const uint32_t dst = ring + s * Cfg::kStageBytes;
                        // one load per block and tensor: its 16 rows as D/64 swizzled tiles
                        tma_load_3d(dst, &tm_k, fb, 0, row, 0);
                        tma_load_3d(dst + Cfg::kKBytes, &tm_v, fb, 0, row, 0);
                    }
                    if (ok) issued = i + 1;
                }
                if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
            }
            if (*abort_flag) break;
        }
    } else {
        // ---------------------------------------------------------------- consumers
        // query fragments (A operand, natural order): rows g, g + 8 = heads of the group
        uint32_t qa[SL][4];
        {
            const uint16_t* qb = a.q + (static_cast<size_t>(sq) * a.Hq + hkv * G) * D;
#pragma unroll
            for (int s = 0; s < SL; ++s) {
                const int d = 16 * s + 2 * t;
                qa[s][0] = g < G ? *reinterpret_cast<const uint32_t*>(qb + g * D + d) : 0u;
                qa[s][1] = g + 8 < G ? *reinterpret_cast<const uint32_t*>(qb + (g + 8) * D + d) : 0u;
                qa[s][2] = g < G ? *reinterpret_cast<const uint32_t*>(qb + g * D + d + 8) : 0u;
                qa[s][3] = g + 8 < G ? *reinterpret_cast<const uint32_t*>(qb + (g + 8) * D + d + 8) : 0u;
            }
        }
        const float c = a.scale_log2;
        // ldmatrix lane roles: K (x4): token (lane>>4)*8 + lane%8, chunk 2s + (lane>>3)%2;
        // V (x4.trans): token ((lane>>3)&1)*8 + lane%8, chunk 2p + (lane>>4).
        const int k_tok = ((lane >> 4) << 3) + (lane & 7), k_sub = (lane >> 3) & 1;
        const int v_tok = (((lane >> 3) & 1) << 3) + (lane & 7), v_sub = lane >> 4;
        for (int i = warp; i < nb; i += kDecConsumers) {
            const int s = i % kDecStages;
            const bool ready = __all_sync(
                0xffffffffu, wait_phase(smem_u32(&full_bar[s]), (i / kDecStages) & 1, abort_flag));
            if (!ready) break;
            if (!stage_skip[s]) {
                const uint32_t kb = ring + s * Cfg::kStageBytes;
                const uint32_t vb = kb + Cfg::kKBytes;
                float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                for (int sl = 0; sl < SL; ++sl) {
                    uint32_t kf[4];
                    ldsm_x4(kb + swz<D>(k_tok, 2 * sl + k_sub), kf);
                    mma16816<BF16>(sc[0], qa[sl], kf[0], kf[1]);
                    mma16816<BF16>(sc[1], qa[sl], kf[2], kf[3]);
                }
                const int tok0 = (b0 + i) * kPageSize;
                float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const bool in = tok0 + nt * 8 + 2 * t + e < len;
                        sc[nt][e] = in ? sc[nt][e] : -INFINITY;
                        sc[nt][2 + e] = in ? sc[nt][2 + e] : -INFINITY;
                        mx0 = fmaxf(mx0, sc[nt][e]);
                        mx1 = fmaxf(mx1, sc[nt][2 + e]);
                    }
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
                const float mn0 = fmaxf(m0, mx0 * c), mn1 = fmaxf(m1, mx1 * c);
                const float al0 = (mn0 == m0) ? 1.f : ex2_approx(m0 - mn0);
                const float al1 = (mn1 == m1) ? 1.f : ex2_approx(m1 - mn1);
                const float nm0 = (mn0 == -INFINITY) ? 0.f : -mn0;
                const float nm1 = (mn1 == -INFINITY) ? 0.f : -mn1;
                float p[2][4];
                float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    p[nt][0] = ex2_approx(fmaf(sc[nt][0], c, nm0));
                    p[nt][1] = ex2_approx(fmaf(sc[nt][1], c, nm0));
                    p[nt][2] = ex2_approx(fmaf(sc[nt][2], c, nm1));
                    p[nt][3] = ex2_approx(fmaf(sc[nt][3], c, nm1));
                    rs0 += p[nt][0] + p[nt][1];
                    rs1 += p[nt][2] + p[nt][3];
                }
                l0 = l0 * al0 + rs0;
                l1 = l1 * al1 + rs1;
                m0 = mn0;
                m1 = mn1;
                const uint32_t pa[4] = {pack2<BF16>(p[0][0], p[0][1]), pack2<BF16>(p[0][2], p[0][3]),
                                        pack2<BF16>(p[1][0], p[1][1]), pack2<BF16>(p[1][2], p[1][3])};
                // A block that crosses the sequence end: its rows past len weigh nothing,
                // and zeroing them keeps whatever they hold (even NaN) out of P.V. In the
                // B fragments, the low and high halves of b0 are tokens 2t and 2t+1, those
                // of b1 tokens 8+2t and 9+2t.
                uint32_t vm0 = 0xFFFFFFFFu, vm1 = 0xFFFFFFFFu;
                if (tok0 + kPageSize > len) {
                    vm0 = (tok0 + 2 * t < len ? 0x0000FFFFu : 0u) | (tok0 + 2 * t + 1 < len ? 0xFFFF0000u : 0u);
                    vm1 = (tok0 + 8 + 2 * t < len ? 0x0000FFFFu : 0u) |
                          (tok0 + 9 + 2 * t < len ? 0xFFFF0000u : 0u);
                }
#pragma unroll
                for (int pp = 0; pp < NT / 2; ++pp) {
                    uint32_t vf[4];
                    ldsm_x4_t(vb + swz<D>(v_tok, 2 * pp + v_sub), vf);
                    vf[0] &= vm0;
                    vf[1] &= vm1;
                    vf[2] &= vm0;
                    vf[3] &= vm1;
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        float* o = oacc[2 * pp + h2];
                        o[0] *= al0;
                        o[1] *= al0;
                        o[2] *= al1;
                        o[3] *= al1;
                        mma16816<BF16>(oacc[2 * pp + h2], pa, vf[2 * h2], vf[2 * h2 + 1]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&empty_bar[s]));
        }
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    }
    __syncthreads();  // every stage consumed: the ring is free for the merge buffers
    if (*abort_flag) {
        // A wait ran out (reported as ATTN_ERR_TIMEOUT): let the loads already issued
        // land before this CTA's shared memory is reused or released, then stop.
        if (warp == kDecConsumers && lane == 0)
            for (int i = max(0, issued - kDecStages); i < issued; ++i)
                drain_phase(smem_u32(&full_bar[i % kDecStages]), (i / kDecStages) & 1);
        return;
    }

    // ---------------------------------------------------- merge this CTA's warps
    // Per-warp outputs in shared memory (row stride D + 8 floats keeps the fragment
    // stores at most two-way bank conflicted) with each warp's row maximum and sum.
    constexpr int kRow = D + 8;
    float* sm_o = reinterpret_cast<float*>(smem);  // [kDecConsumers][16][kRow]
    if (warp < kDecConsumers) {
        if (t == 0) {
            sm_m[warp][g] = m0;
            sm_l[warp][g] = l0;
            sm_m[warp][g + 8] = m1;
            sm_l[warp][g + 8] = l1;
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float* r0 = sm_o + (warp * kMaxGroup + g) * kRow + nt * 8 + 2 * t;
            float* r1 = sm_o + (warp * kMaxGroup + g + 8) * kRow + nt * 8 + 2 * t;
            *reinterpret_cast<float2*>(r0) = make_float2(oacc[nt][0], oacc[nt][1]);
            *reinterpret_cast<float2*>(r1) = make_float2(oacc[nt][2], oacc[nt][3]);
        }
    }
    __syncthreads();
    __shared__ float s_rowM[kMaxGroup], s_rowL[kMaxGroup];  // the unit merge's row statistics

    // Each thread forms its row's combined maximum and weight from the four warps' (m, l)
    // itself (no further barrier) and writes one 4-float slice of the normalised output.
    const bool direct = nchunk == 1;
    const int cidx = blockIdx.x;  // chunk index (balanced schedule; unused when direct)
    for (int i4 = tid; i4 < G * (D / 4); i4 += blockDim.x) {
        const int r = i4 / (D / 4), d = (i4 % (D / 4)) * 4;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecConsumers; ++w) M = fmaxf(M, sm_m[w][r]);
        float f[kDecConsumers], L = 0.f;
#pragma unroll
        for (int w = 0; w < kDecConsumers; ++w) {
            f[w] = (M == -INFINITY) ? 0.f : ex2_approx(sm_m[w][r] - M);
            L += f[w] * sm_l[w][r];
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kDecConsumers; ++w) {
            const float fw = f[w] * inv;
            const float4 v = *reinterpret_cast<const float4*>(sm_o + (w * kMaxGroup + r) * kRow + d);
            o.x += fw * v.x;
            o.y += fw * v.y;
            o.z += fw * v.z;
            o.w += fw * v.w;
        }
        const float lse2 = L > 0.f ? M + log2f(L) : -INFINITY;
        if (direct) {
            const size_t orow = static_cast<size_t>(sq) * a.Hq + hkv * G + r;
            uint2 pk;
            pk.x = pack2<BF16>(o.x, o.y);
            pk.y = pack2<BF16>(o.z, o.w);
            *reinterpret_cast<uint2*>(a.out + orow * D + d) = pk;
            if (d == 0 && a.lse != nullptr) a.lse[orow] = lse2 * kLn2;
        } else {
            const size_t prow = static_cast<size_t>(cidx) * G + r;
            *reinterpret_cast<float4*>(a.ws_o + prow * D + d) = o;
            if (d == 0) a.ws_lse[prow] = lse2;
        }
    }
    if (direct) return;

    // ---------------------------------------------- the last chunk merges the unit
    // One gpu-scope acquire-release add by thread 0 after the CTA barrier: its release
    // publishes the partial stores of every thread (the barrier orders them before it),
    // its acquire makes the other chunks' partials visible here.
    __syncthreads();
    if (tid == 0) s_last = atom_add_acq_rel_gpu(&a.ws_count[unit], 1) == nchunk - 1;
    __syncthreads();
    if (!s_last) return;
    const float* part = a.ws_o + static_cast<size_t>(chunk0) * G * D;  // [nchunk][G][D]
    const float* plse = a.ws_lse + static_cast<size_t>(chunk0) * G;     // [nchunk][G]
    const int nw = nchunk * G;
    const uint32_t part_bytes = static_cast<uint32_t>(nw) * D * sizeof(float);
    // The unit's partials are contiguous: when they fit the ring they arrive by one bulk
    // copy (one round trip), else every thread loads its slices from L2.
    const bool staged = static_cast<size_t>(nw) * (D + 1) * sizeof(float) <= Cfg::kBufBytes;
    float* s_part = reinterpret_cast<float*>(smem);
    float* s_w = staged ? s_part + static_cast<size_t>(nw) * D : reinterpret_cast<float*>(smem);
    if (staged && tid == 0) {
        // the copy reads what the acquire made visible, and writes ring bytes the
        // barrier above ordered after their last generic use
        fence_proxy_async_global();
        fence_proxy_async_shared();
        mbar_arrive_expect_tx(smem_u32(&merge_bar), part_bytes);
        bulk_load(smem_u32(s_part), part, part_bytes, smem_u32(&merge_bar));
    }
    // All chunks' log2-sum-exp in shared memory (one round of parallel loads).
    for (int i = tid; i < nw; i += blockDim.x) s_w[i] = __ldcg(plse + i);
    // Few chunks: every thread forms its row's maximum and weights from the staged values
    // itself, so one barrier (after the bulk copy has landed) is all the merge waits on.
    constexpr int kFewChunks = 16;
    if (staged && nchunk <= kFewChunks) {
        if (tid == 0 && !wait_phase(smem_u32(&merge_bar), 0, abort_flag))
            drain_phase(smem_u32(&merge_bar), 0);  // gave up (reported): let the copy land
        __syncthreads();
        if (*abort_flag) return;
        for (int i4 = tid; i4 < G * (D / 4); i4 += blockDim.x) {
            const int r = i4 / (D / 4), d = (i4 % (D / 4)) * 4;
            float M = -INFINITY;
            for (int k = 0; k < nchunk; ++k) M = fmaxf(M, s_w[k * G + r]);
            float W = 0.f;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            if (M != -INFINITY) {
                const float4* src = reinterpret_cast<const float4*>(s_part + r * D + d);
                for (int k = 0; k < nchunk; ++k) {
                    const float w = ex2_approx(s_w[k * G + r] - M);
                    const float4 v = src[k * (G * D / 4)];
                    W += w;
                    acc.x = fmaf(w, v.x, acc.x);
                    acc.y = fmaf(w, v.y, acc.y);
                    acc.z = fmaf(w, v.z, acc.z);
                    acc.w = fmaf(w, v.w, acc.w);
                }
            }
            const float inv = W > 0.f ? 1.f / W : 0.f;
            const size_t orow = static_cast<size_t>(sq) * a.Hq + hkv * G + r;
            uint2 pk;
            pk.x = pack2<BF16>(acc.x * inv, acc.y * inv);
            pk.y = pack2<BF16>(acc.z * inv, acc.w * inv);
            *reinterpret_cast<uint2*>(a.out + orow * D + d) = pk;
            if (d == 0 && a.lse != nullptr)
                a.lse[orow] = W > 0.f ? (M + log2f(W)) * kLn2 : -INFINITY;
        }
        if (tid == 0) a.ws_count[unit] = 0;  // leave the workspace as found
        return;
    }
    __syncthreads();
    // Many chunks: per row the maximum, the total weight and each chunk's normalised
    // weight, one warp per row.
    for (int r = warp; r < G; r += kDecThreads / 32) {
        float M = -INFINITY;
        for (int k = lane; k < nchunk; k += 32) M = fmaxf(M, s_w[k * G + r]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float W = 0.f;
        if (M != -INFINITY)
            for (int k = lane; k < nchunk; k += 32) W += ex2_approx(s_w[k * G + r] - M);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
        if (lane == 0) {
            s_rowM[r] = M;
            s_rowL[r] = W;
        }
    }
    __syncthreads();
    for (int i = tid; i < nw; i += blockDim.x) {
        const int r = i % G;
        const float M = s_rowM[r], W = s_rowL[r];
        s_w[i] = (M == -INFINITY || !(W > 0.f)) ? 0.f : ex2_approx(s_w[i] - M) / W;
    }
    if (staged && tid == 0 && !wait_phase(smem_u32(&merge_bar), 0, abort_flag))
        drain_phase(smem_u32(&merge_bar), 0);  // gave up (reported): let the copy land
    __syncthreads();
    if (*abort_flag) return;
    // Each thread owns 4-float slices of the output and sums them over the chunks.
    for (int i4 = tid; i4 < G * (D / 4); i4 += blockDim.x) {
        const int r = i4 / (D / 4), d = (i4 % (D / 4)) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (staged) {
            // four independent sums over the chunks keep four loads in flight
            const float4* src = reinterpret_cast<const float4*>(s_part + r * D + d);
            const int step = G * D / 4;  // float4 stride between chunks
            float4 part4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) part4[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int k = 0; k < nchunk; k += 4) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (k + u < nchunk) {
                        const float w = s_w[(k + u) * G + r];
                        const float4 v = src[(k + u) * step];
                        part4[u].x += w * v.x;
                        part4[u].y += w * v.y;
                        part4[u].z += w * v.z;
                        part4[u].w += w * v.w;
                    }
                }
            }
            acc.x = (part4[0].x + part4[1].x) + (part4[2].x + part4[3].x);
            acc.y = (part4[0].y + part4[1].y) + (part4[2].y + part4[3].y);
            acc.z = (part4[0].z + part4[1].z) + (part4[2].z + part4[3].z);
            acc.w = (part4[0].w + part4[1].w) + (part4[2].w + part4[3].w);
        } else {
            const float4* src = reinterpret_cast<const float4*>(part + r * D + d);
            const size_t step = static_cast<size_t>(G) * D / 4;
            for (int k = 0; k < nchunk; k += 8) {
                float4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    v[u] = (k + u < nchunk) ? __ldcg(src + (k + u) * step) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const float w = (k + u < nchunk) ? s_w[(k + u) * G + r] : 0.f;
                    acc.x += w * v[u].x;
                    acc.y += w * v[u].y;
                    acc.z += w * v[u].z;
                    acc.w += w * v[u].w;
                }
            }
        }
        const size_t orow = static_cast<size_t>(sq) * a.Hq + hkv * G + r;
        uint2 pk;
        pk.x = pack2<BF16>(acc.x, acc.y);
        pk.y = pack2<BF16>(acc.z, acc.w);
        *reinterpret_cast<uint2*>(a.out + orow * D + d) = pk;
        if (d == 0 && a.lse != nullptr) {
            const float M = s_rowM[r], W = s_rowL[r];
            a.lse[orow] = (M == -INFINITY || !(W > 0.f)) ? -INFINITY : (M + log2f(W)) * kLn2;
        }
    }
    if (tid == 0) a.ws_count[unit] = 0;  // leave the workspace as found
}

}  // namespace attn
