// paged_decode.cuh -- decode attention over a paged KV cache (one query token per
// sequence), memory-bound.
//
// The cache is stored in fixed-size blocks of 16 tokens and a block table maps each
// sequence's logical block to a physical one; the kernel resolves every position
// through the table ("Fast attention kernels and operator fusion", the-ai.news,
// section on FlashAttention-style and paged attention; block_size = 16 as in its
// vLLM example). The softmax is exact: per K/V chunk an online softmax, then the
// chunks are merged with log-sum-exp weights.
//
// Work unit = (sequence s, K/V head, chunk of kBlocksPerCta blocks). One CTA of
// kDecWarps warps; each warp owns kBlocksPerWarp whole blocks. All G = H_q / H_kv
// query heads of the K/V head are processed together as the 16 rows of an
// m16n8k16 tensor-core tile (rows >= G are zero), so every K/V byte is read once.
//
// Fragments come straight from global memory into registers with 16-byte loads:
//  - Scores: the dot product over D may take the D positions in any order, so the
//    query and key fragments use the same permutation: mma thread (g, t) holds the
//    D/4 contiguous dims [t*D/4, (t+1)*D/4) of its token row, slab s taking dims
//    t*D/4 + 4s .. 4s+3. Each thread loads two 64-byte runs of K per block.
//  - P·V: output dims are permuted so thread (g, t) holds V columns
//    g*D/8 .. g*D/8 + D/8 - 1 for its four token rows 2t, 2t+1, 2t+8, 2t+9; the
//    accumulator of thread (g, t) then covers output dims [2t*D/8, (2t+2)*D/8).
// The P fragment is the score accumulator itself (the usual register reuse).
//
// Split-KV combine: each CTA reduces its warps in shared memory. A sequence that
// fits one CTA writes O and lse directly. Otherwise each CTA writes its normalised
// partial O and its log2-sum-exp to the workspace, fences, and bumps a per-(s, head)
// counter; the CTA that brings the counter to the number of chunks merges all
// partials and resets the counter to 0.
#pragma once
#include "common.cuh"

namespace attn {

constexpr int kDecWarps = 4;
constexpr int kBlocksPerWarp = 2;
constexpr int kBlocksPerCta = kDecWarps * kBlocksPerWarp;
constexpr int kPageSize = 16;
constexpr int kMaxGroup = 16;

struct PagedArgs {
    const uint16_t* q;
    const uint16_t* kc;
    const uint16_t* vc;
    const int32_t* block_table;
    const int32_t* seq_lens;
    uint16_t* out;
    float* lse;
    float* ws_o;      // [S][Hkv][max_splits][G][D]
    float* ws_lse;    // [S][Hkv][max_splits][G], log2 units
    int* ws_count;    // [S][Hkv]
    int Hq, Hkv, G, max_blocks, num_blocks, max_splits;
    float scale_log2;
};

// Workspace layout shared by the size query and the launcher.
struct PagedLayout {
    int max_splits;
    size_t count_off, lse_off, o_off, total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline PagedLayout paged_layout(int num_seqs, int Hq, int Hkv, int D, int max_blocks) {
    PagedLayout L{};
    L.max_splits = max_blocks <= 0 ? 1 : (max_blocks + kBlocksPerCta - 1) / kBlocksPerCta;
    if (L.max_splits <= 1 || num_seqs <= 0) {
        L.max_splits = 1;
        return L;
    }
    const size_t units = static_cast<size_t>(num_seqs) * Hkv;
    const size_t G = Hq / Hkv;
    L.count_off = 0;
    L.lse_off = align_up(units * sizeof(int), 256);
    L.o_off = L.lse_off + align_up(units * L.max_splits * G * sizeof(float), 256);
    L.total = L.o_off + align_up(units * L.max_splits * G * D * sizeof(float), 256);
    return L;
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
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

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

template <int D, bool BF16>
__global__ void __launch_bounds__(kDecWarps * 32)
    paged_decode_kernel(const PagedArgs a) {
    constexpr int KU = D / 32;   // 16-byte K loads per token run (D/4 elements)
    constexpr int VU = D / 64;   // 16-byte V loads per token run (D/8 elements)
    constexpr int NT = D / 8;    // P·V n-tiles
    constexpr int SL = D / 16;   // score k-slabs
    __shared__ float sm_m[kDecWarps][kMaxGroup];
    __shared__ float sm_l[kDecWarps][kMaxGroup];
    __shared__ __align__(16) float sm_o[kDecWarps][kMaxGroup][D];
    __shared__ int sm_last;

    const int split = blockIdx.x;
    const int hkv = blockIdx.y;
    const int sq = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2;  // mma group id: head row g (and g + 8), or token row
    const int t = lane & 3;   // thread in group

    int len = a.seq_lens[sq];
    const int cap = a.max_blocks * kPageSize;
    if (len < 0 || len > cap) {
        report_status(ATTN_ERR_BAD_INDEX);
        len = len < 0 ? 0 : cap;
    }
    const int nblk = (len + kPageSize - 1) / kPageSize;
    const int nsplit = nblk == 0 ? 1 : (nblk + kBlocksPerCta - 1) / kBlocksPerCta;
    if (split >= nsplit) return;
    const int G = a.G;

    // ---- query fragments (rows = the G heads of this K/V head, zero-padded to 16)
    uint32_t qa[SL][4];
    {
        const uint16_t* qbase = a.q + (static_cast<size_t>(sq) * a.Hq + hkv * G) * D + t * (D / 4);
        uint4 q0[KU], q1[KU];
#pragma unroll
        for (int u = 0; u < KU; ++u) {
            q0[u] = g < G ? *reinterpret_cast<const uint4*>(qbase + static_cast<size_t>(g) * D + u * 8)
                          : make_uint4(0, 0, 0, 0);
            q1[u] = g + 8 < G
                        ? *reinterpret_cast<const uint4*>(qbase + static_cast<size_t>(g + 8) * D + u * 8)
                        : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int s = 0; s < SL; ++s) {
            const int u = s >> 1, w = (s & 1) * 2;
            qa[s][0] = word_of(q0[u], w);      // row g,   dims 4s+0,1 of the run
            qa[s][1] = word_of(q1[u], w);      // row g+8
            qa[s][2] = word_of(q0[u], w + 1);  // row g,   dims 4s+2,3
            qa[s][3] = word_of(q1[u], w + 1);  // row g+8
        }
    }

    // ---- issue every K/V load of this warp's blocks up front
    const int blk_first = split * kBlocksPerCta + warp * kBlocksPerWarp;
    uint4 kr[kBlocksPerWarp][2][KU];
    uint4 vr[kBlocksPerWarp][4][VU];
    bool valid[kBlocksPerWarp];
#pragma unroll
    for (int i = 0; i < kBlocksPerWarp; ++i) {
        const int blk = blk_first + i;
        int phys = -1;
        if (blk < nblk) {
            phys = a.block_table[static_cast<size_t>(sq) * a.max_blocks + blk];
            if (phys < 0 || phys >= a.num_blocks) {
                report_status(ATTN_ERR_BAD_INDEX);
                phys = -1;
            }
        }
        valid[i] = phys >= 0;
        if (valid[i]) {
            const size_t base = (static_cast<size_t>(phys) * a.Hkv + hkv) * kPageSize * D;
            const uint16_t* kb = a.kc + base;
            const uint16_t* vb = a.vc + base;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int u = 0; u < KU; ++u)
                    kr[i][nt][u] = ldg_stream(kb + (nt * 8 + g) * D + t * (D / 4) + u * 8);
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int tok = 2 * t + (r & 1) + (r >> 1) * 8;
#pragma unroll
                for (int u = 0; u < VU; ++u)
                    vr[i][r][u] = ldg_stream(vb + tok * D + g * (D / 8) + u * 8);
            }
        } else {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int u = 0; u < KU; ++u) kr[i][nt][u] = make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int u = 0; u < VU; ++u) vr[i][r][u] = make_uint4(0, 0, 0, 0);
        }
    }

    // ---- online softmax over this warp's blocks (rows g and g+8)
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float oacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) oacc[nt][0] = oacc[nt][1] = oacc[nt][2] = oacc[nt][3] = 0.f;
    const float c = a.scale_log2;

#pragma unroll
    for (int i = 0; i < kBlocksPerWarp; ++i) {
        if (!valid[i]) continue;  // warp-uniform
        const int tok0 = (blk_first + i) * kPageSize;
        float sc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
            for (int s = 0; s < SL; ++s) {
                const int u = s >> 1, w = (s & 1) * 2;
                mma16816<BF16>(sc[nt], qa[s], word_of(kr[i][nt][u], w), word_of(kr[i][nt][u], w + 1));
            }
        }
        // columns of the score tile: token tok0 + nt*8 + 2t + e
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
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            oacc[nt][0] *= al0;
            oacc[nt][1] *= al0;
            oacc[nt][2] *= al1;
            oacc[nt][3] *= al1;
            // column g of this n-tile is output dim g*D/8 + nt: element nt of each token run
            const int u = nt >> 3, wsel = (nt & 7) >> 1;
            const uint32_t sel = (nt & 1) ? 0x7632u : 0x5410u;
            const uint32_t b0 = __byte_perm(word_of(vr[i][0][u], wsel), word_of(vr[i][1][u], wsel), sel);
            const uint32_t b1 = __byte_perm(word_of(vr[i][2][u], wsel), word_of(vr[i][3][u], wsel), sel);
            mma16816<BF16>(oacc[nt], pa, b0, b1);
        }
    }
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

    // ---- reduce the warps of this CTA in shared memory
    if (t == 0) {
        sm_m[warp][g] = m0;
        sm_l[warp][g] = l0;
        sm_m[warp][g + 8] = m1;
        sm_l[warp][g + 8] = l1;
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        // accumulator columns 2t, 2t+1 are output dims 2t*D/8 + nt and (2t+1)*D/8 + nt
        sm_o[warp][g][(2 * t) * (D / 8) + nt] = oacc[nt][0];
        sm_o[warp][g][(2 * t + 1) * (D / 8) + nt] = oacc[nt][1];
        sm_o[warp][g + 8][(2 * t) * (D / 8) + nt] = oacc[nt][2];
        sm_o[warp][g + 8][(2 * t + 1) * (D / 8) + nt] = oacc[nt][3];
    }
    __syncthreads();

    const bool direct = nsplit == 1;
    const size_t unit = static_cast<size_t>(sq) * a.Hkv + hkv;
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int r = idx / D, d = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, sm_m[w][r]);
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kDecWarps; ++w) {
                const float f = ex2_approx(sm_m[w][r] - M);
                L += f * sm_l[w][r];
                O += f * sm_o[w][r][d];
            }
        }
        const float on = L > 0.f ? O / L : 0.f;
        const float lse2 = L > 0.f ? M + log2f(L) : -INFINITY;
        if (direct) {
            const size_t orow = static_cast<size_t>(sq) * a.Hq + hkv * G + r;
            a.out[orow * D + d] = static_cast<uint16_t>(BF16 ? __bfloat16_as_ushort(__float2bfloat16_rn(on))
                                                             : __half_as_ushort(__float2half_rn(on)));
            if (d == 0 && a.lse != nullptr) a.lse[orow] = lse2 * kLn2;
        } else {
            const size_t prow = (unit * a.max_splits + split) * G + r;
            a.ws_o[prow * D + d] = on;
            if (d == 0) a.ws_lse[prow] = lse2;
        }
    }
    if (direct) return;

    // ---- last CTA of this (sequence, head) merges the chunks
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const int prev = atomicAdd(&a.ws_count[unit], 1);
        sm_last = prev == nsplit - 1;
    }
    __syncthreads();
    if (!sm_last) return;
    __threadfence();
    // Row statistics: one warp per head row reduces the chunks' log2-sum-exp values in
    // parallel (32 loads in flight per warp, not a serial chain).
    const size_t lse0 = unit * a.max_splits * G;  // + sp * G + r
    for (int r = warp; r < G; r += kDecWarps) {
        float M = -INFINITY;
        for (int sp = lane; sp < nsplit; sp += 32) M = fmaxf(M, __ldcg(a.ws_lse + lse0 + sp * G + r));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float W = 0.f;
        if (M != -INFINITY)
            for (int sp = lane; sp < nsplit; sp += 32) W += ex2_approx(__ldcg(a.ws_lse + lse0 + sp * G + r) - M);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
        if (lane == 0) {
            sm_m[0][r] = M;
            sm_l[0][r] = W;
        }
    }
    __syncthreads();
    // Weighted sum of the chunks' normalised outputs, kCombineChunk chunks at a time
    // with their weights staged in shared memory (reusing the warp-reduction buffer).
    float* wbuf = &sm_o[0][0][0];
    constexpr int kCombineChunk = (kDecWarps * kMaxGroup * D) / kMaxGroup;  // chunks per pass
    float acc[(kMaxGroup * D + kDecWarps * 32 - 1) / (kDecWarps * 32)];
#pragma unroll
    for (int e = 0; e < (int)(sizeof(acc) / sizeof(float)); ++e) acc[e] = 0.f;
    for (int c0 = 0; c0 < nsplit; c0 += kCombineChunk) {
        const int cn = min(kCombineChunk, nsplit - c0);
        __syncthreads();
        for (int i = threadIdx.x; i < cn * G; i += blockDim.x) {
            const int sp = c0 + i / G, r = i % G;
            const float M = sm_m[0][r], W = sm_l[0][r];
            wbuf[i] = (M == -INFINITY) ? 0.f : ex2_approx(__ldcg(a.ws_lse + lse0 + sp * G + r) - M) / W;
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < (int)(sizeof(acc) / sizeof(float)); ++e) {
            const int idx = threadIdx.x + e * blockDim.x;
            if (idx < G * D) {
                const int r = idx / D;
                const float* src = a.ws_o + (lse0 + static_cast<size_t>(c0) * G) * D + idx;
                float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
                int i = 0;
                for (; i + 4 <= cn; i += 4) {
                    const float o0 = __ldcg(src + static_cast<size_t>(i) * G * D);
                    const float o1 = __ldcg(src + static_cast<size_t>(i + 1) * G * D);
                    const float o2 = __ldcg(src + static_cast<size_t>(i + 2) * G * D);
                    const float o3 = __ldcg(src + static_cast<size_t>(i + 3) * G * D);
                    s0 += wbuf[i * G + r] * o0;
                    s1 += wbuf[(i + 1) * G + r] * o1;
                    s2 += wbuf[(i + 2) * G + r] * o2;
                    s3 += wbuf[(i + 3) * G + r] * o3;
                }
                for (; i < cn; ++i) s0 += wbuf[i * G + r] * __ldcg(src + static_cast<size_t>(i) * G * D);
                acc[e] += (s0 + s1) + (s2 + s3);
            }
        }
    }
#pragma unroll
    for (int e = 0; e < (int)(sizeof(acc) / sizeof(float)); ++e) {
        const int idx = threadIdx.x + e * blockDim.x;
        if (idx < G * D) {
            const int r = idx / D, d = idx % D;
            const size_t orow = static_cast<size_t>(sq) * a.Hq + hkv * G + r;
            a.out[orow * D + d] = static_cast<uint16_t>(BF16 ? __bfloat16_as_ushort(__float2bfloat16_rn(acc[e]))
                                                             : __half_as_ushort(__float2half_rn(acc[e])));
            if (d == 0 && a.lse != nullptr) {
                const float M = sm_m[0][r], W = sm_l[0][r];
                a.lse[orow] = (M == -INFINITY || !(W > 0.f)) ? -INFINITY : (M + log2f(W)) * kLn2;
            }
        }
    }
    if (threadIdx.x == 0) a.ws_count[unit] = 0;  // leave the workspace as found
}

}  // namespace attn
