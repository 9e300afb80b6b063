// api.cu -- the C ABI declared in include/attn.h: argument validation, TMA tensor-map
// encoding and kernel launches. No per-call allocation, no synchronisation, no CPU
// fallback.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn.h"
#include "backward_sm100.cuh"
#include "paged_decode.cuh"
#include "prefill_sm100.cuh"

namespace {

using attn::PagedArgs;
using attn::PrefillArgs;
using attn::PrefillCfg;

constexpr int kMaxSeq = 1 << 22;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// ---------------------------------------------------------------- device check
// The kernels are built for sm_100a only: require compute capability 10.0.
attn_status_t check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_DEVICE;
    }
    static std::mutex mu;
    static int known[64] = {0};  // 0 unknown, 1 ok, -1 unsupported
    if (dev < 0 || dev >= 64) return ATTN_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(mu);
    if (known[dev] == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
            cudaGetLastError();
            return ATTN_ERR_DEVICE;
        }
        known[dev] = (major == 10 && minor == 0) ? 1 : -1;
    }
    return known[dev] == 1 ? ATTN_OK : ATTN_ERR_DEVICE;
}

// Streaming multiprocessors of the current device (0 if unknown).
int sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return 0;
    }
    static std::mutex mu;
    static int known[64] = {0};
    std::lock_guard<std::mutex> lock(mu);
    if (known[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        known[dev] = n;
    }
    return known[dev];
}

// When the usual grid (two query tiles per CTA) would leave SMs idle, each CTA takes one
// query tile and its two softmax warpgroups split the tile's key tiles between them
// (PrefillArgs::split_kv): twice the CTAs, each about half as long. Needs at least two
// key tiles to split.
void choose_split_kv(PrefillArgs& args, long long planes) {
    const int sms = sm_count();
    if (sms > 0 && planes * args.n_q_blocks < sms && args.Lk > attn::kBN) {
        args.split_kv = 1;
        args.n_q_blocks = (args.Lq + attn::kBM - 1) / attn::kBM;
    }
}

// ------------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        cudaGetLastError();
    });
    return fn;
}

// Element strides of a (batch, head, row) tensor with contiguous rows of D elements.
struct Strides {
    long long b, h, l;
};

Strides contiguous_strides(int H, int L, int D) {
    return {static_cast<long long>(H) * L * D, static_cast<long long>(L) * D, D};
}

// Caller strides (NULL: contiguous [B, H, L, D]). Each stride of a dimension longer than
// 1 must be positive, a multiple of 16 bytes (the TMA and vector-store unit) and below
// 2^38 elements; the stride of a dimension of length 1 is never used and is replaced.
attn_status_t take_strides(const attn_strides_t* in, int B, int H, int L, int D, Strides* out,
                           int elem_bytes = 2) {
    *out = contiguous_strides(H, L, D);
    if (in == nullptr) return ATTN_OK;
    const long long v[3] = {in->batch, in->head, in->seq};
    const long long ext[3] = {B, H, L};
    long long* dst[3] = {&out->b, &out->h, &out->l};
    for (int i = 0; i < 3; ++i) {
        if (ext[i] <= 1) continue;  // keep the contiguous value
        if (v[i] <= 0 || v[i] >= (1LL << 38)) return ATTN_ERR_INVALID;
        if ((v[i] * elem_bytes) % 16 != 0) return ATTN_ERR_MISALIGNED;
        *dst[i] = v[i];
    }
    return ATTN_OK;
}

// 4-D view (D, L, H, B) of a tensor with element strides (l, h, b) and contiguous D;
// box (128 bytes of D) x box_rows x 1 x 1 with 128-byte swizzle. Rows past L read as zero.
// u8: 8-bit elements (the bytes of e4m3 values).
bool encode_strided_map(CUtensorMap* tm, const void* base, bool bf16, int D, int L, int H, int B,
                        const Strides& st, int box_rows, bool u8 = false) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t el = u8 ? 1 : 2;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L),
                                static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(st.l) * el, static_cast<cuuint64_t>(st.h) * el,
                                   static_cast<cuuint64_t>(st.b) * el};
    // one 128-byte swizzle row per box row: 64 16-bit or 128 8-bit elements
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / el), static_cast<cuuint32_t>(box_rows), 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapDataType dt = u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                      : (bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                              : CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    return fn(tm, dt, 4,
              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Zeros the D elements of every (batch, head, row) of a strided output.
__global__ void zero_rows_kernel(uint16_t* out, long long sb, long long sh, long long sl, int H,
                                 int L, int D, long long rows) {
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long r = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; r < rows;
         r += stride) {
        const long long i = r % L, bh = r / L;
        uint4* p = reinterpret_cast<uint4*>(out + (bh / H) * sb + (bh % H) * sh + i * sl);
        for (int c = 0; c < D / 8; ++c) p[c] = make_uint4(0u, 0u, 0u, 0u);
    }
}

// ------------------------------------------------------------------ launchers
template <int D, bool BF16, int MASK, bool PAGED = false, bool FP8 = false>
attn_status_t launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const PrefillArgs& args, int planes, cudaStream_t stream) {
    auto kern = attn::prefill_fwd_kernel<D, BF16, MASK, PAGED, FP8>;
    constexpr int smem = PrefillCfg<D, FP8>::kSmemBytes;
    static std::once_flag once;
    static attn_status_t setup = ATTN_OK;
    std::call_once(once, [&] {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess) {
            setup = ATTN_ERR_CUDA;
            return;
        }
        // The kernel moves registers between warpgroups with setmaxnreg; refuse to
        // launch unless the registers it is launched with cover the split.
        cudaFuncAttributes fa{};
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) {
            setup = ATTN_ERR_CUDA;
            return;
        }
        if (static_cast<long long>(fa.numRegs) * attn::kPrefillThreads < attn::kRegBudget)
            setup = ATTN_ERR_UNSUPPORTED;
    });
    if (setup != ATTN_OK) {
        cudaGetLastError();
        return setup;
    }
    // Programmatic stream serialisation, as for the decode: the kernel may be launched
    // while the previous kernel of the stream finishes, and waits for it
    // (griddepcontrol.wait) before touching global memory.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(planes), static_cast<unsigned>(args.n_q_blocks));
    cfg.blockDim = dim3(attn::kPrefillThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, args) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
}

template <int D, bool BF16>
attn_status_t dispatch_mask(int mask, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, const PrefillArgs& args, int planes,
                            cudaStream_t stream) {
    if (mask == attn::kMaskCausal)
        return launch_prefill<D, BF16, attn::kMaskCausal>(tq, tk, tv, args, planes, stream);
    if (mask == attn::kMaskWindow)
        return launch_prefill<D, BF16, attn::kMaskWindow>(tq, tk, tv, args, planes, stream);
    return launch_prefill<D, BF16, attn::kMaskNone>(tq, tk, tv, args, planes, stream);
}

// 2-D view (D, rows) of a paged cache [num_blocks, H_kv, 16, D]: one row per token of
// each (block, head); box 64 x 16 (one block's rows, 64 columns) with 128-byte swizzle.
bool encode_cache_map(CUtensorMap* tm, const void* base, bool bf16, int D, long long rows) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(attn::kPageSize)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(tm, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D view (64, rows, D / 64) of a paged cache [num_blocks, H_kv, 16, D] for the decode:
// one box {64, 16, D / 64} is a whole block's 16 rows as D / 64 swizzled 16 x 64 tiles (the
// second coordinate steps over rows, the third over 64-column chunks), so one TMA load
// brings a block's K (or V).
bool encode_block_map(CUtensorMap* tm, const void* base, bool bf16, int D, long long rows) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(D / 64)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, 128};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(attn::kPageSize),
                               static_cast<cuuint32_t>(D / 64)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(tm, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The decode is launched with programmatic stream serialisation: it may start while the
// kernel before it in the stream finishes, and waits for that kernel (griddepcontrol.wait)
// before it reads or writes any global memory. Back-to-back decode calls then overlap one
// launch's start-up with the previous one's tail.
template <int D, bool BF16>
attn_status_t launch_paged(const CUtensorMap& tk, const CUtensorMap& tv, const PagedArgs& a,
                           int grid, cudaStream_t stream) {
    auto kern = attn::paged_decode_kernel<D, BF16>;
    constexpr int smem = attn::DecodeCfg<D>::kSmemBytes;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [&] {
        attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    });
    if (attr_err != cudaSuccess) return ATTN_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(attn::kDecThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tk, tv, a) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
}

// Dense forward with a band of visible keys: key j is visible to query i iff
// i' - left <= j <= i' + right with i' = i + (Lk - Lq); -1 leaves a side unbounded.
attn_status_t fwd_band(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                       int H_q, int H_kv, int Lq, int Lk, int D, float scale, int left,
                       int right, attn_dtype_t dtype, void* stream_,
                       const attn_strides_t* q_st = nullptr, const attn_strides_t* k_st = nullptr,
                       const attn_strides_t* v_st = nullptr,
                       const attn_strides_t* o_st = nullptr) {
    if (B < 0 || H_q < 1 || H_kv < 1 || Lq < 0 || Lk < 0) return ATTN_ERR_INVALID;
    if (H_q % H_kv != 0) return ATTN_ERR_INVALID;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (dtype != ATTN_F16 && dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
    if (Lq > kMaxSeq || Lk > kMaxSeq) return ATTN_ERR_UNSUPPORTED;
    const long long planes_q = static_cast<long long>(B) * H_q;
    if (planes_q > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    if (B == 0 || Lq == 0) return ATTN_OK;  // nothing to compute; pointers may be NULL
    // k and v may be NULL (empty tensors) only when there are no keys
    if (q == nullptr || out == nullptr || (Lk > 0 && (k == nullptr || v == nullptr)))
        return ATTN_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        (lse != nullptr && !aligned(lse, 4)))
        return ATTN_ERR_MISALIGNED;
    Strides sq, sk, sv, so;
    attn_status_t st = take_strides(q_st, B, H_q, Lq, D, &sq);
    if (st == ATTN_OK) st = take_strides(k_st, B, H_kv, Lk, D, &sk);
    if (st == ATTN_OK) st = take_strides(v_st, B, H_kv, Lk, D, &sv);
    if (st == ATTN_OK) st = take_strides(o_st, B, H_q, Lq, D, &so);
    if (st != ATTN_OK) return st;
    const bool out_contiguous = o_st == nullptr ||
                                (so.b == static_cast<long long>(H_q) * Lq * D &&
                                 so.h == static_cast<long long>(Lq) * D && so.l == D);
    const attn_status_t dev = check_device();
    if (dev != ATTN_OK) return dev;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const bool bf16 = dtype == ATTN_BF16;

    if (Lk == 0 && !out_contiguous) {  // no keys: O = 0 through the strides, lse = -inf
        const long long rows = planes_q * Lq;
        zero_rows_kernel<<<1184, 256, 0, stream>>>(static_cast<uint16_t*>(out), so.b, so.h, so.l,
                                                   H_q, Lq, D, rows);
        if (lse != nullptr)
            attn::fill_empty_kernel<true><<<1184, 256, 0, stream>>>(nullptr, lse, 0,
                                                                    static_cast<size_t>(rows));
        return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
    }
    if (Lk == 0) {  // no keys at all: O = 0, lse = -inf
        const size_t rows = static_cast<size_t>(planes_q) * Lq;
        if (bf16)
            attn::fill_empty_kernel<true><<<1184, 256, 0, stream>>>(static_cast<uint16_t*>(out), lse,
                                                                    rows * D, rows);
        else
            attn::fill_empty_kernel<false><<<1184, 256, 0, stream>>>(static_cast<uint16_t*>(out), lse,
                                                                     rows * D, rows);
        return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
    }

    alignas(64) CUtensorMap tq, tk, tv;
    if (!encode_strided_map(&tq, q, bf16, D, Lq, H_q, B, sq, attn::kBM) ||
        !encode_strided_map(&tk, k, bf16, D, Lk, H_kv, B, sk, attn::kBN) ||
        !encode_strided_map(&tv, v, bf16, D, Lk, H_kv, B, sv, attn::kBN))
        return ATTN_ERR_CUDA;

    PrefillArgs args{};
    args.out = out;
    args.out_sb = so.b;
    args.out_sh = so.h;
    args.out_sl = so.l;
    args.lse = lse;
    args.Hq = H_q;
    args.Hkv = H_kv;
    args.group = H_q / H_kv;
    args.Lq = Lq;
    args.Lk = Lk;
    args.n_q_blocks = (Lq + 2 * attn::kBM - 1) / (2 * attn::kBM);
    args.win_left = left;
    args.win_right = right;
    args.scale_log2 = scale * attn::kLog2e;
    const int planes = static_cast<int>(planes_q);
    const int m = (left < 0 && right < 0) ? attn::kMaskNone
                  : (left < 0 && right == 0) ? attn::kMaskCausal
                                             : attn::kMaskWindow;
    choose_split_kv(args, planes_q);
    if (D == 64)
        return bf16 ? dispatch_mask<64, true>(m, tq, tk, tv, args, planes, stream)
                    : dispatch_mask<64, false>(m, tq, tk, tv, args, planes, stream);
    return bf16 ? dispatch_mask<128, true>(m, tq, tk, tv, args, planes, stream)
                : dispatch_mask<128, false>(m, tq, tk, tv, args, planes, stream);
}

// ------------------------------------------------------------------ backward
template <int D, bool BF16, int MASK, int KIND>
attn_status_t launch_bwd(const CUtensorMap& tx, const CUtensorMap& tw, const CUtensorMap& ty,
                         const CUtensorMap& tz, const attn::BwdArgs& args, long long planes,
                         int tiles, cudaStream_t stream) {
    auto kern = attn::bwd_kernel<D, BF16, MASK, KIND>;
    constexpr int smem = attn::BwdCfg<D, KIND>::kSmemBytes;
    static std::once_flag once;
    static attn_status_t setup = ATTN_OK;
    std::call_once(once, [&] {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess) {
            setup = ATTN_ERR_CUDA;
            return;
        }
        // The kernel moves registers between warpgroups with setmaxnreg; refuse to
        // launch unless the registers it is launched with cover the split.
        cudaFuncAttributes fa{};
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) {
            setup = ATTN_ERR_CUDA;
            return;
        }
        if (static_cast<long long>(fa.numRegs) * attn::kBwdThreads < attn::kBwdRegBudget)
            setup = ATTN_ERR_UNSUPPORTED;
    });
    if (setup != ATTN_OK) {
        cudaGetLastError();
        return setup;
    }
    const dim3 grid(static_cast<unsigned>(planes), static_cast<unsigned>(tiles));
    kern<<<grid, attn::kBwdThreads, smem, stream>>>(tx, tw, ty, tz, args);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Strides of the backward pass's tensors: q, k, v, out, dout (dq, dk, dv go in the args).
struct BwdStrides {
    Strides q, k, v, o, d;
};

template <int D, bool BF16, int MASK>
attn_status_t run_bwd(const void* q, const void* k, const void* v, const void* out,
                      const void* dout, const float* lse, const attn::BwdArgs& args,
                      long long planes_q, long long planes_kv, const BwdStrides& st,
                      cudaStream_t stream) {
    // dK, dV: fixed K and V, streamed Q and dO; dQ: fixed Q and dO, streamed K and V
    // (128-row boxes throughout).
    static_assert(attn::kBwdFix == attn::kBwdSub, "one box height for fixed and streamed tiles");
    alignas(64) CUtensorMap tk, tv, tq, tdo;
    const int B = static_cast<int>(planes_q / args.Hq);
    if (!encode_strided_map(&tk, k, BF16, D, args.Lk, args.Hkv, B, st.k, attn::kBwdFix) ||
        !encode_strided_map(&tv, v, BF16, D, args.Lk, args.Hkv, B, st.v, attn::kBwdFix) ||
        !encode_strided_map(&tq, q, BF16, D, args.Lq, args.Hq, B, st.q, attn::kBwdFix) ||
        !encode_strided_map(&tdo, dout, BF16, D, args.Lq, args.Hq, B, st.d, attn::kBwdFix))
        return ATTN_ERR_CUDA;
    const long long rows_pad = planes_q * args.Lq_pad;  // a multiple of 128: whole warps
    const long long blocks = rows_pad * 8 / 256;
    if (blocks > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    attn::bwd_prep_kernel<D, BF16><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const uint16_t*>(out), static_cast<const uint16_t*>(dout), lse,
        const_cast<float*>(args.nlse2), const_cast<float*>(args.delta), args.Lq, args.Lq_pad,
        rows_pad, args.Hq, st.o.b, st.o.h, st.o.l, st.d.b, st.d.h, st.d.l);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    const attn_status_t rc = launch_bwd<D, BF16, MASK, attn::kDKDV>(
        tk, tv, tq, tdo, args, planes_kv, (args.Lk + attn::kBwdFix - 1) / attn::kBwdFix, stream);
    if (rc != ATTN_OK) return rc;
    return launch_bwd<D, BF16, MASK, attn::kDQ>(tq, tdo, tk, tv, args, planes_q,
                                                (args.Lq + attn::kBwdFix - 1) / attn::kBwdFix,
                                                stream);
}

template <int D, bool BF16>
attn_status_t dispatch_bwd(int mask, const void* q, const void* k, const void* v,
                           const void* out, const void* dout, const float* lse,
                           const attn::BwdArgs& args, long long planes_q, long long planes_kv,
                           const BwdStrides& st, cudaStream_t stream) {
    if (mask == attn::kMaskCausal)
        return run_bwd<D, BF16, attn::kMaskCausal>(q, k, v, out, dout, lse, args, planes_q,
                                                   planes_kv, st, stream);
    if (mask == attn::kMaskWindow)
        return run_bwd<D, BF16, attn::kMaskWindow>(q, k, v, out, dout, lse, args, planes_q,
                                                   planes_kv, st, stream);
    return run_bwd<D, BF16, attn::kMaskNone>(q, k, v, out, dout, lse, args, planes_q, planes_kv,
                                             st, stream);
}

size_t bwd_workspace_bytes(long long planes_q, int Lq) {
    const long long pad = (static_cast<long long>(Lq) + attn::kBwdFix - 1) / attn::kBwdFix *
                          attn::kBwdFix;
    return static_cast<size_t>(planes_q) * static_cast<size_t>(pad) * 2 * sizeof(float);
}

attn_status_t bwd_band(const void* q, const void* k, const void* v, const void* out,
                       const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                       int H_q, int H_kv, int Lq, int Lk, int D, float scale, int left, int right,
                       attn_dtype_t dtype, void* workspace, size_t workspace_bytes, void* stream_,
                       const attn_strides_t* const* strides = nullptr) {
    if (B < 0 || H_q < 1 || H_kv < 1 || Lq < 0 || Lk < 0) return ATTN_ERR_INVALID;
    if (H_q % H_kv != 0) return ATTN_ERR_INVALID;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (dtype != ATTN_F16 && dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
    if (Lq > kMaxSeq || Lk > kMaxSeq) return ATTN_ERR_UNSUPPORTED;
    const long long planes_q = static_cast<long long>(B) * H_q;
    const long long planes_kv = static_cast<long long>(B) * H_kv;
    if (planes_q > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    if (B == 0 || (Lq == 0 && Lk == 0)) return ATTN_OK;  // nothing to write
    const bool have_q = Lq > 0, have_k = Lk > 0;
    if ((have_q && (q == nullptr || dq == nullptr)) ||
        (have_k && (k == nullptr || v == nullptr || dk == nullptr || dv == nullptr)) ||
        (have_q && have_k && (out == nullptr || dout == nullptr || lse == nullptr)))
        return ATTN_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
        !aligned(lse, 4))
        return ATTN_ERR_MISALIGNED;
    // strides: q, k, v, out, dout, dq, dk, dv (NULL array or entry: contiguous)
    Strides sts[8];
    {
        const int hs[8] = {H_q, H_kv, H_kv, H_q, H_q, H_q, H_kv, H_kv};
        const int ls[8] = {Lq, Lk, Lk, Lq, Lq, Lq, Lk, Lk};
        for (int i = 0; i < 8; ++i) {
            const attn_status_t st = take_strides(strides ? strides[i] : nullptr, B, hs[i], ls[i], D,
                                                  &sts[i]);
            if (st != ATTN_OK) return st;
        }
    }
    if (have_q && have_k) {
        if (workspace == nullptr || workspace_bytes < bwd_workspace_bytes(planes_q, Lq))
            return ATTN_ERR_WORKSPACE;
        if (!aligned(workspace, 16)) return ATTN_ERR_MISALIGNED;
    }
    const attn_status_t dev = check_device();
    if (dev != ATTN_OK) return dev;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const bool bf16 = dtype == ATTN_BF16;
    if (!have_q || !have_k) {  // no queries: dK = dV = 0; no keys: dQ = 0
        if (!have_q) {
            zero_rows_kernel<<<1184, 256, 0, stream>>>(static_cast<uint16_t*>(dk), sts[6].b, sts[6].h,
                                                       sts[6].l, H_kv, Lk, D, planes_kv * Lk);
            zero_rows_kernel<<<1184, 256, 0, stream>>>(static_cast<uint16_t*>(dv), sts[7].b, sts[7].h,
                                                       sts[7].l, H_kv, Lk, D, planes_kv * Lk);
        } else {
            zero_rows_kernel<<<1184, 256, 0, stream>>>(static_cast<uint16_t*>(dq), sts[5].b, sts[5].h,
                                                       sts[5].l, H_q, Lq, D, planes_q * Lq);
        }
        return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
    }

    attn::BwdArgs args{};
    args.Lq_pad = static_cast<int>((static_cast<long long>(Lq) + attn::kBwdFix - 1) /
                                   attn::kBwdFix * attn::kBwdFix);
    float* ws = static_cast<float*>(workspace);
    args.nlse2 = ws;
    args.delta = ws + static_cast<size_t>(planes_q) * args.Lq_pad;
    args.dq = dq;
    args.dk = dk;
    args.dv = dv;
    const Strides* outs[3] = {&sts[5], &sts[6], &sts[7]};
    long long* dst[3] = {args.dq_s, args.dk_s, args.dv_s};
    for (int i = 0; i < 3; ++i) {
        dst[i][0] = outs[i]->b;
        dst[i][1] = outs[i]->h;
        dst[i][2] = outs[i]->l;
    }
    const BwdStrides bst{sts[0], sts[1], sts[2], sts[3], sts[4]};
    args.Hq = H_q;
    args.Hkv = H_kv;
    args.group = H_q / H_kv;
    args.Lq = Lq;
    args.Lk = Lk;
    args.win_left = left;
    args.win_right = right;
    args.scale = scale;
    args.scale_log2 = scale * attn::kLog2e;
    const int m = (left < 0 && right < 0) ? attn::kMaskNone
                  : (left < 0 && right == 0) ? attn::kMaskCausal
                                             : attn::kMaskWindow;
    if (D == 64)
        return bf16 ? dispatch_bwd<64, true>(m, q, k, v, out, dout, lse, args, planes_q, planes_kv, bst, stream)
                    : dispatch_bwd<64, false>(m, q, k, v, out, dout, lse, args, planes_q, planes_kv, bst, stream);
    return bf16 ? dispatch_bwd<128, true>(m, q, k, v, out, dout, lse, args, planes_q, planes_kv, bst, stream)
                : dispatch_bwd<128, false>(m, q, k, v, out, dout, lse, args, planes_q, planes_kv, bst, stream);
}

// Dense forward on e4m3 inputs (8-bit tensor-core products), bf16 output.
attn_status_t fwd_fp8(const void* q, const attn_strides_t* q_st, const void* k,
                      const attn_strides_t* k_st, const void* v, const attn_strides_t* v_st,
                      void* out, const attn_strides_t* o_st, float* lse, int B, int H_q, int H_kv,
                      int Lq, int Lk, int D, float scale, float descale_q, float descale_k,
                      float descale_v, int causal, void* stream_) {
    if (B < 0 || H_q < 1 || H_kv < 1 || Lq < 0 || Lk < 0) return ATTN_ERR_INVALID;
    if (H_q % H_kv != 0) return ATTN_ERR_INVALID;
    const float sc = scale * descale_q * descale_k;
    if (!std::isfinite(scale) || !(scale > 0.f) || !std::isfinite(sc) || !(sc > 0.f) ||
        !std::isfinite(descale_v) || !(descale_v > 0.f))
        return ATTN_ERR_INVALID;
    if (D != 128) return ATTN_ERR_UNSUPPORTED;
    if (Lq > kMaxSeq || Lk > kMaxSeq) return ATTN_ERR_UNSUPPORTED;
    const long long planes_q = static_cast<long long>(B) * H_q;
    if (planes_q > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    if (B == 0 || Lq == 0) return ATTN_OK;  // nothing to compute; pointers may be NULL
    if (q == nullptr || out == nullptr || (Lk > 0 && (k == nullptr || v == nullptr)))
        return ATTN_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        (lse != nullptr && !aligned(lse, 4)))
        return ATTN_ERR_MISALIGNED;
    Strides sq, sk, sv, so;
    attn_status_t st = take_strides(q_st, B, H_q, Lq, D, &sq, 1);
    if (st == ATTN_OK) st = take_strides(k_st, B, H_kv, Lk, D, &sk, 1);
    if (st == ATTN_OK) st = take_strides(v_st, B, H_kv, Lk, D, &sv, 1);
    if (st == ATTN_OK) st = take_strides(o_st, B, H_q, Lq, D, &so, 2);
    if (st != ATTN_OK) return st;
    const attn_status_t dev = check_device();
    if (dev != ATTN_OK) return dev;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (Lk == 0) {  // no keys: O = 0, lse = -inf
        const long long rows = planes_q * Lq;
        zero_rows_kernel<<<1184, 256, 0, stream>>>(static_cast<uint16_t*>(out), so.b, so.h, so.l,
                                                   H_q, Lq, D, rows);
        if (lse != nullptr)
            attn::fill_empty_kernel<true><<<1184, 256, 0, stream>>>(nullptr, lse, 0,
                                                                    static_cast<size_t>(rows));
        return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
    }
    alignas(64) CUtensorMap tq, tk, tv;
    if (!encode_strided_map(&tq, q, false, D, Lq, H_q, B, sq, attn::kBM, true) ||
        !encode_strided_map(&tk, k, false, D, Lk, H_kv, B, sk, attn::kBN, true) ||
        !encode_strided_map(&tv, v, false, D, Lk, H_kv, B, sv, attn::kBN, true))
        return ATTN_ERR_CUDA;
    PrefillArgs args{};
    args.out = out;
    args.out_sb = so.b;
    args.out_sh = so.h;
    args.out_sl = so.l;
    args.lse = lse;
    args.Hq = H_q;
    args.Hkv = H_kv;
    args.group = H_q / H_kv;
    args.Lq = Lq;
    args.Lk = Lk;
    args.n_q_blocks = (Lq + 2 * attn::kBM - 1) / (2 * attn::kBM);
    args.win_left = -1;
    args.win_right = causal ? 0 : -1;
    args.scale_log2 = sc * attn::kLog2e;
    args.o_scale = descale_v;
    choose_split_kv(args, planes_q);
    const int planes = static_cast<int>(planes_q);
    return causal ? launch_prefill<128, true, attn::kMaskCausal, false, true>(tq, tk, tv, args, planes, stream)
                  : launch_prefill<128, true, attn::kMaskNone, false, true>(tq, tk, tv, args, planes, stream);
}

// Prefill over a paged cache: the dense forward kernel with its K/V tiles gathered
// block by block through the table.
attn_status_t paged_prefill(const void* q, const attn_strides_t* q_st, const void* k_cache,
                            const void* v_cache, const int32_t* block_table,
                            const int32_t* seq_lens, const int32_t* q_lens, int block_size,
                            void* out, const attn_strides_t* o_st, float* lse, int num_seqs,
                            int H_q, int H_kv, int Lq, int D, int max_blocks, int num_blocks,
                            float scale, int causal, attn_dtype_t dtype, void* stream_) {
    if (num_seqs < 0 || H_q < 1 || H_kv < 1 || Lq < 0 || max_blocks < 0 || num_blocks < 0)
        return ATTN_ERR_INVALID;
    if (H_q % H_kv != 0) return ATTN_ERR_INVALID;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID;
    if (block_size != attn::kPageSize) return ATTN_ERR_UNSUPPORTED;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (dtype != ATTN_F16 && dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
    if (Lq > kMaxSeq || static_cast<long long>(max_blocks) * attn::kPageSize > kMaxSeq)
        return ATTN_ERR_UNSUPPORTED;
    const long long planes_q = static_cast<long long>(num_seqs) * H_q;
    if (planes_q > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    if (num_seqs == 0 || Lq == 0) return ATTN_OK;  // nothing to write; pointers may be NULL
    if (q == nullptr || out == nullptr || seq_lens == nullptr ||
        (max_blocks > 0 && (block_table == nullptr || k_cache == nullptr || v_cache == nullptr)))
        return ATTN_ERR_INVALID;
    if (max_blocks > 0 && num_blocks < 1) return ATTN_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_table, 4) || !aligned(seq_lens, 4) || !aligned(q_lens, 4) ||
        (lse != nullptr && !aligned(lse, 4)))
        return ATTN_ERR_MISALIGNED;
    Strides sq, so;
    attn_status_t st = take_strides(q_st, num_seqs, H_q, Lq, D, &sq);
    if (st == ATTN_OK) st = take_strides(o_st, num_seqs, H_q, Lq, D, &so);
    if (st != ATTN_OK) return st;
    const attn_status_t dev = check_device();
    if (dev != ATTN_OK) return dev;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const bool bf16 = dtype == ATTN_BF16;
    if (max_blocks == 0) {  // every sequence is empty: O = 0, lse = -inf
        const long long rows = planes_q * Lq;
        zero_rows_kernel<<<1184, 256, 0, stream>>>(static_cast<uint16_t*>(out), so.b, so.h, so.l,
                                                   H_q, Lq, D, rows);
        if (lse != nullptr)
            attn::fill_empty_kernel<true><<<1184, 256, 0, stream>>>(nullptr, lse, 0,
                                                                    static_cast<size_t>(rows));
        return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
    }

    alignas(64) CUtensorMap tq, tk, tv;
    const long long cache_rows = static_cast<long long>(num_blocks) * H_kv * attn::kPageSize;
    if (!encode_strided_map(&tq, q, bf16, D, Lq, H_q, num_seqs, sq, attn::kBM) ||
        !encode_cache_map(&tk, k_cache, bf16, D, cache_rows) ||
        !encode_cache_map(&tv, v_cache, bf16, D, cache_rows))
        return ATTN_ERR_CUDA;
    PrefillArgs args{};
    args.out = out;
    args.out_sb = so.b;
    args.out_sh = so.h;
    args.out_sl = so.l;
    args.lse = lse;
    args.Hq = H_q;
    args.Hkv = H_kv;
    args.group = H_q / H_kv;
    args.Lq = Lq;
    args.Lk = max_blocks * attn::kPageSize;  // replaced per sequence by seq_lens[b]
    args.n_q_blocks = (Lq + 2 * attn::kBM - 1) / (2 * attn::kBM);
    args.win_left = -1;
    args.win_right = causal ? 0 : -1;
    args.scale_log2 = scale * attn::kLog2e;
    args.block_table = block_table;
    args.seq_lens = seq_lens;
    args.q_lens = q_lens;
    args.max_blocks = max_blocks;
    args.num_blocks = num_blocks;
    const int planes = static_cast<int>(planes_q);
    if (D == 64) {
        if (bf16)
            return causal ? launch_prefill<64, true, attn::kMaskCausal, true>(tq, tk, tv, args, planes, stream)
                          : launch_prefill<64, true, attn::kMaskNone, true>(tq, tk, tv, args, planes, stream);
        return causal ? launch_prefill<64, false, attn::kMaskCausal, true>(tq, tk, tv, args, planes, stream)
                      : launch_prefill<64, false, attn::kMaskNone, true>(tq, tk, tv, args, planes, stream);
    }
    if (bf16)
        return causal ? launch_prefill<128, true, attn::kMaskCausal, true>(tq, tk, tv, args, planes, stream)
                      : launch_prefill<128, true, attn::kMaskNone, true>(tq, tk, tv, args, planes, stream);
    return causal ? launch_prefill<128, false, attn::kMaskCausal, true>(tq, tk, tv, args, planes, stream)
                  : launch_prefill<128, false, attn::kMaskNone, true>(tq, tk, tv, args, planes, stream);
}

// Decode tensor maps of paged caches (encode_block_map), cached by what they encode (base address, rows, D,
// dtype, device): a map holds nothing else, so a cached map is exact even if the
// memory behind an address was freed and reallocated with the same extent.
struct CacheMapKey {
    const void* base;
    long long rows;
    int D, bf16, dev;
    bool operator==(const CacheMapKey& o) const {
        return base == o.base && rows == o.rows && D == o.D && bf16 == o.bf16 && dev == o.dev;
    }
};

bool cached_cache_map(CUtensorMap* tm, const void* base, bool bf16, int D, long long rows) {
    constexpr int kSlots = 16;
    static std::mutex mu;
    static CacheMapKey keys[kSlots];
    alignas(64) static CUtensorMap maps[kSlots];
    static int used = 0, next = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    const CacheMapKey key{base, rows, D, bf16 ? 1 : 0, dev};
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (keys[i] == key) {
            *tm = maps[i];
            return true;
        }
    if (!encode_block_map(tm, base, bf16, D, rows)) return false;
    const int slot = used < kSlots ? used++ : (next++ % kSlots);
    keys[slot] = key;
    maps[slot] = *tm;
    return true;
}

// A paged-decode call: paged_prepare checks the arguments and fills in the kernel's
// arguments, paged_encode checks the device and encodes the cache tensor maps, and
// paged_launch enqueues the kernel. Nothing is enqueued before paged_launch.
struct PagedCall {
    bool empty = false;  // num_seqs == 0: nothing to launch
    int D = 0;
    bool bf16 = false;
    attn::PagedLayout L{};
    const void* k_cache = nullptr;
    const void* v_cache = nullptr;
    long long rows = 1;  // cache rows the tensor maps span
    alignas(64) CUtensorMap tk, tv;
    PagedArgs a{};
};

attn_status_t paged_prepare(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_table, const int32_t* seq_lens, int block_size,
                            void* out, float* lse, int num_seqs, int H_q, int H_kv, int D,
                            int max_blocks_per_seq, int num_blocks, float scale,
                            attn_dtype_t dtype, PagedCall* c) {
    if (num_seqs < 0 || H_q < 1 || H_kv < 1 || max_blocks_per_seq < 0 || num_blocks < 0)
        return ATTN_ERR_INVALID;
    if (num_seqs == 0) {  // nothing to compute; pointers may be NULL
        c->empty = true;
        return ATTN_OK;
    }
    if (q == nullptr || k_cache == nullptr || v_cache == nullptr || block_table == nullptr ||
        seq_lens == nullptr || out == nullptr)
        return ATTN_ERR_INVALID;
    if (H_q % H_kv != 0) return ATTN_ERR_INVALID;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID;
    if (block_size != attn::kPageSize) return ATTN_ERR_UNSUPPORTED;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (dtype != ATTN_F16 && dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
    if (H_q / H_kv > attn::kMaxGroup) return ATTN_ERR_UNSUPPORTED;
    if (static_cast<long long>(max_blocks_per_seq) * attn::kPageSize > kMaxSeq || num_seqs > 65535 ||
        H_kv > 65535)
        return ATTN_ERR_UNSUPPORTED;
    const long long rows = static_cast<long long>(num_blocks) * H_kv * attn::kPageSize;
    if (rows > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
        !aligned(block_table, 4) || !aligned(seq_lens, 4) || (lse != nullptr && !aligned(lse, 4)))
        return ATTN_ERR_MISALIGNED;
    c->D = D;
    c->bf16 = dtype == ATTN_BF16;
    c->L = attn::paged_layout(num_seqs, H_q, H_kv, D, max_blocks_per_seq);
    c->k_cache = k_cache;
    c->v_cache = v_cache;
    c->rows = rows > 0 ? rows : 1;
    PagedArgs& a = c->a;
    a.q = static_cast<const uint16_t*>(q);
    a.block_table = block_table;
    a.seq_lens = seq_lens;
    a.out = static_cast<uint16_t*>(out);
    a.lse = lse;
    a.num_seqs = num_seqs;
    a.Hq = H_q;
    a.Hkv = H_kv;
    a.G = H_q / H_kv;
    a.max_blocks = max_blocks_per_seq;
    a.num_blocks = num_blocks;
    a.balanced = c->L.balanced;
    a.scale_log2 = scale * attn::kLog2e;
    return ATTN_OK;
}

attn_status_t paged_encode(PagedCall& c) {
    const attn_status_t dev = check_device();
    if (dev != ATTN_OK) return dev;
    if (!cached_cache_map(&c.tk, c.k_cache, c.bf16, c.D, c.rows) ||
        !cached_cache_map(&c.tv, c.v_cache, c.bf16, c.D, c.rows))
        return ATTN_ERR_CUDA;
    return ATTN_OK;
}

// Launches a prepared, encoded call with its split-KV scratch at `workspace` (unused
// when the layout needs none).
attn_status_t paged_launch(PagedCall& c, void* workspace, cudaStream_t stream) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const attn::PagedLayout& L = c.L;
    c.a.ws_count = L.total ? reinterpret_cast<int*>(ws + L.count_off) : nullptr;
    c.a.ws_lse = L.total ? reinterpret_cast<float*>(ws + L.lse_off) : nullptr;
    c.a.ws_o = L.total ? reinterpret_cast<float*>(ws + L.o_off) : nullptr;
    if (c.D == 64)
        return c.bf16 ? launch_paged<64, true>(c.tk, c.tv, c.a, L.grid, stream)
                      : launch_paged<64, false>(c.tk, c.tv, c.a, L.grid, stream);
    return c.bf16 ? launch_paged<128, true>(c.tk, c.tv, c.a, L.grid, stream)
                  : launch_paged<128, false>(c.tk, c.tv, c.a, L.grid, stream);
}

}  // namespace

extern "C" {

attn_status_t attn_fwd_fp8(const void* q, const attn_strides_t* q_strides, const void* k,
                           const attn_strides_t* k_strides, const void* v,
                           const attn_strides_t* v_strides, void* out,
                           const attn_strides_t* out_strides, float* lse, int B, int H_q, int H_kv,
                           int Lq, int Lk, int D, float scale, float descale_q, float descale_k,
                           float descale_v, int causal, void* stream) {
    return fwd_fp8(q, q_strides, k, k_strides, v, v_strides, out, out_strides, lse, B, H_q, H_kv,
                   Lq, Lk, D, scale, descale_q, descale_k, descale_v, causal, stream);
}

attn_status_t attn_fwd_paged_prefill(const void* q, const attn_strides_t* q_strides,
                                     const void* k_cache, const void* v_cache,
                                     const int32_t* block_table, const int32_t* seq_lens,
                                     const int32_t* q_lens, int block_size, void* out,
                                     const attn_strides_t* out_strides, float* lse, int num_seqs,
                                     int H_q, int H_kv, int Lq, int D, int max_blocks_per_seq,
                                     int num_blocks, float scale, int causal, attn_dtype_t dtype,
                                     void* stream) {
    return paged_prefill(q, q_strides, k_cache, v_cache, block_table, seq_lens, q_lens,
                         block_size, out, out_strides, lse, num_seqs, H_q, H_kv, Lq, D,
                         max_blocks_per_seq, num_blocks, scale, causal, dtype, stream);
}

size_t attn_bwd_workspace_size(int B, int H_q, int Lq) {
    if (B < 0 || H_q < 1 || Lq < 0) return 0;
    return bwd_workspace_bytes(static_cast<long long>(B) * H_q, Lq);
}

attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* out,
                       const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                       int H_q, int H_kv, int Lq, int Lk, int D, float scale, int causal,
                       attn_dtype_t dtype, void* workspace, size_t workspace_bytes, void* stream) {
    return bwd_band(q, k, v, out, dout, lse, dq, dk, dv, B, H_q, H_kv, Lq, Lk, D, scale, -1,
                    causal ? 0 : -1, dtype, workspace, workspace_bytes, stream);
}

attn_status_t attn_bwd_strided(const void* q, const attn_strides_t* q_strides, const void* k,
                               const attn_strides_t* k_strides, const void* v,
                               const attn_strides_t* v_strides, const void* out,
                               const attn_strides_t* out_strides, const void* dout,
                               const attn_strides_t* dout_strides, const float* lse, void* dq,
                               const attn_strides_t* dq_strides, void* dk,
                               const attn_strides_t* dk_strides, void* dv,
                               const attn_strides_t* dv_strides, int B, int H_q, int H_kv, int Lq,
                               int Lk, int D, float scale, int causal, int window_left,
                               int window_right, attn_dtype_t dtype, void* workspace,
                               size_t workspace_bytes, void* stream) {
    if (window_left < -1 || window_right < -1) return ATTN_ERR_INVALID;
    const attn_strides_t* st[8] = {q_strides, k_strides,  v_strides,  out_strides,
                                   dout_strides, dq_strides, dk_strides, dv_strides};
    return bwd_band(q, k, v, out, dout, lse, dq, dk, dv, B, H_q, H_kv, Lq, Lk, D, scale,
                    window_left, causal ? 0 : window_right, dtype, workspace, workspace_bytes,
                    stream, st);
}

attn_status_t attn_bwd_window(const void* q, const void* k, const void* v, const void* out,
                              const void* dout, const float* lse, void* dq, void* dk, void* dv,
                              int B, int H_q, int H_kv, int Lq, int Lk, int D, float scale,
                              int causal, int window_left, int window_right, attn_dtype_t dtype,
                              void* workspace, size_t workspace_bytes, void* stream) {
    if (window_left < -1 || window_right < -1) return ATTN_ERR_INVALID;
    return bwd_band(q, k, v, out, dout, lse, dq, dk, dv, B, H_q, H_kv, Lq, Lk, D, scale,
                    window_left, causal ? 0 : window_right, dtype, workspace, workspace_bytes,
                    stream);
}


attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                       int H_q, int H_kv, int Lq, int Lk, int D, float scale, int causal,
                       attn_dtype_t dtype, void* stream) {
    return fwd_band(q, k, v, out, lse, B, H_q, H_kv, Lq, Lk, D, scale, -1, causal ? 0 : -1, dtype,
                    stream);
}

attn_status_t attn_fwd_window(const void* q, const void* k, const void* v, void* out, float* lse,
                              int B, int H_q, int H_kv, int Lq, int Lk, int D, float scale,
                              int causal, int window_left, int window_right, attn_dtype_t dtype,
                              void* stream) {
    if (window_left < -1 || window_right < -1) return ATTN_ERR_INVALID;
    return fwd_band(q, k, v, out, lse, B, H_q, H_kv, Lq, Lk, D, scale, window_left,
                    causal ? 0 : window_right, dtype, stream);
}

attn_status_t attn_fwd_strided(const void* q, const attn_strides_t* q_strides, const void* k,
                               const attn_strides_t* k_strides, const void* v,
                               const attn_strides_t* v_strides, void* out,
                               const attn_strides_t* out_strides, float* lse, int B, int H_q,
                               int H_kv, int Lq, int Lk, int D, float scale, int causal,
                               int window_left, int window_right, attn_dtype_t dtype,
                               void* stream) {
    if (window_left < -1 || window_right < -1) return ATTN_ERR_INVALID;
    return fwd_band(q, k, v, out, lse, B, H_q, H_kv, Lq, Lk, D, scale, window_left,
                    causal ? 0 : window_right, dtype, stream, q_strides, k_strides, v_strides,
                    out_strides);
}

size_t attn_paged_workspace_size(int num_seqs, int H_q, int H_kv, int D, int max_blocks_per_seq,
                                 int block_size) {
    if (num_seqs < 0 || H_q < 1 || H_kv < 1 || H_q % H_kv != 0 || (D != 64 && D != 128) ||
        max_blocks_per_seq < 0 || block_size != attn::kPageSize)
        return 0;
    return attn::paged_layout(num_seqs, H_q, H_kv, D, max_blocks_per_seq).total;
}

attn_status_t attn_fwd_paged(const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_table, const int32_t* seq_lens, int block_size,
                             void* out, float* lse, int num_seqs, int H_q, int H_kv, int D,
                             int max_blocks_per_seq, int num_blocks, float scale,
                             attn_dtype_t dtype, void* workspace, size_t workspace_bytes,
                             void* stream_) {
    PagedCall c;
    const attn_status_t st =
        paged_prepare(q, k_cache, v_cache, block_table, seq_lens, block_size, out, lse, num_seqs,
                      H_q, H_kv, D, max_blocks_per_seq, num_blocks, scale, dtype, &c);
    if (st != ATTN_OK || c.empty) return st;
    if (c.L.total > 0 && (workspace == nullptr || workspace_bytes < c.L.total))
        return ATTN_ERR_WORKSPACE;
    if (workspace != nullptr && !aligned(workspace, 256)) return ATTN_ERR_MISALIGNED;
    const attn_status_t enc = paged_encode(c);
    if (enc != ATTN_OK) return enc;
    return paged_launch(c, workspace, static_cast<cudaStream_t>(stream_));
}

// ------------------------------------------------------------ failure detection
namespace attn {
// One CTA waits on an mbarrier that nothing ever completes, through the same bounded
// wait the attention kernels use: the wait must give up, report ATTN_ERR_TIMEOUT in the
// device status word and let the kernel return.
__global__ void selftest_wait_kernel() {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) wait_phase(smem_u32(&bar), 0, &abort_flag);
}
}  // namespace attn

extern "C" attn_status_t attn_selftest_bounded_wait(void* stream_) {
    const attn_status_t dev = check_device();
    if (dev != ATTN_OK) return dev;
    attn::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream_)>>>();
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// ----------------------------------------------------------- no-allocation decode
// Scratch for attn_fwd_paged_noalloc: a fixed 4 MiB array in this library's own device
// module. Every GPU that loads the library holds it until the process exits. In host
// code the name g_paged_scratch is only a host-side stand-in for the device array, so
// it is never passed to a kernel; its device address is looked up once per device.
}  // extern "C"
namespace {
constexpr size_t kStaticScratchBytes = static_cast<size_t>(4) << 20;
static __device__ __align__(256) uint8_t g_paged_scratch[kStaticScratchBytes];

// The calling thread's current CUDA context (nullptr if none or if the driver entry
// point is unavailable).
CUcontext current_context() {
    using CtxGetCurrentFn = CUresult (*)(CUcontext*);
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
        cudaGetLastError();
    });
    CUcontext ctx = nullptr;
    if (fn == nullptr || fn(&ctx) != CUDA_SUCCESS) return nullptr;
    return ctx;
}

// Device address of g_paged_scratch in the current device's context. It is looked up
// (cudaGetSymbolAddress) by the first call made with that device current, and again
// whenever the device's current context differs from the one it was looked up in
// (after a device reset the module is loaded anew, at a new address).
void* static_scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return nullptr;
    }
    static std::mutex mu;
    static void* addr[64] = {nullptr};
    static CUcontext ctx_of[64] = {nullptr};
    std::lock_guard<std::mutex> lock(mu);
    const CUcontext ctx = current_context();
    if (addr[dev] == nullptr || ctx == nullptr || ctx != ctx_of[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_paged_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        addr[dev] = p;
        ctx_of[dev] = current_context();  // the lookup made the device's context current
    }
    return addr[dev];
}
}  // namespace
extern "C" {

attn_status_t attn_fwd_paged_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* block_table, const int32_t* seq_lens,
                                     int block_size, void* out, float* lse, int num_seqs,
                                     int H_q, int H_kv, int D, int max_blocks_per_seq,
                                     int num_blocks, float scale, attn_dtype_t dtype,
                                     void* stream_) {
    // Every check and the tensor-map encoding run first, so that a rejected call
    // enqueues nothing (not even the counter clear).
    PagedCall c;
    const attn_status_t st =
        paged_prepare(q, k_cache, v_cache, block_table, seq_lens, block_size, out, lse, num_seqs,
                      H_q, H_kv, D, max_blocks_per_seq, num_blocks, scale, dtype, &c);
    if (st != ATTN_OK || c.empty) return st;
    if (c.L.total > kStaticScratchBytes) return ATTN_ERR_SCRATCH_LIMIT;
    const attn_status_t enc = paged_encode(c);
    if (enc != ATTN_OK) return enc;
    void* scratch = nullptr;
    if (c.L.total > 0) {
        scratch = static_scratch_address();
        if (scratch == nullptr) return ATTN_ERR_CUDA;
    }
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (c.L.total > 0) {
        // The completion counters must start at zero; the partial results need not.
        const size_t counters = static_cast<size_t>(num_seqs) * H_kv * sizeof(int);
        if (cudaMemsetAsync(static_cast<uint8_t*>(scratch) + c.L.count_off, 0, counters, stream) !=
            cudaSuccess) {
            cudaGetLastError();
            return ATTN_ERR_CUDA;
        }
    }
    return paged_launch(c, scratch, stream);
}

attn_status_t attn_selftest_fill_noalloc_scratch(int byte_value, void* stream_) {
    const attn_status_t dev = check_device();
    if (dev != ATTN_OK) return dev;
    void* scratch = static_scratch_address();
    if (scratch == nullptr) return ATTN_ERR_CUDA;
    if (cudaMemsetAsync(scratch, byte_value & 0xFF, kStaticScratchBytes,
                        static_cast<cudaStream_t>(stream_)) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
}

const char* attn_error_string(attn_status_t status) {
    switch (status) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_INVALID: return "invalid argument";
        case ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
        case ATTN_ERR_MISALIGNED: return "misaligned pointer";
        case ATTN_ERR_DEVICE: return "no supported device (compute capability 10.0 required)";
        case ATTN_ERR_CUDA: return "CUDA call failed";
        case ATTN_ERR_TIMEOUT: return "device-side bounded wait expired";
        case ATTN_ERR_WORKSPACE: return "workspace missing or too small";
        case ATTN_ERR_BAD_INDEX: return "block-table entry or sequence length out of range";
        case ATTN_ERR_SCRATCH_LIMIT:
            return "problem needs more scratch than the library's fixed 4 MiB device buffer";
    }
    return "unknown status";
}

attn_status_t attn_get_device_status(void* stream_) {
    const attn_status_t dev = check_device();
    if (dev != ATTN_OK) return dev;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    int host = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbolAsync(&host, attn::g_attn_status, sizeof(int), 0,
                                  cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaMemcpyToSymbolAsync(attn::g_attn_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice,
                                stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    return static_cast<attn_status_t>(host);
}

}  // extern "C"
