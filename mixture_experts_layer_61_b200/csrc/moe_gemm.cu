// moe_gemm.cu -- host side of the tcgen05 grouped GEMM: TMA tensor maps,
// variant dispatch (operand dtype, SwiGLU or plain epilogue, token-tile cap)
// and the persistent launch.
#include <mutex>

#include "moe_ffn_stream.cuh"
#include "moe_gemm.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        cudaGetLastError();
    });
    return fn;
}

// [rows, kdim] row-major, box = box_rows x row_bytes (128 or 64) with the
// swizzle of that width, out-of-range elements read as zero.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int elt_bytes, const void* base, long long rows, int kdim,
              int box_rows, int row_bytes = 128) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(kdim), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(kdim) * elt_bytes};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(row_bytes / elt_bytes), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <typename T, typename OutT, int kEpi, int kMaxN, int kCta = 1>
int launch_variant(const GemmLaunch& L, const GemmCtl& ctl, int num_sms, cudaStream_t stream) {
    using C = GemmCfg<T, kEpi, kMaxN, kCta>;
    auto kern = moe_gemm_kernel<T, OutT, kEpi, kMaxN, kCta>;
    if (kCta == 2 && (num_sms & 1)) return -1;
    static int grid_blocks = 0;  // per instantiation: CTAs that can be resident at once
    static bool attr_done = false;  // per instantiation
    if (!attr_done) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess) {
            cudaGetLastError();
            return -3;
        }
        grid_blocks = num_sms;
        if (kCta > 1) {
            // pairs must sit in one GPC: size the persistent grid by the clusters that fit
            cudaLaunchConfig_t oc = {};
            oc.gridDim = dim3(num_sms);
            oc.blockDim = dim3(kGemmThreads);
            oc.dynamicSmemBytes = C::kSmemBytes;
            cudaLaunchAttribute ca;
            ca.id = cudaLaunchAttributeClusterDimension;
            ca.val.clusterDim.x = kCta;
            ca.val.clusterDim.y = 1;
            ca.val.clusterDim.z = 1;
            oc.attrs = &ca;
            oc.numAttrs = 1;
            int nclusters = 0;
            if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &oc) != cudaSuccess || nclusters <= 0) {
                cudaGetLastError();
                return -3;
            }
            grid_blocks = nclusters * kCta < num_sms ? nclusters * kCta : num_sms;
        }
        attr_done = true;
    }
    CUtensorMap tm_w, tm_x, tm_x64, tm_xbig;
    constexpr int rb = C::kRowBytes;
    if (!make_map(&tm_w, Elt<T>::kTma, Elt<T>::kBytes, L.w, L.w_rows, L.kdim, 128, rb)) return -3;
    if (!make_map(&tm_x, Elt<T>::kTma, Elt<T>::kBytes, L.x, L.x_rows, L.kdim, C::kXBoxRows, rb)) return -3;
    if (!make_map(&tm_x64, Elt<T>::kTma, Elt<T>::kBytes, L.x, L.x_rows, L.kdim, C::kXBoxMid, rb)) return -3;
    if (!make_map(&tm_xbig, Elt<T>::kTma, Elt<T>::kBytes, L.x, L.x_rows, L.kdim, kMaxN / kCta, rb)) return -3;
    GemmParams p;
    p.seg_offsets = L.seg_offsets;
    p.n_groups = L.n_groups;
    p.seg_rows = L.seg_rows;
    p.n_out = L.n_out;
    p.kdim = L.kdim;
    p.w_group_stride = L.w_group_stride;
    p.up_offset = L.up_offset;
    p.out = L.out;
    p.out_ld = L.out_ld;
    p.counters = ctl.counters;
    p.partials = ctl.partials;
    p.status = ctl.status;
    p.wait_limit_ns = wait_limit_ns();
    p.withhold_first_load = take_withhold_flag();
    p.sk_min_units = 4;
    p.max_split = L.max_split > 0 ? L.max_split : 4;
    p.split_tail = split_tail_mode();
    int grid = grid_blocks;
    if (L.sms > 0 && L.sms < grid) grid = L.sms >= 2 * kCta ? L.sms - L.sms % kCta : kCta;
    cudaError_t e = launch_kernel_cluster(kern, dim3(grid), dim3(kGemmThreads), C::kSmemBytes, stream, kCta,
                                          tm_w, tm_x, tm_x64, tm_xbig, p);
    count_launch();
    if (e != cudaSuccess) cudaGetLastError();
    return e == cudaSuccess ? 0 : -3;
}

template <typename T, typename OutT, int kEpi>
int dispatch_n(const GemmLaunch& L, const GemmCtl& ctl, int num_sms, cudaStream_t s) {
    switch (L.max_n) {
        case 32: return launch_variant<T, OutT, kEpi, 32>(L, ctl, num_sms, s);
        case 64: return launch_variant<T, OutT, kEpi, 64>(L, ctl, num_sms, s);
        case 128: return launch_variant<T, OutT, kEpi, 128>(L, ctl, num_sms, s);
        case 256: return launch_variant<T, OutT, kEpi, 256>(L, ctl, num_sms, s);
        default: return -1;
    }
}

bool g_cta_pairs = true;

// Plain epilogue: 256-feature tiles (two weight tiles per stage, halving the
// token-tile bytes per flop) once token tiles are large; 128 otherwise.
template <typename T, typename OutT>
int dispatch_plain(const GemmLaunch& L, const GemmCtl& ctl, int num_sms, cudaStream_t s) {
    if (L.max_n == 128 && L.n_out >= 256) return launch_variant<T, OutT, kEpiWide, 128>(L, ctl, num_sms, s);
    if (L.max_n == 256 && L.n_out >= 256) return launch_variant<T, OutT, kEpiWide, 256>(L, ctl, num_sms, s);
    return dispatch_n<T, OutT, kEpiPlain>(L, ctl, num_sms, s);
}

// bf16 at the 256-token cap: CTA pairs (2-SM MMA, M = 256 weight rows per
// pair, each CTA staging half of the 256 token rows); without SwiGLU a pair
// takes 512 output features (wide) when there are that many.
int dispatch_bf16(const GemmLaunch& L, const GemmCtl& ctl, int num_sms, cudaStream_t s) {
    using bf = __nv_bfloat16;
    if (g_cta_pairs && L.max_n == 256 && !L.out_f32 && (num_sms % 2) == 0) {
        if (L.swiglu) return launch_variant<bf, bf, kEpiSwiGLU, 256, 2>(L, ctl, num_sms, s);
        if (L.n_out >= 512) return launch_variant<bf, bf, kEpiWide, 256, 2>(L, ctl, num_sms, s);
    }
    if (L.out_f32) return dispatch_n<bf, float, kEpiPlain>(L, ctl, num_sms, s);
    return L.swiglu ? dispatch_n<bf, bf, kEpiSwiGLU>(L, ctl, num_sms, s) : dispatch_plain<bf, bf>(L, ctl, num_sms, s);
}

}  // namespace

size_t gemm_ctl_bytes(int num_sms) {
    return kCtlHeaderBytes + sizeof(int) * 2 * (size_t)num_sms + kSlotBytesMax * 2 * (size_t)num_sms + 256;
}

size_t gemm_ctl_zero_bytes(int num_sms) { return kCtlHeaderBytes + sizeof(int) * 2 * (size_t)num_sms; }

GemmCtl gemm_ctl(void* workspace, int num_sms) {
    uint8_t* b = static_cast<uint8_t*>(workspace);
    GemmCtl c;
    c.status = reinterpret_cast<unsigned*>(b);
    c.counters = reinterpret_cast<int*>(b + kCtlHeaderBytes);
    size_t off = kCtlHeaderBytes + sizeof(int) * 2 * (size_t)num_sms;
    off = (off + 255) & ~size_t(255);
    c.partials = reinterpret_cast<float*>(b + off);
    c.ffn_ctl = reinterpret_cast<int*>(b + ((gemm_ctl_bytes(num_sms) + 255) & ~size_t(255)));
    return c;
}

size_t ctl_block_bytes(int num_sms) {
    return ((gemm_ctl_bytes(num_sms) + 255) & ~size_t(255)) + ((sizeof(int) * kFfnCtlInts + 255) & ~size_t(255));
}

namespace {

template <typename T, int kMaxN, bool kFp8>
int launch_ffn_variant(const FfnLaunch& L, const GemmCtl& ctl, int num_sms, cudaStream_t stream) {
    using C = FfnCfg<T, kMaxN, kFp8>;
    auto kern = moe_ffn_stream_kernel<T, kMaxN, kFp8>;
    static bool attr_done = false;
    if (!attr_done) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess) {
            cudaGetLastError();
            return -3;
        }
        attr_done = true;
    }
    // partial slots of 128 x (2 * kMaxN) fp32 share the GEMM slot area (2 x 256 KB per SM)
    const int slots_total = (int)((kSlotBytesMax * 2 * (size_t)num_sms) / ((size_t)C::kSlotFloats * 4));
    CUtensorMap w13, w2, xa, xa64, xb, xb64;
    const int eb = Elt<T>::kBytes;
    const CUtensorMapDataType dt = Elt<T>::kTma;
    if (kFp8) {
        // E4M3 codes: 64-code rows (one stage's K) with the 64-byte swizzle, which
        // spreads the converters' row-per-thread reads over all banks
        if (!make_map(&w13, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, L.w13, (long long)L.n_groups * 2 * L.I, L.H, 128,
                      C::kBK))
            return -3;
        if (!make_map(&w2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, L.w2, (long long)L.n_groups * L.H, L.I, 128, C::kBK))
            return -3;
    } else {
        if (!make_map(&w13, dt, eb, L.w13, (long long)L.n_groups * 2 * L.I, L.H, 128)) return -3;
        if (!make_map(&w2, dt, eb, L.w2, (long long)L.n_groups * L.H, L.I, 128)) return -3;
    }
    // token operands: on the FP8 path the gate/up operand is the rows' E4M3 hi
    // and lo codes ([2 x_rows, H] bytes, 128-code boxes) and the activations are
    // f16 (split into codes in shared memory); otherwise both are in the
    // activation dtype
    const CUtensorMapDataType xdt = kFp8 ? Elt<__half>::kTma : dt;
    if (kFp8) {
        // the per-row activation maxima live in the control block
        if (!L.x_scale || L.x_rows > kFfnMaxRows) return -1;
        if (!make_map(&xa, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, L.x, 2 * L.x_rows, L.H, 16)) return -3;
        if (!make_map(&xa64, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, L.x, 2 * L.x_rows, L.H, 64)) return -3;
    } else {
        if (!make_map(&xa, xdt, eb, L.x, L.x_rows, L.H, 16)) return -3;
        if (!make_map(&xa64, xdt, eb, L.x, L.x_rows, L.H, 64)) return -3;
    }
    if (!make_map(&xb, xdt, eb, L.act, L.x_rows, L.I, 16)) return -3;
    if (!make_map(&xb64, xdt, eb, L.act, L.x_rows, L.I, 64)) return -3;
    FfnParams p;
    p.seg_offsets = L.seg_offsets;
    p.n_groups = L.n_groups;
    p.seg_rows = L.seg_rows;
    p.H = L.H;
    p.I = L.I;
    p.act = L.act;
    p.y = L.y;
    p.ctl = ctl.ffn_ctl;
    p.partials = ctl.partials;
    p.status = ctl.status;
    p.wait_limit_ns = wait_limit_ns();
    p.withhold_first_load = take_withhold_flag();
    p.max_slots_phase = slots_total / 2;
    p.s13 = L.s13;
    p.s2 = L.s2;
    p.x_scale = L.x_scale;
    p.lo_rows = L.x_rows;
    const int grid = L.sms > 0 && L.sms < num_sms ? L.sms : num_sms;
    cudaError_t e = launch_kernel(kern, dim3(grid), dim3(C::kThreads), C::kSmemBytes, stream, w13, w2, xa, xa64,
                                  xb, xb64, p);
    count_launch();
    if (e != cudaSuccess) cudaGetLastError();
    return e == cudaSuccess ? 0 : -3;
}

}  // namespace

int launch_ffn_stream(const FfnLaunch& L, const GemmCtl& ctl, cudaStream_t stream) {
    DeviceInfo d;
    int rc = current_device(&d);
    if (rc != 0) return rc;
    if (L.max_n != 32 && L.max_n != 64 && L.max_n != 128) return 1;
    if (L.n_groups < 1 || L.n_groups > kMaxGroups || L.max_chunks > kFfnMaxChunks) return 1;
    // split-tile counters: each phase's tiles must fit half the counter array when split
    const long long ntiles_a = L.max_chunks * ((L.I + 127) / 128);
    const long long ntiles_b = L.max_chunks * ((L.H + 255) / 256);
    const long long G = L.sms > 0 && L.sms < d.num_sms ? L.sms : d.num_sms;
    if ((ntiles_a < 2LL * G && ntiles_a > kFfnTileCtrs / 2) || (ntiles_b < 2LL * G && ntiles_b > kFfnTileCtrs / 2))
        return 1;
    if (L.x_rows <= 0) return 0;
    if (L.fp8) {
        if (L.dtype != 0 || !L.s13 || !L.s2) return -1;
        if (L.max_n == 32) return launch_ffn_variant<__nv_bfloat16, 32, true>(L, ctl, d.num_sms, stream);
        if (L.max_n == 64) return launch_ffn_variant<__nv_bfloat16, 64, true>(L, ctl, d.num_sms, stream);
        return launch_ffn_variant<__nv_bfloat16, 128, true>(L, ctl, d.num_sms, stream);
    }
    if (L.dtype == 0) {
        if (L.max_n == 32) return launch_ffn_variant<__nv_bfloat16, 32, false>(L, ctl, d.num_sms, stream);
        if (L.max_n == 64) return launch_ffn_variant<__nv_bfloat16, 64, false>(L, ctl, d.num_sms, stream);
        return launch_ffn_variant<__nv_bfloat16, 128, false>(L, ctl, d.num_sms, stream);
    }
    if (L.dtype == 1) {
        if (L.max_n == 32) return launch_ffn_variant<float, 32, false>(L, ctl, d.num_sms, stream);
        if (L.max_n == 64) return launch_ffn_variant<float, 64, false>(L, ctl, d.num_sms, stream);
        return launch_ffn_variant<float, 128, false>(L, ctl, d.num_sms, stream);
    }
    return -1;
}

namespace {
int g_token_tile_cap = 0;  // 0: automatic
int g_split_tail = 1;      // aligned k-slices for the last partial wave
}

void set_token_tile_cap(int n) { g_token_tile_cap = n; }
int token_tile_cap() { return g_token_tile_cap; }
void set_split_tail(int mode) { g_split_tail = mode; }
int split_tail_mode() { return g_split_tail; }
void set_cta_pairs(bool on) { g_cta_pairs = on; }

int pick_max_n(double rows_per_group) {
    if (g_token_tile_cap == 32 || g_token_tile_cap == 64 || g_token_tile_cap == 128 || g_token_tile_cap == 256)
        return g_token_tile_cap;
    if (rows_per_group <= 24.0) return 32;
    if (rows_per_group <= 56.0) return 64;
    if (rows_per_group <= 128.0) return 128;
    return 256;
}

int launch_gemm(const GemmLaunch& L, const GemmCtl& ctl, cudaStream_t stream) {
    DeviceInfo d;
    int rc = current_device(&d);
    if (rc != 0) return rc;
    if (L.n_groups < 1 || L.n_groups > kMaxGroups || L.kdim <= 0 || L.n_out <= 0) return -1;
    if (L.x_rows <= 0 || L.w_rows <= 0) return 0;
    if (L.dtype == 0) {
        if (L.out_f32 && L.swiglu) return -1;
        return dispatch_bf16(L, ctl, d.num_sms, stream);
    }
    if (L.dtype == 1) {
        return L.swiglu ? dispatch_n<float, float, kEpiSwiGLU>(L, ctl, d.num_sms, stream)
                        : dispatch_plain<float, float>(L, ctl, d.num_sms, stream);
    }
    return -1;
}

}  // namespace moe
