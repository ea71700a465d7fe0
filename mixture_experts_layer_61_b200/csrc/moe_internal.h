// moe_internal.h -- host-side declarations shared by the libmoe translation
// units (launchers, device properties, the launch counter).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

namespace moe {

// Programmatic dependent launch (on by default): kernels may begin while the
// previous kernel on the stream drains; each kernel waits (griddepcontrol)
// before it touches data a predecessor produced.
bool pdl_enabled();
void set_pdl(bool on);

// Launch with programmatic dependent launch (when enabled) and, for
// cluster_x > 1, thread-block clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                  int cluster_x, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int n = 0;
    if (pdl_enabled()) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (cluster_x > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          Args&&... args) {
    return launch_kernel_cluster(kern, grid, block, smem, s, 1, std::forward<Args>(args)...);
}

// Cached properties of the current device.
struct DeviceInfo {
    int device;
    int num_sms;
    int cc_major, cc_minor;
};
// Returns 0 and fills *info for the current device; -5 if it is not sm_100.
int current_device(DeviceInfo* info);

// Workspace control block: status word, stream-K counters (2 per SM) and
// partial-tile slots (2 per SM, each 128 rows x at most 512 fp32 columns).
constexpr size_t kCtlHeaderBytes = 256;
constexpr size_t kSlotBytesMax = 128ull * 512ull * 4ull;
size_t gemm_ctl_bytes(int num_sms);
// Bytes of the control words that must be zero between calls (status + counters).
size_t gemm_ctl_zero_bytes(int num_sms);

struct GemmCtl {
    unsigned* status;
    int* counters;
    float* partials;
    int* ffn_ctl;  // control words of the fused decode FFN kernel
};
GemmCtl gemm_ctl(void* workspace, int num_sms);
// Bytes of the whole control block at the start of a workspace: the GEMM
// control words and partial slots, then the fused FFN's control words.
size_t ctl_block_bytes(int num_sms);

// One GEMM launch.  X rows are tokens ([x_rows, kdim]), W rows are output
// features ([w_rows, kdim]); out[row][feature] with row stride out_ld.
struct GemmLaunch {
    const void* x;
    long long x_rows;
    const void* w;
    long long w_rows;
    int kdim;
    int n_out;
    const int32_t* seg_offsets;  // device, n_groups + 1, or nullptr
    int n_groups;
    int seg_rows;                // one segment [0, seg_rows) when seg_offsets == nullptr
    int w_group_stride;
    int up_offset;
    bool swiglu;
    bool out_f32;                // fp32 output (router logits) instead of the activation dtype
    void* out;
    int out_ld;
    int dtype;                   // 0 bf16, 1 fp32
    int max_n;                   // token-tile cap: 32, 64, 128 or 256
    int max_split;               // stream-K: most blocks per tile (0 = default 4)
    int sms;                     // persistent blocks at most (0 = one per SM): an SM share
};

int launch_gemm(const GemmLaunch& L, const GemmCtl& ctl, cudaStream_t stream);

// The expert FFN (gate/up + SwiGLU, then down) over n_groups segments of X in
// one launch, for token-tile caps 32, 64 and 128 (memory-bound sizes).  Returns 1 when the
// configuration is outside what the fused kernel handles (caller falls back
// to two GEMM launches).
struct FfnLaunch {
    const void* x;
    long long x_rows;
    const void* w13;
    const void* w2;
    int H, I;
    const int32_t* seg_offsets;
    int n_groups;
    int seg_rows;
    void* act;
    void* y;
    int dtype;
    int max_n;
    long long max_chunks;  // upper bound on token chunks (host side)
    int sms;               // persistent blocks at most (0 = one per SM)
    bool fp8 = false;      // w13 / w2 are E4M3 codes with fp32 row scales s13 [n_groups*2I], s2 [n_groups*H]
    const float* s13 = nullptr;
    const float* s2 = nullptr;
    // FP8 weights: x holds the token rows' E4M3 hi codes [x_rows, H], then their
    // lo codes [x_rows, H]; x_scale [x_rows] their power-of-two scales
    const float* x_scale = nullptr;
};
int launch_ffn_stream(const FfnLaunch& L, const GemmCtl& ctl, cudaStream_t stream);

// Token-tile cap for an expected number of rows per group (or the cap forced
// by set_token_tile_cap, 0 = automatic).
int pick_max_n(double rows_per_group);
void set_token_tile_cap(int n);
int token_tile_cap();  // the forced cap, 0 = automatic
// How the GEMM shares out the tiles after its whole data-parallel waves:
// 0 contiguous stream-K over the last one to two waves, 1 aligned k-slices of
// the last partial wave (default).
void set_split_tail(int mode);
int split_tail_mode();
// CTA-pair (2-SM MMA) tiles for bf16 launches at the 256-token cap (default on).
void set_cta_pairs(bool on);

// Elementwise / routing kernels.
// k_per_token (nullable): per-token expert count, clamped to [0, K]; slots
// from it on get id -1 and weight 0.
int launch_topk(int T, int E, int K, int score_fn, int renorm, const float* logits, const int32_t* k_per_token,
                int32_t* ids, float* w, cudaStream_t stream);
// mode 0: block-wise padding, 1: max-value padding (every expert padded to the
// most loaded one's rounded count).
int launch_align(int T, int K, int E, int B, int mode, long long P_max, const int32_t* ids, int32_t* counts,
                 int32_t* offsets, int32_t* sorted_ids, int32_t* block_expert, int32_t* pos, int32_t* scalars,
                 int32_t* stats_copy, cudaStream_t stream);
// Router logits (CUDA cores) + top-K + alignment in one launch, for small T
// and a small router matrix (E H <= kSmallRouteMaxEH), or any router matrix
// with few logits (T E <= kSmallRouteMaxTE): with many logits of a large
// router the single block that reduces the partial sums and runs top-K and
// the alignment outlasts the three separate launches (DeepSeek-V3-shaped
// layer at T = 8: 6 us slower per layer, at T = 32: 56 us), while with one
// token it saves two launch hand-overs (T = 1: DeepSeek-V3-shaped 8 us,
// Qwen2-MoE-shaped 7 us faster).
constexpr int kSmallRouteMaxT = 64;
constexpr long long kSmallRouteMaxEH = 1 << 17;
constexpr long long kSmallRouteMaxTE = 256;
// `part` holds (H/256 + 1) * T * E floats of partial router sums.
int launch_route_small(int T, int H, int E, int K, int score_fn, int renorm, int B, int mode, long long P_max,
                       int dtype, const void* x, const void* w_r, const float* logits_override,
                       const int32_t* k_per_token, float* part, float* logits, int32_t* ids, float* w,
                       int32_t* counts, int32_t* offsets, int32_t* sorted_ids, int32_t* block_expert, int32_t* pos,
                       int32_t* scalars, int32_t* stats_copy, int* done_ctr, cudaStream_t stream);
int launch_permute(int H, int K, int dtype, long long P_max, const void* x, const int32_t* sorted_ids,
                   const int32_t* scalars, void* x_perm, cudaStream_t stream);
// The exact two-term E4M3 split of bf16 rows [rows, H] (gathered by
// sorted_ids with the count in scalars[0] when sorted_ids is given): codes
// [rows, H] hi then, lo_rows rows on, lo; power-of-two scales [rows].
int launch_split_e4m3(int H, int K, long long rows, const void* x, const int32_t* sorted_ids, const int32_t* scalars,
                      uint8_t* codes, long long lo_rows, float* scales, cudaStream_t stream);
// col0 / ncols (elements, multiples of 16 bytes): only those columns, into
// rows of ncols; ncols < 0: all H columns
int launch_combine(int T, int H, int K, int dtype, const void* y_perm, const int32_t* pos, const float* w,
                   const void* shared_out, void* out, cudaStream_t stream, bool out_f32 = false, int col0 = 0,
                   int ncols = -1);
// out [T, H] from n column blocks parts[c] [T, H / n] (fp32), rounded to dtype
int launch_tp_gather(int n, const float* const* parts, int T, int H, int dtype, void* out, cudaStream_t stream);
constexpr int kTpMaxParts = 16;  // ranks of one TP reduction
// router logits on the CUDA cores for small router matrices (E <= 16, E*H*elt
// bytes <= kRouterCcMaxBytes, H % 8 == 0); -1 when the shape does not fit
constexpr int kRouterCcMaxBytes = 96 * 1024;
bool router_cc_fits(int H, int E, int dtype);
int launch_router_cc(int T, int H, int E, int dtype, const void* x, const void* w_r, float* logits,
                     cudaStream_t stream);
int launch_tp_reduce(int n, const float* const* parts, long long count, int dtype, void* out, cudaStream_t stream);
// Router logits (CUDA cores, router matrix in shared memory) + top-K + gate
// weights + alignment in one launch, for router_cc_fits shapes at any T.
struct RouteCcArgs {
    int T, H, E, K, score_fn, renorm, B, mode, dtype;
    long long P_max;
    const void* x;
    const void* w_r;
    const float* logits_override;
    const int32_t* k_per_token;
    float* logits;
    int32_t* ids;
    float* w;
    int32_t *counts, *offsets, *sorted_ids, *block_expert, *pos, *scalars, *stats_copy;
    int* done_ctr;
};
int launch_route_cc(const RouteCcArgs& a, cudaStream_t stream);

// Row-wise FP8 E4M3 quantisation: q [rows, cols] codes, scales [rows].
int launch_quantize_fp8(long long rows, int cols, int dtype, const void* w, uint8_t* q, float* scales,
                        cudaStream_t stream);

// Launch bookkeeping.
void count_launch();
uint64_t wait_limit_ns();
int take_withhold_flag();

}  // namespace moe
