// moe_api.cu -- the extern "C" entry points of libmoe.so (declared in
// include/moe.h): argument checks, workspace layout and the launch sequence of
// the MoE layer forward.  Every compute step runs in the kernels of
// moe_kernels.cu and moe_gemm.cu; nothing here touches tensor data.
#include <atomic>
#include <climits>
#include <cmath>
#include <mutex>

#include "../../include/moe.h"
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {
std::atomic<uint64_t> g_launches{0};
std::atomic<uint64_t> g_wait_limit{2000000000ull};
std::atomic<int> g_withhold{0};

constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
int g_dev_state[kMaxDevices];  // 0 unknown, 1 ok, -1 unsupported
std::mutex g_dev_mu;
}  // namespace

std::atomic<bool> g_pdl{true};
bool pdl_enabled() { return g_pdl.load(std::memory_order_relaxed); }
void set_pdl(bool on) { g_pdl.store(on); }

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
uint64_t wait_limit_ns() { return g_wait_limit.load(std::memory_order_relaxed); }
int take_withhold_flag() { return g_withhold.exchange(0); }

int current_device(DeviceInfo* info) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return -3;
    }
    if (dev < 0 || dev >= kMaxDevices) return -5;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (g_dev_state[dev] == 0) {
        DeviceInfo d;
        d.device = dev;
        if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
            cudaGetLastError();
            return -3;
        }
        g_dev[dev] = d;
        g_dev_state[dev] = (d.cc_major == 10 && d.cc_minor == 0) ? 1 : -1;
    }
    if (g_dev_state[dev] < 0) return -5;
    *info = g_dev[dev];
    return 0;
}

}  // namespace moe

using namespace moe;

namespace {

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int elt_bytes(int dtype) { return dtype == 0 ? 2 : (dtype == 1 ? 4 : 0); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_cfg(const moe_config_t* c) {
    if (!c) return MOE_ERR_ARG;
    const int eb = elt_bytes(c->dtype);
    if (eb == 0) return MOE_ERR_ARG;
    const int vec = 16 / eb;
    if (c->T < 0 || c->H <= 0 || c->E < 1 || c->E > 1024 || c->K < 1 || c->K > 16 || c->K > c->E || c->I <= 0)
        return MOE_ERR_ARG;
    if (c->n_shared < 0 || c->I_shared < 0 || (c->n_shared > 0 && c->I_shared <= 0)) return MOE_ERR_ARG;
    if (c->tile_B < 1 || c->tile_B > 256) return MOE_ERR_ARG;
    if (c->score_fn != 0 && c->score_fn != 1) return MOE_ERR_ARG;
    if (c->renorm != 0 && c->renorm != 1) return MOE_ERR_ARG;
    if (c->pad_mode != 0 && c->pad_mode != 1) return MOE_ERR_ARG;
    if (c->H % vec != 0 || c->I % vec != 0) return MOE_ERR_ARG;
    const long long I_sh = (long long)c->n_shared * c->I_shared;
    if (I_sh % vec != 0 || I_sh > (1LL << 30)) return MOE_ERR_ARG;
    const long long A = (long long)c->T * c->K;
    if (A > (1LL << 30)) return MOE_ERR_ARG;
    if ((long long)c->E * 2 * c->I >= (1LL << 31) || (long long)c->E * c->H >= (1LL << 31)) return MOE_ERR_ARG;
    return MOE_OK;
}

long long p_max(const moe_config_t* c) {
    const long long A = (long long)c->T * c->K;
    if (c->pad_mode == 1) {
        // an expert holds at most one assignment per token
        const long long n = A < c->T ? A : c->T;
        return (long long)c->E * ((n + c->tile_B - 1) / c->tile_B) * c->tile_B;
    }
    return A + (A < c->E ? A : c->E) * (long long)(c->tile_B - 1);
}

struct Layout {
    size_t ctl, ctl_sh, logits, route_part, ids, w, counts, offsets, scalars, sorted_ids, block_expert, pos, x_perm,
        act, act_sh, sh_out, x16, x_scale, y8, sh_scale;
    size_t total;
};

int routed_max_n(const moe_config_t* c);
int routed_max_n_avg(const moe_config_t* c);

// The layer's routing runs as one small-batch launch (route_small_kernel).
bool small_route(const moe_config_t* c) {
    return c->T <= kSmallRouteMaxT && c->H % 8 == 0 &&
           ((long long)c->E * c->H <= kSmallRouteMaxEH || (long long)c->T * c->E <= kSmallRouteMaxTE);
}

// FP8 expert weights run at decode sizes only (the fused expert FFN)
bool fp8_sized(const moe_config_t* c) { return c->dtype == 0 && routed_max_n_avg(c) <= 128; }

Layout layout(const moe_config_t* c, int num_sms) {
    Layout L;
    const size_t eb = elt_bytes(c->dtype);
    const long long P = p_max(c);
    const long long A = (long long)c->T * c->K;
    const long long I_sh = (long long)c->n_shared * c->I_shared;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t r = o;
        o = align256(o + bytes);
        return r;
    };
    L.ctl = take(ctl_block_bytes(num_sms));
    // the shared experts' own control block: they run beside the routed experts
    L.ctl_sh = take(I_sh > 0 ? ctl_block_bytes(num_sms) : 0);
    L.logits = take(sizeof(float) * (size_t)c->T * c->E);
    // partial router sums of the small-batch routing kernel (slices of 256 hidden elements)
    L.route_part = take(small_route(c) ? sizeof(float) * ((size_t)c->H / 256 + 1) * c->T * c->E : 0);
    L.ids = take(sizeof(int32_t) * (size_t)A);
    L.w = take(sizeof(float) * (size_t)A);
    L.counts = take(sizeof(int32_t) * (size_t)c->E);
    L.offsets = take(sizeof(int32_t) * ((size_t)c->E + 1));
    L.scalars = take(sizeof(int32_t) * 4);
    L.sorted_ids = take(sizeof(int32_t) * (size_t)P);
    L.block_expert = take(sizeof(int32_t) * (size_t)((P + c->tile_B - 1) / c->tile_B));
    L.pos = take(sizeof(int32_t) * (size_t)A);
    // also holds y_perm once x_perm is consumed; with FP8 weights the token rows'
    // E4M3 hi and lo codes (the same 2 bytes an element)
    L.x_perm = take(eb * (size_t)P * c->H);
    L.act = take(eb * (size_t)P * c->I);
    L.act_sh = take(I_sh > 0 ? eb * (size_t)c->T * I_sh : 0);
    L.sh_out = take(I_sh > 0 ? eb * (size_t)c->T * c->H : 0);
    // the shared FFN on FP8 weights: x's E4M3 hi and lo codes and its row scales
    L.x16 = take(I_sh > 0 && c->dtype == 0 ? 2 * (size_t)c->T * c->H : 0);
    L.sh_scale = take(I_sh > 0 && c->dtype == 0 ? sizeof(float) * (size_t)c->T : 0);
    // the routed FFN on FP8 weights: the permuted rows' scales, and its
    // outputs (x_perm holds the codes, which other chunks still read)
    const bool f8 = fp8_sized(c);
    L.x_scale = take(f8 ? sizeof(float) * (size_t)P : 0);
    L.y8 = take(f8 ? eb * (size_t)P * c->H : 0);
    L.total = o;
    return L;
}

template <typename P>
P* at(void* base, size_t off) {
    return reinterpret_cast<P*>(static_cast<uint8_t*>(base) + off);
}

int status_of(int rc) { return rc == 0 ? MOE_OK : (rc == -5 ? MOE_ERR_DEVICE : (rc == -1 ? MOE_ERR_ARG : MOE_ERR_CUDA)); }

GemmLaunch gate_up_launch(const void* x, long long x_rows, const int32_t* seg_offsets, int n_groups, int seg_rows,
                          int H, int I, int dtype, const void* w13, void* act, int max_n) {
    GemmLaunch g{};
    g.x = x;
    g.x_rows = x_rows;
    g.w = w13;
    g.w_rows = (long long)n_groups * 2 * I;
    g.kdim = H;
    g.n_out = I;
    g.seg_offsets = seg_offsets;
    g.n_groups = n_groups;
    g.seg_rows = seg_rows;
    g.w_group_stride = 2 * I;
    g.up_offset = I;
    g.swiglu = true;
    g.out_f32 = false;
    g.out = act;
    g.out_ld = I;
    g.dtype = dtype;
    g.max_n = max_n;
    return g;
}

GemmLaunch down_launch(const void* act, long long x_rows, const int32_t* seg_offsets, int n_groups, int seg_rows,
                       int H, int I, int dtype, const void* w2, void* y, int max_n) {
    GemmLaunch d{};
    d.x = act;
    d.x_rows = x_rows;
    d.w = w2;
    d.w_rows = (long long)n_groups * H;
    d.kdim = I;
    d.n_out = H;
    d.seg_offsets = seg_offsets;
    d.n_groups = n_groups;
    d.seg_rows = seg_rows;
    d.w_group_stride = H;
    d.up_offset = 0;
    d.swiglu = false;
    d.out_f32 = false;
    d.out = y;
    d.out_ld = H;
    d.dtype = dtype;
    d.max_n = max_n;
    return d;
}

// gate/up (SwiGLU) + down over `n_groups` segments of X: one fused launch at
// decode sizes (token-tile cap 32, 64 or 128), else two GEMM launches.
// `max_chunks` bounds the number of token chunks the segments can form;
// `sms` / `ffn_sms` cap the persistent grid of the GEMMs / of the fused
// kernel (0 = one block per SM).
int run_ffn(const void* x, long long x_rows, const int32_t* seg_offsets, int n_groups, int seg_rows, int H, int I,
            int dtype, const void* w13, const void* w2, void* act, void* y, int max_n, const GemmCtl& ctl,
            cudaStream_t s, long long max_chunks, int sms = 0, int ffn_sms = 0, const float* s13 = nullptr,
            const float* s2 = nullptr, const float* x_scale = nullptr) {
    const bool fp8 = s13 != nullptr;  // w13 / w2 hold E4M3 codes with these row scales
    if (fp8 && max_n > 128) return -1;  // FP8 weights run on the fused (decode-size) kernel only
    if (max_n <= 128) {
        FfnLaunch f;
        f.x = x;
        f.x_rows = x_rows;
        f.w13 = w13;
        f.w2 = w2;
        f.H = H;
        f.I = I;
        f.seg_offsets = seg_offsets;
        f.n_groups = n_groups;
        f.seg_rows = seg_rows;
        f.act = act;
        f.y = y;
        f.dtype = dtype;
        f.max_n = max_n;
        f.max_chunks = max_chunks;
        f.sms = ffn_sms;
        f.fp8 = fp8;
        f.s13 = s13;
        f.s2 = s2;
        f.x_scale = x_scale;
        int rc = launch_ffn_stream(f, ctl, s);
        if (rc != 1) return rc;  // 1: not handled, use two launches
        if (fp8) return -1;
    }
    GemmLaunch g = gate_up_launch(x, x_rows, seg_offsets, n_groups, seg_rows, H, I, dtype, w13, act, max_n);
    g.sms = sms;
    int rc = launch_gemm(g, ctl, s);
    if (rc != 0) return rc;
    g = down_launch(act, x_rows, seg_offsets, n_groups, seg_rows, H, I, dtype, w2, y, max_n);
    g.sms = sms;
    return launch_gemm(g, ctl, s);
}

// ------------------------------------------ shared experts beside the routed ones
// The shared experts read only x, so they run from the start of the layer on a
// second stream, concurrently with routing and the routed experts, on their
// own share of the SMs and with their own control block; the combine waits
// for both.  One side stream and a fork/join event pair per device, created on
// first use; the mutex keeps the record/wait pairs of concurrent callers apart.
struct SideStream {
    std::mutex mu;
    int state = 0;  // 0 not yet created, 1 ready, -1 creation failed (run serially)
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
SideStream g_side[kMaxDevices];
std::atomic<int> g_shared_sms{0};  // 0 automatic, -1 serial, n > 0 fixed share

// Called with side.mu held.
bool side_ready(SideStream& side) {
    if (side.state == 0) {
        side.state = -1;
        if (cudaStreamCreateWithFlags(&side.s, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&side.fork, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&side.join, cudaEventDisableTiming) == cudaSuccess)
            side.state = 1;
        else
            cudaGetLastError();
    }
    return side.state == 1;
}

// SMs given to the shared experts (even, for CTA pairs), or 0 to run them after
// the routed experts on the caller's stream.  Calibrated on B200 with the
// Qwen2-MoE- and DeepSeek-V3-shaped layers (a sweep of the share per T):
//  * T <= 128 (the shared FFN is one fused launch): the shared experts start
//    with a large share while routing runs, and the routed FFN's blocks take
//    over their SMs as they exit: 0.35 N + 0.4 N f, at most 0.55 N, where f is
//    the shared experts' fraction of the weight bytes.
//  * larger T (the shared FFN is a GEMM pair, near per-SM tensor peak on a
//    few SMs, beside the routed stream at HBM speed): 12 + rho / 2 SMs, at most
//    40, with rho = shared flops / routed weight bytes; serially once the
//    routed experts reach 128 rows each, where they need every SM.
int shared_sms(const moe_config_t* c, int num_sms) {
    const int forced = g_shared_sms.load(std::memory_order_relaxed);
    if (forced < 0 || num_sms < 8) return 0;
    if (forced > 0) {
        const int n = forced & ~1;
        return n < 2 ? 2 : (n > num_sms - 2 ? num_sms - 2 : n);
    }
    const double eb = elt_bytes(c->dtype), T = c->T, H = c->H, I = c->I, E = c->E, K = c->K;
    const double I_sh = (double)c->n_shared * c->I_shared;
    const double e_act = E * (1.0 - std::pow(1.0 - K / E, T));
    const double B_r = e_act * 3.0 * H * I * eb, B_s = 3.0 * H * I_sh * eb;
    double n;
    if (pick_max_n(T) <= 128) {
        const double f = B_s / (B_s + B_r);
        n = num_sms * std::fmin(0.55, 0.35 + 0.4 * f);
    } else {
        if (T * K / E >= 128.0) return 0;
        const double rho = 6.0 * T * H * I_sh / B_r;
        n = std::fmin(40.0, 12.0 + 0.5 * rho);
    }
    int ni = 2 * (int)std::lround(n / 2.0);
    return ni < 2 ? 2 : (ni > num_sms - 2 ? num_sms - 2 : ni);
}

// The router's output has only E features, so its tiles are few: cut the
// tokens into 64-row tiles (32 for decode batches) and let up to 8 blocks
// share a tile, so that more SMs stream x.
void router_tiling(GemmLaunch& g, int T) {
    g.max_n = T > 32 ? 64 : 32;
    g.max_split = 8;
}

// The routed experts' token tile: by the average rows per expert (the FP8
// path, and every layer but the one case below) ...
int routed_max_n_avg(const moe_config_t* c) { return pick_max_n((double)c->T * c->K / (double)c->E); }

// ... except that bf16 layers of large experts (H I >= 2^25) whose largest
// expert is expected past the fused FFN's 128-row chunk (binomial rows under
// uniform routing: mean + 2.5 standard deviations) take the 256-token
// CTA-pair GEMMs: there the fused kernel, MMA-issue-bound at 128 rows, would
// stream and issue a whole large expert once more for each remainder chunk
// (Mixtral-shaped layer at 128 rows per expert: 0.619 ms fused, 0.573 ms
// pairs; at 96 rows 0.509 fused, 0.556 pairs; Qwen2-MoE's small experts at
// 128 rows: 1.152 fused, 1.172 pairs).
int routed_max_n(const moe_config_t* c) {
    const int n = routed_max_n_avg(c);
    if (n != 128 || c->dtype != 0 || token_tile_cap() != 0) return n;
    const double A = (double)c->T * c->K, pe = 1.0 / c->E;
    const double hi = A * pe + 2.5 * std::sqrt(A * pe * (1.0 - pe));
    return (double)c->H * c->I >= 33554432.0 && hi > 128.0 ? 256 : n;
}

// Upper bounds on the token chunks of the routed segments (every chunk holds
// at least one 16-row unit) and of a dense segment of T rows.
long long routed_max_chunks(const moe_config_t* c) { return (long long)c->E + p_max(c) / 16 + 1; }
long long dense_max_chunks(long long T) { return T / 16 + 1; }

}  // namespace

extern "C" {

const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_ARG: return "invalid argument";
        case MOE_ERR_WORKSPACE: return "workspace too small";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_TIMEOUT: return "device wait timed out";
        case MOE_ERR_DEVICE: return "unsupported device (needs sm_100)";
        default: return "unknown status";
    }
}

int64_t moe_padded_rows_max(const moe_config_t* cfg) {
    if (check_cfg(cfg) != MOE_OK) return -1;
    return p_max(cfg);
}

size_t moe_workspace_size(const moe_config_t* cfg) {
    if (check_cfg(cfg) != MOE_OK) return 0;
    DeviceInfo d;
    if (current_device(&d) != 0) return 0;
    return layout(cfg, d.num_sms).total;
}

int64_t moe_layer_logits_offset(const moe_config_t* cfg) {
    if (check_cfg(cfg) != MOE_OK) return -1;
    DeviceInfo d;
    if (current_device(&d) != 0) return -1;
    return (int64_t)layout(cfg, d.num_sms).logits;
}

size_t moe_gemm_workspace_size(void) {
    DeviceInfo d;
    if (current_device(&d) != 0) return 0;
    return ctl_block_bytes(d.num_sms);
}

size_t dense_ffn_workspace_size(int T, int H, int I, int dtype) {
    const int eb = elt_bytes(dtype);
    if (eb == 0 || T < 0 || H <= 0 || I <= 0) return 0;
    DeviceInfo d;
    if (current_device(&d) != 0) return 0;
    return align256(ctl_block_bytes(d.num_sms)) + align256((size_t)eb * T * I);
}

int moe_router_gemm(const moe_config_t* cfg, const void* x, const void* w_router, float* logits, void* workspace,
                    size_t ws_bytes, moe_stream_t stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->T == 0) return MOE_OK;
    if (!x || !w_router || !logits || !workspace) return MOE_ERR_ARG;
    if (!aligned16(x) || !aligned16(w_router) || !aligned16(workspace)) return MOE_ERR_ARG;
    DeviceInfo d;
    if ((rc = current_device(&d)) != 0) return status_of(rc);
    if (ws_bytes < ctl_block_bytes(d.num_sms)) return MOE_ERR_WORKSPACE;
    if (router_cc_fits(cfg->H, cfg->E, cfg->dtype))  // a small router matrix: CUDA cores, w_r in shared memory
        return status_of(launch_router_cc(cfg->T, cfg->H, cfg->E, cfg->dtype, x, w_router, logits,
                                          (cudaStream_t)stream));
    GemmLaunch g{};
    g.x = x;
    g.x_rows = cfg->T;
    g.w = w_router;
    g.w_rows = cfg->E;
    g.kdim = cfg->H;
    g.n_out = cfg->E;
    g.n_groups = 1;
    g.seg_rows = cfg->T;
    g.swiglu = false;
    g.out_f32 = true;
    g.out = logits;
    g.out_ld = cfg->E;
    g.dtype = cfg->dtype;
    router_tiling(g, cfg->T);
    return status_of(launch_gemm(g, gemm_ctl(workspace, d.num_sms), (cudaStream_t)stream));
}

int moe_route_k(const moe_config_t* cfg, const float* logits, const int32_t* k_per_token, int32_t* topk_ids,
                float* topk_w, moe_stream_t stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->T == 0) return MOE_OK;
    if (!logits || !topk_ids || !topk_w) return MOE_ERR_ARG;
    DeviceInfo d;
    if ((rc = current_device(&d)) != 0) return status_of(rc);
    return status_of(launch_topk(cfg->T, cfg->E, cfg->K, cfg->score_fn, cfg->renorm, logits, k_per_token, topk_ids,
                                 topk_w, (cudaStream_t)stream));
}

int moe_route(const moe_config_t* cfg, const float* logits, int32_t* topk_ids, float* topk_w, moe_stream_t stream) {
    return moe_route_k(cfg, logits, nullptr, topk_ids, topk_w, stream);
}

int moe_align_pad(const moe_config_t* cfg, const int32_t* topk_ids, int32_t* counts, int32_t* offsets,
                  int32_t* sorted_ids, int32_t* block_expert, int32_t* pos, int32_t* scalars, moe_stream_t stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (!counts || !offsets || !scalars || !block_expert) return MOE_ERR_ARG;
    if (cfg->T > 0 && (!topk_ids || !sorted_ids || !pos)) return MOE_ERR_ARG;
    DeviceInfo d;
    if ((rc = current_device(&d)) != 0) return status_of(rc);
    return status_of(launch_align(cfg->T, cfg->K, cfg->E, cfg->tile_B, cfg->pad_mode, p_max(cfg), topk_ids,
                                  counts, offsets,
                                  sorted_ids, block_expert, pos, scalars, nullptr, (cudaStream_t)stream));
}

int moe_permute(const moe_config_t* cfg, const void* x, const int32_t* sorted_ids, const int32_t* scalars,
                void* x_perm, moe_stream_t stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->T == 0) return MOE_OK;
    if (!x || !sorted_ids || !scalars || !x_perm || !aligned16(x) || !aligned16(x_perm)) return MOE_ERR_ARG;
    return status_of(launch_permute(cfg->H, cfg->K, cfg->dtype, p_max(cfg), x, sorted_ids, scalars, x_perm,
                                    (cudaStream_t)stream));
}

int moe_grouped_ffn(const moe_config_t* cfg, const void* x_perm, const void* w13, const void* w2,
                    const int32_t* offsets, void* act, void* y_perm, void* workspace, size_t ws_bytes,
                    moe_stream_t stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->T == 0) return MOE_OK;
    if (!x_perm || !w13 || !w2 || !offsets || !act || !y_perm || !workspace) return MOE_ERR_ARG;
    if (!aligned16(x_perm) || !aligned16(w13) || !aligned16(w2) || !aligned16(act) || !aligned16(y_perm) ||
        !aligned16(workspace))
        return MOE_ERR_ARG;
    DeviceInfo d;
    if ((rc = current_device(&d)) != 0) return status_of(rc);
    if (ws_bytes < ctl_block_bytes(d.num_sms)) return MOE_ERR_WORKSPACE;
    return status_of(run_ffn(x_perm, p_max(cfg), offsets, cfg->E, 0, cfg->H, cfg->I, cfg->dtype, w13, w2, act,
                             y_perm, routed_max_n(cfg), gemm_ctl(workspace, d.num_sms), (cudaStream_t)stream,
                             routed_max_chunks(cfg)));
}

int moe_grouped_ffn_fp8(const moe_config_t* cfg, const uint8_t* x_codes, const float* x_scales,
                        const uint8_t* w13_q, const float* w13_s, const uint8_t* w2_q, const float* w2_s,
                        const int32_t* offsets, void* act, void* y_perm, void* workspace, size_t ws_bytes,
                        moe_stream_t stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->dtype != 0 || cfg->H % 16 || cfg->I % 16) return MOE_ERR_ARG;
    if (cfg->T == 0) return MOE_OK;
    if (!x_codes || !x_scales || !w13_q || !w13_s || !w2_q || !w2_s || !offsets || !act || !y_perm || !workspace)
        return MOE_ERR_ARG;
    if (!aligned16(x_codes) || !aligned16(w13_q) || !aligned16(w2_q) || !aligned16(act) || !aligned16(y_perm) ||
        !aligned16(workspace))
        return MOE_ERR_ARG;
    if (routed_max_n_avg(cfg) > 128) return MOE_ERR_ARG;
    DeviceInfo d;
    if ((rc = current_device(&d)) != 0) return status_of(rc);
    if (ws_bytes < ctl_block_bytes(d.num_sms)) return MOE_ERR_WORKSPACE;
    return status_of(run_ffn(x_codes, p_max(cfg), offsets, cfg->E, 0, cfg->H, cfg->I, cfg->dtype, w13_q, w2_q, act,
                             y_perm, routed_max_n_avg(cfg), gemm_ctl(workspace, d.num_sms), (cudaStream_t)stream,
                             routed_max_chunks(cfg), 0, 0, w13_s, w2_s, x_scales));
}

int moe_grouped_gate_up(const moe_config_t* cfg, const void* x_perm, const void* w13, const int32_t* offsets,
                        void* act, void* workspace, size_t ws_bytes, moe_stream_t stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->T == 0) return MOE_OK;
    if (!x_perm || !w13 || !offsets || !act || !workspace) return MOE_ERR_ARG;
    if (!aligned16(x_perm) || !aligned16(w13) || !aligned16(act) || !aligned16(workspace)) return MOE_ERR_ARG;
    DeviceInfo d;
    if ((rc = current_device(&d)) != 0) return status_of(rc);
    if (ws_bytes < ctl_block_bytes(d.num_sms)) return MOE_ERR_WORKSPACE;
    return status_of(launch_gemm(gate_up_launch(x_perm, p_max(cfg), offsets, cfg->E, 0, cfg->H, cfg->I, cfg->dtype,
                                                w13, act, routed_max_n(cfg)),
                                 gemm_ctl(workspace, d.num_sms), (cudaStream_t)stream));
}

int moe_grouped_down(const moe_config_t* cfg, const void* act, const void* w2, const int32_t* offsets, void* y_perm,
                     void* workspace, size_t ws_bytes, moe_stream_t stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->T == 0) return MOE_OK;
    if (!act || !w2 || !offsets || !y_perm || !workspace) return MOE_ERR_ARG;
    if (!aligned16(act) || !aligned16(w2) || !aligned16(y_perm) || !aligned16(workspace)) return MOE_ERR_ARG;
    DeviceInfo d;
    if ((rc = current_device(&d)) != 0) return status_of(rc);
    if (ws_bytes < ctl_block_bytes(d.num_sms)) return MOE_ERR_WORKSPACE;
    return status_of(launch_gemm(down_launch(act, p_max(cfg), offsets, cfg->E, 0, cfg->H, cfg->I, cfg->dtype, w2,
                                             y_perm, routed_max_n(cfg)),
                                 gemm_ctl(workspace, d.num_sms), (cudaStream_t)stream));
}

int moe_combine(const moe_config_t* cfg, const void* y_perm, const int32_t* pos, const float* topk_w,
                const void* shared_out, void* out, moe_stream_t stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->T == 0) return MOE_OK;
    if (!y_perm || !pos || !topk_w || !out || !aligned16(y_perm) || !aligned16(out) ||
        (shared_out && !aligned16(shared_out)))
        return MOE_ERR_ARG;
    return status_of(launch_combine(cfg->T, cfg->H, cfg->K, cfg->dtype, y_perm, pos, topk_w, shared_out, out,
                                    (cudaStream_t)stream));
}

int moe_layer_forward(const moe_config_t* cfg, const void* x, const void* w_router, const void* w13, const void* w2,
                      const void* w13_shared, const void* w2_shared, const float* logits_override, void* out,
                      void* workspace, size_t ws_bytes, int32_t* stats_out, moe_stream_t stream) {
    return moe_layer_forward_k(cfg, x, w_router, w13, w2, w13_shared, w2_shared, logits_override, nullptr, out,
                               workspace, ws_bytes, stats_out, stream);
}

namespace {
struct Fp8Scales {
    const float *s13, *s2, *s13_sh, *s2_sh;
};
}  // namespace

// stage 0: the whole layer; stage 1 (TP over I, overlapped all-reduce): up to
// the routed experts' gate/up and the whole shared FFN, no down projection and
// no combine (those run per output-feature block in moe_layer_forward_partial_down)
static int layer_forward_impl(const moe_config_t* cfg, const void* x, const void* w_router, const void* w13,
                              const void* w2, const void* w13_shared, const void* w2_shared,
                              const Fp8Scales* fp8, const float* logits_override, const int32_t* k_per_token,
                              void* out, void* workspace, size_t ws_bytes, int32_t* stats_out, moe_stream_t stream,
                              bool out_f32 = false, int stage = 0);

int moe_layer_forward_k(const moe_config_t* cfg, const void* x, const void* w_router, const void* w13,
                        const void* w2, const void* w13_shared, const void* w2_shared, const float* logits_override,
                        const int32_t* k_per_token, void* out, void* workspace, size_t ws_bytes, int32_t* stats_out,
                        moe_stream_t stream) {
    return layer_forward_impl(cfg, x, w_router, w13, w2, w13_shared, w2_shared, nullptr, logits_override,
                              k_per_token, out, workspace, ws_bytes, stats_out, stream);
}

int moe_layer_forward_fp8(const moe_config_t* cfg, const void* x, const void* w_router, const uint8_t* w13_q,
                          const float* w13_s, const uint8_t* w2_q, const float* w2_s, const uint8_t* w13_shared_q,
                          const float* w13_shared_s, const uint8_t* w2_shared_q, const float* w2_shared_s,
                          const float* logits_override, const int32_t* k_per_token, void* out, void* workspace,
                          size_t ws_bytes, int32_t* stats_out, moe_stream_t stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->dtype != 0) return MOE_ERR_ARG;  // bf16 activations
    if (cfg->T == 0) return MOE_OK;
    const long long I_sh = (long long)cfg->n_shared * cfg->I_shared;
    if (!w13_s || !w2_s || (I_sh > 0 && (!w13_shared_s || !w2_shared_s))) return MOE_ERR_ARG;
    if (cfg->H % 16 || cfg->I % 16 || I_sh % 16) return MOE_ERR_ARG;  // 16-byte rows of codes
    // decode sizes: the routed and shared FFNs must run on the fused kernel
    if (routed_max_n_avg(cfg) > 128 || (I_sh > 0 && pick_max_n(cfg->T) > 128)) return MOE_ERR_ARG;
    const Fp8Scales sc{w13_s, w2_s, w13_shared_s, w2_shared_s};
    return layer_forward_impl(cfg, x, w_router, w13_q, w2_q, w13_shared_q, w2_shared_q, &sc, logits_override,
                              k_per_token, out, workspace, ws_bytes, stats_out, stream);
}

}  // extern "C"

static int layer_forward_impl(const moe_config_t* cfg, const void* x, const void* w_router, const void* w13,
                              const void* w2, const void* w13_shared, const void* w2_shared,
                              const Fp8Scales* fp8, const float* logits_override, const int32_t* k_per_token,
                              void* out, void* workspace, size_t ws_bytes, int32_t* stats_out, moe_stream_t stream,
                              bool out_f32, int stage) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->T == 0) return MOE_OK;
    const long long I_sh = (long long)cfg->n_shared * cfg->I_shared;
    const bool front = stage == 1;
    if (front && (fp8 || routed_max_n(cfg) <= 128)) return MOE_ERR_ARG;  // the two-launch expert FFN only
    if (!x || !w_router || !w13 || (!w2 && !front) || (!out && !front) || !workspace) return MOE_ERR_ARG;
    if (I_sh > 0 && (!w13_shared || !w2_shared)) return MOE_ERR_ARG;
    if (!aligned16(x) || !aligned16(w_router) || !aligned16(w13) || (!front && !aligned16(w2)) ||
        (!front && !aligned16(out)) || !aligned16(workspace) ||
        (I_sh > 0 && (!aligned16(w13_shared) || !aligned16(w2_shared))))
        return MOE_ERR_ARG;
    DeviceInfo d;
    if ((rc = current_device(&d)) != 0) return status_of(rc);
    const Layout L = layout(cfg, d.num_sms);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    const GemmCtl ctl = gemm_ctl(at<uint8_t>(workspace, L.ctl), d.num_sms);
    float* logits = at<float>(workspace, L.logits);
    int32_t* ids = at<int32_t>(workspace, L.ids);
    float* w = at<float>(workspace, L.w);
    int32_t* counts = at<int32_t>(workspace, L.counts);
    int32_t* offsets = at<int32_t>(workspace, L.offsets);
    int32_t* scalars = at<int32_t>(workspace, L.scalars);
    int32_t* sorted_ids = at<int32_t>(workspace, L.sorted_ids);
    int32_t* block_expert = at<int32_t>(workspace, L.block_expert);
    int32_t* pos = at<int32_t>(workspace, L.pos);
    void* x_perm = at<void>(workspace, L.x_perm);
    void* act = at<void>(workspace, L.act);
    void* y_perm = x_perm;
    const long long P = p_max(cfg);

    // shared experts first, on the side stream, when they run beside the routed ones
    SideStream* side = nullptr;
    std::unique_lock<std::mutex> side_lock;
    const void* sh = nullptr;
    int n_sh = 0;
    if (I_sh > 0) {
        SideStream& sd = g_side[d.device];
        side_lock = std::unique_lock<std::mutex>(sd.mu);
        n_sh = shared_sms(cfg, d.num_sms);
        if (n_sh > 0 && side_ready(sd)) {
            if (cudaEventRecord(sd.fork, s) != cudaSuccess || cudaStreamWaitEvent(sd.s, sd.fork, 0) != cudaSuccess) {
                cudaGetLastError();
                return MOE_ERR_CUDA;
            }
            GemmCtl ctl_sh = gemm_ctl(at<uint8_t>(workspace, L.ctl_sh), d.num_sms);
            ctl_sh.status = ctl.status + 1;  // the header's second status word
            void* sh_out = at<void>(workspace, L.sh_out);
            const void* x_sh = x;
            if (fp8) {  // the FP8 path's token operand: x split into E4M3 hi and lo codes
                x_sh = at<void>(workspace, L.x16);
                if ((rc = launch_split_e4m3(cfg->H, 1, cfg->T, x, nullptr, nullptr, at<uint8_t>(workspace, L.x16),
                                            cfg->T, at<float>(workspace, L.sh_scale), sd.s)) != 0) {
                    cudaEventRecord(sd.join, sd.s);
                    cudaStreamWaitEvent(s, sd.join, 0);
                    return status_of(rc);
                }
            }
            rc = run_ffn(x_sh, cfg->T, nullptr, 1, cfg->T, cfg->H, (int)I_sh, cfg->dtype, w13_shared, w2_shared,
                         at<void>(workspace, L.act_sh), sh_out, pick_max_n(cfg->T), ctl_sh, sd.s,
                         dense_max_chunks(cfg->T), n_sh, n_sh, fp8 ? fp8->s13_sh : nullptr,
                         fp8 ? fp8->s2_sh : nullptr, fp8 ? at<float>(workspace, L.sh_scale) : nullptr);
            if (cudaEventRecord(sd.join, sd.s) != cudaSuccess) {
                cudaGetLastError();
                return MOE_ERR_CUDA;
            }
            side = &sd;
            if (rc != 0) {
                cudaStreamWaitEvent(s, sd.join, 0);
                return status_of(rc);
            }
            sh = sh_out;
        } else {
            side_lock.unlock();
        }
    }
    // Every return from here on makes the caller's stream wait for the side
    // stream first, so that a capturing caller stream stays joined.
    struct JoinOnExit {
        SideStream* side;
        cudaStream_t s;
        ~JoinOnExit() {
            if (side && cudaStreamWaitEvent(s, side->join, 0) != cudaSuccess) cudaGetLastError();
        }
    };
    JoinOnExit join_guard{side, s};
    // The router and routed GEMMs take the SMs the shared experts leave.  The
    // routed fused FFN fetches its work dynamically: beside a fused (one-launch)
    // shared FFN it launches a block per SM, and those that find no free SM
    // start when the shared experts' blocks exit; beside the shared GEMM pair it
    // keeps to its share, so that the shared down GEMM finds its SMs free.
    const int n_routed = side ? d.num_sms - n_sh : 0;
    const int n_routed_ffn = side && pick_max_n(cfg->T) > 128 ? n_routed : 0;
    if (small_route(cfg)) {
        // router logits, top-K and alignment in one launch (decode-sized batches)
        int* route_ctr = reinterpret_cast<int*>(at<uint8_t>(workspace, L.ctl)) + 16;  // in the control header
        if ((rc = launch_route_small(cfg->T, cfg->H, cfg->E, cfg->K, cfg->score_fn, cfg->renorm, cfg->tile_B,
                                     cfg->pad_mode, P,
                                     cfg->dtype, x, w_router, logits_override, k_per_token,
                                     at<float>(workspace, L.route_part),
                                     logits, ids, w, counts, offsets, sorted_ids, block_expert, pos, scalars,
                                     stats_out, route_ctr, s)) != 0)
            return status_of(rc);
    } else if (router_cc_fits(cfg->H, cfg->E, cfg->dtype)) {
        // a small router matrix (E * H fits shared memory): router logits on the
        // CUDA cores, top-K and alignment in the same launch
        RouteCcArgs a{};
        a.T = cfg->T;
        a.H = cfg->H;
        a.E = cfg->E;
        a.K = cfg->K;
        a.score_fn = cfg->score_fn;
        a.renorm = cfg->renorm;
        a.B = cfg->tile_B;
        a.mode = cfg->pad_mode;
        a.dtype = cfg->dtype;
        a.P_max = P;
        a.x = x;
        a.w_r = w_router;
        a.logits_override = logits_override;
        a.k_per_token = k_per_token;
        a.logits = logits;
        a.ids = ids;
        a.w = w;
        a.counts = counts;
        a.offsets = offsets;
        a.sorted_ids = sorted_ids;
        a.block_expert = block_expert;
        a.pos = pos;
        a.scalars = scalars;
        a.stats_copy = stats_out;
        a.done_ctr = reinterpret_cast<int*>(at<uint8_t>(workspace, L.ctl)) + 16;  // in the control header
        if ((rc = launch_route_cc(a, s)) != 0) return status_of(rc);
    } else {
        // the tensor-core router GEMM, then top-K and the alignment
        GemmLaunch g{};
        g.x = x;
        g.x_rows = cfg->T;
        g.w = w_router;
        g.w_rows = cfg->E;
        g.kdim = cfg->H;
        g.n_out = cfg->E;
        g.n_groups = 1;
        g.seg_rows = cfg->T;
        g.out_f32 = true;
        g.out = logits;
        g.out_ld = cfg->E;
        g.dtype = cfg->dtype;
        router_tiling(g, cfg->T);
        g.sms = n_routed;
        if ((rc = launch_gemm(g, ctl, s)) != 0) return status_of(rc);
        if ((rc = launch_topk(cfg->T, cfg->E, cfg->K, cfg->score_fn, cfg->renorm,
                              logits_override ? logits_override : logits, k_per_token, ids, w, s)) != 0)
            return status_of(rc);
        if ((rc = launch_align(cfg->T, cfg->K, cfg->E, cfg->tile_B, cfg->pad_mode, P, ids, counts, offsets,
                               sorted_ids, block_expert,
                               pos, scalars, stats_out, s)) != 0)
            return status_of(rc);
    }
    if (fp8) {
        // the permuted token rows split into E4M3 hi and lo codes with their scales;
        // the expert outputs get their own rows (other chunks still read the codes)
        if ((rc = launch_split_e4m3(cfg->H, cfg->K, P, x, sorted_ids, scalars, static_cast<uint8_t*>(x_perm), P,
                                    at<float>(workspace, L.x_scale), s)) != 0)
            return status_of(rc);
        y_perm = at<void>(workspace, L.y8);
    } else if ((rc = launch_permute(cfg->H, cfg->K, cfg->dtype, P, x, sorted_ids, scalars, x_perm, s)) != 0) {
        return status_of(rc);
    }
    if (front) {
        GemmLaunch g = gate_up_launch(x_perm, P, offsets, cfg->E, 0, cfg->H, cfg->I, cfg->dtype, w13, act,
                                      routed_max_n(cfg));
        g.sms = n_routed;
        if ((rc = launch_gemm(g, ctl, s)) != 0) return status_of(rc);
    } else if ((rc = run_ffn(x_perm, P, offsets, cfg->E, 0, cfg->H, cfg->I, cfg->dtype, w13, w2, act, y_perm,
                             fp8 ? routed_max_n_avg(cfg) : routed_max_n(cfg), ctl, s, routed_max_chunks(cfg),
                             n_routed, n_routed_ffn,
                             fp8 ? fp8->s13 : nullptr, fp8 ? fp8->s2 : nullptr,
                             fp8 ? at<float>(workspace, L.x_scale) : nullptr)) != 0) {
        return status_of(rc);
    }
    if (I_sh > 0 && !side) {
        void* sh_out = at<void>(workspace, L.sh_out);
        const void* x_sh = x;
        if (fp8) {
            x_sh = at<void>(workspace, L.x16);
            if ((rc = launch_split_e4m3(cfg->H, 1, cfg->T, x, nullptr, nullptr, at<uint8_t>(workspace, L.x16), cfg->T,
                                        at<float>(workspace, L.sh_scale), s)) != 0)
                return status_of(rc);
        }
        if ((rc = run_ffn(x_sh, cfg->T, nullptr, 1, cfg->T, cfg->H, (int)I_sh, cfg->dtype, w13_shared, w2_shared,
                          at<void>(workspace, L.act_sh), sh_out, pick_max_n(cfg->T), ctl, s,
                          dense_max_chunks(cfg->T), 0, 0, fp8 ? fp8->s13_sh : nullptr,
                          fp8 ? fp8->s2_sh : nullptr, fp8 ? at<float>(workspace, L.sh_scale) : nullptr)) != 0)
            return status_of(rc);
        sh = sh_out;
    }
    if (side) {
        join_guard.side = nullptr;
        if (cudaStreamWaitEvent(s, side->join, 0) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
    }
    if (front) return MOE_OK;  // act, the routing and the shared output wait in the workspace
    return status_of(launch_combine(cfg->T, cfg->H, cfg->K, cfg->dtype, y_perm, pos, w, sh, out, s, out_f32));
}

extern "C" {

// ------------------------------------------------ tensor parallelism over I

int moe_layer_forward_partial(const moe_config_t* cfg, const void* x, const void* w_router, const void* w13,
                              const void* w2, const void* w13_shared, const void* w2_shared,
                              const float* logits_override, const int32_t* k_per_token, float* out_partial,
                              void* workspace, size_t ws_bytes, int32_t* stats_out, moe_stream_t stream) {
    return layer_forward_impl(cfg, x, w_router, w13, w2, w13_shared, w2_shared, nullptr, logits_override,
                              k_per_token, out_partial, workspace, ws_bytes, stats_out, stream, true);
}

int moe_layer_forward_partial_front(const moe_config_t* cfg, const void* x, const void* w_router, const void* w13,
                                    const void* w13_shared, const void* w2_shared, const float* logits_override,
                                    const int32_t* k_per_token, void* workspace, size_t ws_bytes, int32_t* stats_out,
                                    moe_stream_t stream) {
    return layer_forward_impl(cfg, x, w_router, w13, nullptr, w13_shared, w2_shared, nullptr, logits_override,
                              k_per_token, nullptr, workspace, ws_bytes, stats_out, stream, true, 1);
}

int moe_layer_forward_partial_down(const moe_config_t* cfg, const void* w2, int chunk, int n_chunks, float* part,
                                   void* workspace, size_t ws_bytes, moe_stream_t stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (n_chunks < 1 || chunk < 0 || chunk >= n_chunks || cfg->H % n_chunks) return MOE_ERR_ARG;
    const int eb = elt_bytes(cfg->dtype);
    const int Hc = cfg->H / n_chunks, c0 = chunk * Hc;
    if ((Hc * eb) % 16 || Hc % 4) return MOE_ERR_ARG;  // 16-byte vectors in, float4 out
    if (routed_max_n(cfg) <= 128) return MOE_ERR_ARG;   // the two-launch expert FFN only
    if (cfg->T == 0) return MOE_OK;
    if (!w2 || !part || !workspace || !aligned16(w2) || !aligned16(part) || !aligned16(workspace)) return MOE_ERR_ARG;
    DeviceInfo d;
    if ((rc = current_device(&d)) != 0) return status_of(rc);
    const Layout L = layout(cfg, d.num_sms);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    const GemmCtl ctl = gemm_ctl(at<uint8_t>(workspace, L.ctl), d.num_sms);
    const long long I_sh = (long long)cfg->n_shared * cfg->I_shared;
    uint8_t* y_perm = at<uint8_t>(workspace, L.x_perm);
    // output features [c0, c0 + Hc) of every expert: rows c0 .. of w2 [E, H, I]
    // with the expert stride kept, into the same columns of y_perm
    GemmLaunch g = down_launch(at<void>(workspace, L.act), p_max(cfg), at<int32_t>(workspace, L.offsets), cfg->E, 0,
                               cfg->H, cfg->I, cfg->dtype, static_cast<const uint8_t*>(w2) + (size_t)c0 * cfg->I * eb,
                               y_perm + (size_t)c0 * eb, routed_max_n(cfg));
    g.n_out = Hc;
    g.w_rows = (long long)cfg->E * cfg->H - c0;
    if ((rc = launch_gemm(g, ctl, s)) != 0) return status_of(rc);
    return status_of(launch_combine(cfg->T, cfg->H, cfg->K, cfg->dtype, y_perm, at<int32_t>(workspace, L.pos),
                                    at<float>(workspace, L.w), I_sh > 0 ? at<void>(workspace, L.sh_out) : nullptr,
                                    part, s, true, c0, Hc));
}

int moe_tp_gather(int n_chunks, const float* const* parts, int T, int H, int dtype, void* out, moe_stream_t stream) {
    if (n_chunks < 1 || n_chunks > kTpMaxParts || T < 0 || H <= 0 || H % n_chunks || (H / n_chunks) % 4 || !parts)
        return MOE_ERR_ARG;
    if (dtype != 0 && dtype != 1) return MOE_ERR_ARG;
    if (T == 0) return MOE_OK;
    if (!out || !aligned16(out)) return MOE_ERR_ARG;
    for (int c = 0; c < n_chunks; ++c)
        if (!parts[c] || !aligned16(parts[c])) return MOE_ERR_ARG;
    return status_of(launch_tp_gather(n_chunks, parts, T, H, dtype, out, (cudaStream_t)stream));
}

int moe_tp_reduce(int n_parts, const float* const* parts, long long count, int dtype, void* out,
                  moe_stream_t stream) {
    if (n_parts < 1 || n_parts > kTpMaxParts || count < 0 || count % 4 || !parts || !out) return MOE_ERR_ARG;
    if (dtype != 0 && dtype != 1) return MOE_ERR_ARG;
    if (count == 0) return MOE_OK;
    for (int r = 0; r < n_parts; ++r)
        if (!parts[r] || !aligned16(parts[r])) return MOE_ERR_ARG;
    if (!aligned16(out)) return MOE_ERR_ARG;
    return status_of(launch_tp_reduce(n_parts, parts, count, dtype, out, (cudaStream_t)stream));
}

int moe_tp_shard(int E, int H, int I, int dtype, int rank, int n_ranks, const void* w13, const void* w2,
                 void* w13_local, void* w2_local, moe_stream_t stream) {
    const int eb = elt_bytes(dtype);
    if (eb == 0 || E < 1 || H < 1 || I < 1 || n_ranks < 1 || rank < 0 || rank >= n_ranks || I % n_ranks)
        return MOE_ERR_ARG;
    if (!w13 || !w2 || !w13_local || !w2_local) return MOE_ERR_ARG;
    const size_t n = (size_t)(I / n_ranks);
    const size_t row = (size_t)H * eb;
    cudaStream_t s = (cudaStream_t)stream;
    // w13: the 2E blocks [gate of e, up of e] are I rows apart; each gives its
    // n rows starting at rank * n
    cudaError_t e = cudaMemcpy2DAsync(w13_local, n * row, static_cast<const uint8_t*>(w13) + rank * n * row,
                                      (size_t)I * row, n * row, (size_t)2 * E, cudaMemcpyDeviceToDevice, s);
    // w2: the E*H rows of I columns each give columns [rank * n, rank * n + n)
    if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(w2_local, n * eb, static_cast<const uint8_t*>(w2) + rank * n * eb, (size_t)I * eb,
                              n * eb, (size_t)E * H, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}


int dense_ffn(int T, int H, int I, int dtype, const void* x, const void* w13, const void* w2, void* out,
              void* workspace, size_t ws_bytes, moe_stream_t stream) {
    const int eb = elt_bytes(dtype);
    if (eb == 0 || T < 0 || H <= 0 || I <= 0 || H % (16 / eb) || I % (16 / eb)) return MOE_ERR_ARG;
    if ((long long)2 * I >= (1LL << 31)) return MOE_ERR_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !w13 || !w2 || !out || !workspace) return MOE_ERR_ARG;
    if (!aligned16(x) || !aligned16(w13) || !aligned16(w2) || !aligned16(out) || !aligned16(workspace))
        return MOE_ERR_ARG;
    DeviceInfo d;
    int rc = current_device(&d);
    if (rc != 0) return status_of(rc);
    const size_t ctl_bytes = align256(ctl_block_bytes(d.num_sms));
    if (ws_bytes < ctl_bytes + (size_t)eb * T * I) return MOE_ERR_WORKSPACE;
    void* act = at<void>(workspace, ctl_bytes);
    return status_of(run_ffn(x, T, nullptr, 1, T, H, I, dtype, w13, w2, act, out, pick_max_n(T),
                             gemm_ctl(workspace, d.num_sms), (cudaStream_t)stream, dense_max_chunks(T)));
}

int dense_ffn_fp8(int T, int H, int I, const void* x, const uint8_t* w13_q, const float* w13_s, const uint8_t* w2_q,
                  const float* w2_s, void* out, void* workspace, size_t ws_bytes, moe_stream_t stream) {
    if (T < 0 || H <= 0 || I <= 0 || H % 16 || I % 16) return MOE_ERR_ARG;
    if ((long long)2 * I >= (1LL << 31)) return MOE_ERR_ARG;
    if (T == 0) return MOE_OK;
    if (pick_max_n(T) > 128) return MOE_ERR_ARG;  // decode sizes: the fused kernel
    if (!x || !w13_q || !w13_s || !w2_q || !w2_s || !out || !workspace) return MOE_ERR_ARG;
    if (!aligned16(x) || !aligned16(w13_q) || !aligned16(w2_q) || !aligned16(out) || !aligned16(workspace))
        return MOE_ERR_ARG;
    DeviceInfo d;
    int rc = current_device(&d);
    if (rc != 0) return status_of(rc);
    const size_t ctl_bytes = align256(ctl_block_bytes(d.num_sms));
    const size_t act_bytes = align256((size_t)2 * T * I);
    const size_t code_bytes = align256((size_t)2 * T * H);
    if (ws_bytes < ctl_bytes + act_bytes + code_bytes + sizeof(float) * (size_t)T) return MOE_ERR_WORKSPACE;
    void* act = at<void>(workspace, ctl_bytes);
    // the token operand: x split into E4M3 hi and lo codes, and the rows' scales
    uint8_t* codes = at<uint8_t>(workspace, ctl_bytes + act_bytes);
    float* scales = at<float>(workspace, ctl_bytes + act_bytes + code_bytes);
    if ((rc = launch_split_e4m3(H, 1, T, x, nullptr, nullptr, codes, T, scales, (cudaStream_t)stream)) != 0)
        return status_of(rc);
    return status_of(run_ffn(codes, T, nullptr, 1, T, H, I, 0, w13_q, w2_q, act, out, pick_max_n(T),
                             gemm_ctl(workspace, d.num_sms), (cudaStream_t)stream, dense_max_chunks(T), 0, 0, w13_s,
                             w2_s, scales));
}

size_t dense_ffn_fp8_workspace_size(int T, int H, int I) {
    if (T < 0 || H <= 0 || I <= 0) return 0;
    DeviceInfo d;
    if (current_device(&d) != 0) return 0;
    return align256(ctl_block_bytes(d.num_sms)) + align256((size_t)2 * T * I) + align256((size_t)2 * T * H) +
           sizeof(float) * (size_t)T;
}

int moe_permute_e4m3x2(const moe_config_t* cfg, const void* x, const int32_t* sorted_ids, const int32_t* scalars,
                       uint8_t* x_codes, float* x_scales, moe_stream_t stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->dtype != 0) return MOE_ERR_ARG;
    if (cfg->T == 0) return MOE_OK;
    if (!x || !sorted_ids || !scalars || !x_codes || !x_scales || !aligned16(x) || !aligned16(x_codes))
        return MOE_ERR_ARG;
    const long long P = p_max(cfg);
    return status_of(launch_split_e4m3(cfg->H, cfg->K, P, x, sorted_ids, scalars, x_codes, P, x_scales,
                                       (cudaStream_t)stream));
}

int moe_quantize_fp8(int64_t rows, int cols, int dtype, const void* w, uint8_t* q, float* scales,
                     moe_stream_t stream) {
    if (rows < 0 || rows > INT32_MAX || cols <= 0 || cols % 16 || (dtype != 0 && dtype != 1)) return MOE_ERR_ARG;
    if (rows == 0) return MOE_OK;
    if (!w || !q || !scales) return MOE_ERR_ARG;
    DeviceInfo d;
    int rc = current_device(&d);
    if (rc != 0) return status_of(rc);
    return status_of(launch_quantize_fp8(rows, cols, dtype, w, q, scales, (cudaStream_t)stream));
}

int moe_check_status(void* workspace, moe_stream_t stream) {
    if (!workspace) return MOE_ERR_ARG;
    DeviceInfo d;
    int rc = current_device(&d);
    if (rc != 0) return status_of(rc);
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    // word 0: every kernel on the caller's stream; word 1: the shared experts'
    // kernels of moe_layer_forward, whose control block follows the first
    unsigned st[2] = {0, 0};
    if (cudaMemcpy(st, workspace, sizeof st, cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    auto rezero = [&](void* block) {
        // status and stream-K counters, and the fused FFN's counters
        const GemmCtl c = gemm_ctl(block, d.num_sms);
        const bool ok =
            cudaMemset(block, 0, gemm_ctl_zero_bytes(d.num_sms)) == cudaSuccess &&
            cudaMemset(c.ffn_ctl, 0, ctl_block_bytes(d.num_sms) - ((uint8_t*)c.ffn_ctl - (uint8_t*)block)) ==
                cudaSuccess;
        if (!ok) cudaGetLastError();
        return ok;
    };
    const unsigned kBad = kStatusTimeout | kStatusCapacity;
    if ((st[0] | st[1]) & kBad) {
        if (!rezero(workspace)) return MOE_ERR_CUDA;
        if ((st[1] & kBad) && !rezero(static_cast<uint8_t*>(workspace) + align256(ctl_block_bytes(d.num_sms))))
            return MOE_ERR_CUDA;
        // a wait that ran out is a timeout; work that did not fit the kernel's
        // tables came from segment offsets inconsistent with the configuration
        return ((st[0] | st[1]) & kStatusTimeout) ? MOE_ERR_TIMEOUT : MOE_ERR_ARG;
    }
    return MOE_OK;
}

void moe_set_wait_limit_ns(uint64_t ns) { g_wait_limit.store(ns ? ns : 2000000000ull); }

int moe_set_token_tile_cap(int n) {
    if (n != 0 && n != 32 && n != 64 && n != 128 && n != 256) return MOE_ERR_ARG;
    set_token_tile_cap(n);
    return MOE_OK;
}

void moe_set_programmatic_launch(int enable) { set_pdl(enable != 0); }

int moe_set_split_tail(int mode) {
    if (mode != 0 && mode != 1) return MOE_ERR_ARG;
    set_split_tail(mode);
    return MOE_OK;
}

int moe_set_shared_sms(int n) {
    if (n < -1) return MOE_ERR_ARG;
    g_shared_sms.store(n);
    return MOE_OK;
}

int moe_shared_sms(const moe_config_t* cfg) {
    if (check_cfg(cfg) != MOE_OK || (long long)cfg->n_shared * cfg->I_shared == 0) return 0;
    DeviceInfo d;
    if (current_device(&d) != 0) return 0;
    return shared_sms(cfg, d.num_sms);
}

int moe_ffn_fused(const moe_config_t* cfg) {
    if (check_cfg(cfg) != MOE_OK) return 0;
    return routed_max_n(cfg) <= 128 ? 1 : 0;
}

void moe_set_cta_pairs(int enable) { set_cta_pairs(enable != 0); }

void moe_debug_withhold_first_load(int enable) { g_withhold.store(enable ? 1 : 0); }

uint64_t moe_kernel_launch_count(void) { return g_launches.load(); }

}  // extern "C"
