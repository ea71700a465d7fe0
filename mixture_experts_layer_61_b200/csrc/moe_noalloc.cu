// moe_noalloc.cu -- a router GEMM entry point that needs no workspace from
// the caller.
//
// Some callers cannot allocate device memory at the moment they enqueue
// work: a plugin inside another inference engine whose enqueue hook must not
// allocate, or a runtime that plans every byte of device memory up front.
// For them, moe_router_gemm_noalloc runs the same tensor-core router GEMM as
// moe_router_gemm but keeps its scratch -- the status word, the stream-K tile
// counters and the partial tiles -- in a fixed array in the library's own
// device memory.  That array (kScratchBytes, about 5 MiB) exists on every GPU
// that loads the library, until the process exits.
//
// Limits: at most kMaxTokens tokens per call (decode-sized batches, which
// keep each partial tile at 128 x 32 fp32) and at most kMaxSms SMs.  All calls
// share the one array: two calls that overlap on the GPU (different streams,
// no ordering between them) race on it.
//
// A bounded device wait that runs out sets the status word inside the array.
// moe_router_gemm_noalloc_status() reads and clears it; the next
// moe_router_gemm_noalloc call clears it too, so read it before that call.
#include "../../include/moe.h"
#include "moe_common.cuh"
#include "moe_internal.h"

#include <mutex>

namespace {

constexpr int kMaxTokens = 32;
constexpr int kMaxSms = 160;
constexpr int kTokenTile = 32;                                  // token-tile cap of the launch
constexpr size_t kSlotBytes = 128ull * kTokenTile * 4ull;        // one partial tile
constexpr size_t kCtlBytes = (moe::kCtlHeaderBytes + sizeof(int) * 2 * kMaxSms + 255) & ~size_t(255);
constexpr size_t kScratchBytes = kCtlBytes + kSlotBytes * 2 * kMaxSms;

// Zero at module load; the status word and counters are cleared again by
// every call before its launch.
static __device__ __align__(256) unsigned char g_router_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];
std::mutex g_mu;

// Device address of g_router_scratch on the current device (looked up once
// per device; the host-side name of the array is not a device address).
int scratch_for(int dev, void** out) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_router_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" int moe_router_gemm_noalloc(const moe_config_t* cfg, const void* x, const void* w_router, float* logits,
                                       moe_stream_t stream) {
    if (!cfg) return MOE_ERR_ARG;
    const int eb = cfg->dtype == 0 ? 2 : (cfg->dtype == 1 ? 4 : 0);
    if (eb == 0 || cfg->T < 0 || cfg->H <= 0 || cfg->H % (16 / eb) != 0 || cfg->E < 1 || cfg->E > 1024)
        return MOE_ERR_ARG;
    if (cfg->T > kMaxTokens) return MOE_ERR_ARG;  // beyond the fixed scratch: use moe_router_gemm
    if (cfg->T == 0) return MOE_OK;
    if (!x || !w_router || !logits) return MOE_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(w_router)) & 15u) return MOE_ERR_ARG;
    moe::DeviceInfo d;
    int rc = moe::current_device(&d);
    if (rc != 0) return rc == -5 ? MOE_ERR_DEVICE : MOE_ERR_CUDA;
    if (d.num_sms > kMaxSms || d.device >= kMaxDevices) return MOE_ERR_DEVICE;
    void* scratch = nullptr;
    if ((rc = scratch_for(d.device, &scratch)) != MOE_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the status word and the stream-K counters must start at zero
    if (cudaMemsetAsync(scratch, 0, moe::gemm_ctl_zero_bytes(d.num_sms), s) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    moe::GemmLaunch g{};
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
    g.max_n = kTokenTile;
    rc = moe::launch_gemm(g, moe::gemm_ctl(scratch, d.num_sms), s);
    return rc == 0 ? MOE_OK : (rc == -1 ? MOE_ERR_ARG : MOE_ERR_CUDA);
}

extern "C" int moe_router_gemm_noalloc_status(moe_stream_t stream) {
    moe::DeviceInfo d;
    int rc = moe::current_device(&d);
    if (rc != 0) return rc == -5 ? MOE_ERR_DEVICE : MOE_ERR_CUDA;
    if (d.num_sms > kMaxSms || d.device >= kMaxDevices) return MOE_ERR_DEVICE;
    void* scratch = nullptr;
    if ((rc = scratch_for(d.device, &scratch)) != MOE_OK) return rc;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    unsigned st = 0;
    if (cudaMemcpy(&st, scratch, sizeof st, cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (st & moe::kStatusTimeout) {
        // the timed-out launch may have left stream-K counters set: clear them with the status word
        if (cudaMemset(scratch, 0, moe::gemm_ctl_zero_bytes(d.num_sms)) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        return MOE_ERR_TIMEOUT;
    }
    return MOE_OK;
}
