// moe_ffn_stream.cuh -- the expert FFN for small per-expert batches (decode):
// gate/up + SwiGLU and down in ONE persistent tcgen05 kernel with dynamic work
// fetching.
//
// At decode sizes the layer is bound by streaming the activated experts'
// weights from HBM (the "weight amplification" of the talk notes' "Decode
// phase").  Two separate GEMM launches each pay a prologue, a pipeline ramp
// and a tail in which the SMs that drew slower HBM service finish last.  Here
// every block repeatedly takes the next work item from a global counter
// (faster SMs simply take more), and the down projection's items follow the
// gate/up items in the same launch, so the down weights start streaming while
// the last gate/up tiles drain.
//
// Work items.  Phase A: gate/up tiles (expert chunk x 128 features), phase B:
// down tiles (expert chunk x 256 features, two weight tiles per stage).  When
// a phase has fewer tiles than about twice the SMs, each tile is cut into S
// K-slices; the slice that completes a tile last (per-tile counter) sums all
// slices' fp32 partials in slice order (deterministic) and runs the epilogue.
// A phase-B item reads the SwiGLU activations of its token chunk, so before
// loading them its producer waits (bounded) until every phase-A tile of that
// chunk has been stored (per-chunk counter).  No block waits on work that is
// not already held by a running block, so the wait always ends.
//
// Roles as in the grouped GEMM (warp 0 TMA, warp 1 TMEM + MMA, warps 2..5
// epilogue); the producer publishes each item id to the other roles through a
// small shared-memory ring.
//
// FP8 weights (kFp8): the weight tiles stream as E4M3 codes (half the bytes),
// 128 rows x 128 codes per tile with the 128-byte swizzle (the same 128-byte
// row pieces as a bf16 tile: 64-code pieces left the weight stream at about
// half the copy bandwidth).
//  * gate/up: the token rows arrive split exactly into two E4M3 terms with a
//    power-of-two scale per row (x = s (hi + lo)); each stage's MMAs are
//    kind::f8f6f4 with both operands in shared memory -- weights x hi, then
//    weights x lo into the same accumulator -- so no code is widened; the
//    epilogue multiplies by the weight row's scale and the token row's s;
//  * down: warps 6..13 widen each stage's two tiles to f16 in registers by
//    moving the code's bits into an f16 pattern (value x 2^-8, exact: E4M3
//    subnormals land on f16 subnormals) and store them into a ring of TMEM
//    buffers, from which the f16 MMA takes its A operand (the activations are
//    f16, two 64-column boxes per stage); the epilogue multiplies each output
//    row by its fp32 row scale x 2^8.
// Widening costs 4 bytes of tensor-memory traffic per weight byte (the f16
// store and the MMA's read): at the gate/up projections, two thirds of the
// bytes, the direct FP8 MMAs avoid it.
// Widening through shared memory instead costs 6 bytes of shared-memory
// traffic per weight (TMA write, read, f16 write, tensor-core read) against 2
// for bf16 weights, which caps the stream below the bf16 rate; through TMEM
// the shared-memory traffic stays at 2 bytes per weight.
// The MMAs run on f16 operands: x_perm arrives in f16 and the SwiGLU
// activations are stored in f16 (the output stays in the activation dtype).
#pragma once

#include <type_traits>

#include "moe_gemm.cuh"

namespace moe {

constexpr int kFfnMaxChunks = 4096;   // token chunks (per-chunk phase-A counters)
constexpr int kFfnTileCtrs = 4096;    // split-tile counters (phase A, then phase B)
constexpr int kFfnRing = 4;
// control ints: [0] work counter, [1] finished blocks, [2, 2+kFfnMaxChunks) chunk
// counters, then kFfnTileCtrs tile counters
constexpr int kFfnCtlInts = 2 + kFfnMaxChunks + kFfnTileCtrs;

struct FfnParams {
    const int32_t* seg_offsets;  // [n_groups + 1] row offsets, or nullptr: one group [0, seg_rows)
    int n_groups;
    int seg_rows;
    int H, I;
    void* act;           // [rows, I] SwiGLU activations (written in phase A, read in phase B)
    void* y;             // [rows, H] output
    int* ctl;            // kFfnCtlInts, zero on entry, left zero
    float* partials;     // split-tile partial slots (up to 8 x gridDim.x)
    unsigned* status;
    uint64_t wait_limit_ns;
    int withhold_first_load;
    int max_slots_phase;  // partial slots available to each phase
    const float* s13;     // FP8 weights: row scales [n_groups * 2I] (gate rows, then up rows), else nullptr
    const float* s2;      // FP8 weights: row scales [n_groups * H], else nullptr
    const float* x_scale; // FP8 weights: the token rows' power-of-two scales (phase A operand)
    long long lo_rows;    // FP8 weights: rows from a token row's hi codes to its lo codes
};

template <typename T, int kMaxN, bool kFp8 = false>
struct FfnCfg {
    // K per stage: 64 bf16 / fp32-as-tf32 elements, or 128 E4M3 codes; either
    // way a weight tile is 128 rows of 128 bytes
    static constexpr int kBK = kFp8 ? 128 : 128 / Elt<T>::kBytes;
    static constexpr int kWTileBytes = 128 * 128;  // a weight tile as it streams in (and, bf16, as the MMA reads it)
    static constexpr int kRawWBytes = kWTileBytes;
    static constexpr int kXBoxRows = 16, kXBoxMid = 64;
    static constexpr int kXBoxes = kFp8 ? 2 : 1;   // 64-column f16 boxes of the token tile per stage (FP8: K 128)
    static constexpr int kXTileBytes = kXBoxes * kMaxN * 128;
    static constexpr int kStageBytes = 2 * kRawWBytes + kXTileBytes;
    static constexpr int kConv = kFp8 ? (kMaxN <= 32 ? 3 : 2) : 0;  // TMEM buffers of widened weights
    static constexpr int kConvCols = 128;  // a stage's two 128 x 128 f16 tiles: 2 x 64 TMEM columns
    static constexpr int kConvThreads = kFp8 ? 256 : 0;   // converter warps 6..13
    static constexpr int kThreads = kFfnThreads + kConvThreads;
    static constexpr int kAccCols = 2 * kMaxN;
    static constexpr int kNumAcc = (kFp8 && kMaxN == 128) ? 1 : 2;  // leaves TMEM room for the weight buffers
    static constexpr int kConvCol0 = kNumAcc * kAccCols;
    static constexpr int kTableBytes = 2 * (kMaxGroups + 1) * 4;
    static constexpr int kMiscBytes = 768;
    static constexpr int kBudget = 227 * 1024 - 1024 - kTableBytes - kMiscBytes;
    static constexpr int kStagesRaw = kBudget / kStageBytes;
    static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kTableBytes + kMiscBytes;
    static_assert(kStageBytes % 1024 == 0, "stages keep the swizzle atoms aligned");
    static_assert(!kFp8 || sizeof(T) == 2, "FP8 weights: 16-bit activations");
    // barriers (full/empty per stage, 2 TMEM pairs, the item ring, the conversion
    // ring, the drain barrier) and the ring / TMEM / flag words fit the misc area
    static_assert((2 * kStages + 2 * kNumAcc + 2 * kFfnRing + 2 * kConv + 1) * 8 + 4 * kFfnRing + 16 <= kMiscBytes,
                  "misc area");
    static constexpr int kSlotFloats = 128 * kAccCols;
    static_assert(kMaxN == 32 || kMaxN == 64 || kMaxN == 128, "decode token tiles");
    static_assert(kAccCols * kNumAcc + kConv * kConvCols <= 512, "TMEM columns");
};

// One phase's split: S slices per tile (S = 1: whole tiles).
__device__ __forceinline__ int ffn_slices(long long tiles, int KI, int G, int max_slots) {
    if (tiles <= 0 || tiles >= 2LL * G) return 1;
    long long s = (2LL * G + tiles - 1) / tiles;
    long long cap = (4LL * G < max_slots ? 4LL * G : max_slots) / tiles;
    if (s > cap) s = cap;
    if (s > 16) s = 16;
    if (s > KI / 4) s = KI / 4;
    return s < 1 ? 1 : (int)s;
}

struct FfnItem {
    int phase;      // 0 gate/up, 1 down
    long long tile; // within the phase
    int slice, S;
    int kb, ke;
    long long slot;  // partial slot (split tiles)
    long long ctr;   // tile counter index (split tiles)
};

__device__ __forceinline__ uint32_t ld_acquire_u32(const int* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Two E4M3 codes at bits [7:0] and [23:16] -> two f16 holding value x 2^-8:
// the sign moves to bit 15, the 4 exponent and 3 mantissa bits to bits 13:7,
// so an E4M3 exponent field e becomes the f16 exponent field e (bias 15 vs 7)
// and e = 0 (subnormal) stays subnormal -- exact for every finite code.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2_scaled(uint32_t two) {
    return ((two << 8) & 0x80008000u) | ((two << 7) & 0x3F803F80u);
}
// 16 codes -> 16 f16 (value x 2^-8) in two 16-byte chunks
__device__ __forceinline__ void e4m3x16_to_f16(const uint4 v, uint4& lo, uint4& hi) {
    lo = make_uint4(e4m3x2_to_f16x2_scaled(__byte_perm(v.x, 0, 0x4140)),
                    e4m3x2_to_f16x2_scaled(__byte_perm(v.x, 0, 0x4342)),
                    e4m3x2_to_f16x2_scaled(__byte_perm(v.y, 0, 0x4140)),
                    e4m3x2_to_f16x2_scaled(__byte_perm(v.y, 0, 0x4342)));
    hi = make_uint4(e4m3x2_to_f16x2_scaled(__byte_perm(v.z, 0, 0x4140)),
                    e4m3x2_to_f16x2_scaled(__byte_perm(v.z, 0, 0x4342)),
                    e4m3x2_to_f16x2_scaled(__byte_perm(v.w, 0, 0x4140)),
                    e4m3x2_to_f16x2_scaled(__byte_perm(v.w, 0, 0x4342)));
}

template <typename T, int kMaxN, bool kFp8 = false>
__global__ void __launch_bounds__(FfnCfg<T, kMaxN, kFp8>::kThreads, 1)
    moe_ffn_stream_kernel(const __grid_constant__ CUtensorMap tm_w13, const __grid_constant__ CUtensorMap tm_w2,
                          const __grid_constant__ CUtensorMap tm_xa, const __grid_constant__ CUtensorMap tm_xa64,
                          const __grid_constant__ CUtensorMap tm_xb, const __grid_constant__ CUtensorMap tm_xb64,
                          const FfnParams p) {
    using C = FfnCfg<T, kMaxN, kFp8>;
    using OutT = T;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stage_base = smem;
    int* seg = reinterpret_cast<int*>(smem + C::kStages * C::kStageBytes);
    int* cbase = seg + (kMaxGroups + 1);
    uint8_t* misc = reinterpret_cast<uint8_t*>(cbase + (kMaxGroups + 1));
    uint64_t* full = reinterpret_cast<uint64_t*>(misc);
    uint64_t* empty = full + C::kStages;
    uint64_t* tfull = empty + C::kStages;
    uint64_t* tempty = tfull + C::kNumAcc;
    uint64_t* ring_full = tempty + C::kNumAcc;
    uint64_t* ring_empty = ring_full + kFfnRing;
    uint64_t* conv_full = ring_empty + kFfnRing;  // C::kConv barriers each (none without FP8 weights)
    uint64_t* conv_empty = conv_full + C::kConv;
    uint64_t* drain_bar = conv_empty + C::kConv;
    int* ring = reinterpret_cast<int*>(drain_bar + 1);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(ring + kFfnRing);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    int* bcast = const_cast<int*>(abort_flag) + 1;
    int* last_block = bcast + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_groups = p.n_groups;
    const uint64_t limit = p.wait_limit_ns;
    int* work_ctr = p.ctl;
    int* done_ctr = p.ctl + 1;
    int* chunk_done = p.ctl + 2;
    int* tile_ctr = p.ctl + 2 + kFfnMaxChunks;

    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < C::kNumAcc; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 128);
        }
        for (int r = 0; r < kFfnRing; ++r) {
            mbar_init(&ring_full[r], 1);
            // the MMA thread, every epilogue thread and (FP8) every converter thread
            mbar_init(&ring_empty[r], 1 + 128 + C::kConvThreads);
        }
        for (int c = 0; c < C::kConv; ++c) {
            mbar_init(&conv_full[c], C::kConvThreads / 32);  // one arrival per converter warp
            mbar_init(&conv_empty[c], 1);
        }
        mbar_init(drain_bar, 1);
        fence_barrier_init();
        *abort_flag = 0;
        tma_prefetch_desc(&tm_w13);
        tma_prefetch_desc(&tm_w2);
        tma_prefetch_desc(&tm_xa);
        tma_prefetch_desc(&tm_xa64);
        tma_prefetch_desc(&tm_xb);
        tma_prefetch_desc(&tm_xb64);
    }
    if (warp == 1) tmem_alloc(tmem_holder, 512);
    pdl_wait();
    for (int g = threadIdx.x; g <= n_groups; g += blockDim.x)
        seg[g] = p.seg_offsets ? p.seg_offsets[g] : (g == 0 ? 0 : p.seg_rows);
    __syncthreads();
    if (warp == 0) {
        int running = 0;
        for (int base = 0; base < n_groups; base += 32) {
            int g = base + lane;
            int n = g < n_groups ? chunks_of(seg[g + 1] - seg[g], kMaxN, 16) : 0;
            int incl = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (g < n_groups) cbase[g] = running + incl - n;
            running += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) cbase[n_groups] = running;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    // ---- the item space (identical in every thread)
    const int G = gridDim.x;
    const long long n_chunks = cbase[n_groups];
    const int NFA = (p.I + 127) / 128, NFB = (p.H + 255) / 256;
    const int KIA = (p.H + C::kBK - 1) / C::kBK, KIB = (p.I + C::kBK - 1) / C::kBK;
    const long long tilesA = n_chunks * NFA, tilesB = n_chunks * NFB;
    const int SA = ffn_slices(tilesA, KIA, G, p.max_slots_phase), SB = ffn_slices(tilesB, KIB, G, p.max_slots_phase);
    const long long nA = tilesA * SA, nB = tilesB * SB;
    const long long total = nA + nB;
    const long long slotsA = SA > 1 ? nA : 0;
    const bool oversize = n_chunks > kFfnMaxChunks || (SA > 1 && tilesA > kFfnTileCtrs / 2) ||
                          (SB > 1 && tilesB > kFfnTileCtrs / 2);

    auto item_of = [&](long long id, FfnItem& it, Tile& t) {
        if (id < nA) {
            it.phase = 0;
            it.tile = id / SA;
            it.slice = (int)(id - it.tile * SA);
            it.S = SA;
            it.kb = (int)((long long)it.slice * KIA / SA);
            it.ke = (int)((long long)(it.slice + 1) * KIA / SA);
            it.slot = id;
            it.ctr = it.tile;
            t = decode_tile_w(it.tile, seg, cbase, n_groups, NFA, 128, 16, 2 * p.I);
        } else {
            const long long j = id - nA;
            it.phase = 1;
            it.tile = j / SB;
            it.slice = (int)(j - it.tile * SB);
            it.S = SB;
            it.kb = (int)((long long)it.slice * KIB / SB);
            it.ke = (int)((long long)(it.slice + 1) * KIB / SB);
            it.slot = slotsA + j;
            it.ctr = kFfnTileCtrs / 2 + it.tile;
            t = decode_tile_w(it.tile, seg, cbase, n_groups, NFB, 256, 16, p.H);
        }
    };

    if (warp == 0) {
        // ------------------------------------------- item fetch + TMA loads
        if (lane == 0) {
            const uint64_t pol_w_once = policy_evict_first();
            const uint64_t pol_w_shared = policy_evict_normal();
            const uint64_t pol_x = policy_evict_last();
            int fills[C::kStages];
#pragma unroll
            for (int s = 0; s < C::kStages; ++s) fills[s] = 0;
            uint32_t kc = 0, n = 0;
            bool withhold = false;  // test hook: armed for work item 0, whichever block takes it
            bool ok = !oversize;
            if (oversize) atomicOr(p.status, kStatusCapacity);  // not a wait: the item space does not fit
            while (true) {
                const int rs = n % kFfnRing;
                const uint32_t rph = (n / kFfnRing) & 1u;
                long long id = -1;
                if (ok) {
                    if (!mbar_wait_bounded(&ring_empty[rs], rph ^ 1u, limit, abort_flag)) {
                        ok = false;
                    } else {
                        id = atomicAdd(work_ctr, 1);
                        if (id >= total) id = -1;
                    }
                }
                if (!ok) {
                    // wake the consumers with the end marker (they may also give up on their own)
                    ring[rs] = -1;
                    mbar_arrive(&ring_full[rs]);
                    break;
                }
                ring[rs] = (int)id;
                mbar_arrive(&ring_full[rs]);
                ++n;
                if (id < 0) break;
                FfnItem it;
                Tile t;
                item_of(id, it, t);
                if (id == 0 && p.withhold_first_load) withhold = true;
                const CUtensorMap* tw = it.phase == 0 ? &tm_w13 : &tm_w2;
                const CUtensorMap* tx = it.phase == 0 ? &tm_xa : &tm_xb;
                const CUtensorMap* tx64 = it.phase == 0 ? &tm_xa64 : &tm_xb64;
                const int second = it.phase == 0 ? p.I : 128;  // up rows, or the next 128 features
                const uint32_t bytes = 2 * C::kRawWBytes + C::kXBoxes * t.mma_n * 128;
                const uint64_t pol_w = t.nch > 1 ? pol_w_shared : pol_w_once;
                auto load_w = [&](int s, int k) {
                    uint8_t* st = stage_base + s * C::kStageBytes;
                    const int kx = k * C::kBK;
                    tma_load_2d(st, tw, &full[s], kx, t.wrow, pol_w);
                    tma_load_2d(st + C::kRawWBytes, tw, &full[s], kx, t.wrow + second, pol_w);
                };
                auto load_x = [&](int s, int k) {
#pragma unroll
                    for (int xb = 0; xb < C::kXBoxes; ++xb) {
                        uint8_t* xs = stage_base + s * C::kStageBytes + 2 * C::kRawWBytes + xb * kMaxN * 128;
                        // FP8 gate/up: box xb holds the hi (0) or lo (1) codes of columns
                        // k*128..+127; otherwise 64 16-bit columns each
                        const bool codes = kFp8 && it.phase == 0;
                        const int kx = codes ? k * C::kBK : k * C::kBK + xb * 64;
                        const int rbase = codes ? (int)(xb * p.lo_rows) : 0;
                        int r = 0;
                        if (kMaxN >= C::kXBoxMid)
                            for (; r + C::kXBoxMid <= t.mma_n; r += C::kXBoxMid)
                                tma_load_2d(xs + r * 128, tx64, &full[s], kx, rbase + t.row0 + r, pol_x);
                        for (; r < t.mma_n; r += C::kXBoxRows)
                            tma_load_2d(xs + r * 128, tx, &full[s], kx, rbase + t.row0 + r, pol_x);
                    }
                };
                int pre = 0;  // stages of this item whose weight tiles went out before the activation wait
                if (it.phase == 1) {
                    // The weights do not depend on phase A: stream the first stages'
                    // weight tiles now, then wait until every gate/up tile of this
                    // token chunk has stored its activations, then load those.
                    const int want = it.ke - it.kb < C::kStages ? it.ke - it.kb : C::kStages;
                    for (; pre < want; ++pre) {
                        const int s = (kc + pre) % C::kStages;
                        const uint32_t ph = ((kc + pre) / C::kStages) & 1u;
                        if (!mbar_wait_bounded(&empty[s], ph ^ 1u, limit, abort_flag)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&full[s], bytes);
                        load_w(s, it.kb + pre);
                        ++fills[s];
                    }
                    if (ok) {
                        const uint64_t t0 = global_ns();
                        while ((int)ld_acquire_u32(&chunk_done[t.chunk]) < NFA) {
                            if (*abort_flag || global_ns() - t0 > limit) {
                                ok = false;
                                break;
                            }
                            __nanosleep(64);
                        }
                        if (ok) fence_proxy_async_global();
                    }
                    // the stages already expecting their activations get them even
                    // when the wait gave up (in-bounds rows; the launch is reported
                    // as timed out), so that every started stage completes
                    for (int j = 0; j < pre; ++j) load_x((kc + j) % C::kStages, it.kb + j);
                    kc += pre;
                    if (!ok) continue;  // next turn publishes the end marker
                }
                for (int k = it.kb + pre; k < it.ke; ++k, ++kc) {
                    const int s = kc % C::kStages;
                    const uint32_t ph = (kc / C::kStages) & 1u;
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1u, limit, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (withhold) {
                        withhold = false;
                        continue;
                    }
                    mbar_arrive_expect_tx(&full[s], bytes);
                    load_w(s, k);
                    load_x(s, k);
                    ++fills[s];
                }
                if (!ok) continue;
            }
            if (!ok) {
                *abort_flag = 1;
                if (!oversize) atomicOr(p.status, kStatusTimeout);
            }
            for (int s = 0; s < C::kStages; ++s)
                if (fills[s] > 0) mbar_drain(&full[s], (uint32_t)(fills[s] - 1) & 1u, limit);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            uint32_t kc = 0, ac = 0, n = 0;
            uint32_t cc = 0;  // FP8: stages widened so far (the conversion ring's own count)
            bool ok = true;
            while (true) {
                const int rs = n % kFfnRing;
                const uint32_t rph = (n / kFfnRing) & 1u;
                if (!mbar_wait_bounded(&ring_full[rs], rph, limit, abort_flag)) {
                    ok = false;
                    break;
                }
                const long long id = ring[rs];
                mbar_arrive(&ring_empty[rs]);
                ++n;
                if (id < 0) break;
                FfnItem it;
                Tile t;
                item_of(id, it, t);
                const int b = ac % C::kNumAcc;
                const uint32_t aph = (ac / C::kNumAcc) & 1u;
                if (!mbar_wait_bounded(&tempty[b], aph ^ 1u, limit, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d0 = tmem_base + b * C::kAccCols;
                const uint32_t d1 = d0 + kMaxN;
                // (FP8: f16 operands in phase B; in phase A E4M3 x E4M3, whose format
                // code in the kind::f8f6f4 descriptor is also 0)
                const uint32_t idesc = umma_idesc(kFp8 ? Elt<__half>::kMmaFmt : Elt<T>::kMmaFmt, 128, t.mma_n);
                for (int k = it.kb; k < it.ke; ++k, ++kc) {
                    const int s = kc % C::kStages;
                    const uint32_t ph = (kc / C::kStages) & 1u;
                    if (!mbar_wait_bounded(&full[s], ph, limit, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = stage_base + s * C::kStageBytes;
                    const uint64_t bx = umma_desc_sw128(smem_u32(st + 2 * C::kRawWBytes));
                    int cv = -1;
                    if (kFp8 && it.phase == 0) {
                        // E4M3 weights x the token rows' hi codes, then x their lo codes,
                        // into the same accumulator: K 32 per MMA, four steps per stage
                        tc_fence_after();
                        const uint64_t a0 = umma_desc_sw128(smem_u32(st));
                        const uint64_t a1 = umma_desc_sw128(smem_u32(st + C::kWTileBytes));
#pragma unroll
                        for (int part = 0; part < 2; ++part) {
                            const uint64_t b = umma_desc_sw128(smem_u32(st + 2 * C::kRawWBytes + part * kMaxN * 128));
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint32_t acc = (k > it.kb || kk > 0 || part > 0) ? 1u : 0u;
                                umma_e4m3(d0, a0 + 2 * kk, b + 2 * kk, idesc, acc);
                                umma_e4m3(d1, a1 + 2 * kk, b + 2 * kk, idesc, acc);
                            }
                        }
                    } else if constexpr (kFp8) {
                        // A: the stage's two tiles, widened to f16 in TMEM by the converter warps
                        cv = (int)(cc % C::kConv);
                        if (!mbar_wait_bounded(&conv_full[cv], (cc / C::kConv) & 1u, limit, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a0 = tmem_base + C::kConvCol0 + cv * C::kConvCols;
                        // K 128 per stage: eight 16-deep steps, the token operand's
                        // first four in its first 64-column box, the rest in the second
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t acc = (k > it.kb || kk > 0) ? 1u : 0u;
                            const uint64_t b = umma_desc_sw128(smem_u32(st + 2 * C::kRawWBytes + (kk >> 2) * kMaxN * 128)) +
                                               2 * (kk & 3);
                            umma_f16_tmem_a(d0, a0 + 8 * kk, b, idesc, acc);
                            umma_f16_tmem_a(d1, a0 + 64 + 8 * kk, b, idesc, acc);
                        }
                    } else {
                        tc_fence_after();
                        const uint64_t a0 = umma_desc_sw128(smem_u32(st));
                        const uint64_t a1 = umma_desc_sw128(smem_u32(st + C::kWTileBytes));
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint32_t acc = (k > it.kb || kk > 0) ? 1u : 0u;
                            umma<T>(d0, a0 + 2 * kk, bx + 2 * kk, idesc, acc);
                            umma<T>(d1, a1 + 2 * kk, bx + 2 * kk, idesc, acc);
                        }
                    }
                    umma_commit(&empty[s]);
                    if (cv >= 0) {  // FP8 down: the conversion buffer is free too
                        umma_commit(&conv_empty[cv]);
                        ++cc;
                    }
                }
                if (!ok) break;
                umma_commit(&tfull[b]);
                ++ac;
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(p.status, kStatusTimeout);
                umma_commit(drain_bar);
                mbar_drain(drain_bar, 0, limit);
            }
        }
    } else if (kFp8 && warp >= 6) {  // converter warps 6 .. 5 + kConvThreads / 32
        // ------------------------------------------- FP8 -> f16 converters
        // warps 6..9 widen a stage's first weight tile, warps 10..13 its second;
        // a warp may only store to its TMEM lane quadrant (warp mod 4), so each
        // thread takes one row (quadrant x 32 + lane): its 128 codes are eight
        // 16-byte chunks, chunk c of row r at chunk position c ^ (r mod 8) under
        // the 128-byte swizzle (8 consecutive rows hit 8 distinct bank groups),
        // widened to 64 f16 pairs and stored as 64 TMEM columns
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const int tt = (warp - 6) >> 2;
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        uint32_t kc = 0, n = 0, cc = 0;  // stages, items, widened stages
        bool ok = true;
        while (ok) {
            const int rs = n % kFfnRing;
            const uint32_t rph = (n / kFfnRing) & 1u;
            if (!mbar_wait_bounded(&ring_full[rs], rph, limit, abort_flag)) {
                ok = false;
                break;
            }
            const long long id = ring[rs];
            mbar_arrive(&ring_empty[rs]);
            ++n;
            if (id < 0) break;
            FfnItem it;
            Tile t;
            item_of(id, it, t);
            if (it.phase == 0) {  // gate/up stages use the codes as they are
                kc += it.ke - it.kb;
                continue;
            }
            for (int k = it.kb; k < it.ke; ++k, ++kc, ++cc) {
                const int s = kc % C::kStages;
                const int cv = (int)(cc % C::kConv);
                const bool got = mbar_wait_bounded(&full[s], (kc / C::kStages) & 1u, limit, abort_flag) &&
                                 mbar_wait_bounded(&conv_empty[cv], ((cc / C::kConv) & 1u) ^ 1u, limit, abort_flag);
                if (!__all_sync(0xffffffffu, got)) {  // the whole warp leaves together (warp-wide TMEM stores)
                    ok = false;
                    break;
                }
                tc_fence_after();  // the MMAs that read this buffer before have completed
                const uint8_t* src = stage_base + s * C::kStageBytes + tt * C::kRawWBytes + row * 128;
#pragma unroll
                for (int h = 0; h < 2; ++h) {  // codes 64 h .. 64 h + 63 -> 32 columns
                    uint32_t w[32];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int cc = 4 * h + c;
                        const uint4 v = *reinterpret_cast<const uint4*>(src + ((cc ^ (row & 7)) << 4));
                        uint4 lo, hi;
                        e4m3x16_to_f16(v, lo, hi);
                        w[8 * c + 0] = lo.x;
                        w[8 * c + 1] = lo.y;
                        w[8 * c + 2] = lo.z;
                        w[8 * c + 3] = lo.w;
                        w[8 * c + 4] = hi.x;
                        w[8 * c + 5] = hi.y;
                        w[8 * c + 6] = hi.z;
                        w[8 * c + 7] = hi.w;
                    }
                    tmem_st32(tmem_base + lane_base + C::kConvCol0 + cv * C::kConvCols + tt * 64 + h * 32, w);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&conv_full[cv]);
            }
        }
        if (!ok) {
            *abort_flag = 1;
            atomicOr(p.status, kStatusTimeout);
        }
    } else {
        // --------------------------------------------------------- epilogue
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        uint32_t ac = 0, n = 0;
        while (true) {
            const int rs = n % kFfnRing;
            const uint32_t rph = (n / kFfnRing) & 1u;
            if (!mbar_wait_bounded(&ring_full[rs], rph, limit, abort_flag)) {
                *abort_flag = 1;
                atomicOr(p.status, kStatusTimeout);
                break;
            }
            const long long id = ring[rs];
            mbar_arrive(&ring_empty[rs]);
            ++n;
            if (id < 0) break;
            FfnItem it;
            Tile t;
            item_of(id, it, t);
            const int b = ac % C::kNumAcc;
            const uint32_t aph = (ac / C::kNumAcc) & 1u;
            if (!mbar_wait_bounded(&tfull[b], aph, limit, abort_flag)) {
                *abort_flag = 1;
                atomicOr(p.status, kStatusTimeout);
                break;
            }
            tc_fence_after();
            const uint32_t tacc = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + b * C::kAccCols;
            const bool gate_up = it.phase == 0;
            const int n_out = gate_up ? p.I : p.H;
            const int f = t.f0 + r;
            const bool v0 = f < n_out;
            const bool v1 = gate_up ? v0 : (f + 128 < n_out);
            // FP8 weights: the activations are f16 (the next MMA's operand)
            using ActT = typename std::conditional<kFp8, __half, OutT>::type;
            OutT* orow = reinterpret_cast<OutT*>(p.y) + (long long)t.row0 * n_out + f;
            ActT* arow = reinterpret_cast<ActT*>(p.act) + (long long)t.row0 * n_out + f;
            // FP8 weights: the row scales of the two accumulators' weight rows,
            // times 2^8 (the widened codes hold value x 2^-8)
            float sc0 = 1.f, sc1 = 1.f;
            if constexpr (kFp8) {
                if (gate_up) {  // direct E4M3 products: no widening factor; the token scale per column below
                    const float* sr = p.s13 + (long long)t.group * 2 * p.I;
                    sc0 = v0 ? __ldg(sr + f) : 0.f;
                    sc1 = v0 ? __ldg(sr + p.I + f) : 0.f;
                } else {
                    const float* sr = p.s2 + (long long)t.group * p.H;
                    sc0 = v0 ? __ldg(sr + f) * 256.f : 0.f;
                    sc1 = v1 ? __ldg(sr + f + 128) * 256.f : 0.f;
                }
            }
            auto emit = [&](int c0, float (&g)[16], float (&u)[16]) {
                if constexpr (kFp8) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        // the token row's scale (phase A operand), read for real rows only
                        const float xs = gate_up && c0 + i < t.nrows ? __ldg(p.x_scale + t.row0 + c0 + i) : 1.f;
                        g[i] *= sc0 * xs;
                        u[i] *= sc1 * xs;
                    }
                }
                if (gate_up) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) g[i] = silu_mul(g[i], u[i]);
                }
                if (v0 && gate_up) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c0 + i < t.nrows) store_out<ActT>(arow + (long long)(c0 + i) * n_out, g[i]);
                } else if (v0) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c0 + i < t.nrows) store_out<OutT>(orow + (long long)(c0 + i) * n_out, g[i]);
                }
                if (!gate_up && v1) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c0 + i < t.nrows) store_out<OutT>(orow + 128 + (long long)(c0 + i) * n_out, u[i]);
                }
            };
            bool finished = true;  // this item completed its tile
            if (it.S == 1) {
                for (int c0 = 0; c0 < t.nrows; c0 += 32) {
                    uint32_t ga[32], ua[32];
                    tmem_ld32_nowait(tacc + c0, ga);
                    tmem_ld32_nowait(tacc + kMaxN + c0, ua);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float g[16], u[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            g[i] = __uint_as_float(ga[16 * h + i]);
                            u[i] = __uint_as_float(ua[16 * h + i]);
                        }
                        if (c0 + 16 * h < t.nrows) emit(c0 + 16 * h, g, u);
                    }
                }
            } else {
                // split tile: publish this slice, the last slice sums them all in order
                float4* mine = reinterpret_cast<float4*>(p.partials + it.slot * C::kSlotFloats);
                for (int c0 = 0; c0 < t.nrows; c0 += 16) {
                    float g[16];
                    tmem_ld16(tacc + c0, g);
                    if (v0) {
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            mine[slot_f4((c0 >> 2) + q, r)] = make_float4(g[4 * q], g[4 * q + 1], g[4 * q + 2], g[4 * q + 3]);
                    }
                    tmem_ld16(tacc + kMaxN + c0, g);
                    if (v1) {
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            mine[slot_f4(((kMaxN + c0) >> 2) + q, r)] =
                                make_float4(g[4 * q], g[4 * q + 1], g[4 * q + 2], g[4 * q + 3]);
                    }
                }
                __threadfence();
                named_sync(1, 128);
                if (r == 0) *bcast = atomicAdd(&tile_ctr[it.ctr], 1);
                named_sync(1, 128);
                finished = *bcast == it.S - 1;
                if (finished) {
                    __threadfence();
                    const long long slot0 = it.slot - it.slice;  // slot of slice 0 of this tile
                    for (int c0 = 0; c0 < t.nrows; c0 += 16) {
                        float g[16], u[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) g[i] = u[i] = 0.f;
                        for (int sl = 0; sl < it.S; ++sl) {
                            if (sl == it.slice) {
                                float v[16];
                                tmem_ld16(tacc + c0, v);
#pragma unroll
                                for (int i = 0; i < 16; ++i) g[i] += v[i];
                                tmem_ld16(tacc + kMaxN + c0, v);
#pragma unroll
                                for (int i = 0; i < 16; ++i) u[i] += v[i];
                            } else {
                                const float4* other =
                                    reinterpret_cast<const float4*>(p.partials + (slot0 + sl) * C::kSlotFloats);
                                const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
                                float4 a4[4], b4[4];
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    a4[q] = v0 ? __ldcg(other + slot_f4((c0 >> 2) + q, r)) : z;
                                    b4[q] = v1 ? __ldcg(other + slot_f4(((kMaxN + c0) >> 2) + q, r)) : z;
                                }
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    g[4 * q] += a4[q].x;
                                    g[4 * q + 1] += a4[q].y;
                                    g[4 * q + 2] += a4[q].z;
                                    g[4 * q + 3] += a4[q].w;
                                    u[4 * q] += b4[q].x;
                                    u[4 * q + 1] += b4[q].y;
                                    u[4 * q + 2] += b4[q].z;
                                    u[4 * q + 3] += b4[q].w;
                                }
                            }
                        }
                        emit(c0, g, u);
                    }
                    if (r == 0) tile_ctr[it.ctr] = 0;
                }
            }
            if (gate_up && finished) {
                // this gate/up tile's activations are stored: count it for its token chunk
                fence_proxy_async_global();
                __threadfence();
                named_sync(1, 128);
                if (r == 0) atomicAdd(&chunk_done[t.chunk], 1);
            }
            tc_fence_before();
            mbar_arrive(&tempty[b]);
            ++ac;
        }
    }

    tc_fence_before();
    __syncthreads();
    // the last block to finish re-zeroes the control words for the next launch
    if (threadIdx.x == 0) {
        __threadfence();
        *last_block = atomicAdd(done_ctr, 1) == (int)gridDim.x - 1;
    }
    __syncthreads();
    if (*last_block) {
        __threadfence();
        const long long nc = n_chunks < kFfnMaxChunks ? n_chunks : kFfnMaxChunks;
        for (long long c = threadIdx.x; c < nc; c += blockDim.x) chunk_done[c] = 0;
        if (threadIdx.x == 0) {
            *work_ctr = 0;
            *done_ctr = 0;
        }
    }
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace moe
