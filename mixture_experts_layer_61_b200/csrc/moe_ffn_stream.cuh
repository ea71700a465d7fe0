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
// A phase-B item reads the SwiGLU activations of its token chunk over its
// k-slice of features, so before loading them its producer waits (bounded)
// until the phase-A tiles that produce those features have been stored: a
// chunk's gate/up feature blocks count in kFfnBands bands, and the item waits
// for the bands its slice overlaps (FP8: all of them, as its activation split
// takes each row's maximum over every feature).  Within a token chunk the
// phase-B items go slice by slice, so the slices that need the chunk's last
// gate/up tiles come last.  No block waits on work that is not already held
// by a running block, so the wait always ends.
//
// Roles as in the grouped GEMM (warp 0 TMA, warp 1 TMEM + MMA, warps 2..5
// epilogue); the producer publishes each item id to the other roles through a
// small shared-memory ring.
//
// FP8 weights (kFp8): the weight tiles stream as E4M3 codes (half the bytes),
// 128 rows x 128 codes per tile with the 128-byte swizzle (the same 128-byte
// row pieces as a bf16 tile), and every MMA is kind::f8f6f4 with both
// operands E4M3 in shared memory (K 32 per instruction), fp32 accumulation.
// The token operand is split exactly into two E4M3 terms with a power-of-two
// scale per row, x = s (hi + lo), and each stage runs weights x hi, then
// weights x lo, into the same accumulator; the epilogue multiplies by the
// weight row's fp32 scale and the token row's s.
//  * gate/up: the token rows arrive split (hi codes, then lo codes lo_rows
//    rows further on, and their scales x_scale);
//  * down: phase A stores the SwiGLU activations in f16 and raises, per token
//    row, the maximum |activation| (atomicMax on the fp32 bits) before its
//    band counter; a phase-B item (which waits for every band of its chunk)
//    brings those maxima along on its first stage
//    (bulk copy on the stage's barrier), and warps 6..13 split each stage's
//    f16 activation tile in place into hi and lo E4M3 codes (row scale from
//    the maximum) before the MMA thread issues.  The split keeps about 8
//    significant bits of each activation (bf16's precision); the weights
//    meet no rounding at all.
// Widening the weight codes instead (to f16, in tensor memory, for kind::f16
// MMAs) cost 4 bytes of tensor-memory traffic per weight byte and ran at half
// the copy bandwidth; splitting the token operand touches kMaxN x 128 values
// per stage against 32 K weights.
#pragma once

#include <type_traits>

#include "moe_gemm.cuh"

namespace moe {

constexpr int kFfnMaxChunks = 4096;   // token chunks
constexpr int kFfnBands = 8;          // phase-A counters per chunk (bands of its gate/up feature blocks)
constexpr int kFfnTileCtrs = 4096;    // split-tile counters (phase A, then phase B)
constexpr int kFfnRing = 4;
constexpr int kFfnMaxRows = 1 << 17;  // token rows of an FP8 launch (per-row activation maxima)
// control ints: [0] work counter, [1] finished blocks, [2, 2+kFfnMaxChunks) chunk
// counters, then kFfnTileCtrs tile counters, then (16-byte aligned, for the
// bulk copies) the FP8 path's per-row activation maxima (fp32 bits) with a
// margin for the copies' rounding to 16 bytes
constexpr int kFfnAmaxOff = (2 + kFfnMaxChunks * kFfnBands + kFfnTileCtrs + 63) / 64 * 64;
constexpr int kFfnCtlInts = kFfnAmaxOff + kFfnMaxRows + 256;

struct FfnParams {
    const int32_t* seg_offsets;  // [n_groups + 1] row offsets, or nullptr: one group [0, seg_rows)
    int n_groups;
    int seg_rows;
    int H, I;
    void* act;           // [rows, I] SwiGLU activations (written in phase A, read in phase B)
    void* y;             // [rows, H] output
    int* ctl;            // kFfnCtlInts, zero on entry, left zero (ctl 16-byte aligned)
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
    // 128-byte rows of the token tile per stage: one box of 64 16-bit columns,
    // or (FP8) two: the hi and lo codes of 128 columns (phase B: the two f16
    // boxes of 64 activation columns, split in place into hi and lo codes)
    static constexpr int kXBoxes = kFp8 ? 2 : 1;
    static constexpr int kXTileBytes = kXBoxes * kMaxN * 128;
    static constexpr int kStageBytes = 2 * kRawWBytes + kXTileBytes;
    static constexpr int kSplitThreads = kFp8 ? 256 : 0;  // activation splitters, warps 6..13
    static constexpr int kUnits = kMaxN * 8 / 256;         // (row, 16 columns) units per splitter per stage
    // per stage: the activation maxima of a phase-B item's rows (first stage
    // only), fetched 16-byte aligned: up to 3 rows before the item's first
    static constexpr int kSideBytes = kFp8 ? (kMaxN + 8) * 4 : 0;
    static constexpr int kThreads = kFfnThreads + kSplitThreads;
    // FP8 with tiles of at most 64 token rows: the hi and lo rows sit one after
    // the other in the stage (lo at row mma_n) and one MMA with N = 2 mma_n
    // covers both -- the per-MMA cost is flat up to N = 64 and at the tensor
    // rate beyond, so this halves the MMAs of a stage; each accumulator then
    // holds the hi and lo products side by side (2 kMaxN columns each), which
    // the epilogue adds.  128-row tiles keep two MMAs into one accumulator
    // (TMEM holds two 2 x 256-column buffers only that way).
    static constexpr bool kStack = kFp8 && kMaxN <= 64;
    static constexpr int kUOff = kStack ? 2 * kMaxN : kMaxN;  // the up (or second) accumulator's first column
    static constexpr int kAccCols = 2 * kUOff;
    static constexpr int kNumAcc = 2;
    // FP8: per stage, a barrier on which phase-B fills complete (their own
    // phases, so the splitters, which skip phase-A stages, wait on exact
    // phases) and one for the split tile being ready (at most 8 stages)
    static constexpr int kXReady = kFp8 ? 8 : 0;
    static constexpr int kTableBytes = 2 * (kMaxGroups + 1) * 4;
    static constexpr int kMiscBytes = 768;
    static constexpr int kBudget = 227 * 1024 - 1024 - kTableBytes - kMiscBytes;
    static constexpr int kStagesRaw = kBudget / (kStageBytes + kSideBytes);
    static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
    static constexpr int kSmemBytes = 1024 + kStages * (kStageBytes + kSideBytes) + kTableBytes + kMiscBytes;
    static_assert(kStageBytes % 1024 == 0, "stages keep the swizzle atoms aligned");
    static_assert(kSideBytes % 16 == 0, "bulk copies land 16-byte aligned");
    static_assert(!kFp8 || sizeof(T) == 2, "FP8 weights: 16-bit activations");
    // barriers (full/empty per stage, 2 TMEM pairs, the item ring, the split
    // barriers, the drain barrier) and the ring / TMEM / flag words fit the misc area
    static_assert((2 * kStages + 2 * kNumAcc + 2 * kFfnRing + 2 * kXReady + 1) * 8 + 4 * kFfnRing + 16 <= kMiscBytes,
                  "misc area");
    static constexpr int kSlotFloats = 128 * 2 * kMaxN;  // a split tile's partial gate and up sums
    static_assert(kMaxN == 32 || kMaxN == 64 || kMaxN == 128, "decode token tiles");
    static_assert(kAccCols * kNumAcc <= 512, "TMEM columns");
};

// One phase's split: S slices per tile (S = 1: whole tiles), about two items
// per block.  A tile's last slice sums the S partial slots (128 x 2 n fp32
// each, n token columns) on one SM, so S also balances that sum against the
// streaming it shortens: a slice streams KI / S stages of 32 KB of weights,
// the sum reads (S - 1) slots of n KB, and the two balance near
// S = sqrt(32 KI / n).
__device__ __forceinline__ int ffn_slices(long long tiles, int KI, int G, int max_slots, int n) {
    if (tiles <= 0 || tiles >= 2LL * G) return 1;
    long long s = (2LL * G + tiles - 1) / tiles;
    long long cap = (4LL * G < max_slots ? 4LL * G : max_slots) / tiles;
    if (s > cap) s = cap;
    if (s > 16) s = 16;
    if (s > KI / 4) s = KI / 4;
    const long long bal = (long long)sqrtf(32.f * (float)KI / (float)n);
    if (s > bal) s = bal;
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

// 16 activations (two 16-byte chunks of f16) times 2^e -> their E4M3 hi and
// lo codes: hi = E4M3(y), lo = E4M3(y - hi), y = a 2^e.  For e <= 15 in packed
// f16: a 2^e is exact (it only loses what falls below 2^-24, far under the lo
// codes' grid) and y - hi is exact (both are multiples of y's unit in the last
// place and |y - hi| is below hi's); for larger e (rows whose largest
// activation is below 448 x 2^-16) in fp32, where 2^e is representable.
__device__ __forceinline__ uint32_t e4m3x2_of_h2(__half2 v) {
    return (uint32_t)__nv_cvt_halfraw2_to_fp8x2(static_cast<__half2_raw>(v), __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ void split_f16x16_e4m3(const uint4 a, const uint4 b, int e, uint4& hi, uint4& lo) {
    const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t h[4], l[4];
    if (e <= 15) {
        const __half2 m = __half2half2(__ushort_as_half((unsigned short)((e + 15) << 10)));
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t hw = 0, lw = 0;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const uint32_t w = in[2 * q + j];
                const __half2 y = __hmul2(*reinterpret_cast<const __half2*>(&w), m);
                const uint32_t hc = e4m3x2_of_h2(y);
                const __half2 hv(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)hc, __NV_E4M3));
                hw |= hc << (16 * j);
                lw |= e4m3x2_of_h2(__hsub2(y, hv)) << (16 * j);
            }
            h[q] = hw;
            l[q] = lw;
        }
    } else {
        const float inv = __uint_as_float((uint32_t)(e + 127) << 23);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t hw = 0, lw = 0;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const uint32_t w = in[2 * q + j];
                float2 y = __half22float2(*reinterpret_cast<const __half2*>(&w));
                y.x *= inv;
                y.y *= inv;
                const __nv_fp8x2_storage_t hc = __nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3);
                const float2 hv = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(hc, __NV_E4M3)));
                const __nv_fp8x2_storage_t lc =
                    __nv_cvt_float2_to_fp8x2(make_float2(y.x - hv.x, y.y - hv.y), __NV_SATFINITE, __NV_E4M3);
                hw |= (uint32_t)hc << (16 * j);
                lw |= (uint32_t)lc << (16 * j);
            }
            h[q] = hw;
            l[q] = lw;
        }
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
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
    uint8_t* side_base = smem + C::kStages * C::kStageBytes;  // FP8: per-stage activation maxima
    int* seg = reinterpret_cast<int*>(side_base + C::kStages * C::kSideBytes);
    int* cbase = seg + (kMaxGroups + 1);
    uint8_t* misc = reinterpret_cast<uint8_t*>(cbase + (kMaxGroups + 1));
    uint64_t* full = reinterpret_cast<uint64_t*>(misc);
    uint64_t* empty = full + C::kStages;
    uint64_t* tfull = empty + C::kStages;
    uint64_t* tempty = tfull + C::kNumAcc;
    uint64_t* ring_full = tempty + C::kNumAcc;
    uint64_t* ring_empty = ring_full + kFfnRing;
    uint64_t* xready = ring_empty + kFfnRing;  // FP8: a stage's split activation tile is ready
    uint64_t* bfull = xready + C::kXReady;     // FP8: a phase-B fill of the stage landed
    uint64_t* drain_bar = bfull + C::kXReady;
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
    int* band_done = p.ctl + 2;  // [chunk][band]: gate/up tiles stored
    int* tile_ctr = p.ctl + 2 + kFfnMaxChunks * kFfnBands;
    unsigned* act_amax = reinterpret_cast<unsigned*>(p.ctl + kFfnAmaxOff);  // FP8: per-row max |activation|

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
            // the MMA thread, every epilogue thread and (FP8) every splitter thread
            mbar_init(&ring_empty[r], 1 + 128 + C::kSplitThreads);
        }
        for (int c = 0; c < C::kXReady; ++c) {
            mbar_init(&xready[c], C::kSplitThreads / 32);  // one arrival per splitter warp
            mbar_init(&bfull[c], 1);
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
    const int BS = (NFA + kFfnBands - 1) / kFfnBands;  // gate/up feature blocks per band
    const int KIA = (p.H + C::kBK - 1) / C::kBK, KIB = (p.I + C::kBK - 1) / C::kBK;
    const long long tilesA = n_chunks * NFA, tilesB = n_chunks * NFB;
    const int SA = ffn_slices(tilesA, KIA, G, p.max_slots_phase, kMaxN),
              SB = ffn_slices(tilesB, KIB, G, p.max_slots_phase, kMaxN);
    const long long nA = tilesA * SA, nB = tilesB * SB;
    const long long total = nA + nB;
    const long long slotsA = SA > 1 ? nA : 0;
    const bool oversize = n_chunks > kFfnMaxChunks || (SA > 1 && tilesA > kFfnTileCtrs / 2) ||
                          (SB > 1 && tilesB > kFfnTileCtrs / 2) || (kFp8 && seg[n_groups] > kFfnMaxRows);

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
            // expert by expert (a group's tiles hold its items' range, SB per
            // tile), and inside an expert slice by slice over its tiles
            const long long j = id - nA;
            const Tile tg = decode_tile_w(j / SB, seg, cbase, n_groups, NFB, 256, 16, p.H);
            const long long gt0 = (long long)cbase[tg.group] * NFB;  // the expert's first tile
            const long long per = (long long)tg.nch * NFB;          // its tiles
            const long long r = j - gt0 * SB;
            it.phase = 1;
            it.slice = (int)(r / per);
            it.tile = gt0 + (r - (long long)it.slice * per);
            it.S = SB;
            it.kb = (int)((long long)it.slice * KIB / SB);
            it.ke = (int)((long long)(it.slice + 1) * KIB / SB);
            it.slot = slotsA + it.tile * SB + it.slice;
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
            int fills[C::kStages], bfills[C::kStages];  // completions owed on full[s] / bfull[s]
#pragma unroll
            for (int s = 0; s < C::kStages; ++s) fills[s] = bfills[s] = 0;
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
                // FP8 down: the item's first stage also brings its rows' activation
                // maxima, from the 16-byte boundary at or below row0
                const uint32_t side_bytes =
                    kFp8 && it.phase == 1 ? 4u * (uint32_t)(((t.row0 & 3) + t.mma_n + 3) & ~3) : 0u;
                const uint64_t pol_w = t.nch > 1 ? pol_w_shared : pol_w_once;
                // FP8 phase B: the stage's loads complete on bfull[s] (the splitters'
                // barrier); every other stage on full[s] (the MMA thread's)
                const bool to_b = kFp8 && it.phase == 1;
                auto bar_of = [&](int s) { return to_b ? &bfull[s] : &full[s]; };
                auto owe = [&](int s) {
                    if (to_b)
                        ++bfills[s];
                    else
                        ++fills[s];
                };
                auto load_w = [&](int s, int k) {
                    uint8_t* st = stage_base + s * C::kStageBytes;
                    const int kx = k * C::kBK;
                    tma_load_2d(st, tw, bar_of(s), kx, t.wrow, pol_w);
                    tma_load_2d(st + C::kRawWBytes, tw, bar_of(s), kx, t.wrow + second, pol_w);
                };
                // FP8: the second box (lo codes, or activation columns 64..127)
                const int box_off = (C::kStack ? t.mma_n : kMaxN) * 128;
                auto load_x = [&](int s, int k) {
                    if (to_b && k == it.kb)
                        bulk_load_g2s(side_base + s * C::kSideBytes, act_amax + (t.row0 & ~3), side_bytes, bar_of(s));
#pragma unroll
                    for (int xb = 0; xb < C::kXBoxes; ++xb) {
                        uint8_t* xs = stage_base + s * C::kStageBytes + 2 * C::kRawWBytes + xb * box_off;
                        // FP8 gate/up: box xb holds the hi (0) or lo (1) codes of columns
                        // k*128..+127; otherwise 64 16-bit columns each
                        const bool codes = kFp8 && it.phase == 0;
                        const int kx = codes ? k * C::kBK : k * C::kBK + xb * 64;
                        const int rbase = codes ? (int)(xb * p.lo_rows) : 0;
                        int r = 0;
                        if (kMaxN >= C::kXBoxMid)
                            for (; r + C::kXBoxMid <= t.mma_n; r += C::kXBoxMid)
                                tma_load_2d(xs + r * 128, tx64, bar_of(s), kx, rbase + t.row0 + r, pol_x);
                        for (; r < t.mma_n; r += C::kXBoxRows)
                            tma_load_2d(xs + r * 128, tx, bar_of(s), kx, rbase + t.row0 + r, pol_x);
                    }
                };
                int pre = 0;  // stages of this item whose weight tiles went out before the activation wait
                if (it.phase == 1) {
                    // The weights do not depend on phase A: stream the first stages'
                    // weight tiles now, then wait until the gate/up tiles of this
                    // token chunk that produce the slice's features (FP8: all of
                    // them) have stored their activations, then load those.
                    const int want = it.ke - it.kb < C::kStages ? it.ke - it.kb : C::kStages;
                    for (; pre < want; ++pre) {
                        const int s = (kc + pre) % C::kStages;
                        const uint32_t ph = ((kc + pre) / C::kStages) & 1u;
                        if (!mbar_wait_bounded(&empty[s], ph ^ 1u, limit, abort_flag)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(bar_of(s), bytes + (pre == 0 ? side_bytes : 0u));
                        load_w(s, it.kb + pre);
                        owe(s);
                    }
                    if (ok) {
                        // the bands of the 128-feature gate/up blocks that hold
                        // features [kb kBK, ke kBK)
                        const int fa1 = (it.ke * C::kBK - 1) / 128;
                        const int b0 = kFp8 ? 0 : (it.kb * C::kBK / 128) / BS;
                        const int b1 = (kFp8 || fa1 >= NFA ? NFA - 1 : fa1) / BS;
                        const uint64_t t0 = global_ns();
                        for (int bd = b0; bd <= b1 && ok; ++bd) {
                            const int need = NFA - bd * BS < BS ? NFA - bd * BS : BS;
                            while ((int)ld_acquire_u32(&band_done[t.chunk * kFfnBands + bd]) < need) {
                                if (*abort_flag || global_ns() - t0 > limit) {
                                    ok = false;
                                    break;
                                }
                                __nanosleep(64);
                            }
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
                    mbar_arrive_expect_tx(bar_of(s), bytes + (k == it.kb ? side_bytes : 0u));
                    load_w(s, k);
                    load_x(s, k);
                    owe(s);
                }
                if (!ok) continue;
            }
            if (!ok) {
                *abort_flag = 1;
                if (!oversize) atomicOr(p.status, kStatusTimeout);
            }
            for (int s = 0; s < C::kStages; ++s) {
                if (fills[s] > 0) mbar_drain(&full[s], (uint32_t)(fills[s] - 1) & 1u, limit);
                if (bfills[s] > 0) mbar_drain(&bfull[s], (uint32_t)(bfills[s] - 1) & 1u, limit);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            uint32_t kc = 0, ac = 0, n = 0;
            uint32_t xpar = 0;  // FP8: per-stage parity of the split barriers (bit s)
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
                const uint32_t d1 = d0 + C::kUOff;
                const uint32_t idesc = umma_idesc(kFp8 ? kFmtE4M3 : Elt<T>::kMmaFmt, 128, C::kStack ? 2 * t.mma_n : t.mma_n);
                for (int k = it.kb; k < it.ke; ++k, ++kc) {
                    const int s = kc % C::kStages;
                    const uint32_t ph = (kc / C::kStages) & 1u;
                    if (kFp8 && it.phase == 1) {
                        // the splitters' hi / lo codes of the activation tile (they waited
                        // for the stage's loads; a block's phase-B items follow all of
                        // its phase-A items, so full[s]'s phases count phase-A fills only)
                        if (!mbar_wait_bounded(&xready[s], (xpar >> s) & 1u, limit, abort_flag)) {
                            ok = false;
                            break;
                        }
                        xpar ^= 1u << s;
                    } else if (!mbar_wait_bounded(&full[s], ph, limit, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = stage_base + s * C::kStageBytes;
                    const uint64_t a0 = umma_desc_sw128(smem_u32(st));
                    const uint64_t a1 = umma_desc_sw128(smem_u32(st + C::kWTileBytes));
                    if constexpr (kFp8) {
                        tc_fence_after();
                        if constexpr (C::kStack) {
                            // E4M3 weights x [hi rows; lo rows] in one MMA (N = 2 mma_n):
                            // K 32 per MMA, four steps per stage
                            const uint64_t bx = umma_desc_sw128(smem_u32(st + 2 * C::kRawWBytes));
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint32_t acc = (k > it.kb || kk > 0) ? 1u : 0u;
                                umma_e4m3(d0, a0 + 2 * kk, bx + 2 * kk, idesc, acc);
                                umma_e4m3(d1, a1 + 2 * kk, bx + 2 * kk, idesc, acc);
                            }
                        } else {
                            // E4M3 weights x the hi rows, then x the lo rows, into the same
                            // accumulator
#pragma unroll
                            for (int part = 0; part < 2; ++part) {
                                const uint64_t bx =
                                    umma_desc_sw128(smem_u32(st + 2 * C::kRawWBytes + part * kMaxN * 128));
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk) {
                                    const uint32_t acc = (k > it.kb || kk > 0 || part > 0) ? 1u : 0u;
                                    umma_e4m3(d0, a0 + 2 * kk, bx + 2 * kk, idesc, acc);
                                    umma_e4m3(d1, a1 + 2 * kk, bx + 2 * kk, idesc, acc);
                                }
                            }
                        }
                    } else {
                        tc_fence_after();
                        const uint64_t bx = umma_desc_sw128(smem_u32(st + 2 * C::kRawWBytes));
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint32_t acc = (k > it.kb || kk > 0) ? 1u : 0u;
                            umma<T>(d0, a0 + 2 * kk, bx + 2 * kk, idesc, acc);
                            umma<T>(d1, a1 + 2 * kk, bx + 2 * kk, idesc, acc);
                        }
                    }
                    umma_commit(&empty[s]);
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
    } else if (kFp8 && warp >= 6) {  // splitter warps 6 .. 13
        // ------------------------------------- activation splitters (phase B)
        // Unit u = (row u / 8, columns 16 (u % 8) .. + 15) of a stage's 128
        // activation columns; thread i takes units i, i + 256, ...  A unit reads
        // two 16-byte f16 chunks of box (u % 8) / 4 and writes one 16-byte chunk
        // of hi codes (box 0) and one of lo codes (box 1), all under the 128-byte
        // swizzle (chunk c of row r at c ^ (r mod 8)).  Every read of the stage
        // precedes every write (in place), so the 256 threads meet in between at
        // a reducing barrier, which also decides whether all of them go on: an
        // exit is always agreed there, so no thread is left waiting at one.
        const int ct = threadIdx.x - 6 * 32;
        uint32_t kc = 0, n = 0;
        uint32_t bpar = 0;  // per-stage parity of bfull (bit s): phase-B fills seen so far
        bool ok = true;
        while (true) {
            const int rs = n % kFfnRing;
            const bool got = mbar_wait_bounded(&ring_full[rs], (n / kFfnRing) & 1u, limit, abort_flag);
            if (!named_all(2, C::kSplitThreads, got)) {
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
            if (it.phase == 0) {  // gate/up stages carry split token rows already
                kc += it.ke - it.kb;
                continue;
            }
            int ex[C::kUnits];  // per unit: the row's scale is 2^-ex
            for (int k = it.kb; k < it.ke; ++k, ++kc) {
                const int s = kc % C::kStages;
                const bool g = mbar_wait_bounded(&bfull[s], (bpar >> s) & 1u, limit, abort_flag);
                bpar ^= 1u << s;
                uint8_t* xt = stage_base + s * C::kStageBytes + 2 * C::kRawWBytes;
                const int box_off = (C::kStack ? t.mma_n : kMaxN) * 128;  // second box: f16 columns 64.., then lo codes
                uint4 va[C::kUnits], vb[C::kUnits];
                if (g) {
                    if (k == it.kb) {  // the rows' scales, from the maxima that came with this stage
                        const unsigned* side = reinterpret_cast<const unsigned*>(side_base + s * C::kSideBytes);
#pragma unroll
                        for (int j = 0; j < C::kUnits; ++j) {
                            const int r = (ct + 256 * j) >> 3;
                            ex[j] = r < t.nrows ? -e4m3_pow2_exp(__uint_as_float(side[(t.row0 & 3) + r])) : 0;
                        }
                    }
#pragma unroll
                    for (int j = 0; j < C::kUnits; ++j) {
                        const int u = ct + 256 * j, r = u >> 3, c = u & 7;
                        if (r < t.nrows) {
                            const uint8_t* src = xt + (c >> 2) * box_off + r * 128;
                            va[j] = *reinterpret_cast<const uint4*>(src + (((2 * (c & 3)) ^ (r & 7)) << 4));
                            vb[j] = *reinterpret_cast<const uint4*>(src + (((2 * (c & 3) + 1) ^ (r & 7)) << 4));
                        }
                    }
                }
                // every read of the stage precedes every write (in place), and all
                // leave together if any wait gave up
                if (!named_all(2, C::kSplitThreads, g)) {
                    ok = false;
                    break;
                }
#pragma unroll
                for (int j = 0; j < C::kUnits; ++j) {
                    const int u = ct + 256 * j, r = u >> 3, c = u & 7;
                    if (r < t.mma_n) {  // rows past the chunk's own: zero codes
                        uint4 hi = make_uint4(0u, 0u, 0u, 0u), lo = hi;
                        if (r < t.nrows) split_f16x16_e4m3(va[j], vb[j], ex[j], hi, lo);
                        const int off = r * 128 + ((c ^ (r & 7)) << 4);
                        *reinterpret_cast<uint4*>(xt + off) = hi;
                        *reinterpret_cast<uint4*>(xt + box_off + off) = lo;
                    }
                }
                fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) mbar_arrive(&xready[s]);
            }
            if (!ok) break;
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
            // every wait ends in an agreement of the 128 epilogue threads: all go
            // on or all leave (the split path meets at named barriers, which a
            // thread that left would never reach)
            const bool got_item = mbar_wait_bounded(&ring_full[rs], rph, limit, abort_flag);
            if (!named_all(1, 128, got_item)) {
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
            const bool got_acc = mbar_wait_bounded(&tfull[b], aph, limit, abort_flag);
            if (!named_all(1, 128, got_acc)) {
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
            // FP8 weights: the row scales of the two accumulators' weight rows
            float sc0 = 1.f, sc1 = 1.f;
            if constexpr (kFp8) {
                if (gate_up) {
                    const float* sr = p.s13 + (long long)t.group * 2 * p.I;
                    sc0 = v0 ? __ldg(sr + f) : 0.f;
                    sc1 = v0 ? __ldg(sr + p.I + f) : 0.f;
                } else {
                    const float* sr = p.s2 + (long long)t.group * p.H;
                    sc0 = v0 ? __ldg(sr + f) : 0.f;
                    sc1 = v1 ? __ldg(sr + f + 128) : 0.f;
                }
            }
            // FP8: the token rows' scales, one column per lane (column 32 j + lane
            // in tsc[j]), read once per item for real rows only: the split of x
            // (gate/up), or the one the splitters took from the row's maximum
            // activation (down; the MMAs are done, so its chunk's maxima are final)
            constexpr int kTsc = kFp8 ? kMaxN / 32 : 1;
            float tsc[kTsc];
#pragma unroll
            for (int j = 0; j < kTsc; ++j) {
                const int c = 32 * j + lane;
                tsc[j] = 1.f;
                if (kFp8 && c < t.nrows)
                    tsc[j] = gate_up ? __ldg(p.x_scale + t.row0 + c)
                                     : e4m3_pow2_scale(__uint_as_float(__ldcg(act_amax + t.row0 + c)));
            }
            auto emit = [&](int c0, float (&g)[16], float (&u)[16]) {
                if constexpr (kFp8) {
                    // columns c0 .. c0 + 15 sit in one register of the lanes (c0 & 31) + i
                    float base = tsc[0];
#pragma unroll
                    for (int j = 1; j < kTsc; ++j)
                        if (j == (c0 >> 5)) base = tsc[j];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float xs = __shfl_sync(0xffffffffu, base, (c0 & 31) + i);
                        g[i] *= sc0 * xs;
                        u[i] *= sc1 * xs;
                    }
                }
                if (gate_up) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) g[i] = silu_mul(g[i], u[i]);
                    if constexpr (kFp8) {
                        // raise each row's maximum |activation| (as stored, in f16) by
                        // this warp's 32 features; non-negative floats order as their bits
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float a = v0 && c0 + i < t.nrows ? fabsf(__half2float(__float2half_rn(g[i]))) : 0.f;
                            const unsigned m = __reduce_max_sync(0xffffffffu, __float_as_uint(a));
                            if (lane == i && m != 0u) atomicMax(act_amax + t.row0 + c0 + i, m);
                        }
                    }
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
            // 16 columns of an accumulator (FP8 stacked: its hi and lo products added)
            auto ld_acc = [&](uint32_t col, float (&v)[16]) {
                tmem_ld16(col, v);
                if constexpr (C::kStack) {
                    float w[16];
                    tmem_ld16(col + t.mma_n, w);
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] += w[i];
                }
            };
            bool finished = true;  // this item completed its tile
            if (C::kStack && it.S == 1) {
                for (int c0 = 0; c0 < t.nrows; c0 += 16) {
                    float g[16], u[16];
                    ld_acc(tacc + c0, g);
                    ld_acc(tacc + C::kUOff + c0, u);
                    emit(c0, g, u);
                }
            } else if (it.S == 1) {
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
                // split tile: publish this slice, the last slice sums them all in
                // order; only the columns of real token rows travel (4 at a time)
                float4* mine = reinterpret_cast<float4*>(p.partials + it.slot * C::kSlotFloats);
                for (int c0 = 0; c0 < t.nrows; c0 += 16) {
                    float g[16];
                    ld_acc(tacc + c0, g);
                    if (v0) {
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            if (c0 + 4 * q < t.nrows)
                                mine[slot_f4((c0 >> 2) + q, r)] =
                                    make_float4(g[4 * q], g[4 * q + 1], g[4 * q + 2], g[4 * q + 3]);
                    }
                    ld_acc(tacc + C::kUOff + c0, g);
                    if (v1) {
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            if (c0 + 4 * q < t.nrows)
                                mine[slot_f4(((kMaxN + c0) >> 2) + q, r)] =
                                    make_float4(g[4 * q], g[4 * q + 1], g[4 * q + 2], g[4 * q + 3]);
                    }
                }
                named_sync(1, 128);
                if (r == 0) *bcast = atomic_add_acq_rel_gpu(&tile_ctr[it.ctr], 1);
                named_sync(1, 128);
                finished = *bcast == it.S - 1;
                if (finished) {
                    const long long slot0 = it.slot - it.slice;  // slot of slice 0 of this tile
                    // g / u = sums over slices, in slice order, of the two accumulators'
                    // 16 columns: this slice's from TMEM, the others' from their slots,
                    // requested kSumBatch slices per L2 round trip -- both accumulators
                    // together, or (FP8: 448 threads at 128 registers each) one at a time
                    constexpr int kSumBatch = kFp8 ? 2 : 4;
                    constexpr int kAccs = kFp8 ? 1 : 2;  // accumulators summed per pass
                    auto sum_pass = [&](int c0, int col, float (&acc0)[16], float (&acc1)[16]) {
                        float own0[16], own1[16];
                        ld_acc(tacc + (col ? C::kUOff : 0) + c0, own0);
                        if (kAccs == 2) ld_acc(tacc + C::kUOff + c0, own1);
#pragma unroll
                        for (int i = 0; i < 16; ++i) acc0[i] = acc1[i] = 0.f;
                        for (int sl0 = 0; sl0 < it.S; sl0 += kSumBatch) {
                            float4 a4[kSumBatch][kAccs][4];
#pragma unroll
                            for (int j = 0; j < kSumBatch; ++j) {
                                const int sl = sl0 + j;
                                const bool other_slice = sl < it.S && sl != it.slice;
                                const float4* other =
                                    reinterpret_cast<const float4*>(p.partials + (slot0 + sl) * C::kSlotFloats);
#pragma unroll
                                for (int h = 0; h < kAccs; ++h) {
                                    const int cb = (h == 1 || col) ? kMaxN : 0;
                                    const bool valid = (h == 1 || col) ? v1 : v0;
#pragma unroll
                                    for (int q = 0; q < 4; ++q)
                                        a4[j][h][q] = valid && other_slice && c0 + 4 * q < t.nrows
                                                          ? __ldcg(other + slot_f4(((cb + c0) >> 2) + q, r))
                                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                                }
                            }
#pragma unroll
                            for (int j = 0; j < kSumBatch; ++j) {
                                const int sl = sl0 + j;
                                if (sl >= it.S) break;
#pragma unroll
                                for (int h = 0; h < kAccs; ++h) {
                                    float* acc = h == 0 ? acc0 : acc1;
                                    const float* own = h == 0 ? own0 : own1;
                                    if (sl == it.slice) {
#pragma unroll
                                        for (int i = 0; i < 16; ++i) acc[i] += own[i];
                                    } else {
#pragma unroll
                                        for (int q = 0; q < 4; ++q) {
                                            acc[4 * q] += a4[j][h][q].x;
                                            acc[4 * q + 1] += a4[j][h][q].y;
                                            acc[4 * q + 2] += a4[j][h][q].z;
                                            acc[4 * q + 3] += a4[j][h][q].w;
                                        }
                                    }
                                }
                            }
                        }
                    };
                    for (int c0 = 0; c0 < t.nrows; c0 += 16) {
                        float g[16], u[16];
                        if (kAccs == 2) {
                            sum_pass(c0, 0, g, u);
                        } else {
                            float unused[16];
                            sum_pass(c0, 0, g, unused);
                            sum_pass(c0, kMaxN, u, unused);
                        }
                        emit(c0, g, u);
                    }
                    if (r == 0) tile_ctr[it.ctr] = 0;
                }
            }
            if (gate_up && finished) {
                // this gate/up tile's activations are stored: count it for its token chunk
                fence_proxy_async_global();
                named_sync(1, 128);
                if (r == 0) red_add_release_gpu(&band_done[t.chunk * kFfnBands + (t.f0 / 128) / BS], 1);
            }
            tc_fence_before();
            mbar_arrive(&tempty[b]);
            ++ac;
        }
    }

    tc_fence_before();
    __syncthreads();
    // the last block to finish re-zeroes the control words for the next launch
    if (threadIdx.x == 0) *last_block = atomic_add_acq_rel_gpu(done_ctr, 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (*last_block) {
        const long long nc = n_chunks < kFfnMaxChunks ? n_chunks : kFfnMaxChunks;
        for (long long c = threadIdx.x; c < nc * kFfnBands; c += blockDim.x) band_done[c] = 0;
        if (kFp8) {
            const int rows = seg[n_groups] < kFfnMaxRows ? seg[n_groups] : kFfnMaxRows;
            for (int r = threadIdx.x; r < rows; r += blockDim.x) act_amax[r] = 0u;
        }
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
