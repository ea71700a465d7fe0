// moe_ffn_pair.cuh -- the fused decode expert FFN with FP8 (E4M3) weights on
// CTA pairs (thread-block clusters of 2, 2-SM tcgen05 MMAs).
//
// At decode sizes the FP8 stream is bound by MMA issue, not by bytes: one
// kind::f16 MMA of 128 weight rows x 16 K covers 2048 weights whatever the
// (tiny) token count, so a single CTA spends about as long issuing a stage's
// MMAs as the stage's codes take to stream.  On a CTA pair one MMA covers
// M = 256 weight rows, the 128 of each CTA, so each SM's weight bytes need
// half the instructions.
//
// Work items as in moe_ffn_stream_kernel, per pair: phase A = (token chunk,
// block of 256 features: each CTA the gate and up rows of its 128), phase B =
// (token chunk, block of 512 features: each CTA two 128-row tiles); tiles
// with few items are cut into K-slices finished by their last slice; phase B
// of a chunk waits until both halves of every phase-A tile of that chunk have
// stored their activations.
//
// Roles in each CTA: warp 0 lane 0 the TMA producer, warp 1 the TMEM owner
// (and, in the leader, the MMA issuer), warps 2..5 the epilogue, warps 6..13
// the converters that widen this CTA's codes into its own tensor memory.
//  * The leader's producer takes each item from the global counter and writes
//    its id into both CTAs' item rings (a remote store and a release-arrive on
//    the peer's ring barrier); every consumer of either CTA frees the slot on
//    the leader's ring barrier.
//  * Each CTA loads its own weight tiles (completing on its own barrier, for
//    its converters) and its half of the token rows with the 2-CTA TMA form
//    (completing on the leader's barrier, for the MMA).
//  * The converters of both CTAs arrive on the leader's conversion barrier;
//    the leader issues the stage's MMAs (A from each CTA's tensor memory, B
//    from each CTA's shared memory) and commits the stage, the conversion
//    buffer and finished accumulators to the barriers of both CTAs.
//  * Each CTA's epilogue reads its own 128 accumulator rows and frees the
//    accumulator on the leader's barrier.
// Every wait is bounded (status word, abort flag); both CTAs leave together
// through a cluster barrier before tensor memory is freed.
#pragma once

#include "moe_ffn_stream.cuh"

namespace moe {

template <int kMaxN>
struct FfnPairCfg {
    static constexpr int kBK = 64;                     // K (codes) per stage
    static constexpr int kRawWBytes = 128 * kBK;       // one 128-row tile of E4M3 codes
    static constexpr int kXRows = kMaxN / 2;           // this CTA's half of the token rows
    static constexpr int kXTileBytes = kXRows * 128;   // f16 rows of 64 elements
    static constexpr int kStageBytes = 2 * kRawWBytes + kXTileBytes;
    static constexpr int kConv = kMaxN <= 64 ? 3 : 2;  // TMEM buffers of widened weights
    static constexpr int kConvCols = 64;               // two 128 x 64 f16 tiles: 2 x 32 columns
    static constexpr int kConvThreads = 256;           // converter warps 6..13
    static constexpr int kThreads = kFfnThreads + kConvThreads;
    static constexpr int kAccCols = 2 * kMaxN;
    static constexpr int kNumAcc = kMaxN == 128 ? 1 : 2;
    static constexpr int kConvCol0 = kNumAcc * kAccCols;
    static constexpr int kUnit = 32;                   // token rows per MMA N step (2-CTA, A in TMEM)
    static constexpr int kTableBytes = 2 * (kMaxGroups + 1) * 4;
    static constexpr int kMiscBytes = 1024;
    static constexpr int kBudget = 227 * 1024 - 1024 - kTableBytes - kMiscBytes;
    static constexpr int kStagesRaw = kBudget / kStageBytes;
    static constexpr int kStages = kStagesRaw > 10 ? 10 : kStagesRaw;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kTableBytes + kMiscBytes;
    static constexpr int kSlotFloats = 128 * kAccCols;
    // consumers of an item-ring slot, counted on the leader's barrier: the
    // leader's MMA thread, epilogue threads and converter threads, then the
    // peer's producer and its epilogue and converter warps (one arrival each)
    static constexpr int kRingConsumers = 1 + 128 + kConvThreads + 1 + 4 + kConvThreads / 32;
    static_assert(kStageBytes % 1024 == 0, "stages keep the swizzle atoms aligned");
    static_assert(kMaxN == 32 || kMaxN == 64 || kMaxN == 128, "decode token tiles");
    static_assert(kAccCols * kNumAcc + kConv * kConvCols <= 512, "TMEM columns");
    static_assert((3 * kStages + 2 * kNumAcc + 2 * kFfnRing + 2 * kConv + 1) * 8 + 4 * kFfnRing + 16 <= kMiscBytes,
                  "misc area");
};

template <int kMaxN>
__global__ void __launch_bounds__(FfnPairCfg<kMaxN>::kThreads, 1)
    moe_ffn_fp8_pair_kernel(const __grid_constant__ CUtensorMap tm_w13, const __grid_constant__ CUtensorMap tm_w2,
                            const __grid_constant__ CUtensorMap tm_xa, const __grid_constant__ CUtensorMap tm_xb,
                            const FfnParams p) {
    using C = FfnPairCfg<kMaxN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stage_base = smem;
    int* seg = reinterpret_cast<int*>(smem + C::kStages * C::kStageBytes);
    int* cbase = seg + (kMaxGroups + 1);
    uint8_t* misc = reinterpret_cast<uint8_t*>(cbase + (kMaxGroups + 1));
    uint64_t* full = reinterpret_cast<uint64_t*>(misc);  // leader: both CTAs' token halves
    uint64_t* wfull = full + C::kStages;                 // this CTA's weight tiles
    uint64_t* empty = wfull + C::kStages;                // this CTA's stage free (MMA commit)
    uint64_t* tfull = empty + C::kStages;
    uint64_t* tempty = tfull + C::kNumAcc;               // leader: both CTAs' epilogues
    uint64_t* ring_full = tempty + C::kNumAcc;
    uint64_t* ring_empty = ring_full + kFfnRing;         // leader: consumers of both CTAs
    uint64_t* conv_full = ring_empty + kFfnRing;         // leader: converter warps of both CTAs
    uint64_t* conv_empty = conv_full + C::kConv;
    uint64_t* drain_bar = conv_empty + C::kConv;
    int* ring = reinterpret_cast<int*>(drain_bar + 1);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(ring + kFfnRing);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    int* bcast = const_cast<int*>(abort_flag) + 1;
    int* last_block = bcast + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int n_groups = p.n_groups;
    const uint64_t limit = p.wait_limit_ns;
    int* work_ctr = p.ctl;
    int* done_ctr = p.ctl + 1;
    int* chunk_done = p.ctl + 2;
    int* tile_ctr = p.ctl + 2 + kFfnMaxChunks;
    // cluster addresses of the leader's shared barriers and of the peer's ring
    auto at_leader = [](const void* a) { return map_to_rank(smem_u32(a), 0); };
    auto at_peer = [](const void* a) { return map_to_rank(smem_u32(a), 1); };

    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&wfull[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < C::kNumAcc; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 2 * 128);
        }
        for (int r = 0; r < kFfnRing; ++r) {
            mbar_init(&ring_full[r], 1);
            mbar_init(&ring_empty[r], C::kRingConsumers);
        }
        for (int c = 0; c < C::kConv; ++c) {
            mbar_init(&conv_full[c], 2 * (C::kConvThreads / 32));
            mbar_init(&conv_empty[c], 1);
        }
        mbar_init(drain_bar, 1);
        fence_barrier_init();
        *abort_flag = 0;
        tma_prefetch_desc(&tm_w13);
        tma_prefetch_desc(&tm_w2);
        tma_prefetch_desc(&tm_xa);
        tma_prefetch_desc(&tm_xb);
    }
    if (warp == 1) tmem_alloc_pair(tmem_holder, 512);
    cluster_sync_all();  // both CTAs' barriers exist before any remote arrive or commit targets them
    pdl_wait();
    for (int g = threadIdx.x; g <= n_groups; g += blockDim.x)
        seg[g] = p.seg_offsets ? p.seg_offsets[g] : (g == 0 ? 0 : p.seg_rows);
    __syncthreads();
    if (warp == 0) {
        int running = 0;
        for (int base = 0; base < n_groups; base += 32) {
            const int g = base + lane;
            const int n = g < n_groups ? chunks_of(seg[g + 1] - seg[g], kMaxN, C::kUnit) : 0;
            int incl = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
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

    // ---- the item space (identical in every thread of both CTAs)
    const int G = gridDim.x / 2;  // pairs
    const long long n_chunks = cbase[n_groups];
    const int NFA = (p.I + 255) / 256, NFB = (p.H + 511) / 512;
    const int KIA = (p.H + C::kBK - 1) / C::kBK, KIB = (p.I + C::kBK - 1) / C::kBK;
    const long long tilesA = n_chunks * NFA, tilesB = n_chunks * NFB;
    // each item of a split tile takes one partial slot per CTA
    const int SA = ffn_slices(tilesA, KIA, G, p.max_slots_phase / 2);
    const int SB = ffn_slices(tilesB, KIB, G, p.max_slots_phase / 2);
    const long long nA = tilesA * SA, nB = tilesB * SB;
    const long long total = nA + nB;
    const long long slotsA = SA > 1 ? nA : 0;
    const bool oversize = n_chunks > kFfnMaxChunks || (SA > 1 && 2 * tilesA > kFfnTileCtrs / 2) ||
                          (SB > 1 && 2 * tilesB > kFfnTileCtrs / 2);

    auto item_of = [&](long long id, FfnItem& it, Tile& t) {
        if (id < nA) {
            it.phase = 0;
            it.tile = id / SA;
            it.slice = (int)(id - it.tile * SA);
            it.S = SA;
            it.kb = (int)((long long)it.slice * KIA / SA);
            it.ke = (int)((long long)(it.slice + 1) * KIA / SA);
            it.slot = id * 2 + rank;
            it.ctr = it.tile * 2 + rank;
            t = decode_tile_w(it.tile, seg, cbase, n_groups, NFA, 256, C::kUnit, 2 * p.I);
        } else {
            const long long j = id - nA;
            it.phase = 1;
            it.tile = j / SB;
            it.slice = (int)(j - it.tile * SB);
            it.S = SB;
            it.kb = (int)((long long)it.slice * KIB / SB);
            it.ke = (int)((long long)(it.slice + 1) * KIB / SB);
            it.slot = (slotsA + j) * 2 + rank;
            it.ctr = kFfnTileCtrs / 2 + it.tile * 2 + rank;
            t = decode_tile_w(it.tile, seg, cbase, n_groups, NFB, 512, C::kUnit, p.H);
        }
    };
    // a consumer has read ring slot rs: the leader's threads arrive one by one,
    // the peer's warps once each (after every lane has read it)
    auto ring_release = [&](int rs) {
        if (leader) {
            mbar_arrive(&ring_empty[rs]);
        } else {
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(at_leader(&ring_empty[rs]));
        }
    };
    auto ring_wait = [&](int rs, uint32_t rph) {
        return leader ? mbar_wait_bounded(&ring_full[rs], rph, limit, abort_flag)
                      : mbar_wait_bounded_cluster(&ring_full[rs], rph, limit, abort_flag);
    };

    if (warp == 0) {
        // ------------------------------------------- item fetch + TMA loads
        if (lane == 0) {
            const uint64_t pol_w_once = policy_evict_first();
            const uint64_t pol_w_shared = policy_evict_normal();
            const uint64_t pol_x = policy_evict_last();
            int fills_w[C::kStages], fills_x[C::kStages];
#pragma unroll
            for (int s = 0; s < C::kStages; ++s) fills_w[s] = fills_x[s] = 0;
            uint32_t kc = 0, n = 0;
            bool ok = !oversize;
            if (oversize) atomicOr(p.status, kStatusCapacity);  // not a wait: the item space does not fit
            while (true) {
                const int rs = n % kFfnRing;
                const uint32_t rph = (n / kFfnRing) & 1u;
                long long id = -1;
                if (leader) {
                    if (ok) {
                        if (!mbar_wait_bounded(&ring_empty[rs], rph ^ 1u, limit, abort_flag)) {
                            ok = false;
                        } else {
                            id = atomicAdd(work_ctr, 1);
                            if (id >= total) id = -1;
                        }
                    }
                    if (!ok) id = -1;  // the end marker wakes every consumer of both CTAs
                    ring[rs] = (int)id;
                    mbar_arrive(&ring_full[rs]);
                    st_shared_cluster_u32(at_peer(&ring[rs]), (uint32_t)(int)id);
                    mbar_arrive_cluster(at_peer(&ring_full[rs]));  // release: the store above is visible
                } else {
                    if (!ring_wait(rs, rph)) {
                        ok = false;
                        break;
                    }
                    id = ring[rs];
                    mbar_arrive_cluster(at_leader(&ring_empty[rs]));
                }
                ++n;
                if (id < 0) break;
                FfnItem it;
                Tile t;
                item_of(id, it, t);
                const bool gate_up = it.phase == 0;
                const CUtensorMap* tw = gate_up ? &tm_w13 : &tm_w2;
                const CUtensorMap* tx = gate_up ? &tm_xa : &tm_xb;
                const int wrow = t.wrow + (int)rank * (gate_up ? 128 : 256);
                const int second = gate_up ? p.I : 128;  // up rows, or the next 128 features
                const int xn = t.mma_n / 2;
                const int xrow = t.row0 + (int)rank * xn;
                const uint64_t pol_w = t.nch > 1 ? pol_w_shared : pol_w_once;
                auto load_w = [&](int s, int k) {
                    uint8_t* st = stage_base + s * C::kStageBytes;
                    mbar_arrive_expect_tx(&wfull[s], 2 * C::kRawWBytes);
                    tma_load_2d(st, tw, &wfull[s], k * C::kBK, wrow, pol_w);
                    tma_load_2d(st + C::kRawWBytes, tw, &wfull[s], k * C::kBK, wrow + second, pol_w);
                    ++fills_w[s];
                };
                auto load_x = [&](int s, int k) {
                    uint8_t* xs = stage_base + s * C::kStageBytes + 2 * C::kRawWBytes;
                    // both CTAs' halves complete on the leader's barrier, which
                    // the leader expects in full (a negative count in between is
                    // allowed: the phase cannot complete before the expect)
                    if (leader) mbar_arrive_expect_tx(&full[s], (uint32_t)t.mma_n * 128u);
                    const uint32_t fb = at_leader(&full[s]);
                    for (int r = 0; r < xn; r += 16)
                        tma_load_2d_pair(xs + r * 128, tx, fb, k * C::kBK, xrow + r, pol_x);
                    ++fills_x[s];
                };
                int pre = 0;
                if (!gate_up) {
                    // weights first, then the activations once both halves of every
                    // phase-A tile of this chunk are stored
                    const int want = it.ke - it.kb < C::kStages ? it.ke - it.kb : C::kStages;
                    for (; pre < want; ++pre) {
                        const int s = (kc + pre) % C::kStages;
                        const uint32_t ph = ((kc + pre) / C::kStages) & 1u;
                        if (!mbar_wait_bounded(&empty[s], ph ^ 1u, limit, abort_flag)) {
                            ok = false;
                            break;
                        }
                        load_w(s, it.kb + pre);
                    }
                    if (ok) {
                        const uint64_t t0 = global_ns();
                        while ((int)ld_acquire_u32(&chunk_done[t.chunk]) < 2 * NFA) {
                            if (*abort_flag || global_ns() - t0 > limit) {
                                ok = false;
                                break;
                            }
                            __nanosleep(64);
                        }
                        if (ok) fence_proxy_async_global();
                    }
                    for (int j = 0; j < pre; ++j) load_x((kc + j) % C::kStages, it.kb + j);
                    kc += pre;
                    if (!ok) {
                        if (leader) continue;  // the next turn publishes the end marker
                        break;
                    }
                }
                for (int k = it.kb + pre; k < it.ke; ++k, ++kc) {
                    const int s = kc % C::kStages;
                    const uint32_t ph = (kc / C::kStages) & 1u;
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1u, limit, abort_flag)) {
                        ok = false;
                        break;
                    }
                    load_w(s, k);
                    load_x(s, k);
                }
                if (!ok && !leader) break;
            }
            if (!ok) {
                *abort_flag = 1;
                if (!oversize) atomicOr(p.status, kStatusTimeout);
            }
            // every issued copy lands before the pair leaves: this CTA's weight
            // tiles on its own barriers, both halves of the tokens on the leader's
            for (int s = 0; s < C::kStages; ++s) {
                if (fills_w[s] > 0) mbar_drain(&wfull[s], (uint32_t)(fills_w[s] - 1) & 1u, limit);
                if (leader && fills_x[s] > 0) mbar_drain(&full[s], (uint32_t)(fills_x[s] - 1) & 1u, limit);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer (leader)
        if (lane == 0 && leader) {
            uint32_t kc = 0, ac = 0, n = 0;
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
                if (!mbar_wait_bounded_cluster(&tempty[b], aph ^ 1u, limit, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d0 = tmem_base + b * C::kAccCols;
                const uint32_t d1 = d0 + kMaxN;
                const uint32_t idesc = umma_idesc(Elt<__half>::kMmaFmt, 256, t.mma_n);
                for (int k = it.kb; k < it.ke; ++k, ++kc) {
                    const int s = kc % C::kStages;
                    const uint32_t ph = (kc / C::kStages) & 1u;
                    const int cv = (int)(kc % C::kConv);
                    if (!mbar_wait_bounded(&full[s], ph, limit, abort_flag) ||
                        !mbar_wait_bounded_cluster(&conv_full[cv], (kc / C::kConv) & 1u, limit, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t bx = umma_desc_sw128(smem_u32(stage_base + s * C::kStageBytes + 2 * C::kRawWBytes));
                    const uint32_t a0 = tmem_base + C::kConvCol0 + cv * C::kConvCols;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t acc = (k > it.kb || kk > 0) ? 1u : 0u;
                        umma_pair_f16_tmem_a(d0, a0 + 8 * kk, bx + 2 * kk, idesc, acc);
                        umma_pair_f16_tmem_a(d1, a0 + 32 + 8 * kk, bx + 2 * kk, idesc, acc);
                    }
                    // the stage and the conversion buffer are free in both CTAs
                    umma_commit_pair(smem_u32(&empty[s]));
                    umma_commit_pair(at_peer(&empty[s]));
                    umma_commit_pair(smem_u32(&conv_empty[cv]));
                    umma_commit_pair(at_peer(&conv_empty[cv]));
                }
                if (!ok) break;
                umma_commit_pair(smem_u32(&tfull[b]));
                umma_commit_pair(at_peer(&tfull[b]));
                ++ac;
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(p.status, kStatusTimeout);
                umma_commit_pair(smem_u32(drain_bar));
                mbar_drain(drain_bar, 0, limit);
            }
        }
    } else if (warp >= 6) {
        // ------------------------------------------- FP8 -> f16 converters
        // as in moe_ffn_stream_kernel: warps 6..9 widen the stage's first
        // weight tile of this CTA, warps 10..13 its second, one row per thread
        // (the warp's TMEM lane quadrant), into this CTA's tensor memory
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const int tt = (warp - 6) >> 2;
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        uint32_t kc = 0, n = 0;
        bool ok = true;
        while (ok) {
            const int rs = n % kFfnRing;
            const uint32_t rph = (n / kFfnRing) & 1u;
            if (!__all_sync(0xffffffffu, ring_wait(rs, rph))) {
                ok = false;
                break;
            }
            const long long id = ring[rs];
            ring_release(rs);
            ++n;
            if (id < 0) break;
            FfnItem it;
            Tile t;
            item_of(id, it, t);
            for (int k = it.kb; k < it.ke; ++k, ++kc) {
                const int s = kc % C::kStages;
                const int cv = (int)(kc % C::kConv);
                const bool got = mbar_wait_bounded(&wfull[s], (kc / C::kStages) & 1u, limit, abort_flag) &&
                                 mbar_wait_bounded(&conv_empty[cv], ((kc / C::kConv) & 1u) ^ 1u, limit, abort_flag);
                if (!__all_sync(0xffffffffu, got)) {  // the whole warp leaves together (warp-wide TMEM stores)
                    ok = false;
                    break;
                }
                tc_fence_after();  // the MMAs that read this buffer before have completed
                const uint8_t* src = stage_base + s * C::kStageBytes + tt * C::kRawWBytes + row * C::kBK;
                uint32_t w[32];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint4 v = *reinterpret_cast<const uint4*>(src + ((c ^ ((row >> 1) & 3)) << 4));
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
                tmem_st32(tmem_base + lane_base + C::kConvCol0 + cv * C::kConvCols + tt * 32, w);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (leader) mbar_arrive(&conv_full[cv]);
                    else mbar_arrive_cluster(at_leader(&conv_full[cv]));
                }
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
            if (!__all_sync(0xffffffffu, ring_wait(rs, rph))) {
                *abort_flag = 1;
                atomicOr(p.status, kStatusTimeout);
                break;
            }
            const long long id = ring[rs];
            ring_release(rs);
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
            const int f = t.f0 + (int)rank * (gate_up ? 128 : 256) + r;
            const bool v0 = f < n_out;
            const bool v1 = gate_up ? v0 : (f + 128 < n_out);
            __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.y) + (long long)t.row0 * n_out + f;
            __half* arow = reinterpret_cast<__half*>(p.act) + (long long)t.row0 * n_out + f;
            // the row scales of the two accumulators' weight rows, times 2^8 (the
            // widened codes hold value x 2^-8)
            float sc0, sc1;
            if (gate_up) {
                const float* sr = p.s13 + (long long)t.group * 2 * p.I;
                sc0 = v0 ? __ldg(sr + f) * 256.f : 0.f;
                sc1 = v0 ? __ldg(sr + p.I + f) * 256.f : 0.f;
            } else {
                const float* sr = p.s2 + (long long)t.group * p.H;
                sc0 = v0 ? __ldg(sr + f) * 256.f : 0.f;
                sc1 = v1 ? __ldg(sr + f + 128) * 256.f : 0.f;
            }
            auto emit = [&](int c0, float (&g)[16], float (&u)[16]) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    g[i] *= sc0;
                    u[i] *= sc1;
                }
                if (gate_up) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) g[i] = silu_mul(g[i], u[i]);
                    if (v0) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c0 + i < t.nrows) store_out<__half>(arow + (long long)(c0 + i) * n_out, g[i]);
                    }
                } else {
                    if (v0) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c0 + i < t.nrows) store_out<__nv_bfloat16>(orow + (long long)(c0 + i) * n_out, g[i]);
                    }
                    if (v1) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c0 + i < t.nrows)
                                store_out<__nv_bfloat16>(orow + 128 + (long long)(c0 + i) * n_out, u[i]);
                    }
                }
            };
            bool finished = true;  // this item completed its tile half
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
                // split tile: publish this slice's half, the last slice of this
                // half sums them all in slice order
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
                    const long long slot0 = it.slot - 2LL * it.slice;  // this half's slot of slice 0
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
                                    reinterpret_cast<const float4*>(p.partials + (slot0 + 2LL * sl) * C::kSlotFloats);
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
                // this half of a gate/up tile has stored its activations
                fence_proxy_async_global();
                __threadfence();
                named_sync(1, 128);
                if (r == 0) atomicAdd(&chunk_done[t.chunk], 1);
            }
            tc_fence_before();
            if (leader) mbar_arrive(&tempty[b]);
            else mbar_arrive_cluster(at_leader(&tempty[b]));
            ++ac;
        }
    }

    tc_fence_before();
    cluster_sync_all();  // neither CTA frees TMEM or leaves while the pair's MMAs or arrivals may target it
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
        tmem_dealloc_pair(tmem_base, 512);
    }
}

}  // namespace moe
