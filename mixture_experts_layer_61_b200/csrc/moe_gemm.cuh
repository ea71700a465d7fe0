// moe_gemm.cuh -- persistent grouped GEMM on the sm_100a tensor cores
// (tcgen05.mma, accumulators in TMEM, operands staged by TMA with the
// 128-byte swizzle), used for every contraction of the layer:
//   * the routed experts' gate/up projections with the SwiGLU epilogue and
//     their down projections (the "GroupGEMM" of the talk notes' Table 1 and
//     "Key findings 5"), one group per expert segment of the padded rows;
//   * the dense SwiGLU FFN (shared experts, DenseFA, DensePA) as one group;
//   * the router GEMM (fp32 logits) as one group.
//
// Orientation.  The weight rows are the MMA's M side (128 output features
// per tile) and the token rows its N side (16..kMaxN tokens per tile, a
// multiple of 16).  Decode (one or two tokens per expert) then costs a
// 128 x 16 MMA per 128 weight rows instead of a 128-row tile of padding, and
// prefill uses N up to 256.  The accumulator D[feature][token] lives in TMEM
// (lane = feature, column = token).
//
// Tiles.  A group g owns rows [seg[g], seg[g+1]) of the token matrix X.  The
// rows are cut into chunks of at most kMaxN rows (in units of 16, balanced);
// a tile is (group, 128-feature block f, chunk j), ordered f-major inside a
// group so that the chunks sharing one weight block run side by side and
// reuse it from L2.  Each tile reduces over K = kdim in steps of 128 bytes.
//
// Schedule.  gridDim.x persistent blocks (one per SM).  Whole waves of tiles
// are dealt round-robin; the remaining one to two waves (all but the first
// wave, with fewer than two) are split evenly by k-iterations across the
// blocks (stream-K), so every block streams the same
// number of weight bytes even when there are fewer tiles than SMs (decode).
// A tile split across blocks is finished by the last block to arrive: each
// contributor stores its fp32 partial tile, then increments the tile's
// counter; the block that brings the counter to the number of contributors
// sums all partials in block order (deterministic) and runs the epilogue.
// No block ever waits on another block.
//
// Roles (320 threads): warp 0 issues TMA loads, warp 1 owns TMEM and issues
// the MMAs, warps 2..9 run the epilogue (TMEM -> registers -> global), two
// warps per TMEM lane quadrant, each on half of the tile's token columns.
// Where the packed results fit in registers, the epilogue reads the whole
// accumulator, frees it for the next tile's MMAs and only then stores.  All
// waits are bounded by a deadline; a wait that runs out sets the status word
// and every role winds down (in-flight copies and MMAs are drained first).
#pragma once

#include "moe_common.cuh"

namespace moe {

constexpr int kMaxGroups = 1024;
constexpr int kGemmEpiWarps = 8;                      // two per TMEM lane quadrant
constexpr int kGemmThreads = 64 + 32 * kGemmEpiWarps;  // producer warp, MMA warp, epilogue
constexpr int kFfnThreads = 192;

// Partial-tile slot layout: column c of row r (r < 128) at float index
// ((c / 4) * 128 + r) * 4 + c % 4, so that a warp moves 32 consecutive
// float4 (512 contiguous bytes) per access.
__device__ __forceinline__ long long slot_f4(int c4, int r) { return (long long)c4 * 128 + r; }

struct GemmParams {
    const int32_t* seg_offsets;  // [n_groups + 1] row offsets into X, or nullptr: one group [0, seg_rows)
    int n_groups;
    int seg_rows;
    int n_out;            // output features
    int kdim;             // reduction length
    int w_group_stride;   // weight rows from one group to the next
    int up_offset;        // weight rows from a gate row to its up row (SwiGLU)
    void* out;            // output rows (same row index as X), out_ld elements apart
    int out_ld;
    int* counters;        // >= 2 * gridDim.x ints; zero on entry and on exit
    float* partials;      // 2 * gridDim.x slots of 128 * kAccCols floats
    unsigned* status;     // status word (bit kStatusTimeout)
    uint64_t wait_limit_ns;
    int withhold_first_load;
    int sk_min_units;     // minimum k-iterations per stream-K block
    int max_split;        // stream-K: most blocks contributing to one tile
    int split_tail;       // 1: whole waves data-parallel, the last partial wave in aligned k-slices
};

// Epilogue kinds: one 128-row weight tile per stage (plain store); gate and
// up tiles of the same 128 features (SwiGLU); two adjacent 128-feature
// blocks sharing one token tile (wide plain store, 256 features per tile).
constexpr int kEpiPlain = 0, kEpiSwiGLU = 1, kEpiWide = 2;

template <typename T, int kEpi, int kMaxN, int kCta = 1>
struct GemmCfg {
    // Operand tiles are K-major rows of kRowBytes with the swizzle of that
    // width.  128-byte rows: 64-byte rows (twice the stages in the same
    // shared memory) measured slower on B200, the per-stage barrier and TMA
    // overhead outweighing the deeper lookahead.
    static constexpr int kRowBytes = 128;
    static constexpr int kBK = kRowBytes / Elt<T>::kBytes;  // K elements per stage
    static constexpr int kMmaK = 32 / Elt<T>::kBytes;       // K per MMA instruction
    static constexpr int kKSteps = kBK / kMmaK;             // MMAs per operand pair and stage
    static constexpr int kNW = kEpi == kEpiPlain ? 1 : 2;  // weight tiles per stage
    static constexpr int kFeat = kEpi == kEpiWide ? 256 : 128;  // output features per CTA and tile
    static constexpr int kFeatTile = kFeat * kCta;                 // output features per tile
    static constexpr int kUnit = 16 * kCta;                        // token-row granularity of the MMA
    static constexpr int kWTileBytes = 128 * kRowBytes;
    static constexpr int kXBoxRows = 16;       // token rows per TMA box: 16, 64 and kMaxN
    static constexpr int kXBoxMid = 64;
    static constexpr int kXTileBytes = (kMaxN / kCta) * kRowBytes;  // this CTA's share of the token tile
    static constexpr int kStageBytes = kNW * kWTileBytes + kXTileBytes;
    static constexpr int kAccCols = kNW * kMaxN;
    static constexpr int kNumAcc = (512 / kAccCols) >= 2 ? 2 : 1;
    static constexpr int kTableBytes = 2 * (kMaxGroups + 1) * 4;
    static constexpr int kMiscBytes = 512;
    static constexpr int kMaxStages = 16;
    static constexpr int kBudget = 227 * 1024 - 1024 - kTableBytes - kMiscBytes;
    static constexpr int kStagesRaw = kBudget / kStageBytes;
    static constexpr int kStages = kStagesRaw > kMaxStages ? kMaxStages : kStagesRaw;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kTableBytes + kMiscBytes;
    static_assert(kStages >= 2, "pipeline needs two stages");
    static_assert(kMaxN % kUnit == 0 && kMaxN >= kUnit && kMaxN <= 256, "MMA N range");
    static_assert(kCta == 1 || kCta == 2, "one CTA or a CTA pair");
    static_assert(kAccCols * kNumAcc <= 512, "TMEM columns");
    static_assert(2 * kMaxStages * 8 + 2 * kNumAcc * 8 + 8 + 12 <= kMiscBytes, "barriers fit");
    static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte alignment of the swizzle atoms");
};

// ------------------------------------------------------------- scheduling
struct Tile {
    int group, f0, row0, nrows, mma_n, wrow, nch, chunk;
};

// Two ways to share out the tiles left after the whole data-parallel waves:
//  * contiguous stream-K (split_tail 0): the last one to two waves of tiles
//    as one range of (tile, k-iteration) units cut evenly across the blocks;
//  * aligned slices (split_tail 1): every whole wave data-parallel, and the
//    tiles of the last partial wave each cut into S equal k-slices, taken
//    slice-major and dealt round-robin (block c takes units c and c + G).
//    Tiles that share a weight block (adjacent token chunks) or a token chunk
//    (feature blocks of one expert) then stream the same k-slice at the same
//    time, so the shared operand is read from DRAM once; with contiguous
//    ranges the sharing tiles sit at different k-offsets and each reads it.
struct Sched {
    int n_groups, NF, KI, G, cta;
    long long total_tiles, dp_waves, dp_tiles, sk_tiles, U;
    int G_sk;
    int S;              // aligned slices per tail tile (0: contiguous stream-K)
    // iteration state
    long long w;        // next DP wave
    long long u, u_end; // stream-K cursor
    bool sk_first;
    int next_unit;      // aligned slices: this block's next local unit (0 or 1)

    __device__ long long beg(int c) const { return (long long)c * U / G_sk; }
    // block owning stream-K unit q
    __device__ int owner(long long q) const { return (int)(((q + 1) * (long long)G_sk - 1) / U); }
};

// Slices per tail tile for the aligned split: at most 2 units per block (the
// two partial slots), at least min_units k-iterations per slice, at most
// max_split contributors per tile; among those, the fewest slices with the
// shortest tail, ceil(tail * S / G) / S tile-times.
__device__ __forceinline__ int aligned_slices(long long tail, int G, int KI, long long min_units, int max_split) {
    if (tail <= 0) return 1;
    long long smax = (2LL * G) / tail;
    if (smax > max_split) smax = max_split;
    if (smax > KI / min_units) smax = KI / min_units;
    int best = 1;
    double best_t = (double)((tail + G - 1) / G);
    for (int s = 2; s <= smax; ++s) {
        const double t = (double)((tail * s + G - 1) / G) / s;
        if (t < best_t - 1e-9) {
            best_t = t;
            best = s;
        }
    }
    return best;
}

struct Item {
    long long tile;
    int kb, ke;
    bool split;   // partial tile (stream-K fixup)
    int slot;     // partial slot of this block (0 or 1)
    long long sk_tile;
};

// Scheduling unit: one CTA, or one CTA pair (cluster of 2) sharing each tile.
__device__ __forceinline__ void sched_init(Sched& s, const GemmParams& p, int total_chunks, int NF, int KI, int ncta) {
    s.n_groups = p.n_groups;
    s.NF = NF;
    s.KI = KI;
    s.G = gridDim.x / ncta;
    s.cta = blockIdx.x / ncta;
    s.total_tiles = (long long)total_chunks * NF;
    // at most max_split blocks share one tile: every block takes >= KI / kMaxSplit k-iterations
    long long min_units = (KI + p.max_split - 1) / p.max_split;
    if (min_units < p.sk_min_units) min_units = p.sk_min_units;
    s.S = 0;
    s.next_unit = 0;
    if (p.split_tail) {
        s.dp_waves = s.total_tiles / s.G;
        s.dp_tiles = s.dp_waves * s.G;
        s.sk_tiles = s.total_tiles - s.dp_tiles;  // < G: fits the counters and two slots per block
        s.S = aligned_slices(s.sk_tiles, s.G, KI, min_units, p.max_split);
        s.U = 0;
        s.G_sk = s.G;
        s.w = 0;
        s.u = s.u_end = 0;
        s.sk_first = true;
        return;
    }
    // Whole waves first, keeping one to two waves for the stream-K tail; with
    // fewer than two waves of tiles, one whole wave and the rest as stream-K,
    // so that the token chunks sharing a weight block (adjacent tiles) stream
    // it together at least in that wave.
    s.dp_waves = s.total_tiles >= 2LL * s.G ? s.total_tiles / s.G - 1 : (s.total_tiles >= s.G ? 1 : 0);
    s.dp_tiles = s.dp_waves * s.G;
    s.sk_tiles = s.total_tiles - s.dp_tiles;
    s.U = s.sk_tiles * KI;
    long long gsk = s.U / min_units;
    if (gsk < 1) gsk = 1;
    if (gsk > s.G) gsk = s.G;
    s.G_sk = (int)gsk;
    s.w = 0;
    if (s.U > 0 && s.cta < s.G_sk) {
        s.u = s.beg(s.cta);
        s.u_end = s.beg(s.cta + 1);
    } else {
        s.u = s.u_end = 0;
    }
    s.sk_first = true;
}

__device__ __forceinline__ bool sched_next(Sched& s, Item& it) {
    if (s.w < s.dp_waves) {
        it.tile = s.w * s.G + s.cta;
        it.kb = 0;
        it.ke = s.KI;
        it.split = false;
        it.slot = 0;
        it.sk_tile = -1;
        ++s.w;
        return true;
    }
    if (s.u < s.u_end) {
        long long st = s.u / s.KI;
        int kb = (int)(s.u - st * s.KI);
        long long left = s.u_end - s.u;
        int ke = (int)((long long)kb + left < s.KI ? kb + left : s.KI);
        it.tile = s.dp_tiles + st;
        it.kb = kb;
        it.ke = ke;
        it.sk_tile = st;
        it.split = !(kb == 0 && ke == s.KI);
        it.slot = s.sk_first ? 0 : 1;
        s.sk_first = false;
        s.u += ke - kb;
        return true;
    }
    if (s.S > 0 && s.next_unit < 2) {
        // aligned slices: unit q = cta + j G is slice q / tail of tail tile q % tail
        const long long q = (long long)s.cta + (long long)s.next_unit * s.G;
        if (q >= s.sk_tiles * s.S) return false;
        const long long st = q % s.sk_tiles;
        const int sl = (int)(q / s.sk_tiles);
        it.tile = s.dp_tiles + st;
        it.kb = (int)((long long)sl * s.KI / s.S);
        it.ke = (int)((long long)(sl + 1) * s.KI / s.S);
        it.sk_tile = st;
        it.split = s.S > 1;
        it.slot = s.next_unit;
        ++s.next_unit;
        return true;
    }
    return false;
}

// Rows of chunk j of a group of `rows` rows cut into `nch` chunks, in units of `unit` rows.
__device__ __forceinline__ void chunk_rows(int rows, int nch, int j, int unit, int& start, int& n, int& mma_n) {
    int units = (rows + unit - 1) / unit;
    int base = units / nch, extra = units % nch;
    int su = j * base + (j < extra ? j : extra);
    int mu = base + (j < extra ? 1 : 0);
    start = su * unit;
    mma_n = mu * unit;
    int left = rows - start;
    n = mma_n < left ? mma_n : left;
}

__device__ __forceinline__ int chunks_of(int rows, int max_n, int unit) {
    if (rows <= 0) return 0;
    int units = (rows + unit - 1) / unit;
    int per = max_n / unit;
    return (units + per - 1) / per;
}

__device__ __forceinline__ Tile decode_tile_w(long long tile, const int* seg, const int* cbase, int n_groups, int NF,
                                              int feat, int unit, int w_group_stride) {
    // group: largest g with cbase[g] * NF <= tile
    int lo = 0, hi = n_groups - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if ((long long)cbase[mid] * NF <= tile) lo = mid;
        else hi = mid - 1;
    }
    int g = lo;
    int nch = cbase[g + 1] - cbase[g];
    long long local = tile - (long long)cbase[g] * NF;
    int f = (int)(local / nch);
    int j = (int)(local - (long long)f * nch);
    Tile t;
    int start, n, mn;
    chunk_rows(seg[g + 1] - seg[g], nch, j, unit, start, n, mn);
    t.group = g;
    t.f0 = f * feat;
    t.row0 = seg[g] + start;
    t.nrows = n;
    t.mma_n = mn;
    t.wrow = g * w_group_stride + f * feat;
    t.nch = nch;
    t.chunk = cbase[g] + j;
    return t;
}

__device__ __forceinline__ Tile decode_tile(long long tile, const int* seg, const int* cbase, int n_groups, int NF,
                                            int feat, int unit, const GemmParams& p) {
    return decode_tile_w(tile, seg, cbase, n_groups, NF, feat, unit, p.w_group_stride);
}

template <typename OutT>
__device__ __forceinline__ void store_out(OutT* ptr, float v);
template <>
__device__ __forceinline__ void store_out<float>(float* ptr, float v) { *ptr = v; }
template <>
__device__ __forceinline__ void store_out<__half>(__half* ptr, float v) {
    *ptr = __float2half_rn(v);
}
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* ptr, float v) {
    *ptr = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// ------------------------------------------------------------------ kernel
template <typename T, typename OutT, int kEpi, int kMaxN, int kCta>
__global__ void __launch_bounds__(kGemmThreads, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                    const __grid_constant__ CUtensorMap tm_x64, const __grid_constant__ CUtensorMap tm_xbig,
                    const GemmParams p) {
    using C = GemmCfg<T, kEpi, kMaxN, kCta>;
    constexpr bool kSwiGLU = kEpi == kEpiSwiGLU;
    constexpr bool kTwo = C::kNW == 2;
    constexpr bool kPair = kCta == 2;
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
    uint64_t* drain_bar = tempty + C::kNumAcc;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    int* bcast = const_cast<int*>(abort_flag) + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_groups = p.n_groups;
    const uint64_t deadline = p.wait_limit_ns;  // per-wait limit
    // CTA pair: rank 0 (the leader) issues the MMAs for both; each CTA stages
    // its own 128 weight rows and half of the token rows, and holds in TMEM
    // the accumulators of its own 128 weight rows.
    const uint32_t rank = kPair ? cluster_rank() : 0u;

    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < C::kNumAcc; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 32 * kGemmEpiWarps * kCta);
        }
        mbar_init(drain_bar, 1);
        fence_barrier_init();
        *abort_flag = 0;
        tma_prefetch_desc(&tm_w);
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_x64);
        tma_prefetch_desc(&tm_xbig);
    }
    if (warp == 1) {
        if (kPair) tmem_alloc_pair(tmem_holder, 512);
        else tmem_alloc(tmem_holder, 512);
    }
    if (kPair) cluster_sync_all();  // the peer's barriers are initialised before any TMA or commit targets them
    pdl_wait();  // everything below reads or writes data shared with earlier kernels
    // segment table
    for (int g = threadIdx.x; g <= n_groups; g += blockDim.x)
        seg[g] = p.seg_offsets ? p.seg_offsets[g] : (g == 0 ? 0 : p.seg_rows);
    __syncthreads();
    if (warp == 0) {
        int running = 0;
        for (int base = 0; base < n_groups; base += 32) {
            int g = base + lane;
            int n = g < n_groups ? chunks_of(seg[g + 1] - seg[g], kMaxN, C::kUnit) : 0;
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

    const int NF = (p.n_out + C::kFeatTile - 1) / C::kFeatTile;
    const int KI = (p.kdim + C::kBK - 1) / C::kBK;
    Sched sch;
    sched_init(sch, p, cbase[n_groups], NF, KI, kCta);

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer
        if (lane == 0) {
            // weights read by one tile only are streamed with evict-first; weight
            // blocks that several token chunks share stay at normal priority
            const uint64_t pol_w_once = policy_evict_first();
            const uint64_t pol_w_shared = policy_evict_normal();
            const uint64_t pol_x = policy_evict_last();
            int fills[C::kStages];
#pragma unroll
            for (int s = 0; s < C::kStages; ++s) fills[s] = 0;
            uint32_t kc = 0;
            bool withhold = p.withhold_first_load && blockIdx.x == 0;
            bool ok = true;
            Item it;
            while (ok && sched_next(sch, it)) {
                Tile t = decode_tile(it.tile, seg, cbase, n_groups, NF, C::kFeatTile, C::kUnit, p);
                // this CTA's weight rows and token rows of the tile
                const int wrow = t.wrow + (int)rank * C::kFeat;
                const int xn = t.mma_n / kCta;
                const int xrow = t.row0 + (int)rank * xn;
                // bytes landing on the (leader's) full barrier per stage: both CTAs' shares
                const uint32_t bytes = kCta * (C::kNW * C::kWTileBytes + xn * C::kRowBytes);
                const uint64_t pol_w = t.nch > 1 ? pol_w_shared : pol_w_once;
                for (int k = it.kb; k < it.ke; ++k, ++kc) {
                    const int s = kc % C::kStages;
                    const uint32_t ph = (kc / C::kStages) & 1u;
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1u, deadline, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (withhold) {  // test hook: this stage is never filled
                        withhold = false;
                        continue;
                    }
                    uint8_t* st = stage_base + s * C::kStageBytes;
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], bytes);
                    const uint32_t fb = kPair ? map_to_rank(smem_u32(&full[s]), 0) : 0u;
                    auto load = [&](void* dst, const CUtensorMap* m, int c1, uint64_t pol) {
                        if (kPair) tma_load_2d_pair(dst, m, fb, k * C::kBK, c1, pol);
                        else tma_load_2d(dst, m, &full[s], k * C::kBK, c1, pol);
                    };
                    load(st, &tm_w, wrow, pol_w);
                    if (kTwo) load(st + C::kWTileBytes, &tm_w, wrow + (kSwiGLU ? p.up_offset : 128), pol_w);
                    uint8_t* xs = st + C::kNW * C::kWTileBytes;
                    int r = 0;
                    if (kMaxN / kCta > C::kXBoxMid && xn == kMaxN / kCta) {
                        load(xs, &tm_xbig, xrow, pol_x);
                        r = xn;
                    }
                    if (kMaxN / kCta >= C::kXBoxMid)
                        for (; r + C::kXBoxMid <= xn; r += C::kXBoxMid)
                            load(xs + r * C::kRowBytes, &tm_x64, xrow + r, pol_x);
                    for (; r < xn; r += C::kXBoxRows) load(xs + r * C::kRowBytes, &tm_x, xrow + r, pol_x);
                    ++fills[s];
                }
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(p.status, kStatusTimeout);
            }
            // every issued copy lands before the block exits (the leader's full
            // barriers count both CTAs' copies; the pair leaves together)
            if (rank == 0)
                for (int s = 0; s < C::kStages; ++s)
                    if (fills[s] > 0) mbar_drain(&full[s], (uint32_t)(fills[s] - 1) & 1u, p.wait_limit_ns);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0 && rank == 0) {
            uint32_t kc = 0, ac = 0;
            bool ok = true;
            Item it;
            while (ok && sched_next(sch, it)) {
                Tile t = decode_tile(it.tile, seg, cbase, n_groups, NF, C::kFeatTile, C::kUnit, p);
                const int b = ac % C::kNumAcc;
                const uint32_t aph = (ac / C::kNumAcc) & 1u;
                if (!mbar_wait_bounded(&tempty[b], aph ^ 1u, deadline, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_gate = tmem_base + b * C::kAccCols;
                const uint32_t d_up = d_gate + kMaxN;
                const uint32_t idesc = umma_idesc(Elt<T>::kMmaFmt, 128 * kCta, t.mma_n);
                for (int k = it.kb; k < it.ke; ++k, ++kc) {
                    const int s = kc % C::kStages;
                    const uint32_t ph = (kc / C::kStages) & 1u;
                    if (!mbar_wait_bounded(&full[s], ph, deadline, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint8_t* st = stage_base + s * C::kStageBytes;
                    auto desc = [](uint32_t a) { return C::kRowBytes == 128 ? umma_desc_sw128(a) : umma_desc_sw64(a); };
                    const uint64_t a0 = desc(smem_u32(st));
                    const uint64_t a1 = desc(smem_u32(st + C::kWTileBytes));
                    const uint64_t bx = desc(smem_u32(st + C::kNW * C::kWTileBytes));
#pragma unroll
                    for (int kk = 0; kk < C::kKSteps; ++kk) {
                        const uint32_t acc = (k > it.kb || kk > 0) ? 1u : 0u;
                        if (kPair) {
                            umma_pair_bf16(d_gate, a0 + 2 * kk, bx + 2 * kk, idesc, acc);
                            if (kTwo) umma_pair_bf16(d_up, a1 + 2 * kk, bx + 2 * kk, idesc, acc);
                        } else {
                            umma<T>(d_gate, a0 + 2 * kk, bx + 2 * kk, idesc, acc);
                            if (kTwo) umma<T>(d_up, a1 + 2 * kk, bx + 2 * kk, idesc, acc);
                        }
                    }
                    if (kPair) {  // the stage is free in both CTAs
                        umma_commit_pair(smem_u32(&empty[s]));
                        umma_commit_pair(map_to_rank(smem_u32(&empty[s]), 1));
                    } else {
                        umma_commit(&empty[s]);
                    }
                }
                if (!ok) break;
                if (kPair) {
                    umma_commit_pair(smem_u32(&tfull[b]));
                    umma_commit_pair(map_to_rank(smem_u32(&tfull[b]), 1));
                } else {
                    umma_commit(&tfull[b]);
                }
                ++ac;
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(p.status, kStatusTimeout);
                if (kPair) umma_commit_pair(smem_u32(drain_bar));
                else umma_commit(drain_bar);
                mbar_drain(drain_bar, 0, p.wait_limit_ns);
            }
        }
    } else {
        // -------------------------------------------------------- epilogue
        const int quad = warp & 3;                // TMEM lane quadrant this warp may access
        const int half = (warp - 2) >> 2;         // which share of the token columns
        const int r = quad * 32 + lane;           // TMEM lane = feature row within a 128-row block
        const int e = (warp - 2) * 32 + lane;     // epilogue thread 0 .. 255
        constexpr int kEpiThreads = 32 * kGemmEpiWarps;
        constexpr int kHalfN = kMaxN / (kGemmEpiWarps / 4);  // token columns per warp
        constexpr int kCh = kHalfN >= 32 ? 32 : 16;
        constexpr bool kBf16Out = sizeof(OutT) == 2;
        constexpr int kRegs = kBf16Out ? kHalfN / 2 : kHalfN;  // packed results of one accumulator
        constexpr bool kEarly = kEpi != kEpiWide && kRegs <= 64;
        const int cbeg = half * kHalfN;
        OutT* out = reinterpret_cast<OutT*>(p.out);
        uint32_t ac = 0;
        Item it;
        while (sched_next(sch, it)) {
            Tile t = decode_tile(it.tile, seg, cbase, n_groups, NF, C::kFeatTile, C::kUnit, p);
            const int b = ac % C::kNumAcc;
            const uint32_t aph = (ac / C::kNumAcc) & 1u;
            // every epilogue thread goes on, or all leave (the split path below
            // meets at named barriers, which a thread that left would never reach)
            const bool got = mbar_wait_bounded(&tfull[b], aph, deadline, abort_flag);
            if (!named_all(1, kEpiThreads, got)) {
                *abort_flag = 1;
                atomicOr(p.status, kStatusTimeout);
                break;
            }
            tc_fence_after();
            const uint32_t tacc = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + b * C::kAccCols;
            const int f = t.f0 + (int)rank * C::kFeat + r;
            // valid rows of the first and second accumulator
            const bool v0 = f < p.n_out;
            const bool v1 = kEpi == kEpiWide ? (f + 128 < p.n_out) : (kSwiGLU && v0);
            OutT* orow = out + (long long)t.row0 * p.out_ld + f;
            const int cend = t.nrows < cbeg + kHalfN ? t.nrows : cbeg + kHalfN;  // this half's real columns
            // kCh columns of the first (and second) accumulator from column c0, one wait
            auto load_cols = [&](int c0, float (&g)[kCh], float (&u)[kCh]) {
                uint32_t ga[kCh], ua[kCh];
                if constexpr (kCh == 32) {
                    tmem_ld32_nowait(tacc + c0, ga);
                    if (kTwo) tmem_ld32_nowait(tacc + kMaxN + c0, ua);
                } else {
                    tmem_ld16_nowait(tacc + c0, ga);
                    if (kTwo) tmem_ld16_nowait(tacc + kMaxN + c0, ua);
                }
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < kCh; ++i) {
                    g[i] = __uint_as_float(ga[i]);
                    u[i] = kTwo ? __uint_as_float(ua[i]) : 0.f;
                }
            };
            auto release = [&]() {
                tc_fence_before();
                if (kPair && rank != 0) mbar_arrive_cluster(map_to_rank(smem_u32(&tempty[b]), 0));
                else mbar_arrive(&tempty[b]);
            };
            // g: first accumulator, u: second (up projection, or features f + 128)
            const int nrows = t.nrows;
            const long long out_ld = p.out_ld;
            // (callers skip blocks that start past the last real column; whole
            // blocks store without per-element predicates, which measured
            // markedly faster than predicating every store)
            auto emit = [orow, nrows, out_ld, v0, v1](int c0, float (&g)[16], float (&u)[16]) {
                const int n = nrows - c0 < 16 ? nrows - c0 : 16;
                if (n == 16) {
                    if (v0) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) store_out<OutT>(orow + (c0 + i) * out_ld, g[i]);
                    }
                    if (kEpi == kEpiWide && v1) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) store_out<OutT>(orow + 128 + (c0 + i) * out_ld, u[i]);
                    }
                } else {
                    if (v0) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (i < n) store_out<OutT>(orow + (c0 + i) * out_ld, g[i]);
                    }
                    if (kEpi == kEpiWide && v1) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (i < n) store_out<OutT>(orow + 128 + (c0 + i) * out_ld, u[i]);
                    }
                }
            };
            if (!it.split && kEarly) {
                // whole half into registers (SwiGLU applied, packed), accumulator freed, then stores
                uint32_t res[kRegs];
#pragma unroll
                for (int j = 0; j < kHalfN / kCh; ++j) {
                    const int c0 = cbeg + j * kCh;
                    if (c0 < cend) {
                        float g[kCh], u[kCh];
                        load_cols(c0, g, u);
#pragma unroll
                        for (int i = 0; i < kCh; ++i)
                            if (kSwiGLU) g[i] = silu_mul(g[i], u[i]);
                        if constexpr (kBf16Out) {
#pragma unroll
                            for (int i = 0; i < kCh; i += 2) {
                                __nv_bfloat162 h2 = __floats2bfloat162_rn(g[i], g[i + 1]);
                                res[(j * kCh + i) / 2] = *reinterpret_cast<uint32_t*>(&h2);
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < kCh; ++i) res[j * kCh + i] = __float_as_uint(g[i]);
                        }
                    }
                }
                release();
                // column i of this warp's share from the packed registers
                auto store_res = [&](int i) {
                    OutT* dst = orow + (long long)(cbeg + i) * out_ld;
                    if constexpr (kBf16Out) {
                        const uint32_t w2 = res[i / 2];
                        *reinterpret_cast<uint16_t*>(dst) = (i & 1) ? (uint16_t)(w2 >> 16) : (uint16_t)(w2 & 0xffffu);
                    } else {
                        *reinterpret_cast<float*>(dst) = __uint_as_float(res[i]);
                    }
                };
                if (v0) {
#pragma unroll
                    for (int j = 0; j < kHalfN / 16; ++j) {
                        const int c0 = cbeg + 16 * j;
                        if (c0 + 16 <= cend) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) store_res(16 * j + i);
                        } else if (c0 < cend) {
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                if (c0 + i < cend) store_res(16 * j + i);
                        }
                    }
                }
            } else if (!it.split) {
                // kCh columns of both accumulators per TMEM round trip, stored 16 at a time
                for (int c0 = cbeg; c0 < cend; c0 += kCh) {
                    uint32_t ga[kCh], ua[kCh];
                    if constexpr (kCh == 32) {
                        tmem_ld32_nowait(tacc + c0, ga);
                        if (kTwo) tmem_ld32_nowait(tacc + kMaxN + c0, ua);
                    } else {
                        tmem_ld16_nowait(tacc + c0, ga);
                        if (kTwo) tmem_ld16_nowait(tacc + kMaxN + c0, ua);
                    }
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < kCh / 16; ++h) {
                        float g[16], u[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            g[i] = __uint_as_float(ga[16 * h + i]);
                            u[i] = kTwo ? __uint_as_float(ua[16 * h + i]) : 0.f;
                            if (kSwiGLU) g[i] = silu_mul(g[i], u[i]);
                        }
                        if (c0 + 16 * h < cend) emit(c0 + 16 * h, g, u);
                    }
                }
                release();
            } else {
                // stream-K: publish this block's partial tile (rows of real
                // output features and columns of real tokens only)
                const long long slot_floats = 128LL * C::kAccCols;
                float4* mine = reinterpret_cast<float4*>(p.partials + ((long long)blockIdx.x * 2 + it.slot) * slot_floats);
                const long long counter = it.sk_tile * kCta + rank;  // one counter per tile half
                for (int c0 = cbeg; c0 < cend; c0 += kCh) {
                    float g[kCh], u[kCh];
                    load_cols(c0, g, u);
                    if (v0) {
#pragma unroll
                        for (int q = 0; q < kCh / 4; ++q)
                            mine[slot_f4((c0 >> 2) + q, r)] =
                                make_float4(g[4 * q], g[4 * q + 1], g[4 * q + 2], g[4 * q + 3]);
                    }
                    if (kTwo && v1) {
#pragma unroll
                        for (int q = 0; q < kCh / 4; ++q)
                            mine[slot_f4(((kMaxN + c0) >> 2) + q, r)] =
                                make_float4(u[4 * q], u[4 * q + 1], u[4 * q + 2], u[4 * q + 3]);
                    }
                }
                named_sync(1, kEpiThreads);
                if (e == 0) *bcast = atomic_add_acq_rel_gpu(&p.counters[counter], 1);
                named_sync(1, kEpiThreads);
                const int arrived = *bcast;
                // contributors: blocks whose stream-K range meets this tile, or
                // (aligned slices) the S slices' units
                const bool aligned = sch.S > 0;
                const long long q0 = it.sk_tile * sch.KI;
                const int c_first = aligned ? 0 : sch.owner(q0);
                const int c_last = aligned ? sch.S - 1 : sch.owner(q0 + sch.KI - 1);
                int ncontrib = 0;
                if (aligned) {
                    ncontrib = sch.S;
                } else {
                    for (int c = c_first; c <= c_last; ++c)
                        if (sch.beg(c) < sch.beg(c + 1)) ++ncontrib;
                }
                if (arrived == ncontrib - 1) {
                    // last to arrive: sum every contribution in block order, then the epilogue
                    for (int c0 = cbeg; c0 < cend; c0 += 16) {
                        float g[16], u[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) g[i] = u[i] = 0.f;
                        for (int i = c_first; i <= c_last; ++i) {
                            // contributor i: a block (contiguous) or a slice (aligned), in k order
                            int c, slot;
                            if (aligned) {
                                const long long q = it.sk_tile + (long long)i * sch.sk_tiles;
                                c = (int)(q % sch.G);
                                slot = (int)(q / sch.G);
                            } else {
                                c = i;
                                const long long bc = sch.beg(c);
                                if (bc >= sch.beg(c + 1)) continue;
                                slot = (bc / sch.KI == it.sk_tile) ? 0 : 1;
                            }
                            if (c == sch.cta && slot == it.slot) {
                                uint32_t va[16], vb[16];
                                tmem_ld16_nowait(tacc + c0, va);
                                if (kTwo) tmem_ld16_nowait(tacc + kMaxN + c0, vb);
                                tmem_wait_ld();
#pragma unroll
                                for (int i = 0; i < 16; ++i) {
                                    g[i] += __uint_as_float(va[i]);
                                    if (kTwo) u[i] += __uint_as_float(vb[i]);
                                }
                            } else {
                                const float4* other =
                                    reinterpret_cast<const float4*>(p.partials + (((long long)c * kCta + rank) * 2 + slot) *
                                                                                     slot_floats);
                                const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
                                float4 a4[4], b4[4];
#pragma unroll
                                for (int q = 0; q < 4; ++q) a4[q] = v0 ? __ldcg(other + slot_f4((c0 >> 2) + q, r)) : z;
                                if (kTwo) {
#pragma unroll
                                    for (int q = 0; q < 4; ++q)
                                        b4[q] = v1 ? __ldcg(other + slot_f4(((kMaxN + c0) >> 2) + q, r)) : z;
                                }
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    g[4 * q] += a4[q].x;
                                    g[4 * q + 1] += a4[q].y;
                                    g[4 * q + 2] += a4[q].z;
                                    g[4 * q + 3] += a4[q].w;
                                }
                                if (kTwo) {
#pragma unroll
                                    for (int q = 0; q < 4; ++q) {
                                        u[4 * q] += b4[q].x;
                                        u[4 * q + 1] += b4[q].y;
                                        u[4 * q + 2] += b4[q].z;
                                        u[4 * q + 3] += b4[q].w;
                                    }
                                }
                            }
                        }
                        if (kSwiGLU) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) g[i] = silu_mul(g[i], u[i]);
                        }
                        emit(c0, g, u);
                    }
                    if (e == 0) p.counters[counter] = 0;  // leave the counter zero for the next launch
                }
                release();
            }
            ++ac;
        }
    }

    tc_fence_before();
    if (kPair) cluster_sync_all();  // neither CTA frees TMEM or leaves while the pair's MMAs may run
    else __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        if (kPair) tmem_dealloc_pair(tmem_base, 512);
        else tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace moe
