// moe_kernels.cu -- the non-GEMM stages of the MoE block ("top-K selection",
// "alignment" and the "local sum" of the talk notes' "Key findings 5", plus
// the permute that feeds the grouped GEMM).  All bandwidth-light: one warp
// per token for top-K, one block for the alignment, 16-byte vector copies for
// permute and combine.
#include <climits>
#include <type_traits>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {
int launched(cudaError_t e) {
    if (e != cudaSuccess) {
        cudaGetLastError();
        return -3;
    }
    return 0;
}
}  // namespace

// ------------------------------------------------------------------ top-K
// Order: larger logit first, lower expert index on equal logits.
__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
    return v > bv || (v == bv && i < bi);
}

// Order-preserving 32-bit key of a logit: a larger value has a larger key,
// -0 and +0 share one key, and every NaN takes key 0, below every number, so
// a NaN logit is picked only once nothing else is left.
__device__ __forceinline__ uint32_t logit_key(float v) {
    uint32_t u = __float_as_uint(v);
    if (u == 0x80000000u) u = 0u;
    const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return v != v ? 0u : k;
}

// One warp per token.  Lane l owns experts l, l+32, ... (at most kPL of them,
// E <= 32 kPL), read through L2 (they may have been written by other blocks
// of the same kernel): once into registers, or (kStream, for the largest E in
// kernels with few registers per thread) again on every scan.  kt rounds
// (kt = K, or the token's own count 0..K under per-token dynamic K; slots
// kt..K-1 get id -1 and weight 0) each take the largest remaining logit, the
// lower expert index on equal logits: every lane keeps its own best expert not
// yet taken; a warp max of the lanes' keys, then a warp min of the expert
// index over the lanes holding that key, name the winner, whose lane alone
// rescans.  Lane k keeps the k-th pick and computes its weight.
template <int kPL, bool kStream = false>
__device__ __forceinline__ void topk_one_token_r(const float* __restrict__ l, int E, int K, int kt, int score_fn,
                                                 int renorm, int32_t* __restrict__ ids_t, float* __restrict__ w_t,
                                                 int lane) {
    float lv[kStream ? 1 : kPL];
    if constexpr (!kStream) {
#pragma unroll
        for (int j = 0; j < kPL; ++j) {
            const int e = lane + 32 * j;
            lv[j] = e < E ? __ldcg(l + e) : 0.f;
        }
    }
    auto val = [&](int j) -> float {
        if constexpr (kStream)
            return __ldcg(l + lane + 32 * j);
        else
            return lv[j];
    };
    // the register variant unrolls fully; the streaming one four loads at a time
    constexpr int kU = kStream ? 4 : kPL;
    uint32_t taken = 0;  // bit j: expert lane + 32 j
    // this lane's best expert not yet taken: key, index (INT_MAX: none), logit
    uint32_t bk = 0;
    int be = INT_MAX;
    float bv = 0.f;
    auto rescan = [&]() {
        bk = 0;
        be = INT_MAX;
        bv = 0.f;
#pragma unroll kU
        for (int j = 0; j < kPL; ++j) {
            const int e = lane + 32 * j;
            if (e < E && !((taken >> j) & 1u)) {
                const float v = val(j);
                const uint32_t k = logit_key(v);
                if (be == INT_MAX || k > bk) {  // ascending j: the lower index keeps a tie
                    bk = k;
                    be = e;
                    bv = v;
                }
            }
        }
    };
    rescan();
    float my_v = 0.f;  // lane k < kt: the k-th pick's logit and expert
    int my_i = -1;
#pragma unroll 1
    for (int k = 0; k < kt; ++k) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
        // lanes without a candidate hold INT_MAX; kt <= E leaves a real one
        const int win = __reduce_min_sync(0xffffffffu, bk == m ? be : INT_MAX);
        const float wv = __shfl_sync(0xffffffffu, bv, win & 31);
        if (lane == k) {
            my_v = wv;
            my_i = win;
        }
        if ((win & 31) == lane) {
            taken |= 1u << (win >> 5);
            rescan();
        }
    }
    // gate weights: lane k < kt computes its own
    const bool mine = lane < kt;
    float wk = 0.f;
    if (score_fn == 0) {
        float m, den;
        if (renorm) {
            // the first pick is the largest selected logit (all NaN if it is)
            m = __shfl_sync(0xffffffffu, my_v, 0);
            float e = mine ? expf(my_v - m) : 0.f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
            den = e;
        } else {
            m = -INFINITY;
#pragma unroll kU
            for (int j = 0; j < kPL; ++j)
                if (lane + 32 * j < E) m = fmaxf(m, val(j));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            float part = 0.f;
#pragma unroll kU
            for (int j = 0; j < kPL; ++j)
                if (lane + 32 * j < E) part += expf(val(j) - m);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            den = part;
        }
        if (mine) wk = expf(my_v - m) / den;
    } else {
        const float sg = mine ? 1.f / (1.f + expf(-my_v)) : 0.f;
        float den = sg;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
        wk = renorm ? (mine ? sg / den : 0.f) : sg;
    }
    if (lane < K) {
        ids_t[lane] = mine ? my_i : -1;
        w_t[lane] = wk;
    }
}

// The same for any E <= 1024: the register count sized by E (E > 512 reloads).
__device__ __forceinline__ void topk_one_token(const float* __restrict__ l, int E, int K, int kt, int score_fn,
                                               int renorm, int32_t* __restrict__ ids_t, float* __restrict__ w_t,
                                               int lane) {
    if (E <= 32)
        topk_one_token_r<1>(l, E, K, kt, score_fn, renorm, ids_t, w_t, lane);
    else if (E <= 64)
        topk_one_token_r<2>(l, E, K, kt, score_fn, renorm, ids_t, w_t, lane);
    else if (E <= 128)
        topk_one_token_r<4>(l, E, K, kt, score_fn, renorm, ids_t, w_t, lane);
    else if (E <= 256)
        topk_one_token_r<8>(l, E, K, kt, score_fn, renorm, ids_t, w_t, lane);
    else if (E <= 512)
        topk_one_token_r<16>(l, E, K, kt, score_fn, renorm, ids_t, w_t, lane);
    else
        topk_one_token_r<32, true>(l, E, K, kt, score_fn, renorm, ids_t, w_t, lane);
}

// The token's expert count: K, or k_per_token[t] clamped to [0, K].
__device__ __forceinline__ int token_k(const int32_t* __restrict__ k_per_token, int t, int K) {
    if (!k_per_token) return K;
    const int k = __ldg(k_per_token + t);
    return k < 0 ? 0 : (k > K ? K : k);
}

__global__ void __launch_bounds__(256) topk_gate_kernel(int T, int E, int K, int score_fn, int renorm,
                                                        const float* __restrict__ logits,
                                                        const int32_t* __restrict__ k_per_token,
                                                        int32_t* __restrict__ ids, float* __restrict__ w) {
    pdl_launch_dependents();
    pdl_wait();
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (t >= T) return;
    topk_one_token(logits + (size_t)t * E, E, K, token_k(k_per_token, t, K), score_fn, renorm, ids + (size_t)t * K,
                   w + (size_t)t * K, lane);
}

int launch_topk(int T, int E, int K, int score_fn, int renorm, const float* logits, const int32_t* k_per_token,
                int32_t* ids, float* w, cudaStream_t stream) {
    if (T == 0) return 0;
    const int warps_per_block = 8;
    const int blocks = (T + warps_per_block - 1) / warps_per_block;
    cudaError_t e = launch_kernel(topk_gate_kernel, dim3(blocks), dim3(warps_per_block * 32), 0, stream, T, E, K,
                                  score_fn, renorm, logits, k_per_token, ids, w);
    count_launch();
    return launched(e);
}

// -------------------------------------------------------------- alignment
// One block of 1024 threads.  (1) the counts N_e (with the ranks of the fast
// path below, or a shared-memory histogram); (2) block scan of the padded
// counts ceil(N_e/B)*B into offsets; (3) stable scatter: every assignment's
// slot keeps ascending a within its expert; (4) -1 in the padding slots,
// block_expert per B-row block.
constexpr int kAlignThreads = 1024;

__device__ __forceinline__ int block_excl_scan(int v, int* warp_tot, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int s = warp_tot[lane];
        int si = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, si, o);
            if (lane >= o) si += x;
        }
        warp_tot[lane] = si - s;  // exclusive prefix of warp totals
        if (lane == 31) warp_tot[32] = si;
    }
    __syncthreads();
    const int r = warp_tot[warp] + incl - v;
    total = warp_tot[32];
    __syncthreads();
    return r;
}

// The alignment of T*K assignments by one block of kAlignThreads threads;
// `sm` is dynamic shared memory of align_smem_bytes(E) bytes.
//
// Fast path (A <= kAlignFastItems * kAlignThreads, E <= kAlignFastMaxE): warp
// w owns the contiguous assignments [w C, (w + 1) C), C = 32 R, each lane R of
// them held in registers (all loaded up front).  Walking its chunk in order,
// the warp ranks each assignment among equal ids with __match_any_sync on top
// of a per-warp running count per expert (a [32][E] table); one scan over the
// 32 warps per expert then gives every warp's base inside each segment, and
// the totals are the counts N_e.  Chunks are in assignment order, so the ranks
// keep ascending a within each expert (stable).  Otherwise the rounds of the
// general path below.
constexpr int kAlignFastItems = 16;   // assignments per lane on the fast path
constexpr int kAlignFastMaxE = 512;   // [32][E] int table within the shared-memory budget

// The same alignment for at most 32 x kAlignTinyItems assignments, by warp 0
// alone (no block barrier; the other warps have nothing to do): lane l holds
// assignments l, l + 32, ...; ranks inside an expert follow the assignment
// index, as in align_block.
constexpr int kAlignTinyItems = 4;
__device__ __forceinline__ void align_warp(int A, int E, int B, int mode, long long P_max, const int32_t* ids,
                                           int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                           int32_t* __restrict__ sorted_ids, int32_t* __restrict__ block_expert,
                                           int32_t* __restrict__ pos, int32_t* __restrict__ scalars,
                                           int32_t* __restrict__ stats_copy, int* sm, int lane) {
    int* run = sm;           // E: assignments per expert so far
    int* off = run + E;      // E + 1: padded segment starts
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int e = lane; e < E; e += 32) run[e] = 0;
    __syncwarp();
    int bad = 0;
    int ie[kAlignTinyItems], ir[kAlignTinyItems];
#pragma unroll
    for (int i = 0; i < kAlignTinyItems; ++i) {
        const int a = lane + 32 * i;
        // ids may come from other blocks (or warps) of the same kernel: read through L2
        int e = a < A ? __ldcg(ids + a) : -1;
        if ((unsigned)e >= (unsigned)E) {
            if (e != -1) bad = 1;  // -1: an empty slot (per-token dynamic K)
            e = -1;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int r = (e >= 0 ? run[e] : 0) + __popc(peers & lt_mask);
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) run[e] += __popc(peers);
        __syncwarp();
        ie[i] = e;
        ir[i] = r;
    }
    bad = __any_sync(0xffffffffu, bad) ? 1 : 0;
    // padded sizes (block-wise, or every expert at the most loaded one's) and
    // their exclusive scan, 32 experts at a time
    long long rows = 0;
    bool overflow = false;
    if (mode == 1) {
        int m = 0;
        for (int e = lane; e < E; e += 32) m = max(m, run[e]);
        m = __reduce_max_sync(0xffffffffu, m);
        rows = ((long long)m + B - 1) / B * B;
        overflow = (long long)E * rows > P_max;
        if (overflow) bad |= 2;
    }
    int carry = 0, n_active = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        const int n = e < E ? run[e] : 0;
        int v = e < E ? (mode == 1 ? (overflow ? 0 : (int)rows) : (n + B - 1) / B * B) : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        if (e < E) {
            off[e] = carry + incl - v;
            counts[e] = n;
            offsets[e] = carry + incl - v;
        }
        n_active += __popc(__ballot_sync(0xffffffffu, e < E && n > 0));
        carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    const int P = carry;
    if (overflow) n_active = 0;
    if (lane == 0) {
        off[E] = P;
        offsets[E] = P;
        scalars[0] = P;
        scalars[1] = n_active;
        scalars[2] = bad;
        scalars[3] = 0;
        if (stats_copy) {
            stats_copy[0] = P;
            stats_copy[1] = n_active;
            stats_copy[2] = bad;
            stats_copy[3] = 0;
        }
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < kAlignTinyItems; ++i) {
        const int a = lane + 32 * i;
        if (ie[i] >= 0 && !overflow) {
            const int p = off[ie[i]] + ir[i];
            sorted_ids[p] = (int32_t)a;
            pos[a] = p;
        } else if (a < A) {
            pos[a] = -1;  // empty slot (or an out-of-range id, flagged above)
        }
    }
    // padding slots inside each segment, then everything past P
    if (!overflow)
        for (int e = lane; e < E; e += 32)
            for (int p = off[e] + run[e]; p < off[e + 1]; ++p) sorted_ids[p] = -1;
    for (long long p = (long long)P + lane; p < P_max; p += 32) sorted_ids[p] = -1;
    const long long nblk = (P_max + B - 1) / B;
    for (long long b = lane; b < nblk; b += 32) {
        const long long p = b * B;
        int r = -1;
        if (p < P) {
            int lo = 0, hi = E - 1;  // largest e with off[e] <= p
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (off[mid] <= p) lo = mid;
                else hi = mid - 1;
            }
            r = lo;
        }
        block_expert[b] = r;
    }
}

__device__ __forceinline__ void align_block(int T, int K, int E, int B, int mode, long long P_max, const int32_t* ids,
                                            int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                            int32_t* __restrict__ sorted_ids, int32_t* __restrict__ block_expert,
                                            int32_t* __restrict__ pos, int32_t* __restrict__ scalars,
                                            int32_t* __restrict__ stats_copy, int* sm) {
    int* cnt = sm;                 // E
    int* off = cnt + E;            // E + 1
    int* cursor = off + E + 1;     // E
    int* rt = cursor + E;          // E
    int* warp_tot = rt + E;        // 33
    int* bad = warp_tot + 33;      // 1
    int* nmax = bad + 1;           // 1
    uint16_t* tbl = reinterpret_cast<uint16_t*>(nmax + 1);  // general path: 32 x E per round
    int* wt = nmax + 1;                                       // fast path: 32 x E running counts
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long A = (long long)T * K;
    if (A <= 32LL * kAlignTinyItems) {  // a handful of assignments: one warp, no block barrier
        if (warp == 0)
            align_warp((int)A, E, B, mode, P_max, ids, counts, offsets, sorted_ids, block_expert, pos, scalars,
                       stats_copy, sm, lane);
        return;
    }
    const unsigned lt_mask = (1u << lane) - 1u;
    const bool fast = A <= (long long)kAlignFastItems * kAlignThreads && E <= kAlignFastMaxE;
    // fast path: item i of this lane is assignment a0 + 32 i; packed as
    // (rank << 11) | (expert + 1), 0 in the low bits for no expert
    const int R = fast ? (int)((A + kAlignThreads - 1) / kAlignThreads) : 0;
    const long long a0 = (long long)warp * 32 * R + lane;
    uint32_t item[kAlignFastItems];

    if (fast) {
        for (int i = tid; i < 32 * E; i += kAlignThreads) wt[i] = 0;
        if (tid == 0) *bad = 0, *nmax = 0;
        // ids may come from other blocks of the same kernel: read through L2
#pragma unroll
        for (int i = 0; i < kAlignFastItems; ++i) {
            const long long a = a0 + 32LL * i;
            item[i] = (i < R && a < A) ? (uint32_t)__ldcg(ids + a) : 0xFFFFFFFFu;
        }
        __syncthreads();
        int* row = wt + warp * E;
        int badl = 0;
#pragma unroll
        for (int i = 0; i < kAlignFastItems; ++i) {
            if (i < R) {  // the same R in every lane
                int e = (int)item[i];
                if ((unsigned)e >= (unsigned)E) {
                    if (e != -1) badl = 1;  // -1: an empty slot (per-token dynamic K) or past A
                    e = -1;
                }
                const unsigned peers = __match_any_sync(0xffffffffu, e);
                const int run = e >= 0 ? row[e] : 0;
                const int rank = run + __popc(peers & lt_mask);
                __syncwarp();
                if (e >= 0 && lane == __ffs(peers) - 1) row[e] = run + __popc(peers);
                __syncwarp();
                item[i] = ((uint32_t)rank << 11) | (uint32_t)(e + 1);
            }
        }
        if (badl) atomicOr(bad, 1);
        __syncthreads();
        // per expert: exclusive scan of the warps' counts in warp order; the total is N_e
        for (int e = tid; e < E; e += kAlignThreads) {
            int run = 0;
            for (int w = 0; w < 32; ++w) {
                const int c = wt[w * E + e];
                wt[w * E + e] = run;
                run += c;
            }
            cnt[e] = run;
        }
        __syncthreads();
    } else {
        for (int e = tid; e < E; e += kAlignThreads) cnt[e] = 0;
        if (tid == 0) *bad = 0, *nmax = 0;
        __syncthreads();
        for (long long a = tid; a < A; a += kAlignThreads) {
            const int e = __ldcg(ids + a);
            if ((unsigned)e < (unsigned)E) atomicAdd(&cnt[e], 1);
            else if (e != -1) atomicOr(bad, 1);  // -1: an empty slot (per-token dynamic K)
        }
        __syncthreads();
    }

    // padded counts -> offsets (E <= 1024: one expert per thread).  Block-wise
    // padding rounds each count up to B; max-value padding gives every expert
    // the rounded size of the most loaded one.
    const int n = tid < E ? cnt[tid] : 0;
    int padded = ((n + B - 1) / B) * B;
    // Block-wise padding stays within P_max for any ids (at most min(E, A)
    // experts each add fewer than B rows).  Max-value padding assumes an
    // expert holds at most one assignment per token; ids that repeat within a
    // token can push E * ceil(max N / B) * B past P_max.  Such a routing is
    // flagged (bit 2 of the bad-input word) and aligned as empty: no rows, no
    // write at or past P_max.
    bool overflow = false;
    if (mode == 1) {
        const int wmax = __reduce_max_sync(0xffffffffu, n);
        if (lane == 0 && wmax > 0) atomicMax(nmax, wmax);
        __syncthreads();
        const long long rows = ((long long)*nmax + B - 1) / B * B;
        overflow = (long long)E * rows > P_max;
        padded = tid < E && !overflow ? (int)rows : 0;
        if (overflow && tid == 0) *bad |= 2;
    }
    int P = 0;
    const int excl = block_excl_scan(padded, warp_tot, P);
    const int n_active = overflow ? 0 : __syncthreads_count(tid < E && n > 0);
    if (tid < E) {
        off[tid] = excl;
        cursor[tid] = excl;
        counts[tid] = n;
        offsets[tid] = excl;
    }
    if (tid == 0) {
        off[E] = P;
        offsets[E] = P;
        scalars[0] = P;
        scalars[1] = n_active;
        scalars[2] = *bad;
        scalars[3] = 0;
        if (stats_copy) {
            stats_copy[0] = P;
            stats_copy[1] = n_active;
            stats_copy[2] = *bad;
            stats_copy[3] = 0;
        }
    }
    __syncthreads();

    if (fast) {
        // slot = segment start + this warp's base in the segment + rank in the warp
#pragma unroll
        for (int i = 0; i < kAlignFastItems; ++i) {
            if (i < R) {
                const long long a = a0 + 32LL * i;
                const int e = (int)(item[i] & 0x7FFu) - 1;
                if (e >= 0 && !overflow) {
                    const int p = off[e] + wt[warp * E + e] + (int)(item[i] >> 11);
                    sorted_ids[p] = (int32_t)a;
                    pos[a] = p;
                } else if (a < A) {
                    pos[a] = -1;  // empty slot (or an out-of-range id, flagged above)
                }
            }
        }
    } else {
        // stable scatter in rounds of kAlignThreads assignments: the rank among
        // equal ids inside a warp from __match_any_sync, across the warps of a
        // round from a per-(warp, expert) count table scanned over the warps,
        // across rounds from a per-expert cursor
        for (long long base = 0; base < A; base += kAlignThreads) {
            const long long a = base + tid;
            int e = a < A && !overflow ? __ldcg(ids + a) : -1;
            if ((unsigned)e >= (unsigned)E) e = -1;
            for (int i = tid; i < 32 * E; i += kAlignThreads) tbl[i] = 0;
            __syncthreads();
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            const int rank = __popc(peers & lt_mask);
            if (e >= 0 && lane == __ffs(peers) - 1) tbl[warp * E + e] = (uint16_t)__popc(peers);
            __syncthreads();
            if (tid < E) {
                int run = 0;
                for (int w = 0; w < 32; ++w) {
                    const int c = tbl[w * E + tid];
                    tbl[w * E + tid] = (uint16_t)run;
                    run += c;
                }
                rt[tid] = run;
            }
            __syncthreads();
            if (e >= 0) {
                const int p = cursor[e] + tbl[warp * E + e] + rank;
                sorted_ids[p] = (int32_t)a;
                pos[a] = p;
            } else if (a < A) {
                pos[a] = -1;  // empty slot (or an out-of-range id, flagged above)
            }
            __syncthreads();
            if (tid < E) cursor[tid] += rt[tid];
            __syncthreads();
        }
    }

    // padding slots inside each segment, then everything past P
    if (!overflow)
        for (int e = warp; e < E; e += kAlignThreads / 32)
            for (int p = off[e] + cnt[e] + lane; p < off[e + 1]; p += 32) sorted_ids[p] = -1;
    for (long long p = (long long)P + tid; p < P_max; p += kAlignThreads) sorted_ids[p] = -1;
    const long long nblk = (P_max + B - 1) / B;
    for (long long b = tid; b < nblk; b += kAlignThreads) {
        const long long p = b * B;
        int r = -1;
        if (p < P) {
            int lo = 0, hi = E - 1;  // largest e with off[e] <= p
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (off[mid] <= p) lo = mid;
                else hi = mid - 1;
            }
            r = lo;
        }
        block_expert[b] = r;
    }
}

__global__ void __launch_bounds__(kAlignThreads, 1)
    align_kernel(int T, int K, int E, int B, int mode, long long P_max, const int32_t* __restrict__ ids,
                 int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ sorted_ids,
                 int32_t* __restrict__ block_expert, int32_t* __restrict__ pos, int32_t* __restrict__ scalars,
                 int32_t* __restrict__ stats_copy) {
    extern __shared__ int sm[];
    pdl_launch_dependents();
    pdl_wait();
    align_block(T, K, E, B, mode, P_max, ids, counts, offsets, sorted_ids, block_expert, pos, scalars, stats_copy,
                sm);
}

// cnt, off, cursor, rt, the scan words and flags, then the [32][E] table (int
// counts on the fast path when E allows it, uint16 per round otherwise)
size_t align_smem_bytes(int E) {
    const size_t table = E <= kAlignFastMaxE ? sizeof(int) * 32 * (size_t)E : sizeof(uint16_t) * 32 * (size_t)E;
    return sizeof(int) * (4 * (size_t)E + 1 + 35) + table;
}

// ----------------------------------------------------- small-batch routing
// Router logits, top-K gating and alignment in one launch for small T.
// Stage 1 (every block): partial dot products of the router GEMV on the CUDA
// cores -- one warp per (expert, group of 8 tokens, slice of the hidden
// dimension), fp32 sums of the exact products -- written to `part`.
// Stage 2 (the last block to finish, found with a counter; no block waits):
// logits[t][e] = sum over slices in slice order (deterministic), then top-K
// for every token and the alignment.  `logits_override` (nullable) replaces
// the computed logits in the routing decision.
constexpr int kRouteTokGroup = 8;

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* f) {
    const int4 v = __ldg(reinterpret_cast<const int4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}
__device__ __forceinline__ void load8(const float* p, float* f) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p + 4));
    f[0] = a.x, f[1] = a.y, f[2] = a.z, f[3] = a.w, f[4] = b.x, f[5] = b.y, f[6] = b.z, f[7] = b.w;
}

template <typename T>
__global__ void __launch_bounds__(kAlignThreads, 1)
    route_small_kernel(int T_, int H, int E, int K, int score_fn, int renorm, int B, int mode, long long P_max,
                       int nslices,
                       int slice_w, const T* __restrict__ x, const T* __restrict__ w_r,
                       const float* __restrict__ logits_override, const int32_t* __restrict__ k_per_token,
                       float* __restrict__ part, float* __restrict__ logits,
                       int32_t* __restrict__ ids, float* __restrict__ w, int32_t* __restrict__ counts,
                       int32_t* __restrict__ offsets, int32_t* __restrict__ sorted_ids,
                       int32_t* __restrict__ block_expert, int32_t* __restrict__ pos, int32_t* __restrict__ scalars,
                       int32_t* __restrict__ stats_copy, int* __restrict__ done_ctr) {
    extern __shared__ int sm[];
    __shared__ int is_last;
    pdl_launch_dependents();
    pdl_wait();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ngroups = (T_ + kRouteTokGroup - 1) / kRouteTokGroup;
    const long long units = (long long)E * ngroups * nslices;
    const long long u = (long long)blockIdx.x * (kAlignThreads / 32) + warp;
    if (u < units) {
        const int e = (int)(u % E);
        const int tg = (int)((u / E) % ngroups);
        const int sl = (int)(u / ((long long)E * ngroups));
        const int t0 = tg * kRouteTokGroup;
        const int nt = T_ - t0 < kRouteTokGroup ? T_ - t0 : kRouteTokGroup;
        const int h0 = sl * slice_w;
        const int h1 = h0 + slice_w < H ? h0 + slice_w : H;
        float acc[kRouteTokGroup];
#pragma unroll
        for (int i = 0; i < kRouteTokGroup; ++i) acc[i] = 0.f;
        const T* wrow = w_r + (size_t)e * H;
        for (int h = h0 + lane * 8; h < h1; h += 256) {
            float wv[8];
            load8(wrow + h, wv);
#pragma unroll
            for (int i = 0; i < kRouteTokGroup; ++i) {
                if (i < nt) {
                    float xv[8];
                    load8(x + (size_t)(t0 + i) * H + h, xv);
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[i] = fmaf(wv[j], xv[j], acc[i]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kRouteTokGroup; ++i) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
        }
        if (lane == 0)
            for (int i = 0; i < nt; ++i) part[((size_t)sl * T_ + t0 + i) * E + e] = acc[i];
    }
    __syncthreads();
    if (threadIdx.x == 0) is_last = atomic_add_acq_rel_gpu(done_ctr, 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (!is_last) return;
    for (long long i = threadIdx.x; i < (long long)T_ * E; i += kAlignThreads) {
        float v = 0.f;
        for (int sl = 0; sl < nslices; ++sl) v += __ldcg(part + (size_t)sl * T_ * E + i);
        logits[i] = v;
    }
    __syncthreads();
    const float* src = logits_override ? logits_override : logits;
    for (int t = warp; t < T_; t += kAlignThreads / 32)
        topk_one_token(src + (size_t)t * E, E, K, token_k(k_per_token, t, K), score_fn, renorm, ids + (size_t)t * K,
                       w + (size_t)t * K, lane);
    __syncthreads();
    align_block(T_, K, E, B, mode, P_max, ids, counts, offsets, sorted_ids, block_expert, pos, scalars, stats_copy,
                sm);
    if (threadIdx.x == 0) *done_ctr = 0;  // ready for the next launch
}

// ------------------------------------------------ router on the CUDA cores
// logits[t][e] = sum over h of x[t][h] * w_r[e][h] in fp32, for layers whose
// router matrix fits shared memory (E <= 16, E * H * elt <= kRouterCcMaxBytes;
// the Mixtral-shaped layer's is 64 KB).  Every block keeps w_r in shared
// memory and each warp takes whole tokens: lane l reads 16-byte chunks l,
// l + 32, ... of the token row (each row is read once, coalesced), multiplies
// them with the E weight chunks at the same position (consecutive lanes,
// consecutive chunks: no bank conflict) and the E per-lane sums go through a
// shuffle tree.  The tensor-core GEMM would fill 8 of the 128 rows of each
// MMA here and pay a pipeline ramp and split-K fixups for what is one read of x.
__device__ __forceinline__ void load8_shared(const __nv_bfloat16* p, float* f) {
    const int4 v = *reinterpret_cast<const int4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}
__device__ __forceinline__ void load8_shared(const float* p, float* f) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    f[0] = a.x, f[1] = a.y, f[2] = a.z, f[3] = a.w, f[4] = b.x, f[5] = b.y, f[6] = b.z, f[7] = b.w;
}

template <typename T, int kE>
__global__ void __launch_bounds__(256) router_cc_kernel(int T_, int H, const T* __restrict__ x,
                                                        const T* __restrict__ w_r, float* __restrict__ logits) {
    extern __shared__ int4 router_sm[];
    const T* ws = reinterpret_cast<const T*>(router_sm);
    pdl_launch_dependents();
    // the router weights are not written by the previous kernel: stage them
    // before waiting for it, 8 independent 16-byte loads per thread in flight
    const int n16 = (int)((long long)kE * H * sizeof(T) / 16);
    const int4* wsrc = reinterpret_cast<const int4*>(w_r);
    for (int i0 = threadIdx.x; i0 < n16; i0 += 8 * blockDim.x) {
        int4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (i0 + j * (int)blockDim.x < n16) v[j] = __ldg(wsrc + i0 + j * blockDim.x);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (i0 + j * (int)blockDim.x < n16) router_sm[i0 + j * blockDim.x] = v[j];
    }
    pdl_wait();
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int warps = blockDim.x >> 5;
    for (int t = blockIdx.x * warps + (threadIdx.x >> 5); t < T_; t += gridDim.x * warps) {
        float acc[kE];
#pragma unroll
        for (int e = 0; e < kE; ++e) acc[e] = 0.f;
        const T* xr = x + (size_t)t * H;
        // the token row in groups of 8 chunks per lane, all 8 loads issued before the first use
        for (int h0 = lane * 8; h0 < H; h0 += 8 * 256) {
            float xv[8][8];
#pragma unroll
            for (int c = 0; c < 8; ++c)
                if (h0 + c * 256 < H) load8(xr + h0 + c * 256, xv[c]);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int h = h0 + c * 256;
                if (h < H) {
#pragma unroll
                    for (int e = 0; e < kE; ++e) {
                        float wv[8];
                        load8_shared(ws + (size_t)e * H + h, wv);
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[e] = fmaf(wv[j], xv[c][j], acc[e]);
                    }
                }
            }
        }
#pragma unroll
        for (int e = 0; e < kE; ++e) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
        }
#pragma unroll
        for (int e = 0; e < kE; ++e)
            if (lane == e) logits[(size_t)t * kE + e] = acc[e];
    }
}

// Router logits, top-K gating and alignment in one launch for router
// matrices that fit shared memory (the layer's routing above the small-batch
// size): blocks of 1024 threads stage w_r in shared memory; each warp takes
// whole tokens, computes the E logits as router_cc_kernel does (the same
// products and summation order), stores them, and runs the top-K and gate
// weights of topk_gate_kernel on the stored row (or on logits_override).  The
// last block to finish (a counter; no block waits) runs the alignment over all
// T, reusing its shared memory.
template <typename T, int kE>
__global__ void __launch_bounds__(kAlignThreads, 1)
    route_cc_kernel(int T_, int H, int K, int score_fn, int renorm, int B, int mode, long long P_max,
                    const T* __restrict__ x, const T* __restrict__ w_r, const float* __restrict__ logits_override,
                    const int32_t* __restrict__ k_per_token, float* __restrict__ logits, int32_t* __restrict__ ids,
                    float* __restrict__ w, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                    int32_t* __restrict__ sorted_ids, int32_t* __restrict__ block_expert, int32_t* __restrict__ pos,
                    int32_t* __restrict__ scalars, int32_t* __restrict__ stats_copy, int* __restrict__ done_ctr) {
    extern __shared__ int4 route_sm[];
    __shared__ int is_last;
    const T* ws = reinterpret_cast<const T*>(route_sm);
    pdl_launch_dependents();
    const int n16 = (int)((long long)kE * H * sizeof(T) / 16);
    const int4* wsrc = reinterpret_cast<const int4*>(w_r);
    for (int i0 = threadIdx.x; i0 < n16; i0 += 4 * blockDim.x) {
        int4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (i0 + j * (int)blockDim.x < n16) v[j] = __ldg(wsrc + i0 + j * blockDim.x);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (i0 + j * (int)blockDim.x < n16) route_sm[i0 + j * blockDim.x] = v[j];
    }
    pdl_wait();
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int warps = blockDim.x >> 5;
    // 1024-thread blocks leave 64 registers a thread: the token row's 16-byte
    // words stay packed while in flight (32 registers: 8 chunks of bf16, 4 of
    // fp32) and each chunk is widened when it is used; the products and their
    // order are those of router_cc_kernel
    constexpr int kChunks = sizeof(T) == 2 ? 8 : 4;
    constexpr int kWords = 8 * sizeof(T) / 16;  // 16-byte words per chunk of 8 elements
    for (int t = blockIdx.x * warps + (threadIdx.x >> 5); t < T_; t += gridDim.x * warps) {
        float acc[kE];
#pragma unroll
        for (int e = 0; e < kE; ++e) acc[e] = 0.f;
        const T* xr = x + (size_t)t * H;
        for (int h0 = lane * 8; h0 < H; h0 += kChunks * 256) {
            int4 raw[kChunks * kWords];
#pragma unroll
            for (int c = 0; c < kChunks; ++c)
                if (h0 + c * 256 < H) {
#pragma unroll
                    for (int q = 0; q < kWords; ++q)
                        raw[c * kWords + q] = __ldg(reinterpret_cast<const int4*>(xr + h0 + c * 256) + q);
                }
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                const int h = h0 + c * 256;
                if (h < H) {
                    float xv[8];
                    load8_shared(reinterpret_cast<const T*>(&raw[c * kWords]), xv);
#pragma unroll
                    for (int e = 0; e < kE; ++e) {
                        float wv[8];
                        load8_shared(ws + (size_t)e * H + h, wv);
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[e] = fmaf(wv[j], xv[j], acc[e]);
                    }
                }
            }
        }
#pragma unroll
        for (int e = 0; e < kE; ++e) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
        }
#pragma unroll
        for (int e = 0; e < kE; ++e)
            if (lane == e) logits[(size_t)t * kE + e] = acc[e];
        __syncwarp();  // the row is complete before the warp reads it back
        const float* src = logits_override ? logits_override + (size_t)t * kE : logits + (size_t)t * kE;
        topk_one_token_r<(kE + 31) / 32>(src, kE, K, token_k(k_per_token, t, K), score_fn, renorm,
                                         ids + (size_t)t * K, w + (size_t)t * K, lane);
    }
    __syncthreads();
    if (threadIdx.x == 0) is_last = atomic_add_acq_rel_gpu(done_ctr, 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (!is_last) return;
    align_block(T_, K, kE, B, mode, P_max, ids, counts, offsets, sorted_ids, block_expert, pos, scalars, stats_copy,
                reinterpret_cast<int*>(route_sm));
    if (threadIdx.x == 0) *done_ctr = 0;  // ready for the next launch
}

bool router_cc_fits(int H, int E, int dtype) {
    const long long eb = dtype == 0 ? 2 : 4;
    return E >= 1 && E <= 16 && H > 0 && H % 8 == 0 && (long long)E * H * eb <= kRouterCcMaxBytes;
}

template <typename T, int kE>
cudaError_t launch_router_cc_e(int n_tok, int H, const void* x, const void* w_r, float* logits, int num_sms,
                               cudaStream_t stream) {
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(router_cc_kernel<T, kE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kRouterCcMaxBytes);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    long long blocks = (n_tok + 7) / 8;
    if (blocks > 2LL * num_sms) blocks = 2LL * num_sms;
    const size_t smem = (size_t)kE * H * sizeof(T);
    return launch_kernel(router_cc_kernel<T, kE>, dim3((int)blocks), dim3(256), smem, stream, n_tok, H,
                         static_cast<const T*>(x), static_cast<const T*>(w_r), logits);
}

template <typename T>
cudaError_t launch_router_cc_t(int n_tok, int H, int E, const void* x, const void* w_r, float* logits, int num_sms,
                               cudaStream_t s) {
    switch (E) {
#define MOE_ROUTER_CC_CASE(n) \
    case n: return launch_router_cc_e<T, n>(n_tok, H, x, w_r, logits, num_sms, s);
        MOE_ROUTER_CC_CASE(1) MOE_ROUTER_CC_CASE(2) MOE_ROUTER_CC_CASE(3) MOE_ROUTER_CC_CASE(4)
        MOE_ROUTER_CC_CASE(5) MOE_ROUTER_CC_CASE(6) MOE_ROUTER_CC_CASE(7) MOE_ROUTER_CC_CASE(8)
        MOE_ROUTER_CC_CASE(9) MOE_ROUTER_CC_CASE(10) MOE_ROUTER_CC_CASE(11) MOE_ROUTER_CC_CASE(12)
        MOE_ROUTER_CC_CASE(13) MOE_ROUTER_CC_CASE(14) MOE_ROUTER_CC_CASE(15) MOE_ROUTER_CC_CASE(16)
#undef MOE_ROUTER_CC_CASE
        default: return cudaErrorInvalidValue;
    }
}

int launch_router_cc(int T, int H, int E, int dtype, const void* x, const void* w_r, float* logits,
                     cudaStream_t stream) {
    if (T == 0) return 0;
    if (!router_cc_fits(H, E, dtype)) return -1;
    DeviceInfo d;
    int rc = current_device(&d);
    if (rc != 0) return rc;
    cudaError_t e = dtype == 0 ? launch_router_cc_t<__nv_bfloat16>(T, H, E, x, w_r, logits, d.num_sms, stream)
                               : launch_router_cc_t<float>(T, H, E, x, w_r, logits, d.num_sms, stream);
    count_launch();
    return launched(e);
}

template <typename T, int kE>
cudaError_t launch_route_cc_e(const RouteCcArgs& a, int num_sms, cudaStream_t stream) {
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(route_cc_kernel<T, kE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kRouterCcMaxBytes);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    // one token per warp where T allows, at most two blocks per SM
    long long blocks = (a.T + 31) / 32;
    if (blocks > 2LL * num_sms) blocks = 2LL * num_sms;
    const size_t wr = (size_t)kE * a.H * sizeof(T), al = align_smem_bytes(kE);
    return launch_kernel(route_cc_kernel<T, kE>, dim3((int)blocks), dim3(kAlignThreads), wr > al ? wr : al, stream,
                         a.T, a.H, a.K, a.score_fn, a.renorm, a.B, a.mode, a.P_max, static_cast<const T*>(a.x),
                         static_cast<const T*>(a.w_r), a.logits_override, a.k_per_token, a.logits, a.ids, a.w,
                         a.counts, a.offsets, a.sorted_ids, a.block_expert, a.pos, a.scalars, a.stats_copy,
                         a.done_ctr);
}

template <typename T>
cudaError_t launch_route_cc_t(const RouteCcArgs& a, int num_sms, cudaStream_t s) {
    switch (a.E) {
#define MOE_ROUTE_CC_CASE(n) \
    case n: return launch_route_cc_e<T, n>(a, num_sms, s);
        MOE_ROUTE_CC_CASE(1) MOE_ROUTE_CC_CASE(2) MOE_ROUTE_CC_CASE(3) MOE_ROUTE_CC_CASE(4)
        MOE_ROUTE_CC_CASE(5) MOE_ROUTE_CC_CASE(6) MOE_ROUTE_CC_CASE(7) MOE_ROUTE_CC_CASE(8)
        MOE_ROUTE_CC_CASE(9) MOE_ROUTE_CC_CASE(10) MOE_ROUTE_CC_CASE(11) MOE_ROUTE_CC_CASE(12)
        MOE_ROUTE_CC_CASE(13) MOE_ROUTE_CC_CASE(14) MOE_ROUTE_CC_CASE(15) MOE_ROUTE_CC_CASE(16)
#undef MOE_ROUTE_CC_CASE
        default: return cudaErrorInvalidValue;
    }
}

int launch_route_cc(const RouteCcArgs& a, cudaStream_t stream) {
    if (a.T == 0) return 0;
    if (!router_cc_fits(a.H, a.E, a.dtype)) return -1;
    DeviceInfo d;
    int rc = current_device(&d);
    if (rc != 0) return rc;
    cudaError_t e = a.dtype == 0 ? launch_route_cc_t<__nv_bfloat16>(a, d.num_sms, stream)
                                 : launch_route_cc_t<float>(a, d.num_sms, stream);
    count_launch();
    return launched(e);
}

// Slices of the hidden dimension (multiples of 256 elements) so that the
// router GEMV covers about one wave of warps on the device.
void route_small_slices(int T, int H, int E, int num_sms, int* nslices, int* slice_w) {
    const long long pairs = (long long)E * ((T + kRouteTokGroup - 1) / kRouteTokGroup);
    const long long target = (long long)num_sms * (kAlignThreads / 32);
    const int max_sl = (H + 255) / 256;
    long long ns = (target + pairs - 1) / pairs;
    if (ns > max_sl) ns = max_sl;
    if (ns < 1) ns = 1;
    const int w = (int)(((H + ns - 1) / ns + 255) / 256 * 256);
    *slice_w = w;
    *nslices = (H + w - 1) / w;
}

int launch_route_small(int T, int H, int E, int K, int score_fn, int renorm, int B, int mode, long long P_max,
                       int dtype,
                       const void* x, const void* w_r, const float* logits_override, const int32_t* k_per_token,
                       float* part, float* logits, int32_t* ids, float* w, int32_t* counts, int32_t* offsets,
                       int32_t* sorted_ids, int32_t* block_expert, int32_t* pos, int32_t* scalars,
                       int32_t* stats_copy, int* done_ctr, cudaStream_t stream) {
    DeviceInfo d;
    int rc = current_device(&d);
    if (rc != 0) return rc;
    const size_t smem = align_smem_bytes(E);
    static bool attr_done = false;
    if (!attr_done) {
        if (cudaFuncSetAttribute(route_small_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 96 * 1024) != cudaSuccess ||
            cudaFuncSetAttribute(route_small_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024) !=
                cudaSuccess) {
            cudaGetLastError();
            return -3;
        }
        attr_done = true;
    }
    int ns, sw;
    route_small_slices(T, H, E, d.num_sms, &ns, &sw);
    const long long units = (long long)E * ((T + kRouteTokGroup - 1) / kRouteTokGroup) * ns;
    const int blocks = (int)((units + kAlignThreads / 32 - 1) / (kAlignThreads / 32));
    cudaError_t e;
    if (dtype == 0)
        e = launch_kernel(route_small_kernel<__nv_bfloat16>, dim3(blocks), dim3(kAlignThreads), smem, stream, T, H, E,
                          K, score_fn, renorm, B, mode, P_max, ns, sw, static_cast<const __nv_bfloat16*>(x),
                          static_cast<const __nv_bfloat16*>(w_r), logits_override, k_per_token, part, logits, ids, w,
                          counts,
                          offsets, sorted_ids, block_expert, pos, scalars, stats_copy, done_ctr);
    else
        e = launch_kernel(route_small_kernel<float>, dim3(blocks), dim3(kAlignThreads), smem, stream, T, H, E, K,
                          score_fn, renorm, B, mode, P_max, ns, sw, static_cast<const float*>(x),
                          static_cast<const float*>(w_r), logits_override, k_per_token, part, logits, ids, w, counts,
                          offsets,
                          sorted_ids, block_expert, pos, scalars, stats_copy, done_ctr);
    count_launch();
    return launched(e);
}

int launch_align(int T, int K, int E, int B, int mode, long long P_max, const int32_t* ids, int32_t* counts,
                 int32_t* offsets, int32_t* sorted_ids, int32_t* block_expert, int32_t* pos, int32_t* scalars,
                 int32_t* stats_copy, cudaStream_t stream) {
    const size_t smem = align_smem_bytes(E);
    static bool attr_done = false;
    if (!attr_done) {
        if (cudaFuncSetAttribute(align_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024) !=
            cudaSuccess) {
            cudaGetLastError();
            return -3;
        }
        attr_done = true;
    }
    cudaError_t e = launch_kernel(align_kernel, dim3(1), dim3(kAlignThreads), smem, stream, T, K, E, B, mode, P_max, ids,
                                  counts, offsets, sorted_ids, block_expert, pos, scalars, stats_copy);
    count_launch();
    return launched(e);
}

// ---------------------------------------------------------------- permute
// x_perm[p] = x[sorted_ids[p] / K] (zero row for a padding slot), p < P.
__global__ void __launch_bounds__(256) permute_kernel(int row_vec, int K, const int4* __restrict__ x,
                                                      const int32_t* __restrict__ sorted_ids,
                                                      const int32_t* __restrict__ scalars, int4* __restrict__ x_perm) {
    pdl_launch_dependents();
    pdl_wait();
    const int P = scalars[0];
    const int rows_per_block = blockDim.x / 64;  // 64 threads per row
    const int sub = threadIdx.x / 64, l = threadIdx.x % 64;
    for (long long p = (long long)blockIdx.x * rows_per_block + sub; p < P; p += (long long)gridDim.x * rows_per_block) {
        const int src = sorted_ids[p];
        int4* dst = x_perm + p * row_vec;
        if (src >= 0) {
            const int4* s = x + (long long)(src / K) * row_vec;
            for (int v = l; v < row_vec; v += 64) dst[v] = __ldg(s + v);
        } else {
            const int4 z = make_int4(0, 0, 0, 0);
            for (int v = l; v < row_vec; v += 64) dst[v] = z;
        }
    }
}

int launch_permute(int H, int K, int dtype, long long P_max, const void* x, const int32_t* sorted_ids,
                   const int32_t* scalars, void* x_perm, cudaStream_t stream) {
    if (P_max <= 0) return 0;
    DeviceInfo d;
    int rc = current_device(&d);
    if (rc != 0) return rc;
    const int elt = dtype == 0 ? 2 : 4;
    const int row_vec = H * elt / 16;
    long long rows_per_block = 4;
    long long blocks = (P_max + rows_per_block - 1) / rows_per_block;
    const long long cap = (long long)d.num_sms * 8;
    if (blocks > cap) blocks = cap;
    cudaError_t e = launch_kernel(permute_kernel, dim3((int)blocks), dim3(256), 0, stream, row_vec, K,
                                  static_cast<const int4*>(x), sorted_ids, scalars, static_cast<int4*>(x_perm));
    count_launch();
    return launched(e);
}

// Exact two-term E4M3 split of bf16 token rows, the token operand of the FP8
// gate/up MMAs: with s the smallest power of two for which max |x| <= 448 s
// (at least 2^-126),
// x / s is exact, hi = E4M3(x / s) keeps its leading four significant bits,
// and the rest r = x / s - hi (exact in fp32; at most four significant bits
// for the eight of a bf16 value) is lo = E4M3(r), so x = s (hi + lo) except
// where r falls below the E4M3 subnormal grid (2^-9, i.e. below 2^-17 of the
// row's largest value).  One warp per row; rows gathered by sorted_ids
// (padding slots: zero codes, scale 1) or taken in order.  codes holds the hi
// rows, then, lo_rows rows further on, the lo rows.
__device__ __forceinline__ uint8_t e4m3_rn(float v) { return __nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3); }
__device__ __forceinline__ float e4m3_value(uint8_t c) {
    __nv_fp8_e4m3 f;
    f.__x = c;
    return static_cast<float>(f);
}

template <bool kGather>
__global__ void __launch_bounds__(256) split_e4m3_kernel(int H, int K, long long rows, const int4* __restrict__ x,
                                                         const int32_t* __restrict__ sorted_ids,
                                                         const int32_t* __restrict__ scalars, uint8_t* __restrict__ codes,
                                                         long long lo_rows, float* __restrict__ scales) {
    pdl_launch_dependents();
    pdl_wait();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nv = H / 8;  // 16-byte vectors of 8 bf16 per row
    const long long n = kGather ? (long long)scalars[0] : rows;
    for (long long p = (long long)blockIdx.x * 8 + warp; p < n; p += (long long)gridDim.x * 8) {
        const int4* src = nullptr;
        if (kGather) {
            const int a = sorted_ids[p];
            if (a >= 0) src = x + (long long)(a / K) * nv;
        } else {
            src = x + p * nv;
        }
        uint2* hi = reinterpret_cast<uint2*>(codes + p * H);
        uint2* lo = reinterpret_cast<uint2*>(codes + (lo_rows + p) * H);
        if (!src) {
            for (int v = lane; v < nv; v += 32) hi[v] = lo[v] = make_uint2(0u, 0u);
            if (lane == 0) scales[p] = 1.f;
            continue;
        }
        float amax = 0.f;
        for (int v = lane; v < nv; v += 32) {
            const int4 q = __ldg(src + v);
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(h[i]);
                amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float sc = e4m3_pow2_scale(amax);
        const float inv = e4m3_pow2_inv_scale(amax);
        for (int v = lane; v < nv; v += 32) {
            const int4 q = __ldg(src + v);
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
            uint32_t hw[2] = {0u, 0u}, lw[2] = {0u, 0u};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(h[i]);
                const float y0 = f.x * inv, y1 = f.y * inv;
                const uint8_t h0 = e4m3_rn(y0), h1 = e4m3_rn(y1);
                const uint8_t l0 = e4m3_rn(y0 - e4m3_value(h0)), l1 = e4m3_rn(y1 - e4m3_value(h1));
                const int sh = 16 * (i & 1);
                hw[i >> 1] |= ((uint32_t)h0 | ((uint32_t)h1 << 8)) << sh;
                lw[i >> 1] |= ((uint32_t)l0 | ((uint32_t)l1 << 8)) << sh;
            }
            hi[v] = make_uint2(hw[0], hw[1]);
            lo[v] = make_uint2(lw[0], lw[1]);
        }
        if (lane == 0) scales[p] = sc;
    }
}

int launch_split_e4m3(int H, int K, long long rows, const void* x, const int32_t* sorted_ids, const int32_t* scalars,
                      uint8_t* codes, long long lo_rows, float* scales, cudaStream_t stream) {
    if (rows <= 0) return 0;
    if (H % 8) return -1;
    DeviceInfo d;
    int rc = current_device(&d);
    if (rc != 0) return rc;
    long long blocks = (rows + 7) / 8;
    const long long cap = (long long)d.num_sms * 8;
    if (blocks > cap) blocks = cap;
    cudaError_t e = sorted_ids
                        ? launch_kernel(split_e4m3_kernel<true>, dim3((int)blocks), dim3(256), 0, stream, H, K, rows,
                                        static_cast<const int4*>(x), sorted_ids, scalars, codes, lo_rows, scales)
                        : launch_kernel(split_e4m3_kernel<false>, dim3((int)blocks), dim3(256), 0, stream, H, K, rows,
                                        static_cast<const int4*>(x), sorted_ids, scalars, codes, lo_rows, scales);
    count_launch();
    return launched(e);
}

// ---------------------------------------------------------------- combine
// out[t] = sum_k w[t,k] * y_perm[pos[t*K+k]] (+ shared[t]), fp32, ascending k.
template <typename T>
struct Vec16 {
    static constexpr int N = 16 / sizeof(T);
};

__device__ __forceinline__ void unpack(const int4& v, float* f, const __nv_bfloat16*) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}
__device__ __forceinline__ void unpack(const int4& v, float* f, const float*) {
    const float* x = reinterpret_cast<const float*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = x[i];
}
__device__ __forceinline__ int4 pack(const float* f, const __nv_bfloat16*) {
    int4 v;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return v;
}
__device__ __forceinline__ int4 pack(const float* f, const float*) {
    int4 v;
    float* x = reinterpret_cast<float*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = f[i];
    return v;
}

// Stores the N fp32 sums of one 16-byte input vector: rounded once to the
// activation dtype, or (TP partials, which an all-reduce sums next) unrounded.
template <int N>
__device__ __forceinline__ void store_sums(const float* acc, __nv_bfloat16* out) {
    *reinterpret_cast<int4*>(out) = pack(acc, (const __nv_bfloat16*)nullptr);
}
template <int N>
__device__ __forceinline__ void store_sums(const float* acc, float* out) {
#pragma unroll
    for (int i = 0; i < N; i += 4)
        *reinterpret_cast<float4*>(out + i) = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
}

// One thread per 16-byte vector of one token's output row: the K expert rows'
// vectors are all requested before the first is used (K <= 16, unrolled), then
// summed in fp32 in ascending k (empty slots skipped), the shared output added
// last, one rounding.  The output holds the columns [col0, col0 + ncol) (in
// 16-byte vectors of the input rows; ncol vectors per output row).
template <typename T, typename TOut, int kMaxK>
__global__ void __launch_bounds__(256) combine_kernel(int T_, int row_vec, int K, int col0, int ncol,
                                                      const int4* __restrict__ y_perm,
                                                      const int32_t* __restrict__ pos, const float* __restrict__ w,
                                                      const int4* __restrict__ sh, TOut* __restrict__ out) {
    constexpr int N = Vec16<T>::N;
    pdl_launch_dependents();
    pdl_wait();
    const long long total = (long long)T_ * ncol;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long t = i / ncol;
        const int v = col0 + (int)(i - t * ncol);
        int p[kMaxK];
        int4 yv[kMaxK];
#pragma unroll
        for (int k = 0; k < kMaxK; ++k)
            if (k < K) p[k] = __ldg(pos + t * K + k);
#pragma unroll
        for (int k = 0; k < kMaxK; ++k)
            if (k < K && p[k] >= 0) yv[k] = __ldcs(y_perm + (long long)p[k] * row_vec + v);
        int4 sv = make_int4(0, 0, 0, 0);
        if (sh) sv = __ldcs(sh + t * row_vec + v);
        float acc[N];
#pragma unroll
        for (int j = 0; j < N; ++j) acc[j] = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxK; ++k) {
            if (k < K && p[k] >= 0) {  // empty slot (per-token dynamic K): skipped
                float y[N];
                unpack(yv[k], y, (const T*)nullptr);
                const float wk = __ldg(w + t * K + k);
#pragma unroll
                for (int j = 0; j < N; ++j) acc[j] += wk * y[j];
            }
        }
        if (sh) {
            float y[N];
            unpack(sv, y, (const T*)nullptr);
#pragma unroll
            for (int j = 0; j < N; ++j) acc[j] += y[j];
        }
        store_sums<N>(acc, out + i * N);
    }
}

int launch_combine(int T, int H, int K, int dtype, const void* y_perm, const int32_t* pos, const float* w,
                   const void* shared_out, void* out, cudaStream_t stream, bool out_f32, int col0, int ncols) {
    if (T == 0) return 0;
    DeviceInfo d;
    int rc = current_device(&d);
    if (rc != 0) return rc;
    const int elt = dtype == 0 ? 2 : 4;
    const int row_vec = H * elt / 16;
    if (ncols < 0) col0 = 0, ncols = H;
    if ((col0 * elt) % 16 || (ncols * elt) % 16 || col0 < 0 || col0 + ncols > H) return -1;
    const int c0 = col0 * elt / 16, nc = ncols * elt / 16;
    const int threads = 256;
    // one thread per output vector (a grid of up to 2^31 - 1 blocks covers
    // every layer this library accepts; beyond that the threads stride)
    long long blocks = ((long long)T * nc + threads - 1) / threads;
    if (blocks > 0x7fffffffLL) blocks = 0x7fffffffLL;
    const int4* y4 = static_cast<const int4*>(y_perm);
    const int4* s4 = static_cast<const int4*>(shared_out);
    const dim3 g((unsigned)blocks), b(threads);
    cudaError_t e;
    // the K expert rows are held in registers: size the array to K's bucket
    auto go = [&](auto kmax) -> cudaError_t {
        constexpr int kK = decltype(kmax)::value;
        if (dtype == 0 && !out_f32)
            return launch_kernel(combine_kernel<__nv_bfloat16, __nv_bfloat16, kK>, g, b, 0, stream, T, row_vec, K, c0,
                                 nc, y4, pos, w, s4, static_cast<__nv_bfloat16*>(out));
        if (dtype == 0)
            return launch_kernel(combine_kernel<__nv_bfloat16, float, kK>, g, b, 0, stream, T, row_vec, K, c0, nc, y4,
                                 pos, w, s4, static_cast<float*>(out));
        return launch_kernel(combine_kernel<float, float, kK>, g, b, 0, stream, T, row_vec, K, c0, nc, y4, pos, w, s4,
                             static_cast<float*>(out));
    };
    if (K <= 2) e = go(std::integral_constant<int, 2>());
    else if (K <= 4) e = go(std::integral_constant<int, 4>());
    else if (K <= 8) e = go(std::integral_constant<int, 8>());
    else e = go(std::integral_constant<int, 16>());
    count_launch();
    return launched(e);
}

// ------------------------------------------------------------ TP reduction
// out[i] = sum over r of parts[r][i], fp32 in rank order, one rounding to the
// output dtype.  parts[r] may live on another GPU (a peer mapping): plain
// coalesced 16-byte loads, 4 elements per thread per step, grid-stride over
// the whole vector with a grid of a few blocks per SM.
struct TpParts {
    const float4* p[kTpMaxParts];
};

template <typename TOut>
__device__ __forceinline__ void store4(TOut* out, long long i, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* out, long long i, float4 v) {
    reinterpret_cast<float4*>(out)[i] = v;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* out, long long i, float4 v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    reinterpret_cast<uint2*>(out)[i] = u;
}

template <typename TOut>
__global__ void __launch_bounds__(256) tp_reduce_kernel(TpParts parts, int n, long long n4, TOut* __restrict__ out) {
    pdl_launch_dependents();
    pdl_wait();
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
        float4 acc = __ldcs(parts.p[0] + i);
        for (int r = 1; r < n; ++r) {
            const float4 v = __ldcs(parts.p[r] + i);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        store4<TOut>(out, i, acc);
    }
}

int launch_tp_reduce(int n, const float* const* parts, long long count, int dtype, void* out, cudaStream_t stream) {
    if (count == 0) return 0;
    DeviceInfo d;
    int rc = current_device(&d);
    if (rc != 0) return rc;
    TpParts tp{};
    for (int r = 0; r < n; ++r) tp.p[r] = reinterpret_cast<const float4*>(parts[r]);
    const long long n4 = count / 4;
    long long blocks = (n4 + 255) / 256;
    const long long cap = (long long)d.num_sms * 8;
    if (blocks > cap) blocks = cap;
    cudaError_t e = dtype == 0 ? launch_kernel(tp_reduce_kernel<__nv_bfloat16>, dim3((int)blocks), dim3(256), 0,
                                               stream, tp, n, n4, static_cast<__nv_bfloat16*>(out))
                               : launch_kernel(tp_reduce_kernel<float>, dim3((int)blocks), dim3(256), 0, stream, tp,
                                               n, n4, static_cast<float*>(out));
    count_launch();
    return launched(e);
}

// One output row from n all-reduced column blocks: out[t][c * Hc + j] =
// parts[c][t * Hc + j], rounded once to the output dtype (4 elements per
// thread, grid-stride over all T * H).
template <typename TOut>
__global__ void __launch_bounds__(256) tp_gather_kernel(TpParts parts, int T_, int hc4, int n, TOut* __restrict__ out) {
    pdl_launch_dependents();
    pdl_wait();
    const long long row4 = (long long)hc4 * n;
    const long long total = (long long)T_ * row4;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
        const long long t = i / row4;
        const int rem = (int)(i - t * row4);
        const int c = rem / hc4, j = rem - c * hc4;
        store4<TOut>(out, i, __ldcs(parts.p[c] + t * hc4 + j));
    }
}

int launch_tp_gather(int n, const float* const* parts, int T, int H, int dtype, void* out, cudaStream_t stream) {
    if (T == 0) return 0;
    DeviceInfo d;
    int rc = current_device(&d);
    if (rc != 0) return rc;
    TpParts tp{};
    for (int r = 0; r < n; ++r) tp.p[r] = reinterpret_cast<const float4*>(parts[r]);
    const int hc4 = H / n / 4;
    const long long total = (long long)T * H / 4;
    long long blocks = (total + 255) / 256;
    const long long cap = (long long)d.num_sms * 8;
    if (blocks > cap) blocks = cap;
    cudaError_t e = dtype == 0 ? launch_kernel(tp_gather_kernel<__nv_bfloat16>, dim3((int)blocks), dim3(256), 0,
                                               stream, tp, T, hc4, n, static_cast<__nv_bfloat16*>(out))
                               : launch_kernel(tp_gather_kernel<float>, dim3((int)blocks), dim3(256), 0, stream, tp,
                                               T, hc4, n, static_cast<float*>(out));
    count_launch();
    return launched(e);
}

// ------------------------------------------------------ FP8 quantisation
// Row-wise E4M3 codes for the decode weight stream: one block per row, the
// row's max |w| by a block reduction, scale = max / 448 (1 for an all-zero
// row), code = E4M3(w / scale) rounded to nearest even with saturation.  The
// divisions are IEEE (correctly rounded) so that the codes are reproducible.
template <typename T>
__global__ void __launch_bounds__(256) quantize_fp8_kernel(int cols, const T* __restrict__ w,
                                                           uint8_t* __restrict__ q, float* __restrict__ scales) {
    __shared__ float red[8];
    const long long row = blockIdx.x;
    const T* wr = w + row * cols;
    float amax = 0.f;
    for (int c = threadIdx.x; c < cols; c += blockDim.x) amax = fmaxf(amax, fabsf(Elt<T>::to_f(wr[c])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = red[0];
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) amax = fmaxf(amax, red[i]);
    const float sc = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    if (threadIdx.x == 0) scales[row] = sc;
    for (int c = threadIdx.x; c < cols; c += blockDim.x)
        q[row * cols + c] = __nv_cvt_float_to_fp8(__fdiv_rn(Elt<T>::to_f(wr[c]), sc), __NV_SATFINITE, __NV_E4M3);
}

int launch_quantize_fp8(long long rows, int cols, int dtype, const void* w, uint8_t* q, float* scales,
                        cudaStream_t stream) {
    if (rows == 0) return 0;
    cudaError_t e = dtype == 0 ? launch_kernel(quantize_fp8_kernel<__nv_bfloat16>, dim3((unsigned)rows), dim3(256), 0,
                                               stream, cols, static_cast<const __nv_bfloat16*>(w), q, scales)
                               : launch_kernel(quantize_fp8_kernel<float>, dim3((unsigned)rows), dim3(256), 0, stream,
                                               cols, static_cast<const float*>(w), q, scales);
    count_launch();
    return launched(e);
}

}  // namespace moe
