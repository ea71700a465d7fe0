/*
 * moe.h -- C ABI of libmoe.so: the single-GPU forward of one
 * Mixture-of-Experts FFN layer on NVIDIA B200 (sm_100a), and the dense SwiGLU
 * FFN used as its FLOP-aligned (DenseFA) and parameter-aligned (DensePA)
 * baselines.
 *
 * The operations follow the pages on "Demystifying the Mixture of Experts
 * Serving Tax" (MLSys 2026):
 *   - talk notes, "Key findings 5": the MoE block runs a router, top-K
 *     selection, alignment, a grouped GEMM (GroupGEMM) and a local sum
 *     (combine);
 *   - talk notes, "Padding model (Section 5.1)": block-wise padding, each
 *     expert's token count N_i rounded up to the block size B,
 *     P = sum_i ceil(N_i / B) * B padded rows;
 *   - talk notes, "Definition": tax tau = T(MoE, b) / T(DenseFA, b) (Eq. 1);
 *     DenseFA = the MoE layer replaced by an FFN whose intermediate size is
 *     scaled by K (same FLOPs per token); DensePA = a dense FFN with the MoE
 *     layer's total parameters;
 *   - talk notes, Table 2: shared experts (always-on FFNs).
 *
 * Symbols: T tokens, H hidden size, E routed experts, K experts per token,
 * I expert intermediate size, S shared experts of width I_s (one dense FFN
 * of width S * I_s), B padding tile, A = T * K assignments, a = t * K + k.
 *
 * Conventions (every entry point):
 *   - Every pointer is a DEVICE pointer unless stated; all arrays are
 *     row-major and contiguous.  The caller owns all memory: the library
 *     never allocates or frees device memory.
 *   - Work is enqueued on `stream`; no call synchronises the stream except
 *     moe_check_status().  A return of MOE_OK means "enqueued".
 *   - Activations and weights are bf16 (dtype 0) or fp32 (dtype 1); router
 *     logits and gate weights are always fp32; indices are int32.
 *   - Weights are laid out like nn.Linear ([out, in]):
 *       w_router [E, H];
 *       w13 [E, 2I, H]: rows 0..I-1 the gate projection W1, rows I..2I-1 the
 *         up projection W3;   w2 [E, H, I];
 *       shared / dense FFN: w13 [2*I_d, H], w2 [H, I_d].
 *   - Row strides must be multiples of 16 bytes: H and I multiples of 8
 *     (bf16) or 4 (fp32).  Device pointers must be 16-byte aligned.
 *   - Errors are returned, never thrown; no CUDA error is left pending.
 *   - T = 0 is a valid no-op (pointers may then be NULL), except that
 *     moe_align_pad still writes zero counts, offsets and scalars.
 *   - The device must be sm_100 (B200); other devices get MOE_ERR_DEVICE.
 *   - Kernel waits are bounded: a wait that exceeds the limit sets a status
 *     word in the workspace and the kernel returns; moe_check_status()
 *     reports it as MOE_ERR_TIMEOUT.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (the same type as cudaStream_t / CUstream). */
typedef struct CUstream_st* moe_stream_t;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_ARG = -1,        /* NULL pointer, bad size or unsupported option */
    MOE_ERR_WORKSPACE = -2,  /* workspace smaller than the *_workspace_size() query */
    MOE_ERR_CUDA = -3,       /* a CUDA launch or runtime call failed */
    MOE_ERR_TIMEOUT = -4,    /* a device-side wait ran out (reported by moe_check_status) */
    MOE_ERR_DEVICE = -5      /* current device is not sm_100 */
} moe_status_t;

typedef struct {
    int T;          /* tokens, >= 0 */
    int H;          /* hidden size */
    int E;          /* routed experts, 1..1024 */
    int K;          /* experts per token, 1..min(E, 16) */
    int I;          /* routed expert intermediate size */
    int n_shared;   /* shared experts S (0 = none) */
    int I_shared;   /* intermediate size of one shared expert I_s */
    int tile_B;     /* padding tile B, 1..256 */
    int score_fn;   /* 0 = softmax, 1 = sigmoid */
    int renorm;     /* 1: weights normalised over the selected K */
    int dtype;      /* 0 = bf16, 1 = fp32 (activations and weights) */
    int pad_mode;   /* 0 = block-wise padding: each expert's rows rounded up to
                       tile_B; 1 = max-value padding: every expert gets the
                       rounded row count of the most loaded expert (Demystifying
                       the MoE Serving Tax, "Padding model (Section 5.1)") */
} moe_config_t;

/* Text for a status code (static storage). */
const char* moe_status_string(int status);

/* Upper bound on padded rows, the length callers give sorted_ids and the
 * permuted buffers (-1 on a bad configuration), A = T * K:
 *   pad_mode 0 (block-wise): P_max = A + min(E, A) * (B - 1);
 *   pad_mode 1 (max-value):  P_max = E * ceil(min(T, A) / B) * B, which
 *     assumes an expert holds at most one assignment per token (true of every
 *     top-K routing); ids that repeat within a token are flagged by the
 *     alignment instead (see moe_align_pad). */
int64_t moe_padded_rows_max(const moe_config_t* cfg);

/* Bytes of workspace moe_layer_forward needs for this configuration on the
 * current device (0 on a bad configuration).  The workspace must be zeroed
 * once before its first use (e.g. cudaMemsetAsync); the library leaves its
 * control words zero after every call that completes without a timeout. */
size_t moe_workspace_size(const moe_config_t* cfg);

/* Byte offset, inside the moe_layer_forward workspace, of the fp32 router
 * logits [T,E] the last forward computed (-1 on a bad configuration).  For
 * T <= 64 and a small router matrix (E * H <= 2^17) the forward computes them
 * on the CUDA cores (fp32 sums of exact products) in the same launch as top-K
 * and alignment, otherwise as moe_router_gemm does; either way they are what
 * top-K selected on unless logits_override was given. */
int64_t moe_layer_logits_offset(const moe_config_t* cfg);

/* Bytes of workspace moe_router_gemm / moe_grouped_ffn / dense_ffn need (the
 * control words and stream-K partial tiles only), same zeroing rule. */
size_t moe_gemm_workspace_size(void);

/* Router GEMM (stage "router"): logits[T,E] (fp32) = x[T,H] . w_router[E,H]^T,
 * products of the inputs accumulated in fp32.  A router matrix that fits
 * shared memory (E <= 16, E*H*elt <= 96 KB, H % 8 == 0) runs on the CUDA cores
 * with exact products (fp32 inputs too); larger ones on the tensor cores (fp32
 * inputs: tf32 products).  The summation order differs between the two, so
 * results agree to fp32 rounding.  `workspace` as returned by
 * moe_gemm_workspace_size() (unused by the CUDA-core form). */
int moe_router_gemm(const moe_config_t* cfg, const void* x, const void* w_router,
                    float* logits, void* workspace, size_t ws_bytes, moe_stream_t stream);

/* Router GEMM for callers that cannot allocate device memory when they
 * enqueue work -- for example a plugin inside another engine whose enqueue
 * step must not allocate, or a runtime that plans every byte of device memory
 * before it starts.  The pages have no counterpart: this is a library
 * convenience, not a step of the method.
 *   Same arguments as moe_router_gemm, minus the workspace, and always the
 *   tensor-core form (equal to moe_router_gemm's result up to fp32 rounding
 *   where that one takes the CUDA-core form): the
 *   scratch (status word, stream-K counters, partial tiles) lives in a fixed
 *   ~5 MiB array in the library's device memory, present on every GPU that
 *   loads the library until the process exits.  No allocation is made.
 *   Limits: T <= 32 (larger T returns MOE_ERR_ARG: use moe_router_gemm) and
 *   at most 160 SMs.  The first call on each device looks up the array's
 *   device address (cudaGetSymbolAddress).  Each call clears the shared
 *   control words before its launch; calls that overlap on the GPU
 *   (unordered streams) race on the shared array.  A device wait that runs out sets a status word in the
 *   array and may leave logits partly written (the tiles whose blocks gave up);
 *   moe_router_gemm_noalloc_status reports it. */
int moe_router_gemm_noalloc(const moe_config_t* cfg, const void* x, const void* w_router,
                            float* logits, moe_stream_t stream);

/* Status of the moe_router_gemm_noalloc calls enqueued on `stream` so far:
 * synchronises the stream, reads the status word of the fixed array and
 * clears it.  MOE_ERR_TIMEOUT when a device wait ran out (the logits of that
 * call are not to be used), MOE_OK otherwise, MOE_ERR_CUDA on a CUDA error.
 * The next moe_router_gemm_noalloc call also clears the word, so call this
 * before it.  No allocation.  The pages have no counterpart. */
int moe_router_gemm_noalloc_status(moe_stream_t stream);

/* Top-K gating (stage "top-K selection"), one token per warp:
 *   topk_ids[T,K]: the K largest logits[t,:], descending, the lower expert
 *     index first on equal values (IEEE comparison: -0.0 ties +0.0; +-inf are
 *     ordered normally; NaN logits give unspecified but in-range ids);
 *   topk_w[T,K]: softmax (score_fn 0) or sigmoid (score_fn 1) weights,
 *     renormalised over the selected K when cfg->renorm (softmax without
 *     renorm: the full softmax over E, restricted to the selected experts;
 *     sigmoid without renorm: the raw sigmoid), computed in fp32. */
int moe_route(const moe_config_t* cfg, const float* logits, int32_t* topk_ids,
              float* topk_w, moe_stream_t stream);

/* Per-token dynamic K (the routing top-k as a per-request runtime knob: the
 * MoE-Prism write-up).  As moe_route, with token t selecting its
 * k_per_token[t] largest logits (device int32 [T]; values clamped to
 * [0, cfg->K]); slots k >= k_per_token[t] get id -1 and weight 0, and the
 * weights are renormalised over the k_per_token[t] selected.  NULL: K for
 * every token (= moe_route).  The alignment treats id -1 as an empty slot
 * (no row, pos -1, not flagged) and the combine skips it. */
int moe_route_k(const moe_config_t* cfg, const float* logits, const int32_t* k_per_token,
                int32_t* topk_ids, float* topk_w, moe_stream_t stream);

/* Token-to-expert alignment (stage "alignment", Section 5.1 padding model).
 * With e(a) = topk_ids[a]:
 *   counts[E]        N_e = #{a : e(a) = e}
 *   offsets[E+1]     exclusive scan of the padded counts; offsets[E] = P.
 *                    cfg->pad_mode 0 (block-wise): ceil(N_e / B) * B;
 *                    1 (max-value): ceil(max_i N_i / B) * B for every expert
 *   sorted_ids[P_max] the assignments of expert e in ascending a at
 *                    offsets[e] .. offsets[e] + N_e - 1; every other slot -1
 *   block_expert[ceil(P_max/B)]  e for blocks inside expert e's segment, -1 after P
 *   pos[A]           the slot p with sorted_ids[p] = a (-1 for an empty slot)
 *   scalars[4]       {P, E_active = #{e : N_e > 0}, 0, 0}
 * Bit-exact and deterministic.  Id -1 is an empty slot (per-token dynamic K):
 * no row, pos -1.  Other out-of-range ids are skipped and flagged in
 * scalars[2] (bit 1; nonzero = bad input).  Max-value padding with ids that
 * repeat within a token (no top-K produces them) can need more than P_max rows:
 * the alignment then sets bit 2 of scalars[2] and writes an empty routing
 * (P = 0, E_active = 0, offsets 0, every pos -1, sorted_ids and block_expert
 * -1), writing nothing at or past P_max. */
int moe_align_pad(const moe_config_t* cfg, const int32_t* topk_ids, int32_t* counts,
                  int32_t* offsets, int32_t* sorted_ids, int32_t* block_expert,
                  int32_t* pos, int32_t* scalars, moe_stream_t stream);

/* Permute (gather): x_perm[p] = x[sorted_ids[p] / K] for p < P, a zero row
 * where sorted_ids[p] = -1; rows >= P are left untouched.  x_perm has P_max
 * rows of H. */
int moe_permute(const moe_config_t* cfg, const void* x, const int32_t* sorted_ids,
                const int32_t* scalars, void* x_perm, moe_stream_t stream);

/* Grouped expert FFN over the padded segments (stage "GroupGEMM"): for each
 * expert e and each row p in [offsets[e], offsets[e+1]):
 *   act[p]    = silu(x_perm[p] . W1_e^T) * (x_perm[p] . W3_e^T)   ([P_max, I])
 *   y_perm[p] = act[p] . W2_e^T                                    ([P_max, H])
 * fp32 accumulation on the tensor cores; act and y_perm are stored in the
 * activation dtype.  `act` is caller-provided scratch of P_max * I elements. */
int moe_grouped_ffn(const moe_config_t* cfg, const void* x_perm, const void* w13,
                    const void* w2, const int32_t* offsets, void* act, void* y_perm,
                    void* workspace, size_t ws_bytes, moe_stream_t stream);

/* The two launches of moe_grouped_ffn, separately (same arguments):
 * gate/up + SwiGLU writes act[P_max, I]; down reads act and writes
 * y_perm[P_max, H]. */
int moe_grouped_gate_up(const moe_config_t* cfg, const void* x_perm, const void* w13,
                        const int32_t* offsets, void* act, void* workspace, size_t ws_bytes,
                        moe_stream_t stream);
int moe_grouped_down(const moe_config_t* cfg, const void* act, const void* w2,
                     const int32_t* offsets, void* y_perm, void* workspace, size_t ws_bytes,
                     moe_stream_t stream);

/* Weighted un-permute and combine (stage "local sum"):
 *   out[t] = sum_{k=0..K-1} topk_w[t,k] * y_perm[pos[t*K+k]]  (+ shared_out[t])
 * summed in fp32 in ascending k, the shared output added last, one final
 * rounding to the activation dtype.  shared_out may be NULL. */
int moe_combine(const moe_config_t* cfg, const void* y_perm, const int32_t* pos,
                const float* topk_w, const void* shared_out, void* out,
                moe_stream_t stream);

/* Whole layer: router GEMM (or logits_override), top-K gating, alignment,
 * permute, grouped gate/up + SwiGLU, grouped down, shared FFN (when
 * n_shared > 0), combine.  out[T,H].  logits_override (nullable, fp32 [T,E])
 * replaces the router output for the routing decision; the router GEMM still
 * runs so its cost is kept.  stats_out (nullable, device int32[4]) receives
 * {P, E_active, bad_ids, 0}.  Nothing is synchronised.  The shared FFN runs
 * concurrently on a library stream forked from and joined back into `stream`
 * (see moe_set_shared_sms); the call is capturable into a CUDA graph, and
 * concurrent calls on one device are serialised while they enqueue. */
int moe_layer_forward(const moe_config_t* cfg, const void* x, const void* w_router,
                      const void* w13, const void* w2, const void* w13_shared,
                      const void* w2_shared, const float* logits_override, void* out,
                      void* workspace, size_t ws_bytes, int32_t* stats_out,
                      moe_stream_t stream);

/* moe_layer_forward with per-token dynamic K (see moe_route_k): token t is
 * routed to its k_per_token[t] top experts (0 = shared experts only);
 * NULL = K for every token.  Same workspace. */
int moe_layer_forward_k(const moe_config_t* cfg, const void* x, const void* w_router,
                        const void* w13, const void* w2, const void* w13_shared,
                        const void* w2_shared, const float* logits_override,
                        const int32_t* k_per_token, void* out, void* workspace,
                        size_t ws_bytes, int32_t* stats_out, moe_stream_t stream);

/* FP8 expert weights for the decode streaming path (talk notes, "Reduction
 * techniques": weight quantisation cuts the expert bytes loaded from HBM).
 * Row-wise E4M3 quantisation of w [rows, cols] (dtype 0 bf16, 1 fp32):
 *   scales[r] = max_c |w[r][c]| / 448 (1 for an all-zero row, fp32),
 *   q[r][c]   = E4M3(w[r][c] / scales[r]), nearest with ties to even,
 *               saturating at +-448 (E4M3: 1 sign, 4 exponent bits with bias
 *               7, 3 mantissa bits, no infinities).
 * cols must be a multiple of 16 (16-byte rows of codes).  Apply it to each
 * expert's w13 rows ([E*2I, H]) and w2 rows ([E*H, I]), and to the shared
 * FFN's; one block per row. */
int moe_quantize_fp8(int64_t rows, int cols, int dtype, const void* w, uint8_t* q,
                     float* scales, moe_stream_t stream);

/* moe_layer_forward_k with FP8 routed (and shared) expert weights: codes
 * w13_q [E,2I,H], w2_q [E,H,I] with row scales w13_s [E,2I], w2_s [E,H]
 * (shared likewise, [2*I_sh,H] / [H,I_sh] with [2*I_sh] / [H]); x, the router
 * and the output stay bf16 (cfg->dtype 0).  The codes stream from HBM and
 * every expert MMA is E4M3 x E4M3 with fp32 accumulation: the token rows
 * enter split exactly into two E4M3 terms with a power-of-two row scale
 * (moe_permute_e4m3x2), the SwiGLU activations are stored in f16 (they must
 * stay within its range) and split the same way on chip (about 8 significant
 * bits kept, bf16's precision); each output is multiplied by its weight
 * row's fp32 scale and its token row's scale.  Decode sizes only: the expert FFNs
 * must run as the fused kernel (at most 128 rows per routed expert and, with
 * shared experts, T <= 128); otherwise MOE_ERR_ARG.  H, I, S*I_s multiples of
 * 16.  Same workspace as moe_layer_forward. */
int moe_layer_forward_fp8(const moe_config_t* cfg, const void* x, const void* w_router,
                          const uint8_t* w13_q, const float* w13_s, const uint8_t* w2_q,
                          const float* w2_s, const uint8_t* w13_shared_q,
                          const float* w13_shared_s, const uint8_t* w2_shared_q,
                          const float* w2_shared_s, const float* logits_override,
                          const int32_t* k_per_token, void* out, void* workspace,
                          size_t ws_bytes, int32_t* stats_out, moe_stream_t stream);

/* moe_permute for the FP8-weight path (bf16 x, cfg->dtype 0): each permuted
 * row p < scalars[0] is split exactly into two E4M3 code rows and a power-of-
 * two scale, x[sorted_ids[p] / K] = x_scales[p] * (hi + lo), with hi the
 * row's codes x_codes[p] and lo the remainder's codes x_codes[P_max + p]
 * (P_max = moe_padded_rows_max(cfg)); x_scales[p] is the smallest power of
 * two with max|row| <= 448 x_scales[p].  The split is exact except where the
 * remainder is below E4M3's subnormal grid (under 2^-17 of the row's largest
 * magnitude), which rounds to the nearest grid value.  Padding rows get zero
 * codes and scale 1.  x_codes: [2 P_max, H] bytes (16-byte aligned); x_scales:
 * [P_max] floats.  The FP8 gate/up products then run as two E4M3 x E4M3
 * tensor-core products per weight tile (Blackwell kind::f8f6f4).  Errors:
 * MOE_ERR_ARG for a bad config, dtype != 0 or a null/misaligned pointer. */
int moe_permute_e4m3x2(const moe_config_t* cfg, const void* x, const int32_t* sorted_ids,
                       const int32_t* scalars, uint8_t* x_codes, float* x_scales,
                       moe_stream_t stream);

/* moe_grouped_ffn with FP8 routed expert weights (codes and row scales as
 * for moe_layer_forward_fp8); decode sizes only (at most 128 rows per
 * expert).  x_codes / x_scales as written by moe_permute_e4m3x2; `act` is
 * f16 scratch ([P_max, I]); y_perm is bf16 [P_max, H] and must not overlap
 * x_codes. */
int moe_grouped_ffn_fp8(const moe_config_t* cfg, const uint8_t* x_codes, const float* x_scales,
                        const uint8_t* w13_q, const float* w13_s, const uint8_t* w2_q,
                        const float* w2_s, const int32_t* offsets, void* act, void* y_perm,
                        void* workspace, size_t ws_bytes, moe_stream_t stream);

/* dense_ffn with FP8 weights (codes [2I,H] / [H,I] and row scales [2I] /
 * [H]), bf16 x and out; decode sizes only (T <= 128); workspace of
 * dense_ffn_fp8_workspace_size bytes (x's E4M3 hi/lo split, as in
 * moe_permute_e4m3x2, is written there). */
size_t dense_ffn_fp8_workspace_size(int T, int H, int I);
int dense_ffn_fp8(int T, int H, int I, const void* x, const uint8_t* w13_q, const float* w13_s,
                  const uint8_t* w2_q, const float* w2_s, void* out, void* workspace,
                  size_t ws_bytes, moe_stream_t stream);

/* Bytes of workspace dense_ffn needs for T tokens of width I (0 if invalid). */
size_t dense_ffn_workspace_size(int T, int H, int I, int dtype);

/* Dense SwiGLU FFN (DenseFA with I = K*I + S*I_s, DensePA with
 * I = E*I + S*I_s, or the shared experts): out[t] = W2 (silu(W1 x_t) * (W3 x_t)),
 * w13 [2I, H], w2 [H, I], same numerics as moe_grouped_ffn. */
int dense_ffn(int T, int H, int I, int dtype, const void* x, const void* w13,
              const void* w2, void* out, void* workspace, size_t ws_bytes,
              moe_stream_t stream);

/* Synchronise `stream`, then read and clear the workspace status words
 * (the caller's-stream kernels' and the concurrent shared FFN's).
 * Returns MOE_OK, MOE_ERR_TIMEOUT (a device wait ran out; the control words
 * are re-zeroed so the workspace stays usable), MOE_ERR_ARG (a fused expert
 * FFN launch was handed segment offsets that form more token chunks than its
 * tables hold -- offsets inconsistent with the configuration; it did no work)
 * or MOE_ERR_CUDA. */
int moe_check_status(void* workspace, moe_stream_t stream);

/* Device-side wait limit in nanoseconds for subsequent launches (default
 * 2e9 = 2 s; 0 restores the default).  Process-wide. */
void moe_set_wait_limit_ns(uint64_t ns);

/* Tuning: force the grouped GEMM's token-tile cap (tokens per MMA tile) to
 * 32, 64, 128 or 256 for subsequent launches; 0 (default) picks it from the
 * expected rows per expert, T*K/E.  Results are unchanged; only speed
 * differs.  Process-wide.  Returns MOE_ERR_ARG for other values. */
int moe_set_token_tile_cap(int n);

/* Tuning: how the grouped GEMM shares out the tiles left after its whole
 * waves of one tile per SM (or SM pair), for subsequent launches.
 *   1 (default): every whole wave data-parallel; the tiles of the last
 *     partial wave cut into equal k-slices, taken slice-major, so that tiles
 *     sharing a weight block or a token chunk stream the same slice together;
 *   0: stream-K over the last one to two waves, in contiguous ranges of
 *     (tile, k-iteration) units.
 * Split tiles are summed in a fixed order by the last contributor; results
 * agree up to fp32 summation order.  Process-wide.  MOE_ERR_ARG for other
 * values. */
int moe_set_split_tail(int mode);

/* 1 when moe_grouped_ffn / moe_layer_forward run this configuration's
 * expert FFN as one fused launch (gate/up + SwiGLU and down in a persistent
 * kernel with dynamic work fetching; decode-sized T*K/E), 0 when as two
 * grouped-GEMM launches.  moe_grouped_gate_up / moe_grouped_down always
 * launch the two GEMMs separately. */
int moe_ffn_fused(const moe_config_t* cfg);

/* Programmatic dependent launch (default on): each kernel may start its
 * prologue while the previous kernel on the stream drains, and waits for it
 * before touching its output.  0 turns it off (plain stream order) for
 * subsequent launches.  Process-wide; results are identical either way. */
void moe_set_programmatic_launch(int enable);

/* CTA pairs (default on): bf16 grouped/dense GEMMs at the 256-token tile
 * cap run on pairs of SMs (thread-block clusters of 2, 2-SM tensor-core MMA
 * with 256 weight rows per pair).  0 keeps single-SM tiles.  Process-wide;
 * results are identical up to fp32 summation order. */
void moe_set_cta_pairs(int enable);

/* Shared experts beside the routed experts.  With n_shared > 0,
 * moe_layer_forward launches the shared FFN first, on a second stream that
 * the library owns (one per device, created on first use), forked from and
 * joined back into the caller's stream with events; it runs concurrently with
 * routing and the routed experts on its own share of the SMs.  n = 0
 * (default): the share comes from a bytes/flops cost model; n > 0: n SMs
 * (rounded down to even, clamped to [2, SMs - 2]); n = -1: no side stream,
 * the shared FFN runs after the routed experts on the caller's stream.
 * Process-wide.  Results agree up to fp32 summation order (the grid size
 * sets the K-splits).  Returns MOE_ERR_ARG for n < -1. */
int moe_set_shared_sms(int n);

/* SMs the shared experts of this configuration get under the current
 * setting (0: they run serially, or there are none). */
int moe_shared_sms(const moe_config_t* cfg);

/* Tensor parallelism over the expert intermediate dimension I (talk notes,
 * "Demystifying the Mixture of Experts Serving Tax": under TP the buckets of
 * the Balls-Bins-Buckets model are the n_tp GPUs; "Key findings" 3: the
 * AllReduce that follows the MoE block).  Rank r of n holds, for every routed
 * expert and for the shared FFN, the gate rows [r*I/n, (r+1)*I/n) of W1, the
 * same rows of W3 and the same columns of W2; the router weights are whole on
 * every rank, so every rank routes identically.  The sum over ranks of the
 * partial outputs is the layer output.
 *
 * moe_tp_shard: rank `rank`'s slice of w13 [E, 2I, H] / w2 [E, H, I] (dtype
 * 0 bf16, 1 fp32) into caller-owned w13_local [E, 2I/n, H] (gate slice, then
 * up slice, per expert) and w2_local [E, H, I/n]; E = 1 slices one dense FFN
 * (the shared experts).  Device-to-device copies enqueued on `stream`.
 * MOE_ERR_ARG unless I % n_ranks == 0 and 0 <= rank < n_ranks. */
int moe_tp_shard(int E, int H, int I, int dtype, int rank, int n_ranks, const void* w13,
                 const void* w2, void* w13_local, void* w2_local, moe_stream_t stream);

/* moe_layer_forward_k on one rank's slice (cfg->I = I/n, cfg->n_shared *
 * cfg->I_shared = the shared FFN's I_sh/n): the same routing, the same
 * kernels, but the combine writes the fp32 sums unrounded into out_partial
 * [T, H] (fp32), ready for the all-reduce.  Same workspace as
 * moe_layer_forward for cfg. */
int moe_layer_forward_partial(const moe_config_t* cfg, const void* x, const void* w_router,
                              const void* w13, const void* w2, const void* w13_shared,
                              const void* w2_shared, const float* logits_override,
                              const int32_t* k_per_token, float* out_partial, void* workspace,
                              size_t ws_bytes, int32_t* stats_out, moe_stream_t stream);

/* TP over I with the all-reduce overlapped with the down projection (talk
 * notes, "Key findings" 3: the AllReduce that follows the MoE block).  The
 * layer on this rank's slice (cfg as for moe_layer_forward_partial) in two
 * parts, so that the all-reduce of one block of output features can run
 * while the down projection of the next block computes:
 *   moe_layer_forward_partial_front: routing, permute, the routed experts'
 *     gate/up + SwiGLU and the whole shared FFN, all into the workspace (the
 *     shared experts' side stream is joined back before it returns);
 *   moe_layer_forward_partial_down: for output features
 *     [chunk * H/n_chunks, (chunk + 1) * H/n_chunks): the routed experts' down
 *     projection and the combine (fp32 sums in ascending k, the shared output
 *     added last, unrounded) into part [T, H/n_chunks] fp32, contiguous and
 *     ready for that block's all-reduce.
 * Call front once, then down for every chunk, on the same stream and
 * workspace (front's results stay there until the next front call).  The sum
 * over ranks of the parts, placed side by side, is the layer output (see
 * moe_tp_gather).  Needs the two-launch expert FFN (moe_ffn_fused(cfg) == 0:
 * more than 128 rows per expert); H/n_chunks a multiple of 8 (bf16) or 4
 * (fp32).  MOE_ERR_ARG otherwise.  Same workspace size as moe_layer_forward. */
int moe_layer_forward_partial_front(const moe_config_t* cfg, const void* x, const void* w_router,
                                    const void* w13, const void* w13_shared, const void* w2_shared,
                                    const float* logits_override, const int32_t* k_per_token,
                                    void* workspace, size_t ws_bytes, int32_t* stats_out,
                                    moe_stream_t stream);
int moe_layer_forward_partial_down(const moe_config_t* cfg, const void* w2, int chunk, int n_chunks,
                                   float* part, void* workspace, size_t ws_bytes, moe_stream_t stream);

/* The layer output from the all-reduced column blocks of
 * moe_layer_forward_partial_down: out[t][c * Hc + j] = parts[c][t * Hc + j]
 * rounded once to dtype (0 bf16, 1 fp32), Hc = H / n_chunks.  `parts` is a
 * HOST array of n_chunks (1..16) device pointers to [T, Hc] fp32 blocks,
 * 16-byte aligned; Hc % 4 == 0. */
int moe_tp_gather(int n_chunks, const float* const* parts, int T, int H, int dtype, void* out,
                  moe_stream_t stream);

/* The reduction of the ranks' partial outputs: out[i] = sum over r of
 * parts[r][i] for i < count, fp32 in rank order, one rounding to dtype (0
 * bf16, 1 fp32).  `parts` is a HOST array of n_parts (1..16) device
 * pointers, each 16-byte aligned; they may point into other GPUs' memory
 * mapped into this one (peer access), which the kernel reads with plain
 * loads.  With n_parts = 1 it rounds an all-reduced sum.  count % 4 == 0.
 * The caller orders the writes of every part before this call (on other
 * GPUs: an event or a barrier) and keeps the parts alive until it ends. */
int moe_tp_reduce(int n_parts, const float* const* parts, long long count, int dtype, void* out,
                  moe_stream_t stream);

/* Test hook: when nonzero, the next GEMM or fused-FFN launch withholds one
 * operand load (the first load of block 0, or of work item 0 in the fused
 * FFN), so the waits that depend on it run out and report MOE_ERR_TIMEOUT
 * through moe_check_status().  Cleared after one launch. */
void moe_debug_withhold_first_load(int enable);

/* Number of kernels this library launched since load (all entry points). */
uint64_t moe_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
