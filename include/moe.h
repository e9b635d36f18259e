/*
 * moe.h -- C ABI of a B200-native (sm_100a) fused Mixture-of-Experts layer.
 *
 * The layer is the "fused MoE" operation: token routing, data reordering and
 * the experts' computation as one batched GPU operation instead of a loop over
 * experts ("Az AWS új MoE-optimalizációkkal gyorsítja a SageMaker AI-t",
 * § "A fused MoE a számítási folyamat több lépését egyesíti").  For tokens
 * x [T,H] and fp32 router logits [T,E]:
 *
 *   ids, w    = top-k of each logits row, softmax over the selected logits
 *   permute   = group the T*k assignments by expert, padded to block_m rows
 *   h         = SiLU(x W_g[e]) * (x W_u[e])          per assignment (SwiGLU)
 *   y         = w * (h W_d[e])
 *   out[t]    = sum over the token's k assignments of y
 *
 * Conventions for every entry point
 *   - Pointers named as device buffers are device memory of the current CUDA
 *     device; the caller allocates and owns every buffer.  The library never
 *     allocates, frees or synchronises, and enqueues work only on the given
 *     stream (NULL = the legacy default stream).
 *   - Argument errors are returned synchronously (MOE_ERR_INVALID_ARG,
 *     MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE) and nothing is launched.
 *   - A failed launch returns MOE_ERR_CUDA.
 *   - Faults found on the device (a bounded wait that ran out, an expert id out
 *     of range) are written to a device status word (int32, 0 = OK, else a
 *     moe_status code); the first fault wins.  moe_check_status reads it.
 *   - Device pointers must be 16-byte aligned; all layouts are row-major.
 *   - T = 0 is a valid no-op.
 *   - Limits: 1 <= k <= E <= 256; H and I multiples of 64; block_m a multiple
 *     of 16 (the token granularity of the tensor-core tiles).
 *   - Process-wide state is limited to two things: the per-device opt-in of
 *     the GEMM kernels to more than 48 KB of shared memory (set on the first
 *     launch on each device, read-only afterwards), and the fixed scratch
 *     array of moe_align_permute_noalloc (see its entry).  The CPU/GPU split
 *     of moe_split.h adds its host thread pool (see there).  Apart from
 *     moe_align_permute_noalloc, calls on different streams with separate
 *     buffers may run concurrently.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle types as cudaStream_t / cudaEvent_t, without the CUDA headers. */
typedef struct CUstream_st* moe_stream_t;
typedef struct CUevent_st* moe_event_t;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,  /* bad pointer, size or alignment */
    MOE_ERR_UNSUPPORTED = 2,  /* valid request outside the supported limits */
    MOE_ERR_WORKSPACE = 3,    /* workspace missing or too small */
    MOE_ERR_CUDA = 4,         /* a CUDA call failed */
    MOE_ERR_TIMEOUT = 5,      /* a bounded device wait ran out (device status) */
    MOE_ERR_DEVICE = 6        /* a device-side check failed, e.g. id >= E */
} moe_status;

typedef enum {
    MOE_BF16 = 0,      /* bf16 weights and activations, fp32 accumulation */
    MOE_FP8_E4M3 = 1   /* e4m3 weights (one scale per expert matrix) and
                          activations (one dynamic scale per tensor), fp32
                          accumulation, bf16 output */
} moe_dtype;

/* Human-readable name of a status code (static string, never NULL). */
MOE_API const char* moe_status_string(moe_status s);

/* Version string of the library. */
MOE_API const char* moe_version(void);

/*
 * a1. Router top-k.  Router selection of the few experts each token activates
 * ("Amazon SageMaker AIにおけるMixture-of-Expertsカーネル最適化の深掘り",
 * § "Mixture-of-Experts (MoE) モデルの原理と推論における課題").
 *   logits  device f32 [T,E]    router logits
 *   ids     device i32 [T,k]    out: selected experts, larger logit first;
 *                               equal logits (and -0/+0) lower index first;
 *                               NaN ranks below every number
 *   w       device f32 [T,k]    out: softmax over the selected logits
 * Errors: T < 0, k < 1, k > E, E > 256, NULL pointers -> MOE_ERR_INVALID_ARG.
 */
MOE_API moe_status moe_route_topk(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                          moe_stream_t stream);

/*
 * a2. Token permutation ("data reordering", same section of the first page
 * cited above): a stable, atomic-free counting sort of the A = T*k assignments
 * (flat index f = t*k + j) by expert.
 *   ids        device i32 [T,k]          expert of each assignment
 *   counts     device i32 [E]            out: c_e
 *   offsets    device i32 [E+1]          out: o_0 = 0,
 *                                        o_{e+1} = o_e + ceil(c_e/block_m)*block_m
 *   sorted_ids device i32 [capacity]     out: sorted_ids[o_e + r] = the r-th
 *                                        smallest f routed to e; every other
 *                                        slot (pads and the tail) = -1
 *   inv_perm   device i32 [T*k]          out: slot of assignment f
 *   tiles      device i32 [capacity/block_m] out: expert owning each block_m
 *                                        rows, -1 past the last
 *   num_tiles  device i32 [1]            out: o_E / block_m
 *   capacity   >= moe_permute_capacity(T, k, E, block_m)
 *   ws         device scratch of moe_align_permute_workspace_size() bytes
 * Errors: invalid sizes or NULL -> MOE_ERR_INVALID_ARG; capacity too small or
 * ws too small -> MOE_ERR_WORKSPACE.  An id outside [0,E) is reported in
 * the status word given to moe_forward/moe_grouped_ffn, not here (it is
 * skipped, and the results are then incomplete).
 */
MOE_API int moe_permute_capacity(int T, int k, int E, int block_m);
MOE_API size_t moe_align_permute_workspace_size(int T, int k, int E);
MOE_API moe_status moe_align_permute(const int32_t* ids, int T, int k, int E, int block_m,
                             int32_t* counts, int32_t* offsets, int32_t* sorted_ids,
                             int32_t* inv_perm, int32_t* tiles, int32_t* num_tiles,
                             int capacity, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * The same permutation for callers that cannot allocate device memory or pass
 * a workspace (for example a plugin of an inference runtime that provides no
 * workspace, or a thread that must not allocate while it enqueues work).  The
 * pages have no counterpart of this entry point; it is a deployment aid.
 * Arguments and outputs are those of moe_align_permute without ws/ws_bytes.
 * Its scratch is a fixed 256 KB device array inside the library (65536
 * int32 counters, held on every GPU that loads the library until exit), so
 * for T*k > 2048, ceil(T*k/512) * E must not exceed 65536; larger problems return
 * MOE_ERR_WORKSPACE with nothing launched.  The first call on a device looks
 * up the array's address for that device; make it before any stream capture.
 * All calls share the array: each overwrites what it reads, but calls that
 * overlap on the GPU race.
 */
MOE_API moe_status moe_align_permute_noalloc(const int32_t* ids, int T, int k, int E,
                                             int block_m, int32_t* counts, int32_t* offsets,
                                             int32_t* sorted_ids, int32_t* inv_perm,
                                             int32_t* tiles, int32_t* num_tiles, int capacity,
                                             moe_stream_t stream);

/*
 * One-time weight packing (not part of the timed layer).  Converts master
 * weights W_g, W_u [E,H,I] and W_d [E,I,H] (device bf16) into the K-major
 * layout the tensor-core GEMMs stream:
 *   W_gu [E][2I][H]: packed row r of expert e holds, for q = r/32, w = r%32,
 *        column j = 16q + (w%16) of W_g (w < 16) or of W_u (w >= 16)
 *   W_dn [E][H][I]:  W_d transposed
 * in bf16 (MOE_BF16) or e4m3 (MOE_FP8_E4M3).  For FP8 each expert matrix gets
 * scale s = amax/448 (amax = 0 gives 1), codes = round-to-nearest-even of
 * w/s saturated to +-448, and scales [E][3] = (s_g, s_u, s_d) is written
 * (device f32); for bf16 scales may be NULL.
 * Errors: MOE_ERR_INVALID_ARG for bad sizes/pointers.
 */
MOE_API size_t moe_packed_weights_size(moe_dtype dtype, int E, int H, int I);
MOE_API moe_status moe_pack_weights(moe_dtype dtype, int E, int H, int I, const void* Wg,
                            const void* Wu, const void* Wd, void* packed, float* scales,
                            moe_stream_t stream);

/*
 * Multi-LoRA adapters (bf16 layers).  Several fine-tuned variants of one MoE
 * model share the GPU, each token naming its adapter ("Amazon SageMaker AIに
 * おけるMixture-of-Expertsカーネル最適化の深掘り", § "SageMakerを活用した
 * MoEモデルのデプロイと性能向上戦略": multi-LoRA serving of MoE models).  The
 * pages give no shapes; this library's definition: adapter a has, for every
 * expert e, rank-r pairs that add s_a A B to each expert matrix the token
 * meets:
 *   g = x W_g + s_a (x A_g) B_g,  u likewise,  h = SiLU(g) * u,
 *   y = h W_d + s_a (h A_d) B_d
 * with A_g, A_u [n][E][H][r], B_g, B_u [n][E][r][I], A_d [n][E][I][r],
 * B_d [n][E][r][H] (device bf16, row-major) and n * r <= 64.
 * moe_pack_lora lays them out once (moe_packed_lora_size bytes, device,
 * 16-byte aligned).  The layer computes each shrink (x A, h A, for all
 * adapters at once, kept only in the token's own adapter's columns and
 * scaled) as one extra 128-row weight tile per expert, and each expand
 * (... B) as one or two extra k-blocks of the base GEMMs.
 * Errors: MOE_ERR_INVALID_ARG for bad sizes or pointers, MOE_ERR_UNSUPPORTED
 * for n * r > 64 or E > 256.
 */
typedef struct {
    int n_adapters;             /* n >= 1 */
    int rank;                   /* r >= 1, n * r <= 64 */
    const int32_t* adapter;     /* device i32 [T]: the token's adapter, -1 = none */
    const void* packed;         /* device, from moe_pack_lora */
    const float* scale;         /* device f32 [n]: s_a */
} moe_lora_args;

MOE_API size_t moe_packed_lora_size(int E, int H, int I, int n_adapters, int rank);
MOE_API moe_status moe_pack_lora(int E, int H, int I, int n_adapters, int rank, const void* Ag,
                                 const void* Bg, const void* Au, const void* Bu, const void* Ad,
                                 const void* Bd, void* packed, moe_stream_t stream);

/*
 * a3-a6. Grouped expert FFN over the permuted assignments: the expert GEMMs
 * A[M,K] x B[K,N] ("Ingénierie de kernels Mixture-of-Experts sur Amazon
 * SageMaker AI"), computed with the expert-weight rows in the tensor core's
 * M slot and the tokens in N (the operand swap of "A mátrixok felcserélése
 * jobban kihasználja a Hopper GPU-kat", re-derived for tcgen05), with the
 * gather of the token rows, the SiLU*up and the routing-weight epilogues
 * fused in:
 *   X_p       = x[sorted_ids[p] / k]      zero for pads; FP8: the e4m3 codes
 *                                         of x with s_x = amax(x)/448, made in
 *                                         token order.  Tiles of up to 64 tokens
 *                                         gather X_p in the gate/up GEMM's
 *                                         operand loads; larger tiles read rows
 *                                         a gather kernel lays out first
 *   h[p]      = SiLU(X_p W_g[e]) * (X_p W_u[e])   (bf16; FP8: then quantised
 *                                                  with s_h)
 *   y_perm[p] = w[sorted_ids[p]] * (h[p] W_d[e])   (bf16; 0 for pads)
 * for every row p of expert e's block.  Inputs come from moe_align_permute.
 * FP8 activations are coded as RNE_sat(v * (1/s)) with the fp32 reciprocal of
 * their scale (a code may differ by one step from RNE(v / s) when v / s lies
 * within an fp32 ulp of a rounding midpoint); weights use v / s exactly.
 * max_ctas > 0 caps the persistent grid (0 = one CTA per SM).
 * Errors: MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED / MOE_ERR_WORKSPACE
 * synchronously; device faults in *status (or, if status is NULL, in the
 * first int32 of ws).
 */
typedef struct {
    moe_dtype dtype;
    int T, k, E, H, I;
    int block_m;                /* padding the permutation used */
    int capacity;               /* rows of sorted_ids / y_perm */
    const void* x;              /* device bf16 [T,H], token order */
    const float* w;             /* device f32 [T*k] routing weights */
    const int32_t* counts;      /* device i32 [E] */
    const int32_t* offsets;     /* device i32 [E+1] */
    const int32_t* sorted_ids;  /* device i32 [capacity] */
    const void* packed;         /* device, from moe_pack_weights */
    const float* scales;        /* device f32 [E][3] (FP8), NULL for bf16 */
    void* y_perm;               /* device bf16 [capacity,H], out */
    int32_t* status;            /* device i32 status word, may be NULL */
    int max_ctas;               /* 0 = one CTA per SM */
} moe_ffn_args;

MOE_API size_t moe_grouped_ffn_workspace_size(moe_dtype dtype, int T, int k, int E, int H, int I,
                                      int block_m);
MOE_API moe_status moe_grouped_ffn(const moe_ffn_args* args, void* ws, size_t ws_bytes,
                           moe_stream_t stream);

/*
 * a7. Weighted top-k combine back to token order (the aggregation of the
 * experts' outputs, "FP8 esetén a Triton backend bizonyult gyorsabbnak"):
 *   out[t] = sum_{j=0..k-1} y_perm[inv_perm[t*k+j]]   (fp32, in j order)
 *   y_perm  device bf16 [*, H], inv_perm device i32 [T*k], out device bf16 [T,H]
 * Errors: MOE_ERR_INVALID_ARG.
 */
MOE_API moe_status moe_combine(const void* y_perm, const int32_t* inv_perm, int T, int k, int H,
                       void* out, moe_stream_t stream);

/*
 * The whole layer in one call: a1 -> a2 -> a3..a6 -> a7 on one stream, with
 * every intermediate carved from ws (size from moe_forward_workspace_size).
 *   x        device bf16 [T,H]; logits device f32 [T,E]
 *   packed / scales  from moe_pack_weights
 *   out      device bf16 [T,H]
 *   ids, w   optional device outputs [T,k] (NULL: kept in ws)
 *   status   optional device status word (NULL: the first int32 of ws)
 *   block_m  0 selects 16
 *   events / n_events  optional: if non-NULL, events[i] is recorded on the
 *            stream after stage i (0 entry, 1 route+permute, 2 a3: the FP8
 *            quantisation of x and, for large token tiles, the gather of the
 *            token rows (empty when the gate/up GEMM gathers them itself and
 *            the route kernel quantises x), 3 gate/up GEMM, 4 h quant (FP8),
 *            5 down GEMM, 6 combine or finalize); used to time the stages.
 *            n_events must be 7 when events is non-NULL.
 *   combine  a moe_combine_mode (0 = auto).
 *   lora     optional adapters (see moe_lora_args); the workspace from
 *            moe_forward_workspace_size always has room for their shrink
 *            outputs.
 * Errors: as for the stages above.
 */
/* How moe_forward forms out[t] = sum_j y(t, j) (a7). */
typedef enum {
    MOE_COMBINE_AUTO = 0,          /* the library's choice: currently the
                                      deterministic form, which measured as fast
                                      as the fused one on B200 */
    MOE_COMBINE_DETERMINISTIC = 1, /* the down GEMM writes y_perm rows (bf16); a
                                      combine kernel sums each token's k rows in
                                      fp32 in j order: bit-reproducible */
    MOE_COMBINE_FUSED = 2          /* the down GEMM's epilogue adds w*y (fp32)
                                      into a token-order accumulator, converted
                                      to bf16 at the end: no y_perm round trip,
                                      but the summation order follows the
                                      schedule, so the last bit may vary */
} moe_combine_mode;

typedef struct {
    moe_dtype dtype;
    int T, k, E, H, I;
    int block_m;
    const void* x;
    const float* logits;
    const void* packed;
    const float* scales;
    void* out;
    int32_t* ids;
    float* w;
    int32_t* status;
    int max_ctas;
    moe_event_t* events;
    int n_events;
    int combine;               /* a moe_combine_mode */
    const moe_lora_args* lora; /* optional multi-LoRA adapters (bf16 only), NULL = none */
} moe_forward_args;

MOE_API size_t moe_forward_workspace_size(moe_dtype dtype, int T, int k, int E, int H, int I,
                                  int block_m);
MOE_API moe_status moe_forward(const moe_forward_args* args, void* ws, size_t ws_bytes,
                       moe_stream_t stream);

/*
 * Reads a device status word: synchronises the stream, then returns
 * MOE_OK or the code the device recorded (MOE_ERR_TIMEOUT, MOE_ERR_DEVICE).
 * Errors: MOE_ERR_INVALID_ARG for NULL, MOE_ERR_CUDA if the copy fails.
 */
MOE_API moe_status moe_check_status(const int32_t* dev_status, moe_stream_t stream);

/*
 * Failure-detection self-test: launches one CTA that waits on a barrier no
 * one arrives at, with a limit of timeout_us microseconds (1..1000000); when
 * it runs out the kernel records MOE_ERR_TIMEOUT in *dev_status and returns.
 * The same bounded-wait routine guards every wait in the GEMM pipeline.
 */
MOE_API moe_status moe_selftest_wait_timeout(int32_t* dev_status, int timeout_us, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
