/*
 * moe_split.h -- CPU/GPU split of the MoE layer for models whose experts do
 * not all fit in GPU memory, after FIDDLER (K. Kamahori et al., "FIDDLER:
 * CPU-GPU orchestration for fast inference of Mixture-of-Experts models", as
 * summarised on aibr.jp/archives/173321):
 *   - offline, the experts hit most often in a profiling run are placed in
 *     GPU memory up to a budget (§ "3.中核となる技術的要素": placement from
 *     offline profiling of hit rates);
 *   - at run time, for each expert a batch routes tokens to but that is not
 *     resident, the runtime compares the expected latency of computing it on
 *     the host with that of copying its weights to the GPU and computing it
 *     there, from the batch's token count, and takes the cheaper (same
 *     section: dynamic scheduling from token counts and expected latencies);
 *   - host experts run in a dedicated CPU kernel using AVX512_BF16 dot
 *     products where the CPU has them (same section, and § "2.先行研究との
 *     差別化ポイント"); on CPUs with AMX, bf16 tile products.
 *
 * Everything else is the layer of moe.h: the GPU routes the batch, permutes
 * it by slot and runs the resident and copied experts in its grouped GEMMs;
 * the host's rows join the combine.  bf16 only.  The conventions of moe.h
 * apply, with the exceptions stated at moe_split_forward (it synchronises its
 * stream, once or twice, and reads and writes host memory).
 *
 * Process-wide state: the host functions share one thread pool (one thread
 * per hardware thread, created on first use, one pool per process: a child
 * made by fork() builds its own; calls from several threads take turns), and
 * the first host call asks Linux once for the AMX tile state where the CPU
 * has AMX.
 */
#ifndef MOE_B200_SPLIT_H
#define MOE_B200_SPLIT_H

#include "moe.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Where one expert runs for one batch (moe_split_plan). */
typedef enum {
    MOE_SPLIT_IDLE = 0,      /* no token of the batch routes to it */
    MOE_SPLIT_RESIDENT = 1,  /* its weights are in GPU memory: GPU */
    MOE_SPLIT_STAGED = 2,    /* its weights are copied to a staging slot: GPU */
    MOE_SPLIT_CPU = 3        /* computed on the host */
} moe_split_where;

/* How moe_split_forward treats active experts that are not resident. */
typedef enum {
    MOE_SPLIT_POLICY_DYNAMIC = 0,   /* moe_split_plan with the given costs */
    MOE_SPLIT_POLICY_ALL_CPU = 1,   /* always the host */
    MOE_SPLIT_POLICY_ALL_STAGED = 2,/* always copy the weights (while staging
                                       slots last; the rest on the host) */
    MOE_SPLIT_POLICY_BALANCED = 3   /* moe_split_plan_balanced with the given
                                       costs */
} moe_split_policy;

/*
 * The runtime's latency model, in microseconds, for an expert that is not
 * resident and receives n tokens:
 *   cpu(n) = cpu_us + cpu_us_per_token * n            (host kernel)
 *   gpu(n) = xfer_us + gpu_us + gpu_us_per_token * n  (copy its weights over
 *                                                      the host link, then run
 *                                                      it on the GPU)
 * moe_split_calibrate (below) measures these on the running system.
 */
typedef struct {
    double cpu_us, cpu_us_per_token;
    double xfer_us, gpu_us, gpu_us_per_token;
} moe_split_costs;

/*
 * Offline placement.  hits: host int64 [E], the number of assignments each
 * expert received in a profiling run.  resident: host int32 [E] out: 1 for
 * the `budget` experts with the most hits (equal hits: lower index first), 0
 * for the others.  0 <= budget <= E.
 * Errors: MOE_ERR_INVALID_ARG for NULL pointers, E < 1, E > 256, a budget
 * outside [0, E] or a negative hit count.
 */
MOE_API moe_status moe_split_place(const int64_t* hits, int E, int budget, int32_t* resident);

/*
 * Runtime plan of one batch.  counts: host int32 [E], tokens routed to each
 * expert; resident: host int32 [E] (0/1); where: host int32 [E] out.
 *   where[e] = IDLE      if counts[e] == 0
 *            = RESIDENT  else if resident[e]
 *            = STAGED    else if gpu(n) < cpu(n) (strictly) and e is among
 *                        the n_stage such experts with the largest saving
 *                        cpu(n) - gpu(n) (equal savings: lower index first)
 *            = CPU       otherwise
 * Errors: MOE_ERR_INVALID_ARG for NULL pointers, E outside [1, 256],
 * n_stage < 0 or a negative count.
 */
MOE_API moe_status moe_split_plan(const int32_t* counts, const int32_t* resident, int E,
                                  const moe_split_costs* costs, int n_stage, int32_t* where);

/*
 * The balanced plan: the same latency model, with the host and the
 * host-to-GPU link counted as two resources that work at the same time (an
 * extension beyond the page, whose rule weighs each expert on its own).  The
 * non-resident experts of a batch then cost
 *   max( sum of cpu(n) over the experts left on the host,
 *        sum of gpu(n) over the staged experts )
 * Candidates (active, not resident) are ranked by cpu(n) / gpu(n), largest
 * first (gpu(n) <= 0 first; equal ratios: lower index first), and the first
 * j of them are staged, j in 0..min(n_stage, #candidates) minimising that
 * maximum (equal maxima: the smaller j).  Sums run in rank order.  Arguments
 * and errors as moe_split_plan.
 */
MOE_API moe_status moe_split_plan_balanced(const int32_t* counts, const int32_t* resident,
                                           int E, const moe_split_costs* costs, int n_stage,
                                           int32_t* where);

/*
 * Host expert weights.  moe_host_pack_weights converts host bf16 master
 * weights W_g, W_u [E,H,I] and W_d [E,I,H] (row-major, as for
 * moe_pack_weights) into the host kernel's layout: per expert a block of
 * moe_host_packed_size(H, I) bytes (= 3*H*I*2) holding, for each 16-column
 * block c of W_g, then of W_u, then of W_d, the block's rows in pairs
 * (rows 2p, 2p+1 of column c*16+i at [c][p][i][0..1]), so that the kernel
 * streams each column block contiguously and multiplies row pairs with
 * bf16 pair dot products.  H and I multiples of 64.
 * Errors: MOE_ERR_INVALID_ARG for bad sizes or NULL pointers.
 */
MOE_API size_t moe_host_packed_size(int H, int I);
MOE_API moe_status moe_host_pack_weights(int E, int H, int I, const uint16_t* Wg,
                                         const uint16_t* Wu, const uint16_t* Wd, void* packed);

/* Instruction-set path the host kernel takes on this CPU: AMX bf16 tiles
 * (where the CPU has them and the OS grants the process the tile state),
 * else AVX512_BF16 pair dot products, else portable C++. */
enum { MOE_HOST_ISA_PORTABLE = 0, MOE_HOST_ISA_AVX512_BF16 = 1, MOE_HOST_ISA_AMX_BF16 = 2 };
MOE_API int moe_host_isa(void);

/*
 * One expert on the host, for n rows (tokens):
 *   h[r] = bf16( SiLU(x[r] W_g) * (x[r] W_u) )    fp32 sums, SiLU(z) = z/(1+e^-z)
 *   y[r] = bf16( w[r] * (h[r] W_d) )
 * the same quantities (and bf16 roundings of h and y) as the GPU's grouped
 * FFN.  All pointers are host memory:
 *   weights  one expert's block from moe_host_pack_weights
 *   x        bf16 [n][H];  w  f32 [n];  h  bf16 [n][I] (out, scratch)
 *   y        bf16 [n][H] (out)
 * threads: worker threads of the library's host pool to use (0 = all; the
 * pool has one thread per hardware thread and is created on first use).
 * flags: MOE_HOST_FLAG_PORTABLE takes the portable path, MOE_HOST_FLAG_NO_AMX
 * the AVX512_BF16 path, even where a faster one is available.  All paths sum
 * in fp32; their results may differ in the last bits (products summed in a
 * different order).
 * Errors: MOE_ERR_INVALID_ARG for bad sizes or NULL pointers.
 */
enum { MOE_HOST_FLAG_PORTABLE = 1, MOE_HOST_FLAG_NO_AMX = 2 };
typedef struct {
    int H, I, n;
    const void* weights;
    const uint16_t* x;
    const float* w;
    uint16_t* h;
    uint16_t* y;
    int threads;
    int flags;
} moe_host_ffn_args;

MOE_API moe_status moe_host_expert_ffn(const moe_host_ffn_args* args);

/*
 * The split layer, for one batch x [T,H], logits [T,E]:
 *   1. GPU: route (a1) into ids, w; copy ids and w to the host; wait.
 *   2. host: counts, then the plan (policy: moe_split_plan for DYNAMIC,
 *      moe_split_plan_balanced for BALANCED); if the plan puts any expert on
 *      the host, x is copied to the host (a second wait, for that copy).
 *   3. GPU: copy each STAGED expert's packed weights into a staging slot;
 *      map every assignment to a slot (0 = host, 1..S = the resident experts
 *      in ascending index, S+1.. = staged experts in ascending index) and
 *      permute by slot (a2); run the grouped FFN (a3..a6) of the resident
 *      slots, then, after the copies, of the staged slots.
 *   4. host (while the GPU runs): each CPU expert's rows with
 *      moe_host_expert_ffn; the rows, in ascending flat index t*k+j (the
 *      order the stable permutation gives slot 0), are copied into the
 *      permuted output's first rows.
 *   5. GPU: combine (a7): out[t] = sum_j y(t,j) in j order.
 * The result is the layer of moe_forward for the same inputs; rows computed
 * on the host may differ from the GPU's in the last bits of bf16.
 *
 * Arguments:
 *   x, logits, out     device, as for moe_forward
 *   resident           host int32 [E] (moe_split_place); S = its number of 1s
 *   resident_packed    device, moe_pack_weights layout of the S resident
 *                      experts in ascending index (E = S); NULL when S = 0
 *   stage_packed       device, moe_pack_weights layout with n_stage experts
 *                      (overwritten by the copies); NULL when n_stage = 0
 *   host_packed        host (page-locked for asynchronous copies): for each
 *                      expert e in turn, the moe_pack_weights output of that
 *                      expert alone (E = 1, moe_packed_weights_size(MOE_BF16,
 *                      1, H, I) bytes each): the source of the copies, so that
 *                      set-up can pack one expert at a time
 *   host_weights       host, moe_host_pack_weights layout of all E experts
 *   costs              latency model (DYNAMIC, BALANCED); may be NULL otherwise
 *   where              optional host int32 [E] out: the plan that ran
 *   copy_stream, copy_event  optional: the weight copies run on copy_stream
 *                      and copy_event orders the staged FFN after them, so
 *                      the resident experts' GEMMs overlap the copies (both
 *                      NULL: the copies run on `stream`)
 *   host_threads       as moe_host_ffn_args.threads
 *   ws                 device workspace, moe_split_workspace_size bytes
 *   host_ws            host workspace (page-locked), moe_split_host_workspace_size
 *                      bytes; it must stay untouched until the stream has
 *                      finished the call
 * Calls that share staging slots or workspaces must be ordered: issue them
 * on one stream (each call's synchronisation then covers the previous one's
 * use of the slots).
 * Exceptions to moe.h's conventions: this call synchronises `stream` (after
 * step 1: the plan needs the batch's routing; and for the copy of x when a
 * host expert needs it) and computes on the calling thread and the host
 * pool; it returns once steps 3-5 are enqueued.
 * Errors: as moe_forward; MOE_ERR_UNSUPPORTED for S + n_stage + 1 > 256.
 */
typedef struct {
    int T, k, E, H, I;
    int block_m;                 /* 0 selects 16 */
    const void* x;
    const float* logits;
    void* out;
    const int32_t* resident;
    const void* resident_packed;
    void* stage_packed;
    int n_stage;
    const void* host_packed;
    const void* host_weights;
    const moe_split_costs* costs;
    int policy;                  /* a moe_split_policy */
    int32_t* where;
    int32_t* status;             /* device status word, may be NULL */
    moe_stream_t copy_stream;
    moe_event_t copy_event;
    int host_threads;
} moe_split_args;

/*
 * Measures the latency model on the running system (a set-up step; it
 * synchronises `stream` and takes a few times the cost of one expert):
 *   cpu_us, cpu_us_per_token  from moe_host_expert_ffn on 1 and n_max rows
 *                             (zero inputs; the best of a few runs each)
 *   xfer_us                   one copy of 3*H*I*2 bytes from host_src
 *                             (page-locked) to dev_dst (device)
 *   gpu_us, gpu_us_per_token  0: the GPU streams an expert's weights ~100x
 *                             faster than the host link carries them, so the
 *                             copy dominates the GPU side
 * host_weights: one expert's block from moe_host_pack_weights; host_ws: at
 * least moe_split_host_workspace_size(n_max, 1, H, I) bytes of host memory.
 * Errors: MOE_ERR_INVALID_ARG for bad sizes or NULL pointers; MOE_ERR_CUDA.
 */
MOE_API moe_status moe_split_calibrate(int H, int I, int n_max, const void* host_weights,
                                       const void* host_src, void* dev_dst, void* host_ws,
                                       size_t host_ws_bytes, int host_threads,
                                       moe_stream_t stream, moe_split_costs* costs);

MOE_API size_t moe_split_workspace_size(int T, int k, int E, int S, int n_stage, int H, int I,
                                        int block_m);
MOE_API size_t moe_split_host_workspace_size(int T, int k, int H, int I);
MOE_API moe_status moe_split_forward(const moe_split_args* args, void* ws, size_t ws_bytes,
                                     void* host_ws, size_t host_ws_bytes, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_SPLIT_H */
