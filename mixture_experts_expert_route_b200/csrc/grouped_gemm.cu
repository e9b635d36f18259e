// grouped_gemm.cu -- a4 (gate/up GEMM + SiLU*up, with the gather of x fused
// into its operand loads) and a6 (down GEMM + routing weight, optionally with
// the top-k combine fused into its epilogue) as one persistent,
// warp-specialised tcgen05 kernel.
//
// The expert GEMM is A[M,K] x B[K,N] with M = tokens, K = hidden and N = the
// expert's output size ("Ingénierie de kernels Mixture-of-Experts sur Amazon
// SageMaker AI").  As in the operand swap of "A mátrixok felcserélése jobban
// kihasználja a Hopper GPU-kat", this kernel puts the expert-weight rows in the
// tensor core's M slot (128 rows per tile) and the tokens routed to the expert
// in N (16..256 in steps of 16), so a token count of 1 still fills the M=128
// datapath and the weights stream at HBM rate.  The same kernel serves decode
// (N = 16) and prefill (N up to 256) -- there is one code path.
//
// Work decomposition ("dynamic scheduling of variable token groups", "FP8
// esetén a Triton backend bizonyult gyorsabbnak"): for every expert e with
// c_e tokens, units = ceil(Mw/128) weight tiles x ceil(c_e/nmax) token tiles,
// each with KB = ceil(K/BK) k-blocks of 128 bytes.  Units are ordered by cost
// (full token tiles first, then partial ones, largest first) and dealt
// round-robin in waves to the persistent CTAs; the last one to two waves are
// cut into equal contiguous k-block ranges instead (stream-K), so all CTAs
// finish together.  Units that straddle a range boundary are finished by
// whichever contributor arrives last, which sums the fp32 partials in CTA
// order -- a fixed order, so the result does not depend on timing.
//
// Fusion ("one pass, no intermediate global round trips", same section): the
// gate/up kernel reads its token rows straight from x (token order) by the
// permutation, so no permuted copy of the activations is written; the down
// kernel can add w * y into an fp32 accumulator in token order (the combine)
// instead of writing permuted rows.
//
// Roles: warp 0 = copy producer (weights; activation rows by TMA where they
// are already in permuted order), warp 1 = MMA issuer (single thread), warp 2
// = TMEM allocator, warps 4-11 = epilogue (two warps per 32-lane TMEM quarter,
// alternating 16-column chunks), and, in the one-CTA gate/up kernel only
// (512 threads; the others run 384), warps 12-15 = gather of the token rows
// (cp.async).
// Shared-memory ring of stages of KPS k-blocks (A KPS*16 KB + B KPS*rows*128 B,
// 128-byte swizzle): 2 stages of 4 k-blocks on one CTA (token tiles of at most
// 64 rows), 3 stages of 2 k-blocks per CTA of a pair (larger tiles).  Two TMEM
// accumulators of nmax fp32 columns let the epilogue of one unit overlap the
// main loop of the next.  Every wait is bounded; on expiry the kernel records
// MOE_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
//
// Token tiles of more than 64 rows run on CTA pairs (cta_group::2): M = 256
// weight rows per MMA, each CTA holding 128 of them and half of the token
// tile; the rank-0 CTA issues the MMAs and its barriers count both CTAs' copies.
//
// Weights (A) are pre-packed as 16 KB tiles that are already the swizzled
// shared-memory image of one stage, so a stage's A operand (one to four
// consecutive k-blocks) is one contiguous copy.  The gate/up kernel's token
// rows (B) of one-CTA tiles (decode-sized, at most 64 tokens) are gathered
// with 16-byte cp.async copies placed in the same swizzled layout
// (zero-filled for pads); the MMA issuer waits for them, makes them visible
// to the tensor core's (async) proxy and issues.  Rows already in permuted
// order (the down kernel's h; the gate/up rows of CTA-pair tiles, which a
// gather kernel lays out first) come through TMA tensor maps with 128-, 64-
// and 16-row boxes.  Measured on B200: pair tiles gathered by cp.async ran
// the gate/up GEMM 1.3x slower than TMA from pre-gathered rows (prefill
// T = 4096: 320 vs 240 us), more than the gather kernel costs, while one-CTA
// tiles gathered in-kernel match the TMA path and save the gather kernel.
// Launched with
// programmatic dependent launch: the producer fetches the first weight tiles
// before waiting for the previous kernel, whose outputs it loads after.
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kBM = 128;            // weight rows per tile (UMMA M)
constexpr int kRowBytes = 128;      // K bytes per stage row (one swizzle atom)
constexpr int kATileBytes = kBM * kRowBytes;
constexpr int kThreads = 512;         // at most; see threads_for
constexpr int kFwdWarp = 2;           // TMEM allocator
constexpr int kEpiWarp0 = 4;          // warps 4..11: two per TMEM lane quarter
constexpr int kEpiThreads = 256;
constexpr int kGatherWarp0 = 12;      // warps 12..15 gather the gate/up token rows
constexpr int kGatherLanes = 128;
constexpr int kGatherRowsPerPass = kGatherLanes / 8;   // 8 lanes per 128-byte row
constexpr int kMaxStages = 8;
constexpr int kMinKbPerCta = 4;
constexpr int kStagingBytes = 16 * 1024;   // 2 KB per epilogue warp
constexpr int kSmemCap = 232448;     // per-block opt-in limit on sm_100
constexpr uint64_t kDrainLimitNs = 10000000ull;  // 10 ms

// Tensor maps of one launch: weight tiles (pairs), activation rows, and the
// adapters' expand tiles and shrink-output rows (multi-LoRA layers).
struct Maps {
    CUtensorMap a;                 // weight tiles, boxes of KPS tiles (pairs)
    CUtensorMap a1;                // weight tiles, one tile per box (pairs, adapters on)
    CUtensorMap al;                // adapter expand tiles, one tile per box (pairs)
    CUtensorMap b128, b64, b16;    // activation rows in permuted order
    CUtensorMap l128, l64, l16;    // adapter shrink outputs (rows in permuted order)
};

struct GemmArgs {
    int E, Mw, K, KB, MT, MTu, Mvalid;   // MTu: weight tiles per unit step (MT, or pairs)
    int KBm, KBx;              // k-blocks of the matrix, and of the adapters' expand
                               // (KB = KBm + KBx)
    const uint8_t* x_tiles;    // adapter expand tiles [E][MT][KBx] (KBx > 0)
    const int32_t* adapter;    // shrink (EPI 3): adapter of each token, -1 = none
    const float* lscale;       // shrink: scale of each adapter
    int lrank, lR;             // shrink: rank r, and n_adapters * r
    int nmax, tmem_cols, stages;
    const uint8_t* a_tiles;
    int ldo;
    void* out;
    const int32_t* counts;
    const int32_t* offsets;
    const int32_t* sorted_ids;
    int ktop;                  // assignments per token (flat index / ktop = token)
    int A;                     // assignments (T * ktop): flat indices are below it
    int capacity;              // rows of the permuted operands
    const uint8_t* gather_src; // gate/up: token-order rows of K elements
    long long src_row_bytes;
    const float* w;            // down: routing weight of flat index f
    const float* w_scales;
    const uint32_t* act_amax;
    uint32_t* out_amax;
    float* acc_zero;           // gate/up: fp32 buffer zeroed for a later reduction
    long long acc_zero_vec4;   // its size in float4
    float* partials;
    int32_t* counters;
    int32_t* status;
    int sched_after_wait;      // counts/offsets are the previous kernel's output
};

struct Ctl {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t gfull[kMaxStages];   // gathered rows of a stage landed (this CTA)
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int flag;
    uint32_t prod_pos;   // k-blocks issued by the producer
    uint32_t mma_pos;    // k-blocks whose full barrier the MMA thread observed
    uint32_t mma_issued; // 1 once any MMA was issued
    int scan_tmp[kThreads / 32 + 1];
    int n_full_units;                  // units of full token tiles (N = nmax)
    int n_partial;                     // experts with a partial last token tile
    int full_prefix[kMaxExperts + 1];  // full-tile units before expert e
    int nfull[kMaxExperts];            // full token tiles of expert e
    int np[kMaxExperts];               // rows of e's partial tile (0: none)
    int key[kMaxExperts];              // sort key of the partial tiles
    int part_expert[kMaxExperts];      // experts with a partial tile, largest first
    int off[kMaxExperts];
    int reuse;                         // some expert has three or more token tiles
};

struct Seg {
    int u, kb0, kb1, e, m, b_row, N;  // N: valid token rows rounded to 16
    int Nm;                           // MMA N (a CTA pair needs a multiple of 32)
};

constexpr int kDynSmemMax = kSmemCap - static_cast<int>(sizeof(Ctl)) - 1024;

// k-blocks per pipeline stage; the number of stages is as many as fit in
// shared memory (at most kMaxStages)
template <bool PAIR>
__host__ __device__ constexpr int kps_for() { return PAIR ? 2 : 4; }

__device__ __forceinline__ int find_expert(const int* prefix, int E, int u) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= u) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Unit order (cost first): all units of full token tiles (N = nmax) in
// (expert, weight tile, token tile) order, then the units of every expert's
// partial last token tile, largest first, in (expert, weight tile) order.
// Dealt round-robin, each wave then holds units of similar cost, and the
// stream-K remainder is made of the cheapest ones.
template <bool PAIR>
__device__ __forceinline__ Seg make_seg(const Ctl& c, const GemmArgs& g, int u, int kb0, int kb1) {
    Seg s;
    s.u = u;
    s.kb0 = kb0;
    s.kb1 = kb1;
    int nt;
    if (u < c.n_full_units) {
        s.e = find_expert(c.full_prefix, g.E, u);
        const int local = u - c.full_prefix[s.e];
        const int nf = c.nfull[s.e];
        s.m = local / nf;
        nt = local - s.m * nf;
        s.N = g.nmax;
    } else {
        const int v = u - c.n_full_units;
        const int r = v / g.MTu;
        s.m = v - r * g.MTu;
        s.e = c.part_expert[r];
        nt = c.nfull[s.e];
        s.N = c.np[s.e];
    }
    s.b_row = c.off[s.e] + nt * g.nmax;
    s.Nm = PAIR ? ((s.N + 31) & ~31) : s.N;
    return s;
}

// Work of one CTA.  With U units and G CTAs: when U > G, all but the last
// full wave are dealt whole and round-robin (CTA c takes units c, c+G, ...;
// each wave works on adjacent units, which share weight and token tiles in
// L2 and stream adjacent weight memory); the remaining G..2G-1 units are cut
// stream-K style into equal contiguous k-block ranges, one per CTA, so every
// CTA ends at the same time.  When U <= G, everything is stream-K.
struct Sched {
    int n_dp;          // whole units dealt round-robin
    int unit0;         // first unit of the stream-K part
    long long L;       // k-blocks of the stream-K part
    int Gsk;           // CTAs sharing the stream-K part
    long long ws, we;  // this CTA's stream-K range
};

struct Cursor {
    int j, n_dp, cta, G, KB, unit0;
    long long x, we;
    __device__ __forceinline__ bool next(int& u, int& kb0, int& kb1) {
        if (j < n_dp) {
            u = cta + j * G;
            kb0 = 0;
            kb1 = KB;
            ++j;
            return true;
        }
        if (x < we) {
            const long long uu = x / KB;
            u = unit0 + static_cast<int>(uu);
            kb0 = static_cast<int>(x - uu * KB);
            const long long left = we - x;
            kb1 = (KB - kb0 <= left) ? KB : kb0 + static_cast<int>(left);
            x += kb1 - kb0;
            return true;
        }
        return false;
    }
};

// CTA whose range [floor(c*L/G), floor((c+1)*L/G)) holds k-block X.
__device__ __forceinline__ int owner_cta(long long X, long long L, int G) {
    return static_cast<int>(((X + 1) * G - 1) / L);
}

__device__ __forceinline__ void named_bar_epi() {
    asm volatile("bar.sync 1, 256;" ::: "memory");
}

__device__ __forceinline__ void raise_abort(Ctl& c, int32_t* status) {
    report(status, MOE_ERR_TIMEOUT);
    *reinterpret_cast<volatile int*>(&c.abort) = 1;
}

// One 16-column chunk (16 tokens) of the accumulator rows this thread owns.
// Epilogue warp w (4..11) owns TMEM lane quarter q = w % 4 (rows 32q..32q+31)
// and every other chunk (half h = (w - 4) / 4).  `sw` is the FP8 dequant
// factor of this row; `wreg` / `treg` hold the routing weights / token
// indices (-1 for pads) of the unit's tokens, token j in lane j/8, register
// j%8.
//   EPI 0: h = SiLU(gate) * up -> bf16 rows of h (permuted order)
//   EPI 1: w * y -> bf16 rows of y_perm (permuted order)
//   EPI 2: w * y added (fp32) into row `token` of the accumulator
//   EPI 3: adapter shrink: output column c (c % 64 = a * r + q) belongs to
//          adapter a; it keeps s_a * value for tokens of adapter a and 0 for
//          every other token (treg holds the tokens' adapters) -> bf16 rows
template <bool FP8, int EPI>
__device__ __forceinline__ void epilogue_chunk(const GemmArgs& g, const Seg& s, int m_own, int c0,
                                               float (&v)[16], float sw, const float (&wreg)[8],
                                               const int (&treg)[8], uint8_t* staging,
                                               float& amax) {
    const int ew = (threadIdx.x >> 5) - kEpiWarp0;
    const int q = (threadIdx.x >> 5) & 3;
    const int lane = threadIdx.x & 31;
    constexpr unsigned kFull = 0xffffffffu;
    if constexpr (FP8) {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] *= sw;
    }
    if constexpr (EPI == 0) {
        __nv_bfloat16* st = reinterpret_cast<__nv_bfloat16*>(staging + ew * 1024);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float p = __shfl_xor_sync(kFull, v[i], 16);
            const float gte = lane < 16 ? v[i] : p;
            const float up = lane < 16 ? p : v[i];
            const __nv_bfloat16 h = __float2bfloat16_rn(silu(gte) * up);
            if (lane < 16) {
                st[i * 16 + lane] = h;
                if constexpr (FP8) amax = fmaxf(amax, fabsf(__bfloat162float(h)));
            }
        }
        __syncwarp();
        const int row = s.b_row + c0 + (lane >> 1);
        const int col = m_own * 64 + 16 * q + 8 * (lane & 1);
        const uint4 val = *reinterpret_cast<const uint4*>(st + (lane >> 1) * 16 + 8 * (lane & 1));
        if (m_own < g.MT)
            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) +
                                      static_cast<long>(row) * g.ldo + col) = val;
        __syncwarp();
    } else if constexpr (EPI == 1 || EPI == 3) {
        __nv_bfloat16* st = reinterpret_cast<__nv_bfloat16*>(staging + ew * 1024);
        if constexpr (EPI == 1) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float wi = __shfl_sync(kFull, wreg[i & 7], (c0 + i) >> 3);
                st[i * 32 + lane] = __float2bfloat16_rn(v[i] * wi);
            }
        } else {
            const int slot = (m_own * kBM + 32 * q + lane) & 63;
            const int ac = slot < g.lR ? slot / g.lrank : -2;   // this column's adapter
            const float sc = ac >= 0 ? __ldg(g.lscale + ac) : 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int ai = __shfl_sync(kFull, treg[i & 7], (c0 + i) >> 3);
                st[i * 32 + lane] = __float2bfloat16_rn(ai == ac ? v[i] * sc : 0.0f);
            }
        }
        __syncwarp();
        const int hcol0 = m_own * kBM + 32 * q;
        if (hcol0 < g.Mvalid && m_own < g.MT) {
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const int piece = lane + 32 * t;
                const int row = piece >> 2, seg = piece & 3;
                const uint4 val = *reinterpret_cast<const uint4*>(st + row * 32 + 8 * seg);
                *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) +
                                          static_cast<long>(s.b_row + c0 + row) * g.ldo + hcol0 +
                                          8 * seg) = val;
            }
        }
        __syncwarp();
    } else {
        // w * y staged as [16 tokens][32 columns] fp32, then added into the
        // accumulator 16 bytes at a time: each lane adds 4 consecutive
        // columns of one token's row (a warp-wide add covers four 128-byte
        // row segments), a quarter of the L2 operations of scalar adds
        float* st = reinterpret_cast<float*>(staging + ew * 2048);
        int tok_of_row = -1;   // lane r < 16 holds the token of chunk row r
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float wi = __shfl_sync(kFull, wreg[i & 7], (c0 + i) >> 3);
            const int ti = __shfl_sync(kFull, treg[i & 7], (c0 + i) >> 3);
            if (lane == i) tok_of_row = ti;
            st[i * 32 + lane] = v[i] * wi;
        }
        __syncwarp();
        const int hcol0 = m_own * kBM + 32 * q;
        float* acc = static_cast<float*>(g.out);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int piece = lane + 32 * t;
            const int row = piece >> 3, seg = piece & 7;
            const int ti = __shfl_sync(kFull, tok_of_row, row);
            if (ti >= 0 && hcol0 < g.Mvalid)
                red_add_v4(acc + static_cast<long>(ti) * g.ldo + hcol0 + 4 * seg,
                           *reinterpret_cast<const float4*>(st + row * 32 + 4 * seg));
        }
        __syncwarp();
    }
}

// Threads of one instantiation: the gather warps (12-15) exist only where a
// one-CTA gate/up kernel gathers its rows; the others run 384 threads, which
// leaves more registers per thread for the epilogue.
template <int EPI, bool PAIR>
__host__ __device__ constexpr int threads_for() { return EPI == 0 && !PAIR ? 512 : 384; }

template <bool FP8, int EPI, bool PAIR>
__global__ void __launch_bounds__(threads_for<EPI, PAIR>(), 1)
    grouped_gemm_kernel(const __grid_constant__ Maps maps, const GemmArgs g) {
    // gate/up token rows: gathered by the kernel itself for one-CTA tiles;
    // CTA-pair tiles (large token tiles) read rows a gather kernel laid out
    // in permuted order, by TMA
    constexpr bool GATHER = EPI == 0 && !PAIR;
    const int S = g.stages;
    // k-blocks per stage: 2 for a pair (large token tiles), 4 for one CTA
    constexpr int KPS = kps_for<PAIR>();
    constexpr int NT = threads_for<EPI, PAIR>();
    extern __shared__ uint8_t dsmem_raw[];
    __shared__ Ctl ctl;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    // stage = KPS consecutive k-blocks: A KPS*16 KB (one bulk copy), B KPS
    // slots of nmax rows x 128 B
    const int rank = PAIR ? static_cast<int>(cluster_ctarank()) : 0;
    const int a_stage_bytes = KPS * kATileBytes;
    // a pair member holds half of each token tile
    const int b_kb_bytes = (PAIR ? g.nmax / 2 : g.nmax) * kRowBytes;
    const int b_stage_bytes = KPS * b_kb_bytes;
    uint8_t* smA = base;
    uint8_t* smB = smA + S * a_stage_bytes;
    uint8_t* staging = smB + S * b_stage_bytes;

    if (g.sched_after_wait) pdl_wait();   // the counts come from the previous kernel

    // ---- schedule tables: per-expert counts, offsets, token tiles, unit prefix
    {
        const int e = threadIdx.x;
        int units = 0;
        int key = 0x7fffffff;
        int tiles = 0;   // token tiles of expert e
        if (e < g.E) {
            int c = __ldcg(g.counts + e);
            const int o = __ldcg(g.offsets + e);
            if constexpr (kDebugChecks) {
                // the expert's rows, padded to 16, must lie inside the capacity
                if (c < 0 || o < 0 || o + ((c + 15) & ~15) > g.capacity) {
                    report(g.status, MOE_ERR_DEVICE);
                    c = 0;
                }
            }
            ctl.off[e] = o;
            int nf = c / g.nmax;
            const int r = c - nf * g.nmax;
            int n = (r + 15) & ~15;
            if (n == g.nmax) {  // rounds up to a full tile
                ++nf;
                n = 0;
            }
            ctl.nfull[e] = nf;
            ctl.np[e] = n;
            tiles = nf + (n > 0 ? 1 : 0);
            units = nf * g.MTu;
            if (n > 0) key = (g.nmax - n) * kMaxExperts + e;
        }
        if (e < kMaxExperts) ctl.key[e] = key;
        int inc = units;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, inc, off);
            if (lane >= off) inc += o;
        }
        if (lane == 31) ctl.scan_tmp[warp] = inc;
        if (threadIdx.x == 0) {
            for (int i = 0; i < S; ++i) {
                // the producer's copies (the gathered rows of a one-CTA
                // gate/up kernel complete on gfull, which the MMA thread
                // waits for itself)
                mbar_init(&ctl.full[i], 1);
                mbar_init(&ctl.empty[i], 1);
                mbar_init(&ctl.gfull[i], kGatherLanes);
            }
            for (int i = 0; i < 2; ++i) {
                mbar_init(&ctl.tfull[i], 1);
                mbar_init(&ctl.tempty[i], (PAIR ? 2 : 1) * (kEpiThreads / 32));
            }
            mbar_init(&ctl.drain, 1);
            fence_mbar_init();
            ctl.abort = 0;
            ctl.prod_pos = 0;
            ctl.mma_pos = 0;
            ctl.mma_issued = 0;
            ctl.reuse = 0;
        }
        if (warp == 0 && lane == 0) {
            if constexpr (PAIR) tma_prefetch_desc(g.KBx ? &maps.a1 : &maps.a);
            if constexpr (!GATHER) {
                tma_prefetch_desc(&maps.b128);
                tma_prefetch_desc(&maps.b64);
                tma_prefetch_desc(&maps.b16);
            }
        }
        if (warp == kFwdWarp) {
            if constexpr (PAIR) {
                tmem_alloc_pair(&ctl.tmem_base, g.tmem_cols);
                tmem_relinquish_pair();
            } else {
                tmem_alloc(&ctl.tmem_base, g.tmem_cols);
                tmem_relinquish();
            }
        }
        __syncthreads();
        if (tiles >= 3) ctl.reuse = 1;   // read after the next barrier
        if (threadIdx.x == 0) {
            int run = 0;
            for (int i = 0; i < NT / 32; ++i) {
                const int t = ctl.scan_tmp[i];
                ctl.scan_tmp[i] = run;
                run += t;
            }
            ctl.scan_tmp[NT / 32] = run;
        }
        __syncthreads();
        if (e < g.E) ctl.full_prefix[e] = ctl.scan_tmp[warp] + inc - units;
        if (threadIdx.x == 0) {
            ctl.full_prefix[g.E] = ctl.scan_tmp[NT / 32];
            ctl.n_full_units = ctl.scan_tmp[NT / 32];
        }
        // rank of e's partial tile among all partial tiles (keys are distinct)
        if (key != 0x7fffffff) {
            int rank_e = 0;
            for (int i = 0; i < g.E; ++i) rank_e += ctl.key[i] < key ? 1 : 0;
            ctl.part_expert[rank_e] = e;
        }
        const int n_has = __popc(__ballot_sync(0xffffffffu, key != 0x7fffffff));
        __syncthreads();
        if (lane == 0) ctl.scan_tmp[warp] = n_has;
        __syncthreads();
        if (threadIdx.x == 0) {
            int t = 0;
            for (int i = 0; i < NT / 32; ++i) t += ctl.scan_tmp[i];
            ctl.n_partial = t;
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // the peer's barriers must be initialised before any cross-CTA signal
        if constexpr (PAIR) cluster_sync();
    }

    const int U = ctl.n_full_units + ctl.n_partial * g.MTu;
    const int G = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
    const int cta = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    Sched sc;
    sc.n_dp = U > G ? U / G - 1 : 0;
    sc.unit0 = sc.n_dp * G;
    sc.L = static_cast<long long>(U - sc.unit0) * g.KB;
    {
        long long gs = (sc.L + kMinKbPerCta - 1) / kMinKbPerCta;
        sc.Gsk = static_cast<int>(gs < G ? gs : G);
        if (sc.Gsk < 1) sc.Gsk = 1;
    }
    const bool in_sk = sc.L > 0 && cta < sc.Gsk;
    sc.ws = in_sk ? static_cast<long long>(cta) * sc.L / sc.Gsk : 0;
    sc.we = in_sk ? static_cast<long long>(cta + 1) * sc.L / sc.Gsk : 0;
    const bool active = sc.n_dp > 0 || in_sk;
    auto cursor = [&]() { return Cursor{0, sc.n_dp, cta, G, g.KB, sc.unit0, sc.ws, sc.we}; };
    const uint32_t tmem_base = ctl.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------ copy producer
        // (both CTAs of a pair run it; their copies complete on the rank-0
        // CTA's barrier, which the rank-0 producer arms for both)
        if (lane == 0) {
            uint32_t it = 0;
            const int bk_elems = FP8 ? 128 : 64;
            // L2 policy of the weight copies, one per launch: each weight tile
            // is read once per token tile of its expert, so evict-first unless
            // some expert has three or more token tiles.  Measured on B200:
            // with skewed routing evict-first re-read the hot experts' weights
            // from DRAM (gate/up 18.0 GB vs 14.9 GB with a normal hint, layer
            // 4.6% slower); where weights are read once or twice, evict-first
            // keeps the activations in L2 (a normal hint slowed decode T = 64
            // by 7% and FP8 T = 2048 by 1%).
            const uint64_t wpol = ctl.reuse ? kEvictNormal : kEvictFirst;
            const int mt_last = g.MT - 1;
            // A pair loads full KPS-tile boxes of weights; a single CTA loads
            // exactly the stage's k-blocks.  The gate/up kernel's token rows
            // are not counted here: the gather warps deliver them.
            // (k-blocks past KBm are an adapter's expand: weights from the
            // adapter tiles, rows from the shrink outputs, both by the
            // producer; with adapters, weights are copied k-block by k-block)
            auto stage_bytes = [&](const Seg& sg, int kb, int nk) -> uint32_t {
                const int rows = PAIR ? sg.Nm / 2 : sg.N;
                const int n64 = rows >> 6, n16 = (rows & 63) >> 4;
                const uint32_t row_bytes = static_cast<uint32_t>((n64 * 64 + n16 * 16) * kRowBytes);
                int nb = nk;   // k-blocks whose rows the producer copies
                if constexpr (GATHER) nb = max(0, kb + nk - max(kb, g.KBm));
                const uint32_t b = static_cast<uint32_t>(nb) * row_bytes;
                const int na = (PAIR && g.KBx == 0) ? KPS : nk;
                return (PAIR ? 2u : 1u) * (static_cast<uint32_t>(na * kATileBytes) + b);
            };
            auto load_a = [&](const Seg& sg, int kb, int nk, int st) {
                int m_own = PAIR ? 2 * sg.m + rank : sg.m;
                if (m_own > mt_last) m_own = mt_last;   // odd tile count: any valid tile
                const size_t em = static_cast<size_t>(sg.e) * g.MT + m_own;
                if (g.KBx == 0) {
                    const size_t tile = em * g.KBm + kb;
                    if constexpr (PAIR)
                        tma_load_2d_pair(smA + st * a_stage_bytes, &maps.a, &ctl.full[st], 0,
                                         static_cast<int>(tile * kTileRows), wpol);
                    else
                        bulk_load(smA + st * a_stage_bytes, g.a_tiles + tile * kTileBytes,
                                  nk * kATileBytes, &ctl.full[st], wpol);
                    return;
                }
                for (int q = 0; q < nk; ++q) {
                    const int k = kb + q;
                    const bool ext = k >= g.KBm;
                    const size_t tile = ext ? em * g.KBx + (k - g.KBm) : em * g.KBm + k;
                    uint8_t* dst = smA + st * a_stage_bytes + q * kATileBytes;
                    if constexpr (PAIR)
                        tma_load_2d_pair(dst, ext ? &maps.al : &maps.a1, &ctl.full[st], 0,
                                         static_cast<int>(tile * kTileRows), wpol);
                    else
                        bulk_load(dst, (ext ? g.x_tiles : g.a_tiles) + tile * kTileBytes,
                                  kATileBytes, &ctl.full[st], wpol);
                }
            };
            auto load_b = [&](const Seg& sg, int kb, int nk, int st) {
                const int rows = PAIR ? sg.Nm / 2 : sg.N;
                const int n128 = rows >> 7, n64 = (rows & 127) >> 6, n16 = (rows & 63) >> 4;
                for (int q = 0; q < nk; ++q) {
                    const int k = kb + q;
                    const bool ext = k >= g.KBm;
                    if (GATHER && !ext) continue;   // the gather warps copy these rows
                    const CUtensorMap* m128 = ext ? &maps.l128 : &maps.b128;
                    const CUtensorMap* m64 = ext ? &maps.l64 : &maps.b64;
                    const CUtensorMap* m16 = ext ? &maps.l16 : &maps.b16;
                    uint8_t* b = smB + st * b_stage_bytes + q * b_kb_bytes;
                    int row = sg.b_row + rank * rows;
                    const int xk = ext ? (k - g.KBm) * 64 : k * bk_elems;
                    for (int j = 0; j < n128; ++j, row += 128, b += 128 * kRowBytes) {
                        if constexpr (PAIR)
                            tma_load_2d_pair(b, m128, &ctl.full[st], xk, row, kEvictLast);
                        else
                            tma_load_2d(b, m128, &ctl.full[st], xk, row, kEvictLast);
                    }
                    for (int j = 0; j < n64; ++j, row += 64, b += 64 * kRowBytes) {
                        if constexpr (PAIR)
                            tma_load_2d_pair(b, m64, &ctl.full[st], xk, row, kEvictLast);
                        else
                            tma_load_2d(b, m64, &ctl.full[st], xk, row, kEvictLast);
                    }
                    for (int j = 0; j < n16; ++j, row += 16, b += 16 * kRowBytes) {
                        if constexpr (PAIR)
                            tma_load_2d_pair(b, m16, &ctl.full[st], xk, row, kEvictLast);
                        else
                            tma_load_2d(b, m16, &ctl.full[st], xk, row, kEvictLast);
                    }
                }
            };
            // Stages whose weight tiles are issued before the wait for the
            // previous kernel; their activation rows follow after it.
            int early = 0;
            if (active) {
                Cursor cur = cursor();
                int u, kb0, kb1;
                while (early < S && cur.next(u, kb0, kb1)) {
                    const Seg sg = make_seg<PAIR>(ctl, g, u, kb0, kb1);
                    for (int kb = sg.kb0; kb < sg.kb1 && early < S; kb += KPS, ++early) {
                        const int nk = min(KPS, sg.kb1 - kb);
                        if (rank == 0)
                            mbar_arrive_expect_tx(&ctl.full[early], stage_bytes(sg, kb, nk));
                        load_a(sg, kb, nk, early);
                    }
                }
            }
            pdl_wait();
            pdl_trigger();
            Cursor cur = cursor();
            int u, kb0, kb1;
            int st = 0;
            uint32_t par = 1;   // parity of the empty-barrier phase the next refill waits for
            while (active && cur.next(u, kb0, kb1)) {
                const Seg sg = make_seg<PAIR>(ctl, g, u, kb0, kb1);
                bool ok = true;
                for (int kb = sg.kb0; kb < sg.kb1; kb += KPS, ++it) {
                    const int nk = min(KPS, sg.kb1 - kb);
                    if (it >= static_cast<uint32_t>(early)) {
                        if (!mbar_wait(&ctl.empty[st], par, &ctl.abort)) {
                            raise_abort(ctl, g.status);
                            ok = false;
                            break;
                        }
                        if (rank == 0) mbar_arrive_expect_tx(&ctl.full[st], stage_bytes(sg, kb, nk));
                        load_a(sg, kb, nk, st);
                    }
                    if (!GATHER || kb + nk > g.KBm) load_b(sg, kb, nk, st);
                    if (++st == S) {
                        st = 0;
                        par ^= 1u;
                    }
                }
                if (!ok) break;
            }
            ctl.prod_pos = it > static_cast<uint32_t>(early) ? it : static_cast<uint32_t>(early);
        }
        __syncwarp();
    } else if (warp >= kGatherWarp0) {
        // ------------------------------------------------ gather (gate/up)
        // Lane gl copies 16-byte chunk c = gl % 8 of rows r0 + 16 i (r0 =
        // gl / 8) of this CTA's token rows, for every k-block of a stage: a
        // warp covers four whole 128-byte row segments per instruction.  In
        // the 128-byte swizzle, chunk c of row r sits at c ^ (r % 8), which is
        // fixed per lane.  Pads (sorted_ids = -1), rows past the tile and
        // bytes past the end of a row are zero-filled.
        if constexpr (GATHER) {
            const int gl = threadIdx.x - kGatherWarp0 * 32;
            const int c = gl & 7, r0 = gl >> 3;
            const uint32_t cs = static_cast<uint32_t>((c ^ (r0 & 7)) << 4);
            constexpr int kMaxRowIters = 128 / kGatherRowsPerPass;   // 8
            const uint32_t smB_u32 = smem_u32(smB);
            // token (row of the source) of each of this lane's rows of a
            // unit, -1 for pads and rows past the tile
            auto load_tokens = [&](const Seg& sg, int (&tok)[kMaxRowIters]) {
                const int rows = PAIR ? sg.Nm / 2 : sg.N;
                const int first = rank * rows;     // this CTA's first row of the tile
#pragma unroll
                for (int i = 0; i < kMaxRowIters; ++i) {
                    const int r = r0 + kGatherRowsPerPass * i;
                    int sid = -1;
                    if (r < rows && first + r < sg.N)
                        sid = __ldg(g.sorted_ids + sg.b_row + first + r);
                    if constexpr (kDebugChecks) {
                        if (sid < -1 || sid >= g.A) {
                            report(g.status, MOE_ERR_DEVICE);
                            sid = -1;
                        }
                    }
                    tok[i] = sid >= 0 ? sid / g.ktop : -1;
                }
            };
            pdl_wait();   // sorted_ids and the source rows come from earlier kernels
            int st = 0;
            uint32_t par = 1;
            Cursor cur = cursor();
            int u, kb0, kb1;
            bool ok = true;
            bool have = active && cur.next(u, kb0, kb1);
            Seg sg{};
            int tok[kMaxRowIters];
            if (have) {
                sg = make_seg<PAIR>(ctl, g, u, kb0, kb1);
                load_tokens(sg, tok);
            }
            while (ok && have) {
                // the next unit's token rows are fetched while this unit's
                // stages are issued, so no unit starts with a dependent load
                int nu, nkb0, nkb1;
                const bool have_next = cur.next(nu, nkb0, nkb1);
                Seg nsg{};
                int ntok[kMaxRowIters];
#pragma unroll
                for (int i = 0; i < kMaxRowIters; ++i) ntok[i] = -1;
                bool fetched = false;
                const int rows = PAIR ? sg.Nm / 2 : sg.N;
                for (int kb = sg.kb0; kb < sg.kb1; kb += KPS) {
                    const int nk = min(KPS, sg.kb1 - kb);
                    if (!mbar_wait(&ctl.empty[st], par, &ctl.abort)) {
                        raise_abort(ctl, g.status);
                        ok = false;
                        break;
                    }
                    for (int q = 0; q < nk && kb + q < g.KBm; ++q) {
                        const long long kofs = static_cast<long long>(kb + q) * kRowBytes + c * 16;
                        const bool in_row = kofs < g.src_row_bytes;
                        const uint32_t dst0 = smB_u32 + st * b_stage_bytes + q * b_kb_bytes + cs;
#pragma unroll
                        for (int i = 0; i < kMaxRowIters; ++i) {
                            const int r = r0 + kGatherRowsPerPass * i;
                            if (r < rows) {
                                const bool v = in_row && tok[i] >= 0;
                                const uint8_t* src =
                                    v ? g.gather_src + static_cast<long long>(tok[i]) * g.src_row_bytes + kofs
                                      : g.gather_src;
                                cp_async16(dst0 + r * kRowBytes, src, v ? 16u : 0u);
                            }
                        }
                    }
                    cp_async_arrive_noinc(&ctl.gfull[st]);
                    if (++st == S) {
                        st = 0;
                        par ^= 1u;
                    }
                    if (!fetched && have_next) {
                        nsg = make_seg<PAIR>(ctl, g, nu, nkb0, nkb1);
                        load_tokens(nsg, ntok);
                        fetched = true;
                    }
                }
                have = have_next;
                if (have) {
                    if (!fetched) {
                        nsg = make_seg<PAIR>(ctl, g, nu, nkb0, nkb1);
                        load_tokens(nsg, ntok);
                    }
                    sg = nsg;
#pragma unroll
                    for (int i = 0; i < kMaxRowIters; ++i) tok[i] = ntok[i];
                }
            }
            // no copy may still target shared memory when the CTA moves on
            cp_async_wait_all();
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0 && active && rank == 0) {
            // The issue loop is kept short: one thread feeds the tensor core,
            // and at N <= 128 an MMA takes only tens of cycles.  Stage index
            // and phase advance incrementally, and descriptors advance by
            // adding (byte offset >> 4) to their start-address field.
            const uint64_t a_desc0 = sw128_desc(smem_u32(smA));
            const uint64_t b_desc0 = sw128_desc(smem_u32(smB));
            const uint32_t a_step = static_cast<uint32_t>(a_stage_bytes) >> 4;
            const uint32_t b_step = static_cast<uint32_t>(b_stage_bytes) >> 4;
            const uint32_t b_kb = static_cast<uint32_t>(b_kb_bytes) >> 4;
            uint64_t ast = a_desc0, bst = b_desc0;
            int st = 0;
            uint32_t ph = 0, it = 0, si = 0;
            bool ok = true;
            Cursor cur = cursor();
            int u, kb0, kb1;
            ctl.mma_issued = 1;
            for (; ok && cur.next(u, kb0, kb1); ++si) {
                const Seg s = make_seg<PAIR>(ctl, g, u, kb0, kb1);
                const int acc = si & 1;
                if (!mbar_wait(&ctl.tempty[acc], ((si >> 1) & 1u) ^ 1u, &ctl.abort)) {
                    raise_abort(ctl, g.status);
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + acc * g.nmax;
                const uint32_t idesc = make_idesc<FP8>(PAIR ? 2 * kBM : kBM, s.Nm);
                for (int kb = s.kb0; kb < s.kb1; kb += KPS, ++it) {
                    const int nk = s.kb1 - kb;
                    bool got = true;
                    if constexpr (GATHER) {
                        // this CTA's gathered rows: wait for their copies,
                        // then make them visible to the tensor core's proxy
                        got = mbar_wait(&ctl.gfull[st], ph, &ctl.abort);
                        if (got) fence_proxy_async_smem();
                    }
                    // weights (and the TMA-loaded activation rows)
                    if (got) got = mbar_wait(&ctl.full[st], ph, &ctl.abort);
                    if (!got) {
                        raise_abort(ctl, g.status);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t first = kb == s.kb0 ? 0u : 1u;
#pragma unroll
                    for (int q = 0; q < KPS; ++q) {
                        if (q == 0 || q < nk) {
                            const uint64_t ad = ast + static_cast<uint32_t>(q * (kATileBytes >> 4));
                            const uint64_t bd = bst + static_cast<uint32_t>(q) * b_kb;
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint32_t accum = (q | kk) ? 1u : first;
                                if constexpr (PAIR)
                                    umma_pair<FP8>(d, ad + 2 * kk, bd + 2 * kk, idesc, accum);
                                else
                                    umma<FP8>(d, ad + 2 * kk, bd + 2 * kk, idesc, accum);
                            }
                        }
                    }
                    if constexpr (PAIR) umma_commit_pair(&ctl.empty[st]);
                    else umma_commit(&ctl.empty[st]);
                    if (++st == S) {
                        st = 0;
                        ph ^= 1u;
                        ast = a_desc0;
                        bst = b_desc0;
                    } else {
                        ast += a_step;
                        bst += b_step;
                    }
                }
                if (!ok) break;
                if constexpr (PAIR) umma_commit_pair(&ctl.tfull[acc]);
                else umma_commit(&ctl.tfull[acc]);
            }
            ctl.mma_pos = it;
        }
        __syncwarp();
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kEpiThreads / 32) {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;                     // TMEM lane quarter
        const int half = (warp - kEpiWarp0) >> 2;   // which chunks: c0 = 16*(2j + half)
        const int row = 32 * q + lane;              // accumulator row = TMEM lane
        const int slot_cta = PAIR ? 2 * cta + rank : cta;   // this CTA's partial slots
        // release of an accumulator: one arrival per warp, on the rank-0 CTA
        auto release = [&](int acc) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (PAIR) mbar_arrive_leader(&ctl.tempty[acc]);
                else mbar_arrive(&ctl.tempty[acc]);
            }
        };
        // the scales and the routing outputs come from earlier kernels
        pdl_wait();
        if constexpr (EPI == 0) {
            // zero this CTA's slice of the fp32 buffer a later down kernel
            // reduces into (its kernel starts only after this one completes)
            if (g.acc_zero) {
                const long long nthreads = static_cast<long long>(gridDim.x) * kEpiThreads;
                const long long tid = static_cast<long long>(blockIdx.x) * kEpiThreads +
                                      (threadIdx.x - kEpiWarp0 * 32);
                float4* z = reinterpret_cast<float4*>(g.acc_zero);
                for (long long i = tid; i < g.acc_zero_vec4; i += nthreads)
                    z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        float act_scale = 1.0f;
        if constexpr (FP8) act_scale = fp8_scale_from_amax(__ldcg(g.act_amax));
        float amax = 0.0f;
        uint32_t si = 0;
        Cursor cur = cursor();
        int u, kb0, kb1;
        for (; active && cur.next(u, kb0, kb1); ++si) {
            const Seg s = make_seg<PAIR>(ctl, g, u, kb0, kb1);
            const int acc = si & 1;
            const int m_own = PAIR ? 2 * s.m + rank : s.m;   // this CTA's 128-row weight tile
            // per-unit constants: FP8 dequant factor of this row, routing
            // weights and token indices of the unit's tokens
            float sw = 1.0f;
            if constexpr (FP8)
                sw = act_scale * __ldg(g.w_scales + s.e * 3 + (EPI != 0 ? 2 : (lane < 16 ? 0 : 1)));
            float wreg[8];
            int treg[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                wreg[i] = 0.0f;
                treg[i] = -1;
            }
            if constexpr (EPI != 0) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int j = 8 * lane + i;
                    if (j < s.N) {
                        int sid = __ldg(g.sorted_ids + s.b_row + j);
                        if constexpr (kDebugChecks) {
                            if (sid < -1 || sid >= g.A) {
                                report(g.status, MOE_ERR_DEVICE);
                                sid = -1;
                            }
                        }
                        if (sid >= 0) {
                            if constexpr (EPI == 3) {
                                treg[i] = __ldg(g.adapter + sid / g.ktop);
                            } else {
                                wreg[i] = __ldg(g.w + sid);
                                treg[i] = sid / g.ktop;
                            }
                        }
                    }
                }
            }
            if (!mbar_wait(&ctl.tfull[acc], (si >> 1) & 1u, &ctl.abort)) {
                raise_abort(ctl, g.status);
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + acc * g.nmax;
            if (s.kb0 == 0 && s.kb1 == g.KB) {
                // this warp's chunks c0 and c0 + 32 loaded together, one wait
                for (int c0 = 16 * half; c0 < s.N; c0 += 64) {
                    const bool two = c0 + 32 < s.N;   // warp-uniform
                    uint32_t r0[16], r1[16];
                    tmem_ld16_async(taddr + c0, r0);
                    if (two) tmem_ld16_async(taddr + c0 + 32, r1);
                    tmem_wait16(r0);
                    if (two) tmem_wait16(r1);
                    float v[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r0[i]);
                    epilogue_chunk<FP8, EPI>(g, s, m_own, c0, v, sw, wreg, treg, staging, amax);
                    if (two) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r1[i]);
                        epilogue_chunk<FP8, EPI>(g, s, m_own, c0 + 32, v, sw, wreg, treg, staging,
                                                 amax);
                    }
                }
                release(acc);
            } else {
                const long long X0 = static_cast<long long>(s.u - sc.unit0) * g.KB;
                const int cf = owner_cta(X0, sc.L, sc.Gsk);
                const int cl = owner_cta(X0 + g.KB - 1, sc.L, sc.Gsk);
                const long long slot_elems = static_cast<long long>(kBM) * g.nmax;
                // partial tiles are column-major (element (row, col) at
                // col * 128 + row): a warp's 32 rows form one 128-byte line
                float* mine = g.partials + (2LL * slot_cta + (cta == cf ? 1 : 0)) * slot_elems + row;
                for (int c0 = 16 * half; c0 < s.N; c0 += 32) {
                    float v[16];
                    tmem_ld16(taddr + c0, v);
#pragma unroll
                    for (int i = 0; i < 16; ++i) __stcg(mine + (c0 + i) * kBM, v[i]);
                }
                release(acc);
                __threadfence();
                named_bar_epi();
                const int ctr = PAIR ? 2 * cf + rank : cf;
                if (threadIdx.x == kEpiWarp0 * 32) {
                    const int old = atomicAdd(&g.counters[ctr], 1);
                    ctl.flag = (old == cl - cf) ? 1 : 0;
                }
                named_bar_epi();
                const int finisher = ctl.flag;
                named_bar_epi();
                if (finisher) {
                    __threadfence();
                    for (int c0 = 16 * half; c0 < s.N; c0 += 32) {
                        float v[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = 0.0f;
                        for (int cc = cf; cc <= cl; ++cc) {
                            const int cc_cta = PAIR ? 2 * cc + rank : cc;
                            const float* p = g.partials +
                                             (2LL * cc_cta + (cc == cf ? 1 : 0)) * slot_elems +
                                             c0 * kBM + row;
#pragma unroll
                            for (int i = 0; i < 16; ++i) v[i] += ld_cg(p + i * kBM);
                        }
                        epilogue_chunk<FP8, EPI>(g, s, m_own, c0, v, sw, wreg, treg, staging,
                                                 amax);
                    }
                    if (threadIdx.x == kEpiWarp0 * 32) g.counters[ctr] = 0;
                }
            }
        }
        if constexpr (FP8 && EPI == 0) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            if (lane == 0 && amax > 0.0f) atomic_max_nonneg(g.out_amax, amax);
        }
    }

    __syncthreads();
    if (*reinterpret_cast<volatile int*>(&ctl.abort)) {
        // Drain: wait (bounded) for this CTA's own MMAs and copies in flight.
        if (warp == 1 && lane == 0 && ctl.mma_issued) {
            if constexpr (PAIR) umma_commit_pair_local(&ctl.drain);
            else umma_commit(&ctl.drain);
            mbar_wait(&ctl.drain, 0, nullptr, kDrainLimitNs);
        }
        // a pair's copies all complete on the rank-0 CTA's barriers
        if (warp == 0 && lane == 0 && rank == 0) {
            for (uint32_t it = ctl.mma_pos; it < ctl.prod_pos; ++it)
                mbar_wait(&ctl.full[it % S], (it / S) & 1u, nullptr, kDrainLimitNs);
        }
        __syncthreads();
    }
    // neither CTA of a pair frees its TMEM before the pair's MMAs, copies
    // and epilogues are all done
    if constexpr (PAIR) cluster_sync();
    if (warp == kFwdWarp) {
        tc_fence_after();
        if constexpr (PAIR) tmem_dealloc_pair(tmem_base, g.tmem_cols);
        else tmem_dealloc(tmem_base, g.tmem_cols);
    }
}

// ---- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_map(CUtensorMap* m, const void* ptr, bool fp8, int K, long rows, int box_rows) {
    // Zero-size tensors are not encodable; a one-row placeholder is never read.
    if (rows < 1) rows = 1;
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * (fp8 ? 1 : 2)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(fp8 ? 128 : 64),
                               static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
              const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Weight tiles viewed as rows of 128 bytes (16 KB tile = 128 rows), copied
// verbatim (the tiles are already swizzled): boxes of kps tiles.
bool make_tile_map(CUtensorMap* m, const void* ptr, long tiles, int kps) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kTileRowBytes),
                                static_cast<cuuint64_t>(tiles) * kTileRows};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kTileRowBytes)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTileRowBytes),
                               static_cast<cuuint32_t>(kps * kTileRows)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The opt-in to more than 48 KB of dynamic shared memory is a function
// attribute held by each device's context, so it is set once per device and
// per kernel instantiation: a process that drives several GPUs must opt in on
// each of them.
constexpr int kMaxDevices = 64;

template <bool FP8, int EPI, bool PAIR>
cudaError_t opt_in_smem() {
    static_assert(sizeof(Maps) % 64 == 0, "tensor maps are 64-byte aligned");
    static std::once_flag once[kMaxDevices];
    static cudaError_t err[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    // Every launch asks for at most kDynSmemMax bytes (see the stage count
    // below); the 1 KB margin in it covers the compiler's padding of the
    // static shared block.
    std::call_once(once[dev], [dev] {
        err[dev] = cudaFuncSetAttribute(grouped_gemm_kernel<FP8, EPI, PAIR>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, kDynSmemMax);
    });
    return err[dev];
}

template <bool FP8, int EPI, bool PAIR>
cudaError_t launch_t(const Maps& maps, const GemmArgs& g, int grid, int smem, cudaStream_t s) {
    auto kern = grouped_gemm_kernel<FP8, EPI, PAIR>;
    const cudaError_t attr = opt_in_smem<FP8, EPI, PAIR>();
    if (attr != cudaSuccess) return attr;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads_for<EPI, PAIR>());
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    at[1].id = cudaLaunchAttributeClusterDimension;
    at[1].val.clusterDim.x = PAIR ? 2 : 1;
    at[1].val.clusterDim.y = 1;
    at[1].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = PAIR ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kern, maps, g);
}

template <bool FP8, bool PAIR>
cudaError_t launch_epi(int epi, const Maps& maps, const GemmArgs& g, int grid, int smem,
                       cudaStream_t s) {
    switch (epi) {
        case 0: return launch_t<FP8, 0, PAIR>(maps, g, grid, smem, s);
        case 1: return launch_t<FP8, 1, PAIR>(maps, g, grid, smem, s);
        case 2: return launch_t<FP8, 2, PAIR>(maps, g, grid, smem, s);
        default:
            // the adapter shrink exists for bf16 layers only
            if constexpr (FP8) return cudaErrorInvalidValue;
            else return launch_t<FP8, 3, PAIR>(maps, g, grid, smem, s);
    }
}

int pow2_at_least(int v) {
    int p = 32;
    while (p < v) p <<= 1;
    return p;
}

}  // namespace

int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
    return n > kMaxCtas ? kMaxCtas : n;
}

int gemm_nmax_for(int T, int k, int E) {
    // Twice the mean tokens per expert, in steps of 16 (16..256); experts with
    // more tokens are split into several token tiles.  Above 64 the tiles run
    // on CTA pairs, whose MMA N is a multiple of 32 (16 token rows per CTA),
    // so the cap is rounded to 32: every tile's MMA N then fits both the
    // per-k-block operand slot (nmax/2 rows per CTA) and the accumulator
    // stride (nmax columns).
    const long mean2 = (2L * T * k + E - 1) / E;
    long n = (mean2 + 15) & ~15L;
    if (n < 16) n = 16;
    if (n > 64) n = (n + 31) & ~31L;
    if (n > 256) n = 256;
    return static_cast<int>(n);
}

size_t gemm_partials_bytes(int nmax) {
    return static_cast<size_t>(kMaxCtas) * 2 * kBM * nmax * sizeof(float);
}

cudaError_t launch_grouped_gemm(const GemmProblem& p, cudaStream_t s) {
    GemmArgs g{};
    g.E = p.E;
    g.Mw = p.Mw;
    g.K = p.K;
    g.Mvalid = p.Mvalid;
    g.nmax = p.nmax;
    g.KBm = p.KB;
    g.KBx = p.KBx;
    g.KB = p.KB + p.KBx;
    g.MT = p.MT;
    g.x_tiles = static_cast<const uint8_t*>(p.x_tiles);
    g.adapter = p.adapter;
    g.lscale = p.lscale;
    g.lrank = p.lrank;
    g.lR = p.lR;
    // Large token tiles run on CTA pairs (M = 256 per MMA, each CTA loads
    // half of every token tile); weight streaming runs one CTA per SM.
    const bool pair = p.nmax > 64;
    g.MTu = pair ? (p.MT + 1) / 2 : p.MT;
    g.a_tiles = static_cast<const uint8_t*>(p.weights);
    // Stages of several k-blocks each: small token tiles (weight streaming)
    // take 2 stages of 4 k-blocks (64 KB weight copies), large ones 3 stages
    // of 2 (32 KB weights + 32 KB activations per CTA).  Measured on B200:
    // fewer, larger copies sustain more bandwidth than many 16 KB stages, for
    // both regimes.
    const int kps = pair ? kps_for<true>() : kps_for<false>();
    const int stage_bytes = kps * (kATileBytes + (pair ? p.nmax / 2 : p.nmax) * kRowBytes);
    int stages = (kDynSmemMax - 1024 - kStagingBytes) / stage_bytes;
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 2) return cudaErrorInvalidValue;
    const int smem = 1024 + stages * stage_bytes + kStagingBytes;
    g.stages = stages;
    g.tmem_cols = pow2_at_least(2 * p.nmax);
    g.ldo = p.ldo;
    g.out = p.out;
    g.counts = p.counts;
    g.offsets = p.offsets;
    g.sorted_ids = p.sorted_ids;
    g.ktop = p.ktop;
    g.A = p.A;
    g.capacity = p.capacity;
    g.gather_src = static_cast<const uint8_t*>(p.gather_src);
    g.src_row_bytes = static_cast<long long>(p.K) * (p.fp8 ? 1 : 2);
    g.w = p.w;
    g.w_scales = p.w_scales;
    g.act_amax = p.act_amax;
    g.out_amax = p.out_amax;
    g.acc_zero = p.acc_zero;
    g.acc_zero_vec4 = static_cast<long long>(p.acc_zero_floats / 4);
    g.partials = p.partials;
    g.counters = p.counters;
    g.status = p.status;
    g.sched_after_wait = p.sched_after_wait ? 1 : 0;
    if (p.epi == 0 && !pair && (!p.gather_src || !p.sorted_ids || p.ktop < 1))
        return cudaErrorInvalidValue;
    if ((p.epi == 1 || p.epi == 2) && (!p.sorted_ids || !p.w)) return cudaErrorInvalidValue;
    if (p.epi == 3 && !p.sorted_ids) return cudaErrorInvalidValue;
    if (p.acc_zero_floats % 4 != 0) return cudaErrorInvalidValue;
    if (p.KBx > 0 && (p.fp8 || !p.x_tiles || !p.x_rows)) return cudaErrorInvalidValue;
    if (p.epi == 3 && (p.fp8 || !p.adapter || !p.lscale || p.lrank < 1 || p.lR > 64))
        return cudaErrorInvalidValue;
    Maps maps;
    memset(&maps, 0, sizeof(maps));
    // activation rows in permuted order come by TMA; a one-CTA gate/up
    // kernel gathers its rows itself and uses no activation maps
    const bool gathers = p.epi == 0 && !pair;
    if (!gathers && (!p.act || !make_map(&maps.b128, p.act, p.fp8, p.K, p.capacity, 128) ||
                     !make_map(&maps.b64, p.act, p.fp8, p.K, p.capacity, 64) ||
                     !make_map(&maps.b16, p.act, p.fp8, p.K, p.capacity, 16)))
        return cudaErrorInvalidValue;
    const long wtiles = static_cast<long>(p.E) * p.MT * p.KB;
    if (pair && !make_tile_map(&maps.a, p.weights, wtiles, kps)) return cudaErrorInvalidValue;
    if (p.KBx > 0) {
        // adapter expand: rows of the shrink outputs (bf16, KBx * 64 wide)
        // and, for pairs, both weight sources one tile per box
        const int xk = p.KBx * 64;
        if (!make_map(&maps.l128, p.x_rows, false, xk, p.capacity, 128) ||
            !make_map(&maps.l64, p.x_rows, false, xk, p.capacity, 64) ||
            !make_map(&maps.l16, p.x_rows, false, xk, p.capacity, 16))
            return cudaErrorInvalidValue;
        if (pair && (!make_tile_map(&maps.a1, p.weights, wtiles, 1) ||
                     !make_tile_map(&maps.al, p.x_tiles,
                                    static_cast<long>(p.E) * p.MT * p.KBx, 1)))
            return cudaErrorInvalidValue;
    }
    int grid = device_sm_count();
    if (p.max_ctas > 0 && p.max_ctas < grid) grid = p.max_ctas;
    if (pair) grid = grid < 2 ? 2 : grid & ~1;
    if (pair)
        return p.fp8 ? launch_epi<true, true>(p.epi, maps, g, grid, smem, s)
                     : launch_epi<false, true>(p.epi, maps, g, grid, smem, s);
    return p.fp8 ? launch_epi<true, false>(p.epi, maps, g, grid, smem, s)
                 : launch_epi<false, false>(p.epi, maps, g, grid, smem, s);
}

}  // namespace moe
