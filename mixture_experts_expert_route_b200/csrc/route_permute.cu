// route_permute.cu -- a1 (router top-k) and a2 (token permutation).
//
// a1: one warp per token.  Each lane holds E/32 logits in registers; k rounds
//     of a warp-wide arg-max under a total order (larger first, equal values
//     and -0/+0 to the lower index, NaN last) pick the experts; the weights are
//     a softmax over the selected logits.  Router of "Amazon SageMaker AIにおける
//     Mixture-of-Expertsカーネル最適化の深掘り", § "Mixture-of-Experts (MoE)
//     モデルの原理と推論における課題".
// a2: the "data reordering" of "Az AWS új MoE-optimalizációkkal gyorsítja a
//     SageMaker AI-t", § "A fused MoE a számítási folyamat több lépését
//     egyesíti": a stable counting sort of the assignments by expert, with no
//     atomics.  Assignments are cut into chunks (all of them, up to 2048, in
//     the single-CTA kernel; 512 per CTA otherwise), a slice per warp; each
//     warp counts its slice with __match_any_sync (the lowest lane of each
//     group of equal ids adds the group size to the warp's private histogram),
//     per-expert prefix sums over (chunk, warp) give every warp a start
//     position per expert, and a second pass places each assignment at
//     start + its rank among equal ids in its 32-wide round.  Lower flat
//     indices always land first, so the result is deterministic and equals the
//     stable sort.
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kThreads = 256;        // multi-CTA kernels: 8 warps
constexpr int kSmallThreads = 512;   // single-CTA kernel: 16 warps
constexpr int kStageFloats = 4096;   // logits staged in smem by the single-CTA kernel
constexpr unsigned kFull = 0xffffffffu;
// Multi-CTA permutation: assignments per chunk (one CTA of 8 warps, 64 per
// warp).  Small chunks give a few-thousand-token batch dozens of CTAs; the
// per-chunk counters (nchunks x E) are scanned in batches of independent loads.
constexpr int kPermChunk = 512;
constexpr int kScanBatch = 16;

// Selection order as one 64-bit key, larger first: an order-preserving map of
// the logit (-0 folded onto +0; NaN below every number) in the high word and
// the complement of the expert index in the low word (equal logits: the lower
// index wins).  Key 0 marks an expert already taken or past E.
__device__ __forceinline__ uint64_t select_key(float f, int e) {
    uint32_t b = __float_as_uint(f);
    if (b == 0x80000000u) b = 0u;
    const uint32_t ord = isnan(f) ? 0u : ((b & 0x80000000u) ? ~b : (b | 0x80000000u));
    return (static_cast<uint64_t>(ord) << 32) | (0xffffffffu - static_cast<uint32_t>(e));
}

// The logit of a key (exact, except -0 reads as +0 and a NaN as the canonical
// NaN; neither changes exp(l - m)).
__device__ __forceinline__ float key_value(uint64_t key) {
    const uint32_t ord = static_cast<uint32_t>(key >> 32);
    if (ord == 0u) return __uint_as_float(0x7fffffffu);
    return __uint_as_float((ord & 0x80000000u) ? (ord & 0x7fffffffu) : ~ord);
}

// Top-k of row[0..E) by one warp (row in global or shared memory).  Each lane
// keys its E/32 logits once; a selection round is a local max of the lane's
// keys and a five-step warp max, after which the owning lane clears the
// winner.  The j-th selection (id and logit) is kept in registers of lane
// j % 32, slot j / 32; the weights are a softmax over the selected logits,
// summed per lane in ascending j and then across the warp.  ids and w are
// written once at the end, lane j for entry j.
template <int EPL>
__device__ void warp_topk(const float* row, int E, int k, int32_t* ids, float* w,
                          int32_t* ids_copy = nullptr) {
    const int lane = threadIdx.x & 31;
    uint64_t key[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        key[i] = e < E ? select_key(row[e], e) : 0ull;
    }
    float sv[EPL];
    int si[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        sv[i] = 0.0f;
        si[i] = 0;
    }
    float m = 0.0f;
    for (int j = 0; j < k; ++j) {
        uint64_t best = key[0];
#pragma unroll
        for (int i = 1; i < EPL; ++i) best = key[i] > best ? key[i] : best;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const uint64_t o = __shfl_xor_sync(kFull, best, off);
            best = o > best ? o : best;
        }
        const int bi = static_cast<int>(0xffffffffu - static_cast<uint32_t>(best));
        const float bv = key_value(best);
        // selects, not indexed stores, so the arrays stay in registers
        const bool won = (bi & 31) == lane, keep = (j & 31) == lane;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            key[i] = (won && i == (bi >> 5)) ? 0ull : key[i];
            const bool here = keep && i == (j >> 5);
            sv[i] = here ? bv : sv[i];
            si[i] = here ? bi : si[i];
        }
        if (j == 0) m = bv;
    }
    float z = 0.0f;
#pragma unroll
    for (int i = 0; i < EPL; ++i)
        if (lane + 32 * i < k) z += expf(sv[i] - m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(kFull, z, off);
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int j = lane + 32 * i;
        if (j < k) {
            ids[j] = si[i];
            if (ids_copy) ids_copy[j] = si[i];
            w[j] = expf(sv[i] - m) / z;
        }
    }
    __syncwarp();
}

__device__ void zero_ctl(int32_t* ctl, int n, int tid, int nthreads) {
    for (int i = tid; i < n; i += nthreads) ctl[i] = 0;
}

template <int EPL>
__global__ void __launch_bounds__(kThreads)
    route_topk_kernel(const float* __restrict__ logits, int T, int E, int k, int32_t* ids,
                      float* w, int32_t* ctl, int ctl_ints) {
    pdl_wait();
    pdl_trigger();
    if (blockIdx.x == 0 && ctl) zero_ctl(ctl, ctl_ints, threadIdx.x, kThreads);
    const int warp = threadIdx.x >> 5;
    const long t = static_cast<long>(blockIdx.x) * (kThreads / 32) + warp;
    if (t >= T) return;
    warp_topk<EPL>(logits + t * E, E, k, ids + t * k, w + t * k);
}

// hist[w][e] += number of assignments of warp w's slice of the chunk routed to e
template <int NW, int CHUNK>
__device__ void chunk_histogram(const int32_t* ids, long A, long chunk_base, int E,
                                int (*hist)[kMaxExperts], int32_t* status) {
    constexpr int kPerWarp = CHUNK / NW;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long wbase = chunk_base + static_cast<long>(warp) * kPerWarp;
    for (int r = 0; r < kPerWarp / 32; ++r) {
        const long f = wbase + r * 32 + lane;
        int e = -1;
        if (f < A) {
            e = ids[f];
            if (e < 0 || e >= E) {
                report(status, MOE_ERR_DEVICE);
                e = -1;
            }
        }
        const unsigned peers = __match_any_sync(kFull, e);
        if (e >= 0 && lane == __ffs(peers) - 1) hist[warp][e] += __popc(peers);
        __syncwarp();
    }
}

// Places the warp's slice: base[w][e] holds the next free slot of expert e.
template <int NW, int CHUNK>
__device__ void chunk_scatter(const int32_t* ids, long A, long chunk_base, int E,
                              int (*base)[kMaxExperts], int32_t* sorted_ids, int32_t* inv_perm) {
    constexpr int kPerWarp = CHUNK / NW;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long wbase = chunk_base + static_cast<long>(warp) * kPerWarp;
    for (int r = 0; r < kPerWarp / 32; ++r) {
        const long f = wbase + r * 32 + lane;
        int e = -1;
        if (f < A) {
            e = ids[f];
            if (e < 0 || e >= E) e = -1;
        }
        const unsigned peers = __match_any_sync(kFull, e);
        if (e >= 0) {
            const int pos = base[warp][e] + __popc(peers & ((1u << lane) - 1u));
            sorted_ids[pos] = static_cast<int32_t>(f);
            inv_perm[f] = pos;
        }
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) base[warp][e] += __popc(peers);
        __syncwarp();
    }
}

// Exclusive scan of one value per thread over the NT threads of the block.
template <int NT>
__device__ int block_exclusive_scan(int v, int* tmp /* NT/32 + 1 */) {
    constexpr int NW = NT / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(kFull, inc, off);
        if (lane >= off) inc += o;
    }
    if (lane == 31) tmp[warp] = inc;
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int i = 0; i < NW; ++i) {
            const int t = tmp[i];
            tmp[i] = run;
            run += t;
        }
        tmp[NW] = run;
    }
    __syncthreads();
    return tmp[warp] + inc - v;
}

// Thread e < E: given the total count c of expert e, writes counts, offsets,
// tiles and the pads of e's block; returns o_e.  All threads must call it.
template <int NT>
__device__ int finish_offsets(int c, int E, int block_m, int32_t* counts, int32_t* offsets,
                              int32_t* sorted_ids, int32_t* tiles, int32_t* num_tiles,
                              int* tmp) {
    const int e = threadIdx.x;
    const int padded = (e < E) ? (c + block_m - 1) / block_m * block_m : 0;
    const int o = block_exclusive_scan<NT>(padded, tmp);
    if (e < E) {
        counts[e] = c;
        offsets[e] = o;
        for (int b = o / block_m; b < (o + padded) / block_m; ++b) tiles[b] = e;
        for (int p = o + c; p < o + padded; ++p) sorted_ids[p] = -1;
        if (e == E - 1) {
            offsets[E] = o + padded;
            *num_tiles = (o + padded) / block_m;
        }
    }
    return o;
}

template <int NT>
__device__ void fill_tail(int total, int block_m, int capacity, int32_t* sorted_ids,
                          int32_t* tiles) {
    for (int p = total + threadIdx.x; p < capacity; p += NT) sorted_ids[p] = -1;
    for (int b = total / block_m + threadIdx.x; b < capacity / block_m; b += NT) tiles[b] = -1;
}

// One CTA of 16 warps: optional routing of all T tokens (logits staged in
// shared memory when they fit), then the whole permutation of A = T*k <=
// kChunk assignments; for FP8 batches with a small x, also amax(x) and the
// e4m3 codes of x.
template <int EPL>
__global__ void __launch_bounds__(kSmallThreads)
    route_permute_small_kernel(const float* __restrict__ logits, int T, int E, int k, int block_m,
                               int capacity, int32_t* ids, float* w, int32_t* counts,
                               int32_t* offsets, int32_t* sorted_ids, int32_t* inv_perm,
                               int32_t* tiles, int32_t* num_tiles, int32_t* status, int32_t* ctl,
                               int ctl_ints, const uint4* __restrict__ x, long x_vecs,
                               uint32_t* amax_out, uint2* __restrict__ xq_out) {
    constexpr int NW = kSmallThreads / 32;
    __shared__ int hist[NW][kMaxExperts];
    __shared__ float slog[kStageFloats];
    __shared__ int tmp[NW + 1];
    __shared__ int32_t sids[kChunk];   // the ids, read twice below
    __shared__ float wmax[NW];
    const int warp = threadIdx.x >> 5;
    const long A = static_cast<long>(T) * k;
    pdl_wait();
    pdl_trigger();
    if (ctl) zero_ctl(ctl, ctl_ints, threadIdx.x, kSmallThreads);
    if (logits) {
        const int n = T * E;
        const float* src = logits;
        if (n <= kStageFloats) {
            for (int i = threadIdx.x; i < n; i += kSmallThreads) slog[i] = logits[i];
            __syncthreads();
            src = slog;
        }
        for (int t = warp; t < T; t += NW)
            warp_topk<EPL>(src + static_cast<long>(t) * E, E, k, ids + static_cast<long>(t) * k,
                           w + static_cast<long>(t) * k, sids + static_cast<long>(t) * k);
    } else {
        for (int i = threadIdx.x; i < A; i += kSmallThreads) sids[i] = ids[i];
    }
    for (int i = threadIdx.x; i < NW * kMaxExperts; i += kSmallThreads) (&hist[0][0])[i] = 0;
    __syncthreads();
    // FP8 small batches: amax of x (a3's scale) here, saving a kernel; the
    // control block was zeroed above, before the barrier
    float xm = 0.0f;
    if (amax_out) {
        for (long i = threadIdx.x; i < x_vecs; i += kSmallThreads) xm = fmaxf(xm, amax8(x[i]));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) xm = fmaxf(xm, __shfl_xor_sync(kFull, xm, off));
        if ((threadIdx.x & 31) == 0) wmax[warp] = xm;
    }
    chunk_histogram<NW, kChunk>(sids, A, 0, E, hist, status);
    __syncthreads();
    if (amax_out) {
        for (int i = 0; i < NW; ++i) xm = fmaxf(xm, wmax[i]);
        if (threadIdx.x == 0) *amax_out = __float_as_uint(xm);
        // and the e4m3 codes of x (token order), which the gate/up GEMM gathers
        if (xq_out) {
            const float sx = fp8_scale_from_amax(__float_as_uint(xm));
            const float inv = 1.0f / sx;
            for (long i = threadIdx.x; i < x_vecs; i += kSmallThreads)
                xq_out[i] = quant8(x[i], inv, sx);
        }
    }
    const int e = threadIdx.x;
    int c = 0;
    if (e < E)
        for (int wq = 0; wq < NW; ++wq) c += hist[wq][e];
    const int o = finish_offsets<kSmallThreads>(c, E, block_m, counts, offsets, sorted_ids, tiles,
                                                num_tiles, tmp);
    if (e < E) {
        int run = o;
        for (int wq = 0; wq < NW; ++wq) {
            const int h = hist[wq][e];
            hist[wq][e] = run;
            run += h;
        }
    }
    const int total = tmp[NW];
    __syncthreads();
    fill_tail<kSmallThreads>(total, block_m, capacity, sorted_ids, tiles);
    chunk_scatter<NW, kChunk>(sids, A, 0, E, hist, sorted_ids, inv_perm);
}

__global__ void __launch_bounds__(kThreads)
    permute_count_kernel(const int32_t* ids, long A, int E, int32_t* __restrict__ chunk_counts,
                         int32_t* status) {
    constexpr int NW = kThreads / 32;
    __shared__ int hist[NW][kMaxExperts];
    pdl_wait();
    pdl_trigger();
    for (int i = threadIdx.x; i < NW * kMaxExperts; i += kThreads) (&hist[0][0])[i] = 0;
    __syncthreads();
    chunk_histogram<NW, kPermChunk>(ids, A, static_cast<long>(blockIdx.x) * kPermChunk, E, hist,
                                    status);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kThreads) {
        int c = 0;
        for (int wq = 0; wq < NW; ++wq) c += hist[wq][e];
        chunk_counts[static_cast<long>(blockIdx.x) * E + e] = c;
    }
}

// Scan + scatter: every CTA sums the per-chunk counts itself (all chunks for
// the expert totals and padded offsets, the chunks before its own for its
// start positions), so no separate scan kernel runs; CTA 0 also writes the
// counts, offsets, tile list and pads.  Then the chunk's assignments are
// placed as in the single-CTA kernel.
__global__ void __launch_bounds__(kThreads)
    scan_scatter_kernel(const int32_t* ids, long A, int E, int block_m, int capacity,
                        int nchunks, const int32_t* __restrict__ chunk_counts, int32_t* counts,
                        int32_t* offsets, int32_t* sorted_ids, int32_t* __restrict__ inv_perm,
                        int32_t* tiles, int32_t* num_tiles) {
    constexpr int NW = kThreads / 32;
    __shared__ int hist[NW][kMaxExperts];
    __shared__ int tmp[NW + 1];
    pdl_wait();
    pdl_trigger();
    const int e = threadIdx.x;
    const int me = blockIdx.x;
    int total = 0, before = 0;
    if (e < E)
        for (int c0 = 0; c0 < nchunks; c0 += kScanBatch) {
            // the batch's loads are independent: issue them all, then add
            int v[kScanBatch];
#pragma unroll
            for (int i = 0; i < kScanBatch; ++i)
                v[i] = c0 + i < nchunks ? chunk_counts[static_cast<long>(c0 + i) * E + e] : 0;
#pragma unroll
            for (int i = 0; i < kScanBatch; ++i) {
                if (c0 + i < me) before += v[i];
                total += v[i];
            }
        }
    int o;
    if (me == 0) {
        o = finish_offsets<kThreads>(total, E, block_m, counts, offsets, sorted_ids, tiles,
                                     num_tiles, tmp);
        const int all = tmp[NW];
        __syncthreads();
        fill_tail<kThreads>(all, block_m, capacity, sorted_ids, tiles);
    } else {
        const int padded = e < E ? (total + block_m - 1) / block_m * block_m : 0;
        o = block_exclusive_scan<kThreads>(padded, tmp);
    }
    for (int i = threadIdx.x; i < NW * kMaxExperts; i += kThreads) (&hist[0][0])[i] = 0;
    __syncthreads();
    const long base = static_cast<long>(me) * kPermChunk;
    chunk_histogram<NW, kPermChunk>(ids, A, base, E, hist, nullptr);
    __syncthreads();
    if (e < E) {
        int run = o + before;
        for (int wq = 0; wq < NW; ++wq) {
            const int h = hist[wq][e];
            hist[wq][e] = run;
            run += h;
        }
    }
    __syncthreads();
    chunk_scatter<NW, kPermChunk>(ids, A, base, E, hist, sorted_ids, inv_perm);
}

int epl_for(int E) { return E <= 32 ? 1 : E <= 64 ? 2 : E <= 128 ? 4 : 8; }

cudaError_t launch_scan_scatter(const int32_t* ids, long A, int E, int block_m, int capacity,
                                int nch, const int32_t* chunk_counts, int32_t* counts,
                                int32_t* offsets, int32_t* sorted_ids, int32_t* inv_perm,
                                int32_t* tiles, int32_t* num_tiles, cudaStream_t s) {
    return launch_pdl(scan_scatter_kernel, dim3(nch), dim3(kThreads), 0, s, ids, A, E, block_m,
                      capacity, nch, chunk_counts, counts, offsets, sorted_ids, inv_perm, tiles,
                      num_tiles);
}

}  // namespace

// 1 when the single-CTA kernel handles all A assignments, else the number of
// chunks (and per-chunk counter rows) of the multi-CTA path.
int permute_chunks(long A) {
    return A <= kChunk ? 1 : static_cast<int>((A + kPermChunk - 1) / kPermChunk);
}

bool fused_route_permute_ok(int T, int k) {
    return T <= kSmallT && static_cast<long>(T) * k <= kChunk;
}

cudaError_t launch_route_topk(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                              cudaStream_t s, int32_t* ctl, int ctl_ints) {
    if (T == 0) return cudaSuccess;
    const dim3 grid((T + kThreads / 32 - 1) / (kThreads / 32));
    switch (epl_for(E)) {
        case 1: return launch_pdl(route_topk_kernel<1>, grid, dim3(kThreads), 0, s, logits, T, E, k, ids, w, ctl, ctl_ints);
        case 2: return launch_pdl(route_topk_kernel<2>, grid, dim3(kThreads), 0, s, logits, T, E, k, ids, w, ctl, ctl_ints);
        case 4: return launch_pdl(route_topk_kernel<4>, grid, dim3(kThreads), 0, s, logits, T, E, k, ids, w, ctl, ctl_ints);
        default: return launch_pdl(route_topk_kernel<8>, grid, dim3(kThreads), 0, s, logits, T, E, k, ids, w, ctl, ctl_ints);
    }
}

cudaError_t launch_route_permute_small(const float* logits, int T, int E, int k, int block_m,
                                       int capacity, int32_t* ids, float* w, int32_t* counts,
                                       int32_t* offsets, int32_t* sorted_ids, int32_t* inv_perm,
                                       int32_t* tiles, int32_t* num_tiles, int32_t* status,
                                       cudaStream_t s, int32_t* ctl, int ctl_ints, const void* x,
                                       long x_elems, uint32_t* amax_out, void* xq_out) {
    const uint4* xv = static_cast<const uint4*>(x);
    uint2* xq = static_cast<uint2*>(xq_out);
    const long nv = x_elems / 8;
#define MOE_SMALL(EPL)                                                                            \
    return launch_pdl(route_permute_small_kernel<EPL>, dim3(1), dim3(kSmallThreads), 0, s, logits, \
                      T, E, k, block_m, capacity, ids, w, counts, offsets, sorted_ids, inv_perm,  \
                      tiles, num_tiles, status, ctl, ctl_ints, xv, nv, amax_out, xq)
    switch (epl_for(E)) {
        case 1: MOE_SMALL(1);
        case 2: MOE_SMALL(2);
        case 4: MOE_SMALL(4);
        default: MOE_SMALL(8);
    }
#undef MOE_SMALL
}

cudaError_t launch_align_permute(const int32_t* ids, int T, int k, int E, int block_m,
                                 int capacity, int32_t* counts, int32_t* offsets,
                                 int32_t* sorted_ids, int32_t* inv_perm, int32_t* tiles,
                                 int32_t* num_tiles, int32_t* chunk_counts, int32_t* status,
                                 cudaStream_t s) {
    const long A = static_cast<long>(T) * k;
    const int nch = permute_chunks(A);
    if (nch <= 1)
        return launch_route_permute_small(nullptr, T, E, k, block_m, capacity,
                                          const_cast<int32_t*>(ids), nullptr, counts, offsets,
                                          sorted_ids, inv_perm, tiles, num_tiles, status, s,
                                          nullptr, 0);
    cudaError_t e = launch_pdl(permute_count_kernel, dim3(nch), dim3(kThreads), 0, s, ids, A, E,
                               chunk_counts, status);
    if (e == cudaSuccess)
        e = launch_scan_scatter(ids, A, E, block_m, capacity, nch, chunk_counts, counts, offsets,
                                sorted_ids, inv_perm, tiles, num_tiles, s);
    return e;
}

}  // namespace moe
