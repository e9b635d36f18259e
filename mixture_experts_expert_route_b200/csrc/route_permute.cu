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
//     atomics.  Assignments are cut into chunks of 2048 (256 per warp); each
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

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kPerWarp = kChunk / kWarps;  // 256 assignments per warp per chunk
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ bool beats(float a, int ia, float b, int ib) {
    const bool na = isnan(a), nb = isnan(b);
    if (na || nb) {
        if (na && nb) return ia < ib;
        return nb;
    }
    if (a != b) return a > b;
    return ia < ib;
}

// Top-k of row[0..E) by one warp; sel is this warp's scratch of >= k floats.
template <int EPL>
__device__ void warp_topk(const float* __restrict__ row, int E, int k, int32_t* __restrict__ ids,
                          float* __restrict__ w, float* sel) {
    const int lane = threadIdx.x & 31;
    float v[EPL];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? row[e] : 0.0f;
        if (e >= E) taken |= 1u << i;
    }
    for (int j = 0; j < k; ++j) {
        float bv = 0.0f;
        int bi = INT_MAX;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            if (taken & (1u << i)) continue;
            const int e = lane + 32 * i;
            if (bi == INT_MAX || beats(v[i], e, bv, bi)) {
                bv = v[i];
                bi = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(kFull, bv, off);
            const int oi = __shfl_xor_sync(kFull, bi, off);
            if (oi != INT_MAX && (bi == INT_MAX || beats(ov, oi, bv, bi))) {
                bv = ov;
                bi = oi;
            }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == 0) {
            ids[j] = bi;
            sel[j] = bv;
        }
    }
    __syncwarp();
    const float m = sel[0];
    float z = 0.0f;
    for (int j = lane; j < k; j += 32) z += expf(sel[j] - m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(kFull, z, off);
    for (int j = lane; j < k; j += 32) w[j] = expf(sel[j] - m) / z;
    __syncwarp();
}

template <int EPL>
__global__ void __launch_bounds__(kThreads) route_topk_kernel(const float* __restrict__ logits,
                                                              int T, int E, int k,
                                                              int32_t* __restrict__ ids,
                                                              float* __restrict__ w) {
    __shared__ float sel[kWarps][kMaxExperts];
    const int warp = threadIdx.x >> 5;
    const long t = static_cast<long>(blockIdx.x) * kWarps + warp;
    if (t >= T) return;
    warp_topk<EPL>(logits + t * E, E, k, ids + t * k, w + t * k, sel[warp]);
}

// hist[w][e] += number of assignments of warp w's slice of the chunk routed to e
__device__ void chunk_histogram(const int32_t* __restrict__ ids, long A, long chunk_base, int E,
                                int (*hist)[kMaxExperts], int32_t* status) {
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
__device__ void chunk_scatter(const int32_t* __restrict__ ids, long A, long chunk_base, int E,
                              int (*base)[kMaxExperts], int32_t* __restrict__ sorted_ids,
                              int32_t* __restrict__ inv_perm) {
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

// Exclusive scan over the 256 threads of the block.
__device__ int block_exclusive_scan(int v, int* tmp /* kWarps + 1 */) {
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
        for (int i = 0; i < kWarps; ++i) {
            const int t = tmp[i];
            tmp[i] = run;
            run += t;
        }
        tmp[kWarps] = run;
    }
    __syncthreads();
    return tmp[warp] + inc - v;
}

// Thread e < E: given the total count c of expert e, writes counts, offsets,
// tiles and the pads of e's block; returns o_e.  All threads must call it.
__device__ int finish_offsets(int c, int E, int block_m, int32_t* counts, int32_t* offsets,
                              int32_t* sorted_ids, int32_t* tiles, int32_t* num_tiles,
                              int* tmp) {
    const int e = threadIdx.x;
    const int padded = (e < E) ? (c + block_m - 1) / block_m * block_m : 0;
    const int o = block_exclusive_scan(padded, tmp);
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

__device__ void fill_tail(int total, int block_m, int capacity, int32_t* sorted_ids,
                          int32_t* tiles) {
    for (int p = total + threadIdx.x; p < capacity; p += kThreads) sorted_ids[p] = -1;
    for (int b = total / block_m + threadIdx.x; b < capacity / block_m; b += kThreads)
        tiles[b] = -1;
}

// One CTA: optional routing of all T tokens, then the whole permutation of
// A = T*k <= kChunk assignments.
template <int EPL>
__global__ void __launch_bounds__(kThreads)
    route_permute_small_kernel(const float* __restrict__ logits, int T, int E, int k, int block_m,
                               int capacity, int32_t* ids, float* w, int32_t* counts,
                               int32_t* offsets, int32_t* sorted_ids, int32_t* inv_perm,
                               int32_t* tiles, int32_t* num_tiles, int32_t* status) {
    __shared__ int hist[kWarps][kMaxExperts];
    __shared__ float sel[kWarps][kMaxExperts];
    __shared__ int tmp[kWarps + 1];
    const int warp = threadIdx.x >> 5;
    const long A = static_cast<long>(T) * k;
    if (logits) {
        for (int t = warp; t < T; t += kWarps)
            warp_topk<EPL>(logits + static_cast<long>(t) * E, E, k, ids + static_cast<long>(t) * k,
                           w + static_cast<long>(t) * k, sel[warp]);
    }
    for (int i = threadIdx.x; i < kWarps * kMaxExperts; i += kThreads) (&hist[0][0])[i] = 0;
    __syncthreads();
    chunk_histogram(ids, A, 0, E, hist, status);
    __syncthreads();
    const int e = threadIdx.x;
    int c = 0;
    if (e < E)
        for (int wq = 0; wq < kWarps; ++wq) c += hist[wq][e];
    const int o = finish_offsets(c, E, block_m, counts, offsets, sorted_ids, tiles, num_tiles, tmp);
    if (e < E) {
        int run = o;
        for (int wq = 0; wq < kWarps; ++wq) {
            const int h = hist[wq][e];
            hist[wq][e] = run;
            run += h;
        }
    }
    const int total = tmp[kWarps];
    __syncthreads();
    fill_tail(total, block_m, capacity, sorted_ids, tiles);
    chunk_scatter(ids, A, 0, E, hist, sorted_ids, inv_perm);
}

__global__ void __launch_bounds__(kThreads)
    permute_count_kernel(const int32_t* __restrict__ ids, long A, int E,
                         int32_t* __restrict__ chunk_counts, int32_t* status) {
    __shared__ int hist[kWarps][kMaxExperts];
    for (int i = threadIdx.x; i < kWarps * kMaxExperts; i += kThreads) (&hist[0][0])[i] = 0;
    __syncthreads();
    chunk_histogram(ids, A, static_cast<long>(blockIdx.x) * kChunk, E, hist, status);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kThreads) {
        int c = 0;
        for (int wq = 0; wq < kWarps; ++wq) c += hist[wq][e];
        chunk_counts[static_cast<long>(blockIdx.x) * E + e] = c;
    }
}

__global__ void __launch_bounds__(kThreads)
    permute_scan_kernel(int nchunks, int E, int block_m, int capacity, int32_t* chunk_counts,
                        int32_t* counts, int32_t* offsets, int32_t* sorted_ids, int32_t* tiles,
                        int32_t* num_tiles) {
    __shared__ int tmp[kWarps + 1];
    const int e = threadIdx.x;
    int run = 0;
    if (e < E)
        for (int c = 0; c < nchunks; ++c) {
            const int v = chunk_counts[static_cast<long>(c) * E + e];
            chunk_counts[static_cast<long>(c) * E + e] = run;
            run += v;
        }
    finish_offsets(run, E, block_m, counts, offsets, sorted_ids, tiles, num_tiles, tmp);
    const int total = tmp[kWarps];
    __syncthreads();
    fill_tail(total, block_m, capacity, sorted_ids, tiles);
}

__global__ void __launch_bounds__(kThreads)
    permute_scatter_kernel(const int32_t* __restrict__ ids, long A, int E,
                           const int32_t* __restrict__ chunk_prefix,
                           const int32_t* __restrict__ offsets, int32_t* __restrict__ sorted_ids,
                           int32_t* __restrict__ inv_perm) {
    __shared__ int hist[kWarps][kMaxExperts];
    for (int i = threadIdx.x; i < kWarps * kMaxExperts; i += kThreads) (&hist[0][0])[i] = 0;
    __syncthreads();
    const long base = static_cast<long>(blockIdx.x) * kChunk;
    chunk_histogram(ids, A, base, E, hist, nullptr);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kThreads) {
        int run = offsets[e] + chunk_prefix[static_cast<long>(blockIdx.x) * E + e];
        for (int wq = 0; wq < kWarps; ++wq) {
            const int h = hist[wq][e];
            hist[wq][e] = run;
            run += h;
        }
    }
    __syncthreads();
    chunk_scatter(ids, A, base, E, hist, sorted_ids, inv_perm);
}

int epl_for(int E) { return E <= 32 ? 1 : E <= 64 ? 2 : E <= 128 ? 4 : 8; }

}  // namespace

int permute_chunks(long A) { return static_cast<int>((A + kChunk - 1) / kChunk); }

bool fused_route_permute_ok(int T, int k) {
    return T <= kSmallT && static_cast<long>(T) * k <= kChunk;
}

cudaError_t launch_route_topk(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                              cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const dim3 grid((T + kWarps - 1) / kWarps);
    switch (epl_for(E)) {
        case 1: route_topk_kernel<1><<<grid, kThreads, 0, s>>>(logits, T, E, k, ids, w); break;
        case 2: route_topk_kernel<2><<<grid, kThreads, 0, s>>>(logits, T, E, k, ids, w); break;
        case 4: route_topk_kernel<4><<<grid, kThreads, 0, s>>>(logits, T, E, k, ids, w); break;
        default: route_topk_kernel<8><<<grid, kThreads, 0, s>>>(logits, T, E, k, ids, w); break;
    }
    return cudaGetLastError();
}

cudaError_t launch_route_permute_small(const float* logits, int T, int E, int k, int block_m,
                                       int capacity, int32_t* ids, float* w, int32_t* counts,
                                       int32_t* offsets, int32_t* sorted_ids, int32_t* inv_perm,
                                       int32_t* tiles, int32_t* num_tiles, int32_t* status,
                                       cudaStream_t s) {
#define MOE_SMALL(EPL)                                                                          \
    route_permute_small_kernel<EPL><<<1, kThreads, 0, s>>>(logits, T, E, k, block_m, capacity, \
                                                           ids, w, counts, offsets, sorted_ids, \
                                                           inv_perm, tiles, num_tiles, status)
    switch (epl_for(E)) {
        case 1: MOE_SMALL(1); break;
        case 2: MOE_SMALL(2); break;
        case 4: MOE_SMALL(4); break;
        default: MOE_SMALL(8); break;
    }
#undef MOE_SMALL
    return cudaGetLastError();
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
                                          sorted_ids, inv_perm, tiles, num_tiles, status, s);
    permute_count_kernel<<<nch, kThreads, 0, s>>>(ids, A, E, chunk_counts, status);
    permute_scan_kernel<<<1, kThreads, 0, s>>>(nch, E, block_m, capacity, chunk_counts, counts,
                                               offsets, sorted_ids, tiles, num_tiles);
    permute_scatter_kernel<<<nch, kThreads, 0, s>>>(ids, A, E, chunk_counts, offsets, sorted_ids,
                                                    inv_perm);
    return cudaGetLastError();
}

}  // namespace moe
