// elementwise.cu -- the layer's memory-bound steps around the GEMMs: the FP8
// quantisation of x (a3; its gather is fused into the gate/up GEMM's operand
// loads) and of h (a5), the combine (a7: the deterministic gather-sum, or the
// conversion of the fused fp32 accumulator), the one-time weight packing, and
// the failure-detection self-test.  All are HBM-bound: 16-byte vector
// accesses, one vector per thread, grids sized from the data.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kThreads = 256;

// One 16-byte vector per thread: a small batch still has thousands of loads
// in flight (measured on B200, FP8 T = 1: h quantisation 25.2 -> 4.9 us
// against one warp per row).
constexpr int kVecBlocksPerSm = 8;

// amax over n bf16 values (n % 8 == 0), folded into *amax_bits with atomicMax.
__global__ void __launch_bounds__(kThreads)
    amax_bf16_kernel(const uint4* __restrict__ src, long nvec, uint32_t* amax_bits) {
    pdl_wait();
    pdl_trigger();
    float m = 0.0f;
    for (long i = static_cast<long>(blockIdx.x) * kThreads + threadIdx.x; i < nvec;
         i += static_cast<long>(gridDim.x) * kThreads)
        m = fmaxf(m, amax8(src[i]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    __shared__ float wm[kThreads / 32];
    if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 1; i < kThreads / 32; ++i) m = fmaxf(m, wm[i]);
        atomic_max_nonneg(amax_bits, m);
    }
}

// a3 (FP8): x in token order -> e4m3 codes with s_x = amax(x)/448; the
// gate/up GEMM gathers the rows of these codes.
__global__ void __launch_bounds__(kThreads)
    quant_x_fp8_kernel(const uint4* __restrict__ x, long nvec,
                       const uint32_t* __restrict__ amax_bits, uint2* __restrict__ xq) {
    pdl_wait();
    pdl_trigger();
    const float s = fp8_scale_from_amax(*amax_bits);
    const float inv_s = 1.0f / s;
    for (long i = static_cast<long>(blockIdx.x) * kThreads + threadIdx.x; i < nvec;
         i += static_cast<long>(gridDim.x) * kThreads)
        xq[i] = quant8(x[i], inv_s, s);
}

// a3 for large token tiles: dst[p] = src[sorted_ids[p] / k] for the rows
// offsets[0] <= p < offsets[E] (pads zero), rows of vpr 16-byte vectors (bf16 x, or the
// e4m3 codes of x).  One warp per row; each lane keeps up to 8 independent
// 16-byte loads in flight before it stores them.
__global__ void __launch_bounds__(kThreads)
    gather_rows_kernel(const uint4* __restrict__ src, const int32_t* __restrict__ sorted_ids,
                       const int32_t* __restrict__ offsets, int E, int k, int vpr, int capacity,
                       uint4* __restrict__ dst) {
    pdl_wait();
    pdl_trigger();
    constexpr int kBatch = 8;
    const int lane = threadIdx.x & 31;
    const int rows = min(capacity, offsets[E]);
    const int wstride = gridDim.x * (kThreads / 32);
    for (int p = offsets[0] + blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); p < rows;
         p += wstride) {
        const int sid = sorted_ids[p];
        uint4* d = dst + static_cast<long>(p) * vpr;
        if (sid < 0) {
            for (int v = lane; v < vpr; v += 32) d[v] = make_uint4(0, 0, 0, 0);
            continue;
        }
        const uint4* s = src + static_cast<long>(sid / k) * vpr;
        for (int v0 = 0; v0 < vpr; v0 += 32 * kBatch) {
            uint4 buf[kBatch];
#pragma unroll
            for (int i = 0; i < kBatch; ++i) {
                const int v = v0 + 32 * i + lane;
                if (v < vpr) buf[i] = __ldg(s + v);
            }
#pragma unroll
            for (int i = 0; i < kBatch; ++i) {
                const int v = v0 + 32 * i + lane;
                if (v < vpr) d[v] = buf[i];
            }
        }
    }
}

// a5: rows p < offsets[E] of a bf16 matrix -> e4m3 with s = amax/448.
__global__ void __launch_bounds__(kThreads)
    quant_rows_fp8_kernel(const uint4* __restrict__ src, const int32_t* __restrict__ offsets,
                          int E, int vec_per_row, int capacity,
                          const uint32_t* __restrict__ amax_bits, uint2* __restrict__ dst) {
    pdl_wait();
    pdl_trigger();
    const int rows = min(capacity, offsets[E]);
    const long n = static_cast<long>(rows) * vec_per_row;
    const float s = fp8_scale_from_amax(*amax_bits);
    const float inv_s = 1.0f / s;
    for (long i = static_cast<long>(blockIdx.x) * kThreads + threadIdx.x; i < n;
         i += static_cast<long>(gridDim.x) * kThreads)
        dst[i] = quant8(src[i], inv_s, s);
}

// a7: out[t] = sum_j y_perm[inv_perm[t*k + j]] in fp32, j ascending.
// Debug builds check each slot against the rows of y_perm (when known).
__global__ void __launch_bounds__(kThreads)
    combine_kernel(const uint4* __restrict__ y, const int32_t* __restrict__ inv_perm, int T,
                   int k, int vec_per_row, int rows, int32_t* status, uint4* __restrict__ out) {
    pdl_wait();
    pdl_trigger();
    const long i = static_cast<long>(blockIdx.x) * kThreads + threadIdx.x;
    if (i >= static_cast<long>(T) * vec_per_row) return;
    // 32-bit division whenever the index fits (a 64-bit one is ~5x the work)
    const long t = (i >> 32) == 0 ? static_cast<long>(static_cast<uint32_t>(i) /
                                                     static_cast<uint32_t>(vec_per_row))
                                  : i / vec_per_row;
    const int v = static_cast<int>(i - t * vec_per_row);
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    // batches of up to 8 rows: all slots, then all row loads, are issued
    // before the (j-ordered) accumulation, so they are in flight together
    constexpr int kB = 8;
    for (int j0 = 0; j0 < k; j0 += kB) {
        int p[kB];
        uint4 q[kB];
#pragma unroll
        for (int b = 0; b < kB; ++b) {
            p[b] = j0 + b < k ? inv_perm[t * k + j0 + b] : -1;
            if constexpr (kDebugChecks) {
                if (j0 + b < k && (p[b] < 0 || p[b] >= rows)) {
                    report(status, MOE_ERR_DEVICE);
                    p[b] = -1;
                }
            }
        }
#pragma unroll
        for (int b = 0; b < kB; ++b)
            q[b] = p[b] >= 0 ? y[static_cast<long>(p[b]) * vec_per_row + v] : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int b = 0; b < kB; ++b) {
            if (p[b] < 0) continue;
            const uint32_t w[4] = {q[b].x, q[b].y, q[b].z, q[b].w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                acc[2 * c] += bf16_lo(w[c]);
                acc[2 * c + 1] += bf16_hi(w[c]);
            }
        }
    }
    uint32_t o[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * c], acc[2 * c + 1]);
        o[c] = *reinterpret_cast<const uint32_t*>(&b);
    }
    out[i] = make_uint4(o[0], o[1], o[2], o[3]);
}

// a7 (fused form): out = bf16(acc), the fp32 token-order sums the down
// GEMM's epilogue accumulated.
__global__ void __launch_bounds__(kThreads)
    finalize_kernel(const float4* __restrict__ acc, long nvec8, uint4* __restrict__ out) {
    pdl_wait();
    pdl_trigger();
    for (long i = static_cast<long>(blockIdx.x) * kThreads + threadIdx.x; i < nvec8;
         i += static_cast<long>(gridDim.x) * kThreads) {
        const float4 a = acc[2 * i], b = acc[2 * i + 1];
        const __nv_bfloat162 p0 = __floats2bfloat162_rn(a.x, a.y);
        const __nv_bfloat162 p1 = __floats2bfloat162_rn(a.z, a.w);
        const __nv_bfloat162 p2 = __floats2bfloat162_rn(b.x, b.y);
        const __nv_bfloat162 p3 = __floats2bfloat162_rn(b.z, b.w);
        out[i] = make_uint4(*reinterpret_cast<const uint32_t*>(&p0),
                            *reinterpret_cast<const uint32_t*>(&p1),
                            *reinterpret_cast<const uint32_t*>(&p2),
                            *reinterpret_cast<const uint32_t*>(&p3));
    }
}

// ---- weight packing (one-time)
// amax of each expert matrix: blockIdx.y = e*3 + m; folded into amax[e*3+m].
__global__ void __launch_bounds__(kThreads)
    matrix_amax_kernel(const uint4* __restrict__ Wg, const uint4* __restrict__ Wu,
                       const uint4* __restrict__ Wd, long vec_per_matrix, uint32_t* amax) {
    const int em = blockIdx.y, e = em / 3, m = em % 3;
    const uint4* src = (m == 0 ? Wg : m == 1 ? Wu : Wd) + static_cast<long>(e) * vec_per_matrix;
    float mx = 0.0f;
    for (long i = static_cast<long>(blockIdx.x) * kThreads + threadIdx.x; i < vec_per_matrix;
         i += static_cast<long>(gridDim.x) * kThreads)
        mx = fmaxf(mx, amax8(src[i]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    __shared__ float wm[kThreads / 32];
    if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 1; i < kThreads / 32; ++i) mx = fmaxf(mx, wm[i]);
        atomic_max_nonneg(&amax[em], mx);
    }
}

// One 16 KB tile of packed weights per CTA: the swizzled shared-memory image
// of 128 weight rows x 128 bytes of K (see PackedGeom).  GU selects the gate/up
// matrix, whose packed row R holds column j = 16*(R/32) + R%16 of W_g
// (R%32 < 16) or W_u; otherwise the down matrix, whose row R is column R of
// W_d (W_d transposed).  Out-of-range rows and K are zero.
// grid = (KB, MT, E).
template <bool FP8, bool GU>
__global__ void __launch_bounds__(kThreads)
    pack_tiles_kernel(const __nv_bfloat16* __restrict__ Wa, const __nv_bfloat16* __restrict__ Wb,
                      int H, int I, int MT, int KB, uint8_t* __restrict__ out,
                      const uint32_t* __restrict__ amax) {
    __shared__ __align__(16) uint8_t tile[kTileBytes];
    constexpr int BK = FP8 ? 128 : 64;
    constexpr int EB = FP8 ? 1 : 2;
    const int kb = blockIdx.x, m = blockIdx.y, e = blockIdx.z;
    const long mat = static_cast<long>(e) * H * I;
    float sa = 1.0f, sb = 1.0f;
    if constexpr (FP8) {
        sa = fp8_scale_from_amax(amax[e * 3 + (GU ? 0 : 2)]);
        sb = fp8_scale_from_amax(amax[e * 3 + 1]);
    }
    for (int idx = threadIdx.x; idx < kTileRows * BK; idx += kThreads) {
        const int r = idx % kTileRows, kk = idx / kTileRows;
        const int R = m * kTileRows + r;
        const int kg = kb * BK + kk;
        float v = 0.0f;
        float sc = sa;
        if (GU) {
            const int j = 16 * (R / 32) + (R & 15);
            const bool up = (R & 31) >= 16;
            if (R < 2 * I && kg < H) {
                v = __bfloat162float((up ? Wb : Wa)[mat + static_cast<long>(kg) * I + j]);
                sc = up ? sb : sa;
            }
        } else if (R < H && kg < I) {
            v = __bfloat162float(Wa[mat + static_cast<long>(kg) * H + R]);
        }
        const int o = r * kTileRowBytes + kk * EB;
        const int sw = o ^ (((o >> 7) & 7) << 4);
        if constexpr (FP8)
            tile[sw] = fp8_quant(v, sc);
        else
            *reinterpret_cast<__nv_bfloat16*>(tile + sw) = __float2bfloat16_rn(v);
    }
    __syncthreads();
    uint4* dst = reinterpret_cast<uint4*>(
        out + (static_cast<size_t>(e * MT + m) * KB + kb) * kTileBytes);
    const uint4* src = reinterpret_cast<const uint4*>(tile);
    for (int i = threadIdx.x; i < kTileBytes / 16; i += kThreads) dst[i] = src[i];
}

// Multi-LoRA adapter tiles (see LoraGeom): one 16 KB tile per CTA, element
// (row rr, k kk) from the section's definition, bf16, swizzled like the
// weights.  Layouts: A_g, A_u [n][E][H][r], B_g, B_u [n][E][r][I],
// A_d [n][E][I][r], B_d [n][E][r][H].  grid = (tiles per expert, 1, E).
template <int SECTION>
__global__ void __launch_bounds__(kThreads)
    pack_lora_kernel(const __nv_bfloat16* __restrict__ Ag, const __nv_bfloat16* __restrict__ Bg,
                     const __nv_bfloat16* __restrict__ Au, const __nv_bfloat16* __restrict__ Bu,
                     const __nv_bfloat16* __restrict__ Ad, const __nv_bfloat16* __restrict__ Bd,
                     int E, int H, int I, int r, int R, int per_expert, uint8_t* __restrict__ out) {
    __shared__ __align__(16) uint8_t tile[kTileBytes];
    const int ti = blockIdx.x, e = blockIdx.z;
    for (int idx = threadIdx.x; idx < kTileRows * 64; idx += kThreads) {
        const int rr = idx % kTileRows, kk = idx / kTileRows;
        float v = 0.0f;
        if constexpr (SECTION == 0) {           // shrink_gu: tile = k-block of H
            const int kg = ti * 64 + kk, slot = rr & 63;
            if (kg < H && slot < R) {
                const int a = slot / r, q = slot % r;
                const __nv_bfloat16* A = rr < 64 ? Ag : Au;
                v = __bfloat162float(A[((static_cast<long>(a) * E + e) * H + kg) * r + q]);
            }
        } else if constexpr (SECTION == 1) {    // expand_gu: tile = (m, x)
            const int m = ti >> 1, x = ti & 1;
            const int Rp = m * kTileRows + rr;
            const int j = 16 * (Rp / 32) + (Rp & 15);
            const bool up = (Rp & 31) >= 16;
            if (Rp < 2 * I && kk < R && up == (x == 1)) {
                const int a = kk / r, q = kk % r;
                const __nv_bfloat16* B = up ? Bu : Bg;
                v = __bfloat162float(B[((static_cast<long>(a) * E + e) * r + q) * I + j]);
            }
        } else if constexpr (SECTION == 2) {    // shrink_d: tile = k-block of I
            const int kg = ti * 64 + kk;
            if (kg < I && rr < R) {
                const int a = rr / r, q = rr % r;
                v = __bfloat162float(Ad[((static_cast<long>(a) * E + e) * I + kg) * r + q]);
            }
        } else {                                // expand_d: tile = m
            const int c = ti * kTileRows + rr;
            if (c < H && kk < R) {
                const int a = kk / r, q = kk % r;
                v = __bfloat162float(Bd[((static_cast<long>(a) * E + e) * r + q) * H + c]);
            }
        }
        const int o = rr * kTileRowBytes + kk * 2;
        const int sw = o ^ (((o >> 7) & 7) << 4);
        *reinterpret_cast<__nv_bfloat16*>(tile + sw) = __float2bfloat16_rn(v);
    }
    __syncthreads();
    uint4* dst = reinterpret_cast<uint4*>(
        out + (static_cast<size_t>(e) * per_expert + ti) * kTileBytes);
    const uint4* src = reinterpret_cast<const uint4*>(tile);
    for (int i = threadIdx.x; i < kTileBytes / 16; i += kThreads) dst[i] = src[i];
}

__global__ void amax_to_scale_kernel(float* scales, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) scales[i] = fp8_scale_from_amax(__float_as_uint(scales[i]));
}

__global__ void wait_timeout_kernel(int32_t* status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // Nothing ever arrives on bar: the bounded wait must give up.
        if (!mbar_wait(&bar, 0, nullptr, limit_ns)) report(status, MOE_ERR_TIMEOUT);
        mbar_arrive(&bar);  // complete the phase so the barrier is left idle
    }
}

int blocks_for(long n, int per_block, int cap) {
    long b = (n + per_block - 1) / per_block;
    if (b < 1) b = 1;
    return static_cast<int>(b < cap ? b : cap);
}

// Grid of the flat vector kernels: one thread per vector of the capacity
// bound, at most kVecBlocksPerSm blocks per SM (grid-stride beyond that;
// measured on B200, an uncapped grid was slower at T = 2048 and above).
int vec_blocks(long nvec) { return blocks_for(nvec, kThreads, kVecBlocksPerSm * device_sm_count()); }

}  // namespace

cudaError_t launch_amax_bf16(const void* src, long n, uint32_t* amax_bits, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    return launch_pdl(amax_bf16_kernel, dim3(blocks_for(n / 8, kThreads * 4, 1184)),
                      dim3(kThreads), 0, s, static_cast<const uint4*>(src), n / 8, amax_bits);
}

cudaError_t launch_quant_x_fp8(const void* x, long n, const uint32_t* amax_bits, void* xq,
                               cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    return launch_pdl(quant_x_fp8_kernel, dim3(vec_blocks(n / 8)), dim3(kThreads), 0, s,
                      static_cast<const uint4*>(x), n / 8, amax_bits, static_cast<uint2*>(xq));
}

cudaError_t launch_gather_rows(const void* src, int row_bytes, const int32_t* sorted_ids,
                               const int32_t* offsets, int E, int k, int capacity, void* dst,
                               cudaStream_t s) {
    if (capacity == 0) return cudaSuccess;
    const int vpr = row_bytes / 16;
    // one warp per row, all rows at once (a capped grid-stride launch measured
    // slower: prefill T = 4096, 31 vs 27 us)
    const int blocks = blocks_for(static_cast<long>(capacity), kThreads / 32, 1 << 30);
    return launch_pdl(gather_rows_kernel, dim3(blocks), dim3(kThreads), 0, s,
                      static_cast<const uint4*>(src), sorted_ids, offsets, E, k, vpr, capacity,
                      static_cast<uint4*>(dst));
}

cudaError_t launch_quant_rows_fp8(const void* h, const int32_t* offsets, int E, int cols,
                                  int capacity, const uint32_t* amax_bits, void* h_q,
                                  cudaStream_t s) {
    if (capacity == 0) return cudaSuccess;
    return launch_pdl(quant_rows_fp8_kernel, dim3(vec_blocks(static_cast<long>(capacity) * (cols / 8))),
                      dim3(kThreads), 0, s, static_cast<const uint4*>(h), offsets, E, cols / 8,
                      capacity, amax_bits, static_cast<uint2*>(h_q));
}

cudaError_t launch_combine(const void* y_perm, const int32_t* inv_perm, int T, int k, int H,
                           void* out, cudaStream_t s, int rows, int32_t* status) {
    const long n = static_cast<long>(T) * (H / 8);
    if (n == 0) return cudaSuccess;
    return launch_pdl(combine_kernel, dim3(static_cast<unsigned>((n + kThreads - 1) / kThreads)),
                      dim3(kThreads), 0, s, static_cast<const uint4*>(y_perm), inv_perm, T, k,
                      H / 8, rows, status, static_cast<uint4*>(out));
}

cudaError_t launch_finalize(const float* acc, long n, void* out, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    return launch_pdl(finalize_kernel, dim3(vec_blocks(n / 8)), dim3(kThreads), 0, s,
                      reinterpret_cast<const float4*>(acc), n / 8, static_cast<uint4*>(out));
}

cudaError_t launch_pack_weights(int fp8, int E, int H, int I, const void* Wg, const void* Wu,
                                const void* Wd, void* packed, float* scales, uint32_t* amax_tmp,
                                cudaStream_t s) {
    const auto* g = static_cast<const __nv_bfloat16*>(Wg);
    const auto* u = static_cast<const __nv_bfloat16*>(Wu);
    const auto* d = static_cast<const __nv_bfloat16*>(Wd);
    const long hi = static_cast<long>(H) * I;
    const PackedGeom geo = packed_geom(fp8, E, H, I);
    uint8_t* gu = static_cast<uint8_t*>(packed);
    uint8_t* dn = gu + geo.gu_bytes;
    const dim3 ggu(geo.kb_gu, geo.mt_gu, E), gdn(geo.kb_dn, geo.mt_dn, E);
    if (fp8) {
        cudaError_t err = cudaMemsetAsync(amax_tmp, 0, sizeof(uint32_t) * 3 * E, s);
        if (err != cudaSuccess) return err;
        matrix_amax_kernel<<<dim3(blocks_for(hi / 8, kThreads * 8, 64), 3 * E), kThreads, 0, s>>>(
            reinterpret_cast<const uint4*>(g), reinterpret_cast<const uint4*>(u),
            reinterpret_cast<const uint4*>(d), hi / 8, amax_tmp);
        pack_tiles_kernel<true, true><<<ggu, kThreads, 0, s>>>(g, u, H, I, geo.mt_gu, geo.kb_gu,
                                                               gu, amax_tmp);
        pack_tiles_kernel<true, false><<<gdn, kThreads, 0, s>>>(d, nullptr, H, I, geo.mt_dn,
                                                                geo.kb_dn, dn, amax_tmp);
        if (static_cast<void*>(scales) != static_cast<void*>(amax_tmp)) {
            err = cudaMemcpyAsync(scales, amax_tmp, sizeof(float) * 3 * E, cudaMemcpyDeviceToDevice,
                                  s);
            if (err != cudaSuccess) return err;
        }
        amax_to_scale_kernel<<<(3 * E + 255) / 256, 256, 0, s>>>(scales, 3 * E);
    } else {
        pack_tiles_kernel<false, true><<<ggu, kThreads, 0, s>>>(g, u, H, I, geo.mt_gu, geo.kb_gu,
                                                                gu, nullptr);
        pack_tiles_kernel<false, false><<<gdn, kThreads, 0, s>>>(d, nullptr, H, I, geo.mt_dn,
                                                                 geo.kb_dn, dn, nullptr);
    }
    return cudaGetLastError();
}

cudaError_t launch_pack_lora(int E, int H, int I, int n_adapters, int rank, const void* Ag,
                             const void* Bg, const void* Au, const void* Bu, const void* Ad,
                             const void* Bd, void* packed, cudaStream_t s) {
    const LoraGeom lg = lora_geom(E, H, I);
    const int R = n_adapters * rank;
    const auto* ag = static_cast<const __nv_bfloat16*>(Ag);
    const auto* bg = static_cast<const __nv_bfloat16*>(Bg);
    const auto* au = static_cast<const __nv_bfloat16*>(Au);
    const auto* bu = static_cast<const __nv_bfloat16*>(Bu);
    const auto* ad = static_cast<const __nv_bfloat16*>(Ad);
    const auto* bd = static_cast<const __nv_bfloat16*>(Bd);
    uint8_t* base = static_cast<uint8_t*>(packed);
    pack_lora_kernel<0><<<dim3(lg.kb_gu, 1, E), kThreads, 0, s>>>(
        ag, bg, au, bu, ad, bd, E, H, I, rank, R, lg.kb_gu, base + lg.shrink_gu);
    pack_lora_kernel<1><<<dim3(lg.mt_gu * 2, 1, E), kThreads, 0, s>>>(
        ag, bg, au, bu, ad, bd, E, H, I, rank, R, lg.mt_gu * 2, base + lg.expand_gu);
    pack_lora_kernel<2><<<dim3(lg.kb_dn, 1, E), kThreads, 0, s>>>(
        ag, bg, au, bu, ad, bd, E, H, I, rank, R, lg.kb_dn, base + lg.shrink_d);
    pack_lora_kernel<3><<<dim3(lg.mt_dn, 1, E), kThreads, 0, s>>>(
        ag, bg, au, bu, ad, bd, E, H, I, rank, R, lg.mt_dn, base + lg.expand_d);
    return cudaGetLastError();
}

cudaError_t launch_wait_timeout_selftest(int32_t* status, int timeout_us, cudaStream_t s) {
    wait_timeout_kernel<<<1, 32, 0, s>>>(status, static_cast<uint64_t>(timeout_us) * 1000ull);
    return cudaGetLastError();
}

}  // namespace moe
