// kernels.h -- host-side launchers of the layer's kernels (internal; the
// public surface is include/moe.h).  Every launcher enqueues on `stream`,
// never synchronises and returns the launch's cudaError_t.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Packed expert weights are stored as 16 KB tiles, each the exact shared-memory
// image (128-byte swizzle) of 128 weight rows x 128 bytes of K, so that one
// contiguous bulk copy fills one pipeline stage.  Tile (m, kb) of expert e of a
// matrix with MT row tiles and KB k-blocks lives at ((e*MT + m)*KB + kb)*16 KB.
// Rows past the matrix and K past its length are zero.
constexpr int kTileRows = 128;
constexpr int kTileRowBytes = 128;
constexpr int kTileBytes = kTileRows * kTileRowBytes;
struct PackedGeom {
    int bk;               // K elements per tile row (64 bf16, 128 e4m3)
    int mt_gu, kb_gu;     // gate/up: 2I/128 row tiles, ceil(H/bk) k-blocks
    int mt_dn, kb_dn;     // down: ceil(H/128) row tiles, ceil(I/bk) k-blocks
    size_t gu_bytes;      // all experts
    size_t dn_bytes;
};
inline PackedGeom packed_geom(int fp8, int E, int H, int I) {
    PackedGeom g;
    g.bk = fp8 ? 128 : 64;
    g.mt_gu = (2 * I + kTileRows - 1) / kTileRows;
    g.kb_gu = (H + g.bk - 1) / g.bk;
    g.mt_dn = (H + kTileRows - 1) / kTileRows;
    g.kb_dn = (I + g.bk - 1) / g.bk;
    g.gu_bytes = static_cast<size_t>(E) * g.mt_gu * g.kb_gu * kTileBytes;
    g.dn_bytes = static_cast<size_t>(E) * g.mt_dn * g.kb_dn * kTileBytes;
    return g;
}

// Packed multi-LoRA adapters (bf16; n_adapters * rank = R <= 64), four
// sections of 16 KB tiles in the same swizzled layout as the weights:
//   shrink_gu [E][ceil(H/64)]   rows 0..63: A_g columns (row a*r+q), rows
//                               64..127: A_u columns; K = H
//   expand_gu [E][MT_gu][2]     per packed gate/up row (interleaved as W_gu):
//                               k-block 0 = B_g (gate rows, else 0), k-block
//                               1 = B_u (up rows, else 0); K index a*r+q
//   shrink_d  [E][ceil(I/64)]   rows 0..R-1: A_d columns; K = I
//   expand_d  [E][MT_dn][1]     per output column c: B_d[a][e][q][c]
struct LoraGeom {
    int kb_gu, kb_dn, mt_gu, mt_dn;
    size_t shrink_gu, expand_gu, shrink_d, expand_d;   // byte offsets
    size_t bytes;
};
inline LoraGeom lora_geom(int E, int H, int I) {
    LoraGeom g;
    g.kb_gu = (H + 63) / 64;
    g.kb_dn = (I + 63) / 64;
    g.mt_gu = (2 * I + kTileRows - 1) / kTileRows;
    g.mt_dn = (H + kTileRows - 1) / kTileRows;
    g.shrink_gu = 0;
    g.expand_gu = g.shrink_gu + static_cast<size_t>(E) * g.kb_gu * kTileBytes;
    g.shrink_d = g.expand_gu + static_cast<size_t>(E) * g.mt_gu * 2 * kTileBytes;
    g.expand_d = g.shrink_d + static_cast<size_t>(E) * g.kb_dn * kTileBytes;
    g.bytes = g.expand_d + static_cast<size_t>(E) * g.mt_dn * kTileBytes;
    return g;
}

// Launch with programmatic dependent launch allowed (see pdl_wait/pdl_trigger).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ---- a1/a2 (route_permute.cu)
// ctl (optional): the layer's control block, zeroed by the first kernel of a
// forward call after it has waited for the previous call's kernels.
cudaError_t launch_route_topk(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                              cudaStream_t s, int32_t* ctl = nullptr, int ctl_ints = 0);
// Single-CTA route + permute for small batches (T <= kSmallT, T*k <= kChunk).
constexpr int kSmallT = 128;
constexpr int kChunk = 2048;  // assignments per permutation chunk
int permute_chunks(long A);
bool fused_route_permute_ok(int T, int k);
cudaError_t launch_route_permute_small(const float* logits, int T, int E, int k, int block_m,
                                       int capacity, int32_t* ids, float* w, int32_t* counts,
                                       int32_t* offsets, int32_t* sorted_ids, int32_t* inv_perm,
                                       int32_t* tiles, int32_t* num_tiles, int32_t* status,
                                       cudaStream_t s, int32_t* ctl = nullptr, int ctl_ints = 0,
                                       const void* x = nullptr, long x_elems = 0,
                                       uint32_t* amax_out = nullptr, void* xq_out = nullptr);
// Batches small enough for the single-CTA kernel to also take amax(x) and
// quantise x (FP8): up to 64 KB of x (measured on B200: at 184 KB the one CTA
// took longer than the separate amax kernel it replaced).
constexpr long kSmallAmaxElems = 32768;
cudaError_t launch_align_permute(const int32_t* ids, int T, int k, int E, int block_m,
                                 int capacity, int32_t* counts, int32_t* offsets,
                                 int32_t* sorted_ids, int32_t* inv_perm, int32_t* tiles,
                                 int32_t* num_tiles, int32_t* chunk_counts, int32_t* status,
                                 cudaStream_t s);

// ---- a3/a5/a7 and packing (elementwise.cu)
cudaError_t launch_amax_bf16(const void* src, long n, uint32_t* amax_bits, cudaStream_t s);
// FP8 x in token order: xq = RNE_sat(x * (1 / s_x)), s_x from amax_bits.
cudaError_t launch_quant_x_fp8(const void* x, long n, const uint32_t* amax_bits, void* xq,
                               cudaStream_t s);
// dst[p] = src[sorted_ids[p] / k] (rows of row_bytes, a multiple of 16), pads
// zero: the permuted token rows of CTA-pair GEMM tiles
cudaError_t launch_gather_rows(const void* src, int row_bytes, const int32_t* sorted_ids,
                               const int32_t* offsets, int E, int k, int capacity, void* dst,
                               cudaStream_t s);
cudaError_t launch_quant_rows_fp8(const void* h, const int32_t* offsets, int E, int cols,
                                  int capacity, const uint32_t* amax_bits, void* h_q,
                                  cudaStream_t s);
// rows: rows of y_perm (debug builds check inv_perm against it; INT32_MAX if
// unknown), status: where such a fault is reported (may be null)
cudaError_t launch_combine(const void* y_perm, const int32_t* inv_perm, int T, int k, int H,
                           void* out, cudaStream_t s, int rows = 0x7fffffff,
                           int32_t* status = nullptr);
// out (bf16) = acc (fp32), n elements (n % 8 == 0)
cudaError_t launch_finalize(const float* acc, long n, void* out, cudaStream_t s);
cudaError_t launch_pack_weights(int fp8, int E, int H, int I, const void* Wg, const void* Wu,
                                const void* Wd, void* packed, float* scales, uint32_t* amax_tmp,
                                cudaStream_t s);
cudaError_t launch_wait_timeout_selftest(int32_t* status, int timeout_us, cudaStream_t s);
cudaError_t launch_pack_lora(int E, int H, int I, int n_adapters, int rank, const void* Ag,
                             const void* Bg, const void* Au, const void* Bu, const void* Ad,
                             const void* Bd, void* packed, cudaStream_t s);

// ---- a4/a6 (grouped_gemm.cu)
struct GemmProblem {
    int fp8;              // 0 bf16, 1 e4m3
    int epi;              // 0: gate/up, rows gathered from gather_src -> SiLU*up -> h
                          // 1: down -> * w -> bf16 rows of out (permuted order)
                          // 2: down -> * w -> added into fp32 row `token` of out
                          // 3: adapter shrink -> masked, scaled bf16 rows of out
    int E, Mw, K;         // weight rows per expert, reduction length
    int Mvalid;           // weight rows per expert that are real (masking)
    int nmax;             // token-tile cap (multiple of 16, <= 256)
    int capacity;         // rows of the permuted operands
    const void* weights;  // packed tiles of this matrix (see PackedGeom)
    int MT, KB;           // row tiles and k-blocks per expert
    const void* act;      // [capacity, K] rows in permuted order (all but the
                          // one-CTA gate/up kernel, which gathers)
    const void* gather_src;  // epi 0, one-CTA tiles: [T, K] rows in token order
    void* out;            // epi 0/1: [capacity, ldo] bf16; epi 2: [T, ldo] f32
    int ldo;
    const int32_t* counts;
    const int32_t* offsets;
    const int32_t* sorted_ids;
    int ktop;                    // k (flat assignment index / k = token)
    int A;                       // T * k
    const float* w;              // epi 1/2: routing weight by flat index [T*k]
    const float* w_scales;       // [E][3] (FP8)
    const uint32_t* act_amax;    // FP8: amax bits of the activation operand
    uint32_t* out_amax;          // FP8 epi 0: amax of h (bits)
    float* acc_zero;             // epi 0: fp32 buffer to zero (may be null)
    long acc_zero_floats;        // its length, a multiple of 4
    float* partials;             // [max_ctas][2][128*nmax] f32
    int32_t* counters;           // [max_ctas] zeroed
    int32_t* status;
    int max_ctas;
    int sched_after_wait;        // counts/offsets are written by the previous kernel
    // multi-LoRA (bf16): the adapters' expand as KBx extra k-blocks of 64,
    // weights from x_tiles [E][MT][KBx], rows from x_rows [capacity, KBx*64]
    int KBx;
    const void* x_tiles;
    const void* x_rows;
    // epi 3 (adapter shrink): the tokens' adapters, their scales, the rank,
    // and n_adapters * rank (<= 64): output column c % 64 = a * rank + q
    const int32_t* adapter;
    const float* lscale;
    int lrank, lR;
};
int gemm_nmax_for(int T, int k, int E);
// Token tiles above 64 rows run on CTA pairs (whose gate/up rows are gathered
// by a separate kernel)
inline bool gemm_uses_pairs(int nmax) { return nmax > 64; }
size_t gemm_partials_bytes(int nmax);
cudaError_t launch_grouped_gemm(const GemmProblem& p, cudaStream_t s);

int device_sm_count();

// ---- the bf16 grouped FFN (a3..a6) over E_sub consecutive segments of a
// permutation (moe_api.cu): counts/offsets point at the first of them and
// may start inside a larger permutation, whose other rows are left alone;
// nmax is the token-tile cap (gemm_nmax_for of the segments' own mean).
// Used by the CPU/GPU split, whose slot permutation spans several weight
// buffers.  ws: segment_ffn_ws_bytes(T, capacity, H, I) bytes.
size_t segment_ffn_ws_bytes(int T, int capacity, int H, int I);
moe_status segment_ffn(int T, int k, int E_sub, int H, int I, int capacity, int nmax,
                       const void* x, const float* w, const int32_t* counts,
                       const int32_t* offsets, const int32_t* sorted_ids, const void* packed,
                       void* y_perm, int32_t* status, void* ws, cudaStream_t s);

}  // namespace moe
