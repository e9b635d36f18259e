// moe_api.cu -- the extern "C" boundary declared in include/moe.h: argument
// validation (nothing is launched on a bad argument), workspace carving, and
// the order of launches on the caller's stream.  Never allocates, never
// synchronises (except moe_check_status, whose job is to read the device).
#include <nvtx3/nvToolsExt.h>

#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

using namespace moe;

namespace {

constexpr size_t kAlign = 256;
// control block: status, amax_x, amax_h, stream-K counters of the gate/up and
// down GEMMs and of the two adapter shrinks (kMaxCtas each)
constexpr int kCtlInts = 64 + 4 * kMaxCtas;
constexpr int kCtlStatus = 0, kCtlAmaxX = 1, kCtlAmaxH = 2, kCtlCountersGu = 64,
              kCtlCountersDn = 64 + kMaxCtas, kCtlCountersSgu = 64 + 2 * kMaxCtas,
              kCtlCountersSdn = 64 + 3 * kMaxCtas;
// widths (bf16 columns) of the adapter shrink outputs: gate|up, and down
constexpr int kLoraGuCols = 128, kLoraDnCols = 64;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

moe_status check_route(int T, int E, int k) {
    if (T < 0 || E < 1 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
    if (E > kMaxExperts) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

moe_status check_layer(moe_dtype dt, int T, int k, int E, int H, int I, int block_m) {
    moe_status s = check_route(T, E, k);
    if (s != MOE_OK) return s;
    if (dt != MOE_BF16 && dt != MOE_FP8_E4M3) return MOE_ERR_INVALID_ARG;
    if (H < 64 || I < 64 || block_m < 16) return MOE_ERR_INVALID_ARG;
    if (H % 64 != 0 || I % 64 != 0 || block_m % 16 != 0) return MOE_ERR_UNSUPPORTED;
    if (block_m > 4096) return MOE_ERR_UNSUPPORTED;
    const long long A = static_cast<long long>(T) * k;
    const long long cap = A + (A < E ? A : E) * (block_m - 1);
    // row coordinates of the tensor maps and row indices are 32-bit
    if (cap > (1LL << 30) || static_cast<long long>(E) * 2 * I > (1LL << 30))
        return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

struct Carver {
    char* base;
    size_t used = 0;
    template <class T>
    T* take(size_t bytes) {
        T* p = reinterpret_cast<T*>(base ? base + used : nullptr);
        used += align_up(bytes);
        return p;
    }
};

struct FfnBuffers {
    int32_t* ctl;
    void* xq;         // FP8: e4m3 codes of x, token order [T, H]
    void* x_perm;     // permuted token rows [cap, H] (bf16 / e4m3): CTA-pair tiles,
                      // and every bf16 layer (adapters' shrink)
    void* t_gu;       // adapters: shrink outputs of x [cap, 128] bf16
    void* t_dn;       // adapters: shrink outputs of h [cap, 64] bf16
    void* h;
    void* h_q;
    float* partials;
};

void carve_ffn_rest(Carver& c, FfnBuffers& b, moe_dtype dt, int T, int cap, int H, int I,
                    int nmax) {
    const bool fp8 = dt == MOE_FP8_E4M3;
    b.xq = fp8 ? c.take<void>(static_cast<size_t>(T) * H) : nullptr;
    // bf16 layers always have room for permuted rows and the adapters'
    // shrink outputs, so one workspace size serves calls with and without
    b.x_perm = (gemm_uses_pairs(nmax) || !fp8)
                   ? c.take<void>(static_cast<size_t>(cap) * H * (fp8 ? 1 : 2))
                   : nullptr;
    b.t_gu = fp8 ? nullptr : c.take<void>(static_cast<size_t>(cap) * kLoraGuCols * 2);
    b.t_dn = fp8 ? nullptr : c.take<void>(static_cast<size_t>(cap) * kLoraDnCols * 2);
    b.h = c.take<void>(static_cast<size_t>(cap) * I * 2);
    b.h_q = fp8 ? c.take<void>(static_cast<size_t>(cap) * I) : nullptr;
    b.partials = c.take<float>(gemm_partials_bytes(nmax));
}

// The control block is carved first, so a missing caller status word means
// the first int32 of the workspace.
FfnBuffers carve_ffn(Carver& c, moe_dtype dt, int T, int cap, int H, int I, int nmax) {
    FfnBuffers b;
    b.ctl = c.take<int32_t>(sizeof(int32_t) * kCtlInts);
    carve_ffn_rest(c, b, dt, T, cap, H, I, nmax);
    return b;
}

// How a forward call forms out[t] = sum_j y(t, j).
enum class Combine {
    kGatherSum,   // y_perm rows written by the down GEMM, summed in fixed j order
    kFused        // the down GEMM's epilogue adds w*y into an fp32 accumulator
};

struct FfnCall {
    moe_dtype dt;
    int T, k, E, H, I, cap;
    const void* x;
    const float* w;
    const int32_t* counts;
    const int32_t* offsets;
    const int32_t* sorted_ids;
    const void* packed;
    const float* scales;
    void* y_out;                 // y_perm [cap, H] bf16, or the fp32 accumulator [T, H]
    int32_t* status;
    int max_ctas;
    bool x_ready = false;        // FP8: amax(x) and the codes of x already written
    bool counts_from_prev = false;  // the permutation is the previous kernel's output
    Combine combine = Combine::kGatherSum;
    const moe_lora_args* lora = nullptr;
    int nmax = 0;                   // token-tile cap; 0 = from T, k and E
};

void record(moe_event_t* ev, int i, cudaStream_t s) {
    if (ev) cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev[i]), s);
}

// NVTX range over the host-side launches of one stage (shown by profilers
// such as Nsight Systems / Compute; free when no tool is attached).
struct Range {
    explicit Range(const char* name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
    Range(const Range&) = delete;
    Range& operator=(const Range&) = delete;
};

// a3..a6 on carved buffers.  The control block must already be zeroed.
moe_status run_ffn(const FfnCall& f, const FfnBuffers& b, moe_event_t* ev, cudaStream_t s) {
    const bool fp8 = f.dt == MOE_FP8_E4M3;
    const int nmax = f.nmax > 0 ? f.nmax : gemm_nmax_for(f.T, f.k, f.E);
    uint32_t* amax_x = reinterpret_cast<uint32_t*>(b.ctl + kCtlAmaxX);
    uint32_t* amax_h = reinterpret_cast<uint32_t*>(b.ctl + kCtlAmaxH);
    const long x_elems = static_cast<long>(f.T) * f.H;
    bool counts_from_prev = f.counts_from_prev;
    if (fp8 && !f.x_ready) {
        // a3 (FP8): amax(x) and the e4m3 codes of x, in token order
        Range r("moe: x quantisation (a3)");
        if (launch_amax_bf16(f.x, x_elems, amax_x, s) != cudaSuccess ||
            launch_quant_x_fp8(f.x, x_elems, amax_x, b.xq, s) != cudaSuccess)
            return MOE_ERR_CUDA;
        counts_from_prev = false;
    }
    const void* rows_src = fp8 ? b.xq : f.x;
    const bool lora = f.lora != nullptr;
    const LoraGeom lgeo = lora_geom(f.E, f.H, f.I);
    const uint8_t* lpk = lora ? static_cast<const uint8_t*>(f.lora->packed) : nullptr;
    if (gemm_uses_pairs(nmax) || lora) {
        // large token tiles: lay the token rows out in permuted order for
        // the pair GEMM's TMA loads
        Range r("moe: gather (a3)");
        if (launch_gather_rows(rows_src, f.H * (fp8 ? 1 : 2), f.sorted_ids, f.offsets, f.E, f.k,
                               f.cap, b.x_perm, s) != cudaSuccess)
            return MOE_ERR_CUDA;
        counts_from_prev = false;
    }

    // the adapters' shrink of x (all adapters, masked to the token's own)
    GemmProblem shr{};
    if (lora) {
        shr.fp8 = 0;
        shr.epi = 3;
        shr.E = f.E;
        shr.Mw = kTileRows;
        shr.Mvalid = kLoraGuCols;
        shr.K = f.H;
        shr.nmax = nmax;
        shr.capacity = f.cap;
        shr.weights = lpk + lgeo.shrink_gu;
        shr.MT = 1;
        shr.KB = lgeo.kb_gu;
        shr.act = b.x_perm;
        shr.out = b.t_gu;
        shr.ldo = kLoraGuCols;
        shr.counts = f.counts;
        shr.offsets = f.offsets;
        shr.sorted_ids = f.sorted_ids;
        shr.ktop = f.k;
        shr.A = f.T * f.k;
        shr.partials = b.partials;
        shr.counters = b.ctl + kCtlCountersSgu;
        shr.status = f.status;
        shr.max_ctas = f.max_ctas;
        shr.adapter = f.lora->adapter;
        shr.lscale = f.lora->scale;
        shr.lrank = f.lora->rank;
        shr.lR = f.lora->n_adapters * f.lora->rank;
        Range r("moe: adapter shrink of x");
        if (launch_grouped_gemm(shr, s) != cudaSuccess) return MOE_ERR_CUDA;
    }
    record(ev, 2, s);

    const PackedGeom geo = packed_geom(fp8, f.E, f.H, f.I);
    const bool fused = f.combine == Combine::kFused;
    GemmProblem gu{};
    gu.fp8 = fp8;
    gu.epi = 0;
    gu.E = f.E;
    gu.Mw = 2 * f.I;
    gu.K = f.H;
    gu.Mvalid = 2 * f.I;
    gu.nmax = nmax;
    gu.capacity = f.cap;
    gu.weights = f.packed;
    gu.MT = geo.mt_gu;
    gu.KB = geo.kb_gu;
    gu.gather_src = rows_src;
    gu.act = b.x_perm;
    gu.out = b.h;
    gu.ldo = f.I;
    gu.counts = f.counts;
    gu.offsets = f.offsets;
    gu.sorted_ids = f.sorted_ids;
    gu.ktop = f.k;
    gu.A = f.T * f.k;
    gu.w_scales = f.scales;
    gu.act_amax = amax_x;
    gu.out_amax = amax_h;
    gu.acc_zero = fused ? static_cast<float*>(f.y_out) : nullptr;
    gu.acc_zero_floats = fused ? x_elems : 0;
    gu.partials = b.partials;
    gu.counters = b.ctl + kCtlCountersGu;
    gu.status = f.status;
    gu.max_ctas = f.max_ctas;
    gu.sched_after_wait = counts_from_prev ? 1 : 0;
    if (lora) {
        gu.KBx = kLoraGuCols / 64;
        gu.x_tiles = lpk + lgeo.expand_gu;
        gu.x_rows = b.t_gu;
    }
    {
        Range r("moe: gate/up GEMM (a3 gather + a4)");
        if (launch_grouped_gemm(gu, s) != cudaSuccess) return MOE_ERR_CUDA;
    }
    record(ev, 3, s);

    if (fp8) {
        Range r("moe: h quantisation (a5)");
        if (launch_quant_rows_fp8(b.h, f.offsets, f.E, f.I, f.cap, amax_h, b.h_q, s) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
    }
    if (lora) {
        // the adapters' shrink of h
        GemmProblem sd = shr;
        sd.Mvalid = kLoraDnCols;
        sd.K = f.I;
        sd.weights = lpk + lgeo.shrink_d;
        sd.KB = lgeo.kb_dn;
        sd.act = b.h;
        sd.out = b.t_dn;
        sd.ldo = kLoraDnCols;
        sd.counters = b.ctl + kCtlCountersSdn;
        Range r("moe: adapter shrink of h");
        if (launch_grouped_gemm(sd, s) != cudaSuccess) return MOE_ERR_CUDA;
    }
    record(ev, 4, s);

    GemmProblem dn = gu;
    dn.epi = fused ? 2 : 1;
    dn.Mw = f.H;
    dn.K = f.I;
    dn.Mvalid = f.H;
    dn.weights = static_cast<const char*>(f.packed) + geo.gu_bytes;
    dn.MT = geo.mt_dn;
    dn.KB = geo.kb_dn;
    dn.act = fp8 ? b.h_q : b.h;
    dn.gather_src = nullptr;
    dn.out = f.y_out;
    dn.ldo = f.H;
    dn.w = f.w;
    dn.act_amax = amax_h;
    dn.out_amax = nullptr;
    dn.acc_zero = nullptr;
    dn.acc_zero_floats = 0;
    dn.counters = b.ctl + kCtlCountersDn;
    if (lora) {
        dn.KBx = kLoraDnCols / 64;
        dn.x_tiles = lpk + lgeo.expand_d;
        dn.x_rows = b.t_dn;
    }
    dn.sched_after_wait = 0;   // the permutation is at least two kernels back
    {
        Range r(fused ? "moe: down GEMM + combine (a6 + a7)" : "moe: down GEMM (a6)");
        if (launch_grouped_gemm(dn, s) != cudaSuccess) return MOE_ERR_CUDA;
    }
    record(ev, 5, s);
    return MOE_OK;
}

size_t ffn_ws_bytes(moe_dtype dt, int T, int k, int E, int H, int I, int block_m) {
    Carver c{nullptr};
    const int cap = moe_permute_capacity(T, k, E, block_m);
    carve_ffn(c, dt, T, cap, H, I, gemm_nmax_for(T, k, E));
    return c.used;
}

struct FwdBuffers {
    int32_t* ids;
    float* w;
    int32_t* counts;
    int32_t* offsets;
    int32_t* num_tiles;
    int32_t* sorted_ids;
    int32_t* inv_perm;
    int32_t* tiles;
    int32_t* chunk_counts;
    void* y_out;      // y_perm (bf16 [cap, H]) or the fp32 accumulator [T, H]
    FfnBuffers ffn;
};

FwdBuffers carve_fwd(Carver& c, moe_dtype dt, int T, int k, int E, int H, int I, int block_m) {
    FwdBuffers b;
    const long A = static_cast<long>(T) * k;
    const int cap = moe_permute_capacity(T, k, E, block_m);
    b.ffn.ctl = c.take<int32_t>(sizeof(int32_t) * kCtlInts);
    b.ids = c.take<int32_t>(sizeof(int32_t) * A);
    b.w = c.take<float>(sizeof(float) * A);
    b.counts = c.take<int32_t>(sizeof(int32_t) * E);
    b.offsets = c.take<int32_t>(sizeof(int32_t) * (E + 1));
    b.num_tiles = c.take<int32_t>(sizeof(int32_t));
    b.sorted_ids = c.take<int32_t>(sizeof(int32_t) * (cap > 0 ? cap : 1));
    b.inv_perm = c.take<int32_t>(sizeof(int32_t) * (A > 0 ? A : 1));
    b.tiles = c.take<int32_t>(sizeof(int32_t) * (cap / block_m + 1));
    b.chunk_counts = c.take<int32_t>(sizeof(int32_t) * permute_chunks(A) * E);
    // one region serves either combine: y_perm or the fp32 accumulator
    const size_t yperm = static_cast<size_t>(cap) * H * 2;
    const size_t acc = static_cast<size_t>(T) * H * 4;
    b.y_out = c.take<void>(yperm > acc ? yperm : acc);
    carve_ffn_rest(c, b.ffn, dt, T, cap, H, I, gemm_nmax_for(T, k, E));
    return b;
}

// The combine a forward call uses.  The gather-sum is deterministic (a fixed
// summation order); the fused reduction skips the y_perm round trip through
// memory but adds in arrival order.  Auto takes the gather-sum: measured on
// B200, the fused form's L2 reductions slowed the down GEMM by about what
// they saved (prefill T = 4096: down +21 us, combine -25 us; skewed T = 8192:
// down +158 us, combine -144 us; FP8 T = 2048: +5 / -4 us).
Combine pick_combine(int mode) {
    return mode == MOE_COMBINE_FUSED ? Combine::kFused : Combine::kGatherSum;
}

}  // namespace

namespace moe {

size_t segment_ffn_ws_bytes(int T, int capacity, int H, int I) {
    Carver c{nullptr};
    carve_ffn(c, MOE_BF16, T, capacity, H, I, 256);   // partials for the largest cap
    return c.used;
}

moe_status segment_ffn(int T, int k, int E_sub, int H, int I, int capacity, int nmax,
                       const void* x, const float* w, const int32_t* counts,
                       const int32_t* offsets, const int32_t* sorted_ids, const void* packed,
                       void* y_perm, int32_t* status, void* ws, cudaStream_t s) {
    if (E_sub < 1 || E_sub > kMaxExperts || nmax < 16 || nmax > 256) return MOE_ERR_INVALID_ARG;
    Carver c{static_cast<char*>(ws)};
    const FfnBuffers b = carve_ffn(c, MOE_BF16, T, capacity, H, I, 256);
    if (cudaMemsetAsync(b.ctl, 0, sizeof(int32_t) * kCtlInts, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    FfnCall f{MOE_BF16, T, k, E_sub, H, I, capacity, x, w, counts, offsets, sorted_ids, packed,
              nullptr, y_perm, status ? status : b.ctl + kCtlStatus, 0};
    f.counts_from_prev = false;   // a memset comes between the permutation and the GEMM
    f.nmax = nmax;
    return run_ffn(f, b, nullptr, s);
}

}  // namespace moe

extern "C" {

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
        case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE";
    }
    return "MOE_ERR_UNKNOWN";
}

const char* moe_version(void) { return "moe-b200 0.1 (sm_100a)"; }

moe_status moe_route_topk(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                          moe_stream_t stream) {
    moe_status st = check_route(T, E, k);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    if (!logits || !ids || !w) return MOE_ERR_INVALID_ARG;
    return from_cuda(launch_route_topk(logits, T, E, k, ids, w, reinterpret_cast<cudaStream_t>(stream)));
}

int moe_permute_capacity(int T, int k, int E, int block_m) {
    if (T < 0 || k < 1 || E < 1 || block_m < 1) return -1;
    const long long A = static_cast<long long>(T) * k;
    const long long ne = A < E ? A : E;
    const long long c = A + ne * (block_m - 1);
    const long long r = (c + block_m - 1) / block_m * block_m;
    return r > INT32_MAX ? -1 : static_cast<int>(r);
}

size_t moe_align_permute_workspace_size(int T, int k, int E) {
    if (T < 0 || k < 1 || E < 1) return 0;
    const long A = static_cast<long>(T) * k;
    const int n = permute_chunks(A);
    return n <= 1 ? 0 : sizeof(int32_t) * static_cast<size_t>(n) * E;
}

moe_status moe_align_permute(const int32_t* ids, int T, int k, int E, int block_m,
                             int32_t* counts, int32_t* offsets, int32_t* sorted_ids,
                             int32_t* inv_perm, int32_t* tiles, int32_t* num_tiles, int capacity,
                             void* ws, size_t ws_bytes, moe_stream_t stream) {
    moe_status st = check_route(T, E, k);
    if (st != MOE_OK) return st;
    if (block_m < 1) return MOE_ERR_INVALID_ARG;
    if (!counts || !offsets || !num_tiles || (T > 0 && (!ids || !inv_perm)))
        return MOE_ERR_INVALID_ARG;
    const int need = moe_permute_capacity(T, k, E, block_m);
    if (need < 0) return MOE_ERR_UNSUPPORTED;
    if (capacity < need) return MOE_ERR_WORKSPACE;
    if (capacity > 0 && (!sorted_ids || !tiles)) return MOE_ERR_INVALID_ARG;
    const size_t wsn = moe_align_permute_workspace_size(T, k, E);
    if (wsn > 0 && (!ws || ws_bytes < wsn)) return MOE_ERR_WORKSPACE;
    return from_cuda(launch_align_permute(ids, T, k, E, block_m, capacity, counts, offsets,
                                          sorted_ids, inv_perm, tiles, num_tiles,
                                          static_cast<int32_t*>(ws), nullptr,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_packed_weights_size(moe_dtype dtype, int E, int H, int I) {
    if (E < 1 || H < 1 || I < 1) return 0;
    const PackedGeom g = packed_geom(dtype == MOE_FP8_E4M3, E, H, I);
    return g.gu_bytes + g.dn_bytes;
}

moe_status moe_pack_weights(moe_dtype dtype, int E, int H, int I, const void* Wg, const void* Wu,
                            const void* Wd, void* packed, float* scales, moe_stream_t stream) {
    if (dtype != MOE_BF16 && dtype != MOE_FP8_E4M3) return MOE_ERR_INVALID_ARG;
    if (E < 1 || H < 64 || I < 64) return MOE_ERR_INVALID_ARG;
    if (E > kMaxExperts || H % 64 || I % 64) return MOE_ERR_UNSUPPORTED;
    if (!Wg || !Wu || !Wd || !packed) return MOE_ERR_INVALID_ARG;
    if (!aligned16(Wg) || !aligned16(Wu) || !aligned16(Wd) || !aligned16(packed))
        return MOE_ERR_INVALID_ARG;
    const bool fp8 = dtype == MOE_FP8_E4M3;
    if (fp8 && (!scales || !aligned16(scales))) return MOE_ERR_INVALID_ARG;
    return from_cuda(launch_pack_weights(fp8, E, H, I, Wg, Wu, Wd, packed, scales,
                                         reinterpret_cast<uint32_t*>(scales),
                                         reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_packed_lora_size(int E, int H, int I, int n_adapters, int rank) {
    if (E < 1 || H < 64 || I < 64 || n_adapters < 1 || rank < 1) return 0;
    if (n_adapters * rank > 64 || E > kMaxExperts || H % 64 || I % 64) return 0;
    return lora_geom(E, H, I).bytes;
}

moe_status moe_pack_lora(int E, int H, int I, int n_adapters, int rank, const void* Ag,
                         const void* Bg, const void* Au, const void* Bu, const void* Ad,
                         const void* Bd, void* packed, moe_stream_t stream) {
    if (E < 1 || H < 64 || I < 64 || n_adapters < 1 || rank < 1) return MOE_ERR_INVALID_ARG;
    if (n_adapters * rank > 64 || E > kMaxExperts || H % 64 || I % 64) return MOE_ERR_UNSUPPORTED;
    if (!Ag || !Bg || !Au || !Bu || !Ad || !Bd || !packed || !aligned16(packed))
        return MOE_ERR_INVALID_ARG;
    return from_cuda(launch_pack_lora(E, H, I, n_adapters, rank, Ag, Bg, Au, Bu, Ad, Bd, packed,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_grouped_ffn_workspace_size(moe_dtype dtype, int T, int k, int E, int H, int I,
                                      int block_m) {
    if (check_layer(dtype, T, k, E, H, I, block_m) != MOE_OK) return 0;
    return ffn_ws_bytes(dtype, T, k, E, H, I, block_m);
}

moe_status moe_grouped_ffn(const moe_ffn_args* a, void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (!a) return MOE_ERR_INVALID_ARG;
    moe_status st = check_layer(a->dtype, a->T, a->k, a->E, a->H, a->I, a->block_m);
    if (st != MOE_OK) return st;
    if (a->T == 0) return MOE_OK;
    const int need = moe_permute_capacity(a->T, a->k, a->E, a->block_m);
    if (a->capacity < need) return MOE_ERR_WORKSPACE;
    if (!a->x || !a->w || !a->counts || !a->offsets || !a->sorted_ids || !a->packed || !a->y_perm)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(a->x) || !aligned16(a->packed) || !aligned16(a->y_perm))
        return MOE_ERR_INVALID_ARG;
    if (a->dtype == MOE_FP8_E4M3 && !a->scales) return MOE_ERR_INVALID_ARG;
    if (a->max_ctas < 0) return MOE_ERR_INVALID_ARG;
    const size_t need_ws = ffn_ws_bytes(a->dtype, a->T, a->k, a->E, a->H, a->I, a->block_m);
    if (!ws || ws_bytes < need_ws || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Carver c{static_cast<char*>(ws)};
    const FfnBuffers b = carve_ffn(c, a->dtype, a->T, a->capacity, a->H, a->I,
                                   gemm_nmax_for(a->T, a->k, a->E));
    if (cudaMemsetAsync(b.ctl, 0, sizeof(int32_t) * kCtlInts, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    FfnCall f{a->dtype, a->T, a->k, a->E, a->H, a->I, a->capacity, a->x, a->w, a->counts,
              a->offsets, a->sorted_ids, a->packed, a->scales, a->y_perm,
              a->status ? a->status : b.ctl + kCtlStatus, a->max_ctas};
    f.counts_from_prev = true;   // made by the caller's earlier calls: read after the wait
    return run_ffn(f, b, nullptr, s);
}

moe_status moe_combine(const void* y_perm, const int32_t* inv_perm, int T, int k, int H, void* out,
                       moe_stream_t stream) {
    if (T < 0 || k < 1 || H < 8 || H % 8) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!y_perm || !inv_perm || !out || !aligned16(y_perm) || !aligned16(out))
        return MOE_ERR_INVALID_ARG;
    return from_cuda(launch_combine(y_perm, inv_perm, T, k, H, out,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_forward_workspace_size(moe_dtype dtype, int T, int k, int E, int H, int I,
                                  int block_m) {
    if (block_m == 0) block_m = 16;
    if (check_layer(dtype, T, k, E, H, I, block_m) != MOE_OK) return 0;
    Carver c{nullptr};
    carve_fwd(c, dtype, T, k, E, H, I, block_m);
    return c.used;
}

moe_status moe_forward(const moe_forward_args* a, void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (!a) return MOE_ERR_INVALID_ARG;
    const int block_m = a->block_m == 0 ? 16 : a->block_m;
    moe_status st = check_layer(a->dtype, a->T, a->k, a->E, a->H, a->I, block_m);
    if (st != MOE_OK) return st;
    if (a->events && a->n_events != 7) return MOE_ERR_INVALID_ARG;
    if (a->max_ctas < 0) return MOE_ERR_INVALID_ARG;
    if (a->combine < MOE_COMBINE_AUTO || a->combine > MOE_COMBINE_FUSED)
        return MOE_ERR_INVALID_ARG;
    if (a->lora) {
        const moe_lora_args* l = a->lora;
        if (a->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
        if (l->n_adapters < 1 || l->rank < 1) return MOE_ERR_INVALID_ARG;
        if (l->n_adapters * l->rank > 64) return MOE_ERR_UNSUPPORTED;
        if (a->T > 0 && (!l->adapter || !l->packed || !l->scale || !aligned16(l->packed)))
            return MOE_ERR_INVALID_ARG;
    }
    if (a->T == 0) return MOE_OK;
    if (!a->x || !a->logits || !a->packed || !a->out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(a->x) || !aligned16(a->packed) || !aligned16(a->out))
        return MOE_ERR_INVALID_ARG;
    if (a->dtype == MOE_FP8_E4M3 && !a->scales) return MOE_ERR_INVALID_ARG;
    Carver probe{nullptr};
    carve_fwd(probe, a->dtype, a->T, a->k, a->E, a->H, a->I, block_m);
    if (!ws || ws_bytes < probe.used || !aligned16(ws)) return MOE_ERR_WORKSPACE;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Carver c{static_cast<char*>(ws)};
    const FwdBuffers b = carve_fwd(c, a->dtype, a->T, a->k, a->E, a->H, a->I, block_m);
    int32_t* ids = a->ids ? a->ids : b.ids;
    float* w = a->w ? a->w : b.w;
    const int cap = moe_permute_capacity(a->T, a->k, a->E, block_m);
    int32_t* status = a->status ? a->status : b.ffn.ctl + kCtlStatus;
    moe_event_t* ev = a->events;

    record(ev, 0, s);
    // The first kernel zeroes the control block (counters, amax words, and
    // the status word when the caller gave none) once the previous call's
    // kernels are done with it.
    cudaError_t e;
    const long x_elems = static_cast<long>(a->T) * a->H;
    const bool fp8 = a->dtype == MOE_FP8_E4M3;
    const bool small = fused_route_permute_ok(a->T, a->k);
    // FP8 with a small x: the single-CTA route kernel also takes amax(x) and
    // writes the codes of x
    const bool x_fused = small && fp8 && x_elems <= kSmallAmaxElems;
    Range whole("moe_forward");
    nvtxRangePushA("moe: route + permute (a1, a2)");
    if (small) {
        e = launch_route_permute_small(
            a->logits, a->T, a->E, a->k, block_m, cap, ids, w, b.counts, b.offsets, b.sorted_ids,
            b.inv_perm, b.tiles, b.num_tiles, status, s, b.ffn.ctl, kCtlInts,
            x_fused ? a->x : nullptr, x_elems,
            x_fused ? reinterpret_cast<uint32_t*>(b.ffn.ctl + kCtlAmaxX) : nullptr,
            x_fused ? b.ffn.xq : nullptr);
    } else {
        e = launch_route_topk(a->logits, a->T, a->E, a->k, ids, w, s, b.ffn.ctl, kCtlInts);
        if (e == cudaSuccess)
            e = launch_align_permute(ids, a->T, a->k, a->E, block_m, cap, b.counts, b.offsets,
                                     b.sorted_ids, b.inv_perm, b.tiles, b.num_tiles,
                                     b.chunk_counts, status, s);
    }
    nvtxRangePop();
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    record(ev, 1, s);
    FfnCall f{a->dtype, a->T, a->k, a->E, a->H, a->I, cap, a->x, w, b.counts, b.offsets,
              b.sorted_ids, a->packed, a->scales, b.y_out, status, a->max_ctas};
    f.x_ready = x_fused;
    // the permutation's last kernel (the single-CTA one, or scan + scatter,
    // which writes the counts) runs right before the gate/up GEMM, unless
    // FP8 or gather kernels come between (run_ffn clears the flag then)
    f.counts_from_prev = true;
    f.combine = pick_combine(a->combine);
    f.lora = a->lora;
    st = run_ffn(f, b.ffn, ev, s);
    if (st != MOE_OK) return st;
    {
        Range r("moe: combine (a7)");
        e = f.combine == Combine::kFused
                ? launch_finalize(static_cast<const float*>(b.y_out), x_elems, a->out, s)
                : launch_combine(b.y_out, b.inv_perm, a->T, a->k, a->H, a->out, s, cap, status);
    }
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    record(ev, 6, s);
    return MOE_OK;
}

moe_status moe_check_status(const int32_t* dev_status, moe_stream_t stream) {
    if (!dev_status) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    int32_t v = 0;
    if (cudaMemcpy(&v, dev_status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (v == 0) return MOE_OK;
    if (v == MOE_ERR_TIMEOUT || v == MOE_ERR_DEVICE) return static_cast<moe_status>(v);
    return MOE_ERR_DEVICE;
}

moe_status moe_selftest_wait_timeout(int32_t* dev_status, int timeout_us, moe_stream_t stream) {
    if (!dev_status || timeout_us < 1 || timeout_us > 1000000) return MOE_ERR_INVALID_ARG;
    return from_cuda(launch_wait_timeout_selftest(dev_status, timeout_us,
                                                  reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
