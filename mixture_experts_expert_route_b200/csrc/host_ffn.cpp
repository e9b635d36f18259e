// host_ffn.cpp -- the host side of the CPU/GPU expert split (include/moe_split.h):
// the host expert kernel, its weight layout, its thread pool, and the
// placement and per-batch plan of which experts run where.
//
// FIDDLER ("FIDDLER: CPU-GPU orchestration for fast inference of
// Mixture-of-Experts models", aibr.jp/archives/173321, § "3.中核となる技術的
// 要素") runs the experts that are not in GPU memory on the CPU with a kernel
// built on AVX512_BF16.  Here one expert for n tokens is two streaming
// passes over its weights:
//   pass 1: for every 16-column block of W_g and W_u, the n rows' dot
//           products over H, two rows of the weights at a time (bf16 pair
//           dot products into fp32), then h = bf16(SiLU(g) * u);
//   pass 2: for every 16-column block of W_d, the n rows' dot products of h
//           over I, then y = bf16(w * .).
// Decode batches give each host expert a handful of tokens, so the passes
// are bound by the host's memory bandwidth: each weight block is read once
// per group of tokens and stays in the core's cache for the next group.
// Where the CPU has AMX tiles the passes multiply 16 tokens x 32 K by 32 K x
// 16 columns per tile instruction (the weight layout is already the tiles'
// pair layout), which keeps them bound by memory up to hundreds of tokens;
// otherwise eight tokens share each 64-byte AVX512_BF16 pair product.
#include <immintrin.h>
#include <sys/syscall.h>
#include <unistd.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <condition_variable>
#include <cstdint>
#include <cstring>
#include <functional>
#include <limits>
#include <mutex>
#include <thread>
#include <vector>

#include "moe_split.h"

namespace {

constexpr int kCols = 16;      // columns per weight block (one fp32 vector)
constexpr int kTokBlock = 8;   // tokens sharing one pass over a block

// ---- thread pool: one worker per hardware thread, the caller included.
class HostPool {
  public:
    explicit HostPool(int n) : size_(n < 1 ? 1 : n) {
        for (int i = 1; i < size_; ++i) workers_.emplace_back([this, i] { loop(i); });
    }
    int size() const { return size_; }

    // Runs fn(task) for task in [0, n_tasks) on up to `threads` threads
    // (the calling thread is one of them) and returns when all are done.
    void run(int n_tasks, int threads, const std::function<void(int)>& fn) {
        std::lock_guard<std::mutex> one_at_a_time(run_mu_);
        const int use = std::max(1, std::min({threads <= 0 ? size_ : threads, size_, n_tasks}));
        {
            std::lock_guard<std::mutex> g(mu_);
            fn_ = &fn;
            n_tasks_ = n_tasks;
            next_.store(0);
            helpers_ = use - 1;
            pending_ = use - 1;
            ++generation_;
        }
        cv_.notify_all();
        work();
        std::unique_lock<std::mutex> g(mu_);
        done_cv_.wait(g, [this] { return pending_ == 0; });
        fn_ = nullptr;
    }

  private:
    void work() {
        for (int t = next_.fetch_add(1); t < n_tasks_; t = next_.fetch_add(1)) (*fn_)(t);
    }
    void loop(int index) {
        uint64_t seen = 0;
        for (;;) {
            {
                std::unique_lock<std::mutex> g(mu_);
                cv_.wait(g, [&] { return generation_ != seen; });
                seen = generation_;
                if (index > helpers_) continue;
            }
            work();
            {
                std::lock_guard<std::mutex> g(mu_);
                --pending_;
            }
            done_cv_.notify_one();
        }
    }

    const int size_;
    std::vector<std::thread> workers_;
    std::mutex run_mu_, mu_;
    std::condition_variable cv_, done_cv_;
    const std::function<void(int)>* fn_ = nullptr;
    int n_tasks_ = 0, helpers_ = 0, pending_ = 0;
    uint64_t generation_ = 0;
    std::atomic<int> next_{0};
};

HostPool& pool() {
    // Created on first use and never destroyed: its threads wait on a
    // condition variable until the process exits.  A child process made by
    // fork() has none of its parent's threads, so it gets a pool of its own
    // (the parent's object is left alone).
    static std::mutex mu;
    static HostPool* p = nullptr;
    static pid_t owner = 0;
    std::lock_guard<std::mutex> g(mu);
    if (!p || owner != getpid()) {
        p = new HostPool(static_cast<int>(std::thread::hardware_concurrency()));
        owner = getpid();
    }
    return *p;
}

// ---- bf16 <-> fp32
inline float bf16_to_f32(uint16_t v) {
    uint32_t u = static_cast<uint32_t>(v) << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}
// round to nearest, ties to even; NaN stays a quiet NaN
inline uint16_t f32_to_bf16(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return static_cast<uint16_t>((u >> 16) | 0x40);
    u += 0x7fffu + ((u >> 16) & 1u);
    return static_cast<uint16_t>(u >> 16);
}
inline float silu(float z) { return z / (1.0f + std::exp(-z)); }
// two consecutive bf16 values as one 32-bit word (the pair a dot product takes)
inline int load_pair(const uint16_t* p) {
    int v;
    std::memcpy(&v, p, 4);
    return v;
}

// ---- layout: per expert, G (W_g), U (W_u), D (W_d) sections; section of a
// [K][N] matrix = [N/16 column blocks][K/2 row pairs][16 columns][2 rows].
inline size_t section_elems(int K, int N) { return static_cast<size_t>(K) * N; }

void pack_section(const uint16_t* W, int K, int N, uint16_t* out) {
    const int nb = N / kCols, kp = K / 2;
    for (int c = 0; c < nb; ++c)
        for (int p = 0; p < kp; ++p) {
            uint16_t* o = out + (static_cast<size_t>(c) * kp + p) * kCols * 2;
            const uint16_t* r0 = W + static_cast<size_t>(2 * p) * N + c * kCols;
            const uint16_t* r1 = r0 + N;
            for (int i = 0; i < kCols; ++i) {
                o[2 * i] = r0[i];
                o[2 * i + 1] = r1[i];
            }
        }
}

// ---- the two passes, portable form: fp32 sums of the row-pair products
// (acc += w0*x0 + w1*x1, the pair summed first, like the bf16 dot product).
void gate_up_block_portable(const uint16_t* G, const uint16_t* U, int H, const uint16_t* x,
                            int n, int c, int I, uint16_t* h) {
    const int hp = H / 2;
    for (int t0 = 0; t0 < n; t0 += kTokBlock) {
        const int nt = std::min(kTokBlock, n - t0);
        float ag[kTokBlock][kCols] = {}, au[kTokBlock][kCols] = {};
        const uint16_t* g = G + static_cast<size_t>(c) * hp * kCols * 2;
        const uint16_t* u = U + static_cast<size_t>(c) * hp * kCols * 2;
        for (int p = 0; p < hp; ++p, g += 2 * kCols, u += 2 * kCols)
            for (int t = 0; t < nt; ++t) {
                const uint16_t* xr = x + static_cast<size_t>(t0 + t) * H + 2 * p;
                const float x0 = bf16_to_f32(xr[0]), x1 = bf16_to_f32(xr[1]);
                for (int i = 0; i < kCols; ++i) {
                    ag[t][i] += bf16_to_f32(g[2 * i]) * x0 + bf16_to_f32(g[2 * i + 1]) * x1;
                    au[t][i] += bf16_to_f32(u[2 * i]) * x0 + bf16_to_f32(u[2 * i + 1]) * x1;
                }
            }
        for (int t = 0; t < nt; ++t)
            for (int i = 0; i < kCols; ++i)
                h[static_cast<size_t>(t0 + t) * I + c * kCols + i] =
                    f32_to_bf16(silu(ag[t][i]) * au[t][i]);
    }
}

void down_block_portable(const uint16_t* D, int I, const uint16_t* h, const float* w, int n, int c,
                         int H, uint16_t* y) {
    const int ip = I / 2;
    for (int t0 = 0; t0 < n; t0 += kTokBlock) {
        const int nt = std::min(kTokBlock, n - t0);
        float acc[kTokBlock][kCols] = {};
        const uint16_t* d = D + static_cast<size_t>(c) * ip * kCols * 2;
        for (int p = 0; p < ip; ++p, d += 2 * kCols)
            for (int t = 0; t < nt; ++t) {
                const uint16_t* hr = h + static_cast<size_t>(t0 + t) * I + 2 * p;
                const float h0 = bf16_to_f32(hr[0]), h1 = bf16_to_f32(hr[1]);
                for (int i = 0; i < kCols; ++i)
                    acc[t][i] += bf16_to_f32(d[2 * i]) * h0 + bf16_to_f32(d[2 * i + 1]) * h1;
            }
        for (int t = 0; t < nt; ++t)
            for (int i = 0; i < kCols; ++i)
                y[static_cast<size_t>(t0 + t) * H + c * kCols + i] =
                    f32_to_bf16(w[t0 + t] * acc[t][i]);
    }
}

// ---- the same passes with AVX512_BF16: one 64-byte load holds a block's
// two rows for all 16 columns, and one vdpbf16ps multiplies them with the
// token's matching bf16 pair and adds both products into 16 fp32 sums.
#define MOE_AVX512BF16 __attribute__((target("avx512f,avx512bw,avx512vl,avx512bf16")))

MOE_AVX512BF16 inline void store_bf16_16(uint16_t* dst, __m512 v) {
    _mm256_storeu_si256(reinterpret_cast<__m256i*>(dst), (__m256i)_mm512_cvtneps_pbh(v));
}

MOE_AVX512BF16 void gate_up_block_avx512(const uint16_t* G, const uint16_t* U, int H,
                                         const uint16_t* x, int n, int c, int I, uint16_t* h) {
    const int hp = H / 2;
    for (int t0 = 0; t0 < n; t0 += kTokBlock) {
        const int nt = std::min(kTokBlock, n - t0);
        __m512 ag[kTokBlock], au[kTokBlock];
        for (int t = 0; t < kTokBlock; ++t) ag[t] = au[t] = _mm512_setzero_ps();
        const uint16_t* g = G + static_cast<size_t>(c) * hp * kCols * 2;
        const uint16_t* u = U + static_cast<size_t>(c) * hp * kCols * 2;
        if (nt == kTokBlock) {
            for (int p = 0; p < hp; ++p, g += 2 * kCols, u += 2 * kCols) {
                const __m512bh wg = (__m512bh)_mm512_loadu_si512(g);
                const __m512bh wu = (__m512bh)_mm512_loadu_si512(u);
#pragma GCC unroll 8
                for (int t = 0; t < kTokBlock; ++t) {
                    const __m512bh xb = (__m512bh)_mm512_set1_epi32(
                        load_pair(x + static_cast<size_t>(t0 + t) * H + 2 * p));
                    ag[t] = _mm512_dpbf16_ps(ag[t], wg, xb);
                    au[t] = _mm512_dpbf16_ps(au[t], wu, xb);
                }
            }
        } else {
            for (int p = 0; p < hp; ++p, g += 2 * kCols, u += 2 * kCols) {
                const __m512bh wg = (__m512bh)_mm512_loadu_si512(g);
                const __m512bh wu = (__m512bh)_mm512_loadu_si512(u);
                for (int t = 0; t < nt; ++t) {
                    const __m512bh xb = (__m512bh)_mm512_set1_epi32(
                        load_pair(x + static_cast<size_t>(t0 + t) * H + 2 * p));
                    ag[t] = _mm512_dpbf16_ps(ag[t], wg, xb);
                    au[t] = _mm512_dpbf16_ps(au[t], wu, xb);
                }
            }
        }
        for (int t = 0; t < nt; ++t) {
            alignas(64) float gv[kCols], uv[kCols];
            _mm512_store_ps(gv, ag[t]);
            _mm512_store_ps(uv, au[t]);
            for (int i = 0; i < kCols; ++i) gv[i] = silu(gv[i]) * uv[i];
            store_bf16_16(h + static_cast<size_t>(t0 + t) * I + c * kCols, _mm512_load_ps(gv));
        }
    }
}

MOE_AVX512BF16 void down_block_avx512(const uint16_t* D, int I, const uint16_t* h, const float* w,
                                      int n, int c, int H, uint16_t* y) {
    const int ip = I / 2;
    for (int t0 = 0; t0 < n; t0 += kTokBlock) {
        const int nt = std::min(kTokBlock, n - t0);
        __m512 acc[kTokBlock];
        for (int t = 0; t < kTokBlock; ++t) acc[t] = _mm512_setzero_ps();
        const uint16_t* d = D + static_cast<size_t>(c) * ip * kCols * 2;
        if (nt == kTokBlock) {
            for (int p = 0; p < ip; ++p, d += 2 * kCols) {
                const __m512bh wd = (__m512bh)_mm512_loadu_si512(d);
#pragma GCC unroll 8
                for (int t = 0; t < kTokBlock; ++t)
                    acc[t] = _mm512_dpbf16_ps(
                        acc[t], wd,
                        (__m512bh)_mm512_set1_epi32(
                            load_pair(h + static_cast<size_t>(t0 + t) * I + 2 * p)));
            }
        } else {
            for (int p = 0; p < ip; ++p, d += 2 * kCols) {
                const __m512bh wd = (__m512bh)_mm512_loadu_si512(d);
                for (int t = 0; t < nt; ++t)
                    acc[t] = _mm512_dpbf16_ps(
                        acc[t], wd,
                        (__m512bh)_mm512_set1_epi32(
                            load_pair(h + static_cast<size_t>(t0 + t) * I + 2 * p)));
            }
        }
        for (int t = 0; t < nt; ++t)
            store_bf16_16(y + static_cast<size_t>(t0 + t) * H + c * kCols,
                          _mm512_mul_ps(acc[t], _mm512_set1_ps(w[t0 + t])));
    }
}

// ---- the same passes on AMX tiles.  TDPBF16PS adds A[M][32] (bf16, M token
// rows) times B[16 pairs][16 columns] (bf16 pairs of consecutive K, one
// 64-byte row per pair: a 1 KB slice of a weight block) into C[M][16] fp32.
// Tiles: 0, 1 = C (gate, up; the down pass uses 0), 2 = A, 3, 4 = B.
// (Measured on the GPU machine's 16-core host: sharing each weight tile between
// two token blocks did not help at 128 tokens and slowed one token by 40%.)
#define MOE_AMX __attribute__((target("amx-tile,amx-bf16,avx512f,avx512bw,avx512vl,avx512bf16")))

struct alignas(64) TileConfig {
    uint8_t palette;
    uint8_t start_row;
    uint8_t reserved[14];
    uint16_t colsb[16];
    uint8_t rows[16];
};

MOE_AMX void amx_config(int M) {
    TileConfig cfg{};
    cfg.palette = 1;
    for (int t : {0, 1, 2}) {
        cfg.rows[t] = static_cast<uint8_t>(M);
        cfg.colsb[t] = 64;
    }
    for (int t : {3, 4}) {
        cfg.rows[t] = 16;
        cfg.colsb[t] = 64;
    }
    _tile_loadconfig(&cfg);
}

MOE_AMX void gate_up_block_amx(const uint16_t* G, const uint16_t* U, int H, const uint16_t* x,
                               int n, int c, int I, uint16_t* h) {
    const int hp = H / 2;
    const uint16_t* g0 = G + static_cast<size_t>(c) * hp * kCols * 2;
    const uint16_t* u0 = U + static_cast<size_t>(c) * hp * kCols * 2;
    constexpr size_t kSlice = 16 * kCols * 2;   // elements of one 1 KB weight slice
    alignas(64) float gv[16 * kCols], uv[16 * kCols];
    for (int t0 = 0; t0 < n; t0 += 16) {
        const int M = std::min(16, n - t0);
        amx_config(M);
        _tile_zero(0);
        _tile_zero(1);
        const uint16_t* xa = x + static_cast<size_t>(t0) * H;
        for (int kk = 0; kk < H / 32; ++kk) {
            _tile_loadd(2, xa + 32 * kk, H * 2);
            _tile_loadd(3, g0 + kk * kSlice, 64);
            _tile_loadd(4, u0 + kk * kSlice, 64);
            _tile_dpbf16ps(0, 2, 3);
            _tile_dpbf16ps(1, 2, 4);
        }
        _tile_stored(0, gv, 64);
        _tile_stored(1, uv, 64);
        _tile_release();
        for (int t = 0; t < M; ++t) {
            float* gr = gv + t * kCols;
            for (int i = 0; i < kCols; ++i) gr[i] = silu(gr[i]) * uv[t * kCols + i];
            store_bf16_16(h + static_cast<size_t>(t0 + t) * I + c * kCols, _mm512_load_ps(gr));
        }
    }
}

MOE_AMX void down_block_amx(const uint16_t* D, int I, const uint16_t* h, const float* w, int n,
                            int c, int H, uint16_t* y) {
    const int ip = I / 2;
    const uint16_t* d0 = D + static_cast<size_t>(c) * ip * kCols * 2;
    constexpr size_t kSlice = 16 * kCols * 2;
    alignas(64) float yv[16 * kCols];
    for (int t0 = 0; t0 < n; t0 += 16) {
        const int M = std::min(16, n - t0);
        amx_config(M);
        _tile_zero(0);
        const uint16_t* ha = h + static_cast<size_t>(t0) * I;
        for (int kk = 0; kk < I / 32; ++kk) {
            _tile_loadd(2, ha + 32 * kk, I * 2);
            _tile_loadd(3, d0 + kk * kSlice, 64);
            _tile_dpbf16ps(0, 2, 3);
        }
        _tile_stored(0, yv, 64);
        _tile_release();
        for (int t = 0; t < M; ++t)
            store_bf16_16(y + static_cast<size_t>(t0 + t) * H + c * kCols,
                          _mm512_mul_ps(_mm512_load_ps(yv + t * kCols),
                                        _mm512_set1_ps(w[t0 + t])));
    }
}

// AMX needs the CPU's tile instructions and, on Linux, the process's
// permission to use the tile state (requested once).
bool cpu_has_amx_bf16() {
    static const bool has = [] {
        if (!__builtin_cpu_supports("amx-tile") || !__builtin_cpu_supports("amx-bf16") ||
            !__builtin_cpu_supports("avx512bf16"))
            return false;
        constexpr long kReqXcompPerm = 0x1023, kXfeatureXtiledata = 18;
        return syscall(SYS_arch_prctl, kReqXcompPerm, kXfeatureXtiledata) == 0;
    }();
    return has;
}

bool cpu_has_avx512_bf16() {
    static const bool has = __builtin_cpu_supports("avx512f") &&
                            __builtin_cpu_supports("avx512bw") &&
                            __builtin_cpu_supports("avx512vl") &&
                            __builtin_cpu_supports("avx512bf16");
    return has;
}

bool valid_dims(int H, int I) { return H >= 64 && I >= 64 && H % 64 == 0 && I % 64 == 0; }

struct WhereItem {
    double saving;
    int e;
};

}  // namespace

extern "C" {

moe_status moe_split_place(const int64_t* hits, int E, int budget, int32_t* resident) {
    if (!hits || !resident || E < 1 || E > 256 || budget < 0 || budget > E)
        return MOE_ERR_INVALID_ARG;
    std::vector<int> order(E);
    for (int e = 0; e < E; ++e) {
        if (hits[e] < 0) return MOE_ERR_INVALID_ARG;
        order[e] = e;
    }
    std::stable_sort(order.begin(), order.end(),
                     [&](int a, int b) { return hits[a] > hits[b]; });
    for (int e = 0; e < E; ++e) resident[e] = 0;
    for (int i = 0; i < budget; ++i) resident[order[i]] = 1;
    return MOE_OK;
}

moe_status moe_split_plan(const int32_t* counts, const int32_t* resident, int E,
                          const moe_split_costs* c, int n_stage, int32_t* where) {
    if (!counts || !resident || !c || !where || E < 1 || E > 256 || n_stage < 0)
        return MOE_ERR_INVALID_ARG;
    std::vector<WhereItem> cand;
    for (int e = 0; e < E; ++e) {
        if (counts[e] < 0) return MOE_ERR_INVALID_ARG;
        if (counts[e] == 0) {
            where[e] = MOE_SPLIT_IDLE;
        } else if (resident[e]) {
            where[e] = MOE_SPLIT_RESIDENT;
        } else {
            where[e] = MOE_SPLIT_CPU;
            const double n = counts[e];
            const double cpu = c->cpu_us + c->cpu_us_per_token * n;
            const double gpu = c->xfer_us + c->gpu_us + c->gpu_us_per_token * n;
            if (gpu < cpu) cand.push_back({cpu - gpu, e});
        }
    }
    std::stable_sort(cand.begin(), cand.end(),
                     [](const WhereItem& a, const WhereItem& b) { return a.saving > b.saving; });
    const int take = std::min<int>(n_stage, static_cast<int>(cand.size()));
    for (int i = 0; i < take; ++i) where[cand[i].e] = MOE_SPLIT_STAGED;
    return MOE_OK;
}

moe_status moe_split_plan_balanced(const int32_t* counts, const int32_t* resident, int E,
                                   const moe_split_costs* c, int n_stage, int32_t* where) {
    if (!counts || !resident || !c || !where || E < 1 || E > 256 || n_stage < 0)
        return MOE_ERR_INVALID_ARG;
    struct Cand {
        double ratio, cpu, gpu;
        int e;
    };
    std::vector<Cand> cand;
    for (int e = 0; e < E; ++e) {
        if (counts[e] < 0) return MOE_ERR_INVALID_ARG;
        if (counts[e] == 0) {
            where[e] = MOE_SPLIT_IDLE;
        } else if (resident[e]) {
            where[e] = MOE_SPLIT_RESIDENT;
        } else {
            where[e] = MOE_SPLIT_CPU;
            const double n = counts[e];
            const double cpu = c->cpu_us + c->cpu_us_per_token * n;
            const double gpu = c->xfer_us + c->gpu_us + c->gpu_us_per_token * n;
            const double ratio = gpu <= 0 ? std::numeric_limits<double>::infinity() : cpu / gpu;
            cand.push_back({ratio, cpu, gpu, e});
        }
    }
    std::stable_sort(cand.begin(), cand.end(),
                     [](const Cand& a, const Cand& b) { return a.ratio > b.ratio; });
    const int m = std::min<int>(n_stage, static_cast<int>(cand.size()));
    int best_j = 0;
    double best = 0;
    for (int j = 0; j <= m; ++j) {
        double host = 0, link = 0;
        for (size_t i = j; i < cand.size(); ++i) host += cand[i].cpu;
        for (int i = 0; i < j; ++i) link += cand[i].gpu;
        const double cost = std::max(host, link);
        if (j == 0 || cost < best) {
            best = cost;
            best_j = j;
        }
    }
    for (int i = 0; i < best_j; ++i) where[cand[i].e] = MOE_SPLIT_STAGED;
    return MOE_OK;
}

size_t moe_host_packed_size(int H, int I) {
    if (!valid_dims(H, I)) return 0;
    return 3 * section_elems(H, I) * sizeof(uint16_t);
}

moe_status moe_host_pack_weights(int E, int H, int I, const uint16_t* Wg, const uint16_t* Wu,
                                 const uint16_t* Wd, void* packed) {
    if (E < 1 || !valid_dims(H, I) || !Wg || !Wu || !Wd || !packed) return MOE_ERR_INVALID_ARG;
    const size_t m = section_elems(H, I);
    uint16_t* out = static_cast<uint16_t*>(packed);
    pool().run(E * 3, 0, [&](int task) {
        const int e = task / 3, which = task % 3;
        uint16_t* dst = out + (static_cast<size_t>(e) * 3 + which) * m;
        if (which == 0) pack_section(Wg + e * m, H, I, dst);
        else if (which == 1) pack_section(Wu + e * m, H, I, dst);
        else pack_section(Wd + e * m, I, H, dst);
    });
    return MOE_OK;
}

int moe_host_isa(void) {
    if (cpu_has_amx_bf16()) return MOE_HOST_ISA_AMX_BF16;
    return cpu_has_avx512_bf16() ? MOE_HOST_ISA_AVX512_BF16 : MOE_HOST_ISA_PORTABLE;
}

moe_status moe_host_expert_ffn(const moe_host_ffn_args* a) {
    if (!a || !valid_dims(a->H, a->I) || a->n < 0) return MOE_ERR_INVALID_ARG;
    if (a->n == 0) return MOE_OK;
    if (!a->weights || !a->x || !a->w || !a->h || !a->y) return MOE_ERR_INVALID_ARG;
    const int H = a->H, I = a->I, n = a->n;
    const size_t m = section_elems(H, I);
    const uint16_t* G = static_cast<const uint16_t*>(a->weights);
    const uint16_t* U = G + m;
    const uint16_t* D = U + m;
    const bool portable = (a->flags & MOE_HOST_FLAG_PORTABLE) != 0;
    const int isa = portable ? MOE_HOST_ISA_PORTABLE
                    : (cpu_has_amx_bf16() && !(a->flags & MOE_HOST_FLAG_NO_AMX))
                        ? MOE_HOST_ISA_AMX_BF16
                        : cpu_has_avx512_bf16() ? MOE_HOST_ISA_AVX512_BF16
                                                : MOE_HOST_ISA_PORTABLE;
    pool().run(I / kCols, a->threads, [&](int c) {
        if (isa == MOE_HOST_ISA_AMX_BF16) gate_up_block_amx(G, U, H, a->x, n, c, I, a->h);
        else if (isa == MOE_HOST_ISA_AVX512_BF16) gate_up_block_avx512(G, U, H, a->x, n, c, I, a->h);
        else gate_up_block_portable(G, U, H, a->x, n, c, I, a->h);
    });
    pool().run(H / kCols, a->threads, [&](int c) {
        if (isa == MOE_HOST_ISA_AMX_BF16) down_block_amx(D, I, a->h, a->w, n, c, H, a->y);
        else if (isa == MOE_HOST_ISA_AVX512_BF16) down_block_avx512(D, I, a->h, a->w, n, c, H, a->y);
        else down_block_portable(D, I, a->h, a->w, n, c, H, a->y);
    });
    return MOE_OK;
}

}  // extern "C"
