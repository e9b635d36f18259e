// split.cu -- the CPU/GPU split layer of include/moe_split.h: routing on the
// GPU, the per-batch plan on the host, weight copies to staging slots, the
// slot permutation, the grouped FFNs of the resident and the staged experts,
// the host experts' rows, and the combine.
//
// After FIDDLER ("FIDDLER: CPU-GPU orchestration for fast inference of
// Mixture-of-Experts models", aibr.jp/archives/173321, § "3.中核となる技術的
// 要素"): experts outside GPU memory are either computed on the host or
// copied in, whichever the latency model expects to be faster for the
// batch's token count.  The slot permutation keeps every GPU expert's rows
// where the layer's grouped GEMMs and combine expect them, and puts the host
// experts' rows first (slot 0), in the order the host produces them.
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <chrono>
#include <cstring>
#include <vector>

#include "../../include/moe_split.h"
#include "kernels.h"

using namespace moe;

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

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

// slot_ids[f] = slot_of[ids[f]]; an id outside [0, E) drops the assignment
// (-1) and records MOE_ERR_DEVICE.
__global__ void slot_map_kernel(const int32_t* __restrict__ ids, long A,
                                const int32_t* __restrict__ slot_of, int E,
                                int32_t* __restrict__ slot_ids, int32_t* status) {
    for (long f = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; f < A;
         f += static_cast<long>(gridDim.x) * blockDim.x) {
        const int e = ids[f];
        if (e >= 0 && e < E) {
            slot_ids[f] = slot_of[e];
        } else {
            slot_ids[f] = -1;
            if (status) atomicCAS(status, 0, static_cast<int32_t>(MOE_ERR_DEVICE));
        }
    }
}

struct DevBuffers {
    int32_t* ctl;        // [64]: status word at 0
    int32_t* ids;
    float* w;
    int32_t* slot_ids;
    int32_t* slot_of;
    int32_t* counts;
    int32_t* offsets;
    int32_t* num_tiles;
    int32_t* sorted_ids;
    int32_t* inv_perm;
    int32_t* tiles;
    int32_t* chunk_counts;
    void* y_perm;
    void* ffn_res;
    void* ffn_stage;
};

DevBuffers carve_dev(Carver& c, int T, int k, int E, int Es, int H, int I, int block_m) {
    DevBuffers b;
    const long A = static_cast<long>(T) * k;
    const int cap = moe_permute_capacity(T, k, Es, block_m);
    b.ctl = c.take<int32_t>(64 * sizeof(int32_t));
    b.ids = c.take<int32_t>(sizeof(int32_t) * A);
    b.w = c.take<float>(sizeof(float) * A);
    b.slot_ids = c.take<int32_t>(sizeof(int32_t) * A);
    b.slot_of = c.take<int32_t>(sizeof(int32_t) * E);
    b.counts = c.take<int32_t>(sizeof(int32_t) * Es);
    b.offsets = c.take<int32_t>(sizeof(int32_t) * (Es + 1));
    b.num_tiles = c.take<int32_t>(sizeof(int32_t));
    b.sorted_ids = c.take<int32_t>(sizeof(int32_t) * (cap > 0 ? cap : 1));
    b.inv_perm = c.take<int32_t>(sizeof(int32_t) * (A > 0 ? A : 1));
    b.tiles = c.take<int32_t>(sizeof(int32_t) * (cap / block_m + 1));
    b.chunk_counts = c.take<int32_t>(sizeof(int32_t) * permute_chunks(A) * Es);
    b.y_perm = c.take<void>(static_cast<size_t>(cap) * H * 2);
    b.ffn_res = c.take<void>(segment_ffn_ws_bytes(T, cap, H, I));
    b.ffn_stage = c.take<void>(segment_ffn_ws_bytes(T, cap, H, I));
    return b;
}

struct HostBuffers {
    int32_t* ids;     // [A]
    float* w;         // [A]
    uint16_t* x;      // [T][H]
    int32_t* slot_of; // [256]
    uint16_t* y;      // [A][H]: the host experts' rows, in slot-0 order
    uint16_t* xg;     // [T][H]: one expert's input rows
    float* wg;        // [T]
    uint16_t* h;      // [T][I]
    uint16_t* yg;     // [T][H]
};

HostBuffers carve_host(Carver& c, int T, int k, int H, int I) {
    HostBuffers b;
    const long A = static_cast<long>(T) * k;
    b.ids = c.take<int32_t>(sizeof(int32_t) * A);
    b.w = c.take<float>(sizeof(float) * A);
    b.x = c.take<uint16_t>(sizeof(uint16_t) * T * static_cast<size_t>(H));
    b.slot_of = c.take<int32_t>(sizeof(int32_t) * 256);
    b.y = c.take<uint16_t>(sizeof(uint16_t) * A * static_cast<size_t>(H));
    b.xg = c.take<uint16_t>(sizeof(uint16_t) * T * static_cast<size_t>(H));
    b.wg = c.take<float>(sizeof(float) * T);
    b.h = c.take<uint16_t>(sizeof(uint16_t) * T * static_cast<size_t>(I));
    b.yg = c.take<uint16_t>(sizeof(uint16_t) * T * static_cast<size_t>(H));
    return b;
}

bool dims_ok(int T, int k, int E, int H, int I, int block_m) {
    return T >= 0 && k >= 1 && E >= 1 && k <= E && E <= 256 && H >= 64 && I >= 64 &&
           H % 64 == 0 && I % 64 == 0 && block_m >= 16 && block_m % 16 == 0 && block_m <= 4096;
}

int count_resident(const int32_t* resident, int E) {
    int S = 0;
    for (int e = 0; e < E; ++e) S += resident[e] != 0;
    return S;
}

// Token-tile cap of a group of experts: twice their mean tokens, as for a layer.
int group_nmax(const std::vector<int>& counts, const int32_t* where, int E, int kind) {
    long A = 0;
    int n = 0;
    for (int e = 0; e < E; ++e)
        if (where[e] == kind) {
            A += counts[e];
            ++n;
        }
    return n ? gemm_nmax_for(static_cast<int>(A), 1, n) : 0;
}

// NVTX range over one step of the split (free when no profiler is attached)
struct Range {
    explicit Range(const char* name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
    Range(const Range&) = delete;
    Range& operator=(const Range&) = delete;
};

double now_us() {
    return std::chrono::duration<double, std::micro>(
               std::chrono::steady_clock::now().time_since_epoch())
        .count();
}

}  // namespace

extern "C" {

size_t moe_split_workspace_size(int T, int k, int E, int S, int n_stage, int H, int I,
                                int block_m) {
    if (block_m == 0) block_m = 16;
    if (!dims_ok(T, k, E, H, I, block_m) || S < 0 || S > E || n_stage < 0) return 0;
    const int Es = 1 + S + n_stage;
    if (Es > 256) return 0;
    Carver c{nullptr};
    carve_dev(c, T, k, E, Es, H, I, block_m);
    return c.used;
}

size_t moe_split_host_workspace_size(int T, int k, int H, int I) {
    if (T < 0 || k < 1 || H < 64 || I < 64) return 0;
    Carver c{nullptr};
    carve_host(c, T, k, H, I);
    return c.used;
}

moe_status moe_split_calibrate(int H, int I, int n_max, const void* host_weights,
                               const void* host_src, void* dev_dst, void* host_ws,
                               size_t host_ws_bytes, int host_threads, moe_stream_t stream,
                               moe_split_costs* costs) {
    if (H < 64 || I < 64 || H % 64 || I % 64 || n_max < 1 || !host_weights || !host_src ||
        !dev_dst || !host_ws || !costs)
        return MOE_ERR_INVALID_ARG;
    if (host_ws_bytes < moe_split_host_workspace_size(n_max, 1, H, I)) return MOE_ERR_WORKSPACE;
    Carver c{static_cast<char*>(host_ws)};
    const HostBuffers hb = carve_host(c, n_max, 1, H, I);
    std::memset(hb.xg, 0, sizeof(uint16_t) * n_max * static_cast<size_t>(H));
    for (int i = 0; i < n_max; ++i) hb.wg[i] = 1.0f;
    auto host_run = [&](int n, int reps) {
        double best = 1e300;
        for (int r = 0; r < reps; ++r) {
            moe_host_ffn_args a{H, I, n, host_weights, hb.xg, hb.wg, hb.h, hb.yg, host_threads, 0};
            const double t0 = now_us();
            if (moe_host_expert_ffn(&a) != MOE_OK) return -1.0;
            best = std::min(best, now_us() - t0);
        }
        return best;
    };
    const double t1 = host_run(1, 3);
    const double tn = n_max > 1 ? host_run(n_max, 2) : t1;
    if (t1 < 0 || tn < 0) return MOE_ERR_INVALID_ARG;
    const double per = n_max > 1 ? std::max(0.0, (tn - t1) / (n_max - 1)) : 0.0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t bytes = 3 * static_cast<size_t>(H) * I * 2;
    double xfer = 1e300;
    for (int r = 0; r < 3; ++r) {
        if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
        const double t0 = now_us();
        if (cudaMemcpyAsync(dev_dst, host_src, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return MOE_ERR_CUDA;
        xfer = std::min(xfer, now_us() - t0);
    }
    costs->cpu_us = std::max(0.0, t1 - per);
    costs->cpu_us_per_token = per;
    costs->xfer_us = xfer;
    costs->gpu_us = 0.0;
    costs->gpu_us_per_token = 0.0;
    return MOE_OK;
}

moe_status moe_split_forward(const moe_split_args* a, void* ws, size_t ws_bytes, void* host_ws,
                             size_t host_ws_bytes, moe_stream_t stream) {
    if (!a) return MOE_ERR_INVALID_ARG;
    const int block_m = a->block_m == 0 ? 16 : a->block_m;
    const int T = a->T, k = a->k, E = a->E, H = a->H, I = a->I;
    if (!dims_ok(T, k, E, H, I, block_m)) return MOE_ERR_INVALID_ARG;
    if (!a->resident || a->n_stage < 0) return MOE_ERR_INVALID_ARG;
    if (a->policy < MOE_SPLIT_POLICY_DYNAMIC || a->policy > MOE_SPLIT_POLICY_BALANCED)
        return MOE_ERR_INVALID_ARG;
    if ((a->policy == MOE_SPLIT_POLICY_DYNAMIC || a->policy == MOE_SPLIT_POLICY_BALANCED) &&
        !a->costs)
        return MOE_ERR_INVALID_ARG;
    if ((a->copy_stream == nullptr) != (a->copy_event == nullptr)) return MOE_ERR_INVALID_ARG;
    const int S = count_resident(a->resident, E);
    const int Es = 1 + S + a->n_stage;
    if (Es > 256) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!a->x || !a->logits || !a->out || !a->host_weights) return MOE_ERR_INVALID_ARG;
    if (S > 0 && !a->resident_packed) return MOE_ERR_INVALID_ARG;
    if (a->n_stage > 0 && (!a->stage_packed || !a->host_packed)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(a->x) || !aligned16(a->out) ||
        (a->resident_packed && !aligned16(a->resident_packed)) ||
        (a->stage_packed && !aligned16(a->stage_packed)))
        return MOE_ERR_INVALID_ARG;
    const size_t need = moe_split_workspace_size(T, k, E, S, a->n_stage, H, I, block_m);
    if (!ws || ws_bytes < need || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    if (!host_ws || host_ws_bytes < moe_split_host_workspace_size(T, k, H, I))
        return MOE_ERR_WORKSPACE;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Carver cd{static_cast<char*>(ws)};
    const DevBuffers d = carve_dev(cd, T, k, E, Es, H, I, block_m);
    Carver chost{static_cast<char*>(host_ws)};
    const HostBuffers hb = carve_host(chost, T, k, H, I);
    const long A = static_cast<long>(T) * k;
    const int cap = moe_permute_capacity(T, k, Es, block_m);
    int32_t* status = a->status ? a->status : d.ctl;

    Range whole("moe_split_forward");
    // 1. route on the GPU, bring the routing and x to the host
    {
        Range r("moe split: route, routing to the host");
        if (!a->status && cudaMemsetAsync(d.ctl, 0, 64 * sizeof(int32_t), s) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (launch_route_topk(a->logits, T, E, k, d.ids, d.w, s) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (cudaMemcpyAsync(hb.ids, d.ids, sizeof(int32_t) * A, cudaMemcpyDeviceToHost, s) !=
                cudaSuccess ||
            cudaMemcpyAsync(hb.w, d.w, sizeof(float) * A, cudaMemcpyDeviceToHost, s) !=
                cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return MOE_ERR_CUDA;
    }

    // 2. the plan
    std::vector<int> counts(E, 0);
    for (long f = 0; f < A; ++f) {
        const int e = hb.ids[f];
        if (e < 0 || e >= E) return MOE_ERR_DEVICE;
        ++counts[e];
    }
    std::vector<int32_t> where(E);
    moe_status st;
    if (a->policy == MOE_SPLIT_POLICY_DYNAMIC) {
        st = moe_split_plan(counts.data(), a->resident, E, a->costs, a->n_stage, where.data());
    } else if (a->policy == MOE_SPLIT_POLICY_BALANCED) {
        st = moe_split_plan_balanced(counts.data(), a->resident, E, a->costs, a->n_stage,
                                     where.data());
    } else {
        // ALL_CPU: no expert gains from a copy; ALL_STAGED: every one does
        // (equal savings, so staging slots go to the lowest indices)
        moe_split_costs fixed{};
        fixed.cpu_us = a->policy == MOE_SPLIT_POLICY_ALL_STAGED ? 1e30 : 0.0;
        fixed.xfer_us = a->policy == MOE_SPLIT_POLICY_ALL_STAGED ? 0.0 : 1e30;
        st = moe_split_plan(counts.data(), a->resident, E, &fixed, a->n_stage, where.data());
    }
    if (st != MOE_OK) return st;
    if (a->where) std::memcpy(a->where, where.data(), sizeof(int32_t) * E);

    // the host experts' assignments, bucketed by expert in ascending flat
    // index; x comes to the host only when some expert runs there (the stream
    // is idle at this point, so the wait is for this copy alone)
    std::vector<std::vector<long>> host_rows(E);
    std::vector<int> pos(A, -1);
    int n_cpu = 0;
    for (long f = 0; f < A; ++f) {
        const int e = hb.ids[f];
        if (where[e] == MOE_SPLIT_CPU) {
            pos[f] = n_cpu++;
            host_rows[e].push_back(f);
        }
    }
    if (n_cpu > 0) {
        Range r("moe split: x to the host");
        if (cudaMemcpyAsync(hb.x, a->x, sizeof(uint16_t) * T * static_cast<size_t>(H),
                            cudaMemcpyDeviceToHost, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return MOE_ERR_CUDA;
    }

    // 3. slots, weight copies, slot permutation, the GPU experts
    Range gpu_part("moe split: weight copies, slot permutation, GPU experts");
    std::vector<int> staged;
    {
        int r = 0;
        for (int e = 0; e < E; ++e) {
            if (a->resident[e]) {
                hb.slot_of[e] = 1 + r++;
            } else if (where[e] == MOE_SPLIT_STAGED) {
                hb.slot_of[e] = 1 + S + static_cast<int>(staged.size());
                staged.push_back(e);
            } else {
                hb.slot_of[e] = 0;
            }
        }
    }
    if (cudaMemcpyAsync(d.slot_of, hb.slot_of, sizeof(int32_t) * E, cudaMemcpyHostToDevice, s) !=
        cudaSuccess)
        return MOE_ERR_CUDA;
    if (!staged.empty()) {
        // host_packed: expert e's own packed layout (E = 1) at e * (gate/up +
        // down bytes); the staging buffer: the packed layout of n_stage experts
        const PackedGeom one = packed_geom(0, 1, H, I);
        const PackedGeom stg = packed_geom(0, a->n_stage, H, I);
        const size_t per_expert = one.gu_bytes + one.dn_bytes;
        cudaStream_t cs = a->copy_stream ? reinterpret_cast<cudaStream_t>(a->copy_stream) : s;
        const char* src = static_cast<const char*>(a->host_packed);
        char* dst = static_cast<char*>(a->stage_packed);
        for (size_t j = 0; j < staged.size(); ++j) {
            const char* se = src + static_cast<size_t>(staged[j]) * per_expert;
            if (cudaMemcpyAsync(dst + j * one.gu_bytes, se, one.gu_bytes, cudaMemcpyHostToDevice,
                                cs) != cudaSuccess ||
                cudaMemcpyAsync(dst + stg.gu_bytes + j * one.dn_bytes, se + one.gu_bytes,
                                one.dn_bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess)
                return MOE_ERR_CUDA;
        }
        if (a->copy_event &&
            cudaEventRecord(reinterpret_cast<cudaEvent_t>(a->copy_event), cs) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    const int blocks = static_cast<int>(std::min<long>((A + 255) / 256, 1024));
    slot_map_kernel<<<blocks, 256, 0, s>>>(d.ids, A, d.slot_of, E, d.slot_ids, status);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    if (launch_align_permute(d.slot_ids, T, k, Es, block_m, cap, d.counts, d.offsets,
                             d.sorted_ids, d.inv_perm, d.tiles, d.num_tiles, d.chunk_counts,
                             status, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    const int nmax_res = group_nmax(counts, where.data(), E, MOE_SPLIT_RESIDENT);
    if (nmax_res > 0) {
        st = segment_ffn(T, k, S, H, I, cap, nmax_res, a->x, d.w, d.counts + 1, d.offsets + 1,
                         d.sorted_ids, a->resident_packed, d.y_perm, status, d.ffn_res, s);
        if (st != MOE_OK) return st;
    }
    if (!staged.empty()) {
        if (a->copy_event &&
            cudaStreamWaitEvent(s, reinterpret_cast<cudaEvent_t>(a->copy_event), 0) != cudaSuccess)
            return MOE_ERR_CUDA;
        const int nmax_stg = group_nmax(counts, where.data(), E, MOE_SPLIT_STAGED);
        st = segment_ffn(T, k, a->n_stage, H, I, cap, nmax_stg, a->x, d.w, d.counts + 1 + S,
                         d.offsets + 1 + S, d.sorted_ids, a->stage_packed, d.y_perm, status,
                         d.ffn_stage, s);
        if (st != MOE_OK) return st;
    }

    // 4. the host experts, while the GPU runs; their rows go to slot 0 in
    // ascending flat index, the order the stable permutation gives them
    Range host_part("moe split: host experts, combine");
    if (n_cpu > 0) {
        const size_t expert_bytes = moe_host_packed_size(H, I);
        for (int e = 0; e < E; ++e) {
            if (where[e] != MOE_SPLIT_CPU) continue;
            const std::vector<long>& rows = host_rows[e];
            const int n = static_cast<int>(rows.size());
            for (int r = 0; r < n; ++r) {
                std::memcpy(hb.xg + static_cast<size_t>(r) * H,
                            hb.x + static_cast<size_t>(rows[r] / k) * H, sizeof(uint16_t) * H);
                hb.wg[r] = hb.w[rows[r]];
            }
            moe_host_ffn_args ha{H, I, n,
                                 static_cast<const char*>(a->host_weights) + e * expert_bytes,
                                 hb.xg, hb.wg, hb.h, hb.yg, a->host_threads, 0};
            st = moe_host_expert_ffn(&ha);
            if (st != MOE_OK) return st;
            for (int r = 0; r < n; ++r)
                std::memcpy(hb.y + static_cast<size_t>(pos[rows[r]]) * H,
                            hb.yg + static_cast<size_t>(r) * H, sizeof(uint16_t) * H);
        }
        if (cudaMemcpyAsync(d.y_perm, hb.y, sizeof(uint16_t) * n_cpu * static_cast<size_t>(H),
                            cudaMemcpyHostToDevice, s) != cudaSuccess)
            return MOE_ERR_CUDA;
    }

    // 5. combine
    if (launch_combine(d.y_perm, d.inv_perm, T, k, H, a->out, s, cap, status) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

}  // extern "C"
