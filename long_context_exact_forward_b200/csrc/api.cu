// api.cu -- the C ABI of include/ra.h: argument validation, the causal block-skip planner, the
// workspace carve-up and the launch sequence of each variant.
//
// Launch sequence of ra_forward (everything on the caller's stream):
//   tensor-core kernel (bf16, D in {64, 128}):
//     1. zigzag only: permute q, k, v into shard-major order (contiguous is already shard-major,
//        S = N * S_loc; striped is read in place through a strided tensor map)
//     2. fused:    one persistent launch walks all N ring steps and writes out / lse in natural
//                  order (the unpermute is folded into its epilogue)
//        per-step: for s = 0 .. N-1 one launch writes the step's partial (O_s, lse_s); an HBM-bound
//                  merge folds it into the running (O, lse); the last merge writes out / lse in
//                  natural order
//   SIMT kernel (fp32, or other head dims): the same two variants, reading natural order directly.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "ra.h"
#include "ra_internal.cuh"

__device__ int g_ra_device_status = 0;

namespace {

using ra::Layout;

thread_local char g_last_error[512] = "";

int cuda_fail(cudaError_t e, const char* what) {
    snprintf(g_last_error, sizeof g_last_error, "%s: %s (%s)", what, cudaGetErrorString(e),
             cudaGetErrorName(e));
    return RA_ERR_CUDA;
}

constexpr int kTcTileM = 128;   // query tile rows of the tensor-core kernel
constexpr int kTcPairRows = 2 * kTcTileM;
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(int64_t B, int64_t H, int64_t S, int64_t D, int n_ring, int layout, int dtype) {
    if (B < 1 || H < 1 || S < 1 || D < 1 || n_ring < 1) return RA_ERR_INVALID_ARG;
    if (layout < RA_LAYOUT_CONTIGUOUS || layout > RA_LAYOUT_ZIGZAG) return RA_ERR_INVALID_ARG;
    if (dtype != RA_DTYPE_FP32 && dtype != RA_DTYPE_BF16) return RA_ERR_INVALID_ARG;
    if (D > 256) return RA_ERR_SHAPE;
    if (S % n_ring != 0) return RA_ERR_SHAPE;
    if (layout == RA_LAYOUT_ZIGZAG && S % (2 * (int64_t)n_ring) != 0) return RA_ERR_SHAPE;
    // TMA coordinates and grid dimensions are 32-bit
    if (S >= (int64_t(1) << 31) || B * H >= (int64_t(1) << 31)) return RA_ERR_SHAPE;
    return RA_OK;
}

Layout make_layout(int64_t S, int n_ring, int layout) {
    return Layout{S, (int64_t)n_ring, S / n_ring, layout};
}

// ------------------------------------------------------------------ device facts (cached)
struct DeviceInfo {
    int sms = 0;
    bool sm100 = false;
    int* status = nullptr;
};

int device_info(DeviceInfo* out) {
    static std::mutex mu;
    static std::map<int, DeviceInfo> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(dev);
    if (it != cache.end()) {
        *out = it->second;
        return RA_OK;
    }
    DeviceInfo d;
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
        return cuda_fail(e, "cudaDeviceGetAttribute");
    if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
        return cuda_fail(e, "cudaDeviceGetAttribute");
    if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return cuda_fail(e, "cudaDeviceGetAttribute");
    d.sm100 = (major == 10 && minor == 0);
    if ((e = cudaGetSymbolAddress(reinterpret_cast<void**>(&d.status), g_ra_device_status)) != cudaSuccess)
        return cuda_fail(e, "cudaGetSymbolAddress");
    cache[dev] = d;
    *out = d;
    return RA_OK;
}

// ------------------------------------------------------------------ planner
int tc_tiles_for(const Layout& L, int causal, int64_t i, int64_t a0, int64_t j) {
    if (a0 >= L.S_loc) return 0;
    const int64_t last = std::min(a0 + kTcTileM - 1, L.S_loc - 1);
    const int64_t n = ra::visible_keys(L, causal, i, last, j);
    return (int)((n + kTcTileM - 1) / kTcTileM);
}

struct PlanKey {
    int64_t B, H, S;
    int n_ring, causal, layout, s_begin, s_end;
    int64_t D;
    bool operator<(const PlanKey& o) const {
        return std::tie(B, H, S, n_ring, causal, layout, s_begin, s_end, D) <
               std::tie(o.B, o.H, o.S, o.n_ring, o.causal, o.layout, o.s_begin, o.s_end, o.D);
    }
};

struct PlanItem {
    int32_t b, h, i, p, cost;
};

// Work list of the tensor-core kernel for ring steps [s_begin, s_end): one item per
// (b, h, shard i, pair of 128-row query tiles), cost = live (query tile, key tile) pairs.
// Order: (b, h) major so that CTAs running at the same time share one head's keys and values in
// L2; inside a head, heaviest first (LPT) so the short items fill the tail -- or, when one head's
// K/V exceeds L2 (plan_groups_by_shard), shard groups heaviest first and LPT inside a group.
const std::vector<PlanItem>& plan_items(int64_t B, int64_t H, const Layout& L, int64_t D_for_plan,
                                        int causal, int s_begin, int s_end) {
    static std::mutex mu;
    static std::map<PlanKey, std::vector<PlanItem>> cache;
    PlanKey key{B, H, L.S, (int)L.N, causal, L.kind, s_begin, s_end, D_for_plan};
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    const int64_t pairs = (L.S_loc + kTcPairRows - 1) / kTcPairRows;
    std::vector<PlanItem> head;
    head.reserve((size_t)(L.N * pairs));
    for (int64_t i = 0; i < L.N; ++i)
        for (int64_t p = 0; p < pairs; ++p) {
            int64_t cost = 0;
            for (int s = s_begin; s < s_end; ++s) {
                const int64_t j = ra::ring_block(i, s, L.N);
                cost += tc_tiles_for(L, causal, i, p * kTcPairRows, j) +
                        tc_tiles_for(L, causal, i, p * kTcPairRows + kTcTileM, j);
            }
            head.push_back(PlanItem{0, 0, (int32_t)i, (int32_t)p, (int32_t)std::min<int64_t>(cost, INT32_MAX)});
        }
    if (ra::plan_groups_by_shard(L.S, D_for_plan)) {
        // one head's K/V does not fit L2: group the items of one shard (they walk the same ring
        // sequence of key/value blocks, so CTAs running together share tiles in L2), groups
        // heaviest first, items heaviest first inside a group
        std::vector<int64_t> group_cost((size_t)L.N, 0);
        for (const PlanItem& x : head) group_cost[(size_t)x.i] += x.cost;
        std::stable_sort(head.begin(), head.end(), [&](const PlanItem& x, const PlanItem& y) {
            if (group_cost[(size_t)x.i] != group_cost[(size_t)y.i])
                return group_cost[(size_t)x.i] > group_cost[(size_t)y.i];
            if (x.i != y.i) return x.i < y.i;
            return x.cost > y.cost;
        });
    } else {
        std::stable_sort(head.begin(), head.end(),
                         [](const PlanItem& x, const PlanItem& y) { return x.cost > y.cost; });
    }
    std::vector<PlanItem> all;
    all.reserve(head.size() * (size_t)(B * H));
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < H; ++h)
            for (PlanItem x : head) {
                x.b = (int32_t)b;
                x.h = (int32_t)h;
                all.push_back(x);
            }
    return cache.emplace(key, std::move(all)).first->second;
}

// All lists of one call flattened into pinned host memory (kept for the life of the process, so
// the asynchronous upload never reads freed or pageable memory).  offsets[s] .. offsets[s + 1]
// delimit the list of step s (per-step) or the single list (fused).
struct FlatList {
    int4* data = nullptr;
    size_t count = 0;
    std::vector<int> offsets;
};

int flat_items(int64_t B, int64_t H, const Layout& L, int64_t D, int causal, bool per_step,
               const FlatList** out) {
    static std::mutex mu;
    static std::map<std::pair<PlanKey, bool>, FlatList> cache;
    const PlanKey key{B, H, L.S, (int)L.N, causal, L.kind, 0, (int)L.N, D};
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find({key, per_step});
        if (it != cache.end()) {
            *out = &it->second;
            return RA_OK;
        }
    }
    FlatList f;
    std::vector<int4> flat;
    const int n_lists = per_step ? (int)L.N : 1;
    for (int s = 0; s < n_lists; ++s) {
        f.offsets.push_back((int)flat.size());
        const auto& items = per_step ? plan_items(B, H, L, D, causal, s, s + 1) : plan_items(B, H, L, D, causal, 0, (int)L.N);
        for (const PlanItem& x : items) flat.push_back(make_int4(x.b, x.h, x.i, x.p));
    }
    f.offsets.push_back((int)flat.size());
    f.count = flat.size();
    if (f.count) {
        cudaError_t e = cudaHostAlloc(reinterpret_cast<void**>(&f.data), f.count * sizeof(int4), cudaHostAllocPortable);
        if (e != cudaSuccess) return cuda_fail(e, "cudaHostAlloc(work list)");
        std::memcpy(f.data, flat.data(), f.count * sizeof(int4));
    }
    std::lock_guard<std::mutex> lock(mu);
    auto ins = cache.emplace(std::make_pair(key, per_step), std::move(f));
    if (!ins.second && f.data) cudaFreeHost(f.data);  // another thread won the race
    *out = &ins.first->second;
    return RA_OK;
}

// ------------------------------------------------------------------ workspace
enum Kernel { kTC, kSIMT };

struct Workspace {
    size_t counters = 0, n_counters = 0;  // one work counter per attention launch (zeroed per call)
    size_t items = 0, n_items_total = 0;
    size_t qp = 0, kp = 0, vp = 0;  // permuted q, k, v
    size_t O_run = 0, lse_run = 0, O_step = 0, lse_step = 0;
    bool permute = false, per_step = false;
    size_t total = 0;
};

Workspace carve(int64_t B, int64_t H, const Layout& L, int64_t D, int causal, int dtype,
                bool per_step, Kernel kernel) {
    Workspace w;
    size_t off = 0;
    const size_t esize = dtype == RA_DTYPE_BF16 ? 2 : 4;
    const size_t elems = (size_t)(B * L.S * H * D);
    w.per_step = per_step && L.N > 1;
    if (kernel == kTC) {
        if (w.per_step) {
            for (int s = 0; s < (int)L.N; ++s) w.n_items_total += plan_items(B, H, L, D, causal, s, s + 1).size();
        } else {
            w.n_items_total = plan_items(B, H, L, D, causal, 0, (int)L.N).size();
        }
        w.counters = off;
        w.n_counters = w.per_step ? (size_t)L.N : 1;
        off = align_up(off + w.n_counters * sizeof(int));
        w.items = off;
        off = align_up(off + w.n_items_total * sizeof(int4));
        // striped is read in place through a strided tensor map; zigzag is gathered shard-major
        w.permute = (L.kind == RA_LAYOUT_ZIGZAG);
        if (w.permute) {
            w.qp = off;
            off = align_up(off + elems * esize);
            w.kp = off;
            off = align_up(off + elems * esize);
            w.vp = off;
            off = align_up(off + elems * esize);
        }
    }
    if (w.per_step) {
        const size_t rows = (size_t)(B * L.S * H);
        w.O_run = off;
        off = align_up(off + elems * 4);
        w.lse_run = off;
        off = align_up(off + rows * 4);
        w.O_step = off;
        off = align_up(off + elems * 4);
        w.lse_step = off;
        off = align_up(off + rows * 4);
    }
    w.total = std::max<size_t>(off, kAlign);
    return w;
}

// ------------------------------------------------------------------ TMA descriptors
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// bf16 q/k/v viewed as 5-D (D, H, a, i, B) -- local token a of shard i -- so that the kernel's
// TMA coordinates are the same for every source:
//   shard-major [B, N, S_loc, H, D] (contiguous layout, or a permuted copy): a-stride H*D, i-stride S_loc*H*D;
//   natural order under the striped layout (token a*N + i):                   a-stride N*H*D, i-stride H*D.
// One box is 64 head-dim elements (128 bytes, the 128-byte swizzle span) x 1 head x 128 tokens;
// tokens past the shard end read as zero.
int encode_qkv_map(CUtensorMap* map, const void* base, int64_t B, const Layout& L, int64_t H, int64_t D,
                   bool striped_natural) {
    auto fn = encode_fn();
    if (!fn) {
        snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled entry point unavailable");
        return RA_ERR_CUDA;
    }
    const cuuint64_t row = (cuuint64_t)(H * D * 2);
    const cuuint64_t dims[5] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)L.S_loc, (cuuint64_t)L.N, (cuuint64_t)B};
    const cuuint64_t strides[4] = {(cuuint64_t)(D * 2), striped_natural ? row * (cuuint64_t)L.N : row,
                                   striped_natural ? row : row * (cuuint64_t)L.S_loc, row * (cuuint64_t)L.S};
    const cuuint32_t box[5] = {64, 1, (cuuint32_t)kTcTileM, 1, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed (%d)", (int)r);
        return RA_ERR_CUDA;
    }
    return RA_OK;
}

// ------------------------------------------------------------------ the forward pass
struct Call {
    const void *q, *k, *v;
    void* out;
    float* lse;
    int64_t B, H, S, D;
    int n_ring, causal, layout, dtype;
    cudaStream_t stream;
};

int select_kernel(const Call& c, int requested, const DeviceInfo& dev, Kernel* k) {
    const bool tc_ok = dev.sm100 && c.dtype == RA_DTYPE_BF16 && (c.D == 64 || c.D == 128);
    if (requested == RA_KERNEL_TC) {
        if (!tc_ok) return RA_ERR_UNSUPPORTED;
        *k = kTC;
    } else if (requested == RA_KERNEL_SIMT) {
        *k = kSIMT;
    } else if (requested == RA_KERNEL_AUTO) {
        *k = tc_ok ? kTC : kSIMT;
    } else {
        return RA_ERR_INVALID_ARG;
    }
    return RA_OK;
}

int run_forward(const Call& c, const ra_options& opt) {
    int rc = check_shape(c.B, c.H, c.S, c.D, c.n_ring, c.layout, c.dtype);
    if (rc != RA_OK) return rc;
    if (!c.q || !c.k || !c.v || !c.out || !c.lse) return RA_ERR_INVALID_ARG;
    if (!aligned16(c.q) || !aligned16(c.k) || !aligned16(c.v) || !aligned16(c.out) ||
        (reinterpret_cast<uintptr_t>(c.lse) & 3u))
        return RA_ERR_ALIGN;
    if (opt.variant < RA_VARIANT_AUTO || opt.variant > RA_VARIANT_PER_STEP) return RA_ERR_INVALID_ARG;
    DeviceInfo dev;
    if ((rc = device_info(&dev)) != RA_OK) return rc;
    Kernel kernel;
    if ((rc = select_kernel(c, opt.kernel, dev, &kernel)) != RA_OK) return rc;

    const Layout L = make_layout(c.S, c.n_ring, c.layout);
    const bool per_step = (opt.variant == RA_VARIANT_PER_STEP);
    const Workspace w = carve(c.B, c.H, L, c.D, c.causal, c.dtype, per_step, kernel);
    uint8_t* ws = static_cast<uint8_t*>(opt.workspace);
    bool own_ws = false;
    if (ws) {
        if (opt.workspace_bytes < w.total) return RA_ERR_NO_WORKSPACE;
        if (reinterpret_cast<uintptr_t>(ws) % kAlign) return RA_ERR_ALIGN;
    } else {
        cudaError_t e = cudaMallocAsync(reinterpret_cast<void**>(&ws), w.total, c.stream);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync(workspace)");
        own_ws = true;
    }
    auto finish = [&](int status) {
        if (own_ws) {
            cudaError_t e = cudaFreeAsync(ws, c.stream);
            if (e != cudaSuccess && status == RA_OK) status = cuda_fail(e, "cudaFreeAsync(workspace)");
        }
        return status;
    };
    cudaError_t e;
    cudaEvent_t ev0 = static_cast<cudaEvent_t>(opt.attn_events[0]);
    cudaEvent_t ev1 = static_cast<cudaEvent_t>(opt.attn_events[1]);

    ra::AttnArgs args{};
    args.L = L;
    args.B = c.B;
    args.H = c.H;
    args.D = c.D;
    args.causal = c.causal ? 1 : 0;
    args.dtype = c.dtype;
    args.scale = (float)(1.0 / std::sqrt((double)c.D));

    // ---- inputs in the order the kernel reads them
    const void *q = c.q, *k = c.k, *v = c.v;
    ra::TcLaunch tc{};
    std::vector<int> step_item_offset;
    if (kernel == kTC) {
        if (w.permute) {
            const void* src[3] = {c.q, c.k, c.v};
            void* dst[3] = {ws + w.qp, ws + w.kp, ws + w.vp};
            if ((e = ra::launch_permute(src, dst, 3, c.B, L, c.H, c.D, 2, false, c.stream)) != cudaSuccess)
                return finish(cuda_fail(e, "permute launch"));
            q = dst[0];
            k = dst[1];
            v = dst[2];
        }
        const bool striped_natural = (L.kind == RA_LAYOUT_STRIPED);
        if ((rc = encode_qkv_map(&tc.tm_q, q, c.B, L, c.H, c.D, striped_natural)) != RA_OK) return finish(rc);
        if ((rc = encode_qkv_map(&tc.tm_k, k, c.B, L, c.H, c.D, striped_natural)) != RA_OK) return finish(rc);
        if ((rc = encode_qkv_map(&tc.tm_v, v, c.B, L, c.H, c.D, striped_natural)) != RA_OK) return finish(rc);
        // upload the work list(s) from the cached pinned copy
        const FlatList* fl = nullptr;
        if ((rc = flat_items(c.B, c.H, L, c.D, args.causal, w.per_step, &fl)) != RA_OK) return finish(rc);
        step_item_offset = fl->offsets;
        if (fl->count > 0 &&
            (e = cudaMemcpyAsync(ws + w.items, fl->data, fl->count * sizeof(int4),
                                 cudaMemcpyHostToDevice, c.stream)) != cudaSuccess)
            return finish(cuda_fail(e, "work list upload"));
        if ((e = cudaMemsetAsync(ws + w.counters, 0, w.n_counters * sizeof(int), c.stream)) != cudaSuccess)
            return finish(cuda_fail(e, "work counter reset"));
        tc.timeout_ns = opt.timeout_ns ? opt.timeout_ns : 2000000000ull;
        tc.debug = opt.debug;
        tc.status = dev.status;
    }

    auto attention = [&](int s_begin, int s_end, int out_mode, void* out, float* lse) -> cudaError_t {
        ra::AttnArgs a = args;
        a.s_begin = s_begin;
        a.s_end = s_end;
        a.out_mode = out_mode;
        a.out = out;
        a.lse = lse;
        if (kernel == kTC) {
            ra::TcLaunch t = tc;
            const int list = w.per_step ? s_begin : 0;
            t.items = reinterpret_cast<const int4*>(ws + w.items) + step_item_offset[list];
            t.n_items = step_item_offset[list + 1] - step_item_offset[list];
            t.grid = std::max(1, std::min(t.n_items, dev.sms));
            t.counter = reinterpret_cast<int*>(ws + w.counters) + list;
            return ra::launch_attn_tc(a, t, c.stream);
        }
        return ra::launch_attn_simt(q, k, v, a, c.stream);
    };

    if (ev0 && (e = cudaEventRecord(ev0, c.stream)) != cudaSuccess) return finish(cuda_fail(e, "cudaEventRecord"));
    if (!w.per_step) {
        if ((e = attention(0, (int)L.N, ra::kOutFinal, c.out, c.lse)) != cudaSuccess)
            return finish(cuda_fail(e, "attention launch"));
    } else {
        float* O_run = reinterpret_cast<float*>(ws + w.O_run);
        float* lse_run = reinterpret_cast<float*>(ws + w.lse_run);
        float* O_step = reinterpret_cast<float*>(ws + w.O_step);
        float* lse_step = reinterpret_cast<float*>(ws + w.lse_step);
        const int64_t rows = c.B * c.S * c.H;
        if ((e = attention(0, 1, ra::kOutPartial, O_run, lse_run)) != cudaSuccess)
            return finish(cuda_fail(e, "attention launch (step 0)"));
        for (int s = 1; s < (int)L.N; ++s) {
            if ((e = attention(s, s + 1, ra::kOutPartial, O_step, lse_step)) != cudaSuccess)
                return finish(cuda_fail(e, "attention launch (step)"));
            if (s + 1 < (int)L.N)
                e = ra::launch_merge_inplace(O_run, lse_run, O_step, lse_step, rows, c.D, c.stream);
            else
                e = ra::launch_merge_final(O_run, lse_run, O_step, lse_step, c.out, c.lse, c.dtype, c.B,
                                           L, c.H, c.D, c.stream);
            if (e != cudaSuccess) return finish(cuda_fail(e, "merge launch"));
        }
    }
    if (ev1 && (e = cudaEventRecord(ev1, c.stream)) != cudaSuccess) return finish(cuda_fail(e, "cudaEventRecord"));
    return finish(RA_OK);
}

ra_options default_options() {
    ra_options o;
    std::memset(&o, 0, sizeof o);
    return o;
}

}  // namespace

// Helpers shared with other entry points of the library (declared in ra_internal.cuh).
namespace ra {
int host_check_shape(int64_t B, int64_t H, int64_t S, int64_t D, int n_ring, int layout, int dtype) {
    return check_shape(B, H, S, D, n_ring, layout, dtype);
}
int host_device_facts(int* sms, bool* sm100, int** status) {
    DeviceInfo d;
    const int rc = device_info(&d);
    if (rc != RA_OK) return rc;
    *sms = d.sms;
    *sm100 = d.sm100;
    *status = d.status;
    return RA_OK;
}
int host_encode_qkv_map(CUtensorMap* map, const void* base, int64_t B, const Layout& L, int64_t H, int64_t D,
                        bool striped_natural) {
    return encode_qkv_map(map, base, B, L, H, D, striped_natural);
}
int host_cuda_fail(cudaError_t e, const char* what) { return cuda_fail(e, what); }
void host_set_error(const char* msg) { snprintf(g_last_error, sizeof g_last_error, "%s", msg); }
}  // namespace ra

extern "C" {

int ra_forward(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B,
               int64_t H, int64_t S, int64_t D, int n_ring, int causal, int layout, int dtype,
               void* stream) {
    return ra_forward_ex(q, k, v, out, lse, B, H, S, D, n_ring, causal, layout, dtype, stream, nullptr);
}

int ra_forward_ex(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B,
                  int64_t H, int64_t S, int64_t D, int n_ring, int causal, int layout, int dtype,
                  void* stream, const ra_options* opt) {
    const ra_options o = opt ? *opt : default_options();
    Call c{q, k, v, out, lse, B, H, S, D, n_ring, causal, layout, dtype, static_cast<cudaStream_t>(stream)};
    return run_forward(c, o);
}

int ra_workspace_size(int64_t B, int64_t H, int64_t S, int64_t D, int n_ring, int causal,
                      int layout, int dtype, int variant, int kernel, size_t* bytes) {
    if (!bytes) return RA_ERR_INVALID_ARG;
    int rc = check_shape(B, H, S, D, n_ring, layout, dtype);
    if (rc != RA_OK) return rc;
    if (variant < RA_VARIANT_AUTO || variant > RA_VARIANT_PER_STEP) return RA_ERR_INVALID_ARG;
    if (kernel < RA_KERNEL_AUTO || kernel > RA_KERNEL_SIMT) return RA_ERR_INVALID_ARG;
    // Host-only: the tensor-core layout is assumed whenever it could apply, which is never smaller.
    const bool tc = (kernel != RA_KERNEL_SIMT) && dtype == RA_DTYPE_BF16 && (D == 64 || D == 128);
    const Layout L = make_layout(S, n_ring, layout);
    *bytes = carve(B, H, L, D, causal ? 1 : 0, dtype, variant == RA_VARIANT_PER_STEP, tc ? kTC : kSIMT).total;
    return RA_OK;
}

int ra_permute(const void* x, void* y, int64_t B, int64_t S, int64_t H, int64_t D, int n_ring,
               int layout, int dtype, void* stream) {
    int rc = check_shape(B, H, S, D, n_ring, layout, dtype);
    if (rc != RA_OK) return rc;
    if (!x || !y) return RA_ERR_INVALID_ARG;
    const void* src[1] = {x};
    void* dst[1] = {y};
    cudaError_t e = ra::launch_permute(src, dst, 1, B, make_layout(S, n_ring, layout), H, D,
                                       dtype == RA_DTYPE_BF16 ? 2 : 4, false, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RA_OK : cuda_fail(e, "permute launch");
}

int ra_unpermute(const void* x, void* y, int64_t B, int64_t S, int64_t H, int64_t D, int n_ring,
                 int layout, int dtype, void* stream) {
    int rc = check_shape(B, H, S, D, n_ring, layout, dtype);
    if (rc != RA_OK) return rc;
    if (!x || !y) return RA_ERR_INVALID_ARG;
    const void* src[1] = {x};
    void* dst[1] = {y};
    cudaError_t e = ra::launch_permute(src, dst, 1, B, make_layout(S, n_ring, layout), H, D,
                                       dtype == RA_DTYPE_BF16 ? 2 : 4, true, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RA_OK : cuda_fail(e, "unpermute launch");
}

int ra_merge_partials(float* O_run, float* lse_run, const float* O_step, const float* lse_step,
                      int64_t rows, int64_t D, void* stream) {
    if (!O_run || !lse_run || !O_step || !lse_step || rows < 0 || D < 1) return RA_ERR_INVALID_ARG;
    if (D % 4 == 0 && (!aligned16(O_run) || !aligned16(O_step))) return RA_ERR_ALIGN;
    cudaError_t e = ra::launch_merge_inplace(O_run, lse_run, O_step, lse_step, rows, D,
                                             static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RA_OK : cuda_fail(e, "merge launch");
}

int ra_layout_positions(int64_t S, int n_ring, int layout, int64_t* pos) {
    if (!pos) return RA_ERR_INVALID_ARG;
    int rc = check_shape(1, 1, S, 1, n_ring, layout, RA_DTYPE_FP32);
    if (rc != RA_OK) return rc;
    const Layout L = make_layout(S, n_ring, layout);
    for (int64_t i = 0; i < L.N; ++i)
        for (int64_t a = 0; a < L.S_loc; ++a) pos[i * L.S_loc + a] = ra::global_position(L, i, a);
    return RA_OK;
}

int ra_plan_tiles(int64_t S, int n_ring, int layout, int causal, int tile, int8_t* cls) {
    if (!cls || tile < 1) return RA_ERR_INVALID_ARG;
    int rc = check_shape(1, 1, S, 1, n_ring, layout, RA_DTYPE_FP32);
    if (rc != RA_OK) return rc;
    const Layout L = make_layout(S, n_ring, layout);
    const int64_t nt = (L.S_loc + tile - 1) / tile;
    for (int64_t i = 0; i < L.N; ++i)
        for (int64_t s = 0; s < L.N; ++s) {
            const int64_t j = ra::ring_block(i, s, L.N);
            for (int64_t qt = 0; qt < nt; ++qt) {
                const int64_t a0 = qt * tile, a1 = std::min(a0 + tile, L.S_loc) - 1;
                const int64_t cmin = ra::visible_keys(L, causal, i, a0, j);
                const int64_t cmax = ra::visible_keys(L, causal, i, a1, j);
                for (int64_t kt = 0; kt < nt; ++kt) {
                    const int64_t k0 = kt * tile;
                    int8_t c;
                    if (k0 >= cmax) c = 0;
                    else if (k0 + tile <= cmin) c = 1;
                    else c = 2;
                    cls[((i * L.N + s) * nt + qt) * nt + kt] = c;
                }
            }
        }
    return RA_OK;
}

int ra_plan_items(int64_t B, int64_t H, int64_t S, int64_t D, int n_ring, int causal, int layout,
                  int32_t* items, int64_t cap, int64_t* n_items) {
    if (!n_items || (cap > 0 && !items)) return RA_ERR_INVALID_ARG;
    int rc = check_shape(B, H, S, D, n_ring, layout, RA_DTYPE_FP32);
    if (rc != RA_OK) return rc;
    const Layout L = make_layout(S, n_ring, layout);
    const auto& list = plan_items(B, H, L, D, causal ? 1 : 0, 0, n_ring);
    *n_items = (int64_t)list.size();
    for (int64_t t = 0; t < std::min<int64_t>(cap, (int64_t)list.size()); ++t) {
        const PlanItem& x = list[(size_t)t];
        int32_t* d = items + 5 * t;
        d[0] = x.b;
        d[1] = x.h;
        d[2] = x.i;
        d[3] = x.p;
        d[4] = x.cost;
    }
    return RA_OK;
}

const char* ra_status_string(int status) {
    switch (status) {
        case RA_OK: return "ok";
        case RA_ERR_INVALID_ARG: return "invalid argument";
        case RA_ERR_SHAPE: return "unsupported shape (S % n_ring, zigzag S % 2 n_ring, or D)";
        case RA_ERR_ALIGN: return "pointer not aligned (16 bytes for tensors, 256 for workspace)";
        case RA_ERR_UNSUPPORTED: return "unsupported device or kernel for these arguments";
        case RA_ERR_NO_WORKSPACE: return "workspace smaller than ra_workspace_size";
        case RA_ERR_CUDA: return "CUDA call failed";
        case RA_ERR_DEVICE_TIMEOUT: return "a bounded in-kernel wait expired";
        default: return "unknown status";
    }
}

const char* ra_last_error_string(void) { return g_last_error; }

int ra_get_device_status(void) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_ra_device_status, sizeof v);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol(status)");
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_ra_device_status, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyToSymbol(status)");
    return v;
}

}  // extern "C"
