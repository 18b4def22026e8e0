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
#include <memory>
#include <mutex>
#include <tuple>
#include <utility>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "ra.h"
#include "ra_internal.cuh"

__device__ int g_ra_device_status = 0;

namespace {

using ra::Layout;

thread_local char g_last_error[512] = "";

// Close the NVTX range an entry point opened and pass its status through (early returns).
int nvtx_pop(int status) {
    nvtxRangePop();
    return status;
}

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
    int shard;  // -1: every shard; otherwise the items of this query shard only
    bool operator<(const PlanKey& o) const {
        return std::tie(B, H, S, n_ring, causal, layout, s_begin, s_end, D, shard) <
               std::tie(o.B, o.H, o.S, o.n_ring, o.causal, o.layout, o.s_begin, o.s_end, o.D, o.shard);
    }
};

// A map from problem shape to a planned object, bounded to kCacheEntries entries: inserting
// beyond that drops the least recently used one.  Entries are shared_ptr, so a caller still
// holding a dropped entry keeps it alive until it lets go.  The cache objects themselves are
// created with new and never destroyed, so no CUDA call runs during static destruction.
constexpr size_t kCacheEntries = 64;

template <class K, class V>
class LruCache {
  public:
    std::shared_ptr<V> get(const K& key) {
        std::lock_guard<std::mutex> lock(mu_);
        auto it = map_.find(key);
        if (it == map_.end()) return nullptr;
        it->second.first = ++tick_;
        return it->second.second;
    }
    // Insert unless another thread got there first; returns the entry that is cached.
    std::shared_ptr<V> put(const K& key, std::shared_ptr<V> value) {
        std::shared_ptr<V> dropped;  // released after the lock, so its destructor runs unlocked
        std::lock_guard<std::mutex> lock(mu_);
        auto it = map_.find(key);
        if (it != map_.end()) return it->second.second;
        map_.emplace(key, std::make_pair(++tick_, value));
        if (map_.size() > kCacheEntries) {
            auto oldest = map_.begin();
            for (auto jt = map_.begin(); jt != map_.end(); ++jt)
                if (jt->second.first < oldest->second.first) oldest = jt;
            dropped = std::move(oldest->second.second);
            map_.erase(oldest);
        }
        return value;
    }
    size_t size() {
        std::lock_guard<std::mutex> lock(mu_);
        return map_.size();
    }

  private:
    std::mutex mu_;
    std::map<K, std::pair<uint64_t, std::shared_ptr<V>>> map_;
    uint64_t tick_ = 0;
};

struct PlanItem {
    int32_t b, h, i, p, cost;
};

using ItemList = std::vector<PlanItem>;

LruCache<PlanKey, const ItemList>& plan_cache() {
    static auto* cache = new LruCache<PlanKey, const ItemList>();
    return *cache;
}

// Work list of the tensor-core kernel for ring steps [s_begin, s_end): one item per
// (b, h, shard i, pair of 128-row query tiles), cost = live (query tile, key tile) pairs; with
// shard >= 0 only the items of that query shard (a ring step on one device's local buffers).
// Order: (b, h) major so that CTAs running at the same time share one head's keys and values in
// L2; inside a head, heaviest first (LPT) so the short items fill the tail -- or, when one head's
// K/V exceeds L2 (plan_groups_by_shard), shard groups heaviest first and LPT inside a group.
std::shared_ptr<const ItemList> plan_items(int64_t B, int64_t H, const Layout& L, int64_t D_for_plan,
                                           int causal, int s_begin, int s_end, int shard = -1) {
    const PlanKey key{B, H, L.S, (int)L.N, causal, L.kind, s_begin, s_end, D_for_plan, shard};
    if (auto hit = plan_cache().get(key)) return hit;
    const int64_t pairs = (L.S_loc + kTcPairRows - 1) / kTcPairRows;
    std::vector<PlanItem> head;
    head.reserve((size_t)(L.N * pairs));
    for (int64_t i = 0; i < L.N; ++i)
        for (int64_t p = 0; p < pairs; ++p) {
            if (shard >= 0 && i != shard) continue;
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
    auto all = std::make_shared<ItemList>();
    all->reserve(head.size() * (size_t)(B * H));
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < H; ++h)
            for (PlanItem x : head) {
                x.b = (int32_t)b;
                x.h = (int32_t)h;
                all->push_back(x);
            }
    return plan_cache().put(key, std::move(all));
}

// All lists of one call flattened into pinned host memory, so that the upload is a true
// asynchronous copy.  offsets[s] .. offsets[s + 1] delimit the list of step s (per-step) or the
// single list (fused).  Pinned memory may only be freed once no copy from it is pending: every
// upload records an event on its stream, and the destructor (run when the bounded cache drops
// the entry and no call holds it any more) waits for those events first.  An upload recorded
// into a CUDA graph reads the buffer at every replay, for as long as the graph lives, which the
// library cannot see; such a buffer is never freed.
struct FlatList {
    int4* data = nullptr;
    size_t count = 0;
    std::vector<int> offsets;
    std::mutex mu;
    std::vector<std::pair<cudaStream_t, cudaEvent_t>> uploads;  // latest upload per stream
    bool in_graph = false;

    FlatList() = default;
    FlatList(const FlatList&) = delete;
    FlatList& operator=(const FlatList&) = delete;
    ~FlatList() {
        if (in_graph) return;  // a captured graph may still copy from data
        for (auto& u : uploads) {
            cudaEventSynchronize(u.second);
            cudaEventDestroy(u.second);
        }
        if (data) cudaFreeHost(data);
    }

    // Upload [first, first + n) items to dst on `stream`, and remember the copy.
    cudaError_t upload(void* dst, size_t first, size_t n, cudaStream_t stream) {
        cudaError_t e = cudaMemcpyAsync(dst, data + first, n * sizeof(int4), cudaMemcpyHostToDevice, stream);
        if (e != cudaSuccess) return e;
        cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
        if ((e = cudaStreamIsCapturing(stream, &cap)) != cudaSuccess) return e;
        std::lock_guard<std::mutex> lock(mu);
        if (cap != cudaStreamCaptureStatusNone) {
            in_graph = true;
            return cudaSuccess;
        }
        cudaEvent_t ev = nullptr;
        for (auto& u : uploads)
            if (u.first == stream) ev = u.second;
        if (!ev) {
            if ((e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming)) != cudaSuccess) return e;
            uploads.emplace_back(stream, ev);
        }
        return cudaEventRecord(ev, stream);
    }
};

struct FlatKey {
    PlanKey plan;
    int chunk;  // ring steps per attention launch (N: one fused launch)
    int device;
    bool operator<(const FlatKey& o) const {
        return std::tie(plan, chunk, device) < std::tie(o.plan, o.chunk, o.device);
    }
};

LruCache<FlatKey, FlatList>& flat_cache() {
    static auto* cache = new LruCache<FlatKey, FlatList>();
    return *cache;
}

// shard >= 0: the list of that query shard for the single step `step` (a ring step on local
// buffers); otherwise every shard, one list per launch of `chunk` ring steps (chunk = N: the single
// list of the fused launch; the last launch takes the steps that remain).
int flat_items(int64_t B, int64_t H, const Layout& L, int64_t D, int causal, int chunk,
               std::shared_ptr<FlatList>* out, int shard = -1, int step = 0) {
    int device = 0;
    cudaError_t e = cudaGetDevice(&device);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    const PlanKey pk = shard >= 0 ? PlanKey{B, H, L.S, (int)L.N, causal, L.kind, step, step + 1, D, shard}
                                  : PlanKey{B, H, L.S, (int)L.N, causal, L.kind, 0, (int)L.N, D, -1};
    if (shard >= 0) chunk = 1;
    const FlatKey key{pk, chunk, device};
    if ((*out = flat_cache().get(key))) return RA_OK;
    auto f = std::make_shared<FlatList>();
    std::vector<int4> flat;
    const int n_lists = shard >= 0 ? 1 : (int)((L.N + chunk - 1) / chunk);
    for (int c = 0; c < n_lists; ++c) {
        f->offsets.push_back((int)flat.size());
        const int s0 = c * chunk, s1 = std::min<int>((int)L.N, s0 + chunk);
        std::shared_ptr<const ItemList> items = shard >= 0 ? plan_items(B, H, L, D, causal, step, step + 1, shard)
                                                           : plan_items(B, H, L, D, causal, s0, s1);
        for (const PlanItem& x : *items) flat.push_back(make_int4(x.b, x.h, x.i, x.p));
    }
    f->offsets.push_back((int)flat.size());
    f->count = flat.size();
    if (f->count) {
        e = cudaHostAlloc(reinterpret_cast<void**>(&f->data), f->count * sizeof(int4), cudaHostAllocPortable);
        if (e != cudaSuccess) return cuda_fail(e, "cudaHostAlloc(work list)");
        std::memcpy(f->data, flat.data(), f->count * sizeof(int4));
    }
    *out = flat_cache().put(key, std::move(f));
    return RA_OK;
}

// ------------------------------------------------------------------ workspace
enum Kernel { kTC, kSIMT };

struct Workspace {
    size_t counters = 0, n_counters = 0;  // one work counter per attention launch (zeroed per call)
    size_t items = 0, n_items_total = 0;
    size_t qp = 0, kp = 0, vp = 0;  // permuted q, k, v
    size_t O_run = 0, lse_run = 0, O_step = 0, lse_step = 0;
    size_t kmax = 0;  // largest query and key norm per (b, h), the score bound of the frozen max
    bool permute = false, per_step = false;
    int chunk = 1, n_launches = 1;  // ring steps per attention launch, and the launches
    size_t total = 0;
};

// Ring steps per attention launch.  FUSED: all N in one launch.  PER_STEP: `steps_per_launch`
// (0 means 1), at most N.  AUTO: fused while one head's keys and values fit comfortably in L2;
// beyond that, launches of as many steps as keep a launch's keys and values per head within the
// same budget, evened out over the N steps.  The reason: a fused work item walks every key/value
// block of its head, and when those do not fit in L2 the CTAs running together (each on its own
// item, at its own pace) spread over more blocks than L2 holds; a launch that covers a few steps
// keeps the blocks its CTAs read together in L2, for the price of one merge of partial results
// per extra launch.
constexpr int64_t kFusedKvBudget = int64_t(96) << 20;

int launch_chunk(const Layout& L, int64_t D, int dtype, int variant, int requested) {
    const int N = (int)L.N;
    if (variant == RA_VARIANT_FUSED) return N;
    if (variant == RA_VARIANT_PER_STEP) return std::min(N, std::max(1, requested));
    const int64_t esize = dtype == RA_DTYPE_BF16 ? 2 : 4;
    const int64_t block_kv = 2 * L.S_loc * D * esize;  // one key/value block of one head
    if (block_kv * N <= kFusedKvBudget) return N;
    const int64_t fit = std::max<int64_t>(1, kFusedKvBudget / std::max<int64_t>(1, block_kv));
    const int64_t launches = (N + fit - 1) / fit;
    return (int)((N + launches - 1) / launches);
}

Workspace carve(int64_t B, int64_t H, const Layout& L, int64_t D, int causal, int dtype,
                int chunk, Kernel kernel) {
    Workspace w;
    size_t off = 0;
    const size_t esize = dtype == RA_DTYPE_BF16 ? 2 : 4;
    const size_t elems = (size_t)(B * L.S * H * D);
    w.chunk = std::max(1, std::min<int>(chunk, (int)L.N));
    w.n_launches = (int)((L.N + w.chunk - 1) / w.chunk);
    w.per_step = w.n_launches > 1;
    if (kernel == kTC) {
        for (int c = 0; c < w.n_launches; ++c) {
            const int s0 = c * w.chunk, s1 = std::min<int>((int)L.N, s0 + w.chunk);
            w.n_items_total += plan_items(B, H, L, D, causal, s0, s1)->size();
        }
        w.counters = off;
        w.n_counters = (size_t)w.n_launches;
        off = align_up(off + w.n_counters * sizeof(int));
        w.items = off;
        off = align_up(off + w.n_items_total * sizeof(int4));
        w.kmax = off;
        off = align_up(off + (size_t)(2 * B * H) * sizeof(float));
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
    if (opt.steps_per_launch < 0) return RA_ERR_INVALID_ARG;
    DeviceInfo dev;
    if ((rc = device_info(&dev)) != RA_OK) return rc;
    Kernel kernel;
    if ((rc = select_kernel(c, opt.kernel, dev, &kernel)) != RA_OK) return rc;

    const Layout L = make_layout(c.S, c.n_ring, c.layout);
    const int chunk = launch_chunk(L, c.D, c.dtype, opt.variant, opt.steps_per_launch);
    const Workspace w = carve(c.B, c.H, L, c.D, c.causal, c.dtype, chunk, kernel);
    uint8_t* ws = static_cast<uint8_t*>(opt.workspace);
    bool own_ws = false;
    if (ws) {
        if (opt.workspace_bytes < w.total) return RA_ERR_NO_WORKSPACE;
        if (reinterpret_cast<uintptr_t>(ws) % kAlign) return RA_ERR_ALIGN;
    } else {
        cudaError_t e = ra::scratch_alloc(reinterpret_cast<void**>(&ws), w.total, c.stream);
        if (e != cudaSuccess) return cuda_fail(e, "stream-ordered allocation (workspace)");
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
            nvtxRangePushA("ra_forward permute");
            e = ra::launch_permute(src, dst, 3, c.B, L, c.H, c.D, 2, false, c.stream);
            nvtxRangePop();
            if (e != cudaSuccess) return finish(cuda_fail(e, "permute launch"));
            q = dst[0];
            k = dst[1];
            v = dst[2];
        }
        const bool striped_natural = (L.kind == RA_LAYOUT_STRIPED);
        if ((rc = encode_qkv_map(&tc.tm_q, q, c.B, L, c.H, c.D, striped_natural)) != RA_OK) return finish(rc);
        if ((rc = encode_qkv_map(&tc.tm_k, k, c.B, L, c.H, c.D, striped_natural)) != RA_OK) return finish(rc);
        if ((rc = encode_qkv_map(&tc.tm_v, v, c.B, L, c.H, c.D, striped_natural)) != RA_OK) return finish(rc);
        // upload the work list(s) from the cached pinned copy
        std::shared_ptr<FlatList> fl;
        if ((rc = flat_items(c.B, c.H, L, c.D, args.causal, w.chunk, &fl)) != RA_OK) return finish(rc);
        step_item_offset = fl->offsets;
        if (fl->count > 0 && (e = fl->upload(ws + w.items, 0, fl->count, c.stream)) != cudaSuccess)
            return finish(cuda_fail(e, "work list upload"));
        if ((e = cudaMemsetAsync(ws + w.counters, 0, w.n_counters * sizeof(int), c.stream)) != cudaSuccess)
            return finish(cuda_fail(e, "work counter reset"));
        if (ra::key_norm_max_applies(c.B, c.H, c.D) &&
            ra::frozen_max_pays((int64_t)w.chunk * L.S_loc, opt.debug == RA_DEBUG_FROZEN_MAX)) {
            // the score bound of every query row (frozen max)
            float* nmax = reinterpret_cast<float*>(ws + w.kmax);
            nvtxRangePushA("ra_forward query and key norms");
            e = ra::launch_norm_max(c.q, c.k, nmax, c.B, c.S, c.H, c.D, dev.sms, c.stream);
            nvtxRangePop();
            if (e != cudaSuccess) return finish(cuda_fail(e, "norm launch"));
            args.qmax = nmax;
            args.kmax = nmax + c.B * c.H;
        }
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
            const int list = s_begin / w.chunk;
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
        // the unpermute is fused into the attention kernel's epilogue (natural-order stores)
        nvtxRangePushA("ra_forward attention (fused ring, unpermute in the epilogue)");
        e = attention(0, (int)L.N, ra::kOutFinal, c.out, c.lse);
        nvtxRangePop();
        if (e != cudaSuccess) return finish(cuda_fail(e, "attention launch"));
    } else {
        float* O_run = reinterpret_cast<float*>(ws + w.O_run);
        float* lse_run = reinterpret_cast<float*>(ws + w.lse_run);
        float* O_step = reinterpret_cast<float*>(ws + w.O_step);
        float* lse_step = reinterpret_cast<float*>(ws + w.lse_step);
        const int64_t rows = c.B * c.S * c.H;
        // launch k covers ring steps [k * chunk, min(N, (k + 1) * chunk)); its partial result is
        // merged into the running one, the last merge writing out and lse in natural order
        nvtxRangePushA("ra_forward attention (first ring steps)");
        e = attention(0, std::min<int>(w.chunk, (int)L.N), ra::kOutPartial, O_run, lse_run);
        nvtxRangePop();
        if (e != cudaSuccess) return finish(cuda_fail(e, "attention launch (step 0)"));
        for (int s = w.chunk; s < (int)L.N; s += w.chunk) {
            const int s_end = std::min<int>((int)L.N, s + w.chunk);
            nvtxRangePushA("ra_forward attention (ring steps)");
            e = attention(s, s_end, ra::kOutPartial, O_step, lse_step);
            nvtxRangePop();
            if (e != cudaSuccess) return finish(cuda_fail(e, "attention launch (step)"));
            // the last merge also unpermutes: it writes out and lse in natural order
            nvtxRangePushA(s_end < (int)L.N ? "ra_forward merge" : "ra_forward merge + unpermute");
            if (s_end < (int)L.N)
                e = ra::launch_merge_inplace(O_run, lse_run, O_step, lse_step, rows, c.D, c.stream);
            else
                e = ra::launch_merge_final(O_run, lse_run, O_step, lse_step, c.out, c.lse, c.dtype, c.B,
                                           L, c.H, c.D, c.stream);
            nvtxRangePop();
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
    // PER_STEP is sized for one step per launch, which covers any steps_per_launch (fewer
    // launches need fewer counters and lists); AUTO is sized for the chunk it picks.
    const bool tc = (kernel != RA_KERNEL_SIMT) && dtype == RA_DTYPE_BF16 && (D == 64 || D == 128);
    const Layout L = make_layout(S, n_ring, layout);
    const int chunk = launch_chunk(L, D, dtype, variant, 1);
    *bytes = carve(B, H, L, D, causal ? 1 : 0, dtype, chunk, tc ? kTC : kSIMT).total;
    return RA_OK;
}

int ra_steps_per_launch(int64_t S, int64_t D, int n_ring, int layout, int dtype, int variant, int steps_per_launch,
                        int* chunk) {
    if (!chunk) return RA_ERR_INVALID_ARG;
    const int rc = check_shape(1, 1, S, D, n_ring, layout, dtype);
    if (rc != RA_OK) return rc;
    if (variant < RA_VARIANT_AUTO || variant > RA_VARIANT_PER_STEP || steps_per_launch < 0) return RA_ERR_INVALID_ARG;
    *chunk = launch_chunk(make_layout(S, n_ring, layout), D, dtype, variant, steps_per_launch);
    return RA_OK;
}

int ra_permute(const void* x, void* y, int64_t B, int64_t S, int64_t H, int64_t D, int n_ring,
               int layout, int dtype, void* stream) {
    int rc = check_shape(B, H, S, D, n_ring, layout, dtype);
    if (rc != RA_OK) return rc;
    if (!x || !y) return RA_ERR_INVALID_ARG;
    const void* src[1] = {x};
    void* dst[1] = {y};
    nvtxRangePushA("ra_permute");
    cudaError_t e = ra::launch_permute(src, dst, 1, B, make_layout(S, n_ring, layout), H, D,
                                       dtype == RA_DTYPE_BF16 ? 2 : 4, false, static_cast<cudaStream_t>(stream));
    nvtxRangePop();
    return e == cudaSuccess ? RA_OK : cuda_fail(e, "permute launch");
}

int ra_unpermute(const void* x, void* y, int64_t B, int64_t S, int64_t H, int64_t D, int n_ring,
                 int layout, int dtype, void* stream) {
    int rc = check_shape(B, H, S, D, n_ring, layout, dtype);
    if (rc != RA_OK) return rc;
    if (!x || !y) return RA_ERR_INVALID_ARG;
    const void* src[1] = {x};
    void* dst[1] = {y};
    nvtxRangePushA("ra_unpermute");
    cudaError_t e = ra::launch_permute(src, dst, 1, B, make_layout(S, n_ring, layout), H, D,
                                       dtype == RA_DTYPE_BF16 ? 2 : 4, true, static_cast<cudaStream_t>(stream));
    nvtxRangePop();
    return e == cudaSuccess ? RA_OK : cuda_fail(e, "unpermute launch");
}

int ra_merge_partials(float* O_run, float* lse_run, const float* O_step, const float* lse_step,
                      int64_t rows, int64_t D, void* stream) {
    if (!O_run || !lse_run || !O_step || !lse_step || rows < 0 || D < 1) return RA_ERR_INVALID_ARG;
    if (D % 4 == 0 && (!aligned16(O_run) || !aligned16(O_step))) return RA_ERR_ALIGN;
    nvtxRangePushA("ra_merge_partials");
    cudaError_t e = ra::launch_merge_inplace(O_run, lse_run, O_step, lse_step, rows, D,
                                             static_cast<cudaStream_t>(stream));
    nvtxRangePop();
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
    const auto list = plan_items(B, H, L, D, causal ? 1 : 0, 0, n_ring);
    *n_items = (int64_t)list->size();
    for (int64_t t = 0; t < std::min<int64_t>(cap, (int64_t)list->size()); ++t) {
        const PlanItem& x = (*list)[(size_t)t];
        int32_t* d = items + 5 * t;
        d[0] = x.b;
        d[1] = x.h;
        d[2] = x.i;
        d[3] = x.p;
        d[4] = x.cost;
    }
    return RA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ one ring step on local buffers
namespace {

struct RingWorkspace {
    size_t counter = 0, items = 0, kmax = 0, O_s = 0, lse_s = 0, total = 0;
    size_t n_items = 0;
};

RingWorkspace ring_carve(int64_t B, int64_t H, const Layout& L, int64_t D, int causal, int shard, int step,
                         bool tc) {
    RingWorkspace w;
    size_t off = 0;
    if (tc) {
        w.n_items = plan_items(B, H, L, D, causal, step, step + 1, shard)->size();
        w.counter = off;
        off = align_up(off + sizeof(int));
        w.items = off;
        off = align_up(off + w.n_items * sizeof(int4));
        w.kmax = off;
        off = align_up(off + (size_t)(2 * B * H) * sizeof(float));
    }
    const size_t rows = (size_t)(B * L.S_loc * H);
    w.O_s = off;
    off = align_up(off + rows * (size_t)D * 4);
    w.lse_s = off;
    off = align_up(off + rows * 4);
    w.total = std::max<size_t>(off, kAlign);
    return w;
}

bool ring_kernel_tc(const DeviceInfo& dev, int dtype, int64_t D) {
    return dev.sm100 && dtype == RA_DTYPE_BF16 && (D == 64 || D == 128);
}

int ring_check(int64_t B, int64_t H, int64_t S, int64_t D, int n_ring, int layout, int dtype, int shard, int step) {
    const int rc = check_shape(B, H, S, D, n_ring, layout, dtype);
    if (rc != RA_OK) return rc;
    if (shard < 0 || shard >= n_ring || step < 0 || step >= n_ring) return RA_ERR_INVALID_ARG;
    return RA_OK;
}

}  // namespace

extern "C" {

int ra_ring_step_workspace_size(int64_t B, int64_t H, int64_t S, int64_t D, int n_ring, int causal, int layout,
                                int dtype, size_t* bytes) {
    if (!bytes) return RA_ERR_INVALID_ARG;
    const int rc = ring_check(B, H, S, D, n_ring, layout, dtype, 0, 0);
    if (rc != RA_OK) return rc;
    // host only: the tensor-core carve-up (a superset) whenever it could apply; the largest
    // work list over every (shard, step) is one item per query-tile pair of each (b, h)
    const bool tc = dtype == RA_DTYPE_BF16 && (D == 64 || D == 128);
    const Layout L = make_layout(S, n_ring, layout);
    const int64_t pairs = (L.S_loc + kTcPairRows - 1) / kTcPairRows;
    size_t off = 0;
    if (tc) off = align_up(sizeof(int)) + align_up((size_t)(B * H * pairs) * sizeof(int4)) +
                  align_up((size_t)(2 * B * H) * sizeof(float));
    const size_t rows = (size_t)(B * L.S_loc * H);
    off = align_up(off + rows * (size_t)D * 4);
    off = align_up(off + rows * 4);
    *bytes = std::max<size_t>(off, kAlign);
    (void)causal;
    return RA_OK;
}

int ra_ring_step(const void* q_i, const void* k_j, const void* v_j, float* O_acc, float* lse_acc, int64_t B,
                 int64_t H, int64_t S, int64_t D, int n_ring, int causal, int layout, int dtype, int shard,
                 int step, int sms_reserved, void* workspace, size_t workspace_bytes, void* stream_handle) {
    int rc = ring_check(B, H, S, D, n_ring, layout, dtype, shard, step);
    if (rc != RA_OK) return rc;
    if (sms_reserved < 0) return RA_ERR_INVALID_ARG;
    if (!q_i || !k_j || !v_j || !O_acc || !lse_acc) return RA_ERR_INVALID_ARG;
    const size_t esize = dtype == RA_DTYPE_BF16 ? 2 : 4;
    auto aligned = [](const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; };
    if (!aligned(O_acc, 16) || !aligned(lse_acc, 4)) return RA_ERR_ALIGN;
    DeviceInfo dev;
    if ((rc = device_info(&dev)) != RA_OK) return rc;
    if (sms_reserved >= dev.sms) return RA_ERR_INVALID_ARG;
    const bool tc = ring_kernel_tc(dev, dtype, D);
    const size_t qkv_align = tc ? 16 : esize;
    if (!aligned(q_i, qkv_align) || !aligned(k_j, qkv_align) || !aligned(v_j, qkv_align)) return RA_ERR_ALIGN;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_handle);
    const Layout L = make_layout(S, n_ring, layout);
    const int j = (int)ra::ring_block(shard, step, n_ring);
    // a later step whose whole block lies in the future of every query of the shard adds nothing
    if (step > 0 && ra::visible_keys(L, causal ? 1 : 0, shard, L.S_loc - 1, j) == 0) return RA_OK;

    const RingWorkspace w = ring_carve(B, H, L, D, causal ? 1 : 0, shard, step, tc);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    bool own_ws = false;
    if (ws) {
        if (workspace_bytes < w.total) return RA_ERR_NO_WORKSPACE;
        if (reinterpret_cast<uintptr_t>(ws) % kAlign) return RA_ERR_ALIGN;
    } else {
        cudaError_t e = ra::scratch_alloc(reinterpret_cast<void**>(&ws), w.total, stream);
        if (e != cudaSuccess) return cuda_fail(e, "stream-ordered allocation (ring step workspace)");
        own_ws = true;
    }
    auto finish = [&](int status) {
        if (own_ws) {
            cudaError_t e = cudaFreeAsync(ws, stream);
            if (e != cudaSuccess && status == RA_OK) status = cuda_fail(e, "cudaFreeAsync(ring step workspace)");
        }
        return status;
    };

    ra::AttnArgs a{};
    a.L = L;
    a.B = B;
    a.H = H;
    a.D = D;
    a.causal = causal ? 1 : 0;
    a.dtype = dtype;
    a.s_begin = step;
    a.s_end = step + 1;
    a.out_mode = ra::kOutPartial;
    a.local = 1;
    a.q_shard = shard;
    a.scale = (float)(1.0 / std::sqrt((double)D));
    // step 0 starts the running result; later steps write a partial that is merged into it
    float* O_s = step == 0 ? O_acc : reinterpret_cast<float*>(ws + w.O_s);
    float* lse_s = step == 0 ? lse_acc : reinterpret_cast<float*>(ws + w.lse_s);
    a.out = O_s;
    a.lse = lse_s;
    cudaError_t e;
    nvtxRangePushA("ra_ring_step attention");
    if (tc) {
        ra::TcLaunch t{};
        const Layout Lloc{L.S_loc, 1, L.S_loc, RA_LAYOUT_CONTIGUOUS};  // one shard per buffer
        if ((rc = encode_qkv_map(&t.tm_q, q_i, B, Lloc, H, D, false)) != RA_OK) return nvtx_pop(finish(rc));
        if ((rc = encode_qkv_map(&t.tm_k, k_j, B, Lloc, H, D, false)) != RA_OK) return nvtx_pop(finish(rc));
        if ((rc = encode_qkv_map(&t.tm_v, v_j, B, Lloc, H, D, false)) != RA_OK) return nvtx_pop(finish(rc));
        std::shared_ptr<FlatList> fl;
        if ((rc = flat_items(B, H, L, D, a.causal, false, &fl, shard, step)) != RA_OK) return nvtx_pop(finish(rc));
        if (fl->count > 0 && (e = fl->upload(ws + w.items, 0, fl->count, stream)) != cudaSuccess)
            return nvtx_pop(finish(cuda_fail(e, "work list upload")));
        if ((e = cudaMemsetAsync(ws + w.counter, 0, sizeof(int), stream)) != cudaSuccess)
            return nvtx_pop(finish(cuda_fail(e, "work counter reset")));
        if (ra::key_norm_max_applies(B, H, D) && ra::frozen_max_pays(L.S_loc, false)) {
            // the score bound over query shard i and key block j
            float* nmax = reinterpret_cast<float*>(ws + w.kmax);
            if ((e = ra::launch_norm_max(q_i, k_j, nmax, B, L.S_loc, H, D, dev.sms, stream)) != cudaSuccess)
                return nvtx_pop(finish(cuda_fail(e, "norm launch")));
            a.qmax = nmax;
            a.kmax = nmax + B * H;
        }
        t.items = reinterpret_cast<const int4*>(ws + w.items);
        t.n_items = (int)fl->count;
        t.counter = reinterpret_cast<int*>(ws + w.counter);
        t.grid = std::max(1, std::min(t.n_items, dev.sms - sms_reserved));
        t.timeout_ns = 2000000000ull;
        t.status = dev.status;
        e = ra::launch_attn_tc(a, t, stream);
    } else {
        e = ra::launch_attn_simt(q_i, k_j, v_j, a, stream);
    }
    nvtxRangePop();
    if (e != cudaSuccess) return finish(cuda_fail(e, "ring step attention launch"));
    if (step > 0) {
        nvtxRangePushA("ra_ring_step merge");
        e = ra::launch_merge_inplace(O_acc, lse_acc, O_s, lse_s, B * L.S_loc * H, D, stream);
        nvtxRangePop();
        if (e != cudaSuccess) return finish(cuda_fail(e, "ring step merge launch"));
    }
    return finish(RA_OK);
}

int ra_ring_finalize(const float* O_acc, const float* lse_acc, void* out, float* lse, int64_t B, int64_t H,
                     int64_t S_loc, int64_t D, int dtype, void* stream) {
    if (!O_acc || !lse_acc || !out || !lse) return RA_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || S_loc < 1 || D < 1 || D > 256) return RA_ERR_INVALID_ARG;
    if (dtype != RA_DTYPE_FP32 && dtype != RA_DTYPE_BF16) return RA_ERR_INVALID_ARG;
    auto aligned = [](const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; };
    if (!aligned(O_acc, 16) || !aligned(out, 16) || !aligned(lse_acc, 4) || !aligned(lse, 4)) return RA_ERR_ALIGN;
    const Layout Lloc{S_loc, 1, S_loc, RA_LAYOUT_CONTIGUOUS};
    nvtxRangePushA("ra_ring_finalize");
    cudaError_t e = ra::launch_merge_final(O_acc, lse_acc, nullptr, nullptr, out, lse, dtype, B, Lloc, H, D,
                                           static_cast<cudaStream_t>(stream));
    nvtxRangePop();
    return e == cudaSuccess ? RA_OK : cuda_fail(e, "ring finalize launch");
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
