// noalloc.cu -- ra_forward_noalloc: the fused tensor-core forward pass without any allocation.
//
// Who needs this.  ra_forward needs scratch memory (the work list of the persistent kernel and,
// for the zigzag layout, shard-major copies of q, k and v) and, unless the caller
// hands it a workspace, allocates it stream-ordered.  Some callers cannot let a library
// allocate device memory at all: code recording a CUDA graph (an allocation inside stream capture
// either fails or becomes part of the graph), engines that own every byte of the GPU through
// their own allocator and budget, and latency-critical loops where an allocator call may stall.
// This entry point serves them: its scratch lives in one fixed array in device memory
// (RA_NOALLOC_SCRATCH_BYTES), part of the library's device code.  The array comes into being on a
// device when the library's code is loaded there -- at the first use of the library on that
// device under CUDA's default lazy module loading, at context creation otherwise -- and stays
// until the process exits.  The call itself allocates nothing.
//
// Rules of use.
//   * The first call on a device, with that device current, looks up the array's device address
//     (cudaGetSymbolAddress) and loads every kernel this entry point launches (both head-dim
//     instantiations of the attention kernel, the permute and key-norm kernels and the list builder), so that
//     no later call loads module code.  Make that first call before any stream capture.
//   * Every call on a device shares the one array and leaves its contents behind.  The one part
//     that must start at zero, the kernel's work counter, is cleared by each call on its stream
//     (cudaMemsetAsync, no allocation); everything else is rewritten before it is read.  Calls
//     whose GPU work overlaps (different streams, or concurrent host threads) race on the array.
//   * Problems whose scratch exceeds the array are rejected with RA_ERR_NO_WORKSPACE (message in
//     ra_last_error_string); nothing is enqueued then.
#include <cuda.h>
#include <cuda_runtime.h>

#include <map>
#include <mutex>

#include "ra.h"
#include "ra_internal.cuh"

namespace {

using ra::Layout;

constexpr size_t kScratchBytes = (size_t)RA_NOALLOC_SCRATCH_BYTES;
constexpr int kTileRows = 128;
constexpr int kPairRows = 256;
// The list builder keeps one cost per item of a head and one total per shard in shared memory;
// it is launched without an opt-in above the default 48 KB of dynamic shared memory, so
// (items per head + shards) * 4 bytes must stay within 48 KB.
constexpr size_t kBuilderSmemBytes = 48 * 1024;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

__global__ void build_work_list(int4* __restrict__ items, int64_t BH, int64_t H, Layout L, int causal,
                                int pairs, int by_shard);

// Device address of g_noalloc_scratch on the current device, looked up once per device; the same
// first call loads every kernel the entry point launches on this device.
int scratch_address(unsigned char** out) {
    static std::mutex mu;
    static std::map<int, unsigned char*> addr;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return ra::host_cuda_fail(e, "cudaGetDevice");
    std::lock_guard<std::mutex> lock(mu);
    auto it = addr.find(dev);
    if (it == addr.end()) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return ra::host_cuda_fail(e, "cudaGetSymbolAddress(noalloc scratch)");
        cudaFuncAttributes fa;
        if ((e = cudaFuncGetAttributes(&fa, build_work_list)) != cudaSuccess)
            return ra::host_cuda_fail(e, "loading the work-list builder");
        if ((e = ra::preload_attn_tc()) != cudaSuccess) return ra::host_cuda_fail(e, "loading the attention kernel");
        if ((e = ra::preload_permute()) != cudaSuccess) return ra::host_cuda_fail(e, "loading the permute kernel");
        if ((e = ra::preload_key_norm()) != cudaSuccess) return ra::host_cuda_fail(e, "loading the key norm kernel");
        it = addr.emplace(dev, static_cast<unsigned char*>(p)).first;
    }
    *out = it->second;
    return RA_OK;
}

// Live 128-key tiles of block j for the 128-row query tile starting at local row a0.
__device__ int live_tiles(const Layout& L, int causal, int64_t i, int64_t a0, int64_t j) {
    if (a0 >= L.S_loc) return 0;
    const int64_t last = (a0 + kTileRows - 1 < L.S_loc - 1) ? a0 + kTileRows - 1 : L.S_loc - 1;
    return (int)((ra::visible_keys(L, causal, i, last, j) + kTileRows - 1) / kTileRows);
}

// One CTA builds the persistent kernel's work list on the device -- the same list, in the same
// order, as the host planner uploads: per head the N * pairs items (shard i, query-tile pair p),
// heaviest first (stable, ties keep (i, p) order), or with `by_shard` grouped by shard (groups
// heaviest first, heaviest first inside), repeated for every (b, h) in head-major order.
__global__ void build_work_list(int4* __restrict__ items, int64_t BH, int64_t H, Layout L, int causal,
                                int pairs, int by_shard) {
    extern __shared__ int smem_i[];
    int* cost = smem_i;                      // [N * pairs]
    int* group = smem_i + L.N * pairs;       // [N]
    const int n = (int)L.N * pairs;
    for (int x = threadIdx.x; x < n; x += blockDim.x) {
        const int64_t i = x / pairs, p = x % pairs;
        int c = 0;
        for (int64_t s = 0; s < L.N; ++s) {
            const int64_t j = ra::ring_block(i, s, L.N);
            c += live_tiles(L, causal, i, p * kPairRows, j) + live_tiles(L, causal, i, p * kPairRows + kTileRows, j);
        }
        cost[x] = c;
    }
    __syncthreads();
    for (int g = threadIdx.x; g < (int)L.N; g += blockDim.x) {
        int t = 0;
        for (int p = 0; p < pairs; ++p) t += cost[g * pairs + p];
        group[g] = t;
    }
    __syncthreads();
    for (int x = threadIdx.x; x < n; x += blockDim.x) {
        const int c = cost[x], gx = x / pairs, gc = group[gx];
        int rank = 0;
        for (int y = 0; y < n; ++y) {
            const int cy = cost[y];
            bool before;
            if (by_shard) {
                const int gy = y / pairs, gcy = group[gy];
                before = (gcy > gc) || (gcy == gc && (gy < gx || (gy == gx && (cy > c || (cy == c && y < x)))));
            } else {
                before = (cy > c) || (cy == c && y < x);
            }
            rank += before;
        }
        const int i = x / pairs, p = x % pairs;
        for (int64_t bh = 0; bh < BH; ++bh)
            items[bh * n + rank] = make_int4((int)(bh / H), (int)(bh % H), i, p);
    }
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

extern "C" int ra_forward_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                                  int64_t B, int64_t H, int64_t S, int64_t D, int n_ring, int causal,
                                  int layout, void* stream_handle) {
    const int dtype = RA_DTYPE_BF16;
    int rc = ra::host_check_shape(B, H, S, D, n_ring, layout, dtype);
    if (rc != RA_OK) return rc;
    if (!q || !k || !v || !out || !lse) return RA_ERR_INVALID_ARG;
    auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!a16(q) || !a16(k) || !a16(v) || !a16(out) || (reinterpret_cast<uintptr_t>(lse) & 3u)) return RA_ERR_ALIGN;
    if (D != 64 && D != 128) return RA_ERR_UNSUPPORTED;
    int sms = 0;
    bool sm100 = false;
    int* status = nullptr;
    if ((rc = ra::host_device_facts(&sms, &sm100, &status)) != RA_OK) return rc;
    if (!sm100) return RA_ERR_UNSUPPORTED;

    const Layout L{S, (int64_t)n_ring, S / n_ring, layout};
    const int pairs = (int)((L.S_loc + kPairRows - 1) / kPairRows);
    const int64_t per_head = L.N * pairs;
    const int64_t n_items = B * H * per_head;
    const size_t tensor_bytes = (size_t)(B * S * H * D) * 2;
    const bool permute = (layout == RA_LAYOUT_ZIGZAG);  // striped is read in place
    const size_t counter_bytes = 256;  // the persistent kernel's work counter, zeroed every call
    const size_t items_bytes = align256((size_t)n_items * sizeof(int4));
    const size_t kmax_bytes = align256((size_t)(2 * B * H) * sizeof(float));
    const size_t need = counter_bytes + items_bytes + kmax_bytes + (permute ? 3 * align256(tensor_bytes) : 0);
    const size_t builder_smem = (size_t)(per_head + L.N) * sizeof(int);
    if (builder_smem > kBuilderSmemBytes) {
        ra::host_set_error("ra_forward_noalloc: too many work items per head for the device list "
                           "builder ((items per head + n_ring) * 4 bytes must stay within 48 KB)");
        return RA_ERR_NO_WORKSPACE;
    }
    if (need > kScratchBytes || n_items > INT32_MAX) {
        ra::host_set_error("ra_forward_noalloc: problem needs more scratch than the fixed "
                           "RA_NOALLOC_SCRATCH_BYTES array");
        return RA_ERR_NO_WORKSPACE;
    }
    unsigned char* scratch = nullptr;
    if ((rc = scratch_address(&scratch)) != RA_OK) return rc;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_handle);

    int* counter = reinterpret_cast<int*>(scratch);
    int4* items = reinterpret_cast<int4*>(scratch + counter_bytes);
    cudaError_t e = cudaMemsetAsync(counter, 0, sizeof(int), stream);
    if (e != cudaSuccess) return ra::host_cuda_fail(e, "work counter reset");
    build_work_list<<<1, 1024, builder_smem, stream>>>(items, B * H, H, L, causal ? 1 : 0, pairs,
                                                ra::plan_groups_by_shard(S, D) ? 1 : 0);
    e = cudaGetLastError();
    if (e != cudaSuccess) return ra::host_cuda_fail(e, "work list launch");

    const void *qs = q, *ks = k, *vs = v;
    if (permute) {
        unsigned char* base = scratch + counter_bytes + items_bytes + kmax_bytes;
        void* dst[3] = {base, base + align256(tensor_bytes), base + 2 * align256(tensor_bytes)};
        const void* src[3] = {q, k, v};
        if ((e = ra::launch_permute(src, dst, 3, B, L, H, D, 2, false, stream)) != cudaSuccess)
            return ra::host_cuda_fail(e, "permute launch");
        qs = dst[0];
        ks = dst[1];
        vs = dst[2];
    }
    ra::TcLaunch t{};
    const bool striped_natural = (layout == RA_LAYOUT_STRIPED);
    if ((rc = ra::host_encode_qkv_map(&t.tm_q, qs, B, L, H, D, striped_natural)) != RA_OK) return rc;
    if ((rc = ra::host_encode_qkv_map(&t.tm_k, ks, B, L, H, D, striped_natural)) != RA_OK) return rc;
    if ((rc = ra::host_encode_qkv_map(&t.tm_v, vs, B, L, H, D, striped_natural)) != RA_OK) return rc;
    t.items = items;
    t.n_items = (int)n_items;
    t.counter = counter;
    t.grid = (int)(n_items < sms ? n_items : sms);
    t.timeout_ns = 2000000000ull;
    t.debug = 0;
    t.status = status;

    ra::AttnArgs a{};
    a.L = L;
    a.B = B;
    a.H = H;
    a.D = D;
    a.causal = causal ? 1 : 0;
    a.dtype = dtype;
    a.s_begin = 0;
    a.s_end = n_ring;
    a.out_mode = ra::kOutFinal;
    a.out = out;
    a.lse = lse;
    a.scale = (float)(1.0 / sqrt((double)D));
    if (ra::key_norm_max_applies(B, H, D) && ra::frozen_max_pays(S, false)) {
        // the score bound of every query row (frozen max)
        float* nmax = reinterpret_cast<float*>(scratch + counter_bytes + items_bytes);
        if ((e = ra::launch_norm_max(q, k, nmax, B, S, H, D, sms, stream)) != cudaSuccess)
            return ra::host_cuda_fail(e, "norm launch");
        a.qmax = nmax;
        a.kmax = nmax + B * H;
    }
    if ((e = ra::launch_attn_tc(a, t, stream)) != cudaSuccess) return ra::host_cuda_fail(e, "attention launch");
    return RA_OK;
}
