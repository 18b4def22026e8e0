// varlen.cu -- ra_forward_varlen: the ring forward pass over packed sequences.
//
// Several sequences of different lengths are packed one after another on the token axis; a query
// attends only to the keys of its own sequence (and, causal, to those at or before it).  Each
// sequence is split into the same n_ring shards with the requested layout, and its items join one
// work list, ordered longest first across all sequences (troisinh.com "Ring Attention", "Trade-off
// thuc te": load balancing with sequences of different lengths is the challenge; one list over every
// sequence lets the scheduler balance it).
//
// Tensor cores (bf16, D in {64, 128}): items are (sequence, head, shard, query-tile pair) for the
// persistent kernel's dynamic scheduler.  The kernel reads the packed tensors in place through TMA
// maps over the whole packed axis; rows past a sequence's end that a tile box still covers are masked
// by the per-row key counts of that sequence.  For the zigzag layout each sequence is first gathered
// into its own shard-major order (shard i's tokens at sequence start + i * S_loc), which the kernel
// addresses like the contiguous layout while it masks, and places its output, by the zigzag
// positions.
//
// CUDA cores (fp32 arithmetic, any dtype, D <= 256): items are (sequence, shard, 64-row query tile),
// one block per item and head, reading natural order through each sequence's layout map.
//
// Either kernel walks all ring steps in one launch, or (per-step variant) a chunk of steps per launch:
// the partial results then sit in natural packed rows and fold into the running result with the
// log-sum-exp merge, the last merge writing out and lse.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <vector>

#include "ra.h"
#include "ra_internal.cuh"

namespace {

constexpr int kTileRows = 128;  // tensor cores: query and key tile
constexpr int kPairRows = 256;  // tensor cores: rows of one work item (two query tiles)
constexpr int kSimtRows = 64;   // CUDA cores: query rows of one work item, keys per tile

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Live key tiles (`rows` keys each) of block j for the query tile of `rows` rows starting at local
// row a0 of shard i.
int64_t live_tiles(const ra::Layout& L, int causal, int64_t i, int64_t a0, int64_t j, int64_t rows) {
    if (a0 >= L.S_loc) return 0;
    const int64_t last = std::min(a0 + rows - 1, L.S_loc - 1);
    return (ra::visible_keys(L, causal, i, last, j) + rows - 1) / rows;
}

struct Item {
    int4 it;
    int64_t cost;
};

constexpr int kRowsPerBlock = 8;  // one warp per token row

struct PackArgs {
    const uint4* src[3];
    uint4* dst[3];
};

// Gather each packed sequence of q, k, v (grid.y) into its shard-major order: destination token t of
// sequence s (first token base_s, length len_s, S_loc = len_s / N) is local token a = u mod S_loc of
// shard i = u / S_loc, u = t - base_s, and comes from token base_s + g(i, a) of the source.  One warp
// copies one token row (row_vecs 16-byte vectors); HBM-bound, each row read once and written once.
__global__ void __launch_bounds__(256) pack_shard_major(PackArgs args, const int2* __restrict__ seqs, int n_seqs,
                                                        int64_t S_total, int N, int kind, int64_t row_vecs) {
    const int tensor = blockIdx.y;
    const int64_t t = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
    if (t >= S_total) return;
    // the sequence holding t: the last entry whose first token is <= t (starts are non-decreasing;
    // an empty sequence shares its start with the next entry, so it is never the last such entry)
    int lo = 0, hi = n_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (seqs[mid].y <= t) lo = mid;
        else hi = mid - 1;
    }
    const int64_t len = seqs[lo].x, base = seqs[lo].y;
    const int64_t S_loc = len / N, u = t - base;
    const ra::Layout L{len, N, S_loc, kind};
    const int64_t src_row = base + ra::global_position(L, u / S_loc, u % S_loc);
    const uint4* __restrict__ s = args.src[tensor] + src_row * row_vecs;
    uint4* __restrict__ d = args.dst[tensor] + t * row_vecs;
    for (int64_t c = threadIdx.x & 31; c < row_vecs; c += 32) d[c] = __ldcs(s + c);
}

}  // namespace

namespace {

// What one call runs: the kernel (tensor cores or CUDA cores) and the ring steps per attention launch.
struct Plan {
    bool tc;
    int chunk;     // ring steps per launch
    int n_chunks;  // attention launches
};

// Host validation shared by every entry point (nothing touches the device).  On success *S_total is
// the packed length and *plan what the call runs: kernel AUTO takes the tensor cores for bf16 with
// D in {64, 128}, the CUDA cores otherwise; variant AUTO and FUSED walk every ring step in one launch,
// PER_STEP walks steps_per_launch steps per launch (0 = 1).
int check_packed(const int64_t* cu_seqlens, int n_seqs, int64_t H, int64_t D, int n_ring, int layout, int dtype,
                 int variant, int kernel, int steps_per_launch, int64_t* S_total, Plan* plan) {
    if (!cu_seqlens || n_seqs < 1 || H < 1 || n_ring < 1 || steps_per_launch < 0) return RA_ERR_INVALID_ARG;
    if (layout != RA_LAYOUT_CONTIGUOUS && layout != RA_LAYOUT_STRIPED && layout != RA_LAYOUT_ZIGZAG)
        return RA_ERR_INVALID_ARG;
    if (dtype != RA_DTYPE_FP32 && dtype != RA_DTYPE_BF16) return RA_ERR_INVALID_ARG;
    if (variant != RA_VARIANT_AUTO && variant != RA_VARIANT_FUSED && variant != RA_VARIANT_PER_STEP)
        return RA_ERR_INVALID_ARG;
    if (kernel != RA_KERNEL_AUTO && kernel != RA_KERNEL_TC && kernel != RA_KERNEL_SIMT) return RA_ERR_INVALID_ARG;
    if (D < 1 || D > 256) return RA_ERR_SHAPE;
    const bool tc_applies = dtype == RA_DTYPE_BF16 && (D == 64 || D == 128);
    if (kernel == RA_KERNEL_TC && !tc_applies) return RA_ERR_UNSUPPORTED;
    if (cu_seqlens[0] != 0) return RA_ERR_INVALID_ARG;
    const int64_t unit = layout == RA_LAYOUT_ZIGZAG ? 2 * (int64_t)n_ring : n_ring;  // zigzag: 2N chunks
    for (int s = 0; s < n_seqs; ++s) {
        const int64_t len = cu_seqlens[s + 1] - cu_seqlens[s];
        if (len < 0) return RA_ERR_INVALID_ARG;
        if (len % unit) return RA_ERR_SHAPE;
    }
    *S_total = cu_seqlens[n_seqs];
    if (*S_total >= (int64_t(1) << 31) || H > 65535) return RA_ERR_SHAPE;
    plan->tc = kernel == RA_KERNEL_TC || (kernel == RA_KERNEL_AUTO && tc_applies);
    plan->chunk = variant == RA_VARIANT_PER_STEP ? std::min(steps_per_launch > 0 ? steps_per_launch : 1, n_ring)
                                                 : n_ring;
    plan->n_chunks = (n_ring + plan->chunk - 1) / plan->chunk;
    return RA_OK;
}

// Scratch of one call, in this order, every part 256-byte aligned: one work counter per attention
// launch, the sequence table {length, first token}, the work list (int4 per item), the largest query
// and key norm of every head (tensor cores, 2 floats per head), for zigzag on the tensor cores the
// shard-major copies of q, k, v, and with more than one launch the running result (fp32 O and lse
// in natural packed rows) and one launch's partial result.  The item count is known before the list
// is built: per non-empty sequence, H * N * ceil(S_loc / 256) tensor-core items (a head and two
// 128-row query tiles each), or N * ceil(S_loc / 64) CUDA-core items (64 rows of every head).
struct Scratch {
    size_t off_seqs, off_items, off_kmax, off_perm, off_acc, tensor_bytes, o_bytes, lse_bytes, bytes;
    int64_t n_items;
};

Scratch scratch_layout(const int64_t* cu_seqlens, int n_seqs, int64_t H, int64_t D, int n_ring, int layout,
                       int dtype, const Plan& plan, int64_t S_total) {
    Scratch w{};
    const int64_t rows_per_item = plan.tc ? kPairRows : kSimtRows;
    for (int s = 0; s < n_seqs; ++s) {
        const int64_t S_loc = (cu_seqlens[s + 1] - cu_seqlens[s]) / n_ring;
        w.n_items += (plan.tc ? H : 1) * n_ring * ((S_loc + rows_per_item - 1) / rows_per_item);
    }
    const size_t esize = dtype == RA_DTYPE_BF16 ? 2 : 4;
    w.tensor_bytes = align256((size_t)S_total * (size_t)H * (size_t)D * esize);
    w.o_bytes = align256((size_t)S_total * (size_t)H * (size_t)D * 4);
    w.lse_bytes = align256((size_t)S_total * (size_t)H * 4);
    w.off_seqs = align256((size_t)plan.n_chunks * sizeof(int));
    w.off_items = w.off_seqs + align256((size_t)n_seqs * sizeof(int2));
    w.off_kmax = w.off_items + align256((size_t)w.n_items * sizeof(int4));
    w.off_perm = w.off_kmax + (plan.tc ? align256((size_t)(2 * H) * sizeof(float)) : 0);
    w.off_acc = w.off_perm + (plan.tc && layout == RA_LAYOUT_ZIGZAG ? 3 * w.tensor_bytes : 0);
    w.bytes = w.off_acc + (plan.n_chunks > 1 ? 2 * (w.o_bytes + w.lse_bytes) : 0);
    return w;
}

// Work lists, longest first (ties in list order).  Tensor cores: (sequence, head, shard, pair of
// 128-row query tiles); CUDA cores: (sequence, shard, 64-row query tile), heads on the grid.  The
// cost of an item is its live key tiles over every ring step.
std::vector<int4> build_items(const int64_t* cu_seqlens, int n_seqs, int64_t H, int64_t N, int causal, int layout,
                              bool tc) {
    std::vector<Item> items;
    for (int s = 0; s < n_seqs; ++s) {
        const int64_t len = cu_seqlens[s + 1] - cu_seqlens[s];
        if (len == 0) continue;
        const ra::Layout L{len, N, len / N, layout};
        if (tc) {
            const int64_t pairs = (L.S_loc + kPairRows - 1) / kPairRows;
            for (int64_t i = 0; i < N; ++i)
                for (int64_t p = 0; p < pairs; ++p) {
                    int64_t cost = 0;
                    for (int64_t st = 0; st < N; ++st) {
                        const int64_t j = ra::ring_block(i, st, N);
                        cost += live_tiles(L, causal, i, p * kPairRows, j, kTileRows) +
                                live_tiles(L, causal, i, p * kPairRows + kTileRows, j, kTileRows);
                    }
                    for (int64_t h = 0; h < H; ++h) items.push_back({make_int4(s, (int)h, (int)i, (int)p), cost});
                }
        } else {
            const int64_t tiles = (L.S_loc + kSimtRows - 1) / kSimtRows;
            for (int64_t i = 0; i < N; ++i)
                for (int64_t t = 0; t < tiles; ++t) {
                    int64_t cost = 0;
                    for (int64_t st = 0; st < N; ++st)
                        cost += live_tiles(L, causal, i, t * kSimtRows, ra::ring_block(i, st, N), kSimtRows);
                    items.push_back({make_int4(s, (int)i, (int)t, 0), cost});
                }
        }
    }
    std::stable_sort(items.begin(), items.end(), [](const Item& a, const Item& b) { return a.cost > b.cost; });
    std::vector<int4> list(items.size());
    for (size_t t = 0; t < items.size(); ++t) list[t] = items[t].it;
    return list;
}

// The forward pass over packed sequences.  ws == nullptr: the scratch is allocated and freed
// stream-ordered here; otherwise ws holds at least scratch_layout(...).bytes.
int varlen_forward(const void* q, const void* k, const void* v, void* out, float* lse, const int64_t* cu_seqlens,
                   int n_seqs, int64_t H, int64_t D, int n_ring, int causal, int layout, int dtype, int variant,
                   int kernel, int steps_per_launch, cudaStream_t stream, uint8_t* ws_given, size_t ws_bytes,
                   uint64_t timeout_ns, int debug, cudaEvent_t ev0, cudaEvent_t ev1) {
    if (!q || !k || !v || !out || !lse) return RA_ERR_INVALID_ARG;
    int64_t S_total = 0;
    Plan plan{};
    int rc = check_packed(cu_seqlens, n_seqs, H, D, n_ring, layout, dtype, variant, kernel, steps_per_launch,
                          &S_total, &plan);
    if (rc != RA_OK) return rc;
    auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!a16(q) || !a16(k) || !a16(v) || !a16(out) || (reinterpret_cast<uintptr_t>(lse) & 3u)) return RA_ERR_ALIGN;
    const Scratch w = scratch_layout(cu_seqlens, n_seqs, H, D, n_ring, layout, dtype, plan, S_total);
    if (w.n_items > (int64_t)INT32_MAX) return RA_ERR_SHAPE;
    if (ws_given) {
        if (reinterpret_cast<uintptr_t>(ws_given) & 255u) return RA_ERR_ALIGN;
        if (ws_bytes < w.bytes) return RA_ERR_NO_WORKSPACE;
    }
    int sms = 0;
    bool sm100 = false;
    int* status = nullptr;
    rc = ra::host_device_facts(&sms, &sm100, &status);
    if (rc != RA_OK) return rc;
    if (plan.tc && !sm100) return RA_ERR_UNSUPPORTED;
    if (S_total == 0) return RA_OK;

    const int64_t N = n_ring;
    const std::vector<int4> list = build_items(cu_seqlens, n_seqs, H, N, causal, layout, plan.tc);
    if ((int64_t)list.size() != w.n_items) {  // the scratch was sized by the same count
        ra::host_set_error("ra_forward_varlen: work list size mismatch");
        return RA_ERR_INVALID_ARG;
    }
    std::vector<int2> seqs(n_seqs);
    for (int s = 0; s < n_seqs; ++s)
        seqs[s] = make_int2((int)(cu_seqlens[s + 1] - cu_seqlens[s]), (int)cu_seqlens[s]);

    uint8_t* ws = ws_given;
    cudaError_t e = cudaSuccess;
    if (!ws_given) {
        e = ra::scratch_alloc(reinterpret_cast<void**>(&ws), w.bytes, stream);
        if (e != cudaSuccess) return ra::host_cuda_fail(e, "stream-ordered allocation (varlen scratch)");
    }
    auto finish = [&](int r) {
        if (ws_given) return r;
        const cudaError_t ef = cudaFreeAsync(ws, stream);
        if (r == RA_OK && ef != cudaSuccess) return ra::host_cuda_fail(ef, "cudaFreeAsync(varlen scratch)");
        return r;
    };
    // pageable sources: each copy returns once its data is staged, so the vectors may go out of scope
    if ((e = cudaMemsetAsync(ws, 0, (size_t)plan.n_chunks * sizeof(int), stream)) != cudaSuccess ||
        (e = cudaMemcpyAsync(ws + w.off_seqs, seqs.data(), seqs.size() * sizeof(int2), cudaMemcpyHostToDevice,
                             stream)) != cudaSuccess ||
        (e = cudaMemcpyAsync(ws + w.off_items, list.data(), list.size() * sizeof(int4), cudaMemcpyHostToDevice,
                             stream)) != cudaSuccess)
        return finish(ra::host_cuda_fail(e, "varlen work list upload"));

    ra::AttnArgs a{};
    a.L = ra::Layout{S_total, N, S_total / N, layout};  // S = S_total; N and the kind apply per sequence
    a.B = 1;
    a.H = H;
    a.D = D;
    a.causal = causal ? 1 : 0;
    a.dtype = dtype;
    a.scale = (float)(1.0 / std::sqrt((double)D));
    a.seqs = reinterpret_cast<const int2*>(ws + w.off_seqs);
    const int4* items = reinterpret_cast<const int4*>(ws + w.off_items);

    ra::TcLaunch t{};
    if (plan.tc) {
        // zigzag: gather every sequence into its shard-major order; the kernel then reads the copies
        // with contiguous addressing (sequence start + i * S_loc + a)
        const bool zigzag = layout == RA_LAYOUT_ZIGZAG;
        const void *qs = q, *ks = k, *vs = v;
        if (zigzag) {
            PackArgs pa{};
            const void* src[3] = {q, k, v};
            for (int x = 0; x < 3; ++x) {
                pa.src[x] = static_cast<const uint4*>(src[x]);
                pa.dst[x] = reinterpret_cast<uint4*>(ws + w.off_perm + x * w.tensor_bytes);
            }
            const dim3 grid((unsigned)((S_total + kRowsPerBlock - 1) / kRowsPerBlock), 3);
            pack_shard_major<<<grid, 256, 0, stream>>>(pa, a.seqs, n_seqs, S_total, n_ring, layout, H * D * 2 / 16);
            if ((e = cudaGetLastError()) != cudaSuccess) return finish(ra::host_cuda_fail(e, "varlen permute launch"));
            qs = pa.dst[0];
            ks = pa.dst[1];
            vs = pa.dst[2];
        }
        // TMA maps over the packed axis: contiguous and zigzag copies (D, H, S_total, 1, 1); striped
        // (D, H, S_total / N, N, 1) with token = a' * N + i (every sequence starts on a multiple of N)
        const bool striped = layout == RA_LAYOUT_STRIPED;
        const ra::Layout Lmap =
            striped ? ra::Layout{S_total, N, S_total / N, layout} : ra::Layout{S_total, 1, S_total, layout};
        if ((rc = ra::host_encode_qkv_map(&t.tm_q, qs, 1, Lmap, H, D, striped)) != RA_OK ||
            (rc = ra::host_encode_qkv_map(&t.tm_k, ks, 1, Lmap, H, D, striped)) != RA_OK ||
            (rc = ra::host_encode_qkv_map(&t.tm_v, vs, 1, Lmap, H, D, striped)) != RA_OK)
            return finish(rc);
        t.items = items;
        t.n_items = (int)list.size();
        t.grid = (int)std::min<int64_t>((int64_t)list.size(), sms);
        t.timeout_ns = timeout_ns ? timeout_ns : 2000000000ull;
        t.debug = debug;
        t.status = status;
        a.varlen_striped = striped ? 1 : 0;
        // keys a query row meets per launch, on average over the packed tokens: sum len^2 / S_total
        // for a whole ring pass, a share chunk / N of it per launch
        double sq = 0.0;
        for (int q_ = 0; q_ < n_seqs; ++q_) {
            const double len = (double)(cu_seqlens[q_ + 1] - cu_seqlens[q_]);
            sq += len * len;
        }
        const int64_t keys_per_row = (int64_t)(sq / (double)S_total * plan.chunk / n_ring);
        if (ra::key_norm_max_applies(1, H, D) && ra::frozen_max_pays(keys_per_row, debug == RA_DEBUG_FROZEN_MAX)) {
            // the score bound of every query row (frozen max)
            float* nmax = reinterpret_cast<float*>(ws + w.off_kmax);
            if ((e = ra::launch_norm_max(q, k, nmax, 1, S_total, H, D, sms, stream)) != cudaSuccess)
                return finish(ra::host_cuda_fail(e, "norm launch"));
            a.qmax = nmax;
            a.kmax = nmax + H;
        }
    }

    // One launch per chunk of ring steps.  A single launch writes the result; otherwise the first
    // writes the running result in natural packed rows, each later one its own partial, which the
    // merge folds in (in place, or, after the last launch, straight to out and lse: the identity
    // layout of the packed axis).
    float* O_acc = reinterpret_cast<float*>(ws + w.off_acc);
    float* lse_acc = reinterpret_cast<float*>(ws + w.off_acc + w.o_bytes);
    float* O_s = reinterpret_cast<float*>(ws + w.off_acc + w.o_bytes + w.lse_bytes);
    float* lse_s = reinterpret_cast<float*>(ws + w.off_acc + 2 * w.o_bytes + w.lse_bytes);
    const ra::Layout Lid{S_total, 1, S_total, RA_LAYOUT_CONTIGUOUS};
    const int64_t rows = S_total * H;
    for (int c = 0; c < plan.n_chunks; ++c) {
        a.s_begin = c * plan.chunk;
        a.s_end = std::min(n_ring, a.s_begin + plan.chunk);
        if (plan.n_chunks == 1) {
            a.out_mode = ra::kOutFinal;
            a.out = out;
            a.lse = lse;
        } else {
            a.out_mode = ra::kOutPartial;
            a.out = c == 0 ? O_acc : O_s;
            a.lse = c == 0 ? lse_acc : lse_s;
        }
        if (c == 0 && ev0 && (e = cudaEventRecord(ev0, stream)) != cudaSuccess)
            return finish(ra::host_cuda_fail(e, "cudaEventRecord"));
        if (plan.tc) {
            t.counter = reinterpret_cast<int*>(ws) + c;
            e = ra::launch_attn_tc(a, t, stream);
        } else {
            e = ra::launch_attn_simt_packed(q, k, v, a, items, (int)list.size(), stream);
        }
        if (e != cudaSuccess) return finish(ra::host_cuda_fail(e, "attention launch"));
        if (c + 1 == plan.n_chunks && ev1 && (e = cudaEventRecord(ev1, stream)) != cudaSuccess)
            return finish(ra::host_cuda_fail(e, "cudaEventRecord"));
        if (c == 0 || plan.n_chunks == 1) continue;
        e = c + 1 < plan.n_chunks
                ? ra::launch_merge_inplace(O_acc, lse_acc, O_s, lse_s, rows, D, stream)
                : ra::launch_merge_final(O_acc, lse_acc, O_s, lse_s, out, lse, dtype, 1, Lid, H, D, stream);
        if (e != cudaSuccess) return finish(ra::host_cuda_fail(e, "merge launch"));
    }
    return finish(RA_OK);
}

}  // namespace

extern "C" int ra_forward_varlen(const void* q, const void* k, const void* v, void* out, float* lse,
                                 const int64_t* cu_seqlens, int n_seqs, int64_t H, int64_t D, int n_ring,
                                 int causal, int layout, int dtype, void* stream_handle) {
    return varlen_forward(q, k, v, out, lse, cu_seqlens, n_seqs, H, D, n_ring, causal, layout, dtype,
                          RA_VARIANT_AUTO, RA_KERNEL_AUTO, 0, static_cast<cudaStream_t>(stream_handle), nullptr, 0,
                          0, RA_DEBUG_NONE, nullptr, nullptr);
}

extern "C" int ra_forward_varlen_ex(const void* q, const void* k, const void* v, void* out, float* lse,
                                    const int64_t* cu_seqlens, int n_seqs, int64_t H, int64_t D, int n_ring,
                                    int causal, int layout, int dtype, void* stream_handle, const ra_options* opt) {
    ra_options o{};
    if (opt) o = *opt;
    if (o.debug != RA_DEBUG_NONE && o.debug != RA_DEBUG_STALL_LOADS && o.debug != RA_DEBUG_FROZEN_MAX)
        return RA_ERR_INVALID_ARG;
    return varlen_forward(q, k, v, out, lse, cu_seqlens, n_seqs, H, D, n_ring, causal, layout, dtype, o.variant,
                          o.kernel, o.steps_per_launch, static_cast<cudaStream_t>(stream_handle),
                          static_cast<uint8_t*>(o.workspace), o.workspace_bytes, o.timeout_ns, o.debug,
                          static_cast<cudaEvent_t>(o.attn_events[0]), static_cast<cudaEvent_t>(o.attn_events[1]));
}

extern "C" int ra_varlen_workspace_size(const int64_t* cu_seqlens, int n_seqs, int64_t H, int64_t D, int n_ring,
                                        int layout, int dtype, int variant, int kernel, size_t* bytes) {
    if (!bytes) return RA_ERR_INVALID_ARG;
    int64_t S_total = 0;
    Plan plan{};
    // PER_STEP: sized for one step per launch, which covers every steps_per_launch
    const int rc = check_packed(cu_seqlens, n_seqs, H, D, n_ring, layout, dtype, variant, kernel, 1, &S_total, &plan);
    if (rc != RA_OK) return rc;
    *bytes = scratch_layout(cu_seqlens, n_seqs, H, D, n_ring, layout, dtype, plan, S_total).bytes;
    return RA_OK;
}
