// attn_simt.cu -- ring-order blockwise attention on CUDA cores with fp32 arithmetic.
//
// This is the exact-fp32 path (tf32 tensor-core products keep 10 mantissa bits and could not meet
// a 1e-5 error bound) and the path for head dims the tensor-core kernel does not cover.  It runs
// the loop of the ultralytics.com "Ring Attention" toy: shard i keeps its query block; at ring step
// s it meets the key/value block of shard j = (i - s) mod N; scores S = Q K^T / sqrt(D) are turned
// into weights exp(S - m) against a running max m (the max subtraction the same page says
// production kernels add), and the running sum l and weighted-value accumulator are rescaled with
// the online-softmax identities (troisinh.com "Ring Attention", "Tai sao no hoat dong") whenever
// m grows; the accumulator is divided by l at the end.
//
// Tiling (register-blocked, like a single-precision GEMM): a CTA of 256 threads owns 64 query rows
// of one shard for one (b, h) and walks 64-key tiles.  Thread (ty, tx) = (tid / 16, tid % 16)
// computes the 4 x 4 block of scores of rows 4ty..4ty+3 and four keys, and the 4 x (kDMax / 16)
// block of the output of the same rows and the columns 4tx + 64c + (0..3) from P^T and V, one float4
// of P^T and kDMax / 64 four-element loads of V per key (16 consecutive threads read consecutive
// bytes of V, free of bank conflicts).  Row maxima and sums are reduced over the 16 threads of a
// row group with shuffles.  Q^T is held in fp32 for the whole item.  Keys and values are gathered
// straight from natural order with the layout map, so no permute is needed.
//
// Two forms of the key/value tile loop:
//   pipelined (every token row a whole number of 16-byte vectors: D * sizeof(T) % 16 == 0): K and V
//     tiles are copied row-major, in the input's own type, by cp.async into two shared-memory
//     stages, the next tile's copies in flight while the current tile is computed.  K rows are
//     padded by 16 bytes so that the four-element K loads of 16 threads (keys tx + 16c, 0 <= c < 4)
//     fall in distinct banks; 8 threads' loads share a 128-byte wavefront.  Per step of 4 over the
//     head dim a thread makes 8 shared-memory loads for 64 FMAs.
//   synchronous (other head dims): K^T and V are gathered as fp32 by the threads between two
//     barriers, and a thread takes keys 4tx..4tx+3, one float4 of Q^T and one of K^T per head-dim
//     step.
//
// Packed sequences (several sequences one after another on the token axis, batch 1): block x takes
// the work item items[x] = {sequence, shard, 64-row query tile} and block z the head; the sequence's
// own layout map (its length split into N shards) places every row, offset by the sequence's first
// token, so a query only meets the keys of its own sequence.
#include <cuda_bf16.h>

#include "ra_internal.cuh"

namespace ra {
namespace {

constexpr int kBQ = 64;        // query rows per CTA
constexpr int kBK = 64;        // keys per tile
constexpr int kThreads = 256;  // 16 x 16 thread grid

template <typename T>
__device__ __forceinline__ float to_float(T x);
template <>
__device__ __forceinline__ float to_float<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_float<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_float(float x);
template <>
__device__ __forceinline__ float from_float<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_float<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Four consecutive elements from shared memory as fp32 (p 16-byte aligned for fp32, 8 for bf16).
template <typename T>
__device__ __forceinline__ float4 load4(const T* p);
template <>
__device__ __forceinline__ float4 load4<float>(const float* p) {
    return *reinterpret_cast<const float4*>(p);
}
template <>
__device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u), __uint_as_float(u.y << 16),
                       __uint_as_float(u.y & 0xffff0000u));
}

// 16-byte asynchronous copy global -> shared, cached in L2 only; with `valid` false nothing is read
// and the 16 bytes are zero-filled.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int kPending>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory");
}

// Token row of local token a of shard `shard`: natural order through the layout map (after the
// first token `base` of a packed sequence), or, for a ring step on local buffers, row a of the
// one-shard buffer.
__device__ __forceinline__ int64_t token_row(const Layout& L, int local, int64_t b, int64_t base, int64_t shard,
                                             int64_t a) {
    return local ? b * L.S_loc + a : b * L.S + base + global_position(L, shard, a);
}

// Gather `kB` token rows of shard `shard` from local row a0 (natural order through the layout map)
// as fp32 into shared memory, transposed: dst[d * kB + r].  Rows past the shard end and columns
// d >= D read as zero.  Thread t takes row t % kB and 4 consecutive columns at a time, so
// consecutive threads write consecutive words and each thread reads whole sectors of its row.
template <typename T, int kDMax, int kB>
__device__ void load_transposed(float* dst, const T* __restrict__ src, const Layout& L, int local, int64_t b,
                                int64_t base, int64_t h, int64_t H, int64_t D, int64_t shard, int64_t a0) {
    const int r = threadIdx.x % kB;
    const int64_t a = a0 + r;
    const T* row = nullptr;
    if (a < L.S_loc) row = src + (token_row(L, local, b, base, shard, a) * H + h) * D;
    for (int d4 = 4 * (threadIdx.x / kB); d4 < kDMax; d4 += 4 * (kThreads / kB)) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int d = d4 + e;
            dst[d * kB + r] = (row && d < D) ? to_float<T>(row[d]) : 0.f;
        }
    }
}

// Same rows, row-major: dst[r * kDMax + d].  Consecutive threads take consecutive columns.
template <typename T, int kDMax, int kB>
__device__ void load_rowmajor(float* dst, const T* __restrict__ src, const Layout& L, int local, int64_t b,
                              int64_t base, int64_t h, int64_t H, int64_t D, int64_t shard, int64_t a0) {
    for (int idx = threadIdx.x; idx < kB * kDMax; idx += kThreads) {
        const int r = idx / kDMax, d = idx % kDMax;
        const int64_t a = a0 + r;
        float x = 0.f;
        if (a < L.S_loc && d < D)
            x = to_float<T>(src[(token_row(L, local, b, base, shard, a) * H + h) * D + d]);
        dst[idx] = x;
    }
}

// P^T is stored key-major, [kBK][kBQ], with the 4-row group g of key `key` at group position
// g ^ swz(key), so that the float4 stores of one instruction (16 keys x 2 row groups) spread over
// all banks and the float4 reads of the P V loop (one key, 2 row groups per warp) hit distinct
// banks.  Synchronous form: keys 4tx + c, swizzled by key / 4; pipelined form: keys tx + 16c,
// swizzled by key mod 16.
__device__ __forceinline__ int pt_index(int key, int row4) {
    return key * kBQ + (((row4 >> 2) ^ ((key >> 2) & 15)) << 2);
}
__device__ __forceinline__ int pt_index_strided(int key, int row4) {
    return key * kBQ + ((((row4 >> 2) ^ key) & 15) << 2);
}

// The item of this block: shard i, batch b, head h, first local query row a0, and the layout of the
// sequence it belongs to (the whole problem, or one packed sequence starting at token `base`).
struct Item {
    Layout L;
    int64_t i, b, h, a0, base;
};

__device__ __forceinline__ Item block_item(const AttnArgs& args, const int4* __restrict__ items) {
    Item it;
    it.L = args.L;
    it.base = 0;
    if (items) {  // packed sequences: this block's item, the sequence's own layout
        const int4 w = items[blockIdx.x];
        const int2 sd = args.seqs[w.x];
        it.L = Layout{sd.x, args.L.N, sd.x / args.L.N, args.L.kind};
        it.base = sd.y;
        it.i = w.y;
        it.a0 = (int64_t)w.z * kBQ;
        it.b = 0;
        it.h = blockIdx.z;
    } else {
        // heaviest shards first: under the causal mask with the contiguous layout shard i meets
        // i + 1 live blocks, so the CTAs of the last shards are launched first (a longest-first order)
        it.i = args.local ? args.q_shard : it.L.N - 1 - blockIdx.y;
        it.b = blockIdx.z / args.H;
        it.h = blockIdx.z % args.H;
        it.a0 = (int64_t)blockIdx.x * kBQ;
    }
    return it;
}

// Online-softmax update of one 4 x 4 score block: masks keys at or past each row's visible count,
// scales, updates the running max m and sum l, turns sc into weights and returns the factor the
// output rows must be rescaled by in alpha.
__device__ __forceinline__ void softmax_block(float (&sc)[4][4], const int64_t (&key)[4], const int64_t (&n_vis)[4],
                                              float scale, float (&m)[4], float (&l)[4], float (&alpha)[4]) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            sc[r][c] = key[c] < n_vis[r] ? sc[r][c] * scale : -INFINITY;
            mx = fmaxf(mx, sc[r][c]);
        }
#pragma unroll
        for (int off = 1; off < 16; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_new = fmaxf(m[r], mx);
        // rows with nothing visible yet keep weight 0 and avoid (-inf) - (-inf)
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        alpha[r] = expf(m[r] - m_use);
        float psum = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            sc[r][c] = expf(sc[r][c] - m_use);
            psum += sc[r][c];
        }
#pragma unroll
        for (int off = 1; off < 16; off <<= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
        l[r] = l[r] * alpha[r] + psum;
        m[r] = m_new;
    }
}

// Write the thread's 4 output rows (O / l and lse = m + ln l): final rows in natural order, or
// partial rows (packed sequences: natural packed rows; batch mode: shard-major, or local rows for a
// ring step on local buffers).
template <typename T, int kOC>
__device__ __forceinline__ void store_rows(const AttnArgs& args, const Item& it, bool packed, int ty, int tx,
                                           const float (&o)[4][kOC], const float (&m)[4], const float (&l)[4]) {
    const Layout& L = it.L;
    const int64_t D = args.D, H = args.H, S_axis = args.L.S;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int64_t a = it.a0 + 4 * ty + r;
        if (a >= L.S_loc) continue;
        const float inv_l = (l[r] > 0.f) ? 1.f / l[r] : 0.f;
        const float lse = (l[r] > 0.f) ? m[r] + logf(l[r]) : -INFINITY;
        if (args.out_mode == kOutFinal) {
            const int64_t g = it.base + global_position(L, it.i, a);
            T* dst = static_cast<T*>(args.out) + ((it.b * S_axis + g) * H + it.h) * D;
#pragma unroll
            for (int c = 0; c < kOC; ++c) {
                const int d = 4 * tx + 64 * (c / 4) + c % 4;
                if (d < D) dst[d] = from_float<T>(o[r][c] * inv_l);
            }
            if (tx == 0) args.lse[(it.b * H + it.h) * S_axis + g] = lse;
        } else {
            const int64_t row = packed       ? (it.base + global_position(L, it.i, a)) * H + it.h
                                : args.local ? (it.b * L.S_loc + a) * H + it.h
                                             : ((it.b * L.N + it.i) * L.S_loc + a) * H + it.h;
            float* dst = static_cast<float*>(args.out) + row * D;
#pragma unroll
            for (int c = 0; c < kOC; ++c) {
                const int d = 4 * tx + 64 * (c / 4) + c % 4;
                if (d < D) dst[d] = o[r][c] * inv_l;
            }
            if (tx == 0) args.lse[row] = lse;
        }
    }
}

// ------------------------------------------------------------------ synchronous form
template <typename T, int kDMax>
__global__ void __launch_bounds__(kThreads, kDMax <= 128 ? 2 : 1)
    attn_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     AttnArgs args, const int4* __restrict__ items) {
    constexpr int kOC = kDMax / 16;  // output columns per thread
    static_assert(kOC % 4 == 0, "kDMax is a multiple of 64");
    extern __shared__ __align__(16) float smem[];
    float* Qt = smem;                 // [kDMax][kBQ]
    float* Kt = Qt + kDMax * kBQ;     // [kDMax][kBK]
    float* Vs = Kt + kDMax * kBK;     // [kBK][kDMax]
    float* Pt = Vs + kBK * kDMax;     // [kBK][kBQ], swizzled (pt_index)

    const int64_t D = args.D, H = args.H;
    const Item it = block_item(args, items);
    const Layout& L = it.L;
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
    const int64_t a_last = (it.a0 + kBQ - 1 < L.S_loc - 1) ? it.a0 + kBQ - 1 : L.S_loc - 1;

    load_transposed<T, kDMax, kBQ>(Qt, q, L, args.local, it.b, it.base, it.h, H, D, it.i, it.a0);

    float m[4], l[4], o[4][kOC];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.f;
#pragma unroll
        for (int c = 0; c < kOC; ++c) o[r][c] = 0.f;
    }

    for (int s = args.s_begin; s < args.s_end; ++s) {
        const int64_t j = ring_block(it.i, s, L.N);
        int64_t n_vis[4];  // visible keys of block j for each of this thread's rows
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int64_t a = it.a0 + 4 * ty + r;
            n_vis[r] = a < L.S_loc ? visible_keys(L, args.causal, it.i, a, j) : 0;
        }
        const int64_t n_vis_cta = visible_keys(L, args.causal, it.i, a_last, j);  // the CTA's widest
        for (int64_t b0 = 0; b0 < n_vis_cta; b0 += kBK) {
            __syncthreads();  // previous tile consumed (and Q loaded on the first pass)
            load_transposed<T, kDMax, kBK>(Kt, k, L, args.local, it.b, it.base, it.h, H, D, j, b0);
            load_rowmajor<T, kDMax, kBK>(Vs, v, L, args.local, it.b, it.base, it.h, H, D, j, b0);
            __syncthreads();

            // S block: rows 4ty + r, keys 4tx + c
            float sc[4][4];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) sc[r][c] = 0.f;
#pragma unroll 4
            for (int d = 0; d < D; ++d) {
                const float4 qa = *reinterpret_cast<const float4*>(Qt + d * kBQ + 4 * ty);
                const float4 kb = *reinterpret_cast<const float4*>(Kt + d * kBK + 4 * tx);
                const float qv[4] = {qa.x, qa.y, qa.z, qa.w}, kv[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int c = 0; c < 4; ++c) sc[r][c] = fmaf(qv[r], kv[c], sc[r][c]);
            }

            const int64_t key[4] = {b0 + 4 * tx, b0 + 4 * tx + 1, b0 + 4 * tx + 2, b0 + 4 * tx + 3};
            float alpha[4];
            softmax_block(sc, key, n_vis, args.scale, m, l, alpha);
#pragma unroll
            for (int c = 0; c < 4; ++c)
                *reinterpret_cast<float4*>(Pt + pt_index(4 * tx + c, 4 * ty)) =
                    make_float4(sc[0][c], sc[1][c], sc[2][c], sc[3][c]);
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < kOC; ++c) o[r][c] *= alpha[r];
            __syncthreads();

            // O block: rows 4ty + r, columns 4tx + 64 (c / 4) + c % 4
#pragma unroll 2
            for (int kk = 0; kk < kBK; ++kk) {
                const float4 pa = *reinterpret_cast<const float4*>(Pt + pt_index(kk, 4 * ty));
                const float pv[4] = {pa.x, pa.y, pa.z, pa.w};
#pragma unroll
                for (int c4 = 0; c4 < kOC / 4; ++c4) {
                    const float4 vb = *reinterpret_cast<const float4*>(Vs + kk * kDMax + 4 * tx + 64 * c4);
                    const float vv[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
                    for (int r = 0; r < 4; ++r)
#pragma unroll
                        for (int c = 0; c < 4; ++c) o[r][4 * c4 + c] = fmaf(pv[r], vv[c], o[r][4 * c4 + c]);
                }
            }
        }
    }
    store_rows<T, kOC>(args, it, items != nullptr, ty, tx, o, m, l);
}

// ------------------------------------------------------------------ pipelined form
template <typename T, int kDMax>
struct PipeShape {
    static constexpr int kVec = 16 / (int)sizeof(T);         // elements per 16-byte copy
    static constexpr int kKStride = kDMax + kVec;            // padded K row (elements)
    static constexpr int kStages = (sizeof(T) == 4 && kDMax > 128) ? 1 : 2;
    static constexpr size_t kQtBytes = sizeof(float) * kDMax * kBQ;
    static constexpr size_t kKBytes = sizeof(T) * kBK * kKStride;  // one stage
    static constexpr size_t kVBytes = sizeof(T) * kBK * kDMax;
    static constexpr size_t kPtBytes = sizeof(float) * kBK * kBQ;
    static constexpr size_t kSmem = kQtBytes + kStages * (kKBytes + kVBytes) + kPtBytes;
    static_assert(kSmem <= 227 * 1024, "shared memory of one CTA");
};

// The (ring step, key tile) sequence of one item: block j = (i - s) mod N, tiles b0 = 0, 64, ... up
// to the widest visible prefix of the item's rows; steps with nothing visible are skipped.
struct TileSeq {
    int s, s_end;
    int64_t j, b0, n;
    bool valid;
    __device__ __forceinline__ void seek(const Layout& L, int causal, int64_t i, int64_t a_last) {
        for (; s < s_end; ++s) {
            j = ring_block(i, s, L.N);
            n = visible_keys(L, causal, i, a_last, j);
            if (n > 0) {
                valid = true;
                return;
            }
        }
        valid = false;
    }
    __device__ __forceinline__ void next(const Layout& L, int causal, int64_t i, int64_t a_last) {
        b0 += kBK;
        if (b0 < n) return;
        b0 = 0;
        ++s;
        seek(L, causal, i, a_last);
    }
};

template <typename T, int kDMax>
__global__ void __launch_bounds__(kThreads, kDMax <= 64 ? 2 : 1)
    attn_simt_pipe_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                          AttnArgs args, const int4* __restrict__ items) {
    using P = PipeShape<T, kDMax>;
    constexpr int kOC = kDMax / 16;
    static_assert(kOC % 4 == 0, "kDMax is a multiple of 64");
    extern __shared__ __align__(16) uint8_t smem_bytes[];
    float* Qt = reinterpret_cast<float*>(smem_bytes);                                  // [kDMax][kBQ]
    T* Ks = reinterpret_cast<T*>(smem_bytes + P::kQtBytes);                            // [stage][kBK][kKStride]
    T* Vs = reinterpret_cast<T*>(smem_bytes + P::kQtBytes + P::kStages * P::kKBytes);  // [stage][kBK][kDMax]
    float* Pt = reinterpret_cast<float*>(smem_bytes + P::kQtBytes + P::kStages * (P::kKBytes + P::kVBytes));

    const int64_t D = args.D, H = args.H;
    const Item it = block_item(args, items);
    const Layout& L = it.L;
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
    const int64_t a_last = (it.a0 + kBQ - 1 < L.S_loc - 1) ? it.a0 + kBQ - 1 : L.S_loc - 1;

    // columns D .. kDMax-1 of the stages are never copied; V's are read by the P V loop, so they
    // hold zeros (K's padding and tail columns are never read)
    if (D < kDMax) {
        for (int x = threadIdx.x; x < P::kStages * kBK * kDMax; x += kThreads) Vs[x] = from_float<T>(0.f);
    }
    load_transposed<T, kDMax, kBQ>(Qt, q, L, args.local, it.b, it.base, it.h, H, D, it.i, it.a0);
    __syncthreads();  // the zero fill is ordered before the copies below

    // issue the copies of one (K, V) tile into `stage`; rows past the block's end are zero-filled
    const int vecs = (int)(D / P::kVec);
    auto issue = [&](int stage, const TileSeq& t) {
        T* ks = Ks + stage * kBK * P::kKStride;
        T* vs = Vs + stage * kBK * kDMax;
        for (int x = threadIdx.x; x < kBK * vecs; x += kThreads) {
            const int r = x / vecs, c = x % vecs;
            const int64_t a = t.b0 + r;
            const bool valid = a < L.S_loc;
            const int64_t row = valid ? (token_row(L, args.local, it.b, it.base, t.j, a) * H + it.h) * D : 0;
            cp_async16(ks + r * P::kKStride + c * P::kVec, k + row + c * P::kVec, valid);
            cp_async16(vs + r * kDMax + c * P::kVec, v + row + c * P::kVec, valid);
        }
        cp_async_commit();
    };

    float m[4], l[4], o[4][kOC];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.f;
#pragma unroll
        for (int c = 0; c < kOC; ++c) o[r][c] = 0.f;
    }

    TileSeq cur{args.s_begin, args.s_end, 0, 0, 0, false};
    cur.seek(L, args.causal, it.i, a_last);
    if (cur.valid) issue(0, cur);
    int stage = 0;
    int s_vis = -1;  // ring step whose visible counts n_vis holds
    int64_t n_vis[4] = {0, 0, 0, 0};
    while (cur.valid) {
        TileSeq nxt = cur;
        nxt.next(L, args.causal, it.i, a_last);
        if (P::kStages == 2 && nxt.valid) {
            issue(stage ^ 1, nxt);  // that stage's last readers passed the barrier ending the last tile
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();  // the current tile's copies are visible to every thread
        if (cur.s != s_vis) {
            s_vis = cur.s;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int64_t a = it.a0 + 4 * ty + r;
                n_vis[r] = a < L.S_loc ? visible_keys(L, args.causal, it.i, a, cur.j) : 0;
            }
        }
        const T* ks = Ks + stage * kBK * P::kKStride;
        const T* vs = Vs + stage * kBK * kDMax;

        // S block: rows 4ty + r, keys tx + 16c
        float sc[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) sc[r][c] = 0.f;
#pragma unroll 2
        for (int d = 0; d < D; d += 4) {
            float4 qa[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) qa[e] = *reinterpret_cast<const float4*>(Qt + (d + e) * kBQ + 4 * ty);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float4 kb = load4<T>(ks + (tx + 16 * c) * P::kKStride + d);
                const float qr[4][4] = {{qa[0].x, qa[1].x, qa[2].x, qa[3].x},
                                        {qa[0].y, qa[1].y, qa[2].y, qa[3].y},
                                        {qa[0].z, qa[1].z, qa[2].z, qa[3].z},
                                        {qa[0].w, qa[1].w, qa[2].w, qa[3].w}};
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    sc[r][c] = fmaf(qr[r][0], kb.x, sc[r][c]);
                    sc[r][c] = fmaf(qr[r][1], kb.y, sc[r][c]);
                    sc[r][c] = fmaf(qr[r][2], kb.z, sc[r][c]);
                    sc[r][c] = fmaf(qr[r][3], kb.w, sc[r][c]);
                }
            }
        }

        const int64_t key[4] = {cur.b0 + tx, cur.b0 + tx + 16, cur.b0 + tx + 32, cur.b0 + tx + 48};
        float alpha[4];
        softmax_block(sc, key, n_vis, args.scale, m, l, alpha);
#pragma unroll
        for (int c = 0; c < 4; ++c)
            *reinterpret_cast<float4*>(Pt + pt_index_strided(tx + 16 * c, 4 * ty)) =
                make_float4(sc[0][c], sc[1][c], sc[2][c], sc[3][c]);
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < kOC; ++c) o[r][c] *= alpha[r];
        __syncthreads();  // P^T complete

        // O block: rows 4ty + r, columns 4tx + 64 (c / 4) + c % 4
#pragma unroll 2
        for (int kk = 0; kk < kBK; ++kk) {
            const float4 pa = *reinterpret_cast<const float4*>(Pt + pt_index_strided(kk, 4 * ty));
            const float pv[4] = {pa.x, pa.y, pa.z, pa.w};
#pragma unroll
            for (int c4 = 0; c4 < kOC / 4; ++c4) {
                const float4 vb = load4<T>(vs + kk * kDMax + 4 * tx + 64 * c4);
                const float vv[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int c = 0; c < 4; ++c) o[r][4 * c4 + c] = fmaf(pv[r], vv[c], o[r][4 * c4 + c]);
            }
        }
        __syncthreads();  // this stage and P^T are free again
        if (P::kStages == 1 && nxt.valid) issue(0, nxt);
        cur = nxt;
        if (P::kStages == 2) stage ^= 1;
    }
    store_rows<T, kOC>(args, it, items != nullptr, ty, tx, o, m, l);
}

template <typename T, int kDMax>
cudaError_t launch_typed(const void* q, const void* k, const void* v, const AttnArgs& a, const int4* items,
                         int n_items, cudaStream_t stream) {
    const dim3 grid = items ? dim3((unsigned)n_items, 1u, (unsigned)a.H)
                            : dim3((unsigned)((a.L.S_loc + kBQ - 1) / kBQ), a.local ? 1u : (unsigned)a.L.N,
                                   (unsigned)(a.B * a.H));
    if ((a.D * (int64_t)sizeof(T)) % 16 == 0) {  // whole 16-byte vectors per row: the pipelined form
        const size_t smem = PipeShape<T, kDMax>::kSmem;
        auto kern = attn_simt_pipe_kernel<T, kDMax>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, kThreads, smem, stream>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                               static_cast<const T*>(v), a, items);
        return cudaGetLastError();
    }
    const size_t smem = sizeof(float) * ((size_t)kDMax * kBQ + 2 * (size_t)kDMax * kBK + (size_t)kBK * kBQ);
    auto kern = attn_simt_kernel<T, kDMax>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, stream>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                           static_cast<const T*>(v), a, items);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dispatch(const void* q, const void* k, const void* v, const AttnArgs& a, const int4* items,
                            int n_items, cudaStream_t stream) {
    if (a.D <= 64) return launch_typed<T, 64>(q, k, v, a, items, n_items, stream);
    if (a.D <= 128) return launch_typed<T, 128>(q, k, v, a, items, n_items, stream);
    return launch_typed<T, 256>(q, k, v, a, items, n_items, stream);
}

}  // namespace

cudaError_t launch_attn_simt(const void* q, const void* k, const void* v, const AttnArgs& a,
                             cudaStream_t stream) {
    if (a.B * a.H * a.L.S == 0) return cudaSuccess;
    if (a.dtype == 0) return launch_dispatch<float>(q, k, v, a, nullptr, 0, stream);
    return launch_dispatch<__nv_bfloat16>(q, k, v, a, nullptr, 0, stream);
}

cudaError_t launch_attn_simt_packed(const void* q, const void* k, const void* v, const AttnArgs& a,
                                    const int4* items, int n_items, cudaStream_t stream) {
    if (n_items == 0 || a.H == 0) return cudaSuccess;
    if (a.dtype == 0) return launch_dispatch<float>(q, k, v, a, items, n_items, stream);
    return launch_dispatch<__nv_bfloat16>(q, k, v, a, items, n_items, stream);
}

}  // namespace ra
