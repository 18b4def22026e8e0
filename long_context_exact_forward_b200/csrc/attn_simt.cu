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
// computes the 4 x 4 block of scores of rows 4ty..4ty+3 and keys 4tx..4tx+3, one float4 of Q^T and
// one of K^T per step over the head dim (16 FMAs per two shared-memory loads), and the
// 4 x (kDMax / 16) block of the output of the same rows and the columns 4tx + 64c + (0..3) from P^T
// and V, one float4 of P^T and kDMax / 64 float4s of V per key (8 consecutive threads read 128
// consecutive bytes of V, so the float4 loads are free of bank conflicts).  Two CTAs share an SM.  Row maxima and sums are reduced over
// the 16 threads of a row group with shuffles.  Keys and values are gathered straight from natural
// order with the layout map, so no permute is needed.
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

// P^T is stored key-major with its 4-row groups permuted by an XOR with (key / 4) mod 16, so that
// both the 16 threads of a row group writing one key each and the float4 reads of the P V loop
// hit distinct banks.
__device__ __forceinline__ int pt_index(int key, int row4) {
    return key * kBQ + (((row4 >> 2) ^ ((key >> 2) & 15)) << 2);
}

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
    const int64_t S_axis = args.L.S;  // token axis of out and lse (the packed length for packed sequences)
    Layout L = args.L;
    int64_t i, b, h, a0, base = 0;
    if (items) {  // packed sequences: this block's item, the sequence's own layout
        const int4 it = items[blockIdx.x];
        const int2 sd = args.seqs[it.x];
        L = Layout{sd.x, args.L.N, sd.x / args.L.N, args.L.kind};
        base = sd.y;
        i = it.y;
        a0 = (int64_t)it.z * kBQ;
        b = 0;
        h = blockIdx.z;
    } else {
        // heaviest shards first: under the causal mask with the contiguous layout shard i meets
        // i + 1 live blocks, so the CTAs of the last shards are launched first (a longest-first order)
        i = args.local ? args.q_shard : L.N - 1 - blockIdx.y;
        b = blockIdx.z / H;
        h = blockIdx.z % H;
        a0 = (int64_t)blockIdx.x * kBQ;
    }
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
    const int64_t a_last = (a0 + kBQ - 1 < L.S_loc - 1) ? a0 + kBQ - 1 : L.S_loc - 1;

    load_transposed<T, kDMax, kBQ>(Qt, q, L, args.local, b, base, h, H, D, i, a0);

    float m[4], l[4], o[4][kOC];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.f;
#pragma unroll
        for (int c = 0; c < kOC; ++c) o[r][c] = 0.f;
    }

    for (int s = args.s_begin; s < args.s_end; ++s) {
        const int64_t j = ring_block(i, s, L.N);
        int64_t n_vis[4];  // visible keys of block j for each of this thread's rows
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int64_t a = a0 + 4 * ty + r;
            n_vis[r] = a < L.S_loc ? visible_keys(L, args.causal, i, a, j) : 0;
        }
        const int64_t n_vis_cta = visible_keys(L, args.causal, i, a_last, j);  // the CTA's widest
        for (int64_t b0 = 0; b0 < n_vis_cta; b0 += kBK) {
            __syncthreads();  // previous tile consumed (and Q loaded on the first pass)
            load_transposed<T, kDMax, kBK>(Kt, k, L, args.local, b, base, h, H, D, j, b0);
            load_rowmajor<T, kDMax, kBK>(Vs, v, L, args.local, b, base, h, H, D, j, b0);
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

            float alpha[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                float mx = -INFINITY;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const bool vis = (b0 + 4 * tx + c) < n_vis[r];
                    sc[r][c] = vis ? sc[r][c] * args.scale : -INFINITY;
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
            for (int key = 0; key < kBK; ++key) {
                const float4 pa = *reinterpret_cast<const float4*>(Pt + pt_index(key, 4 * ty));
                const float pv[4] = {pa.x, pa.y, pa.z, pa.w};
#pragma unroll
                for (int c4 = 0; c4 < kOC / 4; ++c4) {
                    const float4 vb = *reinterpret_cast<const float4*>(Vs + key * kDMax + 4 * tx + 64 * c4);
                    const float vv[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
                    for (int r = 0; r < 4; ++r)
#pragma unroll
                        for (int c = 0; c < 4; ++c) o[r][4 * c4 + c] = fmaf(pv[r], vv[c], o[r][4 * c4 + c]);
                }
            }
        }
    }

#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int64_t a = a0 + 4 * ty + r;
        if (a >= L.S_loc) continue;
        const float inv_l = (l[r] > 0.f) ? 1.f / l[r] : 0.f;
        const float lse = (l[r] > 0.f) ? m[r] + logf(l[r]) : -INFINITY;
        if (args.out_mode == kOutFinal) {
            const int64_t g = base + global_position(L, i, a);
            T* dst = static_cast<T*>(args.out) + ((b * S_axis + g) * H + h) * D;
#pragma unroll
            for (int c = 0; c < kOC; ++c) {
                const int d = 4 * tx + 64 * (c / 4) + c % 4;
                if (d < D) dst[d] = from_float<T>(o[r][c] * inv_l);
            }
            if (tx == 0) args.lse[(b * H + h) * S_axis + g] = lse;
        } else {
            // partial rows: packed sequences in natural packed order, batch mode shard-major (or
            // local rows for a ring step on local buffers)
            const int64_t row = items ? (base + global_position(L, i, a)) * H + h
                                : args.local ? (b * L.S_loc + a) * H + h
                                             : ((b * L.N + i) * L.S_loc + a) * H + h;
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

template <typename T, int kDMax>
cudaError_t launch_typed(const void* q, const void* k, const void* v, const AttnArgs& a, const int4* items,
                         int n_items, cudaStream_t stream) {
    const size_t smem = sizeof(float) * ((size_t)kDMax * kBQ + 2 * (size_t)kDMax * kBK + (size_t)kBK * kBQ);
    auto kern = attn_simt_kernel<T, kDMax>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid = items ? dim3((unsigned)n_items, 1u, (unsigned)a.H)
                            : dim3((unsigned)((a.L.S_loc + kBQ - 1) / kBQ), a.local ? 1u : (unsigned)a.L.N,
                                   (unsigned)(a.B * a.H));
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
