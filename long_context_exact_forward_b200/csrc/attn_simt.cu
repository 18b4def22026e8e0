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
// Tiling: a CTA of 128 threads owns 32 query rows of one shard for one (b, h); 4 threads share a
// row (each scores 8 of the 32 keys of a tile and owns every 4th output column).  Keys and values
// are gathered straight from natural order with the layout map, so no permute is needed.
#include <cuda_bf16.h>

#include "ra_internal.cuh"

namespace ra {
namespace {

constexpr int kBQ = 32;       // query rows per CTA
constexpr int kBK = 32;       // keys per tile
constexpr int kThreads = 128; // 4 threads per query row

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

// Load `rows` token rows of shard `shard` starting at local row a0 into smem [kB][ld] as fp32;
// rows past the shard end read as zero.
template <typename T>
__device__ void load_rows(float* dst, int ld, const T* __restrict__ src, const Layout& L,
                          int64_t b, int64_t h, int64_t H, int64_t D, int64_t shard, int64_t a0,
                          int rows) {
    for (int idx = threadIdx.x; idx < rows * D; idx += kThreads) {
        const int r = idx / (int)D, d = idx % (int)D;
        const int64_t a = a0 + r;
        float x = 0.f;
        if (a < L.S_loc) {
            const int64_t g = global_position(L, shard, a);
            x = to_float<T>(src[((b * L.S + g) * H + h) * D + d]);
        }
        dst[r * ld + d] = x;
    }
}

template <typename T, int kDMax>
__global__ void __launch_bounds__(kThreads) attn_simt_kernel(const T* __restrict__ q,
                                                             const T* __restrict__ k,
                                                             const T* __restrict__ v, AttnArgs args) {
    constexpr int kCols = kDMax / 4;  // output columns owned per thread
    extern __shared__ float smem[];
    const Layout L = args.L;
    const int64_t D = args.D, H = args.H;
    const int ldq = (int)D + 1, ldk = (int)D + 1, ldv = (int)D, ldp = kBK + 1;
    float* Qs = smem;
    float* Ks = Qs + kBQ * ldq;
    float* Vs = Ks + kBK * ldk;
    float* Ps = Vs + kBK * ldv;

    const int64_t i = blockIdx.y;
    const int64_t bh = blockIdx.z;
    const int64_t b = bh / H, h = bh % H;
    const int64_t a0 = (int64_t)blockIdx.x * kBQ;
    const int r = threadIdx.x >> 2, sub = threadIdx.x & 3;
    const int64_t a = a0 + r;

    load_rows<T>(Qs, ldq, q, L, b, h, H, D, i, a0, kBQ);

    float m = -INFINITY, l = 0.f;
    float o[kCols];
#pragma unroll
    for (int c = 0; c < kCols; ++c) o[c] = 0.f;

    const int64_t a_last = (a0 + kBQ - 1 < L.S_loc - 1) ? a0 + kBQ - 1 : L.S_loc - 1;
    for (int s = args.s_begin; s < args.s_end; ++s) {
        const int64_t j = ring_block(i, s, L.N);
        const int64_t n_vis = visible_keys(L, args.causal, i, a, j);           // this row
        const int64_t n_vis_cta = visible_keys(L, args.causal, i, a_last, j);  // the CTA's widest
        for (int64_t b0 = 0; b0 < n_vis_cta; b0 += kBK) {
            __syncthreads();  // previous tile fully consumed (and Q loaded on the first pass)
            load_rows<T>(Ks, ldk, k, L, b, h, H, D, j, b0, kBK);
            load_rows<T>(Vs, ldv, v, L, b, h, H, D, j, b0, kBK);
            __syncthreads();

            // scores for keys b0 + sub*8 + x
            float sc[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) sc[x] = 0.f;
            for (int d = 0; d < D; ++d) {
                const float qd = Qs[r * ldq + d];
#pragma unroll
                for (int x = 0; x < 8; ++x) sc[x] = fmaf(qd, Ks[(sub * 8 + x) * ldk + d], sc[x]);
            }
            float mx = -INFINITY;
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const bool ok = (b0 + sub * 8 + x) < n_vis;
                sc[x] = ok ? sc[x] * args.scale : -INFINITY;
                mx = fmaxf(mx, sc[x]);
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m, mx);
            // rows with nothing visible yet keep weight 0 and avoid (-inf) - (-inf)
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            const float alpha = expf(m - m_use);
            float psum = 0.f;
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const float p = expf(sc[x] - m_use);
                psum += p;
                Ps[r * ldp + sub * 8 + x] = p;
            }
            psum += __shfl_xor_sync(0xffffffffu, psum, 1);
            psum += __shfl_xor_sync(0xffffffffu, psum, 2);
            l = l * alpha + psum;
            m = m_new;
            __syncwarp();
#pragma unroll
            for (int c = 0; c < kCols; ++c) {
                const int d = sub + 4 * c;
                if (d < D) {
                    float acc = o[c] * alpha;
                    for (int kk = 0; kk < kBK; ++kk) acc = fmaf(Ps[r * ldp + kk], Vs[kk * ldv + d], acc);
                    o[c] = acc;
                }
            }
            __syncwarp();
        }
    }

    if (a >= L.S_loc) return;
    const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
    const float lse = (l > 0.f) ? m + logf(l) : -INFINITY;
    if (args.out_mode == kOutFinal) {
        const int64_t g = global_position(L, i, a);
        T* dst = static_cast<T*>(args.out) + ((b * L.S + g) * H + h) * D;
#pragma unroll
        for (int c = 0; c < kCols; ++c) {
            const int d = sub + 4 * c;
            if (d < D) dst[d] = from_float<T>(o[c] * inv_l);
        }
        if (sub == 0) args.lse[(b * H + h) * L.S + g] = lse;
    } else {
        const int64_t row = ((b * L.N + i) * L.S_loc + a) * H + h;
        float* dst = static_cast<float*>(args.out) + row * D;
#pragma unroll
        for (int c = 0; c < kCols; ++c) {
            const int d = sub + 4 * c;
            if (d < D) dst[d] = o[c] * inv_l;
        }
        if (sub == 0) args.lse[row] = lse;
    }
}

template <typename T, int kDMax>
cudaError_t launch_typed(const void* q, const void* k, const void* v, const AttnArgs& a,
                         cudaStream_t stream) {
    const int D = (int)a.D;
    const size_t smem = sizeof(float) * ((size_t)kBQ * (D + 1) + (size_t)kBK * (D + 1) +
                                         (size_t)kBK * D + (size_t)kBQ * (kBK + 1));
    auto kern = attn_simt_kernel<T, kDMax>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((a.L.S_loc + kBQ - 1) / kBQ), (unsigned)a.L.N, (unsigned)(a.B * a.H));
    kern<<<grid, kThreads, smem, stream>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                           static_cast<const T*>(v), a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dispatch(const void* q, const void* k, const void* v, const AttnArgs& a,
                            cudaStream_t stream) {
    if (a.D <= 32) return launch_typed<T, 32>(q, k, v, a, stream);
    if (a.D <= 64) return launch_typed<T, 64>(q, k, v, a, stream);
    if (a.D <= 128) return launch_typed<T, 128>(q, k, v, a, stream);
    return launch_typed<T, 256>(q, k, v, a, stream);
}

}  // namespace

cudaError_t launch_attn_simt(const void* q, const void* k, const void* v, const AttnArgs& a,
                             cudaStream_t stream) {
    if (a.B * a.H * a.L.S == 0) return cudaSuccess;
    if (a.dtype == 0) return launch_dispatch<float>(q, k, v, a, stream);
    return launch_dispatch<__nv_bfloat16>(q, k, v, a, stream);
}

}  // namespace ra
