// merge.cu -- the per-ring-step merge of partial attention results.
//
// Each ring step yields, per query row, a partial output O_s normalised by its own sum and its
// log-sum-exp lse_s = m_s + ln l_s.  The merge identities of troisinh.com "Ring Attention"
// ("Tai sao no hoat dong": m' = max(m_p, m_n), l' = e^{m_p - m'} l_p + e^{m_n - m'} l_n, output
// rescaled the same way) become, with l = e^{lse - m}:
//     lse' = mx + ln(e^{lse_r - mx} + e^{lse_s - mx}),   mx = max(lse_r, lse_s)
//     O'   = e^{lse_r - lse'} O_r + e^{lse_s - lse'} O_s
// A row with lse = -inf (no visible key yet) contributes nothing; two such rows stay empty.
//
// HBM-bound: per row and step it reads O_r and O_s and writes O' (12 bytes per element in fp32)
// plus 12 bytes of lse.  Each thread handles 4 consecutive elements (float4), so a warp moves
// 512 contiguous bytes per access.
#include <cuda_bf16.h>

#include "ra_internal.cuh"

namespace ra {
namespace {

struct Weights {
    float wr, ws, lse;
};

__device__ __forceinline__ Weights merge_weights(float lr, float ls) {
    const float mx = fmaxf(lr, ls);
    if (mx == -INFINITY) return {0.f, 0.f, -INFINITY};
    const float er = expf(lr - mx), es = expf(ls - mx);  // exp(-inf) = 0 for an empty side
    const float sum = er + es;
    return {er / sum, es / sum, mx + logf(sum)};
}

__global__ void __launch_bounds__(256) merge_inplace_vec4(float4* __restrict__ O_r,
                                                          float* __restrict__ lse_r,
                                                          const float4* __restrict__ O_s,
                                                          const float* __restrict__ lse_s,
                                                          int64_t rows, int64_t vecs_per_row) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= rows * vecs_per_row) return;
    const int64_t row = t / vecs_per_row;
    const float lr = lse_r[row], ls = __ldcs(lse_s + row);
    const Weights w = merge_weights(lr, ls);
    const float4 a = O_r[t], b = __ldcs(O_s + t);
    O_r[t] = make_float4(w.wr * a.x + w.ws * b.x, w.wr * a.y + w.ws * b.y, w.wr * a.z + w.ws * b.z,
                         w.wr * a.w + w.ws * b.w);
    // lse_r is updated by merge_lse, launched after this kernel: every thread of a row must read
    // the old value first, and a row may span several blocks.
}

__global__ void merge_lse(float* __restrict__ lse_r, const float* __restrict__ lse_s, int64_t rows) {
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    lse_r[r] = merge_weights(lse_r[r], lse_s[r]).lse;
}

__global__ void __launch_bounds__(256) merge_inplace_scalar(float* __restrict__ O_r,
                                                            const float* __restrict__ lse_r,
                                                            const float* __restrict__ O_s,
                                                            const float* __restrict__ lse_s,
                                                            int64_t rows, int64_t D) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= rows * D) return;
    const int64_t row = t / D;
    const Weights w = merge_weights(lse_r[row], lse_s[row]);
    O_r[t] = w.wr * O_r[t] + w.ws * O_s[t];
}

// Final merge: rows are shard-major (b, i, a, h); the result goes to natural position g(i, a).
// With O_s and lse_s null, the running result alone is converted and written (the last step of a
// ring whose partials were already merged).
template <typename T>
__device__ __forceinline__ void store4(T* p, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* p, float4 v) {
    *reinterpret_cast<float4*>(p) = v;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, float4 v) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&lo);
    u.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p) = u;
}

template <typename T, bool kVec>
__global__ void __launch_bounds__(256) merge_final(const float* __restrict__ O_r,
                                                   const float* __restrict__ lse_r,
                                                   const float* __restrict__ O_s,
                                                   const float* __restrict__ lse_s,
                                                   T* __restrict__ out, float* __restrict__ lse,
                                                   Layout L, int64_t B, int64_t H, int64_t D) {
    const int64_t per_row = kVec ? D / 4 : D;
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t rows = B * L.S * H;
    if (t >= rows * per_row) return;
    const int64_t row = t / per_row, c = t % per_row;
    const int64_t h = row % H;
    const int64_t r = row / H;  // (b * N + i) * S_loc + a
    const int64_t a = r % L.S_loc, bi = r / L.S_loc;
    const int64_t i = bi % L.N, b = bi / L.N;
    const int64_t g = global_position(L, i, a);
    // without a step partial (lse_s null) the running result is written as it is
    const Weights w = lse_s ? merge_weights(lse_r[row], __ldcs(lse_s + row)) : Weights{1.f, 0.f, lse_r[row]};
    T* dst = out + ((b * L.S + g) * H + h) * D;
    if (kVec) {
        const float4 x = reinterpret_cast<const float4*>(O_r)[t];
        const float4 y = lse_s ? __ldcs(reinterpret_cast<const float4*>(O_s) + t) : make_float4(0.f, 0.f, 0.f, 0.f);
        store4<T>(dst + 4 * c, make_float4(w.wr * x.x + w.ws * y.x, w.wr * x.y + w.ws * y.y,
                                           w.wr * x.z + w.ws * y.z, w.wr * x.w + w.ws * y.w));
    } else {
        const float x = w.wr * O_r[t] + (lse_s ? w.ws * O_s[t] : 0.f);
        if constexpr (sizeof(T) == 4) {
            dst[c] = x;
        } else {
            dst[c] = __float2bfloat16_rn(x);
        }
    }
    if (c == 0) lse[(b * H + h) * L.S + g] = w.lse;
}

}  // namespace

cudaError_t launch_merge_inplace(float* O_r, float* lse_r, const float* O_s, const float* lse_s,
                                 int64_t rows, int64_t D, cudaStream_t stream) {
    if (rows == 0) return cudaSuccess;
    if (D % 4 == 0) {
        const int64_t n = rows * (D / 4);
        merge_inplace_vec4<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(
            reinterpret_cast<float4*>(O_r), lse_r, reinterpret_cast<const float4*>(O_s), lse_s,
            rows, D / 4);
    } else {
        const int64_t n = rows * D;
        merge_inplace_scalar<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(O_r, lse_r, O_s,
                                                                              lse_s, rows, D);
    }
    merge_lse<<<(unsigned)((rows + 255) / 256), 256, 0, stream>>>(lse_r, lse_s, rows);
    return cudaGetLastError();
}

cudaError_t launch_merge_final(const float* O_r, const float* lse_r, const float* O_s,
                               const float* lse_s, void* out, float* lse, int dtype, int64_t B,
                               const Layout& L, int64_t H, int64_t D, cudaStream_t stream) {
    const int64_t rows = B * L.S * H;
    if (rows == 0) return cudaSuccess;
    const bool vec = (D % 4 == 0);
    const int64_t n = rows * (vec ? D / 4 : D);
    const unsigned grid = (unsigned)((n + 255) / 256);
    if (dtype == 0) {
        if (vec)
            merge_final<float, true><<<grid, 256, 0, stream>>>(O_r, lse_r, O_s, lse_s,
                                                               static_cast<float*>(out), lse, L, B, H, D);
        else
            merge_final<float, false><<<grid, 256, 0, stream>>>(O_r, lse_r, O_s, lse_s,
                                                                static_cast<float*>(out), lse, L, B, H, D);
    } else {
        if (vec)
            merge_final<__nv_bfloat16, true><<<grid, 256, 0, stream>>>(
                O_r, lse_r, O_s, lse_s, static_cast<__nv_bfloat16*>(out), lse, L, B, H, D);
        else
            merge_final<__nv_bfloat16, false><<<grid, 256, 0, stream>>>(
                O_r, lse_r, O_s, lse_s, static_cast<__nv_bfloat16*>(out), lse, L, B, H, D);
    }
    return cudaGetLastError();
}

}  // namespace ra
