// rope.cu -- ra_rope: rotary position embedding with global token positions.
//
// When K/V blocks travel round the ring, each token must still be rotated by the angle m theta of
// its own position m (troisinh.com "Ring Attention", "RoPE va Position Embedding").  The library
// takes q and k in natural token order, so the position of the token at natural index g is g (plus
// a caller offset, for a sequence that continues an earlier one), whatever the ring layout.  The
// pair (x[2p], x[2p+1]) is rotated by m * theta_p, theta_p = base^(-2p/D).
//
// HBM bound.  The angle m * theta_p is formed and reduced to [-pi, pi] in fp64 (m reaches 2^31,
// where an fp32 angle would lose whole radians), once per token and pair, then sincosf on the
// reduced angle; the rotation itself is fp32.
#include <cuda_bf16.h>

#include <cmath>

#include "ra.h"
#include "ra_internal.cuh"

namespace ra {
namespace {

constexpr int kMaxPairs = 128;  // D <= 256

struct RopeArgs {
    double theta[kMaxPairs];  // base^(-2p/D)
    int64_t rows;             // B * S * H
    int64_t S, H;
    int pairs;                // D / 2
    int64_t pos_offset;
};

template <typename T>
__device__ __forceinline__ float ld_f(const T* p, int64_t i);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p, int64_t i) { return p[i]; }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) { return __bfloat162float(p[i]); }
template <typename T>
__device__ __forceinline__ void st_f(T* p, int64_t i, float x);
template <>
__device__ __forceinline__ void st_f<float>(float* p, int64_t i, float x) { p[i] = x; }
template <>
__device__ __forceinline__ void st_f<__nv_bfloat16>(__nv_bfloat16* p, int64_t i, float x) { p[i] = __float2bfloat16_rn(x); }

constexpr int kTokensPerStep = 4;  // tokens a CTA rotates between two barriers

// 8 consecutive elements (4 pairs) at x + e, as fp32; e is a multiple of 8 and the row is 16-byte
// aligned (the vector path requires D % 8 == 0 and 16-byte aligned tensors).
__device__ __forceinline__ void ld8(const float* x, int64_t e, float (&v)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(x + e), b = *reinterpret_cast<const float4*>(x + e + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void ld8(const __nv_bfloat16* x, int64_t e, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(x + e);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void st8(float* y, int64_t e, const float (&v)[8]) {
    *reinterpret_cast<float4*>(y + e) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(y + e + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void st8(__nv_bfloat16* y, int64_t e, const float (&v)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(y + e) = make_uint4(w[0], w[1], w[2], w[3]);
}

// Grid-stride over groups of kTokensPerStep tokens: the D / 2 angles of each token's position are
// reduced in fp64 and turned into cos / sin once, in shared memory, then every head of those tokens
// is rotated with them, consecutive threads on consecutive pairs (4 pairs per thread on the vector
// path, 1 otherwise).
template <typename T, bool kVec>
__global__ void __launch_bounds__(256) rope_kernel(const T* x, T* y, const RopeArgs A) {  // x may equal y
    __shared__ float cs[kTokensPerStep][kMaxPairs], sn[kTokensPerStep][kMaxPairs];
    const double two_pi = 6.283185307179586476925286766559;
    const double inv_two_pi = 0.15915494309189533576888376337251;
    const int64_t n_tokens = A.rows / A.H;
    const int token_pairs = (int)A.H * A.pairs;
    for (int64_t t0 = (int64_t)blockIdx.x * kTokensPerStep; t0 < n_tokens; t0 += (int64_t)gridDim.x * kTokensPerStep) {
        const int nt = n_tokens - t0 < kTokensPerStep ? (int)(n_tokens - t0) : kTokensPerStep;
        for (int u = threadIdx.x; u < nt * A.pairs; u += blockDim.x) {
            const int k = u / A.pairs, p = u % A.pairs;
            const int64_t g = (t0 + k) % A.S;
            const double angle = (double)(g + A.pos_offset) * A.theta[p];
            sincosf((float)(angle - two_pi * rint(angle * inv_two_pi)), &sn[k][p], &cs[k][p]);
        }
        __syncthreads();
        const int per = kVec ? 4 : 1;  // pairs per thread step
        const int steps = nt * token_pairs / per;
        for (int t = threadIdx.x; t < steps; t += blockDim.x) {
            const int pair0 = t * per;  // pair index within the group of tokens
            const int k = pair0 / token_pairs;
            const int p0 = (pair0 - k * token_pairs) % A.pairs;
            const int64_t e = 2 * (t0 * token_pairs + pair0);
            if (kVec) {
                float v[8];
                ld8(x, e, v);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float c = cs[k][p0 + i], s = sn[k][p0 + i], x0 = v[2 * i], x1 = v[2 * i + 1];
                    v[2 * i] = x0 * c - x1 * s;
                    v[2 * i + 1] = x0 * s + x1 * c;
                }
                st8(y, e, v);
            } else {
                const float x0 = ld_f(x, e), x1 = ld_f(x, e + 1);
                st_f(y, e, x0 * cs[k][p0] - x1 * sn[k][p0]);
                st_f(y, e + 1, x0 * sn[k][p0] + x1 * cs[k][p0]);
            }
        }
        __syncthreads();  // the next group overwrites cs, sn
    }
}

}  // namespace
}  // namespace ra

extern "C" int ra_rope(const void* x, void* y, int64_t B, int64_t S, int64_t H, int64_t D, int64_t pos_offset,
                       double base, int dtype, void* stream_handle) {
    if (!x || !y || B < 0 || S < 0 || H < 0 || D <= 0 || (D & 1) || D > 2 * ra::kMaxPairs) return RA_ERR_INVALID_ARG;
    if (!(base > 0.0) || pos_offset < 0) return RA_ERR_INVALID_ARG;
    if (dtype != RA_DTYPE_FP32 && dtype != RA_DTYPE_BF16) return RA_ERR_INVALID_ARG;
    const uintptr_t esize = dtype == RA_DTYPE_FP32 ? 4 : 2;
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) % esize) return RA_ERR_ALIGN;
    if (B * S * H == 0) return RA_OK;
    if (H * D > (int64_t(1) << 28)) return RA_ERR_SHAPE;  // per-token element counts are int in the kernel
    ra::RopeArgs A{};
    A.pairs = (int)(D / 2);
    for (int p = 0; p < A.pairs; ++p) A.theta[p] = std::pow(base, -2.0 * p / (double)D);
    A.rows = B * S * H;
    A.S = S;
    A.H = H;
    A.pos_offset = pos_offset;
    const int64_t groups = (B * S + ra::kTokensPerStep - 1) / ra::kTokensPerStep;
    const int blocks = (int)(groups < 148 * 16 ? groups : 148 * 16);
    const bool vec = D % 8 == 0 && ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & 15u) == 0;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_handle);
    if (dtype == RA_DTYPE_FP32) {
        auto xf = static_cast<const float*>(x);
        auto yf = static_cast<float*>(y);
        if (vec) ra::rope_kernel<float, true><<<blocks, 256, 0, stream>>>(xf, yf, A);
        else ra::rope_kernel<float, false><<<blocks, 256, 0, stream>>>(xf, yf, A);
    } else {
        auto xb = static_cast<const __nv_bfloat16*>(x);
        auto yb = static_cast<__nv_bfloat16*>(y);
        if (vec) ra::rope_kernel<__nv_bfloat16, true><<<blocks, 256, 0, stream>>>(xb, yb, A);
        else ra::rope_kernel<__nv_bfloat16, false><<<blocks, 256, 0, stream>>>(xb, yb, A);
    }
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return ra::host_cuda_fail(e, "rope launch");
    return RA_OK;
}
