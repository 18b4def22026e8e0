// norms.cu -- the largest query norm and the largest key norm of every (batch, head):
// qmax = max over tokens s of ||q[b, s, h, :]||_2, kmax likewise for k.
//
// The tensor-core forward kernel uses them to bound every score of a head before it sees them: by
// the Cauchy-Schwarz inequality q.k <= ||q|| ||k|| <= qmax * kmax.  When that bound lies within 2^32
// of a row's running max after its first key tile, no later tile can raise the max far enough to
// matter, and the kernel keeps the max fixed for the rest of the row: every later weight
// exp(s - m) stays below 2^32 (no overflow in fp32, no rescale of the accumulator), and the result
// is the same exact attention.  The online-softmax identities hold for any common reference m
// (troisinh.com "Ring Attention", "Tai sao no hoat dong"), so keeping m fixed changes nothing but
// rounding.
//
// HBM-bound: one read of q and of k (2 bytes per element each) and 2 * B * H floats written.  A half-warp takes one
// (token, head) row of D <= 128 elements (16-byte vectors, lane-contiguous), reduces the sum of
// squares with shuffles, and a block keeps one max per head in shared memory before one atomicMax
// per head.  Norms are non-negative, so the float bit patterns order like unsigned integers.
#include <cuda_bf16.h>

#include <algorithm>

#include "ra_internal.cuh"

namespace ra {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxHeadsPerBlock = (int)kKeyNormMaxHeads;  // shared-memory maxima of one block

__global__ void __launch_bounds__(kThreads) key_norm_max(const __nv_bfloat16* __restrict__ q,
                                                         const __nv_bfloat16* __restrict__ k,
                                                         unsigned* __restrict__ nmax, int64_t rows_per_batch,
                                                         int64_t H, int64_t D, int64_t rows_per_block) {
    const __nv_bfloat16* __restrict__ x = blockIdx.z ? k : q;  // grid.z: 0 queries, 1 keys
    unsigned* __restrict__ out = nmax + blockIdx.z * gridDim.y * H;
    __shared__ unsigned smax[kMaxHeadsPerBlock];
    for (int h = threadIdx.x; h < H; h += kThreads) smax[h] = 0u;
    __syncthreads();
    const int64_t b = blockIdx.y;
    const int64_t r0 = (int64_t)blockIdx.x * rows_per_block;
    const int64_t r1 = r0 + rows_per_block < rows_per_batch ? r0 + rows_per_block : rows_per_batch;
    const int half = threadIdx.x >> 4, lane16 = threadIdx.x & 15;
    const int vec_per_row = (int)(D / 8);  // 16-byte vectors of one (token, head) row
    // (token, head) rows of this block, two per warp per pass
    const int64_t pairs0 = r0 * H, pairs1 = r1 * H;
    const __nv_bfloat16* base = x + b * rows_per_batch * H * D;
    // every lane of a warp runs the same passes, so the shuffles always see the whole warp
    for (int64_t p0 = pairs0; p0 < pairs1; p0 += kThreads / 16) {
        const int64_t p = p0 + half;
        const bool live = p < pairs1;
        float ss = 0.f;
        for (int v = lane16; live && v < vec_per_row; v += 16) {
            const uint4 u = __ldcs(reinterpret_cast<const uint4*>(base + p * D) + v);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xffff0000u);
                ss = fmaf(lo, lo, ss);
                ss = fmaf(hi, hi, ss);
            }
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o, 16);
        if (live && lane16 == 0) atomicMax(&smax[p % H], __float_as_uint(sqrtf(ss)));
    }
    __syncthreads();
    for (int h = threadIdx.x; h < H; h += kThreads)
        if (smax[h]) atomicMax(&out[b * H + h], smax[h]);
}

}  // namespace

cudaError_t launch_norm_max(const void* q, const void* k, float* nmax, int64_t B, int64_t rows, int64_t H,
                            int64_t D, int sms, cudaStream_t stream) {
    if (!key_norm_max_applies(B, H, D)) return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(nmax, 0, (size_t)(2 * B * H) * sizeof(float), stream);
    if (e != cudaSuccess || B * rows == 0) return e;
    // about four blocks per SM over the whole tensor
    const int64_t blocks_per_batch = std::max<int64_t>(1, std::min<int64_t>(rows, (4 * (int64_t)sms + B - 1) / B));
    const int64_t rows_per_block = (rows + blocks_per_batch - 1) / blocks_per_batch;
    dim3 grid((unsigned)((rows + rows_per_block - 1) / rows_per_block), (unsigned)B, 2u);
    key_norm_max<<<grid, kThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(q),
                                                static_cast<const __nv_bfloat16*>(k),
                                                reinterpret_cast<unsigned*>(nmax), rows, H, D, rows_per_block);
    return cudaGetLastError();
}

cudaError_t preload_key_norm() {
    cudaFuncAttributes fa;
    return cudaFuncGetAttributes(&fa, key_norm_max);
}

}  // namespace ra
