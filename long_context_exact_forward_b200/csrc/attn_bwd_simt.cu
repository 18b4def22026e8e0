// attn_bwd_simt.cu -- ra_backward: gradients of ring attention on CUDA cores with fp32 arithmetic.
//
// What it computes.  For an upstream gradient dO of out = softmax(Q K^T / sqrt(D)) V (causal mask on
// original positions when asked), the gradients dQ, dK, dV.  The forward statistics are not stored:
// every block recomputes its scores and takes the softmax weights from the saved lse
// (troisinh.com "Ring Attention", "Blockwise Backward": the backward pass recomputes the attention
// statistics, FlashAttention style, each device only on the K/V block visiting it).  Per query row r
// and key c, with Delta_r = dO_r . O_r (O as returned by the forward pass):
//     P_rc  = exp(q_r . k_c / sqrt(D) - lse_r)
//     dP_rc = dO_r . v_c
//     dS_rc = P_rc (dP_rc - Delta_r)
//     dQ_r  = sum_c dS_rc k_c / sqrt(D),  dK_c = sum_r dS_rc q_r / sqrt(D),  dV_c = sum_r P_rc dO_r
//
// Ring order.  dQ of query shard i is accumulated over the key blocks j = (i - s) mod N, s = 0..N-1,
// as in the forward pass.  dK and dV of key block j travel with the block in the distributed form:
// at step s the block visits query shard i = (j + s) mod N, and that is the order here.
//
// Entry points: ra_backward / ra_backward_ex (kernel choice).  bf16 inputs with D in {64, 128} go to
// the tensor-core kernels of attn_bwd_tc.cu; everything else (fp32, other head dims) to the
// CUDA-core kernels below.
//
// Kernels (one CTA of 256 threads per 64-row query tile or 64-key tile, fp32 arithmetic, inputs
// gathered from natural order through the layout map):
//   bwd_delta_kernel  Delta = rowsum(dO * O), one warp per row                        (HBM bound)
//   bwd_dq_kernel     per query tile: S and dP blocks 4 x 4 per thread, dS to shared memory,
//                     dQ block 4 x D/16 per thread (the forward SIMT kernel's tiling)
//   bwd_dkv_kernel    per key tile: S and dP blocks, P and dS to shared memory, dV and dK blocks
//                     4 keys x D/16 per thread
#include <cuda_bf16.h>

#include <cmath>

#include "ra.h"
#include "ra_internal.cuh"

namespace ra {
namespace {

constexpr int kT = 64;         // query rows per tile and keys per tile
constexpr int kThreads = 256;  // 16 x 16 thread grid

template <typename T>
__device__ __forceinline__ float ld_f(const T* p, int64_t i);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p, int64_t i) { return p[i]; }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
    return __bfloat162float(p[i]);
}
template <typename T>
__device__ __forceinline__ void st_f(T* p, int64_t i, float x);
template <>
__device__ __forceinline__ void st_f<float>(float* p, int64_t i, float x) { p[i] = x; }
template <>
__device__ __forceinline__ void st_f<__nv_bfloat16>(__nv_bfloat16* p, int64_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

// Delta[b, h, g] = sum_d dO[b, g, h, d] * O[b, g, h, d]; rows are (b, g, h) in [B, S, H, D] order.
template <typename T>
__global__ void bwd_delta_kernel(const T* __restrict__ o, const T* __restrict__ dout, float* __restrict__ delta,
                                 int64_t B, int64_t S, int64_t H, int64_t D) {
    const int lane = threadIdx.x & 31;
    const int64_t n_rows = B * S * H;
    for (int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < n_rows;
         row += ((int64_t)gridDim.x * blockDim.x) >> 5) {
        float acc = 0.f;
        for (int64_t d = lane; d < D; d += 32) acc = fmaf(ld_f(dout, row * D + d), ld_f(o, row * D + d), acc);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) {
            const int64_t h = row % H, bg = row / H, g = bg % S, b = bg / S;
            delta[(b * H + h) * S + g] = acc;
        }
    }
}

// `kT` rows of shard `shard` from local row a0, transposed into dst[d * kT + r] as fp32 (zero past
// the shard end and for d >= D); thread t takes row t % kT and 4 consecutive columns at a time.
template <typename T, int kDMax>
__device__ void load_t(float* dst, const T* __restrict__ src, const Layout& L, int64_t b, int64_t h,
                       int64_t H, int64_t D, int64_t shard, int64_t a0) {
    const int r = threadIdx.x % kT;
    const int64_t a = a0 + r;
    const T* row = nullptr;
    if (a < L.S_loc) row = src + ((b * L.S + global_position(L, shard, a)) * H + h) * D;
    for (int d4 = 4 * (threadIdx.x / kT); d4 < kDMax; d4 += 4 * (kThreads / kT)) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int d = d4 + e;
            dst[d * kT + r] = (row && d < D) ? ld_f(row, d) : 0.f;
        }
    }
}

// The same rows row-major: dst[r * kDMax + d].
template <typename T, int kDMax>
__device__ void load_r(float* dst, const T* __restrict__ src, const Layout& L, int64_t b, int64_t h,
                       int64_t H, int64_t D, int64_t shard, int64_t a0) {
    for (int idx = threadIdx.x; idx < kT * kDMax; idx += kThreads) {
        const int r = idx / kDMax, d = idx % kDMax;
        const int64_t a = a0 + r;
        float x = 0.f;
        if (a < L.S_loc && d < D) x = ld_f(src, ((b * L.S + global_position(L, shard, a)) * H + h) * D + d);
        dst[idx] = x;
    }
}

// 4 x 4 block of A B^T over the head dim from transposed tiles At, Bt [kDMax][kT]: rows 4ty.., cols 4tx..
__device__ __forceinline__ void block_4x4(float (&acc)[4][4], const float* At, const float* Bt, int64_t D,
                                          int ty, int tx) {
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
#pragma unroll 4
    for (int d = 0; d < D; ++d) {
        const float4 a = *reinterpret_cast<const float4*>(At + d * kT + 4 * ty);
        const float4 b = *reinterpret_cast<const float4*>(Bt + d * kT + 4 * tx);
        const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
    }
}

// Key-major [kT keys][kT rows] store with the 4-row groups XOR-swizzled by (key / 4) mod 16, so the
// writes of one key by 16 threads and the float4 reads of 4 rows are free of bank conflicts.
__device__ __forceinline__ int swz(int key, int row4) {
    return key * kT + (((row4 >> 2) ^ ((key >> 2) & 15)) << 2);
}

struct BwdArgs {
    Layout L;
    int64_t B, H, D;
    int causal;
    float scale;
    const float* lse;    // [B, H, S] natural
    const float* delta;  // [B, H, S] natural
};

// dQ of one 64-row query tile (b, h, shard i), over the key blocks in ring order.
template <typename T, int kDMax>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const T* __restrict__ dout, T* __restrict__ dq, BwdArgs A) {
    constexpr int kOC = kDMax / 16;
    extern __shared__ __align__(16) float smem[];
    float* Qt = smem;                // [kDMax][kT]
    float* dOt = Qt + kDMax * kT;    // [kDMax][kT]
    float* Kt = dOt + kDMax * kT;    // [kDMax][kT]
    float* Vt = Kt + kDMax * kT;     // [kDMax][kT]
    float* Ks = Vt + kDMax * kT;     // [kT][kDMax]
    float* dSt = Ks + kT * kDMax;    // [kT keys][kT rows], swizzled
    const Layout L = A.L;
    const int64_t D = A.D, H = A.H, S = L.S;
    const int64_t i = L.N - 1 - blockIdx.y;  // heaviest shards first
    const int64_t b = blockIdx.z / H, h = blockIdx.z % H;
    const int64_t a0 = (int64_t)blockIdx.x * kT;
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
    const int64_t a_last = (a0 + kT - 1 < L.S_loc - 1) ? a0 + kT - 1 : L.S_loc - 1;

    load_t<T, kDMax>(Qt, q, L, b, h, H, D, i, a0);
    load_t<T, kDMax>(dOt, dout, L, b, h, H, D, i, a0);
    float lse_r[4], del_r[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int64_t a = a0 + 4 * ty + r;
        const int64_t g = a < L.S_loc ? global_position(L, i, a) : 0;
        lse_r[r] = a < L.S_loc ? A.lse[(b * H + h) * S + g] : 0.f;
        del_r[r] = a < L.S_loc ? A.delta[(b * H + h) * S + g] : 0.f;
    }
    float acc[4][kOC];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < kOC; ++c) acc[r][c] = 0.f;

    for (int s = 0; s < L.N; ++s) {
        const int64_t j = ring_block(i, s, L.N);
        int64_t n_vis[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int64_t a = a0 + 4 * ty + r;
            n_vis[r] = a < L.S_loc ? visible_keys(L, A.causal, i, a, j) : 0;
        }
        const int64_t n_vis_cta = visible_keys(L, A.causal, i, a_last, j);
        for (int64_t c0 = 0; c0 < n_vis_cta; c0 += kT) {
            __syncthreads();  // previous tile consumed (and the query tiles loaded on the first pass)
            load_t<T, kDMax>(Kt, k, L, b, h, H, D, j, c0);
            load_t<T, kDMax>(Vt, v, L, b, h, H, D, j, c0);
            load_r<T, kDMax>(Ks, k, L, b, h, H, D, j, c0);
            __syncthreads();
            float sc[4][4], dp[4][4];
            block_4x4(sc, Qt, Kt, D, ty, tx);
            block_4x4(dp, dOt, Vt, D, ty, tx);
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const bool vis = (c0 + 4 * tx + c) < n_vis[r];
                    const float p = vis ? expf(sc[r][c] * A.scale - lse_r[r]) : 0.f;
                    sc[r][c] = p * (dp[r][c] - del_r[r]);  // dS
                }
#pragma unroll
            for (int c = 0; c < 4; ++c)
                *reinterpret_cast<float4*>(dSt + swz(4 * tx + c, 4 * ty)) =
                    make_float4(sc[0][c], sc[1][c], sc[2][c], sc[3][c]);
            __syncthreads();
#pragma unroll 2
            for (int key = 0; key < kT; ++key) {
                const float4 sa = *reinterpret_cast<const float4*>(dSt + swz(key, 4 * ty));
                const float sv[4] = {sa.x, sa.y, sa.z, sa.w};
#pragma unroll
                for (int c4 = 0; c4 < kOC / 4; ++c4) {
                    const float4 kb = *reinterpret_cast<const float4*>(Ks + key * kDMax + 4 * tx + 64 * c4);
                    const float kv[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
                    for (int r = 0; r < 4; ++r)
#pragma unroll
                        for (int c = 0; c < 4; ++c) acc[r][4 * c4 + c] = fmaf(sv[r], kv[c], acc[r][4 * c4 + c]);
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int64_t a = a0 + 4 * ty + r;
        if (a >= L.S_loc) continue;
        const int64_t base = ((b * S + global_position(L, i, a)) * H + h) * D;
#pragma unroll
        for (int c = 0; c < kOC; ++c) {
            const int d = 4 * tx + 64 * (c / 4) + c % 4;
            if (d < D) st_f(dq, base + d, acc[r][c] * A.scale);
        }
    }
}

// dK and dV of one 64-key tile (b, h, key shard j), over the query shards i = (j + s) mod N.
template <typename T, int kDMax>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkv_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   const T* __restrict__ dout, T* __restrict__ dk, T* __restrict__ dv, BwdArgs A) {
    constexpr int kOC = kDMax / 16;
    extern __shared__ __align__(16) float smem[];
    float* Kt = smem;                // [kDMax][kT] keys of this CTA
    float* Vt = Kt + kDMax * kT;     // [kDMax][kT]
    float* Qt = Vt + kDMax * kT;     // [kDMax][kT] rows of the current query tile
    float* dOt = Qt + kDMax * kT;    // [kDMax][kT]
    float* Qs = dOt + kDMax * kT;    // [kT][kDMax]
    float* dOs = Qs + kT * kDMax;    // [kT][kDMax]
    float* Pt = dOs + kT * kDMax;    // [kT keys][kT rows], swizzled
    float* dSt = Pt + kT * kT;       // [kT keys][kT rows], swizzled
    const Layout L = A.L;
    const int64_t D = A.D, H = A.H, S = L.S;
    const int64_t j = blockIdx.y;
    const int64_t b = blockIdx.z / H, h = blockIdx.z % H;
    const int64_t c0 = (int64_t)blockIdx.x * kT;  // first local key of this tile
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;

    load_t<T, kDMax>(Kt, k, L, b, h, H, D, j, c0);
    load_t<T, kDMax>(Vt, v, L, b, h, H, D, j, c0);
    float dk_acc[4][kOC], dv_acc[4][kOC];  // keys 4ty + r, columns 4tx + 64 (c / 4) + c % 4
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < kOC; ++c) dk_acc[r][c] = dv_acc[r][c] = 0.f;

    for (int s = 0; s < L.N; ++s) {
        const int64_t i = (j + s) % L.N;
        for (int64_t a0 = 0; a0 < L.S_loc; a0 += kT) {
            const int64_t a_last = (a0 + kT - 1 < L.S_loc - 1) ? a0 + kT - 1 : L.S_loc - 1;
            // the tile's widest row sees keys [0, n); nothing to do unless n reaches this key tile
            if (visible_keys(L, A.causal, i, a_last, j) <= c0) continue;
            __syncthreads();  // previous query tile consumed (and K, V loaded on the first pass)
            load_t<T, kDMax>(Qt, q, L, b, h, H, D, i, a0);
            load_t<T, kDMax>(dOt, dout, L, b, h, H, D, i, a0);
            load_r<T, kDMax>(Qs, q, L, b, h, H, D, i, a0);
            load_r<T, kDMax>(dOs, dout, L, b, h, H, D, i, a0);
            __syncthreads();
            float sc[4][4], dp[4][4];  // rows 4ty + r, keys 4tx + c
            block_4x4(sc, Qt, Kt, D, ty, tx);
            block_4x4(dp, dOt, Vt, D, ty, tx);
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int64_t a = a0 + 4 * ty + r;
                int64_t n_vis = 0;
                float lse = 0.f, del = 0.f;
                if (a < L.S_loc) {
                    n_vis = visible_keys(L, A.causal, i, a, j);
                    const int64_t g = global_position(L, i, a);
                    lse = A.lse[(b * H + h) * S + g];
                    del = A.delta[(b * H + h) * S + g];
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const bool vis = (c0 + 4 * tx + c) < n_vis;
                    const float p = vis ? expf(sc[r][c] * A.scale - lse) : 0.f;
                    sc[r][c] = p;
                    dp[r][c] = p * (dp[r][c] - del);  // dS
                }
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                *reinterpret_cast<float4*>(Pt + swz(4 * tx + c, 4 * ty)) =
                    make_float4(sc[0][c], sc[1][c], sc[2][c], sc[3][c]);
                *reinterpret_cast<float4*>(dSt + swz(4 * tx + c, 4 * ty)) =
                    make_float4(dp[0][c], dp[1][c], dp[2][c], dp[3][c]);
            }
            __syncthreads();
            // dV_c += sum_r P_rc dO_r,  dK_c += sum_r dS_rc q_r  for keys c = 4ty + kk
#pragma unroll 1
            for (int r4 = 0; r4 < kT; r4 += 4) {
                float pv[4][4], sv[4][4];  // [key kk][row r4 + e]
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const float4 p4 = *reinterpret_cast<const float4*>(Pt + swz(4 * ty + kk, r4));
                    const float4 s4 = *reinterpret_cast<const float4*>(dSt + swz(4 * ty + kk, r4));
                    pv[kk][0] = p4.x; pv[kk][1] = p4.y; pv[kk][2] = p4.z; pv[kk][3] = p4.w;
                    sv[kk][0] = s4.x; sv[kk][1] = s4.y; sv[kk][2] = s4.z; sv[kk][3] = s4.w;
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = r4 + e;
#pragma unroll
                    for (int c4 = 0; c4 < kOC / 4; ++c4) {
                        const float4 o4 = *reinterpret_cast<const float4*>(dOs + r * kDMax + 4 * tx + 64 * c4);
                        const float4 q4 = *reinterpret_cast<const float4*>(Qs + r * kDMax + 4 * tx + 64 * c4);
                        const float ov[4] = {o4.x, o4.y, o4.z, o4.w}, qv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                dv_acc[kk][4 * c4 + c] = fmaf(pv[kk][e], ov[c], dv_acc[kk][4 * c4 + c]);
                                dk_acc[kk][4 * c4 + c] = fmaf(sv[kk][e], qv[c], dk_acc[kk][4 * c4 + c]);
                            }
                    }
                }
            }
        }
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        const int64_t c = c0 + 4 * ty + kk;
        if (c >= L.S_loc) continue;
        const int64_t base = ((b * S + global_position(L, j, c)) * H + h) * D;
#pragma unroll
        for (int cc = 0; cc < kOC; ++cc) {
            const int d = 4 * tx + 64 * (cc / 4) + cc % 4;
            if (d < D) {
                st_f(dk, base + d, dk_acc[kk][cc] * A.scale);
                st_f(dv, base + d, dv_acc[kk][cc]);
            }
        }
    }
}

template <typename T, int kDMax>
cudaError_t launch_grads(const void* q, const void* k, const void* v, const void* dout, void* dq, void* dk,
                         void* dv, const BwdArgs& A, cudaStream_t stream) {
    const size_t smem_dq = sizeof(float) * (5 * (size_t)kDMax * kT + (size_t)kT * kT);
    const size_t smem_dkv = sizeof(float) * (6 * (size_t)kDMax * kT + 2 * (size_t)kT * kT);
    auto kq = bwd_dq_kernel<T, kDMax>;
    auto kkv = bwd_dkv_kernel<T, kDMax>;
    cudaError_t e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_dq);
    if (e != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_dkv)) != cudaSuccess)
        return e;
    const dim3 grid((unsigned)((A.L.S_loc + kT - 1) / kT), (unsigned)A.L.N, (unsigned)(A.B * A.H));
    kq<<<grid, kThreads, smem_dq, stream>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                            static_cast<const T*>(v), static_cast<const T*>(dout),
                                            static_cast<T*>(dq), A);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    kkv<<<grid, kThreads, smem_dkv, stream>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                              static_cast<const T*>(v), static_cast<const T*>(dout),
                                              static_cast<T*>(dk), static_cast<T*>(dv), A);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_delta(const void* out, const void* dout, float* delta, const BwdArgs& A, cudaStream_t stream) {
    const int64_t rows = A.B * A.L.S * A.H;
    const int blocks = (int)((rows + 7) / 8 < 4096 ? (rows + 7) / 8 : 4096);
    bwd_delta_kernel<T><<<blocks, 256, 0, stream>>>(static_cast<const T*>(out), static_cast<const T*>(dout),
                                                     delta, A.B, A.L.S, A.H, A.D);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_grads_simt(const void* q, const void* k, const void* v, const void* dout, void* dq, void* dk,
                              void* dv, const BwdArgs& A, cudaStream_t stream) {
    if (A.D <= 64) return launch_grads<T, 64>(q, k, v, dout, dq, dk, dv, A, stream);
    return launch_grads<T, 128>(q, k, v, dout, dq, dk, dv, A, stream);
}

}  // namespace
}  // namespace ra

extern "C" int ra_backward_ex(const void* q, const void* k, const void* v, const void* out, const float* lse,
                              const void* dout, void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t S,
                              int64_t D, int n_ring, int causal, int layout, int dtype, int kernel,
                              uint64_t timeout_ns, int debug, void* stream_handle) {
    int rc = ra::host_check_shape(B, H, S, D, n_ring, layout, dtype);
    if (rc != RA_OK) return rc;
    if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv) return RA_ERR_INVALID_ARG;
    if (kernel < RA_KERNEL_AUTO || kernel > RA_KERNEL_SIMT) return RA_ERR_INVALID_ARG;
    const uintptr_t esize = dtype == RA_DTYPE_FP32 ? 4 : 2;
    const void* ptrs[8] = {q, k, v, out, dout, dq, dk, dv};
    bool a16 = true;
    for (const void* p : ptrs) {
        if (reinterpret_cast<uintptr_t>(p) % esize) return RA_ERR_ALIGN;
        a16 = a16 && (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
    }
    if (reinterpret_cast<uintptr_t>(lse) & 3u) return RA_ERR_ALIGN;
    if (D > 128) {
        ra::host_set_error("ra_backward: head dims above 128 are not supported");
        return RA_ERR_UNSUPPORTED;
    }
    int sms = 0;
    bool sm100 = false;
    int* status = nullptr;
    if ((rc = ra::host_device_facts(&sms, &sm100, &status)) != RA_OK) return rc;
    // tensor cores: bf16, D in {64, 128}, 16-byte alignment (zigzag through shard-major copies)
    const bool tc_ok = sm100 && dtype == RA_DTYPE_BF16 && (D == 64 || D == 128) && a16;
    if (kernel == RA_KERNEL_TC && !tc_ok) return RA_ERR_UNSUPPORTED;
    const bool use_tc = kernel != RA_KERNEL_SIMT && tc_ok;
    if (B * H * S == 0) return RA_OK;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_handle);
    // scratch: Delta, and for the tensor-core path with zigzag the shard-major q, k, v, dout
    const size_t delta_bytes = (sizeof(float) * (size_t)(B * H * S) + 255) / 256 * 256;
    const size_t copy_bytes = ((size_t)(B * S * H * D) * 2 + 255) / 256 * 256;
    const bool copies = use_tc && layout == RA_LAYOUT_ZIGZAG;
    uint8_t* scratch = nullptr;
    cudaError_t e = ra::scratch_alloc(reinterpret_cast<void**>(&scratch), delta_bytes + (copies ? 4 * copy_bytes : 0),
                                      stream);
    if (e != cudaSuccess) return ra::host_cuda_fail(e, "stream-ordered allocation (backward scratch)");
    float* delta = reinterpret_cast<float*>(scratch);
    ra::BwdArgs A{};
    A.L = ra::Layout{S, (int64_t)n_ring, S / n_ring, layout};
    A.B = B;
    A.H = H;
    A.D = D;
    A.causal = causal ? 1 : 0;
    A.scale = (float)(1.0 / std::sqrt((double)D));
    A.lse = lse;
    A.delta = delta;
    e = dtype == RA_DTYPE_FP32 ? ra::launch_delta<float>(out, dout, delta, A, stream)
                               : ra::launch_delta<__nv_bfloat16>(out, dout, delta, A, stream);
    if (e == cudaSuccess) {
        if (use_tc) {
            rc = ra::launch_backward_tc(q, k, v, dout, dq, dk, dv, lse, delta, B, H, A.L, D, causal, status,
                                        copies ? scratch + delta_bytes : nullptr, timeout_ns, debug, stream);
        } else {
            e = dtype == RA_DTYPE_FP32
                    ? ra::launch_grads_simt<float>(q, k, v, dout, dq, dk, dv, A, stream)
                    : ra::launch_grads_simt<__nv_bfloat16>(q, k, v, dout, dq, dk, dv, A, stream);
        }
    }
    const cudaError_t ef = cudaFreeAsync(scratch, stream);
    if (e != cudaSuccess) return ra::host_cuda_fail(e, "backward launch");
    if (rc != RA_OK) return rc;
    if (ef != cudaSuccess) return ra::host_cuda_fail(ef, "cudaFreeAsync(backward scratch)");
    return RA_OK;
}

extern "C" int ra_backward(const void* q, const void* k, const void* v, const void* out, const float* lse,
                           const void* dout, void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t S,
                           int64_t D, int n_ring, int causal, int layout, int dtype, void* stream_handle) {
    return ra_backward_ex(q, k, v, out, lse, dout, dq, dk, dv, B, H, S, D, n_ring, causal, layout, dtype,
                          RA_KERNEL_AUTO, 0, RA_DEBUG_NONE, stream_handle);
}
