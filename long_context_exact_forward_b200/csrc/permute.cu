// permute.cu -- gather tokens from natural order into shard-major order and back.
//
// Sequence sharding gives each device its own block of tokens (aiunderstanding.org "Sequence
// Parallelism and Ring Attention"; ultralytics.com "Ring Attention": the sequence is cut into N
// blocks, one per device).  On one GPU the shards are views of one buffer laid out
// [B, N, S_loc, H, D]; this kernel builds that buffer for the striped and zigzag layouts
// (contiguous needs no copy) and scatters results back.
//
// A token row is H*D contiguous elements.  One warp moves one row with 16-byte vectors, so every
// load and store is a fully used 512-byte warp transaction; the kernel is HBM-bound:
// algorithmic bytes = 2 * B * S * H * D * esize per tensor (read once, write once).
#include "ra_internal.cuh"

namespace ra {
namespace {

constexpr int kRowsPerBlock = 8;  // 8 warps, one row each

constexpr int kMaxTensors = 4;  // tensors moved by one launch (grid.y)

struct PermuteArgs {
    const void* src[kMaxTensors];
    void* dst[kMaxTensors];
};

// Vector path: row bytes are a multiple of 16.
__global__ void __launch_bounds__(256) permute_rows_vec16(PermuteArgs args, int64_t rows_total,
                                                          Layout L, int64_t row_vecs, int inverse) {
    const int tensor = blockIdx.y;
    const int64_t r = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
    if (r >= rows_total) return;
    // r is a shard-major row: r = (b * N + i) * S_loc + a
    const int64_t a = r % L.S_loc;
    const int64_t bi = r / L.S_loc;
    const int64_t i = bi % L.N, b = bi / L.N;
    const int64_t g = b * L.S + global_position(L, i, a);  // natural row
    const int64_t src_row = inverse ? r : g, dst_row = inverse ? g : r;
    const uint4* __restrict__ s = static_cast<const uint4*>(args.src[tensor]) + src_row * row_vecs;
    uint4* __restrict__ d = static_cast<uint4*>(args.dst[tensor]) + dst_row * row_vecs;
    for (int64_t c = threadIdx.x & 31; c < row_vecs; c += 32) d[c] = __ldcs(s + c);
}

// Element path for rows that are not a multiple of 16 bytes.
template <typename T>
__global__ void __launch_bounds__(256) permute_rows_elem(PermuteArgs args, int64_t rows_total,
                                                         Layout L, int64_t row_elems, int inverse) {
    const int tensor = blockIdx.y;
    const int64_t r = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
    if (r >= rows_total) return;
    const int64_t a = r % L.S_loc;
    const int64_t bi = r / L.S_loc;
    const int64_t i = bi % L.N, b = bi / L.N;
    const int64_t g = b * L.S + global_position(L, i, a);
    const int64_t src_row = inverse ? r : g, dst_row = inverse ? g : r;
    const T* s = static_cast<const T*>(args.src[tensor]) + src_row * row_elems;
    T* d = static_cast<T*>(args.dst[tensor]) + dst_row * row_elems;
    for (int64_t c = threadIdx.x & 31; c < row_elems; c += 32) d[c] = s[c];
}

}  // namespace

cudaError_t launch_permute(const void* const* src, void* const* dst, int n_tensors, int64_t B,
                           const Layout& L, int64_t H, int64_t D, int esize, bool inverse,
                           cudaStream_t stream) {
    if (n_tensors < 1 || n_tensors > kMaxTensors) return cudaErrorInvalidValue;
    PermuteArgs args{};
    for (int t = 0; t < n_tensors; ++t) {
        args.src[t] = src[t];
        args.dst[t] = dst[t];
    }
    const int64_t rows = B * L.S;
    if (rows == 0) return cudaSuccess;
    dim3 grid((unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock), (unsigned)n_tensors);
    const int64_t row_bytes = H * D * esize;
    if (row_bytes % 16 == 0) {
        permute_rows_vec16<<<grid, 256, 0, stream>>>(args, rows, L, row_bytes / 16, inverse);
    } else if (esize == 4) {
        permute_rows_elem<float><<<grid, 256, 0, stream>>>(args, rows, L, H * D, inverse);
    } else {
        permute_rows_elem<unsigned short><<<grid, 256, 0, stream>>>(args, rows, L, H * D, inverse);
    }
    return cudaGetLastError();
}

cudaError_t preload_permute() {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, permute_rows_vec16);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, permute_rows_elem<float>);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, permute_rows_elem<unsigned short>);
    return e;
}

}  // namespace ra
