// ra_internal.cuh -- parameter blocks and launcher declarations shared by the library's .cu files.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "layout.cuh"

namespace ra {

// Where an attention launch puts its result.
//   kOutFinal:   normalised O in the input dtype at natural position g(i, a), lse natural [B, H, S].
//   kOutPartial: normalised O_s fp32 and lse_s fp32, both in shard-major row order
//                row = ((b * N + i) * S_loc + a) * H + h  (O_s [rows, D], lse_s [rows]).
enum OutMode { kOutFinal = 0, kOutPartial = 1 };

struct AttnArgs {
    Layout L;
    int64_t B, H, D;
    int causal;
    int dtype;            // RA_DTYPE_*
    int s_begin, s_end;   // ring steps walked: s in [s_begin, s_end), block j = (i - s) mod N
    int out_mode;         // OutMode
    void* out;            // kOutFinal: [B, S, H, D] dtype; kOutPartial: fp32 [rows, D]
    float* lse;           // kOutFinal: [B, H, S]; kOutPartial: [rows]
    float scale;          // 1 / sqrt(D)
    // Packed sequences (B = 1): work item x indexes `seqs`, each entry {S_k, first token of
    // sequence k}; L then describes the whole packed axis (S = S_total) and every sequence is split
    // into L.N shards with L.kind.  kOutPartial rows are then natural packed rows (token * H + h).
    // Null: batch mode (item x = batch b).
    const int2* seqs;
    int varlen_striped;   // packed sequences with the striped layout inside each sequence
    // One ring step on one device's local buffers (kOutPartial only): q holds query shard
    // q_shard alone and k, v hold key block (q_shard - s_begin) mod N alone, each [B, S_loc, H, D]
    // in the layout's local order.  Masks and positions use the true shard indices; addresses use
    // shard 0 of a one-shard buffer, and the partial rows are local, ((b * S_loc + a) * H + h).
    int local;
    int q_shard;
    // Largest query and key norm per (b, h) -- batch mode -- or per h -- packed sequences -- over
    // every query row and key the launch reads (launch_norm_max).  Null: every tile computes its
    // row max (no freezing).
    const float* qmax;
    const float* kmax;
};

// norms.cu: nmax[b * H + h] = max over the `rows` tokens of ||q[b, token, h, :]||_2 and
// nmax[B * H + b * H + h] the same for k (bf16 q, k of [B, rows, H, D] in any token order, D a
// multiple of 8 up to 128); zeroes nmax first.  Needs H <= kKeyNormMaxHeads and B <= 65535
// (key_norm_max_applies).
constexpr int64_t kKeyNormMaxHeads = 2048;
inline bool key_norm_max_applies(int64_t B, int64_t H, int64_t D) {
    return H <= kKeyNormMaxHeads && B <= 65535 && D % 8 == 0 && D <= 128;
}
cudaError_t launch_norm_max(const void* q, const void* k, float* nmax, int64_t B, int64_t rows, int64_t H,
                            int64_t D, int sms, cudaStream_t stream);
// The pre-pass and the frozen row max it enables pay when each query row of a launch meets many keys
// (the row maxima saved grow with them, the pre-pass's read of q and k does not); `force` is
// RA_DEBUG_FROZEN_MAX.
constexpr int64_t kFrozenMaxMinKeys = 32768;
inline bool frozen_max_pays(int64_t keys_per_row, bool force) { return force || keys_per_row >= kFrozenMaxMinKeys; }

// pool.cu: stream-ordered scratch of the allocating entry points, from a library-owned pool per
// device that keeps freed memory reserved (the default pool when the stream is capturing).
cudaError_t scratch_alloc(void** ptr, size_t bytes, cudaStream_t stream);

// permute.cu
cudaError_t launch_permute(const void* const* src, void* const* dst, int n_tensors, int64_t B,
                           const Layout& L, int64_t H, int64_t D, int esize, bool inverse,
                           cudaStream_t stream);

// merge.cu: fold (O_s, lse_s) into (O_r, lse_r) in place, or (final) write the merged result
// to out (natural order, dtype) and lse natural [B, H, S]; launch_merge_final with O_s and lse_s
// null writes (O_r, lse_r) alone.
cudaError_t launch_merge_inplace(float* O_r, float* lse_r, const float* O_s, const float* lse_s,
                                 int64_t rows, int64_t D, cudaStream_t stream);
cudaError_t launch_merge_final(const float* O_r, const float* lse_r, const float* O_s,
                               const float* lse_s, void* out, float* lse, int dtype, int64_t B,
                               const Layout& L, int64_t H, int64_t D, cudaStream_t stream);

// attn_simt.cu: CUDA-core attention over natural-order q, k, v (any layout, D <= 256).
cudaError_t launch_attn_simt(const void* q, const void* k, const void* v, const AttnArgs& a,
                             cudaStream_t stream);
// Packed sequences (a.seqs set, B = 1, a.L.S the packed length): block x takes items[x] =
// {sequence, shard, 64-row query tile}, block z the head; kOutPartial rows are natural packed rows
// (token * H + h).
cudaError_t launch_attn_simt_packed(const void* q, const void* k, const void* v, const AttnArgs& a,
                                    const int4* items, int n_items, cudaStream_t stream);

// attn_tc.cu: tcgen05 attention over shard-major bf16 q, k, v (D in {64, 128}).
struct TcLaunch {
    CUtensorMap tm_q, tm_k, tm_v;
    const int4* items;     // work list (b, h, i, pair), heaviest first
    int n_items;
    int* counter;          // zero before the launch; CTAs take items in list order
    int grid;
    uint64_t timeout_ns;
    int debug;
    int* status;           // device status word, set to RA_ERR_DEVICE_TIMEOUT on a give-up
};
size_t tc_smem_bytes(int64_t D);

// Load the module code of every instantiation of a kernel family on the current device now
// (cudaFuncGetAttributes forces it), so that a later launch -- possibly inside a stream capture --
// never triggers lazy module loading.
cudaError_t preload_attn_tc();
cudaError_t preload_permute();
cudaError_t preload_key_norm();

// api.cu: host helpers shared by the entry points.
int host_check_shape(int64_t B, int64_t H, int64_t S, int64_t D, int n_ring, int layout, int dtype);
int host_device_facts(int* sms, bool* sm100, int** status);
int host_encode_qkv_map(CUtensorMap* map, const void* base, int64_t B, const Layout& L, int64_t H, int64_t D,
                        bool striped_natural);
int host_cuda_fail(cudaError_t e, const char* what);
void host_set_error(const char* msg);
cudaError_t launch_attn_tc(const AttnArgs& a, const TcLaunch& t, cudaStream_t stream);

// attn_bwd_tc.cu: the gradient kernels of ra_backward on the tensor cores (bf16, D in {64, 128});
// Delta must already be in `delta`; zigzag needs `shard_major` scratch of 4 tensors (see the
// definition).  timeout_ns = 0 means 2 s.  Returns an RA_* status.
int launch_backward_tc(const void* q, const void* k, const void* v, const void* dout, void* dq, void* dk,
                       void* dv, const float* lse, const float* delta, int64_t B, int64_t H, const Layout& L,
                       int64_t D, int causal, int* status, void* shard_major, uint64_t timeout_ns, int debug,
                       cudaStream_t stream);

}  // namespace ra
