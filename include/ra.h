/* ra.h -- C ABI of the Ring Attention exact-forward library for NVIDIA B200 (sm_100a).
 *
 * The operation (all five pages on Ring Attention agree on it): exact softmax attention
 *     out = softmax(Q K^T / sqrt(D)) V
 * over one long sequence whose tokens are split into n_ring shards.  Shard i keeps its queries;
 * at ring step s it meets the key/value block of shard j = (i - s) mod n_ring
 * (ultralytics.com "Ring Attention", section "how ring attention works"; jisaku.com
 * "Ring Attention", 処理フロー), scores it, and merges the partial result into running
 * statistics with the online-softmax identities m' = max(m_p, m_n),
 * l' = e^{m_p - m'} l_p + e^{m_n - m'} l_n (troisinh.com "Ring Attention", "Tai sao no hoat
 * dong"), so that after n_ring steps the result equals full attention.  Here the ring is
 * virtual: every shard lives on the one GPU, and "the next block arrives" means "the next key/value
 * tile address".
 *
 * Conventions shared by every entry point
 *   - Tensors q, k, v, out are [B, S, H, D] row-major (D fastest) in NATURAL token order, the
 *     (batch, seq, heads, head_dim) order of the ring-flash-attn example on jisaku.com.
 *   - lse is [B, H, S] fp32 in natural token order: the natural-log log-sum-exp of the scaled
 *     scores of each query row (lse = m + ln l).
 *   - scale = 1/sqrt(D) (the toy on ultralytics.com divides by dim**0.5).
 *   - causal != 0 masks key position g_k > query position g_q, on ORIGINAL token positions, the
 *     diagonal included, whatever the layout.
 *   - layout chooses which tokens shard i owns (S_loc = S / n_ring):
 *       RA_LAYOUT_CONTIGUOUS: local token a is global token i*S_loc + a (aiunderstanding.org:
 *                             each GPU owns a contiguous chunk);
 *       RA_LAYOUT_STRIPED:    local token a is global token a*n_ring + i (ultralytics.com: tokens
 *                             spread evenly over the sequence);
 *       RA_LAYOUT_ZIGZAG:     with C = S/(2 n_ring), local token a < C is global i*C + a and
 *                             a >= C is global (2 n_ring - 1 - i)*C + (a - C) (aiunderstanding.org
 *                             names zigzag; this two-chunk form is the reading adopted).
 *     The result does not depend on the layout (exactness); the layout only changes how the
 *     causal work is spread over shards and steps.
 *   - dtype: RA_DTYPE_FP32 (exact fp32 arithmetic) or RA_DTYPE_BF16 (bf16 inputs, fp32
 *     accumulation, bf16 output rounded to nearest even).  q, k, v, out share the dtype.
 *   - All device pointers are CUDA device addresses on the current device; the caller owns every
 *     buffer (including any workspace) and the library keeps no pointer past the call.
 *   - stream is a cudaStream_t (NULL = legacy default stream).  Work is enqueued on it and the
 *     call returns after enqueueing; nothing synchronises the device.
 *   - Return value: RA_OK (0) or a negative RA_ERR_* code; no exception crosses the ABI.
 *     Arguments are validated before anything is enqueued; a validation error enqueues nothing.
 */
#ifndef RA_H
#define RA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RA_API __attribute__((visibility("default")))
#else
#define RA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum ra_layout { RA_LAYOUT_CONTIGUOUS = 0, RA_LAYOUT_STRIPED = 1, RA_LAYOUT_ZIGZAG = 2 };
enum ra_dtype { RA_DTYPE_FP32 = 0, RA_DTYPE_BF16 = 1 };

/* Kernel path for ra_forward_ex.
 *   RA_VARIANT_FUSED:    one persistent launch walks all n_ring steps per query tile and keeps the
 *                        running (m, l, O) on chip (ultralytics.com toy loop structure).
 *   RA_VARIANT_PER_STEP: each attention launch covers ra_options.steps_per_launch ring steps (0 or
 *                        1: one step, the pages' per-device loop) and writes a partial (O_s,
 *                        lse_s); an HBM-bound merge launch folds it into the running (O, lse) with
 *                        the log-sum-exp form of the merge identities.
 *   RA_VARIANT_AUTO:     FUSED while one head's keys and values (2*S*D*esize bytes) fit in 96 MB of
 *                        the 126 MB L2; beyond that, PER_STEP with as many steps per launch as keep
 *                        a launch's keys and values per head within 96 MB (a fused item walks every
 *                        key/value block of its head, and CTAs running at their own pace then spread
 *                        over more blocks than L2 holds). */
enum ra_variant { RA_VARIANT_AUTO = 0, RA_VARIANT_FUSED = 1, RA_VARIANT_PER_STEP = 2 };

/* Kernel family for ra_forward_ex.
 *   RA_KERNEL_AUTO:    tcgen05 tensor-core kernel for bf16 with D in {64, 128}; SIMT otherwise.
 *   RA_KERNEL_TC:      require the tensor-core kernel (RA_ERR_UNSUPPORTED if it cannot apply).
 *   RA_KERNEL_SIMT:    CUDA-core kernel with fp32 arithmetic (any dtype, D <= 256). */
enum ra_kernel { RA_KERNEL_AUTO = 0, RA_KERNEL_TC = 1, RA_KERNEL_SIMT = 2 };

enum ra_status {
    RA_OK = 0,
    RA_ERR_INVALID_ARG = -1,     /* null pointer, bad enum, negative size */
    RA_ERR_SHAPE = -2,           /* S % n_ring != 0, zigzag S % (2 n_ring) != 0, D unsupported */
    RA_ERR_ALIGN = -3,           /* a tensor pointer is not 16-byte aligned */
    RA_ERR_UNSUPPORTED = -4,     /* no sm_100 device, or RA_KERNEL_TC cannot apply */
    RA_ERR_NO_WORKSPACE = -5,    /* caller workspace smaller than ra_workspace_size */
    RA_ERR_CUDA = -6,            /* a CUDA runtime/driver call failed (see ra_last_error_string) */
    RA_ERR_DEVICE_TIMEOUT = -7   /* a bounded in-kernel wait expired (from ra_get_device_status) */
};

/* Debug knobs (ra_options.debug).  RA_DEBUG_STALL_LOADS makes the tensor-core kernel's load warp
 * issue no copies, so every consumer wait runs out: a test of the bounded-wait give-up path.
 * RA_DEBUG_FROZEN_MAX runs the forward kernel's score-bound pre-pass (the largest query and key norm
 * per head) and lets it freeze row maxima at any size.  Without it that happens only when a launch's
 * query rows each meet at least 32768 keys (steps per launch x S/n_ring keys, or the mean sequence
 * length for packed sequences): below that, the pre-pass's read of q and k costs more than the row
 * maxima it saves.  Results are exact either way. */
enum ra_debug { RA_DEBUG_NONE = 0, RA_DEBUG_STALL_LOADS = 1, RA_DEBUG_FROZEN_MAX = 2 };

typedef struct ra_options {
    int variant;             /* enum ra_variant */
    int kernel;              /* enum ra_kernel */
    void* workspace;         /* device buffer of >= ra_workspace_size bytes, 256-byte aligned;
                                NULL: the call allocates stream-ordered on `stream` from a pool the
                                library keeps per device, and frees it the same way; freed memory
                                stays reserved in that pool for later calls until the process exits
                                (a stream being captured allocates from the default pool) */
    size_t workspace_bytes;
    uint64_t timeout_ns;     /* limit for every in-kernel wait; 0 = 2 s */
    int debug;               /* enum ra_debug */
    void* attn_events[2];    /* optional cudaEvent_t pair recorded on `stream` right before the
                                first and right after the last attention-kernel launch */
    int steps_per_launch;    /* RA_VARIANT_PER_STEP: ring steps per attention launch (0 = 1; values
                                above n_ring are n_ring); ignored by the other variants; >= 0 */
} ra_options;

/* ra_forward: exact attention as described above, with the defaults of ra_options (variant AUTO,
 * kernel AUTO, stream-ordered workspace).  q, k, v: [B, S, H, D] in dtype; out: [B, S, H, D] in
 * dtype; lse: [B, H, S] fp32.  Requires B, H >= 1, S >= 1, 1 <= D <= 256, n_ring >= 1 dividing S
 * (2 n_ring dividing S for zigzag), 16-byte aligned pointers. */
RA_API int ra_forward(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B,
               int64_t H, int64_t S, int64_t D, int n_ring, int causal, int layout, int dtype,
               void* stream);

/* ra_forward_ex: ra_forward with explicit options (opt may be NULL for the defaults). */
RA_API int ra_forward_ex(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B,
                  int64_t H, int64_t S, int64_t D, int n_ring, int causal, int layout, int dtype,
                  void* stream, const ra_options* opt);

/* ra_workspace_size: bytes of caller workspace ra_forward_ex needs for these arguments and the
 * given variant/kernel (enum values as in ra_options), written to *bytes.  Host only.  For
 * RA_VARIANT_PER_STEP the size covers every steps_per_launch; for RA_VARIANT_AUTO it is the size of
 * the path AUTO takes for these arguments.  (The pages define no such call; the kernel argument
 * and the status return with the size in *bytes let the size depend on the kernel choice and
 * report a bad shape the same way as the other calls.) */
RA_API int ra_workspace_size(int64_t B, int64_t H, int64_t S, int64_t D, int n_ring, int causal,
                      int layout, int dtype, int variant, int kernel, size_t* bytes);

/* ra_steps_per_launch (host only): the ring steps each attention launch of ra_forward_ex covers for
 * these arguments, variant and ra_options.steps_per_launch, written to *chunk (n_ring: one fused
 * launch; below n_ring: ceil(n_ring / *chunk) launches with a merge after each but the first). */
RA_API int ra_steps_per_launch(int64_t S, int64_t D, int n_ring, int layout, int dtype, int variant,
                               int steps_per_launch, int* chunk);

/* ra_permute: gather x [B, S, H, D] (natural order) into shard-major y [B, n_ring, S_loc, H, D]
 * where y[b, i, a] = x[b, g(i, a)] under `layout` (the per-shard chunks of the pages' sequence
 * sharding).  ra_unpermute scatters back: y[b, g(i, a)] = x[b, i, a].  x and y must not overlap.
 * dtype selects the element size (fp32 or bf16).  Asynchronous on `stream`. */
RA_API int ra_permute(const void* x, void* y, int64_t B, int64_t S, int64_t H, int64_t D, int n_ring,
               int layout, int dtype, void* stream);
RA_API int ra_unpermute(const void* x, void* y, int64_t B, int64_t S, int64_t H, int64_t D, int n_ring,
                 int layout, int dtype, void* stream);

/* ra_merge_partials: fold one ring step's partial result into the running result, in place:
 *   lse' = ln(e^{lse_run} + e^{lse_step}),  O' = e^{lse_run - lse'} O_run + e^{lse_step - lse'} O_step
 * (the merge identities in log-sum-exp form, with each O normalised by its own l).  O_* are fp32
 * [rows, D], lse_* fp32 [rows]; a row with lse = -inf is empty and contributes nothing.
 * Exported for callers that drive the per-step path themselves and for tests. */
RA_API int ra_merge_partials(float* O_run, float* lse_run, const float* O_step, const float* lse_step,
                      int64_t rows, int64_t D, void* stream);

/* ra_layout_positions (host only): pos[i * S_loc + a] = global position of local token a of
 * shard i under `layout`.  pos has S entries. */
RA_API int ra_layout_positions(int64_t S, int n_ring, int layout, int64_t* pos);

/* ra_plan_tiles (host only): classify every (query tile, key/value tile) pair of every
 * (shard i, ring step s) under the causal mask, as the block-skip scheduler does.
 * cls has n_ring * n_ring * nqt * nkt entries, nqt = nkt = ceil(S_loc / tile), at index
 * ((i * n_ring + s) * nqt + qt) * nkt + kt; values 0 = EMPTY (skipped), 1 = FULL (no mask),
 * 2 = PARTIAL (element mask).  Without causal every pair inside the shard is FULL, except a
 * ragged last key tile, which is PARTIAL. */
RA_API int ra_plan_tiles(int64_t S, int n_ring, int layout, int causal, int tile, int8_t* cls);

/* ra_plan_items (host only): the fused kernel's work list, in the order CTAs take it.  Each item
 * is four int32 (b, h, shard i, query-tile pair p) followed by its cost in live key/value tiles
 * (int32), 5 entries per item.  Items are (b, h) major; inside a head they are heaviest first
 * (LPT), except that when one head's keys and values (4*S*D bytes) exceed 96 MB the items of each
 * shard are grouped (groups heaviest first, LPT inside).  Writes at most cap items; *n_items
 * receives the full count. */
RA_API int ra_plan_items(int64_t B, int64_t H, int64_t S, int64_t D, int n_ring, int causal,
                         int layout, int32_t* items, int64_t cap, int64_t* n_items);

/* RA_NOALLOC_SCRATCH_BYTES: size of the fixed device array that ra_forward_noalloc uses as
 * scratch.  The array is part of the library's device code: a GPU holds it from the moment that
 * code is loaded there (the first use of the library on the device under CUDA's default lazy
 * module loading; context creation with CUDA_MODULE_LOADING=EAGER) until the process exits. */
#define RA_NOALLOC_SCRATCH_BYTES (64u << 20)

/* ra_forward_noalloc: the pages have no counterpart to this call; it exists for callers that
 * cannot let a library allocate GPU memory -- code recording a CUDA graph, engines that manage
 * every byte of device memory through their own allocator, loops where an allocation could stall.
 * It computes what ra_forward computes for bf16 q, k, v with D in {64, 128} on sm_100 (the fused
 * tensor-core ring), but takes its scratch (work list and counter; shard-major copies of q, k, v
 * for the zigzag layout) from one fixed device array of RA_NOALLOC_SCRATCH_BYTES instead of
 * allocating.  Arguments as for ra_forward (dtype is bf16 implicitly).
 *   - The first call on a device, with that device current, looks up the array's address and
 *     loads the code of every kernel the call launches (both head dims, every layout), so that no
 *     later call loads module code; make that first call before any stream capture.
 *   - All calls on a device share the array and leave their data in it; calls whose GPU work
 *     overlaps (other streams, other host threads) race on it.
 *   - A problem whose scratch does not fit (B*H*n_ring*ceil(S_loc/256) work items of 16 bytes,
 *     plus 3*B*S*H*D*2 bytes for zigzag and 256 bytes of counter), or whose work list the device
 *     builder cannot hold ((n_ring*ceil(S_loc/256) + n_ring) * 4 bytes above 48 KB), is rejected
 *     with RA_ERR_NO_WORKSPACE and a message in ra_last_error_string; nothing is enqueued.
 *   - Other dtypes or head dims return RA_ERR_UNSUPPORTED. */
RA_API int ra_forward_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                              int64_t B, int64_t H, int64_t S, int64_t D, int n_ring, int causal,
                              int layout, void* stream);

/* ra_backward: gradients dq, dk, dv of out = softmax(q k^T / sqrt(D)) v (causal mask on original
 * token positions, diagonal included, when `causal`) for the upstream gradient dout.  The
 * backward pass recomputes the attention statistics block by block from the saved lse instead of
 * storing the S x S weights (troisinh.com "Ring Attention", "Blockwise Backward"): dq of query
 * shard i accumulates over the key blocks j = (i - s) mod N in ring order, and dk, dv of key block
 * j over the query shards (j + s) mod N it visits, s = 0..N-1.
 *   q, k, v, out, dout, dq, dk, dv: [B, S, H, D] row-major in natural token order, `dtype` (fp32 or
 *     bf16); out and lse are the results of ra_forward on the same q, k, v, n_ring, causal
 *     (layout only changes the order of the work, not the result).
 *   lse: [B, H, S] fp32, natural log.
 *   Arithmetic (CUDA-core path; the tensor-core path, taken for bf16 with D in {64, 128}, is
 *   described under ra_backward_ex): Delta = rowsum(dout * out), then per tile
 *   P = exp(q k^T / sqrt(D) - lse), dP = dout v^T, dS = P (dP - Delta), dq = dS k / sqrt(D),
 *   dk = dS^T q / sqrt(D), dv = P^T dout; dq, dk, dv are written once each (no atomics).
 *   D <= 128 (RA_ERR_UNSUPPORTED otherwise); pointers aligned to their element size.
 *   The caller owns every buffer; scratch (B*H*S fp32 for Delta, plus shard-major copies for
 *   zigzag on the tensor-core path) is allocated and freed stream-ordered on `stream`
 *   (from the library's pool, as ra_options.workspace = NULL describes).  Asynchronous on `stream`.
 * Returns RA_OK or a negative status (validation errors before anything is enqueued). */
RA_API int ra_backward(const void* q, const void* k, const void* v, const void* out, const float* lse,
                       const void* dout, void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t S,
                       int64_t D, int n_ring, int causal, int layout, int dtype, void* stream);

/* ra_backward_ex: ra_backward with the kernel choice, the bound of every in-kernel wait of the
 * tensor-core kernels (timeout_ns; 0 = 2 s) and a debug knob (RA_DEBUG_STALL_LOADS: their load warp
 * issues no streamed tile, so the waits run out and report RA_ERR_DEVICE_TIMEOUT -- for tests).
 * No counterpart on the pages.  Kernel choice:
 *   RA_KERNEL_AUTO  tensor cores when they apply, else CUDA cores (what ra_backward does);
 *   RA_KERNEL_TC    tcgen05 kernels: bf16, D in {64, 128}, all eight tensors 16-byte aligned, sm_100
 *                   (RA_ERR_UNSUPPORTED otherwise); zigzag inputs are first copied to shard-major
 *                   order in stream-ordered scratch (4 x B*S*H*D bf16).  S and dP (or
 *                   their transposes) and the three gradient products run on the tensor cores
 *                   with fp32 accumulation; P and dS are rounded to bf16 as the product operands;
 *                   the elementwise step is fp32.  Bounded waits report RA_ERR_DEVICE_TIMEOUT
 *                   through ra_get_device_status;
 *   RA_KERNEL_SIMT  fp32 arithmetic on CUDA cores for every dtype, D <= 128. */
RA_API int ra_backward_ex(const void* q, const void* k, const void* v, const void* out, const float* lse,
                          const void* dout, void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t S,
                          int64_t D, int n_ring, int causal, int layout, int dtype, int kernel,
                          uint64_t timeout_ns, int debug, void* stream);

/* ra_forward_varlen: exact attention over several sequences packed one after another on the token
 * axis -- each query attends only to the keys of its own sequence (and, when `causal`, to those at or
 * before its position inside that sequence).  troisinh.com "Ring Attention", "Trade-off thuc te",
 * names load balancing with sequences of different lengths as the challenge; every sequence is split
 * into n_ring shards with `layout` and all their work items join one longest-first list.
 *   q, k, v, out: [S_total, H, D] in dtype (batch 1), natural order; lse: [H, S_total] fp32, natural
 *     log.
 *   cu_seqlens: HOST array of n_seqs + 1 int64 offsets, cu[0] = 0, non-decreasing, cu[n_seqs] =
 *     S_total; every length a multiple of n_ring, of 2 n_ring for zigzag (RA_ERR_SHAPE otherwise);
 *     empty sequences allowed.  S_total < 2^31, H <= 65535, 1 <= D <= 256.
 *   layout: contiguous, striped or zigzag, applied inside each sequence; dtype RA_DTYPE_FP32 or
 *   RA_DTYPE_BF16; q, k, v, out 16-byte aligned.  The defaults of ra_options apply: the tcgen05
 *   kernel (sm_100) for bf16 with D in {64, 128}, all ring steps in one persistent launch; the
 *   CUDA-core kernel with fp32 arithmetic otherwise.  Scratch (work list, sequence table, counter;
 *   for zigzag on the tensor cores also shard-major copies of q, k, v, 3 x S_total*H*D bf16) is
 *   allocated stream-ordered.  Asynchronous on `stream`; bounded waits report through
 *   ra_get_device_status. */
RA_API int ra_forward_varlen(const void* q, const void* k, const void* v, void* out, float* lse,
                             const int64_t* cu_seqlens, int n_seqs, int64_t H, int64_t D, int n_ring,
                             int causal, int layout, int dtype, void* stream);

/* ra_forward_varlen_ex: ra_forward_varlen with options (opt may be NULL for the defaults).
 *   variant: AUTO and FUSED walk every ring step in one attention launch; PER_STEP walks
 *     opt->steps_per_launch steps per launch (0 = 1) and folds each launch's partial result, kept
 *     in fp32 in natural packed rows, into the running one with the log-sum-exp merge.
 *   kernel: AUTO (tensor cores where they apply, see ra_forward_varlen), TC (bf16 with D in {64, 128}
 *     on sm_100, RA_ERR_UNSUPPORTED otherwise) or SIMT (CUDA cores, fp32 arithmetic, any dtype).
 *   workspace / workspace_bytes: caller scratch of at least ra_varlen_workspace_size bytes (for the
 *     same variant and kernel), 256-byte aligned (RA_ERR_ALIGN otherwise; RA_ERR_NO_WORKSPACE if
 *     smaller); NULL: allocated and freed stream-ordered as ra_forward_varlen does.  A caller that
 *     keeps the buffer between calls saves the allocation, which for zigzag on the tensor cores
 *     holds the 3 x S_total*H*D bf16 shard-major copies and, with more than one launch, the fp32
 *     running and partial results (2 x S_total*H*(D + 1) floats).
 *   timeout_ns, debug: as for ra_forward_ex (the tensor-core kernel's waits).  attn_events: recorded
 *     right before the first and right after the last attention launch (after the zigzag gather). */
RA_API int ra_forward_varlen_ex(const void* q, const void* k, const void* v, void* out, float* lse,
                                const int64_t* cu_seqlens, int n_seqs, int64_t H, int64_t D, int n_ring,
                                int causal, int layout, int dtype, void* stream, const ra_options* opt);

/* ra_varlen_workspace_size: scratch bytes ra_forward_varlen_ex needs for these packed sequences,
 * dtype, variant and kernel (enum values as in ra_options), written to *bytes; for PER_STEP the size
 * covers every steps_per_launch.  Host only; the arguments are validated as for ra_forward_varlen. */
RA_API int ra_varlen_workspace_size(const int64_t* cu_seqlens, int n_seqs, int64_t H, int64_t D, int n_ring,
                                    int layout, int dtype, int variant, int kernel, size_t* bytes);

/* ra_rope: rotary position embedding with global token positions (troisinh.com "Ring Attention",
 * "RoPE va Position Embedding": a token must be rotated by the angle m theta of its own position m
 * wherever its block travels on the ring).  x, y: [B, S, H, D] in natural token order, dtype fp32 or
 * bf16; the token at natural index g takes the position m = g + pos_offset (so a later chunk of a
 * sequence passes the length before it).  The pair (x[2p], x[2p+1]) is rotated by m * theta_p,
 * theta_p = base^(-2p/D) (10000 is the usual base).  y may equal x (in place) but must not overlap it
 * otherwise.  D even, <= 256; H * D <= 2^28 (RA_ERR_SHAPE otherwise);
 * pos_offset >= 0; base > 0; pointers aligned to their element size.  The angle is reduced in fp64,
 * the rotation is fp32, the result rounds to the dtype.  Asynchronous on `stream`; returns RA_OK
 * or a validation error before anything is enqueued. */
RA_API int ra_rope(const void* x, void* y, int64_t B, int64_t S, int64_t H, int64_t D, int64_t pos_offset,
                   double base, int dtype, void* stream);

/* ---- One ring step on one device's own buffers (a real multi-device ring).
 *
 * On a real ring device i keeps its query block Q_i and, at step s, holds the key/value block of
 * device j = (i - s) mod n_ring, which its left neighbour sent it during the previous step; it
 * computes the partial attention of Q_i against that block and merges it into its running result
 * (jisaku.com "Ring Attention", 処理フロー and 通信計算オーバーラップ; ultralytics.com "Ring
 * Attention", "how ring attention works").  These calls are the per-device compute of that loop;
 * moving the blocks between devices is the caller's (for example NCCL send/recv into a local
 * buffer -- the kernels only ever read memory of the current device).
 *
 * Local buffers hold one shard each, in the layout's local order: q_i[b, a] is global token
 * g(i, a) and k_j[b, a], v_j[b, a] are global token g(j, a), with g the layout map described at the
 * top of this file; every buffer is [B, S_loc, H, D], S_loc = S / n_ring.  The causal mask still
 * compares global positions, so the result of n_ring steps equals rows g(i, 0..S_loc-1) of
 * ra_forward on the whole sequence.
 *
 * ra_ring_step: step `step` (0 <= step < n_ring) of query shard `shard`, whose key/value block is
 * j = (shard - step) mod n_ring.
 *   q_i, k_j, v_j: [B, S_loc, H, D] in dtype (bf16 with D in {64, 128} on sm_100 runs on the tensor
 *     cores and needs 16-byte aligned pointers; other cases run the fp32 CUDA-core kernel).
 *   O_acc: [B, S_loc, H, D] fp32, 16-byte aligned; lse_acc: [B, S_loc, H] fp32.  The running
 *     result: O normalised by its own sum and its log-sum-exp.  Step 0 writes it (nothing is read);
 *     a later step merges its partial into it with the log-sum-exp form of the merge identities
 *     (troisinh.com "Ring Attention", "Tai sao no hoat dong").  Every step must see the same
 *     B, H, S, D, n_ring, causal, layout, dtype and shard.  A later step whose whole block is
 *     masked for every query of the shard enqueues nothing.
 *   sms_reserved: SMs the persistent tensor-core kernel leaves free (0 <= sms_reserved < SM count),
 *     so that a transfer kernel running at the same time (an NCCL send/recv of the next block) finds
 *     room on the GPU instead of waiting for the attention kernel to end; the CUDA-core kernel
 *     ignores it.
 *   workspace: device scratch of at least ra_ring_step_workspace_size bytes, 256-byte aligned
 *     (work list, counter, and the step's partial result); NULL: allocated and freed
 *     stream-ordered on `stream`.
 *   Asynchronous on `stream`; bounded in-kernel waits report through ra_get_device_status. */
RA_API int ra_ring_step(const void* q_i, const void* k_j, const void* v_j, float* O_acc, float* lse_acc,
                        int64_t B, int64_t H, int64_t S, int64_t D, int n_ring, int causal, int layout,
                        int dtype, int shard, int step, int sms_reserved, void* workspace,
                        size_t workspace_bytes, void* stream);

/* ra_ring_step_workspace_size: scratch bytes that suffice for ra_ring_step at every (shard, step) of
 * these arguments, written to *bytes.  Host only. */
RA_API int ra_ring_step_workspace_size(int64_t B, int64_t H, int64_t S, int64_t D, int n_ring, int causal,
                                       int layout, int dtype, size_t* bytes);

/* ra_ring_finalize: write the running result of a shard after its last step: out [B, S_loc, H, D] in
 * dtype (bf16 rounded to nearest even) and lse [B, H, S_loc] fp32, both in the shard's local token
 * order.  O_acc and out 16-byte aligned.  Asynchronous on `stream`. */
RA_API int ra_ring_finalize(const float* O_acc, const float* lse_acc, void* out, float* lse, int64_t B,
                            int64_t H, int64_t S_loc, int64_t D, int dtype, void* stream);

/* ra_status_string: static description of a status code. */
RA_API const char* ra_status_string(int status);

/* ra_last_error_string: the message of the last error recorded on the calling host thread: every
 * RA_ERR_CUDA records one, and so do the validation failures whose code alone is ambiguous (for
 * example RA_ERR_NO_WORKSPACE of ra_forward_noalloc).  Messages persist until the next one or until
 * ra_clear_last_error; the string is owned by the library and valid until the thread's next call. */
RA_API const char* ra_last_error_string(void);

/* ra_clear_last_error: empty the calling host thread's message, so that a non-empty message after a
 * failing call belongs to that call. */
RA_API void ra_clear_last_error(void);

/* ra_get_device_status: read and clear the status word that the kernels of this library set on
 * the current device (RA_OK, or RA_ERR_DEVICE_TIMEOUT after a bounded wait ran out).  Call it
 * after synchronising the stream; it synchronises the device itself. */
RA_API int ra_get_device_status(void);

#ifdef __cplusplus
}
#endif

#endif /* RA_H */
