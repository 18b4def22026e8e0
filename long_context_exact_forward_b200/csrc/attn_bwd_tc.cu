// attn_bwd_tc.cu -- the backward pass on the sm_100a tensor cores (tcgen05 + TMEM + TMA), bf16 inputs.
//
// Same mathematics and ring order as attn_bwd_simt.cu (troisinh.com "Ring Attention", "Blockwise
// Backward": the weights are recomputed per block from the saved lse, never stored):
//     P = exp(S / sqrt(D) - lse),  dP = dO V^T,  dS = P (dP - Delta),  Delta = rowsum(dO * O)
//     dQ = dS K / sqrt(D),  dK = dS^T Q / sqrt(D),  dV = P^T dO
// with the four products of a 128 x 128 tile on the tensor cores (bf16 operands, fp32 accumulators
// in TMEM) and the elementwise step on 256 threads, two per TMEM lane (tile row), each on half of
// the tile's columns.
//
// Inputs are read through 5-D TMA maps: in place for the contiguous and striped layouts, from
// shard-major copies for zigzag.
//
// bwd_dq_tc_kernel   one CTA per 128-row query tile of shard i; key tiles of the blocks
//                    j = (i - s) mod N in ring order.  TMEM: S of even / odd tiles [0,128) /
//                    [128,256), dP [256,384), dQ [384,512).  Per key tile t: S = Q K^T and dP = dO V^T
//                    (SS), the elementwise warps write dS (bf16) over S_t (packed_col below),
//                    then dQ += dS K (TS, K as the MN-major operand, like V in the forward P V).
//                    S of tile t + 1 is computed while the elementwise warps work on tile t, and
//                    dP of tile t + 1 goes before dQ of tile t, so the elementwise warps wait only
//                    for one product between tiles.
// bwd_dkv_tc_kernel  one CTA per 128-key tile of shard j; query tiles of the shards
//                    i = (j + s) mod N the block visits.  TMEM: S^T [0,128), dP^T [128,256),
//                    dV [256,384), dK [384,512).  Per query tile: S^T = K Q^T and dP^T = V dO^T (SS),
//                    the elementwise warps write P^T over S^T and dS^T over dP^T (bf16), then
//                    dV += P^T dO and dK += dS^T Q (TS, dO and Q as MN-major operands).
//
// Roles (320 threads): warp 0 TMA producer (lane 0 issues), warp 1 MMA issuer (converged warp,
// elect.sync picks the issuing lane) and TMEM owner, warps 2-9 elementwise: warp w reads TMEM lanes
// 32 (w mod 4) .. +31, warps 2-5 the columns 0..63 of every tile and warps 6-9 the columns 64..127
// (the elementwise steps have no row reductions, so the two halves never meet).  The streamed tiles
// go through two shared-memory stages.  Every wait is bounded; on give-up the CTA records
// RA_ERR_DEVICE_TIMEOUT, lets its copies and MMAs drain, frees TMEM and exits.
#include <cuda_bf16.h>

#include "ra.h"
#include "ra_internal.cuh"
#include "sm100.cuh"

namespace ra {
namespace {
using namespace sm100;

constexpr int kTile = 128;
constexpr int kThreads = 320;
constexpr int kEwWarps = 8;  // elementwise warps: two per TMEM lane quadrant, one per 64-column half
constexpr int kProducerWarp = 0, kMmaWarp = 1;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kColBlockBytes = 128 * 128;  // 128 rows x 64 bf16 (128-byte rows, 128-byte swizzle)

template <int kD>
struct BwdSmem {
    static constexpr int kTileBytes = kTile * kD * 2;
    uint8_t fixed[2][kTileBytes];      // dq: Q, dO of the CTA's query tile; dkv: K, V of its key tile
    uint8_t stream[2][2][kTileBytes];  // [stage][0/1]: dq: K, V of a key tile; dkv: Q, dO of a query tile
    float col_lse2[2][kTile];          // dkv: lse * log2(e) and Delta of the stage's 128 query rows
    float col_delta[2][kTile];
    uint64_t fixed_full, stage_full[2], stage_empty[2], s_full, dp_full, ds_full, acc_full, drain;
    uint32_t tmem_base;
    int abort;
};

struct BwdTcArgs {
    Layout32 L;
    int B, H, D;
    int causal;
    float scale;
    const float* lse;    // [B, H, S] natural
    const float* delta;  // [B, H, S] natural
    __nv_bfloat16* dq;   // [B, S, H, D] natural
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    uint64_t timeout_ns;
    int debug;           // RA_DEBUG_STALL_LOADS: the producer issues no streamed tile (tests)
    int* status;
};

// Each thread reads 16 consecutive 32-bit columns of its own TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Wait for the asynchronous TMEM loads and tie the destination registers to the wait, so that no
// use of them is scheduled before it.
template <int N>
__device__ __forceinline__ void wait_ld_tied(uint32_t (&r)[N]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int x = 0; x < N; ++x) asm volatile("" : "+r"(r[x]));
}
// Tie more registers to the wait just made (the wait covers every load issued before it).
template <int N>
__device__ __forceinline__ void tie_regs(uint32_t (&r)[N]) {
#pragma unroll
    for (int x = 0; x < N; ++x) asm volatile("" : "+r"(r[x]));
}

// mbar_wait preceded by a non-blocking probe: a phase that has already completed (the common case
// for the barriers the elementwise warps check second) costs one test instead of a try_wait.
__device__ __forceinline__ bool bar_wait(uint64_t* bar, uint32_t parity, uint64_t timeout, volatile int* abort) {
    return mbar_test_wait(bar, parity) || mbar_wait(bar, parity, timeout, abort);
}

__device__ __forceinline__ void give_up(volatile int* abort, int* status) {
    *abort = 1;
    atomicExch(status, RA_ERR_DEVICE_TIMEOUT);
}

__device__ __forceinline__ void tma_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int kD, int h,
                                         int a0, int shard, int b) {
    for (int cb = 0; cb < kD / 64; ++cb) tma_load_5d(dst + cb * kColBlockBytes, map, bar, cb * 64, h, a0, shard, b);
}

// D[tmem] (+)= A B^T over the head dim, A and B K-major tiles in shared memory (SS, N = 128)
template <int kD>
__device__ __forceinline__ void mma_tile_ss(uint32_t d_tmem, const uint8_t* a, const uint8_t* b) {
    constexpr uint32_t idesc = idesc_bf16_f32(kTile, kTile, 0, 0);
    const uint32_t aa = smem_addr(a), ba = smem_addr(b);
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kColBlockBytes + (kk & 3) * 32;
        warp_mma_ss(d_tmem, smem_desc_sw128(aa + off, 16, 1024), smem_desc_sw128(ba + off, 16, 1024), idesc,
                    kk > 0);
    }
}

// Packed bf16 A operands of the TS products (dS in the dq kernel; P^T and dS^T in the dk/dv kernel)
// are written over the fp32 tile they are computed from.  The 32 columns of chunk c (c = 0..3) go to
// TMEM columns 64 (c / 2) + 16 (c mod 2) .. +15: each of the two warps of a lane quadrant, which take
// columns 0..63 and 64..127, then overwrites only columns it has already read itself.
__device__ __forceinline__ uint32_t packed_col(int c) { return 64u * (uint32_t)(c >> 1) + 16u * (uint32_t)(c & 1); }

// D[tmem] (+)= A[tmem, bf16, 128 x 128, packed as above] B, B an MN-major 128 x kD tile in shared
// memory (TS, N = kD); K-step kk (16 columns of A = 8 TMEM columns) sits at 64 (kk / 4) + 8 (kk mod 4)
template <int kD>
__device__ __forceinline__ void mma_tile_ts(uint32_t d_tmem, uint32_t a_tmem, const uint8_t* b, bool accumulate) {
    constexpr uint32_t idesc = idesc_bf16_f32(kTile, kD, 0, 1);
    const uint32_t ba = smem_addr(b);
#pragma unroll
    for (int kk = 0; kk < kTile / 16; ++kk)
        warp_mma_ts(d_tmem, a_tmem + 64u * (kk >> 2) + 8u * (kk & 3),
                    smem_desc_sw128(ba + kk * 16 * 128, kColBlockBytes, 1024), idesc, (kk > 0 || accumulate) ? 1u : 0u);
}

// Number of live 128-key tiles of block j for the query tile at a0 of shard i.
__device__ __forceinline__ int key_tiles(const Layout32& L, int causal, int i, int a0, int j) {
    if (a0 >= L.S_loc) return 0;
    const int last = a0 + kTile - 1 < L.S_loc - 1 ? a0 + kTile - 1 : L.S_loc - 1;
    return (visible_keys(L, causal, i, last, j) + kTile - 1) / kTile;
}

// Does the query tile at a0 of shard i see any key of the key tile at c0 of block j?
__device__ __forceinline__ bool query_tile_live(const Layout32& L, int causal, int i, int a0, int j, int c0) {
    const int last = a0 + kTile - 1 < L.S_loc - 1 ? a0 + kTile - 1 : L.S_loc - 1;
    return visible_keys(L, causal, i, last, j) > c0;
}

// Store 32 fp32 values (times `mul`) of one row as bf16 at dst[0..31] (only the first `n` valid).
__device__ __forceinline__ void store_row_chunk(__nv_bfloat16* dst, const uint32_t (&v)[32], float mul, int n) {
    if (n >= 32) {
        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(v[8 * x + 0]) * mul, __uint_as_float(v[8 * x + 1]) * mul);
            u.y = pack_bf16x2(__uint_as_float(v[8 * x + 2]) * mul, __uint_as_float(v[8 * x + 3]) * mul);
            u.z = pack_bf16x2(__uint_as_float(v[8 * x + 4]) * mul, __uint_as_float(v[8 * x + 5]) * mul);
            u.w = pack_bf16x2(__uint_as_float(v[8 * x + 6]) * mul, __uint_as_float(v[8 * x + 7]) * mul);
            d4[x] = u;
        }
    } else {
        for (int x = 0; x < n; ++x) dst[x] = __float2bfloat16_rn(__uint_as_float(v[x]) * mul);
    }
}

// ================================================================ dQ
template <int kD>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const BwdTcArgs A) {
    extern __shared__ uint8_t smem_raw[];
    BwdSmem<kD>& sm = *reinterpret_cast<BwdSmem<kD>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                     ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Layout32 L = A.L;
    const int i = L.N - 1 - (int)blockIdx.y;  // heaviest shards first under the contiguous layout
    const int b = (int)blockIdx.z / A.H, h = (int)blockIdx.z % A.H;
    const int a0 = (int)blockIdx.x * kTile;
    const uint64_t timeout = A.timeout_ns;
    volatile int* abort = &sm.abort;

    if (threadIdx.x == 0) {
        mbar_init(&sm.fixed_full, 1);
        for (int st = 0; st < 2; ++st) {
            mbar_init(&sm.stage_full[st], 1);
            mbar_init(&sm.stage_empty[st], 1);
        }
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.dp_full, 1);
        mbar_init(&sm.ds_full, kEwWarps);
        mbar_init(&sm.acc_full, 1);
        mbar_init(&sm.drain, 1);
        sm.abort = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // S of tile t in [128 (t mod 2), +128): the next tile's S is computed while the elementwise
    // warps work on this one
    constexpr uint32_t kdP = 256, kdQ = 384;

    if (warp == kProducerWarp) {
        bool ok = true;
        uint32_t it = 0;
        if (lane == 0) {
            mbar_arrive_expect_tx(&sm.fixed_full, 2 * BwdSmem<kD>::kTileBytes);
            tma_tile(sm.fixed[0], &tm_q, &sm.fixed_full, kD, h, a0, i, b);
            tma_tile(sm.fixed[1], &tm_do, &sm.fixed_full, kD, h, a0, i, b);
        }
        for (int s = 0; s < L.N && ok; ++s) {
            const int j = ring_block32(i, s, L.N);
            const int nt = key_tiles(L, A.causal, i, a0, j);
            for (int kt = 0; kt < nt && ok; ++kt, ++it) {
                const uint32_t st = it & 1;
                if (A.debug == RA_DEBUG_STALL_LOADS) break;  // consumers must time out
                ok = __all_sync(0xffffffffu, mbar_wait(&sm.stage_empty[st], ((it >> 1) & 1) ^ 1, timeout, abort));
                if (!ok) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&sm.stage_full[st], 2 * BwdSmem<kD>::kTileBytes);
                    tma_tile(sm.stream[st][0], &tm_k, &sm.stage_full[st], kD, h, kt * kTile, j, b);
                    tma_tile(sm.stream[st][1], &tm_v, &sm.stage_full[st], kD, h, kt * kTile, j, b);
                }
            }
        }
        if (!ok) {
            if (lane == 0) give_up(abort, A.status);
            // the copies in flight: the two stages' last tiles and the fixed tiles
            for (uint32_t u = it > 2 ? it - 2 : 0; u < it; ++u)
                mbar_wait(&sm.stage_full[u & 1], (u >> 1) & 1, timeout, nullptr);
            mbar_wait(&sm.fixed_full, 0, timeout, nullptr);
        }
    } else if (warp == kMmaWarp) {
        bool ok = true;
        auto wait = [&](uint64_t* bar, uint32_t parity) {
            if (!ok) return false;
            ok = __all_sync(0xffffffffu, bar_wait(bar, parity, timeout, abort));
            if (ok) tc_fence_after();
            return ok;
        };
        uint32_t n_tiles = 0;  // key tiles of all ring steps, in the order the producer loads them
        for (int s = 0; s < L.N; ++s) n_tiles += key_tiles(L, A.causal, i, a0, ring_block32(i, s, L.N));
        if (wait(&sm.fixed_full, 0) && n_tiles > 0 && wait(&sm.stage_full[0], 0)) {
            mma_tile_ss<kD>(tmem + 0, sm.fixed[0], sm.stream[0][0]);
            mma_tile_ss<kD>(tmem + kdP, sm.fixed[1], sm.stream[0][1]);
            warp_mma_commit(&sm.s_full);
            for (uint32_t t = 0; t < n_tiles && ok; ++t) {
                const uint32_t st = t & 1, sn = (t + 1) & 1;
                const bool more = t + 1 < n_tiles;
                // S of the next tile into the other S buffer (its dS was read by the dQ MMA of tile
                // t - 1, issued before), while the elementwise warps work on tile t
                if (more) {
                    if (!wait(&sm.stage_full[sn], ((t + 1) >> 1) & 1)) break;
                    mma_tile_ss<kD>(tmem + 128 * sn, sm.fixed[0], sm.stream[sn][0]);
                }
                if (!wait(&sm.ds_full, t & 1)) break;
                // dP of the next tile (the elementwise warps have read dP of this one), then
                // dQ += dS K of this tile: dS (bf16) in the first 64 columns of S_t, K MN-major
                if (more) {
                    mma_tile_ss<kD>(tmem + kdP, sm.fixed[1], sm.stream[sn][1]);
                    warp_mma_commit(&sm.s_full);
                }
                mma_tile_ts<kD>(tmem + kdQ, tmem + 128 * st, sm.stream[st][0], t > 0);
                warp_mma_commit(&sm.stage_empty[st]);
            }
        }
        if (ok) warp_mma_commit(&sm.acc_full);
        if (!ok) {
            if (lane == 0) give_up(abort, A.status);
            warp_mma_commit(&sm.drain);
            mbar_wait(&sm.drain, 0, timeout, nullptr);
        }
    } else {
        // elementwise: row r of the query tile, columns 64 half .. 64 half + 63 of each key tile
        const int half = (warp - 2) >> 2;
        const int r = 32 * (warp & 3) + lane;
        const int a = a0 + r;
        const bool row_ok = a < L.S_loc;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        const int g = row_ok ? global_position(L, i, a) : 0;
        const size_t row_stat = ((size_t)b * A.H + h) * L.S + g;
        const float lse2 = row_ok ? A.lse[row_stat] * kLog2e : 0.f;
        const float del = row_ok ? A.delta[row_stat] : 0.f;
        const float sl2 = A.scale * kLog2e;
        bool ok = true;
        auto wait_all = [&](uint64_t* bar, uint32_t parity) {
            ok = __all_sync(0xffffffffu, bar_wait(bar, parity, timeout, abort));
            if (ok) tc_fence_after();
            return ok;
        };
        uint32_t it = 0;
        bool any = false;
        for (int s = 0; s < L.N && ok; ++s) {
            const int j = ring_block32(i, s, L.N);
            const int nt = key_tiles(L, A.causal, i, a0, j);
            const int cnt = row_ok ? visible_keys(L, A.causal, i, a, j) : 0;
            for (int kt = 0; kt < nt && ok; ++kt, ++it) {
                if (!wait_all(&sm.s_full, it & 1)) break;
                any = true;
                const int valid = cnt - kt * kTile;
                const uint32_t kS = 128 * (it & 1);
#pragma unroll 1
                auto chunk = [&](int c, const uint32_t (&sv)[32], const uint32_t (&pv)[32]) {
                    uint32_t pk[16];
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        float ds[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int col = 32 * c + 2 * x + e;
                            const float p = col < valid ? ex2(fmaf(__uint_as_float(sv[2 * x + e]), sl2, -lse2)) : 0.f;
                            ds[e] = p * (__uint_as_float(pv[2 * x + e]) - del);
                        }
                        pk[x] = pack_bf16x2(ds[0], ds[1]);
                    }
                    // dS of columns 32c..32c+31 -> TMEM columns packed_col(c)..+15 (already read)
                    tmem_st16(lane_base + kS + packed_col(c), pk);
                };
                {  // the second chunk's loads run while the first is computed
                    const int c0 = 2 * half;
                    uint32_t sv0[32], pv0[32], sv1[32], pv1[32];
                    tmem_ld32(lane_base + kS + 32 * c0, sv0);
                    tmem_ld32(lane_base + kdP + 32 * c0, pv0);
                    wait_ld_tied(sv0);
                    tie_regs(pv0);
                    tmem_ld32(lane_base + kS + 32 * (c0 + 1), sv1);
                    tmem_ld32(lane_base + kdP + 32 * (c0 + 1), pv1);
                    chunk(c0, sv0, pv0);
                    wait_ld_tied(sv1);
                    tie_regs(pv1);
                    chunk(c0 + 1, sv1, pv1);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.ds_full);
            }
        }
        // each warp of a quadrant stores its half of the head dims
        if (ok && any) {
            if (wait_all(&sm.acc_full, 0)) {
                __nv_bfloat16* dst = A.dq + (((size_t)b * L.S + g) * A.H + h) * A.D;
#pragma unroll 1
                for (int c = half * (kD / 64); c < (half + 1) * (kD / 64); ++c) {
                    uint32_t v[32];
                    tmem_ld32(lane_base + kdQ + 32 * c, v);
                    wait_ld_tied(v);
                    if (row_ok) store_row_chunk(dst + 32 * c, v, A.scale, 32);
                }
            }
        } else if (ok && row_ok) {  // no visible key at all: the gradient is zero
            __nv_bfloat16* dst = A.dq + (((size_t)b * L.S + g) * A.H + h) * A.D;
            for (int d = half * (kD / 2); d < (half + 1) * (kD / 2); ++d) dst[d] = __float2bfloat16_rn(0.f);
        }
        if (!ok && lane == 0) give_up(abort, A.status);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ================================================================ dK, dV
template <int kD>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const BwdTcArgs A) {
    extern __shared__ uint8_t smem_raw[];
    BwdSmem<kD>& sm = *reinterpret_cast<BwdSmem<kD>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                     ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Layout32 L = A.L;
    const int j = (int)blockIdx.y;
    const int b = (int)blockIdx.z / A.H, h = (int)blockIdx.z % A.H;
    const int c0 = (int)blockIdx.x * kTile;  // first local key of this tile
    const uint64_t timeout = A.timeout_ns;
    volatile int* abort = &sm.abort;

    if (threadIdx.x == 0) {
        mbar_init(&sm.fixed_full, 1);
        for (int st = 0; st < 2; ++st) {
            mbar_init(&sm.stage_full[st], 2);  // the copies (expect_tx) + the query statistics
            mbar_init(&sm.stage_empty[st], 1);
        }
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.dp_full, 1);
        mbar_init(&sm.ds_full, kEwWarps);
        mbar_init(&sm.acc_full, 1);
        mbar_init(&sm.drain, 1);
        sm.abort = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    constexpr uint32_t kST = 0, kdPT = 128, kdV = 256, kdK = 384;

    if (warp == kProducerWarp) {
        bool ok = true;
        uint32_t it = 0;
        if (lane == 0) {
            mbar_arrive_expect_tx(&sm.fixed_full, 2 * BwdSmem<kD>::kTileBytes);
            tma_tile(sm.fixed[0], &tm_k, &sm.fixed_full, kD, h, c0, j, b);
            tma_tile(sm.fixed[1], &tm_v, &sm.fixed_full, kD, h, c0, j, b);
        }
        for (int s = 0; s < L.N && ok; ++s) {
            const int i = (j + s) % L.N;
            for (int q0 = 0; q0 < L.S_loc && ok; q0 += kTile) {
                if (!query_tile_live(L, A.causal, i, q0, j, c0)) continue;
                const uint32_t st = it & 1;
                if (A.debug == RA_DEBUG_STALL_LOADS) break;  // consumers must time out
                // lse (log2 units) and Delta of the tile's query rows, for the elementwise warps: read
                // before the stage frees, so that the gather's latency overlaps the wait
                float l2[kTile / 32], dl[kTile / 32];
#pragma unroll
                for (int e = 0; e < kTile / 32; ++e) {
                    const int a = q0 + lane * (kTile / 32) + e;
                    l2[e] = 0.f;
                    dl[e] = 0.f;
                    if (a < L.S_loc) {
                        const size_t ix = ((size_t)b * A.H + h) * L.S + global_position(L, i, a);
                        l2[e] = __ldg(A.lse + ix) * kLog2e;
                        dl[e] = __ldg(A.delta + ix);
                    }
                }
                ok = __all_sync(0xffffffffu, mbar_wait(&sm.stage_empty[st], ((it >> 1) & 1) ^ 1, timeout, abort));
                if (!ok) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&sm.stage_full[st], 2 * BwdSmem<kD>::kTileBytes);
                    tma_tile(sm.stream[st][0], &tm_q, &sm.stage_full[st], kD, h, q0, i, b);
                    tma_tile(sm.stream[st][1], &tm_do, &sm.stage_full[st], kD, h, q0, i, b);
                }
#pragma unroll
                for (int e = 0; e < kTile / 32; ++e) {
                    const int r = lane * (kTile / 32) + e;
                    sm.col_lse2[st][r] = l2[e];
                    sm.col_delta[st][r] = dl[e];
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.stage_full[st]);
                ++it;
            }
        }
        if (!ok) {
            if (lane == 0) give_up(abort, A.status);
            for (uint32_t u = it > 2 ? it - 2 : 0; u < it; ++u)
                mbar_wait(&sm.stage_full[u & 1], (u >> 1) & 1, timeout, nullptr);
            mbar_wait(&sm.fixed_full, 0, timeout, nullptr);
        }
    } else if (warp == kMmaWarp) {
        bool ok = true;
        auto wait = [&](uint64_t* bar, uint32_t parity) {
            if (!ok) return false;
            ok = __all_sync(0xffffffffu, bar_wait(bar, parity, timeout, abort));
            if (ok) tc_fence_after();
            return ok;
        };
        uint32_t n_tiles = 0;  // live query tiles over the ring steps, in the producer's order
        for (int s = 0; s < L.N; ++s)
            for (int q0 = 0; q0 < L.S_loc; q0 += kTile)
                n_tiles += query_tile_live(L, A.causal, (j + s) % L.N, q0, j, c0) ? 1u : 0u;
        if (wait(&sm.fixed_full, 0) && n_tiles > 0 && wait(&sm.stage_full[0], 0)) {
            mma_tile_ss<kD>(tmem + kST, sm.fixed[0], sm.stream[0][0]);
            warp_mma_commit(&sm.s_full);
            mma_tile_ss<kD>(tmem + kdPT, sm.fixed[1], sm.stream[0][1]);
            warp_mma_commit(&sm.dp_full);
            for (uint32_t t = 0; t < n_tiles && ok; ++t) {
                const uint32_t st = t & 1, sn = (t + 1) & 1;
                const bool more = t + 1 < n_tiles;
                if (!wait(&sm.ds_full, t & 1)) break;
                // dV += P^T dO (P^T over S^T), then S^T of the next tile into the columns just read,
                // so the elementwise warps start its exponentials while dK and dP^T run
                mma_tile_ts<kD>(tmem + kdV, tmem + kST, sm.stream[st][1], t > 0);
                if (more) {
                    if (!wait(&sm.stage_full[sn], ((t + 1) >> 1) & 1)) break;
                    mma_tile_ss<kD>(tmem + kST, sm.fixed[0], sm.stream[sn][0]);
                    warp_mma_commit(&sm.s_full);
                }
                // dK += dS^T Q (dS^T over dP^T), then dP^T of the next tile
                mma_tile_ts<kD>(tmem + kdK, tmem + kdPT, sm.stream[st][0], t > 0);
                warp_mma_commit(&sm.stage_empty[st]);
                if (more) {
                    mma_tile_ss<kD>(tmem + kdPT, sm.fixed[1], sm.stream[sn][1]);
                    warp_mma_commit(&sm.dp_full);
                }
            }
        }
        if (ok) warp_mma_commit(&sm.acc_full);
        if (!ok) {
            if (lane == 0) give_up(abort, A.status);
            warp_mma_commit(&sm.drain);
            mbar_wait(&sm.drain, 0, timeout, nullptr);
        }
    } else {
        // elementwise: row r = key c0 + r of this tile, columns = the query rows 64 half .. 64 half + 63
        // of a query tile
        const int half = (warp - 2) >> 2;
        const int r = 32 * (warp & 3) + lane;
        const int key = c0 + r;
        const bool row_ok = key < L.S_loc;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        const float sl2 = A.scale * kLog2e;
        const int gk = row_ok ? global_position(L, j, key) : 0;
        bool ok = true;
        auto wait_all = [&](uint64_t* bar, uint32_t parity) {
            ok = __all_sync(0xffffffffu, bar_wait(bar, parity, timeout, abort));
            if (ok) tc_fence_after();
            return ok;
        };
        uint32_t it = 0;
        bool any = false;
        for (int s = 0; s < L.N && ok; ++s) {
            const int i = (j + s) % L.N;
            // queries a >= a_min of shard i see this key (positions are increasing within a shard)
            const int a_min = !row_ok ? L.S_loc : (A.causal ? key_count(L, i, gk - 1) : 0);
            for (int q0 = 0; q0 < L.S_loc && ok; q0 += kTile) {
                if (!query_tile_live(L, A.causal, i, q0, j, c0)) continue;
                const uint32_t st = it & 1;
                // the query statistics first: they land with the tile's copies, well before S^T, so
                // this check overlaps the wait for S^T instead of following it (no TMEM access
                // depends on it, hence no tcgen05 fence)
                ok = __all_sync(0xffffffffu, bar_wait(&sm.stage_full[st], (it >> 1) & 1, timeout, abort));
                if (!ok) break;
                if (!wait_all(&sm.s_full, it & 1)) break;
                any = true;
                // phase 1 (S^T ready): P^T = exp(S^T / sqrt(D) - lse), bf16, written over S^T
                // (chunk c writes columns packed_col(c).., already read by this warp).  Both of the
                // warp's chunks are loaded at once, so that one TMEM round trip serves them.
                auto phase1 = [&](int c, const uint32_t (&sv)[32]) {
                    uint32_t pk[16];
                    const float4* l4 = reinterpret_cast<const float4*>(&sm.col_lse2[st][32 * c]);
                    // every query of this chunk sees the key: no per-element check (the common case)
                    const bool all_vis = q0 + 32 * c >= a_min && q0 + 32 * c + 31 < L.S_loc;
                    if (all_vis) {
#pragma unroll
                        for (int x = 0; x < 8; ++x) {
                            const float4 lv = l4[x];  // 4 columns' lse per shared-memory load
                            pk[2 * x] = pack_bf16x2(ex2(fmaf(__uint_as_float(sv[4 * x]), sl2, -lv.x)),
                                                    ex2(fmaf(__uint_as_float(sv[4 * x + 1]), sl2, -lv.y)));
                            pk[2 * x + 1] = pack_bf16x2(ex2(fmaf(__uint_as_float(sv[4 * x + 2]), sl2, -lv.z)),
                                                        ex2(fmaf(__uint_as_float(sv[4 * x + 3]), sl2, -lv.w)));
                        }
                    } else {
#pragma unroll
                        for (int x = 0; x < 16; ++x) {
                            float p[2];
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int col = 32 * c + 2 * x + e, a = q0 + col;
                                const bool vis = a >= a_min && a < L.S_loc;
                                p[e] = vis ? ex2(fmaf(__uint_as_float(sv[2 * x + e]), sl2, -sm.col_lse2[st][col])) : 0.f;
                            }
                            pk[x] = pack_bf16x2(p[0], p[1]);
                        }
                    }
                    tmem_st16(lane_base + kST + packed_col(c), pk);
                };
                {
                    const int c0 = 2 * half;
                    uint32_t sv0[32], sv1[32];
                    tmem_ld32(lane_base + kST + 32 * c0, sv0);
                    tmem_ld32(lane_base + kST + 32 * (c0 + 1), sv1);
                    wait_ld_tied(sv0);
                    tie_regs(sv1);
                    phase1(c0, sv0);
                    phase1(c0 + 1, sv1);
                }
                // phase 2 (dP^T ready): dS^T = P^T (dP^T - Delta) from the stored bf16 P^T, written
                // over dP^T in the same packed columns
                tmem_wait_st();
                if (!wait_all(&sm.dp_full, it & 1)) break;
                auto phase2 = [&](int c, const uint32_t (&pv)[32], const uint32_t (&pb)[16]) {
                    uint32_t dk16[16];
                    const float4* d4 = reinterpret_cast<const float4*>(&sm.col_delta[st][32 * c]);
#pragma unroll
                    for (int x = 0; x < 8; ++x) {
                        const float4 dv = d4[x];  // 4 columns' Delta per shared-memory load
                        const uint32_t b0 = pb[2 * x], b1 = pb[2 * x + 1];
                        dk16[2 * x] = pack_bf16x2(__uint_as_float(b0 << 16) * (__uint_as_float(pv[4 * x]) - dv.x),
                                                  __uint_as_float(b0 & 0xffff0000u) * (__uint_as_float(pv[4 * x + 1]) - dv.y));
                        dk16[2 * x + 1] = pack_bf16x2(__uint_as_float(b1 << 16) * (__uint_as_float(pv[4 * x + 2]) - dv.z),
                                                      __uint_as_float(b1 & 0xffff0000u) * (__uint_as_float(pv[4 * x + 3]) - dv.w));
                    }
                    tmem_st16(lane_base + kdPT + packed_col(c), dk16);
                };
                {  // the second chunk's loads run while the first chunk is computed
                    const int c0 = 2 * half;
                    uint32_t pv0[32], pb0[16], pv1[32], pb1[16];
                    tmem_ld32(lane_base + kdPT + 32 * c0, pv0);
                    tmem_ld16(lane_base + kST + packed_col(c0), pb0);
                    wait_ld_tied(pv0);
                    tie_regs(pb0);
                    tmem_ld32(lane_base + kdPT + 32 * (c0 + 1), pv1);
                    tmem_ld16(lane_base + kST + packed_col(c0 + 1), pb1);
                    phase2(c0, pv0, pb0);
                    wait_ld_tied(pv1);
                    tie_regs(pb1);
                    phase2(c0 + 1, pv1, pb1);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.ds_full);
                ++it;
            }
        }
        __nv_bfloat16* dkr = A.dk + (((size_t)b * L.S + gk) * A.H + h) * A.D;
        __nv_bfloat16* dvr = A.dv + (((size_t)b * L.S + gk) * A.H + h) * A.D;
        // each warp of a quadrant stores its half of the head dims
        if (ok && any) {
            if (wait_all(&sm.acc_full, 0)) {
#pragma unroll 1
                for (int c = half * (kD / 64); c < (half + 1) * (kD / 64); ++c) {
                    uint32_t v[32];
                    tmem_ld32(lane_base + kdV + 32 * c, v);
                    wait_ld_tied(v);
                    if (row_ok) store_row_chunk(dvr + 32 * c, v, 1.f, 32);
                    tmem_ld32(lane_base + kdK + 32 * c, v);
                    wait_ld_tied(v);
                    if (row_ok) store_row_chunk(dkr + 32 * c, v, A.scale, 32);
                }
            }
        } else if (ok && row_ok) {  // no query sees these keys: the gradients are zero
            for (int d = half * (kD / 2); d < (half + 1) * (kD / 2); ++d) {
                dkr[d] = __float2bfloat16_rn(0.f);
                dvr[d] = __float2bfloat16_rn(0.f);
            }
        }
        if (!ok && lane == 0) give_up(abort, A.status);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

static_assert(sizeof(BwdSmem<128>) + 1024 <= 232448, "shared memory of one CTA (227 KB)");

// Launch both gradient kernels (after Delta is computed) for bf16 q, k, v, dout in natural order,
// D in {64, 128}.  Contiguous and striped inputs are read in place (striped through the strided
// TMA view); for zigzag, `shard_major` holds room for shard-major copies of q, k, v and dout
// (4 x B*S*H*D bf16, 256-byte aligned each), made here with the permute kernel.  The gradients are
// written in natural order either way.
int launch_backward_tc(const void* q, const void* k, const void* v, const void* dout, void* dq, void* dk,
                       void* dv, const float* lse, const float* delta, int64_t B, int64_t H, const Layout& L,
                       int64_t D, int causal, int* status, void* shard_major, uint64_t timeout_ns, int debug,
                       cudaStream_t stream) {
    CUtensorMap maps[4];
    const void* srcs[4] = {q, k, v, dout};
    const bool striped = L.kind == RA_LAYOUT_STRIPED;
    if (L.kind == RA_LAYOUT_ZIGZAG) {
        if (!shard_major) return RA_ERR_NO_WORKSPACE;
        const size_t bytes = ((size_t)(B * L.S * H * D) * 2 + 255) / 256 * 256;
        void* dst[4];
        for (int t = 0; t < 4; ++t) dst[t] = static_cast<uint8_t*>(shard_major) + t * bytes;
        const cudaError_t e = launch_permute(srcs, dst, 4, B, L, H, D, 2, false, stream);
        if (e != cudaSuccess) return host_cuda_fail(e, "permute launch");
        for (int t = 0; t < 4; ++t) srcs[t] = dst[t];
    }
    for (int t = 0; t < 4; ++t) {
        const int rc = host_encode_qkv_map(&maps[t], srcs[t], B, L, H, D, striped);
        if (rc != RA_OK) return rc;
    }
    BwdTcArgs A{};
    A.L = narrow(L);
    A.B = (int)B;
    A.H = (int)H;
    A.D = (int)D;
    A.causal = causal ? 1 : 0;
    A.scale = (float)(1.0 / sqrt((double)D));
    A.lse = lse;
    A.delta = delta;
    A.dq = static_cast<__nv_bfloat16*>(dq);
    A.dk = static_cast<__nv_bfloat16*>(dk);
    A.dv = static_cast<__nv_bfloat16*>(dv);
    A.timeout_ns = timeout_ns ? timeout_ns : 2000000000ull;
    A.debug = debug;
    A.status = status;
    const dim3 grid((unsigned)((L.S_loc + kTile - 1) / kTile), (unsigned)L.N, (unsigned)(B * H));
    cudaError_t e;
    if (D == 64) {
        const size_t smem = sizeof(BwdSmem<64>) + 1024;
        if ((e = cudaFuncSetAttribute(bwd_dq_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(bwd_dkv_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return host_cuda_fail(e, "backward kernel attributes");
        bwd_dq_tc_kernel<64><<<grid, kThreads, smem, stream>>>(maps[0], maps[1], maps[2], maps[3], A);
        if ((e = cudaGetLastError()) != cudaSuccess) return host_cuda_fail(e, "dq launch");
        bwd_dkv_tc_kernel<64><<<grid, kThreads, smem, stream>>>(maps[0], maps[1], maps[2], maps[3], A);
    } else {
        const size_t smem = sizeof(BwdSmem<128>) + 1024;
        if ((e = cudaFuncSetAttribute(bwd_dq_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(bwd_dkv_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return host_cuda_fail(e, "backward kernel attributes");
        bwd_dq_tc_kernel<128><<<grid, kThreads, smem, stream>>>(maps[0], maps[1], maps[2], maps[3], A);
        if ((e = cudaGetLastError()) != cudaSuccess) return host_cuda_fail(e, "dq launch");
        bwd_dkv_tc_kernel<128><<<grid, kThreads, smem, stream>>>(maps[0], maps[1], maps[2], maps[3], A);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return host_cuda_fail(e, "dkv launch");
    return RA_OK;
}

}  // namespace ra
