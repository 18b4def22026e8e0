// attn_tc.cu -- ring-order blockwise attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// What it computes.  For each work item (batch b, head h, shard i, a pair of 128-row query tiles)
// the kernel walks the ring steps s in [s_begin, s_end); at step s it meets the key/value block of
// shard j = (i - s) mod N (ultralytics.com "Ring Attention" toy loop; jisaku.com 処理フロー) and
// for every live 128-key tile of that block it computes
//     S = Q_i K_j^T                         (tcgen05.mma, bf16 x bf16 -> fp32 in TMEM)
//     m' = max(m, rowmax(S) / sqrt(D));  P = exp(S / sqrt(D) - m')     (softmax warps)
//     l  = e^{m - m'} l + rowsum(P);     O = e^{m - m'} O + P V_j      (tcgen05.mma, P from TMEM)
// i.e. the online-softmax identities of troisinh.com "Ring Attention" ("Tai sao no hoat dong"),
// applied tile by tile and step by step, so that the merge across ring steps (the in-kernel form
// of the pages' per-device accumulation) never leaves the chip.  At the end O / l and
// lse = m + ln l are written, either as the final result in natural token order or as one ring
// step's partial result (per-step variant).
//
// The causal mask is applied on original token positions.  Because every layout keeps positions
// increasing within a shard, a query row sees a prefix of each key block; key tiles past the
// longest prefix of the query tile are never loaded (block skip), tiles inside every row's prefix
// run unmasked, and only the tile holding a row's prefix end is masked.
//
// Layout of one CTA (384 threads, one CTA per SM, persistent; items are taken from a launch-wide
// counter, heaviest first):
//   warps 0-3  softmax for query tile 0 (thread t owns row t = TMEM lane t)
//   warps 4-7  softmax for query tile 1
//   warp  8    TMA producer (lane 0 issues): Q tiles, then K and V tiles into a ring of 4
//              shared-memory slots; also hands out the work items
//   warp  9    MMA issuer (the whole warp runs the loop, one elected lane issues) and TMEM owner
//   warps 10-11 idle
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [384,384+D).  P (bf16) is
// written over the first 64 columns of its S tile and read from there by the P V MMA.
// The MMA order per key tile t is  P0V(t), S0(t+1), P1V(t), S1(t+1), so each query tile's softmax
// overlaps the other tile's MMAs.  Each P V is issued in two halves: keys 0..63 as soon as the
// softmax warps have stored that half of P (they signal it mid-way), keys 64..127 when all of P
// is stored.  Because S0(t+1) is issued after P0V(t), the completion of S0(t+1) also proves P0V(t)
// is done, which lets the softmax warps rescale O in place before they store P of tile t+1.
// Rescaling of O is lazy: it happens only when a row's max grows by more than 2^8.
//
// Every wait is bounded (timeout_ns); on give-up the CTA records RA_ERR_DEVICE_TIMEOUT in the
// status word, lets its own copies and MMAs drain (again bounded), frees TMEM and exits.
#include <cuda_bf16.h>

#include <type_traits>

#include "ra.h"
#include "ra_internal.cuh"
#include "sm100.cuh"

namespace ra {
namespace {
using namespace sm100;

constexpr int kM = 128;           // query rows per tile
constexpr int kN = 128;           // keys per tile
constexpr int kSlots = 4;         // K/V tile slots
constexpr int kThreads = 384;
#ifndef RA_REGS_SOFTMAX
#define RA_REGS_SOFTMAX 184
#endif
#ifndef RA_REGS_OTHER
#define RA_REGS_OTHER 112
#endif
// register split: 256 softmax threads and 128 load / MMA threads, within the 384 x 168 registers
// the CTA is launched with
constexpr int kRegsSoftmax = RA_REGS_SOFTMAX, kRegsOther = RA_REGS_OTHER;
static_assert(256 * kRegsSoftmax + 128 * kRegsOther <= 384 * 168, "register split exceeds the launch budget");
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;  // lazy-rescale threshold (log2 units)
// Frozen max: when the head's score bound (qmax * kmax * scale, log2 units) lies within kFreezeLog2
// of every row's max after the first tile of an item, a warp keeps its rows' max fixed for the rest
// of the item: no later weight exceeds 2^kFreezeLog2, so no max and no rescale is needed.
constexpr float kFreezeLog2 = 32.0f;
constexpr float kBoundSlack = 1.0f + 1.0f / 256.0f;  // covers fp32 rounding of the norms and of S
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr uint32_t kNegInfBits = 0xff800000u;
constexpr int kColBlockBytes = 128 * 128;  // one 128-row x 64-element bf16 block (128-B rows)

// Every kExp2PolyEvery-th pair of P columns can be exponentiated on the FMA pipe instead of the
// MUFU unit (16 384 exponentials per 128x128 tile, as many cycles as the tile's MMAs).  Measured
// on s128k: 0 (all on MUFU) is fastest, 4 costs 4.5 % and 2 costs 8 %: the softmax warps are bound
// by issue latency, not by the MUFU pipe, so the default is 0.
#ifndef RA_EXP2_POLY_EVERY
#define RA_EXP2_POLY_EVERY 0
#endif
constexpr int kExp2PolyEvery = RA_EXP2_POLY_EVERY;

// 2^x for a pair of floats on the FMA pipe (Cody-Waite style range reduction):
//   x is clamped to >= -127, t = x + 1.5*2^23 rounded toward -inf puts floor(x) in t's low
//   mantissa bits, f = x - floor(x) in [0, 1), 2^f ~ 1 + f(c1 + f(c2 + f c3)), and floor(x) is added
//   to the exponent field (t's bits shifted left by 23 equal floor(x) << 23 modulo 2^32).
//   c1..c3 minimise the maximum relative error of the cubic on [0, 1) with p(0) = 1 fixed (a
//   linear program on 4001 points): 8.6e-5, far below the 2^-9 rounding of P to bf16.  At
//   x = -127 the result is exactly +0 (f = 0, p = 1, exponent field 0), so masked scores vanish.
__device__ __forceinline__ uint64_t exp2_poly_f32x2(uint64_t x2) {
    constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
    float x0, x1;
    split_f32x2(x2, x0, x1);
    const uint64_t xc = f32x2(fmaxf(x0, -127.f), fmaxf(x1, -127.f));
    const uint64_t t = add_rm_f32x2(xc, f32x2(kShift, kShift));
    const uint64_t fl = sub_f32x2(t, f32x2(kShift, kShift));
    const uint64_t fr = sub_f32x2(xc, fl);
    uint64_t p = fma_f32x2(fr, f32x2(0.07706724107265472f, 0.07706724107265472f),
                           f32x2(0.22764497995376587f, 0.22764497995376587f));
    p = fma_f32x2(p, fr, f32x2(0.6951166391372681f, 0.6951166391372681f));
    p = fma_f32x2(p, fr, f32x2(1.f, 1.f));
    float t0, t1, p0, p1;
    split_f32x2(t, t0, t1);
    split_f32x2(p, p0, p1);
    const uint32_t r0 = __float_as_uint(p0) + (__float_as_uint(t0) << 23);
    const uint32_t r1 = __float_as_uint(p1) + (__float_as_uint(t1) << 23);
    return f32x2(__uint_as_float(r0), __uint_as_float(r1));
}

template <int kD>
struct TcSmem {
    static constexpr int kTileBytes = kM * kD * 2;
    uint8_t q[2][kTileBytes];         // each tile: kD/64 column blocks of 128 rows x 128 B
    uint8_t kv[kSlots][kTileBytes];
    uint64_t q_full, q_empty, drain;
    uint64_t kv_full[2];              // K and V of key tile n have landed (barrier n % 2)
    uint64_t slot_empty[kSlots];      // key tile n uses slots 2n and 2n+1 (mod kSlots)
    uint64_t s_full[2], p_half[2], p_full[2], o_final[2], o_free[2];  // p_half: P of keys 0..63 stored
    uint64_t item_full[2], item_empty[2];  // ring of work-item indices handed out by the load warp
    int item_idx[2];
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ uint32_t s_col(int q) { return (uint32_t)q * 128u; }
template <int kD>
__device__ __forceinline__ uint32_t o_col(int q) { return 256u + (uint32_t)q * 128u; }

struct ItemGeom {
    Layout32 L;   // the item's sequence: the whole problem, or one packed sequence
    int base;     // first token of the sequence on the packed axis (0 in batch mode)
    int b, h, i;
    int a0[2];    // first local row of each query tile
    int last[2];  // last valid local row of each query tile (clamped to the shard)
};

// kVarlen is a template flag so that the batch-mode kernel keeps the problem's layout in the
// roles' registers instead of a per-item copy.
template <bool kVarlen>
__device__ __forceinline__ ItemGeom item_geom(const AttnArgs& A, const Layout32& Lg, int4 it) {
    ItemGeom G;
    G.h = it.y;
    G.i = it.z;
    if (kVarlen) {  // packed sequences: x is the sequence
        const int2 sd = A.seqs[it.x];
        G.L = Layout32{sd.x, Lg.N, sd.x / Lg.N, Lg.kind};
        G.base = sd.y;
        G.b = 0;
    } else {
        G.L = Lg;
        G.base = 0;
        G.b = it.x;
    }
    for (int q = 0; q < 2; ++q) {
        G.a0[q] = it.w * 2 * kM + q * kM;
        const int e = G.a0[q] + kM - 1;
        G.last[q] = e < G.L.S_loc - 1 ? e : G.L.S_loc - 1;
    }
    return G;
}

// TMA row coordinates (dims 2 and 3 of the 5-D map) of local row a of shard `shard`: in batch mode
// (row, shard); packed contiguous, the map's token axis is the packed axis; packed striped, the
// map is (token / N, token mod N) and sequences start on multiples of N.
template <bool kVarlen>
__device__ __forceinline__ int2 tma_rows(const AttnArgs& A, const ItemGeom& G, int shard, int a) {
    if (!kVarlen) return make_int2(a, A.local ? 0 : shard);
    if (A.varlen_striped) return make_int2(G.base / G.L.N + a, shard);
    return make_int2(G.base + shard * G.L.S_loc + a, 0);
}

// Live key tiles of block j for query tile q (0 if the tile lies past the shard end).
__device__ __forceinline__ int tiles_for(const Layout32& L, int causal, const ItemGeom& G, int q, int j) {
    if (G.a0[q] >= L.S_loc) return 0;
    return (visible_keys(L, causal, G.i, G.last[q], j) + kN - 1) / kN;
}

// Flat sequence of (step, key tile) pairs of one item, skipping dead steps.
struct TileIter {
    int s, s_end, kt, nt0, nt1, j;
    bool valid;
    __device__ __forceinline__ void load_step(const Layout32& L, int causal, const ItemGeom& G) {
        for (; s < s_end; ++s) {
            j = ring_block32(G.i, s, L.N);
            nt0 = tiles_for(L, causal, G, 0, j);
            nt1 = tiles_for(L, causal, G, 1, j);
            if (nt0 > 0 || nt1 > 0) {
                valid = true;
                return;
            }
        }
        valid = false;
    }
    __device__ __forceinline__ void init(const AttnArgs& A, const Layout32& L, const ItemGeom& G) {
        s = A.s_begin;
        s_end = A.s_end;
        kt = 0;
        load_step(L, A.causal, G);
    }
    __device__ __forceinline__ void next(const Layout32& L, int causal, const ItemGeom& G) {
        if (++kt >= (nt0 > nt1 ? nt0 : nt1)) {
            kt = 0;
            ++s;
            load_step(L, causal, G);
        }
    }
    __device__ __forceinline__ bool act(int q) const { return kt < (q ? nt1 : nt0); }
};

__device__ __forceinline__ void give_up(volatile int* abort, int* status) {
    *abort = 1;
    atomicExch(status, RA_ERR_DEVICE_TIMEOUT);
}

// Order uses of r[] after the asynchronous TMEM load has landed.
__device__ __forceinline__ void tmem_wait_ld_regs16(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                   "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                   "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                   "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

template <int kD, bool kVarlen>
struct Roles {
    TcSmem<kD>& sm;
    const AttnArgs& A;
    const int4* __restrict__ items;
    int n_items;
    uint64_t timeout;
    int* status;
    volatile int* abort;
    uint32_t tmem;
    Layout32 L;
    int* counter;  // next work item of this launch (zeroed by the host before the launch)

    // ------------------------------------------------------------ TMA producer (one warp, converged;
    // lane 0 takes work items and issues the copies)
    __device__ void producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                             const CUtensorMap* tm_v, int debug) {
        const bool leader = (threadIdx.x & 31) == 0;
        uint32_t tile_it = 0, q_it = 0, armed = 0;
        bool ok = true;
        auto wait = [&](uint64_t* bar, uint32_t parity) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar, parity, timeout, abort));
            return ok;
        };
        // Dynamic schedule: take the next item from the launch-wide counter and publish its index
        // to the other roles through a two-entry ring (index -1 ends the loop).
        for (uint32_t k = 0; ok; ++k) {
            const uint32_t b = k & 1;
            if (!wait(&sm.item_empty[b], ((k >> 1) & 1) ^ 1)) break;
            int idx = 0;
            if (leader) {
                idx = atomicAdd(counter, 1);
                if (idx >= n_items) idx = -1;
                sm.item_idx[b] = idx;
                mbar_arrive(&sm.item_full[b]);
            }
            idx = __shfl_sync(0xffffffffu, idx, 0);
            if (idx < 0) break;
            const ItemGeom G = item_geom<kVarlen>(A, L, items[idx]);
            TileIter t;
            t.init(A, G.L, G);
            if (!t.valid) continue;
            if (debug == RA_DEBUG_STALL_LOADS) continue;  // consumers must time out
            if (!wait(&sm.q_empty, (q_it & 1) ^ 1)) break;
            if (leader) {
                mbar_arrive_expect_tx(&sm.q_full, 2 * TcSmem<kD>::kTileBytes);
                for (int q = 0; q < 2; ++q) {
                    const int2 rc = tma_rows<kVarlen>(A, G, G.i, G.a0[q]);
                    for (int cb = 0; cb < kD / 64; ++cb)
                        tma_load_5d(sm.q[q] + cb * kColBlockBytes, tm_q, &sm.q_full, cb * 64, G.h, rc.x,
                                    rc.y, G.b);
                }
            }
            ++q_it;
            for (; t.valid && ok; t.next(G.L, A.causal, G)) {
                uint64_t* full = &sm.kv_full[tile_it & 1];
                for (int w = 0; w < 2; ++w) {  // K then V of this tile, each as soon as its slot frees
                    const uint32_t use = 2 * tile_it + w;
                    const uint32_t slot = use % kSlots;
                    if (!wait(&sm.slot_empty[slot], ((use / kSlots) & 1) ^ 1)) break;
                    if (w == 0) armed = tile_it + 1;
                    if (leader) {
                        if (w == 0) mbar_arrive_expect_tx(full, 2 * TcSmem<kD>::kTileBytes);
                        const int2 rc = tma_rows<kVarlen>(A, G, t.j, t.kt * kN);
                        for (int cb = 0; cb < kD / 64; ++cb)
                            tma_load_5d(sm.kv[slot] + cb * kColBlockBytes, w ? tm_v : tm_k, full, cb * 64,
                                        G.h, rc.x, rc.y, G.b);
                    }
                }
                if (ok) ++tile_it;
            }
        }
        if (!ok) {
            if (leader) give_up(abort, status);
            // let the copies already issued land before the CTA can exit (if the last tile's V
            // copy was never issued, its wait runs out after the K copy has landed)
            if (tile_it > 0) mbar_wait(&sm.kv_full[(tile_it - 1) & 1], ((tile_it - 1) >> 1) & 1, timeout, nullptr);
            if (armed > tile_it) mbar_wait(&sm.kv_full[tile_it & 1], (tile_it >> 1) & 1, timeout, nullptr);
            if (q_it > 0) mbar_wait(&sm.q_full, (q_it - 1) & 1, timeout, nullptr);
        }
    }

    // ------------------------------------------------------------ MMA issuer (one warp, converged;
    // the elected lane issues every MMA and commit)
    __device__ void issue_s(int q, uint32_t kslot) {
        constexpr uint32_t idesc = idesc_bf16_f32(kM, kN, 0, 0);
        const uint32_t qa = smem_addr(sm.q[q]), ka = smem_addr(sm.kv[kslot]);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kColBlockBytes + (kk & 3) * 32;
            warp_mma_ss(tmem + s_col(q), smem_desc_sw128(qa + off, 16, 1024),
                   smem_desc_sw128(ka + off, 16, 1024), idesc, kk > 0);
        }
        warp_mma_commit(&sm.s_full[q]);
    }

    // O_q (+)= P_q V for the keys [16 * kk0, 16 * kk1) of the tile
    template <int kk0, int kk1>
    __device__ void issue_pv(int q, uint32_t vslot, bool accumulate) {
        constexpr uint32_t idesc = idesc_bf16_f32(kM, kD, 0, 1);  // V is MN-major (D fastest)
        const uint32_t va = smem_addr(sm.kv[vslot]);
#pragma unroll
        for (int kk = kk0; kk < kk1; ++kk) {
            // 16 keys = 16 rows of 128 B of every column block; P: 16 bf16 = 8 TMEM columns
            warp_mma_ts(tmem + o_col<kD>(q), tmem + s_col(q) + kk * 8,
                   smem_desc_sw128(va + kk * 16 * 128, kColBlockBytes, 1024), idesc,
                   (kk > 0 || accumulate) ? 1u : 0u);
        }
    }

    __device__ void mma() {
        uint32_t tile_it = 0, q_it = 0, p_cnt[2] = {0, 0}, act_items[2] = {0, 0};
        bool ok = true;
        const bool leader = (threadIdx.x & 31) == 0;
        auto wait = [&](uint64_t* bar, uint32_t parity) {
            if (!ok) return false;
            ok = __all_sync(0xffffffffu, mbar_wait(bar, parity, timeout, abort));
            if (ok) tc_fence_after();
            return ok;
        };
        auto& wait_tma = wait;  // K/V/Q tiles landed (TMA)
        for (uint32_t k = 0; ok; ++k) {
            const uint32_t b = k & 1;
            if (!wait(&sm.item_full[b], (k >> 1) & 1)) break;
            const int idx = sm.item_idx[b];
            __syncwarp();
            if (leader) mbar_arrive(&sm.item_empty[b]);
            if (idx < 0) break;
            const ItemGeom G = item_geom<kVarlen>(A, L, items[idx]);
            TileIter cur;
            cur.init(A, G.L, G);
            if (!cur.valid) continue;
            if (!wait_tma(&sm.q_full, q_it & 1)) break;
            ++q_it;
            bool first_pv[2] = {true, true}, any_act[2] = {false, false};
            // one wait per key tile: K and V of tile n complete the same barrier
            if (!wait_tma(&sm.kv_full[tile_it & 1], (tile_it >> 1) & 1)) break;
            uint32_t kslot = (2 * tile_it) % kSlots;
            for (int q = 0; q < 2; ++q)
                if (cur.act(q)) {
                    issue_s(q, kslot);
                    any_act[q] = true;
                }
            warp_mma_commit(&sm.slot_empty[kslot]);
            TileIter nxt = cur;
            nxt.next(G.L, A.causal, G);
            if (!nxt.valid) warp_mma_commit(&sm.q_empty);
            for (;;) {
                const uint32_t vslot = (2 * tile_it + 1) % kSlots;  // landed with K of this tile
                for (int q = 0; q < 2; ++q) {
                    if (cur.act(q)) {
                        // P V in two halves: keys 0..63 as soon as their P is stored, while the
                        // softmax warps still work on keys 64..127
                        if (!wait(&sm.p_half[q], p_cnt[q] & 1)) break;
                        if (first_pv[q] && act_items[q] > 0 &&
                            !wait(&sm.o_free[q], (act_items[q] - 1) & 1))
                            break;
                        issue_pv<0, kN / 32>(q, vslot, !first_pv[q]);
                        if (!wait(&sm.p_full[q], p_cnt[q] & 1)) break;
                        ++p_cnt[q];
                        issue_pv<kN / 32, kN / 16>(q, vslot, true);
                        first_pv[q] = false;
                    }
                    if (q == 0 && nxt.valid) {
                        if (!wait_tma(&sm.kv_full[(tile_it + 1) & 1], ((tile_it + 1) >> 1) & 1)) break;
                        kslot = (2 * (tile_it + 1)) % kSlots;
                        if (nxt.act(0)) {
                            issue_s(0, kslot);
                            any_act[0] = true;
                        }
                    }
                }
                if (!ok) break;
                warp_mma_commit(&sm.slot_empty[vslot]);
                if (!nxt.valid) break;
                if (nxt.act(1)) {
                    issue_s(1, kslot);
                    any_act[1] = true;
                }
                warp_mma_commit(&sm.slot_empty[kslot]);
                cur = nxt;
                ++tile_it;
                nxt.next(G.L, A.causal, G);
                if (!nxt.valid) warp_mma_commit(&sm.q_empty);
            }
            if (!ok) break;
            ++tile_it;  // past the item's last key tile
            for (int q = 0; q < 2; ++q)
                if (any_act[q]) {
                    warp_mma_commit(&sm.o_final[q]);
                    ++act_items[q];
                }
        }
        if (!ok) {
            if (leader) give_up(abort, status);
            warp_mma_commit(&sm.drain);  // every MMA issued so far has finished once this arrives
            mbar_wait(&sm.drain, 0, timeout, nullptr);
        }
    }

    // ------------------------------------------------------------ softmax + epilogue (128 threads per tile)
    __device__ void softmax(int q, int warp, int row) {
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t tS = lane_base + s_col(q), tO = lane_base + o_col<kD>(q);
        const float sl2 = A.scale * kLog2e;
        uint32_t s_cnt = 0, items_act = 0;
        bool ok = true;
        auto wait_all = [&](uint64_t* bar, uint32_t parity) {
            bool w = mbar_wait(bar, parity, timeout, abort);
            ok = __all_sync(0xffffffffu, w);
            if (ok) tc_fence_after();
            return ok;
        };
        for (uint32_t k = 0; ok; ++k) {
            const uint32_t b = k & 1;
            if (!wait_all(&sm.item_full[b], (k >> 1) & 1)) break;
            const int idx = sm.item_idx[b];
            __syncwarp();
            if ((threadIdx.x & 31) == 0) mbar_arrive(&sm.item_empty[b]);
            if (idx < 0) break;
            const ItemGeom G = item_geom<kVarlen>(A, L, items[idx]);
            const int a = G.a0[q] + row;
            float m_run = -INFINITY, l = 0.f;
            int n_act = 0;
            bool frozen = false;  // the row max of this warp's rows stays fixed (see kFreezeLog2)
            for (int s = A.s_begin; s < A.s_end && ok; ++s) {
                const int j = ring_block32(G.i, s, G.L.N);
                const int nt = tiles_for(G.L, A.causal, G, q, j);
                if (nt == 0) continue;
                const int cnt = visible_keys(G.L, A.causal, G.i, a, j);
                // One key tile.  Compiled twice: with the row max and the lazy rescale, and -- once the
                // warp's max is frozen -- without them, so that each copy keeps its own registers.
                auto tile = [&](auto frozen_tag, int kt) -> bool {
                    constexpr bool kFrozen = decltype(frozen_tag)::value;
                    if constexpr (kFrozen) {
                        // Frozen max: no row max and no rescale, so S need not be held whole.  It is
                        // read from TMEM 32 columns at a time, each read issued while the previous
                        // chunk's exponentials run; P of chunk c goes to columns [16c, 16c + 16), which
                        // only chunks already read occupied.
                        if (!wait_all(&sm.s_full[q], s_cnt & 1)) return false;
                        ++s_cnt;
                        const int valid = cnt - kt * kN;
                        const uint64_t scale2 = f32x2(sl2, sl2), neg_m2 = f32x2(-m_run, -m_run);
                        uint64_t lsum[4] = {0, 0, 0, 0};
                        uint32_t ca[32], cb[32];
                        tmem_ld32(tS, ca);
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4) {
                            uint32_t(&cur)[32] = (c4 & 1) ? cb : ca;
                            uint32_t(&nxt)[32] = (c4 & 1) ? ca : cb;
                            tmem_wait_ld_regs(cur);
                            if (c4 < 3) tmem_ld32(tS + (c4 + 1) * 32, nxt);
                            if (valid < (c4 + 1) * 32) {
#pragma unroll
                                for (int x = 0; x < 32; ++x)
                                    if (c4 * 32 + x >= valid) cur[x] = kNegInfBits;
                            }
                            uint32_t pk[16];
#pragma unroll
                            for (int x = 0; x < 16; ++x) {
                                const uint64_t t2 = fma_f32x2(f32x2(__uint_as_float(cur[2 * x]), __uint_as_float(cur[2 * x + 1])),
                                                              scale2, neg_m2);
                                float t0, t1;
                                split_f32x2(t2, t0, t1);
                                const uint64_t p2 = f32x2(ex2(t0), ex2(t1));
                                lsum[x & 3] = add_f32x2(lsum[x & 3], p2);
                                float p0, p1;
                                split_f32x2(p2, p0, p1);
                                pk[x] = pack_bf16x2(p0, p1);
                            }
                            tmem_st16(tS + c4 * 16, pk);
                            if (c4 == 1) {  // P of keys 0..63 visible to the MMA
                                tmem_wait_st();
                                tc_fence_before();
                                __syncwarp();
                                if ((threadIdx.x & 31) == 0) mbar_arrive(&sm.p_half[q]);
                            }
                        }
                        float a0, a1;
                        split_f32x2(add_f32x2(add_f32x2(lsum[0], lsum[1]), add_f32x2(lsum[2], lsum[3])), a0, a1);
                        l += a0 + a1;
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if ((threadIdx.x & 31) == 0) mbar_arrive(&sm.p_full[q]);
                        return true;
                    } else {
                    if (!wait_all(&sm.s_full[q], s_cnt & 1)) return false;
                    ++s_cnt;
                    uint32_t r[128];
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        tmem_wait_ld_regs(*reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
                    const int valid = cnt - kt * kN;
                    if (valid < kN) {
#pragma unroll
                        for (int c = 0; c < kN; ++c)
                            if (c >= valid) r[c] = kNegInfBits;
                    }
#define SF(c) __uint_as_float(r[(c)])
                    // row max, 8 chains of three-input max (not computed once the warp's max is frozen)
                    float m_new = m_run;
                    if (!kFrozen) {
                    float mc[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) mc[k] = fmax3(SF(k), SF(k + 8), SF(k + 16));
#pragma unroll
                    for (int c = 24; c < 120; c += 16)
#pragma unroll
                        for (int k = 0; k < 8; ++k) mc[k] = fmax3(mc[k], SF(c + k), SF(c + k + 8));
#pragma unroll
                    for (int k = 0; k < 8; ++k) mc[k] = fmaxf(mc[k], SF(120 + k));
                    const float mx = fmax3(fmax3(mc[0], mc[1], mc[2]), fmax3(mc[3], mc[4], mc[5]),
                                           fmaxf(mc[6], mc[7]));
                    m_new = fmaxf(m_run, mx * sl2);
                    }
                    bool rescale = false;
                    float alpha = 1.f;
                    if (n_act == 0) {
                        m_run = m_new;
                    } else if (m_new > m_run + kRescaleLog2) {
                        alpha = ex2(m_run - m_new);
                        rescale = true;
                        l *= alpha;
                        m_run = m_new;
                    }
                    // rescale O before any P V of this tile accumulates into it (P_q V of the
                    // previous tile is complete: S_q of this tile was issued after it)
                    if (!kFrozen && __any_sync(0xffffffffu, rescale)) {
                        const uint64_t alpha2 = f32x2(alpha, alpha);
#pragma unroll 1
                        for (int c = 0; c < kD / 16; ++c) {  // 16 columns at a time: all of S is still live
                            uint32_t o[16];
                            tmem_ld16(tO + c * 16, o);
                            tmem_wait_ld_regs16(o);
#pragma unroll
                            for (int x = 0; x < 8; ++x) {
                                float v0, v1;
                                split_f32x2(mul_f32x2(f32x2(__uint_as_float(o[2 * x]), __uint_as_float(o[2 * x + 1])), alpha2), v0, v1);
                                o[2 * x] = __float_as_uint(v0);
                                o[2 * x + 1] = __float_as_uint(v1);
                            }
                            tmem_st16(tO + c * 16, o);
                        }
                    }
                    const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
                    // P = 2^(S * scale * log2 e - m), two columns per packed op; every
                    // kExp2PolyEvery-th pair on the FMA pipe, the rest on MUFU
                    const uint64_t scale2 = f32x2(sl2, sl2), neg_m2 = f32x2(-m_use, -m_use);
                    uint64_t lsum[4] = {0, 0, 0, 0};
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        uint32_t pk[16];
#pragma unroll
                        for (int x = 0; x < 16; ++x) {
                            const int c = c4 * 32 + 2 * x;
                            const uint64_t t2 = fma_f32x2(f32x2(SF(c), SF(c + 1)), scale2, neg_m2);
                            uint64_t p2;
                            if (kExp2PolyEvery > 0 && (x % kExp2PolyEvery) == kExp2PolyEvery - 1) {
                                p2 = exp2_poly_f32x2(t2);
                            } else {
                                float t0, t1;
                                split_f32x2(t2, t0, t1);
                                p2 = f32x2(ex2(t0), ex2(t1));
                            }
                            lsum[x & 3] = add_f32x2(lsum[x & 3], p2);
                            float p0, p1;
                            split_f32x2(p2, p0, p1);
                            pk[x] = pack_bf16x2(p0, p1);
                        }
                        tmem_st16(tS + c4 * 16, pk);
                        if (c4 == 1) {  // P of keys 0..63 (and any rescaled O) visible to the MMA
                            tmem_wait_st();
                            tc_fence_before();
                            __syncwarp();
                            if ((threadIdx.x & 31) == 0) mbar_arrive(&sm.p_half[q]);
                        }
                    }
                    {
                        float a0, a1, b0, b1;
                        split_f32x2(add_f32x2(add_f32x2(lsum[0], lsum[1]), add_f32x2(lsum[2], lsum[3])), a0, a1);
                        (void)b0;
                        (void)b1;
                        l += a0 + a1;
                    }
#undef SF
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if ((threadIdx.x & 31) == 0) mbar_arrive(&sm.p_full[q]);
                    return true;
                    }
                };
                for (int kt = 0; kt < nt && ok; ++kt) {
                    const bool done = frozen ? tile(std::true_type{}, kt) : tile(std::false_type{}, kt);
                    if (!done) break;
                    if (n_act == 0 && A.kmax) {
                        // after the first tile: the score bound of every row of this head, log2 units
                        // (Cauchy-Schwarz with the head's largest query and key norms), against the
                        // max each row has now
                        const int bh = kVarlen ? G.h : G.b * (int)A.H + G.h;
                        const float bound = __ldg(A.qmax + bh) * __ldg(A.kmax + bh) * sl2 * kBoundSlack;
                        frozen = __all_sync(0xffffffffu, bound - m_run <= kFreezeLog2);
                    }
                    ++n_act;
                }
            }
            if (!ok) break;
            epilogue(q, G, a, n_act, m_run, l, tO, ok, wait_all, items_act);
        }
        if (!ok) give_up(abort, status);
    }

    template <typename Wait>
    __device__ void epilogue(int q, const ItemGeom& G, int a, int n_act, float m_run, float l,
                             uint32_t tO, bool& ok, Wait& wait_all, uint32_t& items_act) {
        const bool row_ok = a < G.L.S_loc;
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        const float lse = l > 0.f ? (m_run + log2f(l)) * kLn2 : -INFINITY;
        const int64_t H = A.H, S = A.L.S;
        float* lse_dst;
        uint8_t* row_dst;
        if (A.out_mode == kOutFinal) {
            // token on the (packed) axis: the sequence's first token plus the position inside it
            const int64_t g = G.base + (row_ok ? global_position(G.L, G.i, a) : 0);
            row_dst = static_cast<uint8_t*>(A.out) + (((G.b * S + g) * H + G.h) * kD) * 2;
            lse_dst = A.lse + (G.b * H + G.h) * S + g;
        } else {
            // packed sequences: natural packed rows; batch mode: shard-major (local rows for a ring
            // step on local buffers)
            const int64_t rr = kVarlen ? (G.base + (row_ok ? global_position(G.L, G.i, a) : 0)) * H + G.h
                               : A.local ? ((int64_t)G.b * G.L.S_loc + a) * H + G.h
                                         : (((int64_t)G.b * G.L.N + G.i) * G.L.S_loc + a) * H + G.h;
            row_dst = static_cast<uint8_t*>(A.out) + rr * kD * 4;
            lse_dst = A.lse + rr;
        }
        if (n_act > 0) {
            if (!wait_all(&sm.o_final[q], items_act & 1)) return;
            ++items_act;
#pragma unroll 1
            for (int c = 0; c < kD / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(tO + c * 32, o);
                tmem_wait_ld_regs(o);
                if (row_ok) store_chunk(row_dst, c, o, inv_l);
            }
            tc_fence_before();
            __syncwarp();
            if ((threadIdx.x & 31) == 0) mbar_arrive(&sm.o_free[q]);
        } else if (row_ok) {
            uint32_t o[32];
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] = 0u;
            for (int c = 0; c < kD / 32; ++c) store_chunk(row_dst, c, o, 0.f);
        }
        if (row_ok) *lse_dst = lse;
    }

    __device__ __forceinline__ void store_chunk(uint8_t* row_dst, int c, const uint32_t (&o)[32],
                                                float inv_l) {
        if (A.out_mode == kOutFinal) {  // bf16, 32 values = 64 bytes
            uint4* dst = reinterpret_cast<uint4*>(row_dst + c * 64);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                uint4 u;
                u.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l);
                u.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l);
                u.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l);
                u.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l);
                dst[v] = u;
            }
        } else {  // fp32, 32 values = 128 bytes
            float4* dst = reinterpret_cast<float4*>(row_dst + c * 128);
#pragma unroll
            for (int v = 0; v < 8; ++v)
                dst[v] = make_float4(__uint_as_float(o[4 * v + 0]) * inv_l, __uint_as_float(o[4 * v + 1]) * inv_l,
                                     __uint_as_float(o[4 * v + 2]) * inv_l, __uint_as_float(o[4 * v + 3]) * inv_l);
        }
    }
};

template <int kD, bool kVarlen>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnArgs A,
                   const int4* __restrict__ items, int n_items, int* counter, uint64_t timeout_ns,
                   int debug, int* status) {
    extern __shared__ uint8_t smem_raw[];
    TcSmem<kD>& sm = *reinterpret_cast<TcSmem<kD>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&sm.q_full, 1);
        mbar_init(&sm.q_empty, 1);
        mbar_init(&sm.drain, 1);
        mbar_init(&sm.kv_full[0], 1);
        mbar_init(&sm.kv_full[1], 1);
        for (int k = 0; k < kSlots; ++k) mbar_init(&sm.slot_empty[k], 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.item_full[b], 1);
            mbar_init(&sm.item_empty[b], 9);  // one lane of the MMA warp and of each softmax warp
        }
        for (int q = 0; q < 2; ++q) {
            mbar_init(&sm.s_full[q], 1);
            mbar_init(&sm.p_half[q], 4);  // one arrival per softmax warp
            mbar_init(&sm.p_full[q], 4);
            mbar_init(&sm.o_final[q], 1);
            mbar_init(&sm.o_free[q], 4);
        }
        sm.abort = 0;
        fence_barrier_init();
    }
    if (warp == kLoadWarp && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    Roles<kD, kVarlen> roles{sm, A, items, n_items, timeout_ns, status, &sm.abort, sm.tmem_base, narrow(A.L), counter};
    if (warp >= 8) {
        setmaxnreg_dec<kRegsOther>();
        if (warp == kLoadWarp) {
            roles.producer(&tm_q, &tm_k, &tm_v, debug);
            __syncwarp();
        } else if (warp == kMmaWarp) {
            roles.mma();
            __syncwarp();
        }
    } else {
        setmaxnreg_inc<kRegsSoftmax>();
        roles.softmax(warp >> 2, warp, threadIdx.x & 127);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(sm.tmem_base, kTmemCols);
    }
}

}  // namespace

cudaError_t preload_attn_tc() {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, attn_tc_kernel<64, false>);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, attn_tc_kernel<128, false>);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, attn_tc_kernel<64, true>);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, attn_tc_kernel<128, true>);
    return e;
}

size_t tc_smem_bytes(int64_t D) {
    return (D == 64 ? sizeof(TcSmem<64>) : sizeof(TcSmem<128>)) + 1024;
}

cudaError_t launch_attn_tc(const AttnArgs& a, const TcLaunch& t, cudaStream_t stream) {
    if (t.n_items == 0) return cudaSuccess;
    const size_t smem = tc_smem_bytes(a.D);
    auto kern = a.seqs ? ((a.D == 64) ? attn_tc_kernel<64, true> : attn_tc_kernel<128, true>)
                       : ((a.D == 64) ? attn_tc_kernel<64, false> : attn_tc_kernel<128, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<t.grid, kThreads, smem, stream>>>(t.tm_q, t.tm_k, t.tm_v, a, t.items, t.n_items, t.counter,
                                             t.timeout_ns, t.debug, t.status);
    return cudaGetLastError();
}

}  // namespace ra
