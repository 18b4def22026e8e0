// layout.cuh -- token layouts and causal key counts, shared by host planner and device kernels.
//
// Sequence sharding puts each shard's tokens together (aiunderstanding.org "Sequence Parallelism
// and Ring Attention": each GPU owns a contiguous piece of the tokens); the striped and zigzag
// layouts rebalance the causal work (same page, "Framtiden"; ultralytics.com "Ring Attention":
// tokens spread evenly over the sequence).
//
// Under all three layouts the global position g(i, a) of local token a on shard i is strictly
// increasing in a.  Hence for a query at global position gq, the keys of shard j it may see under
// the causal mask (g_k <= gq, diagonal included) are exactly the local PREFIX a < key_count(j, gq).
// The kernels mask with that one count per row and shard, and the block-skip scheduler derives
// tile classes (EMPTY / FULL / PARTIAL) from the counts of a tile's first and last rows.
#pragma once
#include <stdint.h>

#ifdef __CUDACC__
#define RA_HD __host__ __device__ __forceinline__
#else
#define RA_HD inline
#endif

namespace ra {

struct Layout {
    int64_t S;      // tokens
    int64_t N;      // shards (ring size)
    int64_t S_loc;  // tokens per shard
    int kind;       // 0 contiguous, 1 striped, 2 zigzag
};

RA_HD int64_t clamp64(int64_t x, int64_t lo, int64_t hi) { return x < lo ? lo : (x > hi ? hi : x); }

// Global position of local token a of shard i.
RA_HD int64_t global_position(const Layout& L, int64_t i, int64_t a) {
    if (L.kind == 0) return i * L.S_loc + a;
    if (L.kind == 1) return a * L.N + i;
    const int64_t C = L.S_loc >> 1;  // zigzag chunk
    return a < C ? i * C + a : (2 * L.N - 1 - i) * C + (a - C);
}

// Number of keys of shard j whose global position is <= gq (the causal prefix length).
RA_HD int64_t key_count(const Layout& L, int64_t j, int64_t gq) {
    if (L.kind == 0) return clamp64(gq - j * L.S_loc + 1, 0, L.S_loc);
    if (L.kind == 1) return gq < j ? 0 : clamp64((gq - j) / L.N + 1, 0, L.S_loc);
    const int64_t C = L.S_loc >> 1;
    return clamp64(gq - j * C + 1, 0, C) + clamp64(gq - (2 * L.N - 1 - j) * C + 1, 0, C);
}

// Keys of shard j visible to the query at local row a of shard i (all S_loc without causal).
// Rows past the shard end (padding of a ragged last tile) behave like the last row.
RA_HD int64_t visible_keys(const Layout& L, int causal, int64_t i, int64_t a, int64_t j) {
    if (!causal) return L.S_loc;
    if (a >= L.S_loc) a = L.S_loc - 1;
    return key_count(L, j, global_position(L, i, a));
}

// Ring order: at step s shard i holds the key/value block of shard (i - s) mod N
// (ultralytics.com "Ring Attention" toy loop; jisaku.com 処理フロー t = 0 .. N-1).
RA_HD int64_t ring_block(int64_t i, int64_t s, int64_t N) { return ((i - s) % N + N) % N; }

// Work order of the persistent kernel: when one head's keys and values (4*S*D bytes in bf16) no
// longer fit comfortably in the 126 MB L2, the items of each shard are grouped together so that CTAs
// running at the same time walk the same ring sequence of key/value blocks.
RA_HD bool plan_groups_by_shard(int64_t S, int64_t D) { return S * D * 4 > (int64_t(96) << 20); }

// 32-bit forms of the same maps for device code (the host rejects S >= 2^31, so every position,
// count and index of a shard fits in 32 bits; 32-bit division is far cheaper on the GPU).
struct Layout32 {
    int S, N, S_loc, kind;
};

RA_HD Layout32 narrow(const Layout& L) { return Layout32{(int)L.S, (int)L.N, (int)L.S_loc, L.kind}; }

RA_HD int clamp32(int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); }

RA_HD int global_position(const Layout32& L, int i, int a) {
    if (L.kind == 0) return i * L.S_loc + a;
    if (L.kind == 1) return a * L.N + i;
    const int C = L.S_loc >> 1;
    return a < C ? i * C + a : (2 * L.N - 1 - i) * C + (a - C);
}

RA_HD int key_count(const Layout32& L, int j, int gq) {
    if (L.kind == 0) return clamp32(gq - j * L.S_loc + 1, 0, L.S_loc);
    if (L.kind == 1) return gq < j ? 0 : clamp32((gq - j) / L.N + 1, 0, L.S_loc);
    const int C = L.S_loc >> 1;
    return clamp32(gq - j * C + 1, 0, C) + clamp32(gq - (2 * L.N - 1 - j) * C + 1, 0, C);
}

RA_HD int visible_keys(const Layout32& L, int causal, int i, int a, int j) {
    if (!causal) return L.S_loc;
    if (a >= L.S_loc) a = L.S_loc - 1;
    return key_count(L, j, global_position(L, i, a));
}

RA_HD int ring_block32(int i, int s, int N) { return ((i - s) % N + N) % N; }

}  // namespace ra
