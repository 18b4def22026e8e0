// ra_oracle.cpp -- fp64 CPU oracle for exact softmax attention and its ring-order form.
//
// TEST INFRASTRUCTURE ONLY.  This file is the correctness yardstick for the CUDA library in
// long_context_exact_forward_b200/.  It shares no code, header, table or helper with that
// library, and neither side includes or links the other.  Only the test suite, the smoke check
// and the CPU-baseline leg of the benchmark load it.
//
// What it computes (sources are the five web pages on Ring Attention):
//   * ora_attention      -- the plain definition softmax(Q K^T / sqrt(D)) V with an optional causal
//                            mask, one query row at a time, in fp64 with no blocking.  Ring
//                            Attention is stated to produce exactly full attention
//                            ("Sequence Parallelism and Ring Attention", aiunderstanding.org,
//                            "Teknisk insikt"; troisinh.com "Ring Attention", "Tai sao no hoat
//                            dong"; ultralytics.com "Ring Attention", section "how ring attention
//                            works"), so the definition is the oracle.
//   * ora_ring_blockwise -- the ring loop of the ultralytics.com toy (device i keeps query block i,
//                            at step s it holds key/value block j = (i - s) mod N, accumulates a
//                            numerator and a denominator, divides at the end) written with the
//                            running-max subtraction that the same page says production kernels
//                            use, and with the token layouts (contiguous / striped / zigzag).
//                            Self-check companion; it is compared against ora_attention.
//   * ora_merge          -- the online-softmax merge identities of troisinh.com "Ring Attention",
//                            section "Tai sao no hoat dong": m' = max(m_p, m_n),
//                            l' = e^{m_p - m'} l_p + e^{m_n - m'} l_n, output rescaled alike.
//   * ora_attention_backward -- the gradients dQ, dK, dV of the same plain definition for an
//                            upstream gradient dO (troisinh.com "Ring Attention", "Blockwise
//                            Backward": the backward pass recomputes the attention statistics
//                            instead of storing the S x S weights).  Written out by the chain rule
//                            with no blocking: P = softmax(S), dV = P^T dO, dP = dO V^T,
//                            dS = P * (dP - rowsum(P * dP)), dQ = dS K / sqrt(D),
//                            dK = dS^T Q / sqrt(D).
//   * ora_attention_varlen -- the plain definition for several sequences packed one after another
//                            along the token axis: a query attends only to keys of its own sequence
//                            (and, causal, at or before its own position).  troisinh.com "Ring
//                            Attention", "Trade-off thuc te" (Complexity) names load balancing
//                            with sequences of different lengths as a challenge; the result is
//                            still exact attention per sequence, which is what this writes out.
//   * ora_rope           -- rotary position embedding applied with each token's GLOBAL position m
//                            (troisinh.com "Ring Attention", "RoPE va Position Embedding": when K/V
//                            travel round the ring, each position m must still be rotated by the
//                            angle m theta).  Reading: the pairs (x[2p], x[2p+1]) of the head dim are
//                            rotated by m theta_p with theta_p = base^(-2p/D), the original
//                            rotary embedding, base 10000 by default.
//
// Readings where the pages are silent (listed again in the design notes):
//   * scale = 1/sqrt(D) (the toy divides the scores by dim**0.5);
//   * the causal mask is on ORIGINAL token positions with the diagonal included (key g_k <= g_q);
//   * lse is the natural-log log-sum-exp of the scaled scores: lse = m + ln(l);
//   * striped: token g lives on shard g mod N at local index g / N;
//     zigzag: 2N chunks of C = S/(2N) tokens, shard i holds chunk i then chunk 2N-1-i.
//
// Tensors are [B, S, H, D] row-major in natural token order; lse is [B, H, S].
// Input element types: 0 = fp32, 1 = bf16 (raw 16-bit patterns), 2 = fp64.  Every conversion to
// fp64 is exact, so input quantisation is never counted as error.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

double to_f64(const void* base, int dtype, int64_t idx) {
    if (dtype == 0) return (double)static_cast<const float*>(base)[idx];
    if (dtype == 1) {
        // a bf16 value is the top half of the fp32 with the same bits
        uint32_t bits = (uint32_t)static_cast<const uint16_t*>(base)[idx] << 16;
        float f;
        std::memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    return static_cast<const double*>(base)[idx];
}

// index of element [b, s, h, d] in a [B, S, H, D] tensor
int64_t at(int64_t b, int64_t s, int64_t h, int64_t d, int64_t S, int64_t H, int64_t D) {
    return ((b * S + s) * H + h) * D + d;
}

// One query row of the plain definition: scores over every allowed key, max, normaliser,
// weighted sum of values, division.  Single-threaded and unblocked.
void attend_one_row(const void* q, const void* k, const void* v, int dtype,
                    int64_t S, int64_t H, int64_t D, int64_t b, int64_t h, int64_t r,
                    int causal, std::vector<double>& qrow, std::vector<double>& scores,
                    double* out_row, double* lse_out) {
    const double scale = 1.0 / std::sqrt((double)D);
    for (int64_t d = 0; d < D; ++d) qrow[d] = to_f64(q, dtype, at(b, r, h, d, S, H, D));
    const int64_t n_keys = causal ? r + 1 : S;  // keys c with c <= r when causal
    double m = -std::numeric_limits<double>::infinity();
    for (int64_t c = 0; c < n_keys; ++c) {
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += qrow[d] * to_f64(k, dtype, at(b, c, h, d, S, H, D));
        scores[c] = scale * dot;
        m = std::max(m, scores[c]);
    }
    double l = 0.0;
    for (int64_t d = 0; d < D; ++d) out_row[d] = 0.0;
    for (int64_t c = 0; c < n_keys; ++c) {
        const double p = std::exp(scores[c] - m);
        l += p;
        for (int64_t d = 0; d < D; ++d) out_row[d] += p * to_f64(v, dtype, at(b, c, h, d, S, H, D));
    }
    for (int64_t d = 0; d < D; ++d) out_row[d] /= l;
    *lse_out = m + std::log(l);
}

// Global position of local token a on shard i (the layout readings above).
int64_t global_pos(int layout, int64_t i, int64_t a, int64_t S, int64_t N) {
    const int64_t S_loc = S / N;
    if (layout == 0) return i * S_loc + a;            // contiguous chunks
    if (layout == 1) return a * N + i;                // striped: round robin
    const int64_t C = S / (2 * N);                    // zigzag: chunks i and 2N-1-i
    return a < C ? i * C + a : (2 * N - 1 - i) * C + (a - C);
}

}  // namespace

extern "C" {

// Plain definition on a chosen set of query rows.
//   rows: [B*H, n_rows] natural-order query positions for each (b, h) (row-major over b then h);
//         NULL means every row 0..S-1 (n_rows must then equal S).
//   out:  [B*H, n_rows, D] fp64;  lse: [B*H, n_rows] fp64.
//   threads: host threads; each runs the unchanged single-threaded row routine on whole rows,
//            so results do not depend on the thread count.
// Returns 0, or -1 on a bad argument.
int ora_attention(const void* q, const void* k, const void* v, int dtype, int64_t B, int64_t H,
                  int64_t S, int64_t D, int causal, const int64_t* rows, int64_t n_rows,
                  double* out, double* lse, int threads) {
    if (!q || !k || !v || !out || !lse || B < 0 || H < 0 || S < 0 || D <= 0 || n_rows < 0) return -1;
    if (dtype < 0 || dtype > 2) return -1;
    if (!rows && n_rows != S) return -1;
    if (rows) {
        for (int64_t t = 0; t < B * H * n_rows; ++t)
            if (rows[t] < 0 || rows[t] >= S) return -1;
    }
    const int64_t total = B * H * n_rows;
    std::atomic<int64_t> next{0};
    auto worker = [&]() {
        std::vector<double> qrow(D), scores(std::max<int64_t>(S, 1));
        for (;;) {
            const int64_t t = next.fetch_add(1);
            if (t >= total) break;
            const int64_t bh = t / n_rows, n = t % n_rows;
            const int64_t b = bh / H, h = bh % H;
            const int64_t r = rows ? rows[t] : n;
            attend_one_row(q, k, v, dtype, S, H, D, b, h, r, causal, qrow, scores, out + t * D,
                           lse + t);
        }
    };
    threads = std::max(1, threads);
    if (threads == 1) {
        worker();
    } else {
        std::vector<std::thread> pool;
        for (int t = 0; t < threads; ++t) pool.emplace_back(worker);
        for (auto& th : pool) th.join();
    }
    return 0;
}

// Merge identities for n rows of running statistics (m, l, O) with a second set (m2, l2, O2):
// m' = max(m, m2), l' = e^{m - m'} l + e^{m2 - m'} l2, O' = e^{m - m'} O + e^{m2 - m'} O2.
// Here O is the UN-normalised accumulator (sum of e^{s - m} v).  A side with l = 0 and m = -inf
// is empty and contributes nothing.  Results overwrite (m, l, O).
void ora_merge(int64_t n, int64_t D, double* m, double* l, double* O, const double* m2,
               const double* l2, const double* O2) {
    for (int64_t r = 0; r < n; ++r) {
        const double mp = m[r], mn = m2[r];
        const double mu = std::max(mp, mn);
        if (mu == -std::numeric_limits<double>::infinity()) continue;  // both sides empty
        const double ap = (mp == -std::numeric_limits<double>::infinity()) ? 0.0 : std::exp(mp - mu);
        const double an = (mn == -std::numeric_limits<double>::infinity()) ? 0.0 : std::exp(mn - mu);
        m[r] = mu;
        l[r] = ap * l[r] + an * l2[r];
        for (int64_t d = 0; d < D; ++d) O[r * D + d] = ap * O[r * D + d] + an * O2[r * D + d];
    }
}

// Position of every token under a layout: pos[i * S_loc + a] = global position of local token a
// on shard i.  Returns -1 when S does not split evenly (S % N, or S % 2N for zigzag).
int ora_layout_positions(int64_t S, int64_t N, int layout, int64_t* pos) {
    if (N <= 0 || S % N != 0 || layout < 0 || layout > 2) return -1;
    if (layout == 2 && S % (2 * N) != 0) return -1;
    const int64_t S_loc = S / N;
    for (int64_t i = 0; i < N; ++i)
        for (int64_t a = 0; a < S_loc; ++a) pos[i * S_loc + a] = global_pos(layout, i, a, S, N);
    return 0;
}

// The ring loop, one (b, h) at a time: shard i keeps its query block; at step s it holds the
// key/value block of shard j = (i - s) mod N, scores its queries against that block, and merges
// the block's (max, sum, weighted values) into its running (m, l, acc) with ora_merge's
// identities; after N steps it divides acc by l.  The causal mask compares global positions.
// block_pairs: if not NULL, [N * N] counts of allowed (query, key) pairs of block (shard i,
// step s) at entry i * N + s, for b = 0, h = 0 -- the per-device work at each step.
// out: [B, S, H, D] fp64 natural order; lse: [B, H, S] fp64.
int ora_ring_blockwise(const void* q, const void* k, const void* v, int dtype, int64_t B,
                       int64_t H, int64_t S, int64_t D, int64_t N, int causal, int layout,
                       double* out, double* lse, int64_t* block_pairs) {
    if (N <= 0 || S % N != 0 || layout < 0 || layout > 2 || D <= 0) return -1;
    if (layout == 2 && S % (2 * N) != 0) return -1;
    const int64_t S_loc = S / N;
    const double scale = 1.0 / std::sqrt((double)D);
    const double NEG_INF = -std::numeric_limits<double>::infinity();
    std::vector<double> qb(S_loc * D), kb(S_loc * D), vb(S_loc * D);
    std::vector<double> m(S_loc), l(S_loc), acc(S_loc * D);
    std::vector<double> bm(S_loc), bl(S_loc), bacc(S_loc * D), sc(S_loc);
    if (block_pairs)
        for (int64_t t = 0; t < N * N; ++t) block_pairs[t] = 0;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < H; ++h)
            for (int64_t i = 0; i < N; ++i) {
                // this device's query block, gathered by the layout
                for (int64_t a = 0; a < S_loc; ++a)
                    for (int64_t d = 0; d < D; ++d)
                        qb[a * D + d] = to_f64(q, dtype, at(b, global_pos(layout, i, a, S, N), h, d, S, H, D));
                std::fill(m.begin(), m.end(), NEG_INF);
                std::fill(l.begin(), l.end(), 0.0);
                std::fill(acc.begin(), acc.end(), 0.0);
                for (int64_t s = 0; s < N; ++s) {
                    const int64_t j = ((i - s) % N + N) % N;  // block that has arrived at step s
                    for (int64_t c = 0; c < S_loc; ++c)
                        for (int64_t d = 0; d < D; ++d) {
                            const int64_t gk = global_pos(layout, j, c, S, N);
                            kb[c * D + d] = to_f64(k, dtype, at(b, gk, h, d, S, H, D));
                            vb[c * D + d] = to_f64(v, dtype, at(b, gk, h, d, S, H, D));
                        }
                    // partial attention of the block: its own max, sum and weighted values
                    for (int64_t a = 0; a < S_loc; ++a) {
                        const int64_t gq = global_pos(layout, i, a, S, N);
                        double mx = NEG_INF;
                        for (int64_t c = 0; c < S_loc; ++c) {
                            const int64_t gk = global_pos(layout, j, c, S, N);
                            if (causal && gk > gq) { sc[c] = NEG_INF; continue; }
                            double dot = 0.0;
                            for (int64_t d = 0; d < D; ++d) dot += qb[a * D + d] * kb[c * D + d];
                            sc[c] = scale * dot;
                            mx = std::max(mx, sc[c]);
                            if (block_pairs && b == 0 && h == 0) block_pairs[i * N + s] += 1;
                        }
                        bm[a] = mx;
                        bl[a] = 0.0;
                        for (int64_t d = 0; d < D; ++d) bacc[a * D + d] = 0.0;
                        if (mx == NEG_INF) continue;  // nothing allowed in this block
                        for (int64_t c = 0; c < S_loc; ++c) {
                            if (sc[c] == NEG_INF) continue;
                            const double p = std::exp(sc[c] - mx);
                            bl[a] += p;
                            for (int64_t d = 0; d < D; ++d) bacc[a * D + d] += p * vb[c * D + d];
                        }
                    }
                    ora_merge(S_loc, D, m.data(), l.data(), acc.data(), bm.data(), bl.data(), bacc.data());
                }
                // divide at the end and scatter back to natural order
                for (int64_t a = 0; a < S_loc; ++a) {
                    const int64_t g = global_pos(layout, i, a, S, N);
                    for (int64_t d = 0; d < D; ++d) out[at(b, g, h, d, S, H, D)] = acc[a * D + d] / l[a];
                    lse[(b * H + h) * S + g] = m[a] + std::log(l[a]);
                }
            }
    return 0;
}

// Gradients of the plain definition.  dout, dq, dk, dv: [B, S, H, D] (dout in `dtype`, the
// gradients fp64).  Each (b, h) is one task (its dk and dv rows belong to it alone); `threads`
// host threads take whole tasks, so the result does not depend on the thread count.
// Per query row r, in the order the chain rule gives them:
//   s_c  = scale * q_r . k_c over the allowed keys c, lse_r = max + ln(sum exp(s - max))
//   P_rc = exp(s_c - lse_r)                       (the softmax row)
//   dP_rc = dO_r . v_c                            (gradient of out_r = sum_c P_rc v_c w.r.t. P_rc)
//   dS_rc = P_rc * (dP_rc - sum_c' P_rc' dP_rc')  (softmax Jacobian)
//   dq_r += scale * dS_rc k_c,  dk_c += scale * dS_rc q_r,  dv_c += P_rc dO_r
// Returns 0, or -1 on a bad argument.
int ora_attention_backward(const void* q, const void* k, const void* v, const void* dout, int dtype,
                           int64_t B, int64_t H, int64_t S, int64_t D, int causal, double* dq,
                           double* dk, double* dv, int threads) {
    if (!q || !k || !v || !dout || !dq || !dk || !dv || B < 0 || H < 0 || S < 0 || D <= 0) return -1;
    if (dtype < 0 || dtype > 2) return -1;
    const double scale = 1.0 / std::sqrt((double)D);
    const int64_t n_tasks = B * H;
    std::atomic<int64_t> next{0};
    auto worker = [&]() {
        std::vector<double> qr(D), dor(D), s(std::max<int64_t>(S, 1)), P(std::max<int64_t>(S, 1)),
            dP(std::max<int64_t>(S, 1));
        for (;;) {
            const int64_t t = next.fetch_add(1);
            if (t >= n_tasks) break;
            const int64_t b = t / H, h = t % H;
            for (int64_t r = 0; r < S; ++r)
                for (int64_t d = 0; d < D; ++d) {
                    dq[at(b, r, h, d, S, H, D)] = 0.0;
                    dk[at(b, r, h, d, S, H, D)] = 0.0;
                    dv[at(b, r, h, d, S, H, D)] = 0.0;
                }
            for (int64_t r = 0; r < S; ++r) {
                for (int64_t d = 0; d < D; ++d) {
                    qr[d] = to_f64(q, dtype, at(b, r, h, d, S, H, D));
                    dor[d] = to_f64(dout, dtype, at(b, r, h, d, S, H, D));
                }
                const int64_t n_keys = causal ? r + 1 : S;
                double m = -std::numeric_limits<double>::infinity();
                for (int64_t c = 0; c < n_keys; ++c) {
                    double dot = 0.0;
                    for (int64_t d = 0; d < D; ++d) dot += qr[d] * to_f64(k, dtype, at(b, c, h, d, S, H, D));
                    s[c] = scale * dot;
                    m = std::max(m, s[c]);
                }
                double l = 0.0;
                for (int64_t c = 0; c < n_keys; ++c) l += std::exp(s[c] - m);
                const double lse = m + std::log(l);
                double row_dot = 0.0;  // sum_c P_rc dP_rc
                for (int64_t c = 0; c < n_keys; ++c) {
                    P[c] = std::exp(s[c] - lse);
                    double dot = 0.0;
                    for (int64_t d = 0; d < D; ++d) dot += dor[d] * to_f64(v, dtype, at(b, c, h, d, S, H, D));
                    dP[c] = dot;
                    row_dot += P[c] * dP[c];
                }
                for (int64_t c = 0; c < n_keys; ++c) {
                    const double dS = P[c] * (dP[c] - row_dot);
                    for (int64_t d = 0; d < D; ++d) {
                        dq[at(b, r, h, d, S, H, D)] += scale * dS * to_f64(k, dtype, at(b, c, h, d, S, H, D));
                        dk[at(b, c, h, d, S, H, D)] += scale * dS * qr[d];
                        dv[at(b, c, h, d, S, H, D)] += P[c] * dor[d];
                    }
                }
            }
        }
    };
    const int n_threads = std::max(1, std::min<int>(threads, (int)std::max<int64_t>(n_tasks, 1)));
    std::vector<std::thread> pool;
    for (int w = 1; w < n_threads; ++w) pool.emplace_back(worker);
    worker();
    for (auto& th : pool) th.join();
    return 0;
}

// Rotary embedding of x [B, S, H, D] (dtype as above) into y (fp64), the token at natural index g
// taking the position m = g + pos_offset; D must be even.  Returns 0, or -1 on a bad argument.
int ora_rope(const void* x, int dtype, int64_t B, int64_t S, int64_t H, int64_t D, int64_t pos_offset,
             double base, double* y) {
    if (!x || !y || B < 0 || S < 0 || H < 0 || D <= 0 || (D & 1) || !(base > 0.0)) return -1;
    if (dtype < 0 || dtype > 2) return -1;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t g = 0; g < S; ++g)
            for (int64_t h = 0; h < H; ++h)
                for (int64_t p = 0; p < D / 2; ++p) {
                    const double m = (double)(g + pos_offset);
                    const double theta = std::pow(base, -2.0 * (double)p / (double)D);
                    const double c = std::cos(m * theta), sn = std::sin(m * theta);
                    const double x0 = to_f64(x, dtype, at(b, g, h, 2 * p, S, H, D));
                    const double x1 = to_f64(x, dtype, at(b, g, h, 2 * p + 1, S, H, D));
                    y[at(b, g, h, 2 * p, S, H, D)] = x0 * c - x1 * sn;
                    y[at(b, g, h, 2 * p + 1, S, H, D)] = x0 * sn + x1 * c;
                }
    return 0;
}

// Packed sequences: q, k, v [S_total, H, D] (one batch), sequence k holding tokens
// [cu[k], cu[k+1]).  out [S_total, H, D] fp64 (natural order), lse [H, S_total] fp64.  A query
// attends to the keys of its own sequence only (and, causal, to those at or before it).
// Returns 0, or -1 on a bad argument.
int ora_attention_varlen(const void* q, const void* k, const void* v, int dtype, int64_t S_total, int64_t H,
                         int64_t D, int causal, const int64_t* cu, int64_t n_seqs, double* out, double* lse,
                         int threads) {
    if (!q || !k || !v || !cu || !out || !lse || S_total < 0 || H <= 0 || D <= 0 || n_seqs < 1) return -1;
    if (dtype < 0 || dtype > 2 || cu[0] != 0 || cu[n_seqs] != S_total) return -1;
    for (int64_t s = 0; s < n_seqs; ++s)
        if (cu[s + 1] < cu[s]) return -1;
    const double scale = 1.0 / std::sqrt((double)D);
    const int64_t total = S_total * H;
    std::atomic<int64_t> next{0};
    auto worker = [&]() {
        std::vector<double> qrow(D), sc(std::max<int64_t>(S_total, 1));
        for (;;) {
            const int64_t t = next.fetch_add(1);
            if (t >= total) break;
            const int64_t r = t / H, h = t % H;
            int64_t seq = 0;
            while (cu[seq + 1] <= r) ++seq;
            const int64_t lo = cu[seq], hi = causal ? r + 1 : cu[seq + 1];
            for (int64_t d = 0; d < D; ++d) qrow[d] = to_f64(q, dtype, at(0, r, h, d, S_total, H, D));
            double m = -std::numeric_limits<double>::infinity();
            for (int64_t c = lo; c < hi; ++c) {
                double dot = 0.0;
                for (int64_t d = 0; d < D; ++d) dot += qrow[d] * to_f64(k, dtype, at(0, c, h, d, S_total, H, D));
                sc[c] = scale * dot;
                m = std::max(m, sc[c]);
            }
            double l = 0.0;
            double* o = out + (r * H + h) * D;
            for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
            for (int64_t c = lo; c < hi; ++c) {
                const double p = std::exp(sc[c] - m);
                l += p;
                for (int64_t d = 0; d < D; ++d) o[d] += p * to_f64(v, dtype, at(0, c, h, d, S_total, H, D));
            }
            for (int64_t d = 0; d < D; ++d) o[d] /= l;
            lse[h * S_total + r] = m + std::log(l);
        }
    };
    const int n_threads = std::max(1, std::min<int>(threads, (int)std::max<int64_t>(total, 1)));
    std::vector<std::thread> pool;
    for (int w = 1; w < n_threads; ++w) pool.emplace_back(worker);
    worker();
    for (auto& th : pool) th.join();
    return 0;
}

}  // extern "C"
