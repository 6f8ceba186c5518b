// CPU oracle for SAGA + Atop-N single-token decode attention.
//
// TEST INFRASTRUCTURE ONLY. This file is the slow, obviously-correct CPU
// restatement of what the decode path computes. Only the test suite, the
// package's smoke check and the benchmark's CPU-baseline leg may load it; the
// product path never calls it and shares no code, header or table with it.
//
// Source: "More Value per Key: Asymmetric Sparse Attention for Faster LLM
// Decoding" (arXiv 2610.04753), as summarised on ai.info (sections "Key
// Contributions", "Main Findings", "Methodology in Plain English") and on
// atlas.scime.ai (sections "Approach", "Experimental setup").
//
// Notation: b batch, hq/hk/hv query/key/value heads, d head dim (dk for keys
// and queries, dv for values where they differ: the Sigma-style head layout
// of Main Findings, "Head count beats head dimension"), l cached
// positions (first l rows of a cache with capacity l_cap), N top-N budget,
// n refresh interval, t 0-based decode step.
//
// Readings taken where the pages are silent (each also listed in the design
// notes of the repository):
//   * head maps are contiguous groups: kh(i) = i*hk/hq, vh(i) = i*hv/hq
//     (the pages only say SAGA decouples hk from hv, Key Contributions #3);
//   * one threshold per (batch, query head) (Main Findings: "h_q x l_q x N
//     value vectors");
//   * the compared quantity is the scaled logit q.k/sqrt(d), kept if >= tau;
//   * ties at tau are all kept (an element-wise compare has no tie-break);
//   * N >= l gives tau = -inf (everything kept, i.e. full attention);
//   * a threshold of -0.0 is stored as +0.0;
//   * an empty kept set (every logit below a stale tau) keeps the row's
//     maximal entries: tau_eff = min(tau, max_j s_j).
//
// Precision: bf16 inputs are widened exactly; dot products accumulate in
// double and are rounded once to fp32 (the logits are fp32 on both sides);
// softmax and the value sum run in double and are rounded once to fp32.
//
// Parity pins for every function here live in tests/test_oracle.py: the
// logits against a float64 library matmul, the threshold against a full sort,
// N >= l against library softmax attention, hk == hv against grouped-query
// attention, n == 1 against exact top-N attention, sum(p) == 1, the N == 1
// argmax case, q == 0 (mean of values), permutation equivariance and a
// closed-form worked example.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <limits>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// bf16 -> fp32 is exact: the bf16 bit pattern is the top half of the fp32 one.
inline double widen_bf16(uint16_t bits) {
    uint32_t u = static_cast<uint32_t>(bits) << 16;
    float f;
    std::memcpy(&f, &u, sizeof f);
    return static_cast<double>(f);
}

// Contiguous-group head maps (reading: the pages only state that the key and
// value head counts are decoupled, SAGA in "Key Contributions" #3).
inline long key_head(long i, long hq, long hk) { return i * hk / hq; }
inline long value_head(long i, long hq, long hv) { return i * hv / hq; }

}  // namespace

extern "C" {

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

// Step 1, the query-key product (Main Findings, "bottleneck shift": the
// query-key multiplication is the step every key head pays for).
//   s[b,i,j] = fp32( sum_c q[b,i,c] * K[b,j,kh(i),c] / sqrt(d) ),  j < l.
// q: [b,hq,d] bf16 bits; K: [b,l_cap,hk,d] bf16 bits; s: [b,hq,l] fp32.
int oracle_logits(long b, long hq, long hk, long d, long l, long l_cap,
                  const uint16_t* q, const uint16_t* K, float* s) {
    if (b <= 0 || hq <= 0 || hk <= 0 || d <= 0 || l < 0 || l > l_cap) return -1;
    const double inv_sqrt_d = 1.0 / std::sqrt(static_cast<double>(d));
#pragma omp parallel for schedule(dynamic)
    for (long row = 0; row < b * hq; ++row) {
        const long bb = row / hq, i = row % hq;
        const long kh = key_head(i, hq, hk);
        const uint16_t* qi = q + (bb * hq + i) * d;
        for (long j = 0; j < l; ++j) {
            const uint16_t* kj = K + ((bb * l_cap + j) * hk + kh) * d;
            double acc = 0.0;
            for (long c = 0; c < d; ++c) acc += widen_bf16(qi[c]) * widen_bf16(kj[c]);
            s[row * l + j] = static_cast<float>(acc * inv_sqrt_d);
        }
    }
    return 0;
}

// Step 2, the exact threshold refresh (Key Contributions #2: "exact top-N
// thresholds computed once every n tokens"): tau = the N-th largest logit of
// the row, counting duplicates.  N >= l gives -inf (keep everything).
// Uses std::nth_element (a library selection).
int oracle_nth_largest(const float* s, long rows, long l, long N, float* tau) {
    if (rows < 0 || l < 0 || N <= 0) return -1;
#pragma omp parallel for schedule(dynamic)
    for (long r = 0; r < rows; ++r) {
        if (N >= l) {
            tau[r] = -std::numeric_limits<float>::infinity();
            continue;
        }
        std::vector<float> v(s + r * l, s + (r + 1) * l);
        std::nth_element(v.begin(), v.begin() + (N - 1), v.end(), std::greater<float>());
        float t = v[N - 1];
        if (t == 0.0f) t = 0.0f;  // -0.0 is stored as +0.0
        tau[r] = t;
    }
    return 0;
}

// The same threshold by brute force: sort the row descending and take the
// entry at index N-1.  Used by the tests to cross-check the selection above.
int oracle_nth_largest_sort(const float* s, long rows, long l, long N, float* tau) {
    if (rows < 0 || l < 0 || N <= 0) return -1;
    for (long r = 0; r < rows; ++r) {
        if (N >= l) {
            tau[r] = -std::numeric_limits<float>::infinity();
            continue;
        }
        std::vector<float> v(s + r * l, s + (r + 1) * l);
        std::sort(v.begin(), v.end(), std::greater<float>());
        float t = v[N - 1];
        if (t == 0.0f) t = 0.0f;
        tau[r] = t;
    }
    return 0;
}

// Step 3, selection by per-element comparison (Key Contributions #2 and
// Methodology ¶2: each logit is compared with the stored threshold; nothing
// is sorted).
//   tau_eff = min(tau, max_j s_j);  keep_j  <=>  s_j >= tau_eff.
// mask: [rows,l] bytes (1 = kept); cnt: [rows] number kept.
int oracle_select(const float* s, long rows, long l, const float* tau,
                  uint8_t* mask, int32_t* cnt) {
    if (rows < 0 || l <= 0) return -1;
#pragma omp parallel for schedule(dynamic)
    for (long r = 0; r < rows; ++r) {
        const float* sr = s + r * l;
        float m_all = sr[0];
        for (long j = 1; j < l; ++j) m_all = std::max(m_all, sr[j]);
        const float t_eff = std::min(tau[r], m_all);
        int32_t c = 0;
        for (long j = 0; j < l; ++j) {
            const bool keep = sr[j] >= t_eff;
            mask[r * l + j] = keep ? 1 : 0;
            c += keep ? 1 : 0;
        }
        cnt[r] = c;
    }
    return 0;
}

// Steps 4-5, softmax over the kept entries and the gathered value sum
// (Main Findings, "bottleneck shift": the probability-value product touches
// only the kept value vectors, h_q x N per token).  Value head vh(i).
//   m = max_kept s;  p_j = exp(s_j - m) / sum_kept exp(s_k - m);
//   o[b,i,:] = fp32( sum_kept p_j * V[b,j,vh(i),:] ).
// s: [b,hq,l]; mask: [b,hq,l]; V: [b,l_cap,hv,d] bf16 bits; out: [b,hq,d].
int oracle_attend_masked(long b, long hq, long hv, long d, long l, long l_cap,
                         const float* s, const uint8_t* mask, const uint16_t* V,
                         float* out) {
    if (b <= 0 || hq <= 0 || hv <= 0 || d <= 0 || l <= 0 || l > l_cap) return -1;
    int bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
    for (long row = 0; row < b * hq; ++row) {
        const long bb = row / hq, i = row % hq;
        const long vh = value_head(i, hq, hv);
        const float* sr = s + row * l;
        const uint8_t* mr = mask + row * l;
        double m = -std::numeric_limits<double>::infinity();
        for (long j = 0; j < l; ++j)
            if (mr[j]) m = std::max(m, static_cast<double>(sr[j]));
        if (!(m > -std::numeric_limits<double>::infinity())) {  // nothing kept
            bad |= 1;
            for (long c = 0; c < d; ++c) out[row * d + c] = std::nanf("");
            continue;
        }
        double denom = 0.0;
        std::vector<double> acc(d, 0.0);
        for (long j = 0; j < l; ++j) {
            if (!mr[j]) continue;
            const double p = std::exp(static_cast<double>(sr[j]) - m);
            denom += p;
            const uint16_t* vj = V + ((bb * l_cap + j) * hv + vh) * d;
            for (long c = 0; c < d; ++c) acc[c] += p * widen_bf16(vj[c]);
        }
        for (long c = 0; c < d; ++c) out[row * d + c] = static_cast<float>(acc[c] / denom);
    }
    return bad ? -2 : 0;
}

// Full (dense) attention, the speedup denominator (Main Findings: the
// end-to-end speedups are measured against full attention): every position
// kept.
// dk: key/query head dim (logits), dv: value head dim (output).
int oracle_decode_dense(long b, long hq, long hk, long hv, long dk, long dv, long l, long l_cap,
                        const uint16_t* q, const uint16_t* K, const uint16_t* V,
                        float* out) {
    if (l <= 0) return -1;
    std::vector<float> s(static_cast<size_t>(b * hq * l));
    if (oracle_logits(b, hq, hk, dk, l, l_cap, q, K, s.data()) != 0) return -1;
    std::vector<uint8_t> mask(s.size(), 1);
    return oracle_attend_masked(b, hq, hv, dv, l, l_cap, s.data(), mask.data(), V, out);
}

// One Atop-N decode step in the order the method states it (Key
// Contributions #2, Methodology ¶2): logits; if t mod n == 0 refresh the
// exact thresholds into tau_state, else reuse the stored ones; compare;
// softmax over the kept entries; gathered value sum.
// tau_state [b,hq] is read and, on refresh steps, overwritten.
// s_out [b,hq,l] and mask_out [b,hq,l] / cnt_out [b,hq] are optional.
int oracle_atopn_step(long b, long hq, long hk, long hv, long dk, long dv, long l, long l_cap,
                      long N, long t, long n,
                      const uint16_t* q, const uint16_t* K, const uint16_t* V,
                      float* tau_state, float* out, float* s_out,
                      uint8_t* mask_out, int32_t* cnt_out) {
    if (l <= 0 || N <= 0 || n <= 0 || t < 0) return -1;
    const long rows = b * hq;
    std::vector<float> s(static_cast<size_t>(rows * l));
    if (oracle_logits(b, hq, hk, dk, l, l_cap, q, K, s.data()) != 0) return -1;
    if (t % n == 0) oracle_nth_largest(s.data(), rows, l, N, tau_state);
    std::vector<uint8_t> mask(s.size());
    std::vector<int32_t> cnt(static_cast<size_t>(rows));
    oracle_select(s.data(), rows, l, tau_state, mask.data(), cnt.data());
    const int rc = oracle_attend_masked(b, hq, hv, dv, l, l_cap, s.data(), mask.data(), V, out);
    if (s_out) std::copy(s.begin(), s.end(), s_out);
    if (mask_out) std::copy(mask.begin(), mask.end(), mask_out);
    if (cnt_out) std::copy(cnt.begin(), cnt.end(), cnt_out);
    return rc;
}

}  // extern "C"
