// topk.cu -- exact per-row top-K selection.
//
// The indexer returns positions only: the k highest scores of the row
// ("Sparse Attention의 Indexer", Fig. 1 -- top-k keeps the k largest
// selection scores and hands their positions on, listed by position).
// Equal scores are taken lower position first; -0 equals +0.  Output rows
// list the selected positions in ascending order (a candidate row lists the
// proxy's top-`split` first, then the rest of the top-C, each ascending).
//
// Every entry has a 64-bit key
//     key = ordered(score) << 32 | (0xFFFFFFFF - position)
// (ordered(): order-preserving uint32 of the float), unique per row, so "the
// K largest keys" is exactly the answer.
//
// One CTA per row.  Fast path:
//   1. a lower bound T for the kept scores: the m-th largest of sampled
//      scores (prefix rows: 2048, in 64 runs of 32, by row_threshold_kernel
//      ahead of the select; other long rows: 4096 evenly spaced, inside it),
//      m chosen so about 1.4 K entries of the row should lie at or above it
//      (all entries when the row is short);
//   2. one vectorised pass appends every eligible entry >= T to shared
//      memory (warp-aggregated);
//   3. if between K and the buffer capacity entries were kept, they hold the
//      top K exactly; the exact K-th score is found by radix passes over
//      linear bins (no sort); of the entries tied at it, the lowest
//      positions are taken (the same search over their position words);
//   4. positions go into a bitmap; prefix popcounts give every selected
//      entry its output slot, so rows come out in position order unsorted.
// Otherwise (threshold missed, K > 8192, rows too long for the bitmaps) the
// exact path: histogram of the top 12 key bits, radix select inside the
// boundary bin, then a sort by position.
#include "common.cuh"
#include "kernels.h"

namespace pivot {

namespace {

constexpr int SEL_THREADS = 512;
constexpr int HIST_BINS = 4096;     // top 12 bits of the ordered score; also sample/bin space
constexpr int SAMPLES = 4096;
constexpr int LBINS = 4096;         // linear bins of one threshold-search pass
constexpr float SAMPLE_MARGIN = 1.4f;

__device__ __forceinline__ int row_limit(int kind, int r, int L, int g, int Gm, int maxlen,
                                         const int32_t* cache_len, bool& ok) {
    ok = true;
    switch (kind) {
        case SCAN_PREFILL_DENSE: return r;
        case SCAN_PREFILL_PROXY: {
            int e = (r + 1) * g;
            return (e < L ? e : L) - 1;
        }
        case SCAN_DECODE_DENSE: {
            int b = r / Gm, m = r % Gm;
            int n = cache_len[b];
            if (n < Gm || n > maxlen) { ok = false; return -1; }
            return n - Gm + m;
        }
        default: {
            int n = cache_len[r];
            if (n < 1 || n > maxlen) { ok = false; return -1; }
            return n - 1;
        }
    }
}

// Row r's causal limit for a select launch (ragged batches through the
// launch's segment table).
__device__ __forceinline__ int select_row_limit(const SelectParams& p, int r, bool& ok) {
    if (p.scan_kind == SCAN_VARLEN_DENSE) { ok = true; return seg_dense_lim(p.seg, r); }
    if (p.scan_kind == SCAN_VARLEN_PROXY) { ok = true; return seg_proxy_lim(p.seg, p.g, r); }
    return row_limit(p.scan_kind, r, p.L, p.g, p.Gm, p.maxlen, p.cache_len, ok);
}

struct RowView {
    const float* S;
    const int32_t* cand;   // null: position = entry index
    const float* ksc;      // candidate rows: score = S[i] * ksc[position], or null
    const uint64_t* keys;  // or: entry i is the full key keys[i] (S, cand unused)
    int n;                 // entries
    int lim;               // valid positions are <= lim
};

__device__ __forceinline__ uint64_t make_key(uint32_t u, int pos) {
    return ((uint64_t)u << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)pos);
}
__device__ __forceinline__ uint32_t key_u(uint64_t k) { return (uint32_t)(k >> 32); }
__device__ __forceinline__ int key_pos(uint64_t k) {
    return (int)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFu));
}
// Position as an unsigned value in which a zero (padding) key sorts last.
__device__ __forceinline__ uint32_t key_upos(uint64_t k) {
    return 0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFu);
}

// Key of entry i, or 0 when the entry is not eligible.
// A key whose position lies outside [0, lim] is an empty entry (the keep-
// everything rescan writes none; only a rescan that gave up leaves them).
__device__ __forceinline__ uint64_t listed_key(const RowView& v, int i) {
    const uint64_t k = v.keys[i];
    const int pos = key_pos(k);
    return (pos >= 0 && pos <= v.lim) ? k : 0ull;
}

__device__ __forceinline__ uint64_t entry_key(const RowView& v, int i) {
    if (v.keys) return listed_key(v, i);
    int pos = i;
    float x = v.S[i];
    if (v.cand) {
        pos = v.cand[i];
        if (pos < 0 || pos > v.lim) return 0;
        if (v.ksc) x = x * v.ksc[pos];
    }
    return make_key(ordered_key(x), pos);
}
__device__ __forceinline__ uint32_t entry_key32(const RowView& v, int i) {
    if (v.keys) return key_u(listed_key(v, i));
    float x = v.S[i];
    if (v.cand) {
        const int pos = v.cand[i];
        if (pos < 0 || pos > v.lim) return 0;
        if (v.ksc) x = x * v.ksc[pos];
    }
    return ordered_key(x);
}

// ------------------------------------------------------------ block helpers

__device__ uint32_t block_sum_u32(uint32_t x, uint32_t* scratch) {
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = x;
    __syncthreads();
    uint32_t t = 0;
    for (int w = 0; w < SEL_THREADS / 32; ++w) t += scratch[w];
    __syncthreads();
    return t;
}

__device__ uint32_t block_min_u32(uint32_t x, uint32_t* scratch) {
    for (int o = 16; o > 0; o >>= 1) x = min(x, __shfl_xor_sync(0xffffffffu, x, o));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = x;
    __syncthreads();
    uint32_t t = 0xFFFFFFFFu;
    for (int w = 0; w < SEL_THREADS / 32; ++w) t = min(t, scratch[w]);
    __syncthreads();
    return t;
}

__device__ uint32_t block_max_u32(uint32_t x, uint32_t* scratch) {
    for (int o = 16; o > 0; o >>= 1) x = max(x, __shfl_xor_sync(0xffffffffu, x, o));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = x;
    __syncthreads();
    uint32_t t = 0;
    for (int w = 0; w < SEL_THREADS / 32; ++w) t = max(t, scratch[w]);
    __syncthreads();
    return t;
}

// Exclusive prefix sum over threads (in thread order).
__device__ uint32_t block_excl_scan(uint32_t x, uint32_t* scratch) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint32_t inc = x;
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    __syncthreads();
    if (lane == 31) scratch[wid] = inc;
    __syncthreads();
    uint32_t base = 0;
    for (int w = 0; w < wid; ++w) base += scratch[w];
    __syncthreads();
    return base + inc - x;
}

__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active) {
    const unsigned mask = __ballot_sync(0xffffffffu, active);
    if (!active) return;
    const unsigned peers = __match_any_sync(mask, bin);
    const int leader = __ffs(peers) - 1;
    if ((threadIdx.x & 31) == leader) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
}

// Block-wide: the largest bin b with sum_{bins >= b} hist >= need, over
// `nbins` bins (nbins a multiple of SEL_THREADS, or <= SEL_THREADS).
// Returns b and the count strictly above it in *above.
__device__ int find_threshold_bin(const uint32_t* hist, int nbins, uint32_t need,
                                  uint32_t* scratch, uint32_t* above) {
    __shared__ int s_bin;
    __shared__ uint32_t s_above;
    const int per = nbins >= SEL_THREADS ? nbins / SEL_THREADS : 1;
    const int t = threadIdx.x;
    uint32_t local = 0;
    const int hi = nbins - t * per;        // thread t owns bins [hi - per, hi), descending
    const int lo = hi - per;
    if (lo >= 0)
        for (int b = lo; b < hi; ++b) local += hist[b];
    if (t == 0) { s_bin = -1; s_above = 0; }
    const uint32_t before = block_excl_scan(local, scratch);
    if (lo >= 0 && before < need && before + local >= need) {
        uint32_t acc = before;
        for (int b = hi - 1; b >= lo; --b) {
            if (acc + hist[b] >= need) {
                s_bin = b;
                s_above = acc;
                break;
            }
            acc += hist[b];
        }
    }
    __syncthreads();
    *above = s_above;
    const int r = s_bin;
    __syncthreads();
    return r;
}

// One pass of the linear-bin search: hist[b] = the count of values u in
// [lo, hi] with floor((u - lo) LBINS / (hi - lo + 1)) == b.
template <class F>
__device__ void linear_histogram(F vals, int n, uint32_t lo, uint32_t hi, uint32_t* hist) {
    const uint64_t range = (uint64_t)hi - lo + 1;
    for (int b = threadIdx.x; b < LBINS; b += SEL_THREADS) hist[b] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += SEL_THREADS) {
        const uint32_t u = vals(i);
        if (u && u >= lo && u <= hi) {
            const uint32_t b = (uint32_t)(((uint64_t)(u - lo) * LBINS) / range);
            atomicAdd(&hist[b], 1u);
        }
    }
    __syncthreads();
}

// [lo, hi] narrowed to the values of bin b of that pass.
__device__ __forceinline__ void narrow_to_bin(int b, uint32_t& lo, uint32_t& hi) {
    const uint64_t range = (uint64_t)hi - lo + 1;
    const uint32_t nlo = lo + (uint32_t)(((uint64_t)b * range + LBINS - 1) / LBINS);
    const uint32_t nhi = lo + (uint32_t)(((uint64_t)(b + 1) * range + LBINS - 1) / LBINS) - 1;
    lo = nlo;
    hi = nhi;
}

// The search from a range [lo, hi] that holds the wanted value, `remaining`
// the rank still wanted inside it and `above_total` the values counted above
// it so far.
template <class F>
__device__ uint32_t kth_in_range(F vals, int n, uint32_t remaining, uint32_t lo, uint32_t hi,
                                 uint32_t above_total, uint32_t* hist, uint32_t* scratch,
                                 uint32_t* above_out) {
    while (lo < hi) {
        linear_histogram(vals, n, lo, hi, hist);
        uint32_t above;
        const int b = find_threshold_bin(hist, LBINS, remaining, scratch, &above);
        remaining -= above;
        above_total += above;
        narrow_to_bin(b, lo, hi);
    }
    *above_out = above_total;
    return lo;
}

// The smallest and largest values >= 1 (lo > hi when there are none).
template <class F>
__device__ void value_range(F vals, int n, uint32_t* scratch, uint32_t& lo, uint32_t& hi) {
    uint32_t lo_l = 0xFFFFFFFFu, hi_l = 0;
    for (int i = threadIdx.x; i < n; i += SEL_THREADS) {
        const uint32_t u = vals(i);
        if (u) { lo_l = min(lo_l, u); hi_l = max(hi_l, u); }
    }
    lo = block_min_u32(lo_l, scratch);
    hi = block_max_u32(hi_l, scratch);
}

// The m-th largest value among n uint32 values >= 1 (values 0 are ignored),
// 1 <= m <= the count of such values: repeated histograms over LBINS linear
// bins of the remaining value range.  *above_out = the count of values
// strictly greater than the result.  `vals(i)` yields value i.
template <class F>
__device__ uint32_t kth_largest_linear(F vals, int n, uint32_t m, uint32_t* hist,
                                       uint32_t* scratch, uint32_t* above_out) {
    uint32_t lo, hi;
    value_range(vals, n, scratch, lo, hi);
    return kth_in_range(vals, n, m, lo, hi, 0u, hist, scratch, above_out);
}

// The m1-th and the m2-th largest of the same values (1 <= m1, m2 <= their
// count): exactly the two searches above, with the range and the first
// pass's histogram shared.  Returns the m1-th; the m2-th goes to *t2.
template <class F>
__device__ uint32_t kth_largest_linear_pair(F vals, int n, uint32_t m1, uint32_t m2,
                                            uint32_t* hist, uint32_t* scratch,
                                            uint32_t* above1, uint32_t* above2, uint32_t* t2) {
    uint32_t lo, hi;
    value_range(vals, n, scratch, lo, hi);
    if (!(lo < hi)) {
        *above1 = 0;
        *above2 = 0;
        *t2 = lo;
        return lo;
    }
    linear_histogram(vals, n, lo, hi, hist);
    uint32_t a1, a2;
    const int b1 = find_threshold_bin(hist, LBINS, m1, scratch, &a1);
    const int b2 = find_threshold_bin(hist, LBINS, m2, scratch, &a2);
    uint32_t lo1 = lo, hi1 = hi, lo2 = lo, hi2 = hi;
    narrow_to_bin(b1, lo1, hi1);
    narrow_to_bin(b2, lo2, hi2);
    *t2 = kth_in_range(vals, n, m2 - a2, lo2, hi2, a2, hist, scratch, above2);
    return kth_in_range(vals, n, m1 - a1, lo1, hi1, a1, hist, scratch, above1);
}

// Warp-aggregated append of `key` (where pred) to buf[*cnt++]; entries past
// `cap` are counted but not stored.  All 32 lanes must call it together.
__device__ __forceinline__ void warp_append(uint64_t* buf, uint32_t* cnt, uint32_t cap,
                                            uint64_t key, bool pred) {
    const unsigned m = __ballot_sync(0xffffffffu, pred);
    if (m == 0) return;
    const int lane = threadIdx.x & 31;
    const int leader = __ffs(m) - 1;
    uint32_t base = 0;
    if (lane == leader) base = atomicAdd(cnt, (uint32_t)__popc(m));
    base = __shfl_sync(0xffffffffu, base, leader);
    if (pred) {
        const uint32_t idx = base + (uint32_t)__popc(m & ((1u << lane) - 1u));
        if (idx < cap) buf[idx] = key;
    }
}

// Per-word exclusive prefix popcounts of a bitmap of W words.
__device__ void bitmap_prefix(const uint32_t* bm, uint32_t* pref, int W, uint32_t* scratch) {
    const int per = (W + SEL_THREADS - 1) / SEL_THREADS;
    const int w0 = threadIdx.x * per;
    const int w1 = min(W, w0 + per);
    uint32_t local = 0;
    for (int w = w0; w < w1; ++w) local += __popc(bm[w]);
    uint32_t acc = block_excl_scan(local, scratch);
    for (int w = w0; w < w1; ++w) {
        pref[w] = acc;
        acc += __popc(bm[w]);
    }
    __syncthreads();
}

__device__ __forceinline__ bool bit_of(const uint32_t* bm, int pos) {
    return (bm[pos >> 5] >> (pos & 31)) & 1u;
}
__device__ __forceinline__ uint32_t rank_of(const uint32_t* bm, const uint32_t* pref, int pos) {
    return pref[pos >> 5] + __popc(bm[pos >> 5] & ((1u << (pos & 31)) - 1u));
}

// The need-th largest low key word among the entries whose score key is Tu
// (1 <= need < their count): lower positions have larger low words, and no
// two are equal.  Kept out of line: only rows with many tied scores take it.
__device__ __noinline__ uint32_t tie_bound(const uint64_t* buf, int cnt, uint32_t Tu,
                                           uint32_t need, uint32_t* hist, uint32_t* scratch) {
    uint32_t above;
    return kth_largest_linear(
        [&](int i) {
            const uint64_t k = buf[i];
            return key_u(k) == Tu ? (uint32_t)(k & 0xFFFFFFFFu) : 0u;
        },
        cnt, need, hist, scratch, &above);
}

// Mark in `bm` the kept entries with u > Tu, plus the `need` lowest-position
// entries with u == Tu.  When more entries than that equal Tu, the lowest
// positions among them are found by the linear-bin search over the keys'
// low words (larger for lower positions, and distinct), in `hist`; when every
// entry equal to Tu is taken (the usual case: one of them), that is skipped.
__device__ void mark_top(const uint64_t* buf, int cnt, uint32_t Tu, uint32_t need, uint32_t* bm,
                         int W, uint32_t* hist, uint32_t* scratch) {
    uint32_t nties = 0;
    for (int i = threadIdx.x; i < cnt; i += SEL_THREADS) {
        const uint64_t k = buf[i];
        const uint32_t u = key_u(k);
        const int pos = key_pos(k);
        if (u > Tu) {
            if (PIVOT_CHECK(pos >= 0 && (pos >> 5) < W)) atomicOr(&bm[pos >> 5], 1u << (pos & 31));
        } else if (u == Tu) {
            ++nties;
        }
    }
    nties = block_sum_u32(nties, scratch);   // also orders the marks above
    // tied entries with a low key word >= lowmin are taken
    const uint32_t lowmin = nties > need ? tie_bound(buf, cnt, Tu, need, hist, scratch) : 0u;
    for (int i = threadIdx.x; i < cnt; i += SEL_THREADS) {
        const uint64_t k = buf[i];
        if (key_u(k) == Tu && (uint32_t)(k & 0xFFFFFFFFu) >= lowmin) {
            const int pos = key_pos(k);
            if (PIVOT_CHECK(pos >= 0 && (pos >> 5) < W)) atomicOr(&bm[pos >> 5], 1u << (pos & 31));
        }
    }
    __syncthreads();
}

// Write every kept entry whose position is marked in `bm` at slot
// base + (its rank among the marked positions).
__device__ void write_marked(const uint64_t* buf, int cnt, const uint32_t* bm, uint32_t* pref,
                             int W, uint32_t base, uint32_t* scratch, int32_t* out, float* outs,
                             int kmax) {
    bitmap_prefix(bm, pref, W, scratch);
    for (int i = threadIdx.x; i < cnt; i += SEL_THREADS) {
        const uint64_t k = buf[i];
        if (k == 0) continue;   // an empty slot (candidate rows keep them in place)
        const int pos = key_pos(k);
        if (!PIVOT_CHECK(pos >= 0 && (pos >> 5) < W)) continue;
        if (bit_of(bm, pos)) {
            const uint32_t slot = base + rank_of(bm, pref, pos);
            if (!PIVOT_CHECK(slot < (uint32_t)kmax)) continue;
            out[slot] = pos;
            if (outs) outs[slot] = key_to_float(key_u(k));
        }
    }
    __syncthreads();
}

__device__ void pad_row(uint32_t from, int K, int32_t* out, float* outs) {
    for (int i = (int)from + threadIdx.x; i < K; i += SEL_THREADS) {
        out[i] = -1;
        if (outs) outs[i] = -INFINITY;
    }
}

template <class Less>
__device__ void bitonic_sort(uint64_t* buf, int n, uint64_t pad, Less less);

// Rank order: the kept entries whose positions are marked in `bm` (exactly
// Kp of them), sorted by key descending -- score descending, then position
// ascending -- into out[0, Kp), then -1 padding to K.  Unmarked entries are
// cleared to the padding key 0 (which sorts last) and everything is sorted
// in place.
__device__ void write_rank_order(uint64_t* buf, int n, const uint32_t* bm, uint32_t Kp, int K,
                                 int32_t* out, float* outs) {
    for (int i = threadIdx.x; i < n; i += SEL_THREADS) {
        const uint64_t k = buf[i];
        if (k != 0 && !bit_of(bm, key_pos(k))) buf[i] = 0;
    }
    __syncthreads();
    bitonic_sort(buf, n, 0ull, [](uint64_t a, uint64_t b) { return a > b; });
    for (int i = threadIdx.x; i < (int)Kp; i += SEL_THREADS) {
        const uint64_t k = buf[i];
        out[i] = key_pos(k);
        if (outs) outs[i] = key_to_float(key_u(k));
    }
    pad_row(Kp, K, out, outs);
}

struct FastSmem {
    uint32_t* hist;     // HIST_BINS: samples, then linear bins
    uint32_t* scratch;  // 64
    uint64_t* buf;      // fast_cap kept entries
    uint32_t* bmS;      // selected positions (W words)
    uint32_t* bmA;      // class A, only when split (W words)
    uint32_t* pref;     // W prefix counts (aliases hist when W <= HIST_BINS)
};

// Fast path; returns false (block-uniformly) when the threshold kept fewer
// than K eligible entries or more than the buffer holds.
__device__ bool select_fast(const SelectParams& p, const RowView& v, const FastSmem& sm,
                            uint32_t* s_cnt, uint32_t* s_valid, int32_t* out, float* outs) {
    // bitmap words this row needs: its positions are <= lim
    const int K = p.K, cap = p.fast_cap, W = min(p.bitmap_words, (v.lim + 32) >> 5);
    uint32_t* hist = sm.hist;
    uint32_t* scratch = sm.scratch;
    uint64_t* buf = sm.buf;
    if (threadIdx.x == 0) { *s_cnt = 0; *s_valid = 0; }
    uint32_t T = 1;
    if (p.thresh) {
        T = p.thresh[blockIdx.x];   // row r = row0 + blockIdx.x
    } else if (v.n > cap) {
        for (int j = threadIdx.x; j < SAMPLES; j += SEL_THREADS)
            hist[j] = entry_key32(v, (int)(((long long)j * v.n) / SAMPLES));
        __syncthreads();
        uint32_t elig = 0;
        for (int j = threadIdx.x; j < SAMPLES; j += SEL_THREADS) elig += hist[j] != 0;
        elig = block_sum_u32(elig, scratch);
        long long m = (long long)ceilf(SAMPLE_MARGIN * (float)K * (float)SAMPLES / (float)v.n);
        if (m < 1) m = 1;
        if (m <= (long long)elig) {
            // move the samples out of the bins' way (the buffer is still free)
            uint32_t* samp = reinterpret_cast<uint32_t*>(buf);
            for (int j = threadIdx.x; j < SAMPLES; j += SEL_THREADS) samp[j] = hist[j];
            __syncthreads();
            uint32_t above;
            T = kth_largest_linear([&](int i) { return samp[i]; }, SAMPLES, (uint32_t)m, hist,
                                   scratch, &above);
        }
    }
    __syncthreads();
    // filtering pass
    uint32_t nvalid_local = 0;
    const bool vec = (v.cand == nullptr) && !v.keys &&
                     ((reinterpret_cast<uintptr_t>(v.S) & 15) == 0);
    if (vec) {
        const int n4 = v.n / 4;
        const float4* S4 = reinterpret_cast<const float4*>(v.S);
        // Entries are compared as floats: for finite scores, key >= T exactly
        // when score >= key_to_float(T) (-0 and +0 alike); a bound at or
        // below the key of -FLT_MAX keeps every finite score.  Each thread
        // reserves room for all its kept entries of a step with one
        // shared-memory atomic (a few entries in a hundred pass, so the
        // atomics rarely collide).
        const float Tf = T <= 0x00800000u ? -INFINITY : key_to_float(T);
        // four float4 per thread in flight per step: the loads of a step go
        // out together, so a row pays one memory latency per 8192 scores
        auto bits = [&](const float4& x, bool in) -> uint32_t {
            return in ? ((x.x >= Tf ? 1u : 0u) | (x.y >= Tf ? 2u : 0u) | (x.z >= Tf ? 4u : 0u) |
                         (x.w >= Tf ? 8u : 0u))
                      : 0u;
        };
        const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i0 = 0; i0 < n4; i0 += 4 * SEL_THREADS) {
            const int ia = i0 + threadIdx.x, ib = ia + SEL_THREADS, ic = ib + SEL_THREADS,
                      id = ic + SEL_THREADS;
            const float4 xa = ia < n4 ? __ldcs(S4 + ia) : z4;
            const float4 xb = ib < n4 ? __ldcs(S4 + ib) : z4;
            const float4 xc = ic < n4 ? __ldcs(S4 + ic) : z4;
            const float4 xd = id < n4 ? __ldcs(S4 + id) : z4;
            uint32_t m = bits(xa, ia < n4) | (bits(xb, ib < n4) << 4) | (bits(xc, ic < n4) << 8) |
                         (bits(xd, id < n4) << 12);
            if (m) {
                uint32_t slot = atomicAdd(s_cnt, (uint32_t)__popc(m));
                do {
                    const int e = __ffs(m) - 1;
                    m &= m - 1;
                    const int j = e >> 2, c = e & 3;
                    const float4 x = j == 0 ? xa : (j == 1 ? xb : (j == 2 ? xc : xd));
                    const float f = c == 0 ? x.x : (c == 1 ? x.y : (c == 2 ? x.z : x.w));
                    const int pos = 4 * (ia + j * SEL_THREADS) + c;
                    if (slot < (uint32_t)cap) buf[slot] = make_key(ordered_key(f), pos);
                    ++slot;
                } while (m);
            }
        }
        const int i = n4 * 4 + threadIdx.x;
        const bool a = threadIdx.x < 4 && i < v.n;
        const uint32_t u = a ? ordered_key(v.S[i]) : 0u;
        warp_append(buf, s_cnt, cap, make_key(u, i), a && u >= T);
    } else if (v.cand && v.n <= cap) {
        // Candidate rows that fit the buffer keep every entry in place
        // (slot = entry index, key 0 where the candidate is not eligible,
        // which every later step skips): no compaction, and each thread
        // issues the loads of eight entries together.
        constexpr int U = 8;
        for (int i0 = 0; i0 < v.n; i0 += SEL_THREADS * U) {
            int pos[U];
            float x[U];
#pragma unroll
            for (int j = 0; j < U; ++j) {
                const int i = i0 + j * SEL_THREADS + threadIdx.x;
                pos[j] = i < v.n ? v.cand[i] : -1;
                x[j] = i < v.n ? v.S[i] : 0.0f;
            }
            if (v.ksc) {
#pragma unroll
                for (int j = 0; j < U; ++j)
                    if (pos[j] >= 0 && pos[j] <= v.lim) x[j] = x[j] * v.ksc[pos[j]];
            }
#pragma unroll
            for (int j = 0; j < U; ++j) {
                const int i = i0 + j * SEL_THREADS + threadIdx.x;
                const bool ok = pos[j] >= 0 && pos[j] <= v.lim;
                if (i < v.n) buf[i] = ok ? make_key(ordered_key(x[j]), pos[j]) : 0ull;
                nvalid_local += ok;
            }
        }
        if (threadIdx.x == 0) *s_cnt = (uint32_t)v.n;
    } else {
        for (int i0 = 0; i0 < v.n; i0 += SEL_THREADS) {
            const int i = i0 + threadIdx.x;
            uint32_t u = 0;
            int pos = i;
            if (i < v.n) {
                if (v.keys) {
                    const uint64_t k = listed_key(v, i);
                    u = key_u(k);
                    pos = k ? key_pos(k) : 0;
                } else {
                    u = entry_key32(v, i);
                    if (v.cand) pos = v.cand[i];
                }
            }
            nvalid_local += (u != 0);
            warp_append(buf, s_cnt, cap, make_key(u, pos), u != 0 && u >= T);
        }
    }
    if (v.cand) {
        for (int o = 16; o > 0; o >>= 1) nvalid_local += __shfl_xor_sync(0xffffffffu, nvalid_local, o);
        if ((threadIdx.x & 31) == 0 && nvalid_local) atomicAdd(s_valid, nvalid_local);
    }
    __syncthreads();
    const uint32_t cnt = *s_cnt;
    const uint32_t nvalid = v.cand ? *s_valid : (uint32_t)v.n;
    const uint32_t Kp = nvalid < (uint32_t)K ? nvalid : (uint32_t)K;
    __syncthreads();
    if (cnt > (uint32_t)cap || cnt < Kp) return false;
    if (Kp == 0) {
        pad_row(0, K, out, outs);
        return true;
    }
    const int n = (int)cnt;
    auto uval = [&](int i) { return key_u(buf[i]); };
    uint32_t aboveK, aboveS = 0;
    const int split = (!p.rank_order && p.split > 0 && (uint32_t)p.split < Kp) ? p.split : 0;
    uint32_t TuS = 0;
    const uint32_t TuK = split ? kth_largest_linear_pair(uval, n, Kp, (uint32_t)split, hist,
                                                          scratch, &aboveK, &aboveS, &TuS)
                               : kth_largest_linear(uval, n, Kp, hist, scratch, &aboveK);
    // selected set (mark_top may take the linear bins again for ties; pref,
    // which may alias them, is used only after it)
    for (int w = threadIdx.x; w < W; w += SEL_THREADS) sm.bmS[w] = 0;
    __syncthreads();
    mark_top(buf, n, TuK, Kp - aboveK, sm.bmS, W, hist, scratch);
    if (p.rank_order) {
        write_rank_order(buf, n, sm.bmS, Kp, K, out, outs);
        return true;
    }
    if (!split) {
        write_marked(buf, n, sm.bmS, sm.pref, W, 0, scratch, out, outs, K);
    } else {
        // class A: the top `split`; class B: the rest of the selected set
        // (bmS less class A, in place)
        for (int w = threadIdx.x; w < W; w += SEL_THREADS) sm.bmA[w] = 0;
        __syncthreads();
        mark_top(buf, n, TuS, (uint32_t)split - aboveS, sm.bmA, W, hist, scratch);
        write_marked(buf, n, sm.bmA, sm.pref, W, 0, scratch, out, outs, K);
        for (int w = threadIdx.x; w < W; w += SEL_THREADS) sm.bmS[w] &= ~sm.bmA[w];
        __syncthreads();
        write_marked(buf, n, sm.bmS, sm.pref, W, (uint32_t)split, scratch, out, outs, K);
    }
    pad_row(Kp, K, out, outs);
    return true;
}

// Sort buf[0, n) ascending by `less` (bitonic, pads to a power of two with
// `pad`, which must sort last).
template <class Less>
__device__ void bitonic_sort(uint64_t* buf, int n, uint64_t pad, Less less) {
    int M = 1;
    while (M < n) M <<= 1;
    for (int i = n + threadIdx.x; i < M; i += SEL_THREADS) buf[i] = pad;
    __syncthreads();
    for (int kk = 2; kk <= M; kk <<= 1) {
        for (int j = kk >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < M; i += SEL_THREADS) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const uint64_t a = buf[i], b = buf[ixj];
                    const bool up = (i & kk) == 0;
                    if (up ? less(b, a) : less(a, b)) {
                        buf[i] = b;
                        buf[ixj] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
}

// Radix select among keys k with (k >> 52) == bin0: the `need` largest.
// Source is the shared-memory buffer (tail, ntail) or, when tail == null,
// the row in global memory.  Returns (mask, prefix): the selected keys are
// exactly those with (k & mask) >= prefix among the source's bin-0 keys.
template <bool FROM_SMEM>
__device__ void radix_select_tail(const RowView& v, const uint64_t* tail, int ntail,
                                  uint32_t bin0, uint32_t need, uint32_t* hist,
                                  uint32_t* scratch, uint64_t* out_mask, uint64_t* out_prefix) {
    uint64_t mask = 0xFFF0000000000000ull;
    uint64_t prefix = (uint64_t)bin0 << 52;
    uint32_t remaining = need;
    const int shifts[7] = {44, 36, 28, 20, 12, 4, 0};
    for (int level = 0; level < 7; ++level) {
        const int sh = shifts[level];
        const int width = (sh == 0) ? 4 : 8;
        const int nb = 1 << width;
        const uint64_t dmask = (uint64_t)(nb - 1) << sh;
        for (int b = threadIdx.x; b < 256; b += SEL_THREADS) hist[b] = 0;
        __syncthreads();
        const int n = FROM_SMEM ? ntail : v.n;
        for (int i0 = 0; i0 < n; i0 += SEL_THREADS) {
            const int i = i0 + threadIdx.x;
            uint64_t k = 0;
            if (i < n) k = FROM_SMEM ? tail[i] : entry_key(v, i);
            const bool act = (i < n) && k != 0 && ((k & mask) == prefix);
            hist_add(hist, (uint32_t)((k & dmask) >> sh), act);
        }
        __syncthreads();
        // digit: largest d with count(>= d) >= remaining (nb <= 256 bins)
        uint32_t above;
        const int d = find_threshold_bin(hist, 256, remaining, scratch, &above);
        // bins above nb are empty, so d < nb
        const uint32_t cnt_d = hist[d];
        remaining -= above;
        prefix |= (uint64_t)d << sh;
        mask |= dmask;
        __syncthreads();
        if (cnt_d == remaining) break;   // everything matching the prefix is in
    }
    *out_mask = mask;
    *out_prefix = prefix;
}


// Exact path: histogram of the top 12 key bits over the whole row, exact
// radix select inside the boundary bin, then the selected keys sorted by
// position (the top `split` first when requested).  `sel` has room for
// 2 * pow2(K) keys, `tail` for tail_cap keys.
__device__ void select_exact(const SelectParams& p, const RowView& v, uint32_t* hist,
                             uint32_t* scratch, uint32_t* hist256, uint64_t* sel, uint64_t* tail,
                             int M2, uint32_t* s_nsel, uint32_t* s_ntail, int32_t* out,
                             float* outs) {
    // 1. histogram of the top 12 bits
    for (int b = threadIdx.x; b < HIST_BINS; b += SEL_THREADS) hist[b] = 0;
    if (threadIdx.x == 0) { *s_nsel = 0; *s_ntail = 0; }
    __syncthreads();
    for (int i0 = 0; i0 < v.n; i0 += SEL_THREADS) {
        const int i = i0 + threadIdx.x;
        const uint32_t u = i < v.n ? entry_key32(v, i) : 0;
        hist_add(hist, u >> 20, u != 0);
    }
    __syncthreads();
    uint32_t total_local = 0;
    for (int b = threadIdx.x; b < HIST_BINS; b += SEL_THREADS) total_local += hist[b];
    const uint32_t total = block_sum_u32(total_local, scratch);
    const uint32_t Kp = total < (uint32_t)p.K ? total : (uint32_t)p.K;

    // 2. threshold bin
    int bin = -1;
    uint32_t above = 0;
    if (Kp > 0 && Kp < total) bin = find_threshold_bin(hist, HIST_BINS, Kp, scratch, &above);
    const uint32_t need = Kp - above;

    // 3. collect
    for (int i0 = 0; i0 < v.n; i0 += SEL_THREADS) {
        const int i = i0 + threadIdx.x;
        if (i >= v.n) break;
        const uint64_t k = entry_key(v, i);
        if (k == 0) continue;
        const int b = (int)(k >> 52);
        if (b > bin) {
            sel[atomicAdd(s_nsel, 1u)] = k;
        } else if (b == bin) {
            const uint32_t slot = atomicAdd(s_ntail, 1u);
            if (slot < (uint32_t)p.tail_cap) tail[slot] = k;
        }
    }
    __syncthreads();

    // 4. resolve the boundary bin
    if (bin >= 0 && need > 0) {
        const uint32_t ntail = *s_ntail;
        uint64_t mask, prefix;
        if (ntail == need) {
            mask = 0; prefix = 0;   // take all of them
        } else if (ntail <= (uint32_t)p.tail_cap) {
            radix_select_tail<true>(v, tail, (int)ntail, (uint32_t)bin, need, hist256, scratch,
                                    &mask, &prefix);
        } else {
            radix_select_tail<false>(v, nullptr, 0, (uint32_t)bin, need, hist256, scratch, &mask,
                                     &prefix);
        }
        if (ntail <= (uint32_t)p.tail_cap) {
            for (uint32_t i = threadIdx.x; i < ntail; i += SEL_THREADS) {
                const uint64_t k = tail[i];
                if ((k & mask) >= prefix) sel[atomicAdd(s_nsel, 1u)] = k;
            }
        } else {
            for (int i = threadIdx.x; i < v.n; i += SEL_THREADS) {
                const uint64_t k = entry_key(v, i);
                if (k != 0 && (int)(k >> 52) == bin && (k & mask) >= prefix)
                    sel[atomicAdd(s_nsel, 1u)] = k;
            }
        }
        __syncthreads();
    }

    // 5. order: by key (to split off the top `split`), then by position
    auto by_pos = [](uint64_t a, uint64_t b) { return key_upos(a) < key_upos(b); };
    const int split = (!p.rank_order && p.split > 0 && (uint32_t)p.split < Kp) ? p.split : 0;
    if (p.rank_order) {
        bitonic_sort(sel, (int)Kp, 0ull, [](uint64_t a, uint64_t b) { return a > b; });
    } else if (split) {
        bitonic_sort(sel, (int)Kp, 0ull, [](uint64_t a, uint64_t b) { return a > b; });
        uint64_t* rest = sel + M2;
        for (int i = threadIdx.x; i < (int)Kp - split; i += SEL_THREADS) rest[i] = sel[split + i];
        __syncthreads();
        bitonic_sort(sel, split, 0ull, by_pos);
        bitonic_sort(rest, (int)Kp - split, 0ull, by_pos);
        for (int i = threadIdx.x; i < (int)Kp - split; i += SEL_THREADS) sel[split + i] = rest[i];
        __syncthreads();
    } else {
        bitonic_sort(sel, (int)Kp, 0ull, by_pos);
    }
    for (int i = threadIdx.x; i < p.K; i += SEL_THREADS) {
        if ((uint32_t)i < Kp) {
            const uint64_t k = sel[i];
            out[i] = key_pos(k);
            if (outs) outs[i] = key_to_float(key_u(k));
        } else {
            out[i] = -1;
            if (outs) outs[i] = -INFINITY;
        }
    }
}

// ------------------------------------------------------------ per-row bound
//
// The fast path's lower bound T for prefix rows, computed ahead of the
// select by one warp per row: the m-th largest of 2048 sampled scores (64
// evenly spread runs of 32 consecutive entries), m set so about
// SAMPLE_MARGIN K entries of the row should lie at or above it; 1 (keep
// everything) when the row fits the fast path's buffer.  Exact m-th by
// histograms over 256 power-of-two-wide bins of the remaining key range.

constexpr int THR_WARPS = 8;           // rows per CTA
constexpr int THR_RUNS = 64;
constexpr int THR_SAMPLES = THR_RUNS * 32;
constexpr int THR_BINS = 256;
constexpr size_t THR_SMEM_WARP = (size_t)(THR_SAMPLES + THR_BINS) * 4;

__device__ __forceinline__ uint32_t warp_min_u32(uint32_t x) {
    for (int o = 16; o > 0; o >>= 1) x = min(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ uint32_t warp_max_u32(uint32_t x) {
    for (int o = 16; o > 0; o >>= 1) x = max(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

// The m-th largest of the nonzero values get(0..n), 1 <= m <= their count,
// by one warp; hist (THR_BINS words) in this warp's shared memory.
template <class F>
__device__ uint32_t warp_kth_largest_f(F get, int n, uint32_t m, uint32_t* hist) {
    const int lane = threadIdx.x & 31;
    uint32_t lo = 0xFFFFFFFFu, hi = 0;
    for (int i = lane; i < n; i += 32) {
        const uint32_t u = get(i);
        if (u) { lo = min(lo, u); hi = max(hi, u); }
    }
    lo = warp_min_u32(lo);
    hi = warp_max_u32(hi);
    uint32_t remaining = m;
    while (lo < hi) {
        // bins of width 2^sh: the smallest sh with (hi - lo) >> sh < THR_BINS
        const uint32_t span = hi - lo;
        int sh = (32 - __clz(span)) - 8;
        if (sh < 0) sh = 0;
#pragma unroll
        for (int b = 0; b < THR_BINS / 32; ++b) hist[b * 32 + lane] = 0;
        __syncwarp();
        for (int i = lane; i < n; i += 32) {
            const uint32_t u = get(i);
            if (u && u >= lo && u <= hi) atomicAdd(&hist[(u - lo) >> sh], 1u);
        }
        __syncwarp();
        // lane l owns the 8 bins [THR_BINS - 8 (l + 1), THR_BINS - 8 l)
        constexpr int PER = THR_BINS / 32;
        const int top = THR_BINS - lane * PER;
        uint32_t c[PER];
        uint32_t local = 0;
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            c[j] = hist[top - 1 - j];
            local += c[j];
        }
        uint32_t inc = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        const uint32_t before = inc - local;
        const bool mine = before < remaining && inc >= remaining;
        int b = 0;
        uint32_t above = 0;
        if (mine) {
            uint32_t acc = before;
#pragma unroll
            for (int j = 0; j < PER; ++j) {
                if (acc + c[j] >= remaining) {
                    b = top - 1 - j;
                    above = acc;
                    break;
                }
                acc += c[j];
            }
        }
        const unsigned who = __ballot_sync(0xffffffffu, mine);
        if (who == 0) break;   // m above the count: keep the current lower edge
        const int src = __ffs(who) - 1;
        b = __shfl_sync(0xffffffffu, b, src);
        above = __shfl_sync(0xffffffffu, above, src);
        remaining -= above;
        const uint32_t nlo = lo + ((uint32_t)b << sh);
        const uint64_t ntop = (uint64_t)nlo + ((1ull << sh) - 1);
        hi = ntop < (uint64_t)hi ? (uint32_t)ntop : hi;
        lo = nlo;
        __syncwarp();
    }
    return lo;
}

__device__ uint32_t warp_kth_largest(const uint32_t* v, int n, uint32_t m, uint32_t* hist) {
    return warp_kth_largest_f([&](int i) { return v[i]; }, n, m, hist);
}

__global__ void __launch_bounds__(THR_WARPS * 32) row_threshold_kernel(const SelectParams p,
                                                                        uint32_t* thresh) {
    extern __shared__ __align__(16) uint8_t smem_t[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t* samp = reinterpret_cast<uint32_t*>(smem_t + warp * THR_SMEM_WARP);
    uint32_t* hist = samp + THR_SAMPLES;
    const int rr = blockIdx.x * THR_WARPS + warp;   // row index within the launch
    if (rr >= p.nrows) return;
    const int r = p.row0 + rr;
    bool ok;
    const int lim =
        select_row_limit(p, r, ok) - p.lim_shift;
    const int n = ok && lim >= 0 ? lim + 1 : 0;
    uint32_t T = 1;
    if (n > p.fast_cap) {
        const float* S = p.S + (size_t)rr * p.S_stride;
#pragma unroll 8
        for (int run = 0; run < THR_RUNS; ++run) {
            long long start = ((long long)run * n) / THR_RUNS;
            if (start + 32 > n) start = n - 32;
            samp[run * 32 + lane] = ordered_key(S[start + lane]);
        }
        __syncwarp();
        uint32_t elig = 0;
        for (int i = lane; i < THR_SAMPLES; i += 32) elig += samp[i] != 0;
        for (int o = 16; o > 0; o >>= 1) elig += __shfl_xor_sync(0xffffffffu, elig, o);
        long long m = (long long)ceilf(SAMPLE_MARGIN * (float)p.K * (float)THR_SAMPLES / (float)n);
        if (m < 1) m = 1;
        if (m <= (long long)elig) T = warp_kth_largest(samp, THR_SAMPLES, (uint32_t)m, hist);
    }
    if (lane == 0) thresh[rr] = T;
}

// ------------------------------------------------------------ candidate rows
//
// Warp-level helpers of the fused selection's finish (one warp a row): the
// k-th largest key by warp histograms, stable compaction, bitonic sort.

__host__ __device__ int pow2_at_least(int x) {
    int m = 1;
    while (m < x) m <<= 1;
    return m;
}

constexpr int CW_BATCH = 8;              // independent loads a lane issues at once
constexpr size_t CW_SMEM_LIMIT = 200 * 1024;

// Sort e[0, M) (M a power of two, whole warp) so that before(a, b) holds for
// every earlier a and later b.
template <class Before>
__device__ void warp_bitonic(uint64_t* e, int M, Before before) {
    const int lane = threadIdx.x & 31;
    for (int kk = 2; kk <= M; kk <<= 1) {
        for (int j = kk >> 1; j > 0; j >>= 1) {
            for (int i = lane; i < M; i += 32) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const uint64_t a = e[i], b = e[ixj];
                    const bool up = (i & kk) == 0;
                    if (up ? before(b, a) : before(a, b)) {
                        e[i] = b;
                        e[ixj] = a;
                    }
                }
            }
            __syncwarp();
        }
    }
}

// Compacts the nonzero entries of e[a, b) to the front of that range, in
// order; returns their count.  Whole warp.
__device__ int warp_compact(uint64_t* e, int a, int b) {
    const int lane = threadIdx.x & 31;
    int n = 0;
    for (int i0 = a; i0 < b; i0 += 32) {
        const int i = i0 + lane;
        const uint64_t x = i < b ? e[i] : 0ull;
        const unsigned m = __ballot_sync(0xffffffffu, x != 0);
        __syncwarp();   // every read of this chunk precedes its writes
        if (x != 0) e[a + n + __popc(m & ((1u << lane) - 1u))] = x;
        n += __popc(m);
        __syncwarp();
    }
    return n;
}

// ------------------------------------------------------------ fused selection
//
// Prefix rows whose scan ran in filter mode.  A sample scan scored every
// kts-th key tile of each row; the bound of a row is the m-th largest of its
// samples, m = m0 + 4.5 sqrt(m0) with m0 = K * (samples) / (row length) the
// samples expected at or above the row's K-th score (4.5 is the default
// margin) -- so, for keys in random order, at least K and about
// K (1 + 4.5 / sqrt(m0)) entries of the row lie
// at or above it, far from the warp select's capacity.  Rows no longer than
// the capacity keep everything (bound 1).  The filter-mode scan appended every
// score at or above the bound; one warp per row then takes the exact top K of
// those survivors -- provided at least min(K, n) and at most `cap` survived
// (else the row goes on the miss list, and the fallback rescans it keeping
// everything and selects with the block select).  Every row that passes holds
// all of its entries at or above its K-th score among the survivors, so its
// answer is exact.

constexpr int FB_WARPS = 8;              // bound kernel: rows a block
constexpr int FF_MAX_WARPS = 8;
constexpr int FF_AUX = 1024;             // warp-select words beside its entries: histogram, prefix

// Row r's causal limit (-1 with ok = false for a bad cache length).
__device__ __forceinline__ int fused_lim(const FusedSelectParams& p, int r, bool& ok) {
    return row_limit(p.scan_kind, r, p.L, p.g, p.Gm, p.maxlen, p.cache_len, ok);
}

// Sample columns at positions <= lim (sample j sits at position
// (j / 128) * kts * 128 + j % 128).
__device__ __forceinline__ int samples_upto(int lim, int kts) {
    if (lim < 0) return 0;
    const int span = kts * 128;
    const int full = lim / span;
    const int rem = lim - full * span;
    return full * 128 + (rem < 128 ? rem + 1 : 128);
}

__global__ void __launch_bounds__(FB_WARPS * 32) sample_bound_kernel(const FusedSelectParams p) {
    extern __shared__ __align__(16) uint8_t smem_b[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (blockIdx.x == 0 && threadIdx.x == 0) *p.miss_count = 0;
    const int rr = blockIdx.x * FB_WARPS + warp;
    if (rr >= p.nrows) return;
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem_b) + (size_t)warp * THR_BINS;
    bool ok;
    const int lim = fused_lim(p, p.row0 + rr, ok) - p.lim_shift;
    const int n = lim + 1;
    uint32_t T = 1;
    if (ok && n > p.cap) {
        // every sample of the row, read in place (each pass of the warp
        // select re-reads the row, written just before and still in L2)
        const int ns = samples_upto(lim, p.kts);
        const float* row = p.samp + (size_t)rr * p.samp_stride;
        const double m0 = (double)p.K * ns / n;
        long long m = (long long)ceil(m0 + (double)p.sigmas * sqrt(m0));
        if (m < 1) m = 1;
        if (m <= ns)
            T = warp_kth_largest_f([&](int j) { return ordered_key(row[j]); }, ns, (uint32_t)m,
                                   hist);
        // else: too few samples to bound the row; it keeps everything and
        // takes the fallback
    }
    if (lane == 0) p.bound[rr] = T;
}

// Among the nonzero keys e[0, n), keep exactly the `keep` largest (score,
// then lower position) and clear the rest.  Whole warp; keep <= nonzero count.
__device__ void warp_keep_top(uint64_t* e, int n, uint32_t keep, uint32_t* hist) {
    const int lane = threadIdx.x & 31;
    const uint32_t T = warp_kth_largest_f([&](int i) { return key_u(e[i]); }, n, keep, hist);
    uint32_t above = 0, eq = 0;
    for (int i = lane; i < n; i += 32) {
        const uint32_t u = key_u(e[i]);
        above += u > T;
        eq += u == T;
    }
    for (int o = 16; o > 0; o >>= 1) {
        above += __shfl_xor_sync(0xffffffffu, above, o);
        eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    const uint32_t need = keep - above;
    uint32_t Lmin = 0;
    if (eq > need)
        Lmin = warp_kth_largest_f([&](int i) { return key_u(e[i]) == T ? (uint32_t)e[i] : 0u; },
                                  n, need, hist);
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
        const uint64_t k = e[i];
        const uint32_t u = key_u(k);
        if (u < T || (u == T && (uint32_t)k < Lmin)) e[i] = 0ull;
    }
    __syncwarp();
}

__global__ void __launch_bounds__(FF_MAX_WARPS * 32) fused_finish_kernel(const FusedSelectParams p,
                                                                         int warps) {
    extern __shared__ __align__(16) uint8_t smem_f[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rr = blockIdx.x * warps + warp;
    if (warp >= warps || rr >= p.nrows) return;   // whole warps; no block barriers
    const int M = p.cap;
    uint64_t* e = reinterpret_cast<uint64_t*>(smem_f + (size_t)warp * ((size_t)M * 8 + FF_AUX * 4));
    uint32_t* hist = reinterpret_cast<uint32_t*>(e + M);   // FF_AUX words: histogram / prefix
    const int r = p.row0 + rr;
    bool ok;
    const int lim = fused_lim(p, r, ok) - p.lim_shift;
    if (!ok && lane == 0) raise_error(ERRBIT_DATA);
    const int n = (ok && lim >= 0) ? lim + 1 : 0;
    const int K = p.K;
    const size_t ostride = p.out_stride ? (size_t)p.out_stride : (size_t)K;
    int32_t* out = p.out_idx + (size_t)(r - p.out_base) * ostride;
    float* outs = p.out_score ? p.out_score + (size_t)(r - p.out_base) * ostride : nullptr;
    const uint32_t Kp = n < K ? (uint32_t)n : (uint32_t)K;

    // segments (chunk, sub-region) of the row's survivors
    const int nch = n > 0 ? (n + p.chunk_keys - 1) / p.chunk_keys : 0;
    const int nseg = nch * p.nsub;
    const uint32_t* cnt = p.surv_count + (size_t)rr * p.nchunks * p.nsub;
    // a count above its segment's size (a scan that gave up left it stale)
    // counts as a miss, so the gather below stays inside the regions
    uint32_t total = 0, over = 0;
    for (int c = lane; c < nseg; c += 32) {
        const uint32_t k = cnt[c];
        if (k > (uint32_t)p.sub_keys) over = 1;
        else total += k;
    }
    for (int o = 16; o > 0; o >>= 1) {
        total += __shfl_xor_sync(0xffffffffu, total, o);
        over |= __shfl_xor_sync(0xffffffffu, over, o);
    }
    if (over || total < Kp || total > (uint32_t)M) {
        if (lane == 0) p.miss_list[atomicAdd(p.miss_count, 1u)] = r;
        return;
    }
    if (Kp > 0) {
        // the row's survivors, segment after segment: an exclusive prefix of
        // the segment counts (in the auxiliary space), then every lane copies
        // entries, finding each one's segment by binary search
        const uint64_t* src = p.surv + (size_t)rr * p.surv_stride;
        if (nseg <= FF_AUX) {
            uint32_t carry = 0;
            for (int c0 = 0; c0 < nseg; c0 += 32) {
                const int c = c0 + lane;
                const uint32_t k = c < nseg ? cnt[c] : 0u;
                uint32_t inc = k;
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
                    if (lane >= o) inc += y;
                }
                if (c < nseg) hist[c] = carry + inc - k;
                carry += __shfl_sync(0xffffffffu, inc, 31);
            }
            __syncwarp();
            for (int i0 = 0; i0 < (int)total; i0 += 32 * CW_BATCH) {
                // CW_BATCH independent loads a lane before any store
                uint64_t v[CW_BATCH];
#pragma unroll
                for (int u = 0; u < CW_BATCH; ++u) {
                    const int i = i0 + u * 32 + lane;
                    v[u] = 0ull;
                    if (i < (int)total) {
                        int lo = 0, hi = nseg - 1;   // the last segment whose start is <= i
                        while (lo < hi) {
                            const int mid = (lo + hi + 1) >> 1;
                            if (hist[mid] <= (uint32_t)i) lo = mid;
                            else hi = mid - 1;
                        }
                        if (PIVOT_CHECK(i < M && i - hist[lo] < (uint32_t)p.sub_keys))
                            v[u] = src[(size_t)(lo / p.nsub) * p.chunk_keys +
                                       (size_t)(lo % p.nsub) * p.sub_keys + (i - hist[lo])];
                    }
                }
#pragma unroll
                for (int u = 0; u < CW_BATCH; ++u) {
                    const int i = i0 + u * 32 + lane;
                    if (i < (int)total) e[i] = v[u];
                }
            }
        } else {
            int off = 0;
            for (int c = 0; c < nseg; ++c) {
                const int k = (int)cnt[c];
                const uint64_t* sg =
                    src + (size_t)(c / p.nsub) * p.chunk_keys + (size_t)(c % p.nsub) * p.sub_keys;
                for (int i = lane; i < k; i += 32) e[off + i] = sg[i];
                off += k;
            }
        }
        __syncwarp();
        const int nt = (int)total;
        if (Kp < total) warp_keep_top(e, nt, Kp, hist);
        // class A (position order with a split): the top `split`
        const int split = (!p.rank_order && p.split > 0 && (uint32_t)p.split < Kp) ? p.split : 0;
        uint32_t TA = 0xFFFFFFFFu, LA = 0xFFFFFFFFu;
        if (split) {
            TA = warp_kth_largest_f([&](int i) { return key_u(e[i]); }, nt, (uint32_t)split, hist);
            uint32_t above = 0, eq = 0;
            for (int i = lane; i < nt; i += 32) {
                const uint32_t u = key_u(e[i]);
                above += u > TA;
                eq += u == TA;
            }
            for (int o = 16; o > 0; o >>= 1) {
                above += __shfl_xor_sync(0xffffffffu, above, o);
                eq += __shfl_xor_sync(0xffffffffu, eq, o);
            }
            const uint32_t need = (uint32_t)split - above;
            LA = 0;
            if (eq > need)
                LA = warp_kth_largest_f(
                    [&](int i) { return key_u(e[i]) == TA ? (uint32_t)e[i] : 0u; }, nt, need, hist);
            __syncwarp();
        }
        const int kept = warp_compact(e, 0, nt);   // == Kp
        const int Mk = pow2_at_least(kept);
        if (p.rank_order) {
            for (int i = kept + lane; i < Mk; i += 32) e[i] = 0ull;
            __syncwarp();
            warp_bitonic(e, Mk, [](uint64_t x, uint64_t y) { return x > y; });
            for (int i = lane; i < kept; i += 32) {
                out[i] = key_pos(e[i]);
                if (outs) outs[i] = key_to_float(key_u(e[i]));
            }
        } else if ((M - kept) >= 32) {
            // position order by a bitmap of the row's positions, a window of
            // WW words at a time in the space past the kept entries (bitmap,
            // then per-word prefix counts): each kept entry's slot is its
            // class's base plus its rank among the class's marked positions
            const int W = (lim >> 5) + 1;
            const int WW = min(W, (M - kept) & ~31);
            uint32_t* bm = reinterpret_cast<uint32_t*>(e + kept);
            uint32_t* pref = bm + WW;
            uint32_t base = 0;
            for (int cls = 0; cls < (split ? 2 : 1); ++cls) {
                for (int w0 = 0; w0 < W; w0 += WW) {
                    const int nw = min(WW, W - w0);
                    for (int w = lane; w < nw; w += 32) bm[w] = 0u;
                    __syncwarp();
                    for (int i = lane; i < kept; i += 32) {
                        const uint64_t k = e[i];
                        const uint32_t u = key_u(k);
                        const bool inA = !split || u > TA || (u == TA && (uint32_t)k >= LA);
                        const int wd = (key_pos(k) >> 5) - w0;
                        if (inA == (cls == 0) && wd >= 0 && wd < nw)
                            atomicOr(&bm[wd], 1u << (key_pos(k) & 31));
                    }
                    __syncwarp();
                    const int per = (nw + 31) / 32;
                    const int v0 = lane * per, v1 = min(nw, v0 + per);
                    uint32_t local = 0;
                    for (int w = v0; w < v1; ++w) local += __popc(bm[w]);
                    uint32_t inc = local;
                    for (int o = 1; o < 32; o <<= 1) {
                        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
                        if (lane >= o) inc += y;
                    }
                    uint32_t acc = inc - local;
                    for (int w = v0; w < v1; ++w) {
                        pref[w] = acc;
                        acc += __popc(bm[w]);
                    }
                    const uint32_t nwin = __shfl_sync(0xffffffffu, inc, 31);
                    __syncwarp();
                    for (int i = lane; i < kept; i += 32) {
                        const uint64_t k = e[i];
                        const uint32_t u = key_u(k);
                        const bool inA = !split || u > TA || (u == TA && (uint32_t)k >= LA);
                        const int pos = key_pos(k);
                        const int wd = (pos >> 5) - w0;
                        if (inA != (cls == 0) || wd < 0 || wd >= nw) continue;
                        const uint32_t slot =
                            base + pref[wd] + __popc(bm[wd] & ((1u << (pos & 31)) - 1u));
                        if (!PIVOT_CHECK(slot < Kp)) continue;
                        out[slot] = pos;
                        if (outs) outs[slot] = key_to_float(u);
                    }
                    base += nwin;
                    __syncwarp();
                }
            }
        } else {
            // sort key: class (A first), then position, with the score kept
            for (int i = lane; i < Mk; i += 32) {
                if (i < kept) {
                    const uint64_t k = e[i];
                    const uint32_t u = key_u(k);
                    const bool inA = split && (u > TA || (u == TA && (uint32_t)k >= LA));
                    const uint64_t cls = (split && !inA) ? 1ull : 0ull;
                    e[i] = (cls << 63) | ((uint64_t)(uint32_t)key_pos(k) << 32) | u;
                } else {
                    e[i] = ~0ull;
                }
            }
            __syncwarp();
            warp_bitonic(e, Mk, [](uint64_t x, uint64_t y) { return x < y; });
            for (int i = lane; i < kept; i += 32) {
                out[i] = (int32_t)((e[i] >> 32) & 0x7FFFFFFFu);
                if (outs) outs[i] = key_to_float((uint32_t)e[i]);
            }
        }
    }
    for (int i = (int)Kp + lane; i < K; i += 32) {
        out[i] = -1;
        if (outs) outs[i] = -INFINITY;
    }
}

}  // namespace

// Shared-memory layout, in bytes from the start of the dynamic buffer:
//   hist [HIST_BINS] u32 | scratch [64] u32 | hist256 [256] u32 | exact region
// The exact path's region (after hist256) holds sel [2 * pow2(K)] + tail
// [tail_cap] keys.  The fast path, which has no use for hist256, starts its
// region there: buf [fast_cap] keys, then the bitmaps bmS (and bmA when
// split) and, when W > HIST_BINS, pref.  All offsets are multiples of 16
// bytes up to the bitmaps, which take 32-bit accesses only.
struct SelectLayout {
    size_t exact_total, fast_total, total;
};

constexpr size_t SEL_FAST_OFF = (size_t)(HIST_BINS + 64) * 4;
constexpr size_t SEL_EXACT_OFF = SEL_FAST_OFF + 256 * 4;

static SelectLayout select_layout(int K, int tail_cap, int fast_cap, int W, bool split) {
    SelectLayout L{};
    const size_t m2 = (size_t)pow2_at_least(K);
    L.exact_total = SEL_EXACT_OFF + (2 * m2 + (size_t)tail_cap) * 8;
    L.fast_total = 0;
    if (fast_cap > 0) {
        const int nbm = split ? 2 : 1;
        L.fast_total = SEL_FAST_OFF + (size_t)fast_cap * 8 +
                       (size_t)(nbm + (W > HIST_BINS ? 1 : 0)) * W * 4;
    }
    L.total = L.exact_total > L.fast_total ? L.exact_total : L.fast_total;
    return L;
}

// Two CTAs an SM (64 registers a thread): a row's barrier-separated phases
// leave the SM idle unless another row fills the gaps.
__global__ void __launch_bounds__(SEL_THREADS, 2) select_kernel(const SelectParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem);
    uint32_t* scratch = hist + HIST_BINS;
    uint32_t* hist256 = scratch + 64;
    uint64_t* region = reinterpret_cast<uint64_t*>(hist256 + 256);   // exact path
    const int M2 = pow2_at_least(p.K);
    __shared__ uint32_t s_a, s_b;

    int r = p.row0 + blockIdx.x;
    if (p.row_list) {
        if (blockIdx.x >= *p.row_count) return;
        r = p.row_list[blockIdx.x];
    }
    const size_t ostride = p.out_stride ? (size_t)p.out_stride : (size_t)p.K;
    int32_t* out = p.out_idx + (size_t)(r - p.out_base) * ostride;
    float* outs = p.out_score ? p.out_score + (size_t)(r - p.out_base) * ostride : nullptr;

    bool ok;
    const int lim =
        select_row_limit(p, r, ok) - p.lim_shift;
    RowView v;
    v.S = p.keys ? nullptr : p.S + (size_t)(r - p.row0) * p.S_stride;
    v.keys = p.keys ? p.keys + (size_t)(r - p.row0) * p.S_stride : nullptr;
    v.lim = lim;
    v.ksc = nullptr;
    if (p.kind == SEL_PREFIX) {
        v.cand = nullptr;
        v.n = ok && lim >= 0 ? lim + 1 : 0;
    } else {
        const bool dec = p.scan_kind == SCAN_DECODE_DENSE;
        const bool var = p.scan_kind == SCAN_VARLEN_DENSE;
        const int grp = dec ? r / p.Gm : (var ? seg_group_of(p.seg, p.g, r) : r / p.g);
        v.cand = p.cand + (size_t)(grp - p.cand_base) * p.C;
        // adaptive C: entries past the group's count are not candidates
        int Cg = p.C;
        if (p.cand_count) {
            const int c = p.cand_count[grp - p.cand_base];
            Cg = c < 0 ? 0 : (c < p.C ? c : p.C);
        }
        v.n = ok ? Cg : 0;
        if (p.key_scale)
            v.ksc = p.key_scale + (dec ? (size_t)grp * p.maxlen
                                       : (var ? (size_t)p.seg.tok[seg_find(p.seg.tok, p.seg.nseq, r)]
                                              : 0));
        if (p.s_per_group) v.S = p.S + (size_t)(grp - p.cand_base) * p.S_stride;
    }
    if (!ok && threadIdx.x == 0) raise_error(ERRBIT_DATA);

    if (p.fast_cap > 0) {
        const int W = p.bitmap_words;
        FastSmem sm;
        sm.hist = hist;
        sm.scratch = scratch;
        sm.buf = reinterpret_cast<uint64_t*>(hist256);   // fast path: from hist256 on
        uint32_t* bms = reinterpret_cast<uint32_t*>(sm.buf + p.fast_cap);
        sm.bmS = bms;
        sm.bmA = p.split > 0 ? bms + W : nullptr;
        sm.pref = W > HIST_BINS ? bms + (p.split > 0 ? 2 : 1) * W : hist;
        if (select_fast(p, v, sm, &s_a, &s_b, out, outs)) return;
        __syncthreads();
    }
    select_exact(p, v, hist, scratch, hist256, region, region + 2 * M2, M2, &s_a, &s_b, out,
                 outs);
}

// Kept-entry capacity of the fast path for top-K: twice K rounded up to a
// power of two, at least 2048; 0 (exact path only) when K > 8192.
static int select_fast_cap(int K) {
    if (K > 8192) return 0;
    int c = 2048;
    while (c < 2 * K) c <<= 1;
    return c;
}

constexpr size_t SELECT_SMEM_LIMIT = 220 * 1024;

cudaError_t launch_row_threshold(const SelectParams& p_in, uint32_t* thresh, cudaStream_t stream) {
    if (p_in.nrows <= 0) return cudaSuccess;
    if (p_in.kind != SEL_PREFIX) return cudaErrorInvalidValue;
    SelectParams p = p_in;
    p.fast_cap = select_fast_cap(p.K);
    if (p.fast_cap == 0) p.fast_cap = 0x7fffffff;   // exact path only: no bound needed
    const size_t smem = THR_WARPS * THR_SMEM_WARP;
    cudaError_t e = cudaFuncSetAttribute(row_threshold_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(row_threshold_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    const int grid = (p.nrows + THR_WARPS - 1) / THR_WARPS;
    row_threshold_kernel<<<grid, THR_WARPS * 32, smem, stream>>>(p, thresh);
    return cudaGetLastError();
}

// Survivor capacity of a fused row: 2 pow2(K) keys (K = 2048: 4096 keys,
// 36 KB of shared memory a warp with its auxiliary words, six warps an SM).
// The bound leaves about K (1 + 4.5 / sqrt(m0)) survivors, m0 >= 64 samples
// for rows longer than the capacity: 1.6 K at most on average.
int fused_cap(int K) { return 2 * pow2_at_least(K < 128 ? 128 : K); }

cudaError_t launch_sample_bound(const FusedSelectParams& p, cudaStream_t stream) {
    if (p.nrows <= 0) return cudaSuccess;
    const size_t smem = (size_t)FB_WARPS * THR_BINS * 4;
    cudaError_t e = cudaFuncSetAttribute(sample_bound_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    sample_bound_kernel<<<(p.nrows + FB_WARPS - 1) / FB_WARPS, FB_WARPS * 32, smem, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_fused_finish(const FusedSelectParams& p, cudaStream_t stream) {
    if (p.nrows <= 0) return cudaSuccess;
    const size_t per = (size_t)p.cap * 8 + FF_AUX * 4;
    // one or two warps a block: blocks pack the SM's shared memory more
    // tightly than one large block would
    int warps = per * 2 <= CW_SMEM_LIMIT / 2 ? 2 : 1;
    if (per > CW_SMEM_LIMIT) return cudaErrorInvalidValue;
    const size_t smem = per * (size_t)warps;
    cudaError_t e = cudaFuncSetAttribute(fused_finish_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(fused_finish_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    fused_finish_kernel<<<(p.nrows + warps - 1) / warps, warps * 32, smem, stream>>>(p, warps);
    return cudaGetLastError();
}


// Shared memory a CTA may take for two to fit an SM (228 KB, less 1 KB
// reserved a CTA and the kernel's static words).
constexpr size_t SELECT_TWO_CTAS = 233472 / 2 - 1024 - 64;

cudaError_t launch_select(const SelectParams& p_in, cudaStream_t stream) {
    if (p_in.nrows <= 0) return cudaSuccess;
    SelectParams p = p_in;
    p.bitmap_words = (p.npos + 31) / 32;
    p.fast_cap = select_fast_cap(p.K);
    SelectLayout lay = select_layout(p.K, p.tail_cap, p.fast_cap, p.bitmap_words, p.split > 0);
    // Where the exact path's boundary buffer is what keeps a second CTA off
    // the SM (k = 4096: 2 x 4096 + 4096 keys), trim it a little: a fuller
    // boundary bin is then searched from global memory, with the same result.
    if (lay.exact_total > SELECT_TWO_CTAS && lay.fast_total <= SELECT_TWO_CTAS) {
        const int trim = (int)((lay.exact_total - SELECT_TWO_CTAS + 7) / 8);
        if (trim <= p.tail_cap / 4) {
            p.tail_cap -= trim;
            lay = select_layout(p.K, p.tail_cap, p.fast_cap, p.bitmap_words, p.split > 0);
        }
    }
    if (lay.total > SELECT_SMEM_LIMIT) {   // rows too long for the bitmaps: exact path only
        p.fast_cap = 0;
        lay = select_layout(p.K, p.tail_cap, 0, p.bitmap_words, p.split > 0);
    }
    if (lay.total > SELECT_SMEM_LIMIT) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)lay.total);
    if (e != cudaSuccess) return e;
    // the whole carveout as shared memory, so two CTAs fit where their buffers allow
    e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    select_kernel<<<p.nrows, SEL_THREADS, lay.total, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace pivot
