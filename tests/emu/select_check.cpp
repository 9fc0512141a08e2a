// Host check of the selection kernels (csrc/topk.cu compiled for the host
// with the CUDA features emulated, emu.h): every row the select writes must
// equal a plain sort's answer -- the top K entries by (score desc, position
// asc), listed by ascending position (with `split`, the top `split` first),
// -1 padded.  Built and run by tests/test_select_emu_cpu.py under
// AddressSanitizer and UndefinedBehaviorSanitizer.
//
//   select_check prefix <L> <K> <split> <dist> <rows> <use_bound>
//   select_check cand <C> <K> <mode> <rows> <order> <layout>
//   select_check varlen <kind> <g> <K> <C>     (ragged batch rows, see run_varlen)
//   select_check decode <kind> <K>             (MTP decode rows, see run_decode)
//   select_check backfill <L> <g> <C> <K>      (Reuse with backfill, see run_backfill)
//   select_check planted <L> <K> <npos>        (bitmap too small; debug build only)
//   select_check fused <L> <K> <split> <dist> <rows> <r0> <order> <sigmas> <kind>
//                                              (selection fused into the scan, see run_fused)
// dist: 0 normal, 1 few distinct values (heavy ties), 2 signed zeros and
// small integers, 3 a heavy tail (a few huge scores), 4 normal scores rounded
// to eighths (a few hundred to a thousand ties at the k-th score), 5 one
// value everywhere (every entry tied); mode: 0 plain, 1 ties,
// 2 rows padded with -1, 3 with per-key scales; order: 0 ascending positions,
// 1 rank order; layout: 0 the proxy scan's two ascending runs, 1 shuffled.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <random>
#include <string>
#include <vector>

#include "common.cuh"   // the error bits
#include "kernels.h"

namespace pivot {
uint32_t g_error_word = 0;
}
using namespace pivot;

namespace {

uint32_t okey(float f) {   // the order of (score desc): larger keys first, -0 == +0
    uint32_t u;
    const float g = f + 0.0f;
    std::memcpy(&u, &g, 4);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

std::vector<int> reference(std::vector<std::pair<uint32_t, int>> e, int K, int split) {
    std::sort(e.begin(), e.end(), [](const auto& a, const auto& b) {
        return a.first != b.first ? a.first > b.first : a.second < b.second;
    });
    const int kp = std::min<int>(K, (int)e.size());
    const int sp = (split > 0 && split < kp) ? split : 0;
    std::vector<int> A, B;
    for (int i = 0; i < kp; ++i) (i < sp ? A : B).push_back(e[i].second);
    std::sort(A.begin(), A.end());
    std::sort(B.begin(), B.end());
    A.insert(A.end(), B.begin(), B.end());
    while ((int)A.size() < K) A.push_back(-1);
    return A;
}

float draw(std::mt19937& rng, int dist) {
    switch (dist) {
        case 1: return (float)(rng() % 5);
        case 2: {
            const int v = (int)(rng() % 7) - 3;
            return v == 0 ? ((rng() & 1) ? -0.0f : 0.0f) : (float)v;
        }
        case 3: return (rng() % 997 == 0) ? 1e6f * (1 + (float)(rng() % 9))
                                          : std::normal_distribution<float>(0.f, 1.f)(rng);
        case 4: return std::round(std::normal_distribution<float>(0.f, 1.f)(rng) * 8.f) / 8.f;
        case 5: return 1.5f;
        default: return std::normal_distribution<float>(0.f, 1.f)(rng);
    }
}

int run_prefix(int L, int K, int split, int dist, int nrows, bool use_bound) {
    std::mt19937 rng(11 + 7 * dist + K);
    std::vector<float> S(L);
    std::vector<int32_t> out(K);
    std::vector<float> outs(K);
    int bad = 0;
    for (int r = 0; r < nrows; ++r) {
        // rows of every length class: short (fits the buffer) to the full L
        const int t = r == 0 ? L - 1 : (r == 1 ? std::min(K / 2, L - 1) : (int)(rng() % L));
        for (auto& x : S) x = draw(rng, dist);
        SelectParams sp{};
        sp.kind = SEL_PREFIX;
        sp.scan_kind = SCAN_PREFILL_DENSE;
        sp.row0 = t;
        sp.nrows = 1;
        sp.L = L;
        sp.g = 1;
        sp.Gm = 1;
        sp.S = S.data();
        sp.S_stride = L;
        sp.K = K;
        sp.split = split;
        sp.out_idx = out.data();
        sp.out_score = outs.data();
        sp.out_base = t;
        sp.tail_cap = 4096;
        sp.npos = L;
        uint32_t bound = 0;
        if (use_bound) {
            if (launch_row_threshold(sp, &bound, nullptr) != cudaSuccess) return 2;
            sp.thresh = &bound;
        }
        std::fill(out.begin(), out.end(), -7);
        if (launch_select(sp, nullptr) != cudaSuccess) return 2;
        std::vector<std::pair<uint32_t, int>> e;
        for (int i = 0; i <= t; ++i) e.push_back({okey(S[i]), i});
        if (reference(e, K, split) != std::vector<int>(out.begin(), out.end())) {
            ++bad;
            std::printf("prefix row %d (t = %d): mismatch\n", r, t);
        }
    }
    return bad;
}

// Top K of the entries (score desc, position asc), in that rank order,
// -1 padded.
std::vector<int> reference_rank(std::vector<std::pair<uint32_t, int>> e, int K) {
    std::sort(e.begin(), e.end(), [](const auto& a, const auto& b) {
        return a.first != b.first ? a.first > b.first : a.second < b.second;
    });
    std::vector<int> A;
    for (int i = 0; i < std::min<int>(K, (int)e.size()); ++i) A.push_back(e[i].second);
    while ((int)A.size() < K) A.push_back(-1);
    return A;
}

// Candidate rows of `nrows` consecutive members (one launch; each member its
// own group, g = 1), member t seeing positions <= t.  layout 0: the proxy
// scan's rows (its top-K ascending, then the rest ascending, -1 padded);
// layout 1: the same positions shuffled.  order 0: positions ascending;
// order 1: rank order.
int run_cand(int C, int K, int mode, int nrows, int order, int layout) {
    const int L = 20000;
    std::mt19937 rng(7 + mode + 13 * layout + 29 * order);
    std::vector<int32_t> cand((size_t)nrows * C), out((size_t)nrows * K);
    std::vector<float> S((size_t)nrows * C), outs((size_t)nrows * K), ksc(L);
    for (auto& x : ksc) x = std::uniform_real_distribution<float>(0.5f, 2.0f)(rng);
    std::vector<int> all(L);
    const int t0 = (int)(rng() % (L - nrows));
    for (int r = 0; r < nrows; ++r) {
        for (int i = 0; i < L; ++i) all[i] = i;
        std::shuffle(all.begin(), all.end(), rng);
        const int nreal = mode == 2 ? C / 2 + (int)(rng() % (C / 2 + 1)) : C;
        const int s = std::min(K, nreal);
        std::vector<int> A(all.begin(), all.begin() + s), B(all.begin() + s, all.begin() + nreal);
        std::sort(A.begin(), A.end());
        std::sort(B.begin(), B.end());
        int32_t* c = cand.data() + (size_t)r * C;
        for (int i = 0; i < C; ++i) c[i] = i < s ? A[i] : (i < nreal ? B[i - s] : -1);
        if (layout == 1) std::shuffle(c, c + C, rng);
        for (int i = 0; i < C; ++i)
            S[(size_t)r * C + i] =
                mode == 1 ? (float)(rng() % 7) : std::normal_distribution<float>(1.f, 3.f)(rng);
    }
    SelectParams sp{};
    sp.kind = SEL_CANDIDATES;
    sp.scan_kind = SCAN_PREFILL_DENSE;
    sp.row0 = t0;
    sp.nrows = nrows;
    sp.L = L;
    sp.g = 1;
    sp.Gm = 1;
    sp.S = S.data();
    sp.S_stride = C;
    sp.cand = cand.data();
    sp.cand_base = t0;
    sp.C = C;
    sp.K = K;
    sp.out_idx = out.data();
    sp.out_score = outs.data();
    sp.out_base = t0;
    sp.tail_cap = 2048;
    sp.npos = L;
    sp.rank_order = order;
    sp.key_scale = mode == 3 ? ksc.data() : nullptr;
    std::fill(out.begin(), out.end(), -7);
    if (launch_select(sp, nullptr) != cudaSuccess) return 2;
    int bad = 0;
    for (int r = 0; r < nrows; ++r) {
        const int t = t0 + r;
        const int32_t* c = cand.data() + (size_t)r * C;
        std::vector<std::pair<uint32_t, int>> e;
        for (int i = 0; i < C; ++i)
            if (c[i] >= 0 && c[i] <= t) {
                float x = S[(size_t)r * C + i];
                if (mode == 3) x = x * ksc[c[i]];
                e.push_back({okey(x), c[i]});
            }
        const std::vector<int> want = order ? reference_rank(e, K) : reference(e, K, 0);
        if (want != std::vector<int>(out.begin() + (size_t)r * K,
                                     out.begin() + (size_t)(r + 1) * K)) {
            ++bad;
            std::printf("candidate row %d (t = %d): mismatch\n", r, t);
        }
        // scores line up with the positions
        for (int i = 0; i < K && out[(size_t)r * K + i] >= 0; ++i) {
            const int pos = out[(size_t)r * K + i];
            int at = -1;
            for (int j = 0; j < C; ++j)
                if (c[j] == pos) at = j;
            float x = S[(size_t)r * C + at];
            if (mode == 3) x = x * ksc[pos];
            if (okey(x) != okey(outs[(size_t)r * K + i])) {
                ++bad;
                std::printf("candidate row %d: score of slot %d\n", r, i);
                break;
            }
        }
    }
    return bad;
}

// Ragged batch rows: packed rows of several sequences, mapped through the
// segment tables.  kind 0: dense rows (token r, limit = its position);
// kind 1: proxy rows (group j, limit = its last member, top-C with the top K
// first); kind 2: candidate rows of members (their group's candidates,
// positions <= the member's, key scales from the sequence's first token).
int run_varlen(int kind, int g, int K, int C) {
    const std::vector<int> lens = {0, 5, 1, 300, 0, 33, 26, 9};
    const int B = (int)lens.size();
    std::vector<int32_t> tok(B + 1, 0), grp(B + 1, 0);
    int maxL = 0;
    for (int b = 0; b < B; ++b) {
        tok[b + 1] = tok[b] + lens[b];
        grp[b + 1] = grp[b] + (lens[b] + g - 1) / g;
        maxL = std::max(maxL, lens[b]);
    }
    const int T = tok[B], G = grp[B];
    SegTable seg{tok.data(), grp.data(), nullptr, B, 0, 0};
    std::mt19937 rng(23 + kind);
    const int rows = kind == 1 ? G : T;
    const int width = kind == 2 ? C : maxL;
    const int Kout = kind == 1 ? C : K;
    std::vector<float> S((size_t)rows * width), ksc(T);
    for (auto& x : S) x = (rng() % 3 == 0) ? (float)(rng() % 4) : std::normal_distribution<float>(0.f, 1.f)(rng);
    for (auto& x : ksc) x = std::uniform_real_distribution<float>(0.5f, 2.0f)(rng);
    std::vector<int32_t> cand;
    if (kind == 2) {   // each group's candidates: distinct positions of its sequence
        cand.assign((size_t)G * C, -1);
        for (int b = 0; b < B; ++b)
            for (int j = grp[b]; j < grp[b + 1]; ++j) {
                std::vector<int> all(lens[b]);
                for (int i = 0; i < lens[b]; ++i) all[i] = i;
                std::shuffle(all.begin(), all.end(), rng);
                const int n = std::min(C, lens[b]);
                std::sort(all.begin(), all.begin() + n);
                for (int i = 0; i < n; ++i) cand[(size_t)j * C + i] = all[i];
            }
    }
    std::vector<int32_t> out((size_t)rows * Kout, -7);
    std::vector<float> outs((size_t)rows * Kout);
    std::vector<uint32_t> bound(rows);
    SelectParams sp{};
    sp.kind = kind == 2 ? SEL_CANDIDATES : SEL_PREFIX;
    sp.scan_kind = kind == 1 ? SCAN_VARLEN_PROXY : SCAN_VARLEN_DENSE;
    sp.row0 = 0;
    sp.nrows = rows;
    sp.L = maxL;
    sp.g = g;
    sp.Gm = 1;
    sp.S = S.data();
    sp.S_stride = width;
    sp.K = Kout;
    sp.split = kind == 1 ? K : 0;
    sp.out_idx = out.data();
    sp.out_score = outs.data();
    sp.out_base = 0;
    sp.tail_cap = 4096;
    sp.npos = maxL;
    sp.seg = seg;
    if (kind == 2) {
        sp.cand = cand.data();
        sp.cand_base = 0;
        sp.C = C;
        sp.key_scale = ksc.data();
    }
    // the rows at each sequence's edges (the first two and the last two), in
    // one launch per contiguous range; rows start at row0 in S and thresh
    const std::vector<int32_t>& pre = kind == 1 ? grp : tok;
    std::vector<int> pick;
    for (int b = 0; b < B; ++b)
        for (int r = pre[b]; r < pre[b + 1]; ++r)
            if (r < pre[b] + 2 || r >= pre[b + 1] - 2) pick.push_back(r);
    for (size_t a = 0; a < pick.size();) {
        size_t z = a + 1;
        while (z < pick.size() && pick[z] == pick[z - 1] + 1) ++z;
        SelectParams q = sp;
        q.row0 = pick[a];
        q.nrows = (int)(z - a);
        q.S = S.data() + (size_t)q.row0 * width;
        if (kind != 2) {
            if (launch_row_threshold(q, bound.data() + q.row0, nullptr) != cudaSuccess) return 2;
            q.thresh = bound.data() + q.row0;
        }
        if (launch_select(q, nullptr) != cudaSuccess) return 2;
        a = z;
    }
    int bad = 0;
    for (int r : pick) {
        int b = 0;
        while (!(pre[b] <= r && r < pre[b + 1])) ++b;
        const int len = lens[b];
        std::vector<std::pair<uint32_t, int>> e;
        const float* row = S.data() + (size_t)r * width;
        if (kind == 0) {
            for (int i = 0; i <= r - tok[b]; ++i) e.push_back({okey(row[i]), i});
        } else if (kind == 1) {
            const int lim = std::min((r - grp[b] + 1) * g, len) - 1;
            for (int i = 0; i <= lim; ++i) e.push_back({okey(row[i]), i});
        } else {
            const int t = r - tok[b], j = grp[b] + t / g;
            for (int i = 0; i < C; ++i) {
                const int pos = cand[(size_t)j * C + i];
                if (pos >= 0 && pos <= t) e.push_back({okey(row[i] * ksc[tok[b] + pos]), pos});
            }
        }
        const std::vector<int> want = reference(e, Kout, kind == 1 ? K : 0);
        if (want != std::vector<int>(out.begin() + (size_t)r * Kout, out.begin() + (size_t)(r + 1) * Kout)) {
            ++bad;
            std::printf("ragged kind %d row %d (sequence %d): mismatch\n", kind, r, b);
        }
    }
    return bad;
}

// Reuse with backfill: member t of group j = t / g takes the top K of the
// group's candidates at or before t, ranked by the group's proxy scores
// (one score row per group), lower position first on ties.
int run_backfill(int L, int g, int C, int K) {
    const int G = (L + g - 1) / g;
    std::mt19937 rng(41 + g);
    std::vector<int32_t> cand((size_t)G * C, -1);
    std::vector<float> sc((size_t)G * C);
    for (int j = 0; j < G; ++j) {
        const int e = std::min(L, (j + 1) * g) - 1;
        std::vector<int> all(e + 1);
        for (int i = 0; i <= e; ++i) all[i] = i;
        std::shuffle(all.begin(), all.end(), rng);
        const int n = std::min(C, e + 1);
        std::sort(all.begin(), all.begin() + n);
        for (int i = 0; i < n; ++i) cand[(size_t)j * C + i] = all[i];
        for (int i = 0; i < C; ++i) sc[(size_t)j * C + i] = (float)(rng() % 6);   // many ties
    }
    std::vector<int32_t> out((size_t)L * K, -7);
    SelectParams sp{};
    sp.kind = SEL_CANDIDATES;
    sp.scan_kind = SCAN_PREFILL_DENSE;
    sp.row0 = 0;
    sp.nrows = L;
    sp.L = L;
    sp.g = g;
    sp.Gm = 1;
    sp.S = sc.data();
    sp.S_stride = C;
    sp.s_per_group = 1;
    sp.cand = cand.data();
    sp.cand_base = 0;
    sp.C = C;
    sp.K = K;
    sp.out_idx = out.data();
    sp.out_base = 0;
    sp.tail_cap = 4096;
    sp.npos = L;
    if (launch_select(sp, nullptr) != cudaSuccess) return 2;
    int bad = 0;
    for (int t = 0; t < L; ++t) {
        const int j = t / g;
        std::vector<std::pair<uint32_t, int>> e;
        for (int i = 0; i < C; ++i) {
            const int pos = cand[(size_t)j * C + i];
            if (pos >= 0 && pos <= t) e.push_back({okey(sc[(size_t)j * C + i]), pos});
        }
        if (reference(e, K, 0) != std::vector<int>(out.begin() + (size_t)t * K, out.begin() + (size_t)(t + 1) * K)) {
            ++bad;
            std::printf("backfill row %d: mismatch\n", t);
        }
    }
    return bad;
}

// Decode rows (the MTP members of B sequences with cached keys): kind 0,
// member m of sequence b sees [0, cache_len[b] - Gm + m]; kind 1, the proxy
// of sequence b sees [0, cache_len[b] - 1].  Cache lengths outside the
// valid range give an all -1 row and raise the data error.
int run_decode(int kind, int K) {
    const int B = 6, Gm = 3, maxlen = 700;
    const std::vector<int32_t> cache_len = {3, 700, 41, 2, 900, 260};   // 2 and 900 invalid
    const int rows = kind == 0 ? B * Gm : B;
    std::mt19937 rng(31 + kind);
    std::vector<float> S((size_t)rows * maxlen);
    for (auto& x : S) x = (rng() % 4 == 0) ? (float)(rng() % 3) : std::normal_distribution<float>(0.f, 1.f)(rng);
    std::vector<int32_t> out((size_t)rows * K, -7);
    std::vector<float> outs((size_t)rows * K);
    SelectParams sp{};
    sp.kind = SEL_PREFIX;
    sp.scan_kind = kind == 0 ? SCAN_DECODE_DENSE : SCAN_DECODE_PROXY;
    sp.row0 = 0;
    sp.nrows = rows;
    sp.Gm = Gm;
    sp.g = 1;
    sp.maxlen = maxlen;
    sp.cache_len = cache_len.data();
    sp.S = S.data();
    sp.S_stride = maxlen;
    sp.K = K;
    sp.out_idx = out.data();
    sp.out_score = outs.data();
    sp.out_base = 0;
    sp.tail_cap = 4096;
    sp.npos = maxlen;
    if (launch_select(sp, nullptr) != cudaSuccess) return 2;
    int bad = 0;
    for (int r = 0; r < rows; ++r) {
        const int b = kind == 0 ? r / Gm : r, m = kind == 0 ? r % Gm : 0;
        const int n = cache_len[b];
        const bool valid = kind == 0 ? (n >= Gm && n <= maxlen) : (n >= 1 && n <= maxlen);
        std::vector<std::pair<uint32_t, int>> e;
        if (valid) {
            const int lim = kind == 0 ? n - Gm + m : n - 1;
            for (int i = 0; i <= lim; ++i) e.push_back({okey(S[(size_t)r * maxlen + i]), i});
        }
        if (reference(e, K, 0) != std::vector<int>(out.begin() + (size_t)r * K, out.begin() + (size_t)(r + 1) * K)) {
            ++bad;
            std::printf("decode kind %d row %d: mismatch\n", kind, r);
        }
    }
    // the invalid lengths must have raised the data error (and nothing else)
    if (g_error_word != ERRBIT_DATA) {
        std::printf("error word %u, expected the data error\n", g_error_word);
        ++bad;
    }
    g_error_word = 0;
    return bad;
}

// The selection fused into the scan, on prefix rows [r0, r0 + nrows) of a
// dense (kind 0) or proxy (kind 1, groups of g = 8) scan: sample scores as
// the sample scan writes them, the bound kernel, the filter scan's appends
// emulated here (every score at or above the row's bound, shuffled within
// each 4096-key chunk, as the scan's atomics may leave them), the warp
// finish, then for the rows it listed the keep-everything regions and the
// block select on keys.  Every row must equal the plain sort.  Prints the
// number of rows that took the fallback.
int run_fused(int L, int K, int split, int dist, int nrows, int r0, int order, float sigmas,
              int kind) {
    const int g = kind == 1 ? 8 : 1;
    const int KTS = 32, CK = 32 * 128;
    const int tiles = (L + 127) / 128;
    const long long ss = (long long)((tiles + KTS - 1) / KTS) * 128;
    const int nch = (tiles + 31) / 32;
    const long long sv = (long long)nch * CK;
    std::mt19937 rng(31 + 7 * dist + K + r0);
    std::vector<float> samp((size_t)nrows * ss, 0.0f);
    std::vector<uint64_t> surv((size_t)nrows * sv, 0);
    std::vector<uint32_t> cnt((size_t)nrows * nch * 4, 0xDEADu), bound(nrows);
    std::vector<int32_t> miss(nrows, -9), out((size_t)nrows * K, -7);
    std::vector<float> outs((size_t)nrows * K);
    uint32_t nmiss = 12345;
    std::vector<std::vector<float>> S(nrows);
    auto lim_of = [&](int r) { return kind == 1 ? std::min(L, (r + 1) * g) - 1 : r; };
    for (int i = 0; i < nrows; ++i) {
        const int lim = lim_of(r0 + i);
        S[i].resize(lim + 1);
        for (auto& x : S[i]) x = draw(rng, dist);
        for (long long j = 0; j < ss; ++j) {
            const long long pos = (j / 128) * KTS * 128 + j % 128;
            if (pos <= lim) samp[(size_t)i * ss + j] = S[i][pos];
        }
    }
    FusedSelectParams fp{};
    fp.scan_kind = kind == 1 ? SCAN_PREFILL_PROXY : SCAN_PREFILL_DENSE;
    fp.row0 = r0;
    fp.nrows = nrows;
    fp.L = L;
    fp.g = g;
    fp.K = K;
    fp.split = split;
    fp.rank_order = order;
    fp.samp = samp.data();
    fp.samp_stride = ss;
    fp.kts = KTS;
    fp.sigmas = sigmas;
    fp.bound = bound.data();
    fp.cap = fused_cap(K);
    fp.surv = surv.data();
    fp.surv_stride = sv;
    fp.surv_count = cnt.data();
    fp.nchunks = nch;
    fp.chunk_keys = CK;
    fp.nsub = 4;
    fp.sub_keys = CK / 4;
    fp.out_idx = out.data();
    fp.out_score = outs.data();
    fp.out_base = r0;
    fp.miss_list = miss.data();
    fp.miss_count = &nmiss;
    if (launch_sample_bound(fp, nullptr) != cudaSuccess) return 2;
    if (nmiss != 0) { std::printf("miss count not cleared\n"); return 3; }
    // the filter scan: each epilogue warp appends the survivors among its
    // TMEM lane quarter's keys (32 of every 128-key tile) to its own
    // sub-region of the chunk, in an order the emulation shuffles, and
    // writes the count
    auto key_of = [&](int i, int pos) {
        return ((uint64_t)okey(S[i][pos]) << 32) | (0xFFFFFFFFu - (uint32_t)pos);
    };
    auto fill = [&](int i, uint32_t T) {
        const float tf = T <= 0x00800000u ? -INFINITY : key_to_float(T);
        const int lim = lim_of(r0 + i);
        for (int c = 0; c * CK <= lim; ++c) {
            for (int q = 0; q < 4; ++q) {
                std::vector<uint64_t> kept;
                for (int pos = c * CK; pos <= std::min(lim, (c + 1) * CK - 1); ++pos)
                    if ((pos % 128) / 32 == q && S[i][pos] >= tf) kept.push_back(key_of(i, pos));
                std::shuffle(kept.begin(), kept.end(), rng);
                std::copy(kept.begin(), kept.end(),
                          surv.begin() + (size_t)i * sv + (size_t)c * CK + (size_t)q * (CK / 4));
                cnt[((size_t)i * nch + c) * 4 + q] = (uint32_t)kept.size();
            }
        }
    };
    for (int i = 0; i < nrows; ++i) fill(i, bound[i]);
    if (launch_fused_finish(fp, nullptr) != cudaSuccess) return 2;
    // the fallback: the listed rows' rescan keeps every key, each at its own
    // position, then the block select reads them as keys
    for (uint32_t m = 0; m < nmiss; ++m) {
        const int i = miss[m] - r0;
        for (int pos = 0; pos <= lim_of(r0 + i); ++pos) surv[(size_t)i * sv + pos] = key_of(i, pos);
    }
    SelectParams sp{};
    sp.kind = SEL_PREFIX;
    sp.scan_kind = fp.scan_kind;
    sp.row0 = r0;
    sp.nrows = nrows;
    sp.L = L;
    sp.g = g;
    sp.Gm = 1;
    sp.keys = surv.data();
    sp.S_stride = sv;
    sp.K = K;
    sp.split = split;
    sp.npos = L;
    sp.out_idx = out.data();
    sp.out_score = outs.data();
    sp.out_base = r0;
    sp.tail_cap = 4096;
    sp.rank_order = order;
    sp.row_list = miss.data();
    sp.row_count = &nmiss;
    if (launch_select(sp, nullptr) != cudaSuccess) return 2;
    int bad = 0;
    for (int i = 0; i < nrows; ++i) {
        std::vector<std::pair<uint32_t, int>> e;
        for (int pos = 0; pos < (int)S[i].size(); ++pos) e.push_back({okey(S[i][pos]), pos});
        const std::vector<int> want = order ? reference_rank(e, K) : reference(e, K, split);
        if (want != std::vector<int>(out.begin() + (size_t)i * K, out.begin() + (size_t)(i + 1) * K)) {
            ++bad;
            std::printf("fused row %d: mismatch\n", r0 + i);
        }
    }
    std::printf("fallback rows %u of %d\n", nmiss, nrows);
    return bad;
}

// A planted mistake in the launch parameters: the bitmap sized for only
// `npos` positions while the rows reach L - 1.  Without PIVOT_DEBUG this
// would write past the bitmap; with it every such access is skipped and the
// error word carries the bounds bit.
int run_planted(int L, int K, int npos) {
    std::mt19937 rng(99);
    std::vector<float> S(L);
    for (auto& x : S) x = draw(rng, 0);
    std::vector<int32_t> out(K);
    std::vector<float> outs(K);
    SelectParams sp{};
    sp.kind = SEL_PREFIX;
    sp.scan_kind = SCAN_PREFILL_DENSE;
    sp.row0 = L - 1;
    sp.nrows = 1;
    sp.L = L;
    sp.g = 1;
    sp.Gm = 1;
    sp.S = S.data();
    sp.S_stride = L;
    sp.K = K;
    sp.out_idx = out.data();
    sp.out_score = outs.data();
    sp.out_base = L - 1;
    sp.tail_cap = 4096;
    sp.npos = npos;
    return launch_select(sp, nullptr) == cudaSuccess ? 0 : 2;
}

}  // namespace

int main(int argc, char** argv) {
    if (argc < 2) return 2;
    const std::string what = argv[1];
    int bad;
    if (what == "prefix" && argc == 8)
        bad = run_prefix(atoi(argv[2]), atoi(argv[3]), atoi(argv[4]), atoi(argv[5]), atoi(argv[6]),
                         atoi(argv[7]) != 0);
    else if (what == "cand" && argc == 8)
        bad = run_cand(atoi(argv[2]), atoi(argv[3]), atoi(argv[4]), atoi(argv[5]), atoi(argv[6]),
                       atoi(argv[7]));
    else if (what == "fused" && argc == 11)
        bad = run_fused(atoi(argv[2]), atoi(argv[3]), atoi(argv[4]), atoi(argv[5]), atoi(argv[6]),
                        atoi(argv[7]), atoi(argv[8]), (float)atof(argv[9]), atoi(argv[10]));
    else if (what == "planted" && argc == 5)
        bad = run_planted(atoi(argv[2]), atoi(argv[3]), atoi(argv[4]));
    else if (what == "backfill" && argc == 6)
        bad = run_backfill(atoi(argv[2]), atoi(argv[3]), atoi(argv[4]), atoi(argv[5]));
    else if (what == "decode" && argc == 4)
        bad = run_decode(atoi(argv[2]), atoi(argv[3]));
    else if (what == "varlen" && argc == 6)
        bad = run_varlen(atoi(argv[2]), atoi(argv[3]), atoi(argv[4]), atoi(argv[5]));
    else
        return 2;
    std::printf("%d bad rows, error word %u\n", bad, g_error_word);
    return bad || g_error_word ? 1 : 0;
}
