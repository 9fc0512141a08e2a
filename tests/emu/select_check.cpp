// Host check of the selection kernels (csrc/topk.cu compiled for the host
// with the CUDA features emulated, emu.h): every row the select writes must
// equal a plain sort's answer -- the top K entries by (score desc, position
// asc), listed by ascending position (with `split`, the top `split` first),
// -1 padded.  Built and run by tests/test_select_emu_cpu.py under
// AddressSanitizer and UndefinedBehaviorSanitizer.
//
//   select_check prefix <L> <K> <split> <dist> <rows> <use_bound>
//   select_check cand <C> <K> <mode> <rows>
// dist: 0 normal, 1 few distinct values (heavy ties), 2 signed zeros and
// small integers, 3 a heavy tail (a few huge scores); mode: 0 plain, 1 ties,
// 2 rows padded with -1, 3 with per-key scales.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <random>
#include <string>
#include <vector>

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

int run_cand(int C, int K, int mode, int nrows) {
    const int L = 20000;
    std::mt19937 rng(7 + mode);
    std::vector<int32_t> cand(C), out(K);
    std::vector<float> S(C), outs(K), ksc(L);
    for (auto& x : ksc) x = std::uniform_real_distribution<float>(0.5f, 2.0f)(rng);
    std::vector<int> all(L);
    int bad = 0;
    for (int r = 0; r < nrows; ++r) {
        // the proxy's top-K (ascending), then the rest (ascending), -1 padded
        for (int i = 0; i < L; ++i) all[i] = i;
        std::shuffle(all.begin(), all.end(), rng);
        const int nreal = mode == 2 ? C / 2 + (int)(rng() % (C / 2)) : C;
        const int s = std::min(K, nreal);
        std::vector<int> A(all.begin(), all.begin() + s), B(all.begin() + s, all.begin() + nreal);
        std::sort(A.begin(), A.end());
        std::sort(B.begin(), B.end());
        for (int i = 0; i < C; ++i) cand[i] = i < s ? A[i] : (i < nreal ? B[i - s] : -1);
        for (int i = 0; i < C; ++i)
            S[i] = mode == 1 ? (float)(rng() % 7) : std::normal_distribution<float>(1.f, 3.f)(rng);
        const int t = (int)(rng() % L);   // the member's position
        SelectParams sp{};
        sp.kind = SEL_CANDIDATES;
        sp.scan_kind = SCAN_PREFILL_DENSE;
        sp.row0 = t;
        sp.nrows = 1;
        sp.L = L;
        sp.g = 1;
        sp.Gm = 1;
        sp.S = S.data();
        sp.S_stride = C;
        sp.cand = cand.data();
        sp.cand_base = t;
        sp.C = C;
        sp.K = K;
        sp.out_idx = out.data();
        sp.out_score = outs.data();
        sp.out_base = t;
        sp.tail_cap = 2048;
        sp.npos = L;
        sp.key_scale = mode == 3 ? ksc.data() : nullptr;
        std::fill(out.begin(), out.end(), -7);
        if (launch_select(sp, nullptr) != cudaSuccess) return 2;
        std::vector<std::pair<uint32_t, int>> e;
        for (int i = 0; i < C; ++i)
            if (cand[i] >= 0 && cand[i] <= t) {
                float x = S[i];
                if (mode == 3) x = x * ksc[cand[i]];
                e.push_back({okey(x), cand[i]});
            }
        if (reference(e, K, 0) != std::vector<int>(out.begin(), out.end())) {
            ++bad;
            std::printf("candidate row %d (t = %d): mismatch\n", r, t);
        }
    }
    return bad;
}

}  // namespace

int main(int argc, char** argv) {
    if (argc < 2) return 2;
    const std::string what = argv[1];
    int bad;
    if (what == "prefix" && argc == 8)
        bad = run_prefix(atoi(argv[2]), atoi(argv[3]), atoi(argv[4]), atoi(argv[5]), atoi(argv[6]),
                         atoi(argv[7]) != 0);
    else if (what == "cand" && argc == 6)
        bad = run_cand(atoi(argv[2]), atoi(argv[3]), atoi(argv[4]), atoi(argv[5]));
    else
        return 2;
    std::printf("%d bad rows, error word %u\n", bad, g_error_word);
    return bad || g_error_word ? 1 : 0;
}
