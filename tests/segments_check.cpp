// Host check of the ragged-batch mapping in segments.h (the same inline
// functions the kernels call): on random batches (empty and one-token
// sequences, groups and row blocks cut by launch ranges) every (row, key
// tile) of the causal prefix is covered by exactly one scan work item, a
// work item never mixes two sequences, every Refine member is scored once
// with its own group, and the proxy groups partition the tokens.
// Built with g++ by tests/test_segments_cpu.py; exits non-zero on a failure.
#include <cstdio>
#include <cstdlib>
#include <random>
#include <vector>

#include "segments.h"

using namespace pivot;

namespace {

struct Tabs {
    int B = 0, T = 0, G = 0, maxL = 0;
    std::vector<int32_t> tok, grp, itmD, itmP;
};

int cdiv(int a, int b) { return (a + b - 1) / b; }

Tabs build(const std::vector<int>& lens, int g, int P, int tpi) {
    Tabs t;
    t.B = (int)lens.size();
    t.tok.assign(t.B + 1, 0);
    t.grp.assign(t.B + 1, 0);
    t.itmD.assign(t.B + 1, 0);
    t.itmP.assign(t.B + 1, 0);
    for (int i = 0; i < t.B; ++i) {
        const int len = lens[i], ng = cdiv(len, g), ch = cdiv(cdiv(len, 128), tpi);
        t.tok[i + 1] = t.tok[i] + len;
        t.grp[i + 1] = t.grp[i] + ng;
        t.itmD[i + 1] = t.itmD[i] + cdiv(len, P) * ch;
        t.itmP[i + 1] = t.itmP[i] + cdiv(ng, P) * ch;
        if (len > t.maxL) t.maxL = len;
    }
    t.T = t.tok[t.B];
    t.G = t.grp[t.B];
    return t;
}

[[noreturn]] void fail(const char* what, int a, int b) {
    std::printf("FAIL %s (%d, %d)\n", what, a, b);
    std::exit(1);
}

// the sequence of entry x, by a linear walk
int seq_of(const std::vector<int32_t>& pre, int x) {
    for (int b = 0; b + 1 < (int)pre.size(); ++b)
        if (pre[b] <= x && x < pre[b + 1]) return b;
    fail("entry outside every sequence", x, 0);
}

int brute_dense_lim(const Tabs& t, int r) { return r - t.tok[seq_of(t.tok, r)]; }

int brute_proxy_lim(const Tabs& t, int g, int j) {
    const int b = seq_of(t.grp, j);
    const int len = t.tok[b + 1] - t.tok[b];
    const int last = (j - t.grp[b] + 1) * g;
    return (last < len ? last : len) - 1;
}

void check_scan(const Tabs& t, bool dense, int g, int P, int tpi, int cap) {
    const std::vector<int32_t>& rowpre = dense ? t.tok : t.grp;
    const std::vector<int32_t>& itm = dense ? t.itmD : t.itmP;
    const int total = dense ? t.T : t.G;
    SegTable s{t.tok.data(), t.grp.data(), itm.data(), t.B, 0, tpi};
    std::vector<int> lim(total);
    for (int r = 0; r < total; ++r) {
        lim[r] = dense ? brute_dense_lim(t, r) : brute_proxy_lim(t, g, r);
        const int got = dense ? seg_dense_lim(s, r) : seg_proxy_lim(s, g, r);
        if (got != lim[r]) fail("row limit", r, got);
    }
    std::vector<std::vector<int>> cov(total);
    for (int r = 0; r < total; ++r) cov[r].assign(cdiv(t.maxL, 128) + 1, 0);
    for (int r0 = 0; r0 < total; r0 += cap) {
        const int r1 = r0 + cap < total ? r0 + cap : total;
        int i0, n0, i1, n1;
        seg_block_items(t.tok.data(), rowpre.data(), itm.data(), t.B, P, tpi, r0, &i0, &n0);
        seg_block_items(t.tok.data(), rowpre.data(), itm.data(), t.B, P, tpi, r1 - 1, &i1, &n1);
        s.item0 = i0;
        const int nitems = i1 + n1 - i0;
        if (i0 < 0 || i1 + n1 > itm[t.B]) fail("item range", i0, i1 + n1);
        for (int item = 0; item < nitems; ++item) {
            const SegItem si = seg_scan_item(s, rowpre.data(), P, r0, r1 - r0, item);
            if (si.rows <= 0) continue;
            if (si.rows > P) fail("block taller than P", item, si.rows);
            if (si.first < r0 || si.first + si.rows > r1) fail("rows outside the launch", item, si.first);
            if (seq_of(rowpre, si.first) != si.b || seq_of(rowpre, si.first + si.rows - 1) != si.b)
                fail("block straddles two sequences", item, si.first);
            const int maxlim = dense ? seg_dense_lim(s, si.first + si.rows - 1)
                                     : seg_proxy_lim(s, g, si.first + si.rows - 1);
            const int len = t.tok[si.b + 1] - t.tok[si.b];
            if (maxlim >= len) fail("limit past the sequence", item, maxlim);
            const int nt = (maxlim + 1 + 127) / 128;
            const int t0 = si.chunk * tpi;
            const int t1 = t0 + tpi < nt ? t0 + tpi : nt;
            for (int r = si.first; r < si.first + si.rows; ++r)
                for (int tt = t0; tt < t1; ++tt) cov[r][tt]++;
        }
    }
    for (int r = 0; r < total; ++r)
        for (int tt = 0; tt < (int)cov[r].size(); ++tt) {
            const bool need = tt * 128 <= lim[r];
            if (need && cov[r][tt] != 1) fail("tile not covered exactly once", r, tt);
            if (!need && cov[r][tt] > 1) fail("masked tile covered twice", r, tt);
        }
}

void check_refine(const Tabs& t, int g, int P, int cap) {
    SegTable s{t.tok.data(), t.grp.data(), nullptr, t.B, 0, 0};
    std::vector<int> cov(t.T, 0);
    const int ipb = cdiv(g, P);
    for (int r0 = 0; r0 < t.T; r0 += cap) {
        const int r1 = r0 + cap < t.T ? r0 + cap : t.T;
        const int jA = seg_group_of(s, g, r0), jB = seg_group_of(s, g, r1 - 1) + 1;
        for (int item = 0; item < (jB - jA) * ipb; ++item) {
            const int grp = jA + item / ipb;
            const SegItem si = seg_refine_item(s, g, P, grp, item % ipb, r0, r1 - r0);
            if (si.rows <= 0) continue;
            if (si.first < r0 || si.first + si.rows > r1) fail("members outside the launch", item, si.first);
            for (int r = si.first; r < si.first + si.rows; ++r) {
                const int b = seq_of(t.tok, r);
                if (b != si.b) fail("member of another sequence", r, si.b);
                if (t.grp[b] + (r - t.tok[b]) / g != grp) fail("member of another group", r, grp);
                cov[r]++;
            }
        }
    }
    for (int r = 0; r < t.T; ++r)
        if (cov[r] != 1) fail("member not scored exactly once", r, cov[r]);
}

void check_groups(const Tabs& t, int g) {
    SegTable s{t.tok.data(), t.grp.data(), nullptr, t.B, 0, 0};
    std::vector<int> cov(t.T, 0);
    for (int j = 0; j < t.G; ++j) {
        const SegGroup sg = seg_group(s, g, j);
        if (sg.n < 1 || sg.n > g) fail("group size", j, sg.n);
        for (int m = sg.first; m < sg.first + sg.n; ++m) {
            if (seq_of(t.tok, m) != sg.b) fail("group spans two sequences", j, m);
            if (seg_group_of(s, g, m) != j) fail("member maps to another group", m, j);
            cov[m]++;
        }
    }
    for (int m = 0; m < t.T; ++m)
        if (cov[m] != 1) fail("token not in exactly one group", m, cov[m]);
}

}  // namespace

int main() {
    std::mt19937 rng(1234);
    int cases = 0;
    for (int it = 0; it < 300; ++it) {
        const int B = 1 + (int)(rng() % 24);
        std::vector<int> lens(B);
        for (int& l : lens) {
            const int k = (int)(rng() % 10);
            l = k == 0 ? 0 : (k == 1 ? 1 : (k < 8 ? (int)(rng() % 300) : 300 + (int)(rng() % 900)));
        }
        const int Ps[3] = {3, 4, 8};
        const int gs[4] = {1, 2, 3, 8};
        const int tpis[3] = {1, 2, 32};
        const int P = Ps[rng() % 3], g = gs[rng() % 4], tpi = tpis[rng() % 3];
        const Tabs t = build(lens, g, P, tpi);
        if (t.T == 0) continue;
        const int capD = rng() % 3 == 0 ? t.T : 1 + (int)(rng() % (t.T + 1));
        const int capP = rng() % 3 == 0 ? t.G : 1 + (int)(rng() % (t.G + 1));
        const int capR = rng() % 3 == 0 ? t.T : 1 + (int)(rng() % (t.T + 1));
        check_scan(t, true, g, P, tpi, capD);
        check_scan(t, false, g, P, tpi, capP);
        check_refine(t, g, P < g ? P : g, capR);
        check_groups(t, g);
        ++cases;
    }
    std::printf("ok %d batches\n", cases);
    return 0;
}
