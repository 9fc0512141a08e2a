// segments.h -- the sequences of a ragged (packed) batch as seen by one
// kernel launch.  Plain C++ usable on the host and the device, so the
// mapping can be checked on the CPU.
//
// Sequence b of the batch owns tokens [tok[b], tok[b+1]) of the packed
// q / w / k rows, groups [grp[b], grp[b+1]) of the packed proxy rows
// (ceil(len_b / g) groups, never spanning two sequences: the PIVOT abstract
// groups consecutive queries of one sequence), and scan work items
// [itm[b], itm[b+1]) of a launch: its rows (tokens, or groups for the proxy
// scan) in blocks of P that never straddle two sequences (a block's keys are
// one sequence's), each block split into chunks of `tpi` key tiles of 128
// covering the sequence's keys.  Positions are counted from each sequence's
// first token.
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define SEG_HD __host__ __device__ __forceinline__
#else
#define SEG_HD inline
#endif

namespace pivot {

struct SegTable {
    const int32_t* tok;   // [nseq + 1] token prefix (cu_seqlens)
    const int32_t* grp;   // [nseq + 1] group prefix
    const int32_t* itm;   // [nseq + 1] scan work-item prefix of the launch's row kind
    int nseq;
    int item0;            // first work item of the launch
    int tpi;              // key tiles per work item
};

// The sequence holding entry x of a prefix array pre[0..n] (pre[0] <= x <
// pre[n]): the largest b < n with pre[b] <= x, which skips empty sequences.
SEG_HD int seg_find(const int32_t* pre, int n, int x) {
    int lo = 0, hi = n;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (pre[mid] <= x) lo = mid;
        else hi = mid;
    }
    return lo;
}

// Work items of a sequence of len keys: blocks of P rows x chunks of tpi
// key tiles.
SEG_HD int seg_chunks(int len, int tpi) { return ((len + 127) / 128 + tpi - 1) / tpi; }

// Work item `item` of a launch (relative to item0) over rows whose prefix is
// rowpre (tokens for the dense scan, groups for the proxy scan): rows
// [first, first + rows) of sequence b, key-tile chunk `chunk`.
struct SegItem {
    int b, first, rows, chunk;
};

SEG_HD SegItem seg_item(const SegTable& s, const int32_t* rowpre, int P, int item) {
    SegItem r;
    const int gi = s.item0 + item;
    r.b = seg_find(s.itm, s.nseq, gi);
    int ipb = seg_chunks(s.tok[r.b + 1] - s.tok[r.b], s.tpi);
    if (ipb < 1) ipb = 1;   // an empty sequence owns no items; never divide by 0
    const int li = gi - s.itm[r.b];
    r.chunk = li % ipb;
    r.first = rowpre[r.b] + (li / ipb) * P;
    const int end = rowpre[r.b + 1];
    r.rows = end - r.first < P ? end - r.first : P;
    return r;
}

// Causal limit of a packed dense row (token r): its own position.
SEG_HD int seg_dense_lim(const SegTable& s, int r) {
    return r - s.tok[seg_find(s.tok, s.nseq, r)];
}

// Causal limit of packed proxy row r (group j of sequence b): the last
// position of the group, min(len_b, (j + 1) g) - 1.
SEG_HD int seg_proxy_lim(const SegTable& s, int g, int r) {
    const int b = seg_find(s.grp, s.nseq, r);
    const int len = s.tok[b + 1] - s.tok[b];
    const long long e = (long long)(r - s.grp[b] + 1) * g;
    return (e < len ? (int)e : len) - 1;
}

// Packed group of packed token t.
SEG_HD int seg_group_of(const SegTable& s, int g, int t) {
    const int b = seg_find(s.tok, s.nseq, t);
    return s.grp[b] + (t - s.tok[b]) / g;
}

// Members of packed group j: tokens [first, first + n).
struct SegGroup {
    int b, first, n;
};

SEG_HD SegGroup seg_group(const SegTable& s, int g, int j) {
    SegGroup r;
    r.b = seg_find(s.grp, s.nseq, j);
    r.first = s.tok[r.b] + (j - s.grp[r.b]) * g;
    const int end = s.tok[r.b + 1];
    r.n = end - r.first < g ? end - r.first : g;
    return r;
}

// A scan work item clamped to the launch's rows [row0, row0 + nrows): rows
// [first, first + rows) (rows <= 0: nothing of it in this launch).
SEG_HD SegItem seg_scan_item(const SegTable& s, const int32_t* rowpre, int P, int row0, int nrows,
                             int item) {
    SegItem r = seg_item(s, rowpre, P, item);
    int end = r.first + r.rows;
    if (r.first < row0) r.first = row0;
    if (end > row0 + nrows) end = row0 + nrows;
    r.rows = end - r.first;
    return r;
}

// A Refine work item: member block mb (P members) of packed group grp,
// clamped to the launch's member rows [row0, row0 + nrows).
SEG_HD SegItem seg_refine_item(const SegTable& s, int g, int P, int grp, int mb, int row0,
                               int nrows) {
    const SegGroup sg = seg_group(s, g, grp);
    SegItem r;
    r.b = sg.b;
    r.chunk = 0;
    int first = sg.first + mb * P;
    int end = first + P;
    if (end > sg.first + sg.n) end = sg.first + sg.n;
    if (first < row0) first = row0;
    if (end > row0 + nrows) end = row0 + nrows;
    r.first = first;
    r.rows = end - first;
    return r;
}

// First work item (global) of the row block holding packed row r, and the
// items of that block: the item range a launch over rows [r0, r1) takes is
// [first(r0), first(r1 - 1) + count(r1 - 1)).
SEG_HD void seg_block_items(const int32_t* tok, const int32_t* rowpre, const int32_t* itm,
                            int nseq, int P, int tpi, int r, int* first, int* count) {
    const int b = seg_find(rowpre, nseq, r);
    int ch = seg_chunks(tok[b + 1] - tok[b], tpi);
    if (ch < 1) ch = 1;
    *first = itm[b] + ((r - rowpre[b]) / P) * ch;
    *count = ch;
}

}  // namespace pivot
