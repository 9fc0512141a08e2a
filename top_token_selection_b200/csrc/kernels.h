// kernels.h -- internal launch interfaces of libpivot (not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "segments.h"

namespace pivot {

// Which rows a scan launch scores and how their causal limit is found.
enum ScanKind {
    SCAN_PREFILL_DENSE = 0,   // row r = query t, keys [0, t]
    SCAN_PREFILL_PROXY = 1,   // row r = group j, keys [0, min(L,(j+1)g) - 1]
    SCAN_DECODE_DENSE = 2,    // row r = b*Gm + m, keys [0, cache_len[b] - Gm + m] of seq b
    SCAN_DECODE_PROXY = 3,    // row r = b, keys [0, cache_len[b] - 1] of seq b
    SCAN_VARLEN_DENSE = 4,    // packed token r of sequence b: keys [0, r - tok[b]] of b
    SCAN_VARLEN_PROXY = 5,    // packed group r of sequence b: keys of b up to its last member
};

struct ScanParams {
    int kind;            // ScanKind
    int dtype;           // pivot_dtype_t
    int esize;           // bytes per q/k element
    int H, D;
    int P;               // rows per row block; N = P*H <= 256
    int row0, nrows;     // global rows of this launch
    int qrow_base;       // per-row arrays (q, w, q_scale) are indexed by r - qrow_base
    int L, g;            // prefill
    int Gm, maxlen;      // decode
    const int32_t* cache_len;
    const float* w;
    const float* q_scale;
    const float* k_scale;   // indexed by key row (decode: b*maxlen + s)
    float* S;               // scores of row r at S + (r - row0)*S_stride + s
    long long S_stride;
    int tiles_per_item, items_per_block, nitems;
    // gather mode (Refine): member rows score the candidate keys of their group
    const int32_t* cand;    // group rows at cand + (grp - cand_base)*C
    int cand_base, C;
    int gsize;              // members per group (g in prefill, Gm in decode)
    int nkeys;              // key positions per sequence (L, or maxlen in decode)
    const void* kbase;      // gather mode: key rows (stored format), row stride D*esize
    const int32_t* cand_count;  // gather mode: group g's first cand_count[g - cand_base]
                                // candidates only (adaptive C), or NULL: all C
    SegTable seg;           // SCAN_VARLEN_*: the batch's sequences (rows, keys packed)
    // Sample scan: key tile t of a row is key tile t * key_tile_stride of its
    // prefix; its scores go to columns t*128 + (key in tile).  0 or 1: every tile.
    int key_tile_stride;
    // Filter mode (surv set; the selection fused into the scan): a score
    // >= its row's bound is kept as a 64-bit key (ordered score << 32 |
    // ~position).  Row r's region is surv + (r - row0) * surv_stride; chunk c
    // of it (tiles_per_item * 128 keys) holds four sub-regions of
    // tiles_per_item * 32, one per TMEM lane quarter, each filled by one
    // epilogue warp from the front, its count at
    // surv_count[((r - row0) * nchunks + c) * 4 + quarter].  In row-list mode
    // (the keep-everything rescan) every key goes to its own position in the
    // region instead, and no count is written.  No score is written to S.
    const uint32_t* bound;  // [nrows]: row r's bound (an ordered key) at bound[r - row0];
                            // keys <= 0x00800000 keep every score; NULL keeps every score
    uint64_t* surv;
    long long surv_stride;
    uint32_t* surv_count;
    int nchunks;
    int lim_shift;          // filter mode: positions kept are <= lim(r) - lim_shift
    // Row-list mode (row_list set): the launch's rows are row_list[0, *row_count),
    // one row a block (P = 1); prefill kinds only.
    const int32_t* row_list;
    const uint32_t* row_count;
};

int scan_smem_bytes(int row_bytes);
cudaError_t launch_scan_umma(const CUtensorMap& tk, const CUtensorMap& tq, const ScanParams& p,
                             int grid, cudaStream_t stream);
cudaError_t launch_scan_simt(const void* q, const void* k, const ScanParams& p,
                             cudaStream_t stream);

// Row selection: for each row, the top-K entries by (score desc, position
// asc) among the row's valid entries, written in ascending position order
// (with `split`, the top `split` first, then the rest) with -1 / -inf padding.
enum SelectKind {
    SEL_PREFIX = 0,      // row r: entries 0..lim(r) of S, position = entry index
    SEL_CANDIDATES = 1,  // row r: C entries, position = cand[grp(r)][i], valid iff 0 <= pos <= lim(r)
};

struct SelectParams {
    int kind;             // SelectKind
    int scan_kind;        // ScanKind giving lim(r) (SEL_PREFIX and SEL_CANDIDATES)
    int row0, nrows;
    int L, g, Gm, maxlen;
    const int32_t* cache_len;
    const float* S;       // row r at S + (r - row0)*S_stride
    long long S_stride;
    const int32_t* cand;  // SEL_CANDIDATES: group rows at cand + (grp - cand_base)*C
    const int32_t* cand_count;  // SEL_CANDIDATES: only the group's first cand_count[grp -
                                // cand_base] entries (adaptive C), or NULL: all C
    int cand_base, C;
    int K;
    int32_t* out_idx;     // row r at out_idx + (r - out_base)*K
    float* out_score;     // or NULL
    int out_base;
    int tail_cap;         // capacity of the boundary buffer (entries)
    int split;            // > 0: list the top `split` first, then the rest (each by position)
    int npos;             // positions are < npos (bitmap size)
    int fast_cap;         // set by launch_select: kept-entry capacity of the fast path
    int bitmap_words;     // set by launch_select
    int s_per_group;          // SEL_CANDIDATES: S rows are per group (grp - cand_base), not per row
    int lim_shift;            // positions considered are <= lim(r) - lim_shift (a window kept out)
    int out_stride;           // output row stride in entries (0: K)
    const float* key_scale;   // SEL_CANDIDATES: if set, entry i's score is S * key_scale[kb + pos]
                              // (kb = grp * maxlen for decode rows, else 0)
    const uint32_t* thresh;   // SEL_PREFIX: row r's lower bound at thresh[r - row0]
                              // (launch_row_threshold), or NULL: sampled in the select
    SegTable seg;             // scan_kind SCAN_VARLEN_*: the batch's sequences; candidate
                              // rows of packed token r: group seg_group_of(r), key scales
                              // from the sequence's first token
    int rank_order;           // 1: rows in rank order (score descending, then position
                              // ascending; `split` is then moot); 0: ascending positions
    // SEL_PREFIX rows whose entries are 64-bit keys (ordered score << 32 |
    // ~position) instead of scores: row r's n = lim + 1 keys at
    // keys + (r - row0) * S_stride (the fused scan's regions, every key kept)
    const uint64_t* keys;
    // Row list: block b selects row row_list[b] when b < *row_count (and
    // does nothing otherwise)
    const int32_t* row_list;
    const uint32_t* row_count;
};

// The selection fused into the scan (prefill dense and proxy rows): a sample
// scan gives each row a bound, the filter-mode scan keeps the scores at or
// above it, and one warp per row selects the top K among them.
struct FusedSelectParams {
    int scan_kind;            // SCAN_PREFILL_* or SCAN_DECODE_*
    int row0, nrows, L, g;
    int Gm, maxlen;           // decode rows: limits from the device cache lengths
    const int32_t* cache_len;
    int lim_shift;            // positions considered are <= lim(r) - lim_shift
    int K, split, rank_order;
    // samples: row r's sample scores at samp + (r - row0) * samp_stride,
    // column j = key position (j / 128) * kts * 128 + j % 128
    const float* samp;
    long long samp_stride;
    int kts;
    float sigmas;             // margin of the bound, in standard deviations of the count
    uint32_t* bound;          // [nrows] out: row r's bound (an ordered key; 1 keeps all)
    int cap;                  // survivors a row may have for the warp select
    // survivors: row r's segment s = chunk * nsub + sub at surv + (r - row0) *
    // surv_stride + chunk * chunk_keys + sub * sub_keys, with
    // surv_count[(r - row0) * nchunks * nsub + s] of them
    const uint64_t* surv;
    long long surv_stride;
    const uint32_t* surv_count;
    int nchunks, chunk_keys, nsub, sub_keys;
    int32_t* out_idx;         // row r at out_idx + (r - out_base) * (out_stride or K)
    float* out_score;         // or NULL
    int out_base, out_stride;
    int32_t* miss_list;       // rows whose survivors fell outside [min(K, n), cap]
    uint32_t* miss_count;     // zeroed by the bound kernel
};
// Bound of every row (one warp per row) and a zeroed miss count.
cudaError_t launch_sample_bound(const FusedSelectParams& p, cudaStream_t stream);
// Top K of every row's survivors (one warp per row); rows that miss go to the
// list for the fallback (a keep-everything rescan and launch_select on keys).
cudaError_t launch_fused_finish(const FusedSelectParams& p, cudaStream_t stream);
// Survivor capacity a row may have for K (entries), and the shared memory
// that needs per warp.
int fused_cap(int K);

cudaError_t launch_select(const SelectParams& p, cudaStream_t stream);
// SEL_PREFIX rows: per-row lower bound for the select's fast path, written
// to thresh[r - row0] (one warp per row; p.thresh is ignored).
cudaError_t launch_row_threshold(const SelectParams& p, uint32_t* thresh, cudaStream_t stream);

struct ReduceParams {
    int dtype, esize, H, D;
    int nmembers_total;    // rows available from member 0 of the first group
    int g;                 // members per group
    int ngroups;
    const void* q;         // member rows, q + m*H*D*esize for member m (relative)
    const float* q_scale;
    const float* w;
    void* pq;
    float* pq_scale;
    float* pw;
    long long group_stride_members;  // members between consecutive groups
    SegTable seg;          // seg.tok set: packed groups of a ragged batch (seg_group)
};
cudaError_t launch_proxy_reduce(const ReduceParams& p, cudaStream_t stream);

// lim_shift: members keep candidates <= t - lim_shift; out_stride 0: topk.
cudaError_t launch_reuse(int t_begin, int t_end, int g, const int32_t* cand, int C, int topk,
                         int32_t* idx, cudaStream_t stream, int lim_shift = 0,
                         int out_stride = 0);
// Each index row (ascending, -1 padded, k entries) united with the window
// [t - window + 1, t] (t = positions[r], or t_begin + r): out [rows, k + window].
// idx rows at stride in_stride (0: k); out may be idx with in_stride = k + window.
cudaError_t launch_window_union(const int32_t* idx, int rows, int k, int t_begin,
                                const int32_t* positions, int window, int32_t* out,
                                cudaStream_t stream, int in_stride = 0);
// Adaptive C: group j keeps its first count[j] candidates -- those whose
// proxy score is at least rho times its k-th (the rows rank-ordered, scores
// descending), clamped to [min(topk, valid), C].
cudaError_t launch_adaptive_count(const float* cand_score, int G, int C, int topk, float rho,
                                  int32_t* count, cudaStream_t stream);
// Reuse over a ragged batch: packed token t takes the first topk entries of
// its group's candidate row (seg_group_of) that are <= its position.
cudaError_t launch_reuse_varlen(const SegTable& seg, int T, int g, const int32_t* cand, int C,
                                int topk, int32_t* idx, cudaStream_t stream);
// Copy n (<= 960) host integers, carried as launch parameters, to dst: a
// host-to-device copy that stream capture records like any launch.
cudaError_t launch_write_ints(int32_t* dst, const int32_t* host, int n, cudaStream_t stream);
cudaError_t launch_decode_reuse(int B, int Gm, int maxlen, const int32_t* cache_len,
                                const int32_t* cand, int C, int topk, int32_t* idx,
                                cudaStream_t stream);

// Refine scores: member r of group grp(r) against C candidate keys.
struct RefineParams {
    int dtype, esize, H, D;
    int kind;              // ScanKind for the member rows (PREFILL_DENSE or DECODE_DENSE)
    int row0, nrows;       // member rows
    int qrow_base;
    int L, g, Gm, maxlen;
    const int32_t* cache_len;
    const void* q;
    const float* q_scale;
    const float* w;
    const void* k;
    const float* k_scale;
    const int32_t* cand;   // group rows at cand + (grp - cand_base)*C
    int cand_base, C;
    float* S;              // row r at S + (r - row0)*C
};
cudaError_t launch_refine_simt(const RefineParams& p, cudaStream_t stream);
// Refine scores on the tensor cores: candidate keys gathered from p.kbase
// with cp.async, member queries from tmap_q.  p.kind is SCAN_PREFILL_DENSE
// or SCAN_DECODE_DENSE (member rows); S rows have C entries.
cudaError_t launch_refine_umma(const CUtensorMap& tmap_q, const ScanParams& p, int grid,
                               cudaStream_t stream);

cudaError_t launch_wait_selftest(cudaStream_t stream);

}  // namespace pivot
