// api.cu -- the libpivot C ABI: argument checks, workspace carving, TMA
// descriptors and kernel launches.  See include/pivot.h for the contract.
#include <climits>
#include <cstdio>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "profile.h"

#include <nvtx3/nvToolsExt.h>

namespace pivot {

__device__ uint32_t g_error_word = 0;
__device__ uint64_t g_wait_limit_ns = 4000000000ull;

namespace {

constexpr size_t WS_ALIGN = 256;
constexpr size_t SCORE_BUF_DEFAULT = size_t(4) << 30;   // preferred score buffer, 4 GiB
size_t g_score_buf_cap = SCORE_BUF_DEFAULT;             // pivot_set_score_buffer_cap
constexpr int MAX_K = 8192;   // the select's exact path holds 2 pow2(K) keys in shared memory
// Fused selection: the sample scan scores every FUSED_KTS-th key tile; a scan
// work item covers FUSED_TILES key tiles (its chunk of 4096 keys).
constexpr int FUSED_KTS = 32;
constexpr int FUSED_TILES = 32;
// A work item of the plain prefill scan (every score written) covers 64 key
// tiles: each item pays a fixed start (the block's weights, limits and
// scales, two barriers of the epilogue warps), and at L = 128K the dense
// scan took 1.7 % less time with 64 tiles an item than with 32 (interleaved
// runs: 101.5-102.0 against 102.5-104.4 ms), 7 % more with 16.
constexpr int PLAIN_TILES = 64;
constexpr int TAIL_CAP = 4096;
constexpr int MAX_SMS = 1024;

int esize_of(int dtype) { return dtype == PIVOT_F32 ? 4 : (dtype == PIVOT_BF16 ? 2 : 1); }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (cache[dev] == 0) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cache[dev] = n > 0 ? (n < MAX_SMS ? n : MAX_SMS) : 148;
    }
    return cache[dev];
}

// ------------------------------------------------------------------ TMA maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D map over rows x cols elements (row stride = cols * esize), box of
// 128 bytes x box_rows, 128-byte swizzle, zero fill out of bounds.
bool make_tmap(CUtensorMap* map, int dtype, const void* base, long long rows, int cols,
               int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const int es = esize_of(dtype);
    CUtensorMapDataType dt = dtype == PIVOT_F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                             : dtype == PIVOT_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                   : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t gstride[1] = {(cuuint64_t)cols * es};
    cuuint32_t box[2] = {(cuuint32_t)(128 / es), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dt, 2, const_cast<void*>(base), gdim, gstride, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------- validation
bool dtype_ok(int dt) { return dt == PIVOT_F32 || dt == PIVOT_BF16 || dt == PIVOT_E4M3; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Tensor-core tiling: FP8 and bf16 codes (the tensor cores have no fp32
// kind, and their tf32 kind keeps 10 mantissa bits, so PIVOT_F32 is scored
// on the CUDA cores in full fp32); N = P*H <= 256 with H in {4..64}; key rows
// of 128 or 256 bytes (two 128-byte swizzle atoms).
bool umma_shape_ok(int H, int D, int dtype) {
    if (dtype == PIVOT_F32) return false;
    const int rb = D * esize_of(dtype);
    return (H == 4 || H == 8 || H == 16 || H == 32 || H == 64) && (rb == 128 || rb == 256);
}

bool simt_shape_ok(int H, int D) {
    const size_t smem = ((size_t)D * 128 + (size_t)H * D + H) * 4;
    return smem <= 200 * 1024;
}

bool order_ok(int order) { return order == PIVOT_ORDER_POSITION || order == PIVOT_ORDER_RANK; }

// The output order of the entry point running on this host thread: set for
// the duration of a call from its input struct, read by every selection
// launch the call makes.
thread_local int t_rank_order = 0;
struct OrderScope {
    int prev;
    explicit OrderScope(int order) : prev(t_rank_order) {
        t_rank_order = order == PIVOT_ORDER_RANK ? 1 : 0;
    }
    ~OrderScope() { t_rank_order = prev; }
};

pivot_status_t check_seq(const pivot_seq_t* s, int* t0, int* t1) {
    if (!s || !dtype_ok(s->dtype) || !order_ok(s->order)) return PIVOT_ERR_INVALID_ARG;
    if (s->L < 1 || s->H < 1 || s->D < 1) return PIVOT_ERR_INVALID_ARG;
    if (!s->q || !s->w || !s->k) return PIVOT_ERR_INVALID_ARG;
    const bool fp8 = s->dtype == PIVOT_E4M3;
    if (fp8 != (s->q_scale != nullptr) || fp8 != (s->k_scale != nullptr))
        return PIVOT_ERR_INVALID_ARG;
    *t0 = s->t_begin;
    *t1 = s->t_end == 0 ? s->L : s->t_end;
    if (*t0 < 0 || *t1 > s->L || *t0 >= *t1) return PIVOT_ERR_INVALID_ARG;
    if (!aligned16(s->q) || !aligned16(s->k)) return PIVOT_ERR_INVALID_ARG;
    if ((s->D * esize_of(s->dtype)) % 16) return PIVOT_ERR_UNSUPPORTED;
    if (!umma_shape_ok(s->H, s->D, s->dtype) && !simt_shape_ok(s->H, s->D))
        return PIVOT_ERR_UNSUPPORTED;
    return PIVOT_OK;
}

pivot_status_t check_group_range(const pivot_seq_t* s, int g, int t0, int t1) {
    if (g < 1) return PIVOT_ERR_INVALID_ARG;
    if (t0 % g) return PIVOT_ERR_INVALID_ARG;
    if (t1 != s->L && t1 % g) return PIVOT_ERR_INVALID_ARG;
    return PIVOT_OK;
}

thread_local char g_last_detail[256] = "no CUDA error recorded";

pivot_status_t from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return PIVOT_OK;
    snprintf(g_last_detail, sizeof(g_last_detail), "%s: %s", cudaGetErrorName(e),
             cudaGetErrorString(e));
    return PIVOT_ERR_CUDA;
}

long long score_stride(int nkeys) { return (long long)align_up((size_t)nkeys, 32); }

// Rows per chunk for `total` rows of `rowbytes` each in `bytes` of
// workspace: all of them if they fit; else, when at least one unit fits, a
// multiple of `unit` that splits the rows into as few chunks as fit, of
// about equal size (a last chunk of a few rows would cost a scan pass and a
// selection wave of its own: 64 of 131072 rows, 8 of 16384 groups, at the
// default workspace); else as many as fit (0 if not even one row fits).
long long chunk_rows(size_t bytes, size_t rowbytes, long long total, int unit) {
    const long long fit = (long long)(bytes / rowbytes);
    if (fit >= total) return total;
    if (fit < unit) return fit;
    const long long most = fit / unit * unit;
    const long long n = (total + most - 1) / most;
    return ((total + n - 1) / n + unit - 1) / unit * unit;   // <= most
}

// Causal (row, key) pairs of rows [r0, r1): the algorithmic work of a scan.
// Decode rows depend on device-side cache lengths: reported as 0.
double scan_pairs(int kind, int r0, int r1, int L, int g) {
    double s = 0.0;
    if (kind == SCAN_PREFILL_DENSE) {
        s = 0.5 * ((double)r1 * (r1 + 1) - (double)r0 * (r0 + 1));
    } else if (kind == SCAN_PREFILL_PROXY) {
        for (int j = r0; j < r1; ++j) s += (double)((j + 1) * (long long)g < L ? (j + 1) * g : L);
    }
    return s;
}

// (member, candidate) pairs of prefill Refine rows [r0, r1): sum of min(C, t+1).
double refine_pairs(int r0, int r1, int C) {
    double s = 0.0;
    const int knee = C - 1;   // rows t >= knee see C candidates
    const int a_end = r1 < knee ? r1 : knee;
    if (r0 < a_end) s += 0.5 * ((double)a_end * (a_end + 1) - (double)r0 * (r0 + 1));
    const int b0 = r0 > knee ? r0 : knee;
    if (b0 < r1) s += (double)(r1 - b0) * C;
    return s;
}

// ------------------------------------------------------------------ scans
// Rows [r0, r1) of kind `kind` into S (row r at S + (r - r0)*stride).
// Modes of a tensor-core scan beyond plain scores (see ScanParams).
struct ScanExtra {
    int key_tile_stride = 0;            // sample scan
    const uint32_t* bound = nullptr;    // filter mode
    uint64_t* surv = nullptr;
    long long surv_stride = 0;
    uint32_t* surv_count = nullptr;
    int nchunks = 0;
    int lim_shift = 0;
    const int32_t* row_list = nullptr;  // row-list mode (P = 1)
    const uint32_t* row_count = nullptr;
    double work = -1.0;                 // the launch's algorithmic pairs (profiling)
};

pivot_status_t run_scan(int kind, int dtype, int H, int D, const void* qbase, long long q_rows,
                        int qrow_base, const float* w, const float* q_scale, const void* kbase,
                        long long k_rows, const float* k_scale, int L, int g, int Gm, int maxlen,
                        const int32_t* cache_len, int P, int r0, int r1, int maxlim_total,
                        float* S, long long stride, cudaStream_t st,
                        const ScanExtra* x = nullptr) {
    ScanParams p{};
    if (x) {
        p.key_tile_stride = x->key_tile_stride;
        p.bound = x->bound;
        p.surv = x->surv;
        p.surv_stride = x->surv_stride;
        p.surv_count = x->surv_count;
        p.nchunks = x->nchunks;
        p.lim_shift = x->lim_shift;
        p.row_list = x->row_list;
        p.row_count = x->row_count;
        if (x->row_list) P = 1;
    }
    const double work = (x && x->work >= 0.0) ? x->work : scan_pairs(kind, r0, r1, L, g);
    p.kind = kind;
    p.dtype = dtype;
    p.esize = esize_of(dtype);
    p.H = H;
    p.D = D;
    p.P = P;
    p.row0 = r0;
    p.nrows = r1 - r0;
    p.qrow_base = qrow_base;
    p.L = L;
    p.g = g;
    p.Gm = Gm;
    p.maxlen = maxlen;
    p.cache_len = cache_len;
    p.w = w;
    p.q_scale = q_scale;
    p.k_scale = k_scale;
    p.S = S;
    p.S_stride = stride;
    const int nblocks = ceil_div(p.nrows, P);
    const int kts = p.key_tile_stride > 1 ? p.key_tile_stride : 1;
    const int nt = ceil_div(ceil_div(maxlim_total + 1, 128), kts);
    const int N = P * H;
    if (umma_shape_ok(H, D, dtype) && N >= 16 && N <= 256 && N % 16 == 0) {
        const bool decode = kind == SCAN_DECODE_DENSE || kind == SCAN_DECODE_PROXY;
        const bool fused_mode = x && (x->surv || x->key_tile_stride > 1 || x->row_list);
        p.tiles_per_item = decode ? 8 : (fused_mode ? FUSED_TILES : PLAIN_TILES);
        p.items_per_block = ceil_div(nt, p.tiles_per_item);
        p.nitems = nblocks * p.items_per_block;
        CUtensorMap tk, tq;
        if (!make_tmap(&tk, dtype, kbase, k_rows, D, 128)) return PIVOT_ERR_CUDA;
        if (!make_tmap(&tq, dtype, qbase, q_rows * H, D, P * H)) return PIVOT_ERR_CUDA;
        const int grid = p.nitems < num_sms() ? p.nitems : num_sms();
        return from_cuda(profiled(PK_SCAN, work, st,
                                  [&] { return launch_scan_umma(tk, tq, p, grid, st); }));
    }
    if (x && (x->surv || x->key_tile_stride > 1 || x->row_list)) return PIVOT_ERR_UNSUPPORTED;
    p.tiles_per_item = 1;
    p.items_per_block = nt;
    p.nitems = nblocks * nt;
    return from_cuda(profiled(PK_SCAN, scan_pairs(kind, r0, r1, L, g), st,
                              [&] { return launch_scan_simt(qbase, kbase, p, st); }));
}

// Rows of a tensor-core block (scan and Refine): N = rows * H = 256 columns
// (one row per epilogue warp at H = 64: four warps per TMEM lane quarter).
int umma_rows(int H) { return 256 / H; }

int rows_per_block(int H, int D, int dtype) {
    return umma_shape_ok(H, D, dtype) ? umma_rows(H) : 8;
}

// Decode dense rows: a row block must not straddle two sequences (its keys
// are one sequence's), so its row count divides Gm; on the tensor cores it is
// also at most umma_rows(H) (the epilogue gives each of its four warp groups
// at most 64 / H rows at H >= 32).
int decode_dense_rows(int Gm, int H, int D, int dtype) {
    if (!umma_shape_ok(H, D, dtype)) return Gm;
    const int pmax = umma_rows(H);
    int P = 1;
    for (int d = 1; d <= Gm && d <= pmax; ++d)
        if (Gm % d == 0) P = d;
    return P;
}

pivot_status_t run_select_prefix(int scan_kind, int r0, int r1, int L, int g, int Gm, int maxlen,
                                 const int32_t* cache_len, const float* S, long long stride,
                                 int K, int split, int npos, int32_t* out, float* out_score,
                                 int out_base, cudaStream_t st, uint32_t* thresh = nullptr,
                                 int lim_shift = 0, int out_stride = 0,
                                 const SegTable* seg = nullptr, double work = -1.0) {
    SelectParams sp{};
    if (seg) sp.seg = *seg;
    sp.lim_shift = lim_shift;
    sp.out_stride = out_stride;
    sp.split = split;
    sp.npos = npos;
    sp.kind = SEL_PREFIX;
    sp.scan_kind = scan_kind;
    sp.row0 = r0;
    sp.nrows = r1 - r0;
    sp.L = L;
    sp.g = g;
    sp.Gm = Gm;
    sp.maxlen = maxlen;
    sp.cache_len = cache_len;
    sp.S = S;
    sp.S_stride = stride;
    sp.K = K;
    sp.out_idx = out;
    sp.out_score = out_score;
    sp.out_base = out_base;
    sp.tail_cap = TAIL_CAP;
    sp.rank_order = t_rank_order;
    sp.thresh = thresh;
    if (thresh) {   // a launch of its own (no work of its own: the select's bytes count once)
        const pivot_status_t t = from_cuda(
            profiled(PK_SELECT, 0.0, st, [&] { return launch_row_threshold(sp, thresh, st); }));
        if (t != PIVOT_OK) return t;
    }
    return from_cuda(profiled(PK_SELECT, work >= 0.0 ? work : scan_pairs(scan_kind, r0, r1, L, g),
                              st, [&] { return launch_select(sp, st); }));
}

// Refine rows: S holds the scores without the key scale, which the
// selection multiplies in (key_scale, NULL for unscaled formats).
pivot_status_t run_select_cand(int scan_kind, int r0, int r1, int L, int g, int Gm, int maxlen,
                               const int32_t* cache_len, const float* S, const int32_t* cand,
                               int cand_base, int C, int K, int npos, int32_t* out,
                               float* out_score, int out_base, cudaStream_t st,
                               const float* key_scale, int lim_shift = 0, int out_stride = 0,
                               const SegTable* seg = nullptr, const int32_t* cand_count = nullptr) {
    SelectParams sp{};
    sp.cand_count = cand_count;
    if (seg) sp.seg = *seg;
    sp.npos = npos;
    sp.kind = SEL_CANDIDATES;
    sp.scan_kind = scan_kind;
    sp.row0 = r0;
    sp.nrows = r1 - r0;
    sp.L = L;
    sp.g = g;
    sp.Gm = Gm;
    sp.maxlen = maxlen;
    sp.cache_len = cache_len;
    sp.S = S;
    sp.S_stride = C;
    sp.cand = cand;
    sp.cand_base = cand_base;
    sp.C = C;
    sp.K = K;
    sp.key_scale = key_scale;
    sp.lim_shift = lim_shift;
    sp.out_stride = out_stride;
    sp.out_idx = out;
    sp.out_score = out_score;
    sp.out_base = out_base;
    sp.tail_cap = TAIL_CAP;
    sp.rank_order = t_rank_order;
    return from_cuda(profiled(PK_SELECT, (double)(r1 - r0) * C, st,
                              [&] { return launch_select(sp, st); }));
}

pivot_status_t run_refine_scores(int kind, int dtype, int H, int D, const void* q,
                                 long long q_rows, int qrow_base, const float* q_scale,
                                 const float* w, const void* k, long long k_rows,
                                 const float* k_scale, int L, int g, int Gm, int maxlen,
                                 const int32_t* cache_len, const int32_t* cand, int cand_base,
                                 int C, int r0, int r1, float* S, cudaStream_t st,
                                 const int32_t* cand_count = nullptr) {
    const double work = kind == SCAN_PREFILL_DENSE ? refine_pairs(r0, r1, C) : 0.0;
    const int gsize = kind == SCAN_DECODE_DENSE ? Gm : g;
    int P = umma_shape_ok(H, D, dtype) ? umma_rows(H) : 0;
    if (P > gsize) P = gsize;
    const int N = P * H;
    if (P > 0 && N >= 16 && N <= 256 && N % 16 == 0) {
        // tensor cores: candidate keys gathered with TMA
        ScanParams p{};
        p.kind = kind;
        p.dtype = dtype;
        p.esize = esize_of(dtype);
        p.H = H;
        p.D = D;
        p.P = P;
        p.row0 = r0;
        p.nrows = r1 - r0;
        p.qrow_base = qrow_base;
        p.L = L;
        p.g = g;
        p.Gm = Gm;
        p.maxlen = maxlen;
        p.cache_len = cache_len;
        p.w = w;
        p.q_scale = q_scale;
        p.k_scale = k_scale;
        p.S = S;
        p.S_stride = C;
        p.cand = cand;
        p.cand_base = cand_base;
        p.C = C;
        p.gsize = gsize;
        p.nkeys = kind == SCAN_DECODE_DENSE ? maxlen : L;
        p.tiles_per_item = ceil_div(C, 128);
        p.items_per_block = ceil_div(gsize, P);
        const int ngroups = (r1 - 1) / gsize - cand_base + 1;
        p.nitems = ngroups * p.items_per_block;
        p.kbase = k;
        p.cand_count = cand_count;
        (void)k_rows;
        CUtensorMap tq;
        if (!make_tmap(&tq, dtype, q, q_rows * H, D, N)) return PIVOT_ERR_CUDA;
        const int grid = p.nitems < num_sms() ? p.nitems : num_sms();
        return from_cuda(profiled(PK_REFINE, work, st,
                                  [&] { return launch_refine_umma(tq, p, grid, st); }));
    }
    RefineParams rp{};
    rp.dtype = dtype;
    rp.esize = esize_of(dtype);
    rp.H = H;
    rp.D = D;
    rp.kind = kind;
    rp.row0 = r0;
    rp.nrows = r1 - r0;
    rp.qrow_base = qrow_base;
    rp.L = L;
    rp.g = g;
    rp.Gm = Gm;
    rp.maxlen = maxlen;
    rp.cache_len = cache_len;
    rp.q = q;
    rp.q_scale = q_scale;
    rp.w = w;
    rp.k = k;
    rp.k_scale = k_scale;
    rp.cand = cand;
    rp.cand_base = cand_base;
    rp.C = C;
    rp.S = S;
    // (CUDA-core shapes score all C; the selection drops what the counts exclude)
    return from_cuda(profiled(PK_REFINE, work, st, [&] { return launch_refine_simt(rp, st); }));
}

// Carve `bytes` (256-aligned) from the workspace cursor.
struct Carver {
    uint8_t* base;
    size_t cap, off = 0;
    bool ok = true;
    void* take(size_t bytes) {
        off = align_up(off, WS_ALIGN);
        if (off + bytes > cap) { ok = false; return nullptr; }
        void* p = base + off;
        off += bytes;
        return p;
    }
};

// A prefill score row in the workspace, plus the row's select bound (4 bytes
// after all score rows of the chunk).
size_t dense_rowbytes(int L) { return (size_t)score_stride(L) * 4 + 4; }

// ------------------------------------------------------------ fused selection
// Prefix rows (dense queries, proxies) whose top-K is taken inside the scan:
// a sample scan over every FUSED_KTS-th key tile, a bound per row, the
// filter-mode scan appending the scores at or above it, one warp per row
// selecting among them, and -- for rows whose survivors miss the warp
// select's range -- a keep-everything rescan of just those rows and the
// block select on their keys.  The scores themselves never reach memory.
// Off by default (pivot_set_fused_selection): the separate selection is
// faster where the scan's epilogue is the bound.
bool g_fused_on = false;
float g_fused_sigmas = 4.5f;

bool fused_ok(int H, int D, int dtype, int K) {
    return g_fused_on && umma_shape_ok(H, D, dtype) && H >= 32 && K <= MAX_K;
}
// Key tiles of one work item of the fused selection's scans (their survivor
// regions are laid out per item): prefill FUSED_TILES, decode (few, long
// rows) 8.
int scan_tiles_per_item(int kind) {
    return (kind == SCAN_DECODE_DENSE || kind == SCAN_DECODE_PROXY) ? 8 : FUSED_TILES;
}
int fused_tiles(int L) { return ceil_div(L, 128); }
long long fused_samp_stride(int L) { return (long long)ceil_div(fused_tiles(L), FUSED_KTS) * 128; }
int fused_nchunks(int L, int tpi = FUSED_TILES) { return ceil_div(fused_tiles(L), tpi); }
long long fused_surv_stride(int L, int tpi = FUSED_TILES) {
    return (long long)fused_nchunks(L, tpi) * tpi * 128;
}
// per row: samples, survivor regions, chunk counts, the bound, a miss slot
size_t fused_rowbytes(int L, int tpi = FUSED_TILES) {
    return (size_t)fused_samp_stride(L) * 4 + (size_t)fused_surv_stride(L, tpi) * 8 +
           (size_t)fused_nchunks(L, tpi) * 4 * 4 + 4 + 4;
}
constexpr size_t FUSED_FIXED = 8 * WS_ALIGN;   // alignment of the six arrays, the miss count

struct FusedWs {
    float* samp;
    uint64_t* surv;
    uint32_t* count;
    uint32_t* bound;
    int32_t* miss;
    uint32_t* nmiss;
};

bool fused_carve(void* ws, size_t bytes, long long rows, int L, FusedWs* w,
                 int tpi = FUSED_TILES) {
    Carver c{static_cast<uint8_t*>(ws), bytes};
    w->samp = static_cast<float*>(c.take((size_t)rows * fused_samp_stride(L) * 4));
    w->surv = static_cast<uint64_t*>(c.take((size_t)rows * fused_surv_stride(L, tpi) * 8));
    w->count = static_cast<uint32_t*>(c.take((size_t)rows * fused_nchunks(L, tpi) * 4 * 4));
    w->bound = static_cast<uint32_t*>(c.take((size_t)rows * 4));
    w->miss = static_cast<int32_t*>(c.take((size_t)rows * 4));
    w->nmiss = static_cast<uint32_t*>(c.take(4));
    return c.ok;
}

// Rows a launch of the fused path takes from `bytes` of workspace.
long long fused_chunk_rows(size_t bytes, int L, long long total, int P) {
    return chunk_rows(bytes > FUSED_FIXED ? bytes - FUSED_FIXED : 0, fused_rowbytes(L), total, P);
}

// The keys a fused selection scans: one prefill sequence, or the caches of
// a decode batch.
struct KeySrc {
    int dtype, H, D;
    const void* k;
    long long k_rows;
    const float* k_scale;
    int L;                 // prefill length, or the cache capacity (maxlen) in decode
    int Gm, maxlen;
    const int32_t* cache_len;
};

KeySrc key_src(const pivot_seq_t* s) {
    return KeySrc{s->dtype, s->H, s->D, s->k, s->L, s->k_scale, s->L, 1, 0, nullptr};
}

// The top K of rows [r0, r1) of `kind` (prefill: rows of queries or
// proxies; decode: members or proxies of the batch), written like
// run_select_prefix writes them.
pivot_status_t run_prefix_fused(int kind, const KeySrc& ks, const void* qbase,
                                long long q_rows, int qrow_base, const float* w,
                                const float* q_scale, int g, int P, int r0, int r1, int maxlim,
                                int K, int split, int32_t* out, float* out_score, int out_base,
                                int lim_shift, int out_stride, const FusedWs& fw,
                                cudaStream_t s) {
    const int L = ks.L;
    const int tpi = scan_tiles_per_item(kind);
    const bool dec = kind == SCAN_DECODE_DENSE || kind == SCAN_DECODE_PROXY;
    const double pairs = dec ? 0.0 : scan_pairs(kind, r0, r1, L, g);
    // 1. samples
    ScanExtra xs;
    xs.key_tile_stride = FUSED_KTS;
    xs.work = pairs / FUSED_KTS;
    nvtxRangePushA("fused: sample scan");
    pivot_status_t st =
        run_scan(kind, ks.dtype, ks.H, ks.D, qbase, q_rows, qrow_base, w, q_scale, ks.k,
                 ks.k_rows, ks.k_scale, dec ? 0 : L, g, ks.Gm, ks.maxlen, ks.cache_len, P, r0,
                 r1, maxlim, fw.samp, fused_samp_stride(L), s, &xs);
    nvtxRangePop();
    if (st != PIVOT_OK) return st;
    // 2. bounds
    FusedSelectParams fp{};
    fp.scan_kind = kind;
    fp.row0 = r0;
    fp.nrows = r1 - r0;
    fp.L = dec ? 0 : L;
    fp.g = g;
    fp.Gm = ks.Gm;
    fp.maxlen = ks.maxlen;
    fp.cache_len = ks.cache_len;
    fp.lim_shift = lim_shift;
    fp.K = K;
    fp.split = split;
    fp.rank_order = t_rank_order;
    fp.samp = fw.samp;
    fp.samp_stride = fused_samp_stride(L);
    fp.kts = FUSED_KTS;
    fp.sigmas = g_fused_sigmas;
    fp.bound = fw.bound;
    fp.cap = fused_cap(K);
    fp.surv = fw.surv;
    fp.surv_stride = fused_surv_stride(L, tpi);
    fp.surv_count = fw.count;
    fp.nchunks = fused_nchunks(L, tpi);
    fp.chunk_keys = tpi * 128;
    fp.nsub = 4;                 // one sub-region per TMEM lane quarter
    fp.sub_keys = tpi * 32;
    fp.out_idx = out;
    fp.out_score = out_score;
    fp.out_base = out_base;
    fp.out_stride = out_stride;
    fp.miss_list = fw.miss;
    fp.miss_count = fw.nmiss;
    nvtxRangePushA("fused: bounds");
    st = from_cuda(profiled(PK_SELECT, 0.0, s, [&] { return launch_sample_bound(fp, s); }));
    nvtxRangePop();
    if (st != PIVOT_OK) return st;
    // 3. the scan, keeping the scores at or above each row's bound
    ScanExtra xf;
    xf.bound = fw.bound;
    xf.surv = fw.surv;
    xf.surv_stride = fused_surv_stride(L, tpi);
    xf.surv_count = fw.count;
    xf.nchunks = fused_nchunks(L, tpi);
    xf.lim_shift = lim_shift;
    xf.work = pairs;
    nvtxRangePushA("fused: filter scan");
    st = run_scan(kind, ks.dtype, ks.H, ks.D, qbase, q_rows, qrow_base, w, q_scale, ks.k,
                  ks.k_rows, ks.k_scale, dec ? 0 : L, g, ks.Gm, ks.maxlen, ks.cache_len, P, r0, r1,
                  maxlim, nullptr, 0, s, &xf);
    nvtxRangePop();
    if (st != PIVOT_OK) return st;
    // 4. the top K of every row's survivors
    nvtxRangePushA("fused: warp select");
    st = from_cuda(profiled(PK_SELECT, 0.0, s, [&] { return launch_fused_finish(fp, s); }));
    nvtxRangePop();
    if (st != PIVOT_OK) return st;
    // 5. rows that missed: rescan keeping every score (one row a block) ...
    ScanExtra xr = xf;
    xr.bound = nullptr;
    xr.row_list = fw.miss;
    xr.row_count = fw.nmiss;
    xr.work = 0.0;
    nvtxRangePushA("fused: rescan of missed rows");
    st = run_scan(kind, ks.dtype, ks.H, ks.D, qbase, q_rows, qrow_base, w, q_scale, ks.k,
                  ks.k_rows, ks.k_scale, dec ? 0 : L, g, ks.Gm, ks.maxlen, ks.cache_len, 1, r0, r1,
                  maxlim, nullptr, 0, s, &xr);
    if (st != PIVOT_OK) {
        nvtxRangePop();
        return st;
    }
    // 6. ... and select on their keys
    SelectParams sp{};
    sp.kind = SEL_PREFIX;
    sp.scan_kind = kind;
    sp.row0 = r0;
    sp.nrows = r1 - r0;
    sp.L = dec ? 0 : L;
    sp.g = g;
    sp.Gm = dec ? ks.Gm : 1;
    sp.maxlen = ks.maxlen;
    sp.cache_len = ks.cache_len;
    sp.keys = fw.surv;
    sp.S_stride = fused_surv_stride(L, tpi);
    sp.K = K;
    sp.split = split;
    sp.npos = L;
    sp.out_idx = out;
    sp.out_score = out_score;
    sp.out_base = out_base;
    sp.out_stride = out_stride;
    sp.lim_shift = lim_shift;
    sp.tail_cap = TAIL_CAP;
    sp.rank_order = t_rank_order;
    sp.row_list = fw.miss;
    sp.row_count = fw.nmiss;
    st = from_cuda(profiled(PK_SELECT, 0.0, s, [&] { return launch_select(sp, s); }));
    nvtxRangePop();
    return st;
}

// One thread waits on an mbarrier that nothing arrives on: the bounded wait
// must run out, raise the timeout bit and let the kernel return.
__global__ void wait_selftest_kernel() {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0);
}

}  // namespace

cudaError_t launch_wait_selftest(cudaStream_t stream) {
    wait_selftest_kernel<<<1, 32, 0, stream>>>();
    return cudaGetLastError();
}

}  // namespace pivot

namespace pivot {
pivot_status_t decode_check_args(const pivot_decode_t* b, int32_t mode, int32_t C, int32_t topk,
                                 const int32_t* idx);

// A named NVTX range around an entry point or a stage of it: the profilers'
// timelines show which call (and which step of the fused selection) each
// kernel belongs to.  Header-only NVTX: without a profiler attached a range
// costs a branch.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};
}  // namespace pivot

using namespace pivot;

extern "C" {

int32_t pivot_version(void) { return PIVOT_VERSION; }

const char* pivot_last_error_detail(void) { return g_last_detail; }

const char* pivot_status_string(pivot_status_t s) {
    switch (s) {
        case PIVOT_OK: return "ok";
        case PIVOT_ERR_INVALID_ARG: return "invalid argument";
        case PIVOT_ERR_UNSUPPORTED: return "unsupported shape";
        case PIVOT_ERR_WORKSPACE: return "workspace too small";
        case PIVOT_ERR_CUDA: return "CUDA error";
        case PIVOT_ERR_TIMEOUT: return "a kernel wait timed out";
        case PIVOT_ERR_DEVICE: return "bad device-side data";
    }
    return "unknown status";
}

pivot_status_t pivot_get_device_error(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return PIVOT_ERR_CUDA;
    uint32_t w = 0;
    if (cudaMemcpyFromSymbol(&w, g_error_word, sizeof(w)) != cudaSuccess) return PIVOT_ERR_CUDA;
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return PIVOT_ERR_CUDA;
    if (w & ERRBIT_TIMEOUT) return PIVOT_ERR_TIMEOUT;
    if (w & (ERRBIT_DATA | ERRBIT_BOUNDS)) return PIVOT_ERR_DEVICE;
    return PIVOT_OK;
}

pivot_status_t pivot_set_wait_limit_ns(uint64_t ns) {
    const uint64_t v = ns ? ns : 4000000000ull;
    return cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)) == cudaSuccess ? PIVOT_OK
                                                                            : PIVOT_ERR_CUDA;
}

pivot_status_t pivot_set_fused_selection(int32_t on, float margin_sigmas) {
    if ((on != 0 && on != 1) || !(margin_sigmas > -1e6f && margin_sigmas < 1e6f))
        return PIVOT_ERR_INVALID_ARG;
    g_fused_on = on != 0;
    g_fused_sigmas = margin_sigmas;
    return PIVOT_OK;
}

pivot_status_t pivot_set_score_buffer_cap(size_t bytes) {
    if (bytes != 0 && bytes < 4096) return PIVOT_ERR_INVALID_ARG;
    g_score_buf_cap = bytes ? bytes : SCORE_BUF_DEFAULT;
    return PIVOT_OK;
}

pivot_status_t pivot_selftest_wait_timeout(void* stream) {
    return launch_wait_selftest(static_cast<cudaStream_t>(stream)) == cudaSuccess ? PIVOT_OK
                                                                                  : PIVOT_ERR_CUDA;
}

// ------------------------------------------------------------------ dense
size_t pivot_dense_index_workspace_size(const pivot_seq_t* seq, int32_t topk) {
    int t0, t1;
    if (check_seq(seq, &t0, &t1) != PIVOT_OK || topk < 1) return 0;
    const int P = rows_per_block(seq->H, seq->D, seq->dtype);
    if (fused_ok(seq->H, seq->D, seq->dtype, topk)) {
        const size_t rb = fused_rowbytes(seq->L);
        long long rows = t1 - t0;
        long long cap = (long long)(g_score_buf_cap / rb) / P * P;
        if (cap < 1) cap = 1;
        if (rows > cap) rows = cap;
        return align_up((size_t)rows * rb + FUSED_FIXED, WS_ALIGN);
    }
    const size_t rb = dense_rowbytes(seq->L);
    long long rows = t1 - t0;
    long long cap = (long long)(g_score_buf_cap / rb) / P * P;
    if (cap < 1) cap = 1;
    if (rows > cap) rows = cap;
    return align_up((size_t)rows * rb, WS_ALIGN);
}

// lim_shift > 0 keeps the last lim_shift positions of every row out of the
// choice; out_stride (0: topk) is the row stride of idx / score.
static pivot_status_t dense_index_impl(const pivot_seq_t* seq, int32_t topk, int32_t* idx,
                                       float* score, void* ws, size_t ws_bytes, void* stream,
                                       int lim_shift, int out_stride) {
    int t0, t1;
    pivot_status_t st = check_seq(seq, &t0, &t1);
    if (st != PIVOT_OK) return st;
    if (topk < 1 || !idx) return PIVOT_ERR_INVALID_ARG;
    if (topk > MAX_K) return PIVOT_ERR_UNSUPPORTED;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) % WS_ALIGN)) return PIVOT_ERR_INVALID_ARG;
    const int P = rows_per_block(seq->H, seq->D, seq->dtype);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (fused_ok(seq->H, seq->D, seq->dtype, topk)) {
        const long long chunk = fused_chunk_rows(ws_bytes, seq->L, t1 - t0, P);
        FusedWs fw;
        if (chunk < 1 || !fused_carve(ws, ws_bytes, chunk, seq->L, &fw)) return PIVOT_ERR_WORKSPACE;
        for (long long c0 = t0; c0 < t1; c0 += chunk) {
            const int r0 = (int)c0;
            const int r1 = (int)(c0 + chunk < t1 ? c0 + chunk : t1);
            st = run_prefix_fused(SCAN_PREFILL_DENSE, key_src(seq), seq->q, seq->L, 0, seq->w,
                                  seq->q_scale, 1, P, r0, r1, r1 - 1, topk, 0, idx, score, t0,
                                  lim_shift, out_stride, fw, s);
            if (st != PIVOT_OK) return st;
        }
        return PIVOT_OK;
    }
    const long long stride = score_stride(seq->L);
    const long long chunk = chunk_rows(ws_bytes, dense_rowbytes(seq->L), t1 - t0, P);
    if (chunk < 1) return PIVOT_ERR_WORKSPACE;
    float* S = static_cast<float*>(ws);
    uint32_t* thresh = reinterpret_cast<uint32_t*>(S + chunk * stride);
    for (long long c0 = t0; c0 < t1; c0 += chunk) {
        const int r0 = (int)c0;
        const int r1 = (int)(c0 + chunk < t1 ? c0 + chunk : t1);
        st = run_scan(SCAN_PREFILL_DENSE, seq->dtype, seq->H, seq->D, seq->q, seq->L, 0, seq->w,
                      seq->q_scale, seq->k, seq->L, seq->k_scale, seq->L, 1, 1, 0, nullptr, P, r0,
                      r1, r1 - 1, S, stride, s);
        if (st != PIVOT_OK) return st;
        // positions of these rows are < r1: bitmaps of r1 bits (smaller
        // shared memory for the early chunks, more CTAs an SM)
        st = run_select_prefix(SCAN_PREFILL_DENSE, r0, r1, seq->L, 1, 1, 0, nullptr, S, stride,
                               topk, 0, r1, idx, score, t0, s, thresh, lim_shift, out_stride);
        if (st != PIVOT_OK) return st;
    }
    return PIVOT_OK;
}

pivot_status_t pivot_dense_index(const pivot_seq_t* seq, int32_t topk, int32_t* idx, float* score,
                                 void* ws, size_t ws_bytes, void* stream) {
    NvtxRange nvtx_range("pivot_dense_index");
    OrderScope order_scope(seq ? seq->order : 0);
    return dense_index_impl(seq, topk, idx, score, ws, ws_bytes, stream, 0, 0);
}

// ------------------------------------------------------------ proxy reduce
pivot_status_t pivot_proxy_reduce(const pivot_seq_t* seq, int32_t g, void* pq, float* pq_scale,
                                  float* pw, void* stream) {
    NvtxRange nvtx_range("pivot_proxy_reduce");
    int t0, t1;
    pivot_status_t st = check_seq(seq, &t0, &t1);
    if (st != PIVOT_OK) return st;
    if ((st = check_group_range(seq, g, t0, t1)) != PIVOT_OK) return st;
    if (!pq || !pw || !aligned16(pq)) return PIVOT_ERR_INVALID_ARG;
    if ((seq->dtype == PIVOT_E4M3) != (pq_scale != nullptr)) return PIVOT_ERR_INVALID_ARG;
    ReduceParams rp{};
    rp.dtype = seq->dtype;
    rp.esize = esize_of(seq->dtype);
    rp.H = seq->H;
    rp.D = seq->D;
    rp.nmembers_total = t1 - t0;
    rp.g = g;
    rp.ngroups = ceil_div(t1 - t0, g);
    rp.q = static_cast<const uint8_t*>(seq->q) + (size_t)t0 * seq->H * seq->D * rp.esize;
    rp.q_scale = seq->q_scale ? seq->q_scale + t0 : nullptr;
    rp.w = seq->w + (size_t)t0 * seq->H;
    rp.pq = pq;
    rp.pq_scale = pq_scale;
    rp.pw = pw;
    rp.group_stride_members = g;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const double bytes = ((double)(t1 - t0) + rp.ngroups) * seq->H * (seq->D * rp.esize + 4.0);
    return from_cuda(profiled(PK_REDUCE, bytes, s, [&] { return launch_proxy_reduce(rp, s); }));
}

// -------------------------------------------------------------- proxy scan
size_t pivot_proxy_scan_workspace_size(const pivot_seq_t* seq, int32_t g, int32_t C) {
    int t0, t1;
    if (check_seq(seq, &t0, &t1) != PIVOT_OK || g < 1 || C < 1) return 0;
    const int P = rows_per_block(seq->H, seq->D, seq->dtype);
    if (fused_ok(seq->H, seq->D, seq->dtype, C)) {
        const size_t rb = fused_rowbytes(seq->L);
        long long rows = ceil_div(t1 - t0, g);
        long long cap = (long long)(g_score_buf_cap / rb) / P * P;
        if (cap < 1) cap = 1;
        if (rows > cap) rows = cap;
        return align_up((size_t)rows * rb + FUSED_FIXED, WS_ALIGN);
    }
    const size_t rb = dense_rowbytes(seq->L);
    long long rows = ceil_div(t1 - t0, g);
    long long cap = (long long)(g_score_buf_cap / rb) / P * P;
    if (cap < 1) cap = 1;
    if (rows > cap) rows = cap;
    return align_up((size_t)rows * rb, WS_ALIGN);
}

pivot_status_t pivot_proxy_scan(const pivot_seq_t* seq, int32_t g, const void* pq,
                                 const float* pq_scale, const float* pw, int32_t C, int32_t topk,
                                 int32_t* cand, float* cand_score, void* ws, size_t ws_bytes,
                                 void* stream) {
    NvtxRange nvtx_range("pivot_proxy_scan");
    OrderScope order_scope(seq ? seq->order : 0);
    int t0, t1;
    pivot_status_t st = check_seq(seq, &t0, &t1);
    if (st != PIVOT_OK) return st;
    if ((st = check_group_range(seq, g, t0, t1)) != PIVOT_OK) return st;
    if (!pq || !pw || !cand || !aligned16(pq) || C < 1) return PIVOT_ERR_INVALID_ARG;
    if (topk < 1 || topk > C) return PIVOT_ERR_INVALID_ARG;
    if ((seq->dtype == PIVOT_E4M3) != (pq_scale != nullptr)) return PIVOT_ERR_INVALID_ARG;
    if (C > MAX_K) return PIVOT_ERR_UNSUPPORTED;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) % WS_ALIGN)) return PIVOT_ERR_INVALID_ARG;
    const int P = rows_per_block(seq->H, seq->D, seq->dtype);
    const long long stride = score_stride(seq->L);
    const int j0 = t0 / g, j1 = ceil_div(t1, g);
    const int G = j1 - j0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (fused_ok(seq->H, seq->D, seq->dtype, C)) {
        const long long chunk = fused_chunk_rows(ws_bytes, seq->L, j1 - j0, P);
        FusedWs fw;
        if (chunk < 1 || !fused_carve(ws, ws_bytes, chunk, seq->L, &fw)) return PIVOT_ERR_WORKSPACE;
        for (long long c0 = j0; c0 < j1; c0 += chunk) {
            const int r0 = (int)c0;
            const int r1 = (int)(c0 + chunk < j1 ? c0 + chunk : j1);
            const int e_last = (r1 * g < seq->L ? r1 * g : seq->L) - 1;
            st = run_prefix_fused(SCAN_PREFILL_PROXY, key_src(seq), pq, G, j0, pw, pq_scale, g, P,
                                  r0, r1, e_last, C, topk, cand, cand_score, j0, 0, 0, fw, s);
            if (st != PIVOT_OK) return st;
        }
        return PIVOT_OK;
    }
    const long long chunk = chunk_rows(ws_bytes, dense_rowbytes(seq->L), j1 - j0, P);
    if (chunk < 1) return PIVOT_ERR_WORKSPACE;
    float* S = static_cast<float*>(ws);
    uint32_t* thresh = reinterpret_cast<uint32_t*>(S + chunk * stride);
    for (long long c0 = j0; c0 < j1; c0 += chunk) {
        const int r0 = (int)c0;
        const int r1 = (int)(c0 + chunk < j1 ? c0 + chunk : j1);
        const int e_last = (r1 * g < seq->L ? r1 * g : seq->L) - 1;
        st = run_scan(SCAN_PREFILL_PROXY, seq->dtype, seq->H, seq->D, pq, G, j0, pw, pq_scale,
                      seq->k, seq->L, seq->k_scale, seq->L, g, 1, 0, nullptr, P, r0, r1, e_last, S,
                      stride, s);
        if (st != PIVOT_OK) return st;
        st = run_select_prefix(SCAN_PREFILL_PROXY, r0, r1, seq->L, g, 1, 0, nullptr, S, stride, C,
                               topk, e_last + 1, cand, cand_score, j0, s, thresh);
        if (st != PIVOT_OK) return st;
    }
    return PIVOT_OK;
}

// ------------------------------------------------------------------- reuse
pivot_status_t pivot_reuse(int32_t t_begin, int32_t t_end, int32_t g, const int32_t* cand,
                           int32_t C, int32_t topk, int32_t* idx, void* stream) {
    NvtxRange nvtx_range("pivot_reuse");
    if (g < 1 || t_begin < 0 || t_end <= t_begin || t_begin % g) return PIVOT_ERR_INVALID_ARG;
    if (!cand || !idx || topk < 1 || C < topk) return PIVOT_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const double bytes = 4.0 * topk * ((double)(t_end - t_begin) + ceil_div(t_end - t_begin, g));
    return from_cuda(profiled(PK_REUSE, bytes, s, [&] {
        return launch_reuse(t_begin, t_end, g, cand, C, topk, idx, s);
    }));
}

pivot_status_t pivot_reuse_backfill(int32_t t_begin, int32_t t_end, int32_t g,
                                    const int32_t* cand, const float* cand_score, int32_t C,
                                    int32_t topk, int32_t* idx, void* stream) {
    NvtxRange nvtx_range("pivot_reuse_backfill");
    if (g < 1 || t_begin < 0 || t_end <= t_begin || t_begin % g) return PIVOT_ERR_INVALID_ARG;
    if (!cand || !cand_score || !idx || topk < 1 || C < topk) return PIVOT_ERR_INVALID_ARG;
    if (C > MAX_K) return PIVOT_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the candidate selection over each group's proxy scores, per member limit t
    SelectParams sp{};
    sp.kind = SEL_CANDIDATES;
    sp.scan_kind = SCAN_PREFILL_DENSE;   // lim(t) = t
    sp.row0 = t_begin;
    sp.nrows = t_end - t_begin;
    sp.L = t_end;
    sp.g = g;
    sp.Gm = 1;
    sp.S = cand_score;
    sp.S_stride = C;
    sp.s_per_group = 1;
    sp.cand = cand;
    sp.cand_base = t_begin / g;
    sp.C = C;
    sp.K = topk;
    sp.out_idx = idx;
    sp.out_base = t_begin;
    sp.tail_cap = TAIL_CAP;
    sp.npos = t_end;
    const double bytes = 8.0 * C * ceil_div(t_end - t_begin, g) + 4.0 * topk * (t_end - t_begin);
    return from_cuda(profiled(PK_REUSE, bytes, s, [&] { return launch_select(sp, s); }));
}

pivot_status_t pivot_window_union(const int32_t* idx, int32_t rows, int32_t topk, int32_t t_begin,
                                  const int32_t* positions, int32_t window, int32_t* out,
                                  void* stream) {
    NvtxRange nvtx_range("pivot_window_union");
    if (rows < 0 || topk < 1 || window < 1 || !idx || !out) return PIVOT_ERR_INVALID_ARG;
    if (!positions && t_begin < 0) return PIVOT_ERR_INVALID_ARG;
    if (rows == 0) return PIVOT_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const double bytes = 4.0 * rows * (2.0 * topk + window);
    return from_cuda(profiled(PK_REUSE, bytes, s, [&] {
        return launch_window_union(idx, rows, topk, t_begin, positions, window, out, s);
    }));
}

// ------------------------------------------------------------------ refine
size_t pivot_refine_workspace_size(const pivot_seq_t* seq, int32_t g, int32_t C, int32_t topk) {
    int t0, t1;
    if (check_seq(seq, &t0, &t1) != PIVOT_OK || g < 1 || C < 1 || topk < 1) return 0;
    long long rows = t1 - t0;
    const size_t rb = (size_t)C * 4;
    long long cap = (long long)(g_score_buf_cap / rb) / g * g;
    if (cap < 1) cap = 1;
    if (rows > cap) rows = cap;
    return align_up((size_t)rows * rb, WS_ALIGN);
}

static pivot_status_t refine_impl(const pivot_seq_t* seq, int32_t g, const int32_t* cand,
                                  int32_t C, int32_t topk, int32_t* idx, float* score, void* ws,
                                  size_t ws_bytes, void* stream, int lim_shift, int out_stride,
                                  const int32_t* cand_count = nullptr) {
    int t0, t1;
    pivot_status_t st = check_seq(seq, &t0, &t1);
    if (st != PIVOT_OK) return st;
    if ((st = check_group_range(seq, g, t0, t1)) != PIVOT_OK) return st;
    if (!cand || !idx || topk < 1 || C < topk) return PIVOT_ERR_INVALID_ARG;
    if (C > MAX_K) return PIVOT_ERR_UNSUPPORTED;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) % WS_ALIGN)) return PIVOT_ERR_INVALID_ARG;
    const long long chunk = chunk_rows(ws_bytes, (size_t)C * 4, t1 - t0, g);
    if (chunk < 1) return PIVOT_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float* S = static_cast<float*>(ws);
    const int j0 = t0 / g;
    for (long long c0 = t0; c0 < t1; c0 += chunk) {
        const int r0 = (int)c0;
        const int r1 = (int)(c0 + chunk < t1 ? c0 + chunk : t1);
        const int jc = r0 / g;
        st = run_refine_scores(SCAN_PREFILL_DENSE, seq->dtype, seq->H, seq->D, seq->q, seq->L, 0,
                               seq->q_scale, seq->w, seq->k, seq->L, seq->k_scale, seq->L, g, 1,
                               0, nullptr, cand + (size_t)(jc - j0) * C, jc, C, r0, r1, S, s,
                               cand_count ? cand_count + (jc - j0) : nullptr);
        if (st != PIVOT_OK) return st;
        st = run_select_cand(SCAN_PREFILL_DENSE, r0, r1, seq->L, g, 1, 0, nullptr, S,
                             cand + (size_t)(jc - j0) * C, jc, C, topk, seq->L, idx, score, t0, s,
                             seq->k_scale, lim_shift, out_stride, nullptr,
                             cand_count ? cand_count + (jc - j0) : nullptr);
        if (st != PIVOT_OK) return st;
    }
    return PIVOT_OK;
}

pivot_status_t pivot_refine(const pivot_seq_t* seq, int32_t g, const int32_t* cand, int32_t C,
                            int32_t topk, int32_t* idx, float* score, void* ws, size_t ws_bytes,
                            void* stream) {
    NvtxRange nvtx_range("pivot_refine");
    OrderScope order_scope(seq ? seq->order : 0);
    return refine_impl(seq, g, cand, C, topk, idx, score, ws, ws_bytes, stream, 0, 0);
}

size_t pivot_refine_adaptive_workspace_size(const pivot_seq_t* seq, int32_t g, int32_t C,
                                            int32_t topk) {
    const size_t inner = pivot_refine_workspace_size(seq, g, C, topk);
    if (inner == 0) return 0;
    int t0 = 0, t1 = 0;
    if (check_seq(seq, &t0, &t1) != PIVOT_OK) return 0;
    return inner + align_up((size_t)ceil_div(t1 - t0, g) * 4, WS_ALIGN);
}

pivot_status_t pivot_refine_adaptive(const pivot_seq_t* seq, int32_t g, const int32_t* cand,
                                     const float* cand_score, int32_t C, int32_t topk, float rho,
                                     int32_t* cand_count, int32_t* idx, float* score, void* ws,
                                     size_t ws_bytes, void* stream) {
    NvtxRange nvtx_range("pivot_refine_adaptive");
    OrderScope order_scope(seq ? seq->order : 0);
    int t0, t1;
    pivot_status_t st = check_seq(seq, &t0, &t1);
    if (st != PIVOT_OK) return st;
    if ((st = check_group_range(seq, g, t0, t1)) != PIVOT_OK) return st;
    if (!cand || !cand_score || !idx || topk < 1 || C < topk) return PIVOT_ERR_INVALID_ARG;
    if (!(rho >= 0.0f && rho <= 1.0f)) return PIVOT_ERR_INVALID_ARG;
    if (C > MAX_K) return PIVOT_ERR_UNSUPPORTED;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) % WS_ALIGN)) return PIVOT_ERR_INVALID_ARG;
    const int G = ceil_div(t1 - t0, g);
    const size_t cnt_bytes = align_up((size_t)G * 4, WS_ALIGN);
    if (ws_bytes <= cnt_bytes) return PIVOT_ERR_WORKSPACE;
    int32_t* counts = cand_count ? cand_count : static_cast<int32_t*>(ws);
    void* inner = static_cast<uint8_t*>(ws) + cnt_bytes;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = from_cuda(profiled(PK_REUSE, 0.0, s, [&] {
        return launch_adaptive_count(cand_score, G, C, topk, rho, counts, s);
    }));
    if (st != PIVOT_OK) return st;
    return refine_impl(seq, g, cand, C, topk, idx, score, inner, ws_bytes - cnt_bytes, stream, 0,
                       0, counts);
}

// ------------------------------------------------------------------ ragged batch
namespace {

// Sequence i of a ragged batch as a single-sequence view (positions from 0).
pivot_seq_t varlen_seq(const pivot_varlen_t* b, int i) {
    const long long off = b->cu_seqlens[i];
    const int es = esize_of(b->dtype);
    pivot_seq_t s{};
    s.dtype = b->dtype;
    s.L = b->cu_seqlens[i + 1] - b->cu_seqlens[i];
    s.H = b->H;
    s.D = b->D;
    s.q = static_cast<const uint8_t*>(b->q) + off * b->H * b->D * es;
    s.q_scale = b->q_scale ? b->q_scale + off : nullptr;
    s.w = b->w + off * b->H;
    s.k = static_cast<const uint8_t*>(b->k) + off * b->D * es;
    s.k_scale = b->k_scale ? b->k_scale + off : nullptr;
    s.order = b->order;
    return s;
}

pivot_status_t check_varlen(const pivot_varlen_t* b, int mode, int g, int C, int topk) {
    if (!b || b->nseq < 1 || !b->cu_seqlens || b->cu_seqlens[0] != 0) return PIVOT_ERR_INVALID_ARG;
    if (!order_ok(b->order)) return PIVOT_ERR_INVALID_ARG;
    if (mode < PIVOT_MODE_DENSE || mode > PIVOT_MODE_REFINE || topk < 1) return PIVOT_ERR_INVALID_ARG;
    if (mode != PIVOT_MODE_DENSE && (g < 1 || C < topk)) return PIVOT_ERR_INVALID_ARG;
    if (topk > MAX_K || (mode != PIVOT_MODE_DENSE && C > MAX_K)) return PIVOT_ERR_UNSUPPORTED;
    for (int i = 0; i < b->nseq; ++i)
        if (b->cu_seqlens[i + 1] < b->cu_seqlens[i]) return PIVOT_ERR_INVALID_ARG;
    return PIVOT_OK;
}

// Workspace of the sequence-by-sequence path: proxies and candidates of the
// longest sequence, then the inner workspace the single-sequence calls need.
struct VarlenWs {
    size_t pq, pqs, pw, cand, inner, total;
};

VarlenWs varlen_layout(const pivot_varlen_t* b, int mode, int g, int C, int topk) {
    VarlenWs w{};
    long long maxL = 0;
    size_t inner = 0;
    for (int i = 0; i < b->nseq; ++i) {
        pivot_seq_t s = varlen_seq(b, i);
        if (s.L < 1) continue;
        if (s.L > maxL) maxL = s.L;
        size_t need = mode == PIVOT_MODE_DENSE ? pivot_dense_index_workspace_size(&s, topk)
                                               : pivot_proxy_scan_workspace_size(&s, g, C);
        if (mode == PIVOT_MODE_REFINE) {
            const size_t r = pivot_refine_workspace_size(&s, g, C, topk);
            if (r > need) need = r;
        }
        if (need > inner) inner = need;
    }
    size_t off = 0;
    if (mode != PIVOT_MODE_DENSE && maxL > 0) {
        const size_t G = (size_t)ceil_div((int)maxL, g);
        w.pq = off;
        off = align_up(off + G * b->H * b->D * esize_of(b->dtype), WS_ALIGN);
        w.pqs = off;
        off = align_up(off + G * 4, WS_ALIGN);
        w.pw = off;
        off = align_up(off + G * b->H * 4, WS_ALIGN);
        w.cand = off;
        off = align_up(off + G * C * 4, WS_ALIGN);
    }
    w.inner = off;
    w.total = align_up(off + inner, WS_ALIGN);
    return w;
}

// ---- one launch per stage over all sequences (tensor-core shapes)
constexpr int VAR_TPI = 32;   // key tiles per scan work item, as in the single-sequence prefill
constexpr int TABLE_CHUNK = 960;   // integers per launch_write_ints call (its limit)

// Host copies of the segment prefixes (segments.h): tokens, groups and the
// scan work items of the dense (query rows) and proxy (group rows) scans.
struct VarTabs {
    int B = 0, T = 0, maxL = 0, G = 0;
    std::vector<int32_t> tok, grp, itmD, itmP;
};

bool varlen_tabs(const pivot_varlen_t* b, int g, int P, VarTabs& t) {
    const int B = b->nseq;
    const int gg = g > 0 ? g : 1;
    t.B = B;
    t.tok.assign(b->cu_seqlens, b->cu_seqlens + B + 1);
    t.grp.assign(B + 1, 0);
    t.itmD.assign(B + 1, 0);
    t.itmP.assign(B + 1, 0);
    long long G = 0, ID = 0, IP = 0;
    for (int i = 0; i < B; ++i) {
        const int len = t.tok[i + 1] - t.tok[i];
        if (len > t.maxL) t.maxL = len;
        const int ng = ceil_div(len, gg);
        const long long ch = seg_chunks(len, VAR_TPI);
        G += ng;
        ID += (long long)ceil_div(len, P) * ch;
        IP += (long long)ceil_div(ng, P) * ch;
        if (G > INT32_MAX || ID > INT32_MAX || IP > INT32_MAX) return false;
        t.grp[i + 1] = (int32_t)G;
        t.itmD[i + 1] = (int32_t)ID;
        t.itmP[i + 1] = (int32_t)IP;
    }
    t.T = t.tok[B];
    t.G = (int)G;
    return true;
}

// Rows of the Refine tensor-core block for groups of g members.
int refine_rows(int H, int g) {
    const int P = umma_rows(H);
    return P < g ? P : g;
}

// Whether the batch runs as one launch per stage: the tensor-core scan
// shapes (and, for Refine, a member block the tensor cores take).
bool varlen_single_ok(const pivot_varlen_t* b, int mode, int g) {
    // inputs the single-sequence checks would refuse take that path and its errors
    if (!dtype_ok(b->dtype) || !b->q || !b->w || !b->k) return false;
    const bool fp8 = b->dtype == PIVOT_E4M3;
    if (fp8 != (b->q_scale != nullptr) || fp8 != (b->k_scale != nullptr)) return false;
    if (!umma_shape_ok(b->H, b->D, b->dtype)) return false;
    if (!aligned16(b->q) || !aligned16(b->k)) return false;
    if (mode == PIVOT_MODE_REFINE) {
        const int N = refine_rows(b->H, g) * b->H;
        if (N < 16 || N > 256 || N % 16) return false;
    }
    VarTabs t;
    return varlen_tabs(b, g, umma_rows(b->H), t);
}

struct VarlenWs1 {
    size_t tabs, pq, pqs, pw, cand, S, S_bytes, total;
};

VarlenWs1 varlen_layout1(const pivot_varlen_t* b, const VarTabs& t, int mode, int g, int C) {
    VarlenWs1 w{};
    size_t off = 0;
    w.tabs = off;
    off = align_up(off + (size_t)4 * (t.B + 1) * 4, WS_ALIGN);
    const size_t G = mode != PIVOT_MODE_DENSE ? (size_t)t.G : 0;
    if (G > 0) {
        w.pq = off;
        off = align_up(off + G * b->H * b->D * esize_of(b->dtype), WS_ALIGN);
        w.pqs = off;
        off = align_up(off + G * 4, WS_ALIGN);
        w.pw = off;
        off = align_up(off + G * b->H * 4, WS_ALIGN);
        w.cand = off;
        off = align_up(off + G * C * 4, WS_ALIGN);
    }
    const int P = umma_rows(b->H);
    const size_t rb = dense_rowbytes(t.maxL);
    long long cap = (long long)(g_score_buf_cap / rb) / P * P;
    if (cap < P) cap = P;
    const long long scan_rows = mode == PIVOT_MODE_DENSE ? t.T : t.G;
    size_t sb = (size_t)(scan_rows < cap ? scan_rows : cap) * rb;
    if (mode == PIVOT_MODE_REFINE) {
        long long capr = (long long)(g_score_buf_cap / ((size_t)C * 4)) / g * g;
        if (capr < g) capr = g;
        const size_t rbytes = (size_t)(t.T < capr ? t.T : capr) * C * 4;
        if (rbytes > sb) sb = rbytes;
    }
    w.S = off;
    w.S_bytes = align_up(sb, WS_ALIGN);
    w.total = align_up(off + w.S_bytes, WS_ALIGN);
    return w;
}

// Causal (row, key) pairs of packed dense rows [r0, r1) and of packed proxy
// rows [j0, j1); (member, candidate) pairs of Refine rows [r0, r1).
double varlen_dense_pairs(const VarTabs& t, int r0, int r1) {
    double s = 0.0;
    for (int b = seg_find(t.tok.data(), t.B, r0); b < t.B && t.tok[b] < r1; ++b) {
        const double a = (r0 > t.tok[b] ? r0 : t.tok[b]) - t.tok[b];
        const double z = (r1 < t.tok[b + 1] ? r1 : t.tok[b + 1]) - t.tok[b];
        if (z > a) s += 0.5 * (z * (z + 1) - a * (a + 1));
    }
    return s;
}

double varlen_proxy_pairs(const VarTabs& t, int g, int j0, int j1) {
    double s = 0.0;
    for (int b = seg_find(t.grp.data(), t.B, j0); b < t.B && t.grp[b] < j1; ++b) {
        const int len = t.tok[b + 1] - t.tok[b];
        const int ng = t.grp[b + 1] - t.grp[b];
        const double a = (j0 > t.grp[b] ? j0 : t.grp[b]) - t.grp[b];
        const double z = (j1 < t.grp[b + 1] ? j1 : t.grp[b + 1]) - t.grp[b];
        if (z <= a) continue;
        // groups x < ng - 1 end at (x + 1) g; the last one at len
        s += (double)g * 0.5 * (z * (z + 1) - a * (a + 1));
        if (z == ng) s += (double)len - (double)ng * g;
    }
    return s;
}

double varlen_refine_pairs(const VarTabs& t, int C, int r0, int r1) {
    double s = 0.0;
    for (int b = seg_find(t.tok.data(), t.B, r0); b < t.B && t.tok[b] < r1; ++b) {
        const int a = (r0 > t.tok[b] ? r0 : t.tok[b]) - t.tok[b];
        const int z = (r1 < t.tok[b + 1] ? r1 : t.tok[b + 1]) - t.tok[b];
        if (z > a) s += refine_pairs(a, z, C);
    }
    return s;
}

// The scan of packed rows [r0, r1) (kind SCAN_VARLEN_DENSE: tokens of q;
// SCAN_VARLEN_PROXY: groups of pq) against each row's sequence's keys.
pivot_status_t run_scan_varlen(int kind, const pivot_varlen_t* b, int T, const void* qbase,
                               long long q_rows, const float* w, const float* q_scale, int g,
                               int P, const SegTable& seg, int nitems, int r0, int r1, float* S,
                               long long stride, double work, cudaStream_t st) {
    ScanParams p{};
    p.kind = kind;
    p.dtype = b->dtype;
    p.esize = esize_of(b->dtype);
    p.H = b->H;
    p.D = b->D;
    p.P = P;
    p.row0 = r0;
    p.nrows = r1 - r0;
    p.qrow_base = 0;
    p.g = g;
    p.Gm = 1;
    p.w = w;
    p.q_scale = q_scale;
    p.k_scale = b->k_scale;
    p.S = S;
    p.S_stride = stride;
    p.tiles_per_item = seg.tpi;
    p.items_per_block = 0;
    p.nitems = nitems;
    p.seg = seg;
    CUtensorMap tk, tq;
    if (!make_tmap(&tk, b->dtype, b->k, T, b->D, 128)) return PIVOT_ERR_CUDA;
    if (!make_tmap(&tq, b->dtype, qbase, q_rows * b->H, b->D, P * b->H)) return PIVOT_ERR_CUDA;
    const int grid = nitems < num_sms() ? nitems : num_sms();
    return from_cuda(
        profiled(PK_SCAN, work, st, [&] { return launch_scan_umma(tk, tq, p, grid, st); }));
}

pivot_status_t varlen_single(const pivot_varlen_t* b, int mode, int g, int C, int topk,
                             int32_t* idx, void* ws, size_t ws_bytes, cudaStream_t st) {
    const int P = umma_rows(b->H);
    VarTabs t;
    if (!varlen_tabs(b, g, P, t)) return PIVOT_ERR_UNSUPPORTED;
    const VarlenWs1 lay = varlen_layout1(b, t, mode, g, C);
    if (ws_bytes < lay.total) return PIVOT_ERR_WORKSPACE;
    if (t.T == 0) return PIVOT_OK;
    uint8_t* base = static_cast<uint8_t*>(ws);
    // the segment tables, carried to the device as launch parameters (a
    // pageable host copy could not be captured in a CUDA graph)
    int32_t* d_tab = reinterpret_cast<int32_t*>(base + lay.tabs);
    const int n1 = t.B + 1;
    const std::vector<int32_t>* tabs[4] = {&t.tok, &t.grp, &t.itmD, &t.itmP};
    for (int a = 0; a < 4; ++a)
        for (int i = 0; i < n1; i += TABLE_CHUNK) {
            const int n = n1 - i < TABLE_CHUNK ? n1 - i : TABLE_CHUNK;
            cudaError_t e = launch_write_ints(d_tab + (size_t)a * n1 + i, tabs[a]->data() + i, n, st);
            if (e != cudaSuccess) return from_cuda(e);
            count_launch();
        }
    SegTable seg{};
    seg.tok = d_tab;
    seg.grp = d_tab + n1;
    seg.nseq = t.B;
    seg.tpi = VAR_TPI;
    const int32_t* d_itmD = d_tab + 2 * n1;
    const int32_t* d_itmP = d_tab + 3 * n1;
    float* S = reinterpret_cast<float*>(base + lay.S);
    const long long stride = score_stride(t.maxL);
    const long long cap_scan = (long long)(lay.S_bytes / dense_rowbytes(t.maxL));
    pivot_status_t res;

    // the scan + selection of packed rows [r0, r1) in launches of at most
    // cap_scan rows (a launch may cut a row block: rows outside it are dropped)
    auto scan_select = [&](int kind, const std::vector<int32_t>& rowpre, const int32_t* d_itm,
                           const std::vector<int32_t>& itm, int nrows_total, const void* qb,
                           const float* w, const float* qs, int gg, int K, int split,
                           int32_t* out) -> pivot_status_t {
        for (long long c0 = 0; c0 < nrows_total; c0 += cap_scan) {
            const int r0 = (int)c0;
            const int r1 = (int)(c0 + cap_scan < nrows_total ? c0 + cap_scan : nrows_total);
            int i0, n0, i1, n1b;
            seg_block_items(t.tok.data(), rowpre.data(), itm.data(), t.B, P, VAR_TPI, r0, &i0, &n0);
            seg_block_items(t.tok.data(), rowpre.data(), itm.data(), t.B, P, VAR_TPI, r1 - 1, &i1,
                            &n1b);
            SegTable sg = seg;
            sg.itm = d_itm;
            sg.item0 = i0;
            const int nitems = i1 + n1b - i0;
            const double work = kind == SCAN_VARLEN_DENSE ? varlen_dense_pairs(t, r0, r1)
                                                          : varlen_proxy_pairs(t, gg, r0, r1);
            uint32_t* thresh = reinterpret_cast<uint32_t*>(S + (size_t)(r1 - r0) * stride);
            pivot_status_t r = run_scan_varlen(kind, b, t.T, qb, nrows_total, w, qs, gg, P, sg,
                                               nitems, r0, r1, S, stride, work, st);
            if (r != PIVOT_OK) return r;
            r = run_select_prefix(kind, r0, r1, t.maxL, gg, 1, 0, nullptr, S, stride, K, split,
                                  t.maxL, out, nullptr, 0, st, thresh, 0, 0, &sg, work);
            if (r != PIVOT_OK) return r;
        }
        return PIVOT_OK;
    };

    if (mode == PIVOT_MODE_DENSE)
        return scan_select(SCAN_VARLEN_DENSE, t.tok, d_itmD, t.itmD, t.T, b->q, b->w, b->q_scale,
                           1, topk, 0, idx);

    // proxies of every group of the batch
    void* pq = base + lay.pq;
    float* pqs = b->dtype == PIVOT_E4M3 ? reinterpret_cast<float*>(base + lay.pqs) : nullptr;
    float* pw = reinterpret_cast<float*>(base + lay.pw);
    int32_t* cand = reinterpret_cast<int32_t*>(base + lay.cand);
    {
        ReduceParams rp{};
        rp.dtype = b->dtype;
        rp.esize = esize_of(b->dtype);
        rp.H = b->H;
        rp.D = b->D;
        rp.nmembers_total = t.T;
        rp.g = g;
        rp.ngroups = t.G;
        rp.q = b->q;
        rp.q_scale = b->q_scale;
        rp.w = b->w;
        rp.pq = pq;
        rp.pq_scale = pqs;
        rp.pw = pw;
        rp.group_stride_members = g;
        rp.seg = seg;
        const double bytes = ((double)t.T + t.G) * b->H * (b->D * rp.esize + 4.0);
        res = from_cuda(profiled(PK_REDUCE, bytes, st, [&] { return launch_proxy_reduce(rp, st); }));
        if (res != PIVOT_OK) return res;
    }
    // one full-prefix scan per group, top-C with its top-k first
    res = scan_select(SCAN_VARLEN_PROXY, t.grp, d_itmP, t.itmP, t.G, pq, pw, pqs, g, C, topk, cand);
    if (res != PIVOT_OK) return res;

    if (mode == PIVOT_MODE_REUSE) {
        const double bytes = 4.0 * topk * ((double)t.T + t.G);
        return from_cuda(profiled(PK_REUSE, bytes, st, [&] {
            return launch_reuse_varlen(seg, t.T, g, cand, C, topk, idx, st);
        }));
    }

    // Refine: members re-score their group's candidates, in launches of at
    // most cap_ref member rows
    const int Pr = refine_rows(b->H, g);
    const int N = Pr * b->H;
    CUtensorMap tq;
    if (!make_tmap(&tq, b->dtype, b->q, (long long)t.T * b->H, b->D, N)) return PIVOT_ERR_CUDA;
    const long long cap_ref = (long long)(lay.S_bytes / ((size_t)C * 4));
    const SegTable host_seg{t.tok.data(), t.grp.data(), nullptr, t.B, 0, 0};
    for (long long c0 = 0; c0 < t.T; c0 += cap_ref) {
        const int r0 = (int)c0;
        const int r1 = (int)(c0 + cap_ref < t.T ? c0 + cap_ref : t.T);
        const int jA = seg_group_of(host_seg, g, r0);
        const int jB = seg_group_of(host_seg, g, r1 - 1) + 1;
        ScanParams p{};
        p.kind = SCAN_VARLEN_DENSE;
        p.dtype = b->dtype;
        p.esize = esize_of(b->dtype);
        p.H = b->H;
        p.D = b->D;
        p.P = Pr;
        p.row0 = r0;
        p.nrows = r1 - r0;
        p.qrow_base = 0;
        p.g = g;
        p.Gm = 1;
        p.w = b->w;
        p.q_scale = b->q_scale;
        p.k_scale = b->k_scale;
        p.S = S;
        p.S_stride = C;
        p.cand = cand + (size_t)jA * C;
        p.cand_base = jA;
        p.C = C;
        p.gsize = g;
        p.tiles_per_item = ceil_div(C, 128);
        p.items_per_block = ceil_div(g, Pr);
        p.nitems = (jB - jA) * p.items_per_block;
        p.kbase = b->k;
        p.seg = seg;
        const double work = varlen_refine_pairs(t, C, r0, r1);
        const int grid = p.nitems < num_sms() ? p.nitems : num_sms();
        res = from_cuda(
            profiled(PK_REFINE, work, st, [&] { return launch_refine_umma(tq, p, grid, st); }));
        if (res != PIVOT_OK) return res;
        res = run_select_cand(SCAN_VARLEN_DENSE, r0, r1, t.maxL, g, 1, 0, nullptr, S,
                              cand + (size_t)jA * C, jA, C, topk, t.maxL, idx, nullptr, 0, st,
                              b->k_scale, 0, 0, &seg);
        if (res != PIVOT_OK) return res;
    }
    return PIVOT_OK;
}

}  // namespace

size_t pivot_index_varlen_workspace_size(const pivot_varlen_t* batch, int32_t mode, int32_t g,
                                         int32_t C, int32_t topk) {
    if (check_varlen(batch, mode, g, C, topk) != PIVOT_OK) return 0;
    if (varlen_single_ok(batch, mode, g)) {
        VarTabs t;
        varlen_tabs(batch, g, umma_rows(batch->H), t);
        return varlen_layout1(batch, t, mode, g, C).total;
    }
    return varlen_layout(batch, mode, g, C, topk).total;
}

pivot_status_t pivot_index_varlen(const pivot_varlen_t* batch, int32_t mode, int32_t g, int32_t C,
                                  int32_t topk, int32_t* idx, void* ws, size_t ws_bytes,
                                  void* stream) {
    NvtxRange nvtx_range("pivot_index_varlen");
    OrderScope order_scope(batch ? batch->order : 0);
    pivot_status_t st = check_varlen(batch, mode, g, C, topk);
    if (st != PIVOT_OK) return st;
    if (!idx || !ws || (reinterpret_cast<uintptr_t>(ws) % WS_ALIGN)) return PIVOT_ERR_INVALID_ARG;
    if (varlen_single_ok(batch, mode, g))
        return varlen_single(batch, mode, g, C, topk, idx, ws, ws_bytes,
                             static_cast<cudaStream_t>(stream));
    const VarlenWs lay = varlen_layout(batch, mode, g, C, topk);
    if (ws_bytes < lay.total) return PIVOT_ERR_WORKSPACE;
    uint8_t* base = static_cast<uint8_t*>(ws);
    const size_t inner_bytes = ws_bytes - lay.inner;
    for (int i = 0; i < batch->nseq; ++i) {
        pivot_seq_t s = varlen_seq(batch, i);
        if (s.L < 1) continue;
        int32_t* out = idx + (size_t)batch->cu_seqlens[i] * topk;
        if (mode == PIVOT_MODE_DENSE) {
            st = pivot_dense_index(&s, topk, out, nullptr, base + lay.inner, inner_bytes, stream);
        } else {
            void* pq = base + lay.pq;
            float* pqs = batch->dtype == PIVOT_E4M3 ? reinterpret_cast<float*>(base + lay.pqs)
                                                   : nullptr;
            float* pw = reinterpret_cast<float*>(base + lay.pw);
            int32_t* cand = reinterpret_cast<int32_t*>(base + lay.cand);
            st = pivot_proxy_reduce(&s, g, pq, pqs, pw, stream);
            if (st == PIVOT_OK)
                st = pivot_proxy_scan(&s, g, pq, pqs, pw, C, topk, cand, nullptr, base + lay.inner,
                                      inner_bytes, stream);
            if (st == PIVOT_OK)
                st = mode == PIVOT_MODE_REUSE
                         ? pivot_reuse(0, s.L, g, cand, C, topk, out, stream)
                         : pivot_refine(&s, g, cand, C, topk, out, nullptr, base + lay.inner,
                                        inner_bytes, stream);
        }
        if (st != PIVOT_OK) return st;
    }
    return PIVOT_OK;
}

// ------------------------------------------------------------------ window kept out
namespace {

struct WinWs {
    size_t pq, pqs, pw, cand, inner, total;
};

WinWs window_layout(const pivot_seq_t* seq, int t0, int t1, int mode, int g, int C, int topk) {
    WinWs w{};
    size_t off = 0, inner;
    if (mode == PIVOT_MODE_DENSE) {
        inner = pivot_dense_index_workspace_size(seq, topk);
    } else {
        const size_t G = (size_t)(ceil_div(t1, g) - t0 / g);
        w.pq = off;
        off = align_up(off + G * seq->H * seq->D * esize_of(seq->dtype), WS_ALIGN);
        w.pqs = off;
        off = align_up(off + G * 4, WS_ALIGN);
        w.pw = off;
        off = align_up(off + G * seq->H * 4, WS_ALIGN);
        w.cand = off;
        off = align_up(off + G * C * 4, WS_ALIGN);
        inner = pivot_proxy_scan_workspace_size(seq, g, C);
        if (mode == PIVOT_MODE_REFINE) {
            const size_t r = pivot_refine_workspace_size(seq, g, C, topk);
            if (r > inner) inner = r;
        }
    }
    w.inner = off;
    w.total = align_up(off + inner, WS_ALIGN);
    return w;
}

pivot_status_t check_window(const pivot_seq_t* seq, int mode, int g, int C, int topk,
                            int window, int* t0, int* t1) {
    pivot_status_t st = check_seq(seq, t0, t1);
    if (st != PIVOT_OK) return st;
    if (mode < PIVOT_MODE_DENSE || mode > PIVOT_MODE_REFINE || topk < 1 || window < 1)
        return PIVOT_ERR_INVALID_ARG;
    if (mode != PIVOT_MODE_DENSE) {
        if ((st = check_group_range(seq, g, *t0, *t1)) != PIVOT_OK) return st;
        if (C < topk) return PIVOT_ERR_INVALID_ARG;
        if (C > MAX_K) return PIVOT_ERR_UNSUPPORTED;
    }
    if (topk > MAX_K) return PIVOT_ERR_UNSUPPORTED;
    return PIVOT_OK;
}

}  // namespace

size_t pivot_index_window_outside_workspace_size(const pivot_seq_t* seq, int32_t mode, int32_t g,
                                                 int32_t C, int32_t topk, int32_t window) {
    int t0, t1;
    if (check_window(seq, mode, g, C, topk, window, &t0, &t1) != PIVOT_OK) return 0;
    return window_layout(seq, t0, t1, mode, g, C, topk).total;
}

pivot_status_t pivot_index_window_outside(const pivot_seq_t* seq, int32_t mode, int32_t g,
                                          int32_t C, int32_t topk, int32_t window, int32_t* idx,
                                          void* ws, size_t ws_bytes, void* stream) {
    NvtxRange nvtx_range("pivot_index_window_outside");
    OrderScope order_scope(seq ? seq->order : 0);
    int t0, t1;
    pivot_status_t st = check_window(seq, mode, g, C, topk, window, &t0, &t1);
    if (st != PIVOT_OK) return st;
    if (!idx || !ws || (reinterpret_cast<uintptr_t>(ws) % WS_ALIGN)) return PIVOT_ERR_INVALID_ARG;
    const WinWs lay = window_layout(seq, t0, t1, mode, g, C, topk);
    if (ws_bytes < lay.total) return PIVOT_ERR_WORKSPACE;
    uint8_t* base = static_cast<uint8_t*>(ws);
    void* inner = base + lay.inner;
    const size_t inner_bytes = ws_bytes - lay.inner;
    const int stride = topk + window;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // 1. the indexer's choice among positions <= t - window, rows at stride topk + window
    if (mode == PIVOT_MODE_DENSE) {
        st = dense_index_impl(seq, topk, idx, nullptr, inner, inner_bytes, stream, window, stride);
    } else {
        void* pq = base + lay.pq;
        float* pqs = seq->dtype == PIVOT_E4M3 ? reinterpret_cast<float*>(base + lay.pqs) : nullptr;
        float* pw = reinterpret_cast<float*>(base + lay.pw);
        int32_t* cand = reinterpret_cast<int32_t*>(base + lay.cand);
        st = pivot_proxy_reduce(seq, g, pq, pqs, pw, stream);
        if (st == PIVOT_OK)
            st = pivot_proxy_scan(seq, g, pq, pqs, pw, C, topk, cand, nullptr, inner, inner_bytes,
                                  stream);
        if (st == PIVOT_OK) {
            if (mode == PIVOT_MODE_REUSE)
                st = from_cuda(profiled(PK_REUSE, 0.0, s, [&] {
                    return launch_reuse(t0, t1, g, cand, C, topk, idx, s, window, stride);
                }));
            else
                st = refine_impl(seq, g, cand, C, topk, idx, nullptr, inner, inner_bytes, stream,
                                 window, stride);
        }
    }
    if (st != PIVOT_OK) return st;
    // 2. the window appended after each row's choice, in place
    return from_cuda(profiled(PK_REUSE, 0.0, s, [&] {
        return launch_window_union(idx, t1 - t0, topk, t0, nullptr, window, idx, s, stride);
    }));
}

// ------------------------------------------------------------------ decode
static pivot_status_t check_decode(const pivot_decode_t* b) {
    if (!b || !dtype_ok(b->dtype) || !order_ok(b->order)) return PIVOT_ERR_INVALID_ARG;
    if (b->B < 1 || b->Gm < 1 || b->H < 1 || b->D < 1 || b->maxlen < b->Gm)
        return PIVOT_ERR_INVALID_ARG;
    if (!b->q || !b->w || !b->kc || !b->cache_len) return PIVOT_ERR_INVALID_ARG;
    const bool fp8 = b->dtype == PIVOT_E4M3;
    if (fp8 != (b->q_scale != nullptr) || fp8 != (b->kc_scale != nullptr))
        return PIVOT_ERR_INVALID_ARG;
    if (!aligned16(b->q) || !aligned16(b->kc)) return PIVOT_ERR_INVALID_ARG;
    if ((b->D * esize_of(b->dtype)) % 16) return PIVOT_ERR_UNSUPPORTED;
    if (!umma_shape_ok(b->H, b->D, b->dtype) && !simt_shape_ok(b->H, b->D))
        return PIVOT_ERR_UNSUPPORTED;
    if (b->Gm * b->H > 256 && !simt_shape_ok(b->H, b->D)) return PIVOT_ERR_UNSUPPORTED;
    return PIVOT_OK;
}

struct DecodeWs {
    FusedWs f;      // fused selection (dense or proxy rows), when the shape takes it
    float* S;       // [B*Gm or B, stride] otherwise
    void* pq;       // [B, H, D]
    float* pqs;     // [B]
    float* pw;      // [B, H]
    int32_t* cand;  // [B, C]
    float* R;       // [B*Gm, C]
};

static size_t decode_layout(const pivot_decode_t* b, int mode, int C, int topk, DecodeWs* out,
                            void* base, size_t cap) {
    Carver c{static_cast<uint8_t*>(base), base ? cap : ~size_t(0) / 2};
    if (!base) c.base = reinterpret_cast<uint8_t*>(WS_ALIGN);   // size query only
    const long long stride = score_stride(b->maxlen);
    const int rows = mode == PIVOT_MODE_DENSE ? b->B * b->Gm : b->B;
    DecodeWs w{};
    const int K = mode == PIVOT_MODE_DENSE ? topk : C;
    if (fused_ok(b->H, b->D, b->dtype, K)) {
        const int tpi = scan_tiles_per_item(SCAN_DECODE_DENSE);
        const int L = b->maxlen;
        w.f.samp = static_cast<float*>(c.take((size_t)rows * fused_samp_stride(L) * 4));
        w.f.surv = static_cast<uint64_t*>(c.take((size_t)rows * fused_surv_stride(L, tpi) * 8));
        w.f.count = static_cast<uint32_t*>(c.take((size_t)rows * fused_nchunks(L, tpi) * 4 * 4));
        w.f.bound = static_cast<uint32_t*>(c.take((size_t)rows * 4));
        w.f.miss = static_cast<int32_t*>(c.take((size_t)rows * 4));
        w.f.nmiss = static_cast<uint32_t*>(c.take(4));
    } else {
        w.S = static_cast<float*>(c.take((size_t)rows * stride * 4));
    }
    if (mode != PIVOT_MODE_DENSE) {
        w.pq = c.take((size_t)b->B * b->H * b->D * esize_of(b->dtype));
        w.pqs = static_cast<float*>(c.take((size_t)b->B * 4));
        w.pw = static_cast<float*>(c.take((size_t)b->B * b->H * 4));
        w.cand = static_cast<int32_t*>(c.take((size_t)b->B * C * 4));
        if (mode == PIVOT_MODE_REFINE)
            w.R = static_cast<float*>(c.take((size_t)b->B * b->Gm * C * 4));
    }
    if (out) *out = w;
    return c.ok ? align_up(c.off, WS_ALIGN) : 0;
}

size_t pivot_decode_workspace_size(const pivot_decode_t* b, int32_t mode, int32_t C, int32_t topk) {
    if (check_decode(b) != PIVOT_OK || mode < 0 || mode > 2 || topk < 1) return 0;
    if (mode != PIVOT_MODE_DENSE && C < topk) return 0;
    return decode_layout(b, mode, C, topk, nullptr, nullptr, 0);
}

// The workspace of a whole indexer pass, from sizes alone (no buffers): the
// largest workspace any call of the mode's call chain needs.
size_t pivot_workspace_size(int32_t mode, int32_t dtype, int32_t L_or_maxlen, int32_t B,
                            int32_t H, int32_t D, int32_t g, int32_t C, int32_t topk) {
    if (mode < PIVOT_MODE_DENSE || mode > PIVOT_MODE_REFINE || !dtype_ok(dtype)) return 0;
    // stand-in addresses: only checked for presence and alignment, never read
    const void* dummy = reinterpret_cast<const void*>(uintptr_t(WS_ALIGN));
    const float* fdummy = static_cast<const float*>(dummy);
    const bool fp8 = dtype == PIVOT_E4M3;
    if (B == 0) {
        pivot_seq_t s{};
        s.dtype = dtype;
        s.L = L_or_maxlen;
        s.H = H;
        s.D = D;
        s.q = dummy;
        s.w = fdummy;
        s.k = dummy;
        s.q_scale = fp8 ? fdummy : nullptr;
        s.k_scale = fp8 ? fdummy : nullptr;
        if (mode == PIVOT_MODE_DENSE) return pivot_dense_index_workspace_size(&s, topk);
        if (topk < 1 || C < topk) return 0;
        const size_t scan = pivot_proxy_scan_workspace_size(&s, g, C);
        if (scan == 0 || mode == PIVOT_MODE_REUSE) return scan;
        const size_t ref = pivot_refine_workspace_size(&s, g, C, topk);
        return ref == 0 ? 0 : (scan > ref ? scan : ref);
    }
    pivot_decode_t b{};
    b.dtype = dtype;
    b.B = B;
    b.Gm = g;
    b.H = H;
    b.D = D;
    b.maxlen = L_or_maxlen;
    b.q = dummy;
    b.w = fdummy;
    b.kc = dummy;
    b.q_scale = fp8 ? fdummy : nullptr;
    b.kc_scale = fp8 ? fdummy : nullptr;
    b.cache_len = static_cast<const int32_t*>(dummy);
    return pivot_decode_workspace_size(&b, mode, C, topk);
}

pivot_status_t pivot_decode(const pivot_decode_t* b, int32_t mode, int32_t C, int32_t topk,
                            int32_t* idx, int32_t* cand, void* ws, size_t ws_bytes, void* stream) {
    NvtxRange nvtx_range("pivot_decode");
    OrderScope order_scope(b ? b->order : 0);
    pivot_status_t st = decode_check_args(b, mode, C, topk, idx);
    if (st != PIVOT_OK) return st;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) % WS_ALIGN)) return PIVOT_ERR_INVALID_ARG;
    DecodeWs w;
    if (decode_layout(b, mode, C, topk, &w, ws, ws_bytes) == 0) return PIVOT_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const long long stride = score_stride(b->maxlen);
    const long long krows = (long long)b->B * b->maxlen;
    const KeySrc ks{b->dtype, b->H, b->D, b->kc, krows, b->kc_scale, b->maxlen, b->Gm, b->maxlen,
                    b->cache_len};
    if (mode == PIVOT_MODE_DENSE) {
        const int rows = b->B * b->Gm;
        const int P = decode_dense_rows(b->Gm, b->H, b->D, b->dtype);
        if (w.f.surv)
            return run_prefix_fused(SCAN_DECODE_DENSE, ks, b->q, rows, 0, b->w, b->q_scale, 1, P, 0,
                                    rows, b->maxlen - 1, topk, 0, idx, nullptr, 0, 0, 0, w.f, s);
        st = run_scan(SCAN_DECODE_DENSE, b->dtype, b->H, b->D, b->q, rows, 0, b->w, b->q_scale,
                      b->kc, krows, b->kc_scale, 0, 1, b->Gm, b->maxlen, b->cache_len, P, 0, rows,
                      b->maxlen - 1, w.S, stride, s);
        if (st != PIVOT_OK) return st;
        return run_select_prefix(SCAN_DECODE_DENSE, 0, rows, 0, 1, b->Gm, b->maxlen, b->cache_len,
                                 w.S, stride, topk, 0, b->maxlen, idx, nullptr, 0, s);
    }
    // proxy of each sequence's Gm new tokens
    ReduceParams rp{};
    rp.dtype = b->dtype;
    rp.esize = esize_of(b->dtype);
    rp.H = b->H;
    rp.D = b->D;
    rp.nmembers_total = b->B * b->Gm;
    rp.g = b->Gm;
    rp.ngroups = b->B;
    rp.q = b->q;
    rp.q_scale = b->q_scale;
    rp.w = b->w;
    rp.pq = w.pq;
    rp.pq_scale = b->dtype == PIVOT_E4M3 ? w.pqs : nullptr;
    rp.pw = w.pw;
    rp.group_stride_members = b->Gm;
    if ((st = from_cuda(profiled(PK_REDUCE, 0.0, s, [&] { return launch_proxy_reduce(rp, s); }))) !=
        PIVOT_OK)
        return st;
    if (w.f.surv) {
        st = run_prefix_fused(SCAN_DECODE_PROXY, ks, w.pq, b->B, 0, w.pw,
                              b->dtype == PIVOT_E4M3 ? w.pqs : nullptr, 1, 1, 0, b->B,
                              b->maxlen - 1, C, topk, w.cand, nullptr, 0, 0, 0, w.f, s);
    } else {
        st = run_scan(SCAN_DECODE_PROXY, b->dtype, b->H, b->D, w.pq, b->B, 0, w.pw,
                      b->dtype == PIVOT_E4M3 ? w.pqs : nullptr, b->kc, krows, b->kc_scale, 0, 1,
                      b->Gm, b->maxlen, b->cache_len, 1, 0, b->B, b->maxlen - 1, w.S, stride, s);
        if (st != PIVOT_OK) return st;
        st = run_select_prefix(SCAN_DECODE_PROXY, 0, b->B, 0, 1, b->Gm, b->maxlen, b->cache_len,
                               w.S, stride, C, topk, b->maxlen, w.cand, nullptr, 0, s);
    }
    if (st != PIVOT_OK) return st;
    if (cand)
        if (cudaMemcpyAsync(cand, w.cand, (size_t)b->B * C * 4, cudaMemcpyDeviceToDevice, s) !=
            cudaSuccess)
            return PIVOT_ERR_CUDA;
    if (mode == PIVOT_MODE_REUSE)
        return from_cuda(profiled(PK_REUSE, 0.0, s, [&] {
            return launch_decode_reuse(b->B, b->Gm, b->maxlen, b->cache_len, w.cand, C, topk, idx, s);
        }));
    const int rows = b->B * b->Gm;
    st = run_refine_scores(SCAN_DECODE_DENSE, b->dtype, b->H, b->D, b->q, rows, 0, b->q_scale,
                           b->w, b->kc, krows, b->kc_scale, 0, 1, b->Gm, b->maxlen, b->cache_len,
                           w.cand, 0, C, 0, rows, w.R, s);
    if (st != PIVOT_OK) return st;
    return run_select_cand(SCAN_DECODE_DENSE, 0, rows, 0, 1, b->Gm, b->maxlen, b->cache_len, w.R,
                           w.cand, 0, C, topk, b->maxlen, idx, nullptr, 0, s, b->kc_scale);
}

}  // extern "C"

namespace pivot {

// The argument checks of pivot_decode, shared with pivot_decode_noalloc so
// that both report the same status for the same arguments.
pivot_status_t decode_check_args(const pivot_decode_t* b, int32_t mode, int32_t C, int32_t topk,
                                 const int32_t* idx) {
    pivot_status_t st = check_decode(b);
    if (st != PIVOT_OK) return st;
    if (mode < 0 || mode > 2 || topk < 1 || !idx) return PIVOT_ERR_INVALID_ARG;
    if (mode != PIVOT_MODE_DENSE && C < topk) return PIVOT_ERR_INVALID_ARG;
    if (topk > MAX_K || C > MAX_K) return PIVOT_ERR_UNSUPPORTED;
    return PIVOT_OK;
}

}  // namespace pivot
